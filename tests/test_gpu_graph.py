"""The decode step as a captured CUDA graph: with SPIN_STEP_DEVICE the step
number comes from the state's device counter, which spin_advance_step moves
inside the graph, so one capture replays every step."""
import pytest
import torch

import indexer_sparse_attention_b200 as isa
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from indexer_sparse_attention_b200 import build
    build.build()


def test_decode_step_replays_from_a_cuda_graph():
    """Captured once and replayed with each step's inputs copied into its
    buffers, the graph gives the same masks, top-k and EMA state as eager
    calls with explicit step numbers."""
    wl = workloads.config(2, requests=4, ctx0=(70_000, 50_000, 90_000, 30_011), steps=6, sparsity=0.5)
    cache = workloads.make_key_cache(wl, 0, "cuda")
    q_all, w_all = workloads.make_queries(wl, 0, wl.steps, "cuda")
    ctx0 = torch.tensor(wl.ctx0, dtype=torch.int64, device="cuda")
    Q, k = wl.requests, wl.topk

    def new_state():
        cfg = isa.make_config(num_layers=1, num_requests=Q, max_slots=wl.max_slots, topk=k,
                              target_sparsity=wl.sparsity, gamma=wl.gamma, seed=wl.seed)
        return isa.SpinState(cfg)

    def inputs(t):
        return q_all[:, t:t + 1].contiguous(), w_all[:, t:t + 1].contiguous(), (ctx0 + t + 1).to(torch.int32)

    # eager, explicit step numbers
    st_e = new_state()
    eager = []
    for t in range(wl.steps):
        mask = st_e.new_mask()
        topk = torch.empty((Q, 1, k), dtype=torch.int32, device="cuda")
        q, w, ctx = inputs(t)
        isa.spin_decode_step(st_e, 0, 1, t, cache.keys, cache.kscale, cache.block_table, q, w, ctx, False, mask, topk)
        eager.append((mask.clone(), topk.clone()))
    assert isa.spin_get_error(st_e)[0] == 0

    # one capture: the step, then the counter advance
    st_g = new_state()
    q_buf, w_buf, ctx_buf = (x.clone() for x in inputs(0))
    mask_g = st_g.new_mask()
    topk_g = torch.empty((Q, 1, k), dtype=torch.int32, device="cuda")
    isa.spin_set_step(st_g, 0)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        isa.spin_decode_step(st_g, 0, 1, isa.SPIN_STEP_DEVICE, cache.keys, cache.kscale, cache.block_table, q_buf,
                             w_buf, ctx_buf, False, mask_g, topk_g)
        isa.spin_advance_step(st_g)
    for t in range(wl.steps):
        q, w, ctx = inputs(t)
        q_buf.copy_(q)
        w_buf.copy_(w)
        ctx_buf.copy_(ctx)
        graph.replay()
        assert torch.equal(mask_g, eager[t][0]), t
        assert torch.equal(topk_g, eager[t][1]), t
    assert isa.spin_get_error(st_g)[0] == 0
    V_e, D_e = st_e.ema(0)
    V_g, D_g = st_g.ema(0)
    assert torch.equal(V_e.view(torch.int32), V_g.view(torch.int32))
    assert torch.equal(D_e.view(torch.int32), D_g.view(torch.int32))
    del graph
