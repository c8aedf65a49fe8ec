"""Pipelined one-row decode steps (spin_set_lookahead): each step prepares the
next step's selection from the state its score kernel leaves behind and runs
its own top-k on a second stream beside the next step's predict kernel.  The
results must be those of the sequential step, bit for bit: the same masks,
top-k indices and EMA state, in lock step with the oracle, replayed from a CUDA
graph, and with a request whose ctx_len breaks the one-slot-a-step contract
reported in the device error word."""
import numpy as np
import pytest
import torch

import indexer_sparse_attention_b200 as isa
import oracle
import workloads
from lockstep import Harness

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from indexer_sparse_attention_b200 import build
    build.build()
    oracle.build()


def _wl(steps=9):
    return workloads.config(2, requests=5, ctx0=(70_000, 130, 64 * 700 - 1, 90_011, 64 * 64), steps=steps,
                            sparsity=0.5)


def _states(wl):
    out = []
    for la in (False, True):
        cfg = isa.make_config(num_layers=1, num_requests=wl.requests, max_slots=wl.max_slots, topk=wl.topk,
                              target_sparsity=wl.sparsity, gamma=wl.gamma, seed=wl.seed)
        st = isa.SpinState(cfg)
        if la:
            isa.spin_set_lookahead(st, True)
        out.append(st)
    return out


@pytest.mark.parametrize("device_step", [False, True])
def test_lookahead_matches_sequential_steps(device_step):
    """Sparsity schedule with an all-keep bootstrap, target changes (the
    prepared selection is dropped and made afresh) and an all-keep step in
    the middle; explicit step numbers or the device counter."""
    wl = _wl()
    cache = workloads.make_key_cache(wl, 0, "cuda")
    q_all, w_all = workloads.make_queries(wl, 0, wl.steps, "cuda")
    ctx0 = torch.tensor(wl.ctx0, dtype=torch.int64, device="cuda")
    Q, k = wl.requests, wl.topk
    seq, la = _states(wl)
    for st in (seq, la):
        isa.spin_set_step(st, 0)
    sched = [0.0, 0.5, 0.5, 0.5, 0.4, 0.4, 0.0, 0.5, 0.5]
    for t, s in enumerate(sched):
        q, w = q_all[:, t:t + 1].contiguous(), w_all[:, t:t + 1].contiguous()
        ctx = (ctx0 + t + 1).to(torch.int32)
        outs = []
        for st in (seq, la):
            isa.spin_set_layer_sparsity(st, [s])
            mask = st.new_mask()
            topk = torch.full((Q, 1, k), -7, dtype=torch.int32, device="cuda")
            step = isa.SPIN_STEP_DEVICE if device_step else t
            isa.spin_decode_step(st, 0, 1, step, cache.keys, cache.kscale, cache.block_table, q, w, ctx, False,
                                 mask, topk)
            if device_step:
                isa.spin_advance_step(st)
            outs.append((mask, topk))
        torch.cuda.synchronize()
        assert torch.equal(outs[0][0], outs[1][0]), f"mask differs at step {t}"
        assert torch.equal(outs[0][1], outs[1][1]), f"top-k differs at step {t}"
        for a, b in zip(seq.ema(0), la.ema(0)):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32)), f"state differs at step {t}"
    assert isa.spin_get_error(seq)[0] == 0 and isa.spin_get_error(la)[0] == 0


def test_lookahead_lock_step_with_oracle():
    """Pipelined steps of the serving shape in lock step with the oracle; the
    block-score buffer is checked as the next step's prediction from the
    state each step leaves behind."""
    wl = _wl(steps=6)
    h = Harness(wl, lookahead=True)
    h.set_sparsity([0.0])
    h.run_step(0, check=range(wl.requests))
    h.set_sparsity([0.5])
    for _ in range(wl.steps - 1):
        h.run_step(0, check=range(wl.requests))


def test_lookahead_graph_replay():
    """One pipelined step captured with the device step counter (after an
    eager pipelined step prepared the first selection), replayed with each
    step's inputs: the same results as sequential eager steps."""
    wl = _wl(steps=6)
    cache = workloads.make_key_cache(wl, 0, "cuda")
    q_all, w_all = workloads.make_queries(wl, 0, wl.steps, "cuda")
    ctx0 = torch.tensor(wl.ctx0, dtype=torch.int64, device="cuda")
    Q, k = wl.requests, wl.topk
    seq, la = _states(wl)

    def inputs(t):
        return q_all[:, t:t + 1].contiguous(), w_all[:, t:t + 1].contiguous(), (ctx0 + t + 1).to(torch.int32)

    eager = []
    for t in range(wl.steps):
        mask = seq.new_mask()
        topk = torch.empty((Q, 1, k), dtype=torch.int32, device="cuda")
        q, w, ctx = inputs(t)
        isa.spin_decode_step(seq, 0, 1, t, cache.keys, cache.kscale, cache.block_table, q, w, ctx, False, mask, topk)
        eager.append((mask.clone(), topk.clone()))
    q_buf, w_buf, ctx_buf = (x.clone() for x in inputs(0))
    mask_g = la.new_mask()
    topk_g = torch.empty((Q, 1, k), dtype=torch.int32, device="cuda")
    isa.spin_set_step(la, 0)
    isa.spin_decode_step(la, 0, 1, isa.SPIN_STEP_DEVICE, cache.keys, cache.kscale, cache.block_table, q_buf, w_buf,
                         ctx_buf, False, mask_g, topk_g)
    isa.spin_advance_step(la)
    torch.cuda.synchronize()
    assert torch.equal(mask_g, eager[0][0]) and torch.equal(topk_g, eager[0][1])
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        isa.spin_decode_step(la, 0, 1, isa.SPIN_STEP_DEVICE, cache.keys, cache.kscale, cache.block_table, q_buf,
                             w_buf, ctx_buf, False, mask_g, topk_g)
        isa.spin_advance_step(la)
    for t in range(1, wl.steps):
        q, w, ctx = inputs(t)
        q_buf.copy_(q)
        w_buf.copy_(w)
        ctx_buf.copy_(ctx)
        graph.replay()
        assert torch.equal(mask_g, eager[t][0]), t
        assert torch.equal(topk_g, eager[t][1]), t
    torch.cuda.synchronize()
    assert isa.spin_get_error(la)[0] == 0
    for a, b in zip(seq.ema(0), la.ema(0)):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    del graph


def test_lookahead_reports_a_broken_ctx_contract():
    """A request whose next ctx_len is not the prepared one (here: the same
    ctx_len again) is not scored: ERR_LOOKAHEAD is raised and its top-k rows
    are -1; the other requests match the sequential step."""
    wl = _wl(steps=3)
    cache = workloads.make_key_cache(wl, 0, "cuda")
    q_all, w_all = workloads.make_queries(wl, 0, wl.steps, "cuda")
    ctx0 = torch.tensor(wl.ctx0, dtype=torch.int64, device="cuda")
    Q, k = wl.requests, wl.topk
    seq, la = _states(wl)
    for t in range(2):
        q, w = q_all[:, t:t + 1].contiguous(), w_all[:, t:t + 1].contiguous()
        ctx = (ctx0 + t + 1).to(torch.int32)
        if t == 1:
            ctx_la = ctx.clone()
            ctx_la[2] -= 1                                  # request 2 does not advance
        res = []
        for st, c in ((seq, ctx), (la, ctx if t == 0 else ctx_la)):
            mask = st.new_mask()
            topk = torch.empty((Q, 1, k), dtype=torch.int32, device="cuda")
            isa.spin_decode_step(st, 0, 1, t, cache.keys, cache.kscale, cache.block_table, q, w, c, False, mask,
                                 topk)
            res.append(topk)
        status, word = isa.spin_get_error(la)
        if t == 0:
            assert status == 0
            continue
        assert isa.STATUS_NAMES[status] == "SPIN_EDEVICE" and word & 32, (status, word)
        assert torch.all(res[1][2] == -1)
        keep = [0, 1, 3, 4]
        assert torch.equal(res[0][keep], res[1][keep])
    assert isa.spin_get_error(seq)[0] == 0


@pytest.mark.parametrize("device_step,max_rows,pooling", [(False, 1, isa.SPIN_POOL_MAX), (True, 1, isa.SPIN_POOL_MAX),
                                                          (False, 4, isa.SPIN_POOL_MAX),
                                                          (False, 1, isa.SPIN_POOL_MEAN)])
def test_prepared_selections_match_sequential_steps(device_step, max_rows, pooling):
    """spin_prepare_selections makes every layer's selection of a step up
    front, and each layer's step then scores it.  Masks, top-k and EMA state equal the
    sequential steps', also on steps without a preparation (the pipelined
    path runs instead), after a target change that drops a prepared
    selection, and on all-keep steps; also in a state made for four MTP rows,
    whose block-score layout is four rows wide.  Max pooling takes one launch
    over up to eight layers (nine layers: a launch of eight and one of one);
    mean pooling takes the per-layer kernels over the state's streams."""
    wl = _wl(steps=7)
    Ly = 9                                # one stream takes two layers
    caches = [workloads.make_key_cache(wl, l, "cuda") for l in range(Ly)]
    qw = [workloads.make_queries(wl, l, wl.steps, "cuda") for l in range(Ly)]
    ctx0 = torch.tensor(wl.ctx0, dtype=torch.int64, device="cuda")
    Q, k = wl.requests, wl.topk
    sts = []
    for prep in (False, True):
        cfg = isa.make_config(num_layers=Ly, num_requests=wl.requests, max_slots=wl.max_slots, topk=wl.topk,
                              target_sparsity=wl.sparsity, gamma=wl.gamma, seed=wl.seed, max_rows=max_rows,
                              pooling=pooling)
        st = isa.SpinState(cfg)
        if prep:
            isa.spin_set_lookahead(st, True)
        isa.spin_set_step(st, 0)
        sts.append(st)
    seq, pre = sts
    base = [0.5, 0.4, 0.6, 0.5, 0.3, 0.5, 0.45, 0.5, 0.55]
    sched = [[0.0] * Ly, base, base, [0.0] + base[1:], base, base, base]
    prepared = {1, 2, 3, 5, 6}            # step 4 takes the pipelined path
    for t in range(wl.steps):
        ctx = (ctx0 + t + 1).to(torch.int32)
        step = isa.SPIN_STEP_DEVICE if device_step else t
        for st in sts:
            isa.spin_set_layer_sparsity(st, sched[t])
        if t in prepared:
            isa.spin_prepare_selections(pre, step, ctx)
        if t == 5:                        # layer 2's target changes after its preparation
            changed = list(sched[t])
            changed[2] = 0.45
            for st in sts:
                isa.spin_set_layer_sparsity(st, changed)
        for l in range(Ly):
            q, w = qw[l][0][:, t:t + 1].contiguous(), qw[l][1][:, t:t + 1].contiguous()
            c = caches[l]
            outs = []
            for st in sts:
                mask = st.new_mask()
                topk = torch.full((Q, 1, k), -7, dtype=torch.int32, device="cuda")
                isa.spin_decode_step(st, l, 1, step, c.keys, c.kscale, c.block_table, q, w, ctx, False, mask, topk)
                outs.append((mask, topk))
            torch.cuda.synchronize()
            assert torch.equal(outs[0][0], outs[1][0]), f"mask differs at step {t}, layer {l}"
            assert torch.equal(outs[0][1], outs[1][1]), f"top-k differs at step {t}, layer {l}"
        if device_step:
            for st in sts:
                isa.spin_advance_step(st)
        for l in range(Ly):
            for a, b in zip(seq.ema(l), pre.ema(l)):
                assert torch.equal(a.view(torch.int32), b.view(torch.int32)), f"state differs at step {t}, layer {l}"
    assert isa.spin_get_error(seq)[0] == 0 and isa.spin_get_error(pre)[0] == 0


def test_prepare_selections_needs_lookahead():
    cfg = isa.make_config(num_layers=2, num_requests=2, max_slots=64 * 40, topk=256)
    st = isa.SpinState(cfg)
    ctx = torch.full((2,), 100, dtype=torch.int32, device="cuda")
    with pytest.raises(isa.SpinError):
        isa.spin_prepare_selections(st, 0, ctx)
    isa.spin_set_lookahead(st, True)
    with pytest.raises(isa.SpinError):
        isa.spin_prepare_selections(st, -5, ctx)
    isa.spin_prepare_selections(st, 0, ctx)
    torch.cuda.synchronize()
    assert isa.spin_get_error(st)[0] == 0
