"""The allocation-free top-k entry point (spin_topk_noalloc), for callers that
cannot give the library any device memory -- code running under CUDA graph
capture, or hosts that own every byte of device memory.  It must return
exactly what the state-based spin_topk returns for the same inputs, on
consecutive calls that reuse its fixed scratch, and refuse problems larger
than that scratch.  Kept in a file of its own that pytest collects last."""
import numpy as np
import pytest
import torch

import indexer_sparse_attention_b200 as isa


def _inputs(rng, st, Q, R, ctx):
    m = (rng.uniform(size=(Q, st.mask_stride)) < 0.55).astype(np.uint8)
    for q in range(Q):
        m[q, -(-(int(ctx[q]) + R - 1) // 64):] = 0
    vals = rng.standard_normal((Q, st.cfg.max_rows, st.score_stride)).astype(np.float32) * 8
    vals[:, :, ::7] = np.round(vals[:, :, ::7])                 # plenty of exact ties
    return torch.from_numpy(m).cuda(), torch.from_numpy(vals).cuda()


@pytest.mark.gpu
def test_noalloc_topk_matches_state_topk_on_consecutive_calls():
    from indexer_sparse_attention_b200 import build
    build.build()
    Q, R, k, max_slots = 7, 2, 512, 64 * 300 + 5
    cfg = isa.make_config(num_layers=1, num_requests=Q, max_slots=max_slots, topk=k, max_rows=R)
    st = isa.SpinState(cfg)
    rng = np.random.default_rng(2024)
    for call in range(2):
        ctx = np.array([max_slots - R + 1, 1, 130, 64 * 77, 64 * 299 + 3, 5000, 64 * 8], np.int64)
        if call == 1:
            ctx = ctx[::-1].copy()
            ctx[0] = max_slots - R + 1
        ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
        mask, scores = _inputs(rng, st, Q, R, ctx)
        ref = torch.full((Q, R, k), -7, dtype=torch.int32, device="cuda")
        got = torch.full((Q, R, k), -7, dtype=torch.int32, device="cuda")
        isa.spin_topk(st, R, scores, mask, ctx_t, ref)
        isa.spin_topk_noalloc(Q, R, R, max_slots, 64, k, scores, mask, ctx_t, got)
        torch.cuda.synchronize()
        assert isa.spin_get_error(st)[0] == 0
        # integer outputs: the tolerance is exact equality
        assert torch.equal(got, ref), f"call {call}: {(got != ref).sum().item()} entries differ"


@pytest.mark.gpu
def test_noalloc_topk_refuses_problems_beyond_its_scratch():
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(isa.SpinError):
        # 200 requests at 1M slots need far more than the fixed 4 MiB of scratch
        isa.spin_topk_noalloc(200, 1, 1, 1024 * 1024, 64, 2048, dummy, dummy.view(torch.uint8),
                              dummy.view(torch.int32), dummy.view(torch.int32))
