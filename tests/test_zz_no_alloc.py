"""The allocation-free top-k entry point (spin_topk_noalloc), for callers that
cannot give the library any device memory -- code running under CUDA graph
capture, or hosts that own every byte of device memory.  Its output must be
the oracle's token top-k (higher score first, ties to the lower slot,
ascending, padded with -1) on consecutive calls that reuse its fixed scratch;
a request whose ctx_len is out of range comes back all -1 with bit 0 of the
error word set, readable through spin_topk_noalloc_error; problems larger than
the scratch are refused.  Kept in a file of its own that pytest collects last."""
import numpy as np
import pytest
import torch

import indexer_sparse_attention_b200 as isa
import oracle

B = 64


def _inputs(rng, Q, R, max_slots, ctx):
    n_max = -(-max_slots // B)
    m = (rng.uniform(size=(Q, n_max)) < 0.55).astype(np.uint8)
    for q in range(Q):
        if 1 <= ctx[q] <= max_slots - R + 1:
            m[q, oracle.num_blocks(int(ctx[q]), R - 1, B):] = 0
    vals = rng.standard_normal((Q, R, n_max * B)).astype(np.float32) * 8
    vals[:, :, ::7] = np.round(vals[:, :, ::7])                 # plenty of exact ties
    return m, vals


def _oracle_topk(vals, m, ctx, R, k, max_slots):
    Q = vals.shape[0]
    out = np.full((Q, R, k), -1, np.int32)
    for q in range(Q):
        if not (1 <= ctx[q] <= max_slots - R + 1):
            continue                                         # out of range: all -1
        for r in range(R):
            out[q, r] = oracle.topk_row(vals[q, r].astype(np.float64), m[q], int(ctx[q]), r, B, k)
    return out


def _run(Q, R, k, max_slots, m, vals, ctx):
    got = torch.full((Q, R, k), -7, dtype=torch.int32, device="cuda")
    isa.spin_topk_noalloc(Q, R, R, max_slots, B, k, torch.from_numpy(vals).cuda(), torch.from_numpy(m).cuda(),
                          torch.from_numpy(ctx.astype(np.int32)).cuda(), got)
    status, word = isa.spin_topk_noalloc_error()
    return got.cpu().numpy(), status, word


@pytest.mark.gpu
def test_noalloc_topk_matches_oracle_and_reports_device_errors():
    from indexer_sparse_attention_b200 import build
    build.build()
    oracle.build()
    Q, R, k, max_slots = 7, 2, 512, 64 * 300 + 5
    rng = np.random.default_rng(2024)
    base = np.array([max_slots - R + 1, 1, 130, 64 * 77, 64 * 299 + 3, 5000, 64 * 8], np.int64)
    cases = [base, base[::-1].copy(), base.copy()]
    cases[1][0] = max_slots - R + 1
    cases[2][3] = max_slots                                  # past the last position two rows can take
    for call, ctx in enumerate(cases):
        m, vals = _inputs(rng, Q, R, max_slots, ctx)
        got, status, word = _run(Q, R, k, max_slots, m, vals, ctx)
        ref = _oracle_topk(vals, m, ctx, R, k, max_slots)
        # integer outputs: the tolerance is exact equality
        assert np.array_equal(got, ref), f"call {call}: {(got != ref).sum()} entries differ"
        if call < 2:
            assert status == 0 and word == 0, (call, status, word)   # cleared at the start of each call
        else:
            assert (got[3] == -1).all()
            assert isa.STATUS_NAMES[status] == "SPIN_EDEVICE" and word & 1, (status, word)


@pytest.mark.gpu
def test_noalloc_topk_refuses_problems_beyond_its_scratch():
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(isa.SpinError):
        # 200 requests at 1M slots need far more than the fixed 4 MiB of scratch
        isa.spin_topk_noalloc(200, 1, 1, 1024 * 1024, 64, 2048, dummy, dummy.view(torch.uint8),
                              dummy.view(torch.int32), dummy.view(torch.int32))
