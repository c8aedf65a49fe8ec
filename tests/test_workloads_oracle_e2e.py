"""Synthetic workloads (shapes, planted structure) and a whole oracle
trajectory on the tiny fp32 workload, CPU only."""
import numpy as np
import pytest
import torch

import workloads


def test_workload_shapes_and_capacity():
    for i in range(5):
        wl = workloads.config(i)
        assert len(wl.ctx0) == wl.requests
        assert wl.max_slots >= max(wl.ctx0) + wl.steps * wl.rows
    wl2 = workloads.config(2)
    assert wl2.requests == 96 and wl2.ctx0[0] == 524288 and wl2.max_blocks == 8193
    wl4 = workloads.config(4)
    assert all(256 * 1024 <= c <= 1024 * 1024 for c in wl4.ctx0)


def test_planted_vertical_slots_score_high():
    wl = workloads.config(1, ctx0=(4096,), steps=2, spare_slots=0)
    cache = workloads.make_key_cache(wl, 0)
    q, w = workloads.make_queries(wl, 0, 2)
    keys = cache.keys.view(torch.float8_e4m3fn).float() * cache.kscale[..., None]
    k = keys[cache.block_table[0].long()].reshape(-1, wl.d)[:4096]
    dots = torch.einsum("hd,sd->sh", q[0, 0].float(), k)
    score = (torch.relu(dots) * w[0, 0]).sum(-1)
    vs = workloads.vertical_slots(wl, 0, 0)
    top = torch.topk(score, vs.numel()).indices
    planted = torch.zeros(4096, dtype=torch.bool)
    planted[vs] = True
    # base rate 256 / 4096 = 6%; planted slots share the top scores with the
    # recent-offset band (the last W = 512 slots get a boost of the same size)
    assert planted[top].float().mean() > 0.2
    recent = torch.zeros(4096, dtype=torch.bool)
    recent[-512:] = True
    assert score[recent & ~planted].mean() > 1.5 * score[~recent & ~planted].mean()


def test_pages_permuted_and_unique():
    wl = workloads.config(2, requests=3, ctx0=(1000,) * 3, steps=2)
    cache = workloads.make_key_cache(wl, 0)
    bt = cache.block_table.flatten()
    assert torch.unique(bt).numel() == bt.numel()
    assert not torch.equal(bt, torch.arange(bt.numel(), dtype=torch.int32))


def test_accepted_lengths_mean():
    wl = workloads.config(3)
    a = workloads.accepted_lengths(wl, 4000)
    assert a.min() >= 1 and a.max() <= 4
    assert abs(a.double().mean().item() - 2.40) < 0.05


def test_oracle_trajectory_tiny_workload(oracle_lib):
    """32 steps of the tiny workload through the oracle: step 0 all-keep,
    then 30% target sparsity.  Checks the budget every step and that the
    predicted blocks recover most of the full indexer's top-k."""
    wl = workloads.config(0)
    cache = workloads.make_key_cache(wl, 0)
    q, w = workloads.make_queries(wl, 0, wl.steps)
    keys = cache.keys.numpy()
    bt = cache.block_table[0].numpy()
    nb = wl.max_blocks
    V = np.full(nb * wl.b, np.inf, np.float32)
    D = np.full(nb * wl.b, -np.inf, np.float32)
    misses = []
    for t in range(wl.steps):
        ctx_len = wl.ctx0[0] + t + 1
        s = 0.0 if t == 0 else wl.sparsity
        out = oracle_lib.decode_step_request(
            V=V, D=D, ctx_len=ctx_len, rows=1, b=wl.b, sparsity=s, gamma=wl.gamma, alpha=wl.alpha,
            seed=wl.seed, request=0, layer=0, step=t, topk=wl.topk, q=q[0, t:t + 1].numpy(),
            w=w[0, t:t + 1].numpy(), keys=keys, kscale=None, block_table=bt, key_fp8=False)
        n = -(-ctx_len // wl.b)
        kept = int(np.count_nonzero(out["mask"]))
        assert kept == (n if t == 0 else n - int(np.floor(np.float64(np.float32(s)) * n)))
        assert np.all(out["topk"][0] >= 0)
        if t > 0:
            full_mask = np.ones(nb, np.uint8)
            full = oracle_lib.score_f32(keys, bt, q[0, t:t + 1].numpy(), w[0, t:t + 1].numpy(),
                                        ctx_len, full_mask, nb * wl.b)
            ftop = oracle_lib.topk_row(full[0], full_mask, ctx_len, 0, wl.b, wl.topk)
            misses.append(oracle_lib.miss_fraction(ftop, out["mask"], wl.b))
    assert np.mean(misses) < 0.15, np.mean(misses)
