"""Lock-step comparison of the CUDA decode step with the oracle.

For each checked request the harness snapshots V and D before a step, runs
the step through the C ABI, then replays it in the oracle: block scores and
the mask from the snapshot, scores in fp64 (all kept blocks, or a sample),
and -- fed the GPU's own fp32 scores -- the top-k and the next V, D.  Masks,
top-k indices and states must match bit for bit; scores within
|gpu - ref| <= 1e-4 + 1e-3 |ref|.
"""
from __future__ import annotations

import numpy as np
import torch

import indexer_sparse_attention_b200 as isa
import oracle
import workloads

RTOL, ATOL = 1e-3, 1e-4


def score_close(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.abs(gpu - ref) <= ATOL + RTOL * np.abs(ref)


def pool_close(gpu, ref, zabs_mean=0.0):
    """Mean and Top-4 block scores.  The oracle's value is the exact mean
    rounded once; the kernel sums in double in a fixed order (at most 256
    terms, error <= 255 * 2^-53 * sum|z|) and rounds once to float, so it is
    within one float ulp of the oracle's, plus 2^-45 * mean|z| where z takes
    both signs.  Equal infinities and NaNs match."""
    gpu = np.asarray(gpu, np.float32)
    ref = np.asarray(ref, np.float32)
    same = (gpu.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(gpu) & np.isnan(ref))
    with np.errstate(invalid="ignore", over="ignore"):
        tol = np.spacing(np.abs(ref)).astype(np.float64) + 2.0 ** -45 * np.asarray(zabs_mean, np.float64)
        close = np.abs(gpu.astype(np.float64) - ref.astype(np.float64)) <= tol
    return same | close


class Harness:
    def __init__(self, wl: workloads.Workload, device="cuda", score_kernel=isa.SPIN_SCORE_AUTO, positions=None,
                 layers=None, lookahead=False):
        self.wl = wl
        self.device = device
        self.layers = list(range(wl.layers)) if layers is None else layers
        npos = positions or (wl.steps * wl.rows + wl.rows)
        self.caches = {l: workloads.make_key_cache(wl, l, device) for l in self.layers}
        self.queries = {l: workloads.make_queries(wl, l, npos, device) for l in self.layers}
        cfg = isa.make_config(num_layers=wl.layers, num_requests=wl.requests, max_slots=wl.max_slots,
                              block_size=wl.b, num_heads=wl.H, head_dim=wl.d, topk=wl.topk, max_rows=wl.rows,
                              key_fp8=wl.key_fp8, q_bf16=wl.q_bf16, alpha=wl.alpha, gamma=wl.gamma,
                              target_sparsity=wl.sparsity, seed=wl.seed, pooling=wl.pooling,
                              mtp_policy=wl.mtp_policy)
        self.cfg = cfg
        self.st = isa.SpinState(cfg, device=device)
        isa.spin_set_score_kernel(self.st, score_kernel)
        self.lookahead = lookahead
        if lookahead:
            isa.spin_set_lookahead(self.st, True)
        self.committed = np.array(wl.ctx0, np.int64)
        self.mask = self.st.new_mask()
        self.topk = None
        self.scores = self.st.new_scores()
        self.sparsity = [wl.sparsity] * wl.layers
        self.step_index = 0
        self.host_pages = {}

    # ------------------------------------------------------------------
    def set_sparsity(self, per_layer):
        self.sparsity = list(per_layer)
        isa.spin_set_layer_sparsity(self.st, self.sparsity)

    def step_inputs(self, layer, rows):
        wl = self.wl
        pos0 = torch.from_numpy(self.committed - np.array(wl.ctx0, np.int64))
        qall, wall = self.queries[layer]
        idx = (pos0[:, None] + torch.arange(rows)[None, :]).to(qall.device)
        qstep = torch.stack([qall[i, idx[i]] for i in range(wl.requests)]).contiguous()
        wstep = torch.stack([wall[i, idx[i]] for i in range(wl.requests)]).contiguous()
        ctx = torch.from_numpy(self.committed + 1).to(torch.int32).to(self.device)
        return qstep, wstep, ctx

    def pages_of(self, layer, q):
        key = (layer, q)
        if key not in self.host_pages:
            keys, ks, ident = workloads.request_pages(self.caches[layer], q)
            self.host_pages[key] = (keys.numpy(), ks.numpy(), ident.numpy())
        return self.host_pages[key]

    # ------------------------------------------------------------------
    def run_step(self, layer, rows=None, accepted=None, check=(), sample_blocks=None, step=None,
                 rng=None, defer=None):
        """One decode step of `layer`.  `accepted` (np int [Q]) replays the
        prefix-valid rows after the step.  Returns per-check stats."""
        wl = self.wl
        rows = rows or wl.rows
        step = self.step_index if step is None else step
        qstep, wstep, ctx = self.step_inputs(layer, rows)
        V, D = self.st.ema(layer)
        snap = {q: (V[q].cpu().numpy().copy(), D[q].cpu().numpy().copy()) for q in check}
        cache = self.caches[layer]
        defer = (rows > 1) if defer is None else defer
        self.topk = torch.empty((wl.requests, rows, wl.topk), dtype=torch.int32, device=self.device)
        isa.spin_decode_step(self.st, layer, rows, step, cache.keys, cache.kscale if wl.key_fp8 else None,
                             cache.block_table, qstep, wstep, ctx, defer, self.mask, self.topk, self.scores)
        acc_t = None
        if defer:
            a = np.full(wl.requests, rows, np.int32) if accepted is None else np.asarray(accepted, np.int32)
            acc_t = torch.from_numpy(a).to(self.device)
            isa.spin_ema_update(self.st, layer, rows, self.scores, self.mask, ctx, acc_t)
        status, word = isa.spin_get_error(self.st)
        assert status == 0, f"device error word {word:#x}"
        results = {}
        for q in check:
            results[q] = self._check_request(layer, q, rows, step, snap[q], ctx[q].item(), qstep[q], wstep[q],
                                             acc_t[q].item() if acc_t is not None else rows, sample_blocks, rng)
        adv = rows if acc_t is None else acc_t.cpu().numpy()
        self.committed = self.committed + adv
        self.step_index += 1
        return results

    def _check_request(self, layer, q, rows, step, snap, ctx_len, qstep, wstep, accepted, sample_blocks, rng):
        wl = self.wl
        V0, D0 = snap
        nstride = self.st.mask_stride
        S_ref = oracle.predict_pool(V0, D0, ctx_len, rows, wl.b, nstride, wl.pooling)
        s = float(np.float32(self.sparsity[layer]))
        S_sel = S_ref
        pipelined = self.lookahead and rows == 1 and wl.key_fp8
        if s > 0 and not pipelined:   # pipelined: the buffer already holds the next step's scores
            S_gpu = self.st.block_scores()[q, :rows, :nstride].cpu().numpy()
            predicting = 1 if wl.mtp_policy == oracle.MTP_ROW0 else rows   # rows whose scores are computed
            for r in range(predicting):
                n = oracle.num_blocks(ctx_len, r, wl.b)
                if wl.pooling == oracle.POOL_MAX:   # a max is exact: bit for bit
                    assert np.array_equal(S_gpu[r, :n], S_ref[r, :n]), f"block scores differ q={q} r={r}"
                else:                               # z >= 0 here (EMA of non-negative scores)
                    assert pool_close(S_gpu[r, :n], S_ref[r, :n]).all(), f"block scores differ q={q} r={r}"
            if wl.pooling != oracle.POOL_MAX:
                # the selection is an integer decision taken from the block
                # scores: the oracle takes it from the GPU's
                S_sel = S_gpu
        mask_ref = oracle.select(S_sel, ctx_len, rows, wl.b, s, wl.gamma, wl.seed, q, layer, step, wl.mtp_policy)
        mask_gpu = self.mask[q].cpu().numpy()
        assert np.array_equal(mask_gpu, mask_ref), f"mask differs q={q}: {np.nonzero(mask_gpu != mask_ref)[0][:10]}"
        keys, ks, ident = self.pages_of(layer, q)
        sub = mask_ref.copy()
        if sample_blocks is not None:
            kept = np.nonzero(mask_ref)[0]
            rng = rng or np.random.default_rng(step)
            keep = rng.choice(kept, min(sample_blocks, kept.size), replace=False)
            sub = np.zeros_like(mask_ref)
            sub[keep] = 1
            n_last = oracle.num_blocks(ctx_len, rows - 1, wl.b)
            sub[n_last - 1] = mask_ref[n_last - 1]           # always the ragged last block
        slot_stride = self.st.score_stride
        q_host = qstep.float().cpu().numpy().astype(np.float64)
        w_host = wstep.cpu().numpy()
        if wl.key_fp8:
            q8, wq, _ = oracle.quantize_q(q_host, w_host)
            q8g, wqg = self.st.qquant(rows)
            assert np.array_equal(q8g[q].cpu().numpy(), q8), "quantised queries differ"
            assert np.array_equal(wqg[q].cpu().numpy(), wq), "folded head weights differ"
            ref = oracle.score_fp8(keys, ks, ident, q8, wq, ctx_len, sub, slot_stride)
        else:
            ref = oracle.score_f32(keys, ident, q_host.astype(np.float32), w_host, ctx_len, sub, slot_stride)
        gpu_scores = self.scores[q, :rows].cpu().numpy()
        scored = ~np.isnan(ref)
        ok = score_close(gpu_scores[scored], ref[scored])
        assert ok.all(), (f"scores differ q={q}: worst "
                          f"{np.max(np.abs(gpu_scores[scored] - ref[scored]) / (ATOL + RTOL * np.abs(ref[scored])))}")
        topk_gpu = self.topk[q, :rows].cpu().numpy()
        for r in range(rows):
            # unscored entries hold whatever the buffer held (any bit pattern,
            # signalling NaNs too); the oracle reads scored slots only
            with np.errstate(invalid="ignore"):
                row64 = gpu_scores[r].astype(np.float64)
            t_ref = oracle.topk_row(row64, mask_ref, ctx_len, r, wl.b, wl.topk)
            assert np.array_equal(topk_gpu[r], t_ref), f"top-k differs q={q} r={r}"
        V1, D1 = V0.copy(), D0.copy()
        oracle.ema_update(V1, D1, gpu_scores.astype(np.float32), mask_ref, ctx_len,
                          oracle.update_rows(wl.mtp_policy, accepted), wl.b, wl.alpha)
        Vg, Dg = self.st.ema(layer)
        assert np.array_equal(Vg[q].cpu().numpy().view(np.uint32), V1.view(np.uint32)), f"V differs q={q}"
        assert np.array_equal(Dg[q].cpu().numpy().view(np.uint32), D1.view(np.uint32)), f"D differs q={q}"
        if pipelined and s > 0 and ctx_len + 1 <= self.cfg.max_slots:
            # the block scores of the next step (one slot more), predicted from
            # the state this step left behind
            S_next = oracle.predict_pool(V1, D1, ctx_len + 1, 1, wl.b, nstride, wl.pooling)
            n = oracle.num_blocks(ctx_len + 1, 0, wl.b)
            S_gpu = self.st.block_scores()[q, 0, :nstride].cpu().numpy()
            if wl.pooling == oracle.POOL_MAX:
                assert np.array_equal(S_gpu[:n], S_next[0, :n]), f"next step's block scores differ q={q}"
            else:
                assert pool_close(S_gpu[:n], S_next[0, :n]).all(), f"next step's block scores differ q={q}"
        n_last = oracle.num_blocks(ctx_len, rows - 1, wl.b)
        return {"kept": int(np.count_nonzero(mask_ref)), "n": n_last, "scored_checked": int(scored.sum())}


def run_multilayer(h: Harness, check, check_warmup, sample_blocks=None):
    """The per-layer budget protocol of the multi-layer workload: an all-keep
    step on every layer, warm-up steps at the uniform target with a shadow
    full indexer measuring each layer's miss rate on the GPU, the water-filled
    per-layer sparsities (library against oracle), then the remaining steps
    with them.  Every layer of a step sees the same token.  Lock-step checks
    on `check_warmup` requests during warm-up and `check` afterwards."""
    wl = h.wl
    for layer in range(wl.layers):
        keep = list(h.sparsity)
        h.set_sparsity([0.0] * wl.layers)
        h.run_step(layer, check=check_warmup, step=0, sample_blocks=sample_blocks)
        h.committed -= 1                                    # every layer sees the same token
        h.set_sparsity(keep)
    h.committed += 1
    miss = np.zeros(wl.layers)
    Q, k = wl.requests, wl.topk
    full_scores = h.st.new_scores()
    full_topk = torch.empty((Q, 1, k), dtype=torch.int32, device=h.device)
    missed = torch.zeros((Q, 1), dtype=torch.int32, device=h.device)
    total = torch.zeros((Q, 1), dtype=torch.int32, device=h.device)
    for t in range(1, 1 + wl.warmup_steps):
        for layer in range(wl.layers):
            h.run_step(layer, check=check_warmup, step=t, sample_blocks=sample_blocks)
            h.committed -= 1
            qstep, wstep, ctx = h.step_inputs(layer, 1)
            cache = h.caches[layer]
            allk = torch.ones_like(h.mask)
            isa.spin_indexer_score(h.st, layer, 1, cache.keys, cache.kscale, cache.block_table, qstep, wstep, ctx,
                                   allk, full_scores)
            isa.spin_topk(h.st, 1, full_scores, allk, ctx, full_topk)
            isa.spin_miss_count(h.st, 1, full_topk, h.mask, missed, total)
            miss[layer] += (missed.double() / total.double()).mean().item()
        h.committed += 1
    miss /= wl.warmup_steps
    blocks = np.array([sum(-(-(c + 1) // wl.b) for c in h.committed)] * wl.layers, np.float64)
    lo = np.full(wl.layers, 0.05)
    s = isa.spin_allocate_layer_sparsity(miss, blocks, lo, wl.sparsity)
    ref = oracle.layer_sparsity(miss, blocks, lo, wl.sparsity)
    assert np.allclose(s, ref, atol=2e-6)
    h.set_sparsity(s)
    for t in range(1 + wl.warmup_steps, wl.steps):
        for layer in range(wl.layers):
            h.run_step(layer, check=check, step=t, sample_blocks=sample_blocks)
            h.committed -= 1
        h.committed += 1
    return s, miss
