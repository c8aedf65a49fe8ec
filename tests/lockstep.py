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


class Harness:
    def __init__(self, wl: workloads.Workload, device="cuda", score_kernel=isa.SPIN_SCORE_AUTO, positions=None,
                 layers=None):
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
        if s > 0:
            S_gpu = self.st.block_scores()[q, :rows, :nstride].cpu().numpy()
            predicting = 1 if wl.mtp_policy == oracle.MTP_ROW0 else rows   # rows whose scores are computed
            for r in range(predicting):
                n = oracle.num_blocks(ctx_len, r, wl.b)
                assert np.array_equal(S_gpu[r, :n], S_ref[r, :n]), f"block scores differ q={q} r={r}"
        mask_ref = oracle.select(S_ref, ctx_len, rows, wl.b, s, wl.gamma, wl.seed, q, layer, step, wl.mtp_policy)
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
        n_last = oracle.num_blocks(ctx_len, rows - 1, wl.b)
        return {"kept": int(np.count_nonzero(mask_ref)), "n": n_last, "scored_checked": int(scored.sum())}
