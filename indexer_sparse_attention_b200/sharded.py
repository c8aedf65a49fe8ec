"""Context-sharded SPIN decode: one request's slots split over the ranks of a
process group (the long contexts the SPIN listing's Table 4 and MRCRv2 bins
reach, 256K to 1M slots).

This module is the exchange protocol: which rank owns which slots, blocks and
EMA entries, and what crosses ranks each step.  The per-shard arithmetic
(block max-pool, selection, indexer score, token top-k, EMA update) is done by
a backend object the caller supplies, so the same protocol drives any
implementation of those steps.  Every exchange is an all-gather over the
group, so every rank takes the same collective steps in the same order.

Ownership (rank g of G, request capacity n_max blocks of b slots):
  * blocks [J_g, J_{g+1}) with J_g = floor(g * n_max / G), i.e. the slots
    [lo_g, hi_g) = [J_g b, J_{g+1} b), and V_i for those slots;
  * the diagonal state D_delta for the offsets delta whose row-0 slot
    p_0 - delta is one of its slots: (p_0 - hi_g, p_0 - lo_g], plus read-only
    copies of the R - 1 offsets above that range (owned by rank g - 1), which
    rows r >= 1 read for the first slots.  As p_0 grows by the accepted length
    a, the a lowest offsets of rank g become rank g + 1's.

Per step (rows r = 0..R-1 at positions p_r = p_0 + r):
  1. each rank pools its blocks: S_{r,j} = max over its slots i <= p_r of
     max(V_i, D_{p_r - i});
  2. all-gather of S: every rank holds the request's full S and runs the same
     deterministic selection (budget, exploration draw, row union), keeping
     the mask of its blocks;
  3. each rank scores its kept slots;
  4. each rank takes the top k of its scored slots per row (score descending,
     lower slot first); all-gather of those candidates and an exact merge
     give the request's top k;
  5. score halo: the prefix-valid replay updates D_delta with rows
     r = 0..a-1 at slots p_0 - delta + r, which for the owner's last R - 1
     offsets lie in the next rank's first R - 1 slots; those scores move down
     one rank;
  6. each rank replays its V entries and its D offsets, rows in order;
  7. D halo: each rank passes its a + R - 1 lowest offsets (after the update)
     to the next rank: the first a become that rank's own, the rest its
     read-only copies.  Rank 0 has no rank above: it owns the R - 1 offsets
     above its range too (only its first slot reaches them, at rows r >= 1),
     and the offsets entering at its top are ones no row has reached (-inf).

Bytes crossing ranks per request and step: 4 n_r per row for S, 8 k per row
and rank for the candidates, 4 R (R - 1) for the score halo and
4 (a + R - 1) for the D halo.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np
import torch
import torch.distributed as dist

NEG_INF = np.float32(-np.inf)
POS_INF = np.float32(np.inf)


@dataclass(frozen=True)
class ShardLayout:
    """Block and slot ranges of every rank for one request capacity."""
    max_slots: int
    b: int
    world: int

    @property
    def n_max(self) -> int:
        return (self.max_slots + self.b - 1) // self.b

    def blocks(self, g: int):
        return (g * self.n_max) // self.world, ((g + 1) * self.n_max) // self.world

    def slots(self, g: int):
        j0, j1 = self.blocks(g)
        return j0 * self.b, min(j1 * self.b, self.max_slots)

    def owner_of_slot(self, s: int) -> int:
        for g in range(self.world):
            lo, hi = self.slots(g)
            if lo <= s < hi:
                return g
        raise ValueError(s)


def merge_topk(keys: np.ndarray, slots: np.ndarray, k: int) -> np.ndarray:
    """The k best of the union of per-rank candidate lists (score descending,
    lower slot first on ties), emitted in ascending slot order and padded with
    -1.  keys: float64 scores, slots: int64, -1 marks an empty candidate."""
    ok = slots >= 0
    keys, slots = keys[ok], slots[ok]
    order = np.lexsort((slots, -keys))[:k]
    out = np.full(k, -1, np.int64)
    chosen = np.sort(slots[order])
    out[: chosen.size] = chosen
    return out


class ShardedRequestState:
    """One request's shard on this rank: V of the owned slots and the D
    window (owned offsets plus R - 1 read-only offsets above them), with the
    committed length C (row 0 of the next step sits at p_0 = C - 1 + 1 once
    its own key is appended, so ctx_len = C + 1)."""

    def __init__(self, layout: ShardLayout, rank: int, rows_max: int, committed: int):
        self.layout, self.rank, self.R = layout, rank, rows_max
        self.lo, self.hi = layout.slots(rank)
        self.V = np.full(self.hi - self.lo, POS_INF, np.float32)
        # D_ext[k] holds offset d_lo + k; d_lo = p0 - hi + 1 for the next step
        self.D_ext = np.full(self.hi - self.lo + rows_max - 1, NEG_INF, np.float32)
        self.committed = committed

    # offsets of the window for the step whose row 0 sits at p0
    def d_lo(self, p0: int) -> int:
        return p0 - self.hi + 1

    def d_full(self, p0: int, n: int) -> np.ndarray:
        """The window as a full-length offset array (-inf outside), for
        backends that index D by offset."""
        out = np.full(n, NEG_INF, np.float32)
        lo = self.d_lo(p0)
        k0 = max(0, -lo)
        k1 = min(self.D_ext.size, n - lo)
        if k1 > k0:
            out[lo + k0: lo + k1] = self.D_ext[k0:k1]
        return out

    def v_full(self, n: int) -> np.ndarray:
        out = np.full(n, NEG_INF, np.float32)
        out[self.lo: self.hi] = self.V
        return out


class ShardedSpin:
    """Drives decode steps of Q requests, each sharded over the process
    group.  `backend` supplies the per-shard arithmetic:

      predict(q, V_full, D_full, ctx_len, rows) -> S [rows, n_max] (the
          rank's own blocks are read from it);
      select(q, S_full, ctx_len, rows, step) -> mask [n_max] uint8;
      score(q, mask_own, ctx_len, rows) -> scores [rows, slot_stride] float64
          (NaN where not scored; only the rank's kept slots are scored);
      ema(V_full, D_full, scores32, mask, ctx_len, n_update) -> None
          (the SPIN update in place on full-length arrays; the protocol keeps
          the entries this rank owns).

    Full-length arrays hold -inf / NaN outside what this rank knows; the
    protocol only ever reads back the entries the rank owns."""

    def __init__(self, backend, layout: ShardLayout, rows_max: int, topk: int, ctx0: Sequence[int],
                 group: Optional[dist.ProcessGroup] = None, mtp_row0: bool = False):
        self.backend, self.layout, self.R, self.k = backend, layout, rows_max, topk
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        assert self.world == layout.world
        self.mtp_row0 = mtp_row0
        self.reqs = [ShardedRequestState(layout, self.rank, rows_max, c) for c in ctx0]
        self.n_slots = layout.n_max * layout.b

    # -- collectives ---------------------------------------------------------
    def _all_gather(self, t: torch.Tensor) -> List[torch.Tensor]:
        out = [torch.empty_like(t) for _ in range(self.world)]
        dist.all_gather(out, t.contiguous(), group=self.group)
        return out

    # -- one step --------------------------------------------------------------
    def step(self, rows: int, step: int, accepted: Optional[Sequence[int]] = None):
        """One decode step of every request.  accepted[q] in 1..rows (None:
        all rows).  Returns (masks [Q][n_max], topk [Q][rows][k])."""
        L, R, b, nmax = self.layout, rows, self.layout.b, self.layout.n_max
        Q = len(self.reqs)
        ctxs = [st.committed + 1 for st in self.reqs]
        p0s = [c - 1 for c in ctxs]
        j0, j1 = L.blocks(self.rank)
        # 1. own block scores
        S_own = np.full((Q, R, j1 - j0), NEG_INF, np.float32)
        for q, st in enumerate(self.reqs):
            S = self.backend.predict(q, st.v_full(self.n_slots), st.d_full(p0s[q], self.n_slots), ctxs[q], R)
            S_own[q] = S[:, j0:j1]
        # 2. all-gather of S, replicated selection
        parts = self._all_gather(torch.from_numpy(self._pad_blocks(S_own)))
        S_full = np.full((Q, R, nmax), np.nan, np.float32)
        for g, t in enumerate(parts):
            a0, a1 = L.blocks(g)
            S_full[:, :, a0:a1] = t.numpy()[:, :, : a1 - a0]
        masks = np.stack([self.backend.select(q, S_full[q], ctxs[q], R, step) for q in range(Q)])
        own = np.zeros_like(masks)
        own[:, j0:j1] = masks[:, j0:j1]
        # 3. own scores; 4. local candidates, all-gather, exact merge
        scores = [self.backend.score(q, own[q], ctxs[q], R) for q in range(Q)]
        cand_k = np.full((Q, R, self.k), -np.inf, np.float64)
        cand_s = np.full((Q, R, self.k), -1, np.int64)
        for q in range(Q):
            for r in range(R):
                sc = scores[q][r]
                idx = np.nonzero(~np.isnan(sc))[0]
                order = np.lexsort((idx, -sc[idx]))[: self.k]
                cand_k[q, r, : order.size] = sc[idx[order]]
                cand_s[q, r, : order.size] = idx[order]
        gk = self._all_gather(torch.from_numpy(cand_k))
        gs = self._all_gather(torch.from_numpy(cand_s))
        allk = np.concatenate([t.numpy() for t in gk], axis=2)
        alls = np.concatenate([t.numpy() for t in gs], axis=2)
        topk = np.stack([np.stack([merge_topk(allk[q, r], alls[q, r], self.k) for r in range(R)])
                         for q in range(Q)])
        # 5. score halo: the first R - 1 slots' scores (every row) move down one rank
        a_len = [R if accepted is None else int(accepted[q]) for q in range(Q)]
        halo_w = max(R - 1, 1)
        mine = np.full((Q, R, halo_w), np.nan, np.float64)
        lo, hi = L.slots(self.rank)
        for q in range(Q):
            n = min(halo_w, hi - lo)
            mine[q, :, :n] = scores[q][:, lo: lo + n]
        halos = self._all_gather(torch.from_numpy(mine))
        below = halos[self.rank + 1].numpy() if self.rank + 1 < self.world else None
        # 6. replay of this rank's V entries and D offsets
        n_upd = [1 if (self.mtp_row0 and R > 1) else a_len[q] for q in range(Q)]
        for q, st in enumerate(self.reqs):
            sc = scores[q].copy()
            m = own[q].copy()
            if below is not None:  # the next rank's first slots, for this rank's last offsets
                nlo, nhi = L.slots(self.rank + 1)
                n = min(halo_w, nhi - nlo)
                sc[:, nlo: nlo + n] = below[q, :, :n]
                m[nlo // b: (nlo + n - 1) // b + 1] = masks[q][nlo // b: (nlo + n - 1) // b + 1]
            Vf = st.v_full(self.n_slots)
            Df = st.d_full(p0s[q], self.n_slots)
            with np.errstate(invalid="ignore"):
                self.backend.ema(Vf, Df, sc.astype(np.float32), m, ctxs[q], n_upd[q])
            st.V[:] = Vf[st.lo: st.hi]
            own_lo = st.d_lo(p0s[q])
            own_n = self._owned_offsets(st)
            k0 = max(0, -own_lo)
            k1 = min(own_n, self.n_slots - own_lo)
            if k1 > k0:
                st.D_ext[k0: k1] = Df[own_lo + k0: own_lo + k1]
        # 7. D halo: the a + R - 1 lowest owned offsets (after the update) move to the next rank
        send_w = R - 1 + max(a_len) if a_len else R
        out = np.full((Q, send_w), NEG_INF, np.float32)
        for q, st in enumerate(self.reqs):
            n = min(send_w, st.D_ext.size)
            out[q, :n] = st.D_ext[:n]
        dh = self._all_gather(torch.from_numpy(out))
        above = dh[self.rank - 1].numpy() if self.rank > 0 else None
        for q, st in enumerate(self.reqs):
            a = a_len[q]
            new = np.empty_like(st.D_ext)
            own_n = self._owned_offsets(st)
            # own offsets slide down by a: keep own[a:], then what the rank above
            # passes on (rank 0: offsets no row has reached yet)
            keep = st.D_ext[a: own_n]
            new[: keep.size] = keep
            add = st.D_ext.size - keep.size
            new[keep.size:] = above[q, :add] if above is not None else NEG_INF
            st.D_ext = new
            st.committed += a
        return masks, topk

    def _owned_offsets(self, st: ShardedRequestState) -> int:
        """Entries of the D window this rank owns: its hi - lo offsets, and for
        rank 0 also the R - 1 above them, which only its first slot reaches
        (rows r >= 1 of slot 0) and no other rank holds."""
        return st.D_ext.size if self.rank == 0 else st.hi - st.lo

    def _pad_blocks(self, S_own: np.ndarray) -> np.ndarray:
        width = max(self.layout.blocks(g)[1] - self.layout.blocks(g)[0] for g in range(self.world))
        out = np.full(S_own.shape[:2] + (width,), NEG_INF, np.float32)
        out[:, :, : S_own.shape[2]] = S_own
        return out

    def gather_state(self):
        """V and D of every request as full-length arrays on every rank (the
        owned entries of each rank), for checkpoints and checks."""
        Q = len(self.reqs)
        L = self.layout
        width = max(L.slots(g)[1] - L.slots(g)[0] for g in range(self.world))
        v = np.full((Q, width), np.nan, np.float32)
        d = np.full((Q, width), np.nan, np.float32)
        for q, st in enumerate(self.reqs):
            v[q, : st.V.size] = st.V
            d[q, : st.hi - st.lo] = st.D_ext[: st.hi - st.lo]
        gv = self._all_gather(torch.from_numpy(v))
        gd = self._all_gather(torch.from_numpy(d))
        V = np.full((Q, self.n_slots), np.nan, np.float32)
        D = np.full((Q, self.n_slots), np.nan, np.float32)
        for g in range(self.world):
            lo, hi = L.slots(g)
            V[:, lo:hi] = gv[g].numpy()[:, : hi - lo]
            for q, st in enumerate(self.reqs):
                p0 = st.committed          # row 0 of the next step
                d_lo = p0 - hi + 1
                vals = gd[g].numpy()[q, : hi - lo]
                for k in range(hi - lo):
                    off = d_lo + k
                    if 0 <= off < self.n_slots:
                        D[q, off] = vals[k]
        return V, D
