"""Seeded synthetic inputs shaped like the SPIN pages' workloads.

This module holds none of the SPIN method's arithmetic.  It only draws the
random inputs that both the CUDA path and the oracle consume: a paged index-key
cache (FP8 E4M3 codes plus a per-token fp32 scale, or fp32 keys), a block
table, query index vectors, head weights and, for speculative rows, accepted
lengths.  Every draw comes from a ``torch.Generator`` seeded from
(workload seed, purpose, layer, request), on the device the caller names, so a
test or benchmark generates once and hands copies to both sides.

Structure planted in the keys and queries:

* vertical lines: a fixed set of slots whose keys carry ``3 * u`` while every
  query carries ``sqrt(d) * u`` (u a unit vector per layer and request), so a
  planted slot's dot product sits about three standard deviations above an
  unplanted one for every query;
* diagonal bands: keys carry ``A * (cos(w i) e1 + sin(w i) e2)`` and queries
  ``sqrt(d) * (cos(w p) e1 + sin(w p) e2)`` in a plane orthogonal to u, with
  ``w = pi / (2 W)``, which adds ``A sqrt(d) cos(w (p - i))``: a boost for
  offsets below W that repeats every 4W;
* queries follow AR(1) over positions, ``q_p = 0.95 q_{p-1} + sqrt(1-0.95^2) e``;
  head weights are U(0, 1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import torch

K = 1024  # "512K" context = 524,288 slots


@dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    requests: int
    ctx0: Sequence[int]           # cached slots before the first decode step, per request
    steps: int                    # decode iterations (step 0 is the all-keep history bootstrap)
    rows: int = 1                 # query rows per step (1, or 1 verify + drafts)
    b: int = 64                   # paged-KV block size
    H: int = 64
    d: int = 128
    topk: int = 2048
    sparsity: float = 0.4         # target block sparsity
    gamma: float = 0.05           # exploration share of the block budget
    alpha: float = 0.9            # EMA decay
    seed: int = 0
    key_fp8: bool = True
    q_bf16: bool = True
    permute_pages: bool = False
    vertical: Sequence[float] = (0.01,)    # per layer: fraction (<1) or count (>=1) of planted slots
    diag_window: Sequence[int] = (2048,)   # per layer W
    diag_amp: Sequence[float] = (3.0,)     # per layer A
    accept_probs: Optional[Sequence[float]] = None  # P(a = 1..rows)
    warmup_steps: int = 0         # config with a per-layer budget: uniform-sparsity warm-up steps
    pooling: int = 0              # block reduction of the predicted scores: 0 max, 1 mean, 2 top-4
    mtp_policy: int = 0           # several rows: 0 row-local union + prefix-valid update, 1 row 0 alone
    spare_slots: int = 0          # extra capacity beyond ctx0 + steps * rows

    @property
    def max_slots(self) -> int:
        return max(self.ctx0) + self.steps * self.rows + self.spare_slots

    @property
    def max_blocks(self) -> int:
        return (self.max_slots + self.b - 1) // self.b

    def per_layer(self, seq, layer):
        return seq[layer % len(seq)]


def config(i: int, **over) -> Workload:
    """The five workloads: tiny fp32, DSA-shaped single request, serving batch
    at 512K, MTP rows, multi-layer ragged long context."""
    if i == 0:
        w = Workload("tiny-fp32-4K", layers=1, requests=1, ctx0=(4096,), steps=32, H=8, d=64,
                     topk=256, sparsity=0.3, gamma=0.05, seed=0, key_fp8=False, q_bf16=False,
                     vertical=(16,), diag_window=(128,))
    elif i == 1:
        w = Workload("dsa-1x64K", layers=1, requests=1, ctx0=(65536,), steps=64, sparsity=0.4,
                     seed=1, vertical=(256,), diag_window=(512,))
    elif i == 2:
        w = Workload("serve-96x512K", layers=1, requests=96, ctx0=(512 * K,) * 96, steps=16,
                     sparsity=0.5, seed=2, permute_pages=True, vertical=(0.01,),
                     diag_window=(2048,))
    elif i == 3:
        w = Workload("mtp-32x128K-r4", layers=1, requests=32, ctx0=(128 * K,) * 32, steps=32,
                     rows=4, sparsity=0.4, seed=3, vertical=(0.01,), diag_window=(2048,),
                     accept_probs=(0.30, 0.25, 0.20, 0.25))
    elif i == 4:
        g = torch.Generator().manual_seed(4_000_003)
        ctx = tuple(int(x) for x in torch.randint(256 * K, 1024 * K + 1, (8,), generator=g))
        w = Workload("ragged-8Lx8-256K-1M", layers=8, requests=8, ctx0=ctx, steps=41,
                     sparsity=0.5, gamma=0.10, seed=4, vertical=(0.01, 0.001),
                     diag_window=(2048, 2048), diag_amp=(1.0, 4.0), warmup_steps=16)
    else:
        raise ValueError(f"no workload {i}")
    return replace(w, **over) if over else w


def _gen(seed: int, purpose: int, layer: int, request: int, device) -> torch.Generator:
    s = (seed * 1_000_003 + purpose * 10_007 + layer * 101 + request * 7 + 12345) % (2**63 - 1)
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def _planted_dirs(wl: Workload, layer: int, request: int, device):
    """u, e1, e2: orthonormal, drawn per (layer, request)."""
    g = _gen(wl.seed, 1, layer, request, device)
    m = torch.randn(wl.d, 3, generator=g, device=device, dtype=torch.float64)
    qm, _ = torch.linalg.qr(m)
    return qm[:, 0].float(), qm[:, 1].float(), qm[:, 2].float()


def vertical_slots(wl: Workload, layer: int, request: int, device="cpu") -> torch.Tensor:
    P = wl.ctx0[request]
    v = wl.per_layer(wl.vertical, layer)
    count = int(round(v * P)) if v < 1 else int(v)
    g = _gen(wl.seed, 2, layer, request, device)
    return torch.randperm(P, generator=g, device=device)[:count]


@dataclass
class KeyCache:
    """Paged index-key cache of one layer: ``keys`` [pages, b, d] (uint8 E4M3
    codes, or fp32), ``kscale`` [pages, b] fp32 (ones for fp32 keys) and
    ``block_table`` [requests, max_blocks] int32 (logical block -> page)."""
    keys: torch.Tensor
    kscale: torch.Tensor
    block_table: torch.Tensor


def make_key_cache(wl: Workload, layer: int, device="cpu") -> KeyCache:
    Q, b, d, nb = wl.requests, wl.b, wl.d, wl.max_blocks
    pages = Q * nb
    if wl.permute_pages:
        g = _gen(wl.seed, 3, layer, 0, device)
        perm = torch.randperm(pages, generator=g, device=device).to(torch.int32)
    else:
        perm = torch.arange(pages, device=device, dtype=torch.int32)
    block_table = perm.view(Q, nb).contiguous()
    kdtype = torch.uint8 if wl.key_fp8 else torch.float32
    keys = torch.empty((pages, b, d), dtype=kdtype, device=device)
    kscale = torch.ones((pages, b), dtype=torch.float32, device=device)
    W = wl.per_layer(wl.diag_window, layer)
    A = wl.per_layer(wl.diag_amp, layer)
    omega = math.pi / (2 * W)
    for q in range(Q):
        g = _gen(wl.seed, 4, layer, q, device)
        k = torch.randn((nb * b, d), generator=g, device=device, dtype=torch.float32)
        u, e1, e2 = _planted_dirs(wl, layer, q, device)
        k[vertical_slots(wl, layer, q, device)] += 3.0 * u
        i = torch.arange(nb * b, device=device, dtype=torch.float64)
        k += A * (torch.cos(omega * i).float()[:, None] * e1 + torch.sin(omega * i).float()[:, None] * e2)
        k = k.view(nb, b, d)
        dest = block_table[q].long()
        if wl.key_fp8:
            amax = k.abs().amax(dim=-1)
            sigma = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
            k8 = (k / sigma[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
            keys[dest] = k8
            kscale[dest] = sigma
        else:
            keys[dest] = k
        del k
    return KeyCache(keys, kscale, block_table)


def make_queries(wl: Workload, layer: int, positions: int, device="cpu"):
    """Query vectors and head weights for ``positions`` consecutive positions
    starting at each request's ctx0: q [requests, positions, H, d] (bf16 or
    fp32), w [requests, positions, H] fp32."""
    Q, H, d = wl.requests, wl.H, wl.d
    eps = torch.empty((Q, positions, H, d), dtype=torch.float32, device=device)
    ws = torch.empty((Q, positions, H), dtype=torch.float32, device=device)
    plant = torch.empty((Q, positions, d), dtype=torch.float32, device=device)
    W = wl.per_layer(wl.diag_window, layer)
    omega = math.pi / (2 * W)
    rho = 0.95
    for q in range(Q):
        g = _gen(wl.seed, 5, layer, q, device)
        eps[q] = torch.randn((positions, H, d), generator=g, device=device, dtype=torch.float32)
        ws[q] = torch.rand((positions, H), generator=g, device=device, dtype=torch.float32)
        u, e1, e2 = _planted_dirs(wl, layer, q, device)
        p = wl.ctx0[q] + torch.arange(positions, device=device, dtype=torch.float64)
        plant[q] = math.sqrt(d) * (u[None, :] + torch.cos(omega * p).float()[:, None] * e1[None, :]
                                   + torch.sin(omega * p).float()[:, None] * e2[None, :])
    qs = torch.empty((Q, positions, H, d), dtype=torch.float32, device=device)
    x = eps[:, 0]
    c = math.sqrt(1 - rho * rho)
    for t in range(positions):
        if t > 0:
            x = rho * x + c * eps[:, t]
        qs[:, t] = x + plant[:, t, None, :]
    del eps
    if wl.q_bf16:
        return qs.to(torch.bfloat16), ws
    return qs, ws


def accepted_lengths(wl: Workload, steps: int, device="cpu") -> torch.Tensor:
    """[steps, requests] int32 in 1..rows (all ``rows`` when no distribution)."""
    if wl.accept_probs is None:
        return torch.full((steps, wl.requests), wl.rows, dtype=torch.int32, device=device)
    g = _gen(wl.seed, 6, 0, 0, "cpu")
    p = torch.tensor(wl.accept_probs, dtype=torch.float64)
    a = torch.multinomial(p, steps * wl.requests, replacement=True, generator=g) + 1
    return a.view(steps, wl.requests).to(torch.int32).to(device)


def request_pages(cache: KeyCache, request: int):
    """The pages of one request in logical order, moved to the CPU, with an
    identity block table: (keys [n, b, d], kscale [n, b], block_table [n])."""
    bt = cache.block_table[request].long()
    keys = cache.keys[bt].cpu()
    ks = cache.kscale[bt].cpu()
    ident = torch.arange(bt.numel(), dtype=torch.int32)
    return keys, ks, ident
