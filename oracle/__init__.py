"""Plain CPU oracle for the SPIN decode step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package.  The product library (``indexer_sparse_attention_b200``) never
imports it, and the two share no code: the arithmetic lives in
``spin_oracle.c`` (plain C, fp64 scores, fp32 EMA state with explicit
``fmaf``), this module only marshals numpy arrays and sequences the per-request
steps in the order the pages give them.

Every function cites the passage it follows in ``spin_oracle.c``.  Parity pins
for each function live in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spin_oracle.c")
_SO = os.path.join(_HERE, "libspin_oracle.so")
_lock = threading.Lock()
_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_i64 = ctypes.c_int64
_u64 = ctypes.c_uint64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no contraction, OpenMP over blocks)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", _SO, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_SO)
            lib.orc_philox4x32_10.argtypes = [_u32p, _u32p, _u32p]
            lib.orc_explore_key.argtypes = [_u64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32, _u64]
            lib.orc_explore_key.restype = ctypes.c_uint32
            lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_decode.restype = ctypes.c_double
            lib.orc_e4m3_encode.argtypes = [ctypes.c_double]
            lib.orc_e4m3_encode.restype = ctypes.c_uint8
            lib.orc_q_exponent.argtypes = [ctypes.c_double]
            lib.orc_q_exponent.restype = ctypes.c_int
            lib.orc_quantize_q.argtypes = [_f64p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           _u8p, _f32p, _i32p]
            lib.orc_num_blocks.argtypes = [_i64, ctypes.c_int, ctypes.c_int]
            lib.orc_num_blocks.restype = _i64
            lib.orc_predict_pool.argtypes = [_f32p, _f32p, _i64, ctypes.c_int, ctypes.c_int, _i64, _f32p]
            lib.orc_predict_pool_mode.argtypes = [_f32p, _f32p, _i64, ctypes.c_int, ctypes.c_int, _i64, ctypes.c_int,
                                                  _f32p]
            lib.orc_mean_exact.argtypes = [_f32p, ctypes.c_int]
            lib.orc_mean_exact.restype = ctypes.c_float
            lib.orc_budget.argtypes = [_i64, ctypes.c_double]
            lib.orc_budget.restype = _i64
            lib.orc_explore_count.argtypes = [_i64, ctypes.c_double]
            lib.orc_explore_count.restype = _i64
            lib.orc_select.argtypes = [_f32p, _i64, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                       ctypes.c_float, _u64, ctypes.c_uint32, ctypes.c_uint32, _u64, ctypes.c_int,
                                       _u8p]
            lib.orc_score_fp8.argtypes = [_u8p, _f32p, _i32p, ctypes.c_int, ctypes.c_int, _u8p, _f32p,
                                          ctypes.c_int, ctypes.c_int, _i64, _u8p, _i64, _f64p]
            lib.orc_score_f32.argtypes = [_f32p, _i32p, ctypes.c_int, ctypes.c_int, _f32p, _f32p,
                                          ctypes.c_int, ctypes.c_int, _i64, _u8p, _i64, _f64p]
            lib.orc_topk_row.argtypes = [_f64p, _u8p, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p]
            lib.orc_topk_row.restype = _i64
            lib.orc_ema_beta.argtypes = [ctypes.c_float]
            lib.orc_ema_beta.restype = ctypes.c_float
            lib.orc_ema_update.argtypes = [_f32p, _f32p, _f32p, _u8p, _i64, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_float, _i64]
            lib.orc_slot_prediction.argtypes = [_f32p, _f32p, _i64, ctypes.c_int, _i64, _f32p]
            lib.orc_random_prediction.argtypes = [_u64, ctypes.c_uint32, ctypes.c_uint32, _u64, _i64, ctypes.c_int,
                                                  _i64, _f32p]
            lib.orc_pearson.argtypes = [_f32p, _f32p, _i64]
            lib.orc_pearson.restype = ctypes.c_double
            lib.orc_miss_fraction.argtypes = [_i32p, ctypes.c_int, _u8p, ctypes.c_int]
            lib.orc_miss_fraction.restype = ctypes.c_double
            lib.orc_layer_sparsity.argtypes = [_f64p, _f64p, _f64p, ctypes.c_int, ctypes.c_double, _f64p]
            _lib = lib
    return _lib


def _p(a: np.ndarray, t):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(t)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# primitives
# --------------------------------------------------------------------------
def philox4x32_10(ctr, key) -> np.ndarray:
    lib = _load()
    c = _c(ctr, np.uint32)
    k = _c(key, np.uint32)
    out = np.zeros(4, np.uint32)
    lib.orc_philox4x32_10(_p(c, _u32p), _p(k, _u32p), _p(out, _u32p))
    return out


def explore_key(seed: int, block: int, request: int, layer: int, step: int) -> int:
    return int(_load().orc_explore_key(seed, block, request, layer, step))


def e4m3_decode(code: int) -> float:
    return float(_load().orc_e4m3_decode(code))


def e4m3_encode(x: float) -> int:
    return int(_load().orc_e4m3_encode(float(x)))


def q_exponent(amax: float) -> int:
    return int(_load().orc_q_exponent(float(amax)))


def num_blocks(ctx_len: int, row: int, b: int) -> int:
    return int(_load().orc_num_blocks(ctx_len, row, b))


def budget(n: int, sparsity: float) -> int:
    return int(_load().orc_budget(n, float(np.float32(sparsity))))


def explore_count(budget_row0: int, gamma: float) -> int:
    return int(_load().orc_explore_count(budget_row0, float(np.float32(gamma))))


def ema_beta(alpha: float) -> np.float32:
    return np.float32(_load().orc_ema_beta(alpha))


def quantize_q(q: np.ndarray, w: np.ndarray):
    """q [rows,H,d] (any float dtype, widened exactly), w [rows,H] fp32 ->
    (q8 codes uint8 [rows,H,d], w' fp32 [rows,H], e int32 [rows,H])."""
    lib = _load()
    q = _c(q, np.float64)
    w = _c(w, np.float32)
    rows, H, d = q.shape
    q8 = np.zeros((rows, H, d), np.uint8)
    wq = np.zeros((rows, H), np.float32)
    e = np.zeros((rows, H), np.int32)
    lib.orc_quantize_q(_p(q, _f64p), _p(w, _f32p), rows, H, d, _p(q8, _u8p), _p(wq, _f32p), _p(e, _i32p))
    return q8, wq, e


POOL_MAX, POOL_MEAN, POOL_TOP4 = 0, 1, 2


def mean_exact(z) -> np.float32:
    """The mean of 1..256 floats: the exact sum over the count, rounded once
    to the nearest float (the definition the Mean and Top-4 pools use)."""
    z = _c(np.atleast_1d(z), np.float32)
    return np.float32(_load().orc_mean_exact(_p(z, _f32p), int(z.size)))


def predict_pool(V: np.ndarray, D: np.ndarray, ctx_len: int, rows: int, b: int, n_stride: int, pooling: int = 0):
    """Block scores S [rows, n_stride] (entries past each row's block count are
    NaN); pooling: POOL_MAX (the method's), POOL_MEAN or POOL_TOP4."""
    lib = _load()
    V = _c(V, np.float32)
    D = _c(D, np.float32)
    S = np.full((rows, n_stride), np.nan, np.float32)
    lib.orc_predict_pool_mode(_p(V, _f32p), _p(D, _f32p), ctx_len, rows, b, n_stride, int(pooling), _p(S, _f32p))
    return S


# MTP policies (SPIN listing, Table 7 and Figure 2): the method's row-local
# union of the rows' masks with a prefix-valid EMA replay, or the baseline
# that shares row 0's mask and updates the EMA from row 0 alone.
MTP_UNION_PREFIX, MTP_ROW0 = 0, 1


def select(S: np.ndarray, ctx_len: int, rows: int, b: int, sparsity: float, gamma: float,
           seed: int, request: int, layer: int, step: int, mtp_policy: int = MTP_UNION_PREFIX) -> np.ndarray:
    lib = _load()
    S = _c(S, np.float32)
    n_stride = S.shape[1]
    mask = np.zeros(n_stride, np.uint8)
    lib.orc_select(_p(S, _f32p), n_stride, ctx_len, rows, b, float(sparsity), float(gamma), seed,
                   request, layer, step, int(mtp_policy), _p(mask, _u8p))
    return mask


def update_rows(mtp_policy: int, accepted: int) -> int:
    """Rows whose scores the EMA update replays: the accepted prefix, or row 0
    alone under the row-0 policy."""
    return min(accepted, 1) if mtp_policy == MTP_ROW0 else accepted


def score_fp8(keys8, kscale, block_table, q8, wq, ctx_len, mask, slot_stride):
    """keys8 [pages,b,d] uint8, kscale [pages,b] fp32, block_table [n] int32,
    q8 [rows,H,d] uint8, wq [rows,H] fp32 -> fp64 scores [rows, slot_stride]
    (NaN where not scored)."""
    lib = _load()
    keys8 = _c(keys8, np.uint8)
    kscale = _c(kscale, np.float32)
    bt = _c(block_table, np.int32)
    q8 = _c(q8, np.uint8)
    wq = _c(wq, np.float32)
    mask = _c(mask, np.uint8)
    _, b, d = keys8.shape
    rows, H, _ = q8.shape
    out = np.full((rows, slot_stride), np.nan, np.float64)
    lib.orc_score_fp8(_p(keys8, _u8p), _p(kscale, _f32p), _p(bt, _i32p), b, d, _p(q8, _u8p),
                      _p(wq, _f32p), H, rows, ctx_len, _p(mask, _u8p), slot_stride, _p(out, _f64p))
    return out


def score_f32(keys, block_table, q, w, ctx_len, mask, slot_stride):
    lib = _load()
    keys = _c(keys, np.float32)
    bt = _c(block_table, np.int32)
    q = _c(q, np.float32)
    w = _c(w, np.float32)
    mask = _c(mask, np.uint8)
    _, b, d = keys.shape
    rows, H, _ = q.shape
    out = np.full((rows, slot_stride), np.nan, np.float64)
    lib.orc_score_f32(_p(keys, _f32p), _p(bt, _i32p), b, d, _p(q, _f32p), _p(w, _f32p), H, rows,
                      ctx_len, _p(mask, _u8p), slot_stride, _p(out, _f64p))
    return out


def topk_row(scores_row, mask, ctx_len: int, row: int, b: int, k: int) -> np.ndarray:
    lib = _load()
    sr = _c(scores_row, np.float64)
    mask = _c(mask, np.uint8)
    out = np.zeros(k, np.int32)
    lib.orc_topk_row(_p(sr, _f64p), _p(mask, _u8p), ctx_len, row, b, k, _p(out, _i32p))
    return out


def ema_update(V: np.ndarray, D: np.ndarray, scores32: np.ndarray, mask, ctx_len: int,
               accepted: int, b: int, alpha: float) -> None:
    """In place on V and D (fp32, C-contiguous)."""
    lib = _load()
    assert V.dtype == np.float32 and D.dtype == np.float32
    assert V.flags["C_CONTIGUOUS"] and D.flags["C_CONTIGUOUS"]
    s32 = _c(scores32, np.float32)
    mask = _c(mask, np.uint8)
    lib.orc_ema_update(_p(V, _f32p), _p(D, _f32p), _p(s32, _f32p), _p(mask, _u8p), ctx_len,
                       accepted, b, float(alpha), s32.shape[1])


# --------------------------------------------------------------------------
# predictor quality (SPIN listing, Table 1)
# --------------------------------------------------------------------------
def slot_prediction(V: np.ndarray, D: np.ndarray, ctx_len: int, rows: int, slot_stride: int) -> np.ndarray:
    """z = max(V_s, D_{p_r - s}) per visible slot, -inf where not finite;
    [rows, slot_stride], NaN past each row's position."""
    lib = _load()
    V = _c(V, np.float32)
    D = _c(D, np.float32)
    out = np.full((rows, slot_stride), np.nan, np.float32)
    lib.orc_slot_prediction(_p(V, _f32p), _p(D, _f32p), ctx_len, rows, slot_stride, _p(out, _f32p))
    return out


def random_prediction(seed: int, request: int, layer: int, step: int, ctx_len: int, rows: int,
                      slot_stride: int) -> np.ndarray:
    lib = _load()
    out = np.full((rows, slot_stride), np.nan, np.float32)
    lib.orc_random_prediction(seed, request, layer, step, ctx_len, rows, slot_stride, _p(out, _f32p))
    return out


def pearson(x, y) -> float:
    """Over the entries where both are finite; 0 if fewer than two or constant."""
    lib = _load()
    x = _c(x, np.float32)
    y = _c(y, np.float32)
    assert x.shape == y.shape
    return float(lib.orc_pearson(_p(x, _f32p), _p(y, _f32p), x.size))


def topk_visible(values_row, ctx_len: int, row: int, k: int) -> np.ndarray:
    """Top-k (value desc, lower slot first) over every visible slot of a row:
    the token top-k with all blocks kept, block size 1."""
    v = np.asarray(values_row, np.float64)
    p = ctx_len - 1 + row
    return topk_row(v, np.ones(p + 1, np.uint8), ctx_len, row, 1, k)


def miss_fraction(full_topk, mask, b: int) -> float:
    lib = _load()
    ft = _c(full_topk, np.int32)
    mask = _c(mask, np.uint8)
    return float(lib.orc_miss_fraction(_p(ft, _i32p), ft.shape[0], _p(mask, _u8p), b))


def layer_sparsity(miss, N, lo, s_glob: float) -> np.ndarray:
    lib = _load()
    m = _c(miss, np.float64)
    n = _c(N, np.float64)
    lo = _c(lo, np.float64)
    out = np.zeros(m.shape[0], np.float64)
    lib.orc_layer_sparsity(_p(m, _f64p), _p(n, _f64p), _p(lo, _f64p), m.shape[0], float(s_glob),
                           _p(out, _f64p))
    return out


def p99(values) -> float:
    """Nearest-rank 99th percentile."""
    v = np.sort(np.asarray(values, np.float64))
    if v.size == 0:
        return 0.0
    rank = int(np.ceil(0.99 * v.size))
    return float(v[max(rank, 1) - 1])


# --------------------------------------------------------------------------
# one decode step for one (layer, request): the pages' order of operations
# --------------------------------------------------------------------------
def decode_step_request(*, V, D, ctx_len, rows, b, sparsity, gamma, alpha, seed, request, layer,
                        step, topk, q, w, keys, kscale, block_table, key_fp8: bool,
                        accepted=None, scores_in=None, n_stride=None, update=True,
                        pooling=POOL_MAX, mtp_policy=MTP_UNION_PREFIX):
    """Run predict -> pool -> select -> score -> top-k -> EMA update for one
    request.  V and D (fp32, [max_slots]) are updated in place when ``update``.

    ``scores_in`` (fp32 [rows, slot_stride]) switches to lock-step mode: the
    given scores (e.g. a GPU's) replace the oracle's own for the top-k and the
    update, so that selection and state can be compared bit for bit.
    Returns a dict with S, mask, q8/wq (FP8 only), scores (fp64), topk [rows,k].
    """
    if n_stride is None:
        n_stride = block_table.shape[0]
    slot_stride = n_stride * b
    S = predict_pool(V, D, ctx_len, rows, b, n_stride, pooling)
    mask = select(S, ctx_len, rows, b, sparsity, gamma, seed, request, layer, step, mtp_policy)
    out = {"S": S, "mask": mask}
    if key_fp8:
        q8, wq, e = quantize_q(q, w)
        out.update(q8=q8, wq=wq, e=e)
        scores = score_fp8(keys, kscale, block_table, q8, wq, ctx_len, mask, slot_stride)
    else:
        scores = score_f32(keys, block_table, q, w, ctx_len, mask, slot_stride)
    out["scores"] = scores
    used = scores if scores_in is None else np.asarray(scores_in, np.float64)
    out["topk"] = np.stack([topk_row(used[r], mask, ctx_len, r, b, topk) for r in range(rows)])
    if update:
        s32 = (scores.astype(np.float32) if scores_in is None
               else np.ascontiguousarray(scores_in, np.float32))
        ema_update(V, D, s32, mask, ctx_len, update_rows(mtp_policy, rows if accepted is None else accepted),
                   b, alpha)
    return out
