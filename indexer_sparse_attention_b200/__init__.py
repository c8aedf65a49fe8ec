"""Python binding of libspin.so, the SPIN (Shadow Predictive Indexer) decode
step for B200 (sm_100a).

Argument marshalling only: every function has the name of the C entry point it
calls (``include/spin.h``) and passes raw device pointers and sizes taken from
PyTorch tensors.  All arithmetic runs in the library's CUDA kernels; there is
no fallback of any kind.  Importing the package does not load the library;
the first call does, and raises if ``libspin.so`` has not been built
(``python -m indexer_sparse_attention_b200.build``) or no CUDA device is present.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "SpinConfig", "SpinError", "SpinState", "load", "SPIN_F32", "SPIN_BF16", "SPIN_FP8_E4M3",
    "SPIN_SCORE_AUTO", "SPIN_SCORE_SIMT", "SPIN_SCORE_TCGEN05",
    "spin_state_bytes", "spin_predict_select", "spin_indexer_score", "spin_topk", "spin_ema_update",
    "spin_decode_step", "spin_miss_count", "spin_allocate_layer_sparsity", "spin_get_error",
    "spin_set_layer_sparsity", "spin_set_score_kernel", "spin_reset_requests", "spin_set_fault_injection",
    "spin_state_export", "spin_state_import", "spin_status_string", "spin_set_kernel_timing",
    "spin_kernel_times", "STAGES", "spin_topk_noalloc", "spin_topk_noalloc_error", "spin_set_lookahead", "spin_prepare_selections", "spin_set_kernel_timing_mask",
    "SPIN_STEP_DEVICE", "spin_set_step", "spin_advance_step", "SPIN_POOL_MAX", "SPIN_POOL_MEAN", "SPIN_POOL_TOP4",
    "SPIN_MTP_UNION_PREFIX", "SPIN_MTP_ROW0", "SPIN_PRED_EMA", "SPIN_PRED_RANDOM", "spin_slot_prediction",
    "spin_pearson", "spin_topk_overlap",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspin.so")

SPIN_F32, SPIN_BF16, SPIN_FP8_E4M3 = 0, 1, 2
SPIN_SCORE_AUTO, SPIN_SCORE_SIMT, SPIN_SCORE_TCGEN05 = 0, 1, 2
SPIN_STEP_DEVICE = -1  # step argument: read the state's device step counter
SPIN_POOL_MAX, SPIN_POOL_MEAN, SPIN_POOL_TOP4 = 0, 1, 2  # block reduction of the predicted scores
SPIN_MTP_UNION_PREFIX, SPIN_MTP_ROW0 = 0, 1  # mask / EMA policy for several query rows
SPIN_PRED_EMA, SPIN_PRED_RANDOM = 0, 1  # slot predictors of the quality profile
STATUS_NAMES = {0: "SPIN_OK", 1: "SPIN_EINVAL", 2: "SPIN_ENOMEM", 3: "SPIN_ECUDA", 4: "SPIN_ESTATE",
                5: "SPIN_ETIMEOUT", 6: "SPIN_EDEVICE", 7: "SPIN_EUNSUPPORTED"}


class SpinConfig(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("num_requests", ctypes.c_int32),
                ("max_slots", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("max_rows", ctypes.c_int32),
                ("key_dtype", ctypes.c_int32), ("q_dtype", ctypes.c_int32),
                ("alpha", ctypes.c_float), ("gamma", ctypes.c_float),
                ("target_sparsity", ctypes.c_float), ("seed", ctypes.c_uint64), ("pooling", ctypes.c_int32),
                ("mtp_policy", ctypes.c_int32)]


class SpinError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({_lib_or_none_msg(status)})")


def _lib_or_none_msg(status):
    try:
        return load().spin_status_string(status).decode()
    except Exception:  # library missing: the status code is still meaningful
        return "libspin unavailable"


_lib = None
_vp = ctypes.c_void_p
_i32, _i64, _u32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32


def load():
    """Loads libspin.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libspin.so not built at {LIB_PATH}; run python -m indexer_sparse_attention_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    S = ctypes.c_int
    sig = {
        "spin_state_bytes": (ctypes.c_size_t, [ctypes.POINTER(SpinConfig)]),
        "spin_state_create": (S, [ctypes.POINTER(SpinConfig), _vp, ctypes.c_size_t, _vp, ctypes.POINTER(_vp)]),
        "spin_state_destroy": (S, [_vp]),
        "spin_set_layer_sparsity": (S, [_vp, _vp]),
        "spin_set_score_kernel": (S, [_vp, ctypes.c_int]),
        "spin_set_fault_injection": (S, [_vp, ctypes.c_int]),
        "spin_set_kernel_timing": (S, [_vp, ctypes.c_int]),
        "spin_set_kernel_timing_mask": (S, [_vp, _u32]),
        "spin_set_step": (S, [_vp, _i64, _vp]),
        "spin_set_lookahead": (S, [_vp, ctypes.c_int]),
        "spin_prepare_selections": (S, [_vp, _i64, _vp, _vp]),
        "spin_advance_step": (S, [_vp, _vp]),
        "spin_kernel_times": (S, [_vp, _vp, _vp, ctypes.c_int]),
        "spin_reset_requests": (S, [_vp, ctypes.c_int, _vp, ctypes.c_int, _vp]),
        "spin_predict_select": (S, [_vp, ctypes.c_int, ctypes.c_int, _i64, _vp, _vp, _vp]),
        "spin_indexer_score": (S, [_vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _i32, _vp, _i32, _vp, _vp, _vp,
                                   _vp, _vp, _vp]),
        "spin_topk": (S, [_vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp]),
        "spin_topk_noalloc": (S, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32, ctypes.c_int, ctypes.c_int, _vp,
                                  _vp, _vp, _vp, _vp]),
        "spin_topk_noalloc_error": (S, [_vp, ctypes.POINTER(_u32)]),
        "spin_ema_update": (S, [_vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp]),
        "spin_decode_step": (S, [_vp, ctypes.c_int, ctypes.c_int, _i64, _vp, _vp, _i32, _vp, _i32, _vp, _vp, _vp,
                                 ctypes.c_int, _vp, _vp, _vp, _vp]),
        "spin_miss_count": (S, [_vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp]),
        "spin_slot_prediction": (S, [_vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i64, _vp, _vp, _vp]),
        "spin_pearson": (S, [_vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp]),
        "spin_topk_overlap": (S, [_vp, ctypes.c_int, _vp, _vp, _vp, _vp]),
        "spin_allocate_layer_sparsity": (S, [ctypes.c_int, _vp, _vp, _vp, ctypes.c_double, _vp]),
        "spin_get_error": (S, [_vp, _vp, ctypes.POINTER(_u32)]),
        "spin_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "spin_state_export_bytes": (ctypes.c_size_t, [_vp]),
        "spin_state_export": (S, [_vp, _vp, ctypes.c_size_t, _vp]),
        "spin_state_import": (S, [_vp, _vp, ctypes.c_size_t, _vp]),
        "spin_state_ema": (S, [_vp, ctypes.c_int, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_i64)]),
        "spin_state_vmax": (S, [_vp, ctypes.c_int, ctypes.POINTER(_vp), ctypes.POINTER(_i64)]),
        "spin_state_refresh": (S, [_vp, ctypes.c_int, _vp]),
        "spin_state_block_scores": (S, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_i64)]),
        "spin_state_qquant": (S, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp)]),
        "spin_score_stride": (_i64, [_vp]),
        "spin_mask_stride": (_i64, [_vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise SpinError(status, where)


def _stream(stream) -> _vp:
    if stream is None:
        stream = torch.cuda.current_stream()
    return _vp(stream.cuda_stream)


def _dev(t: Optional[torch.Tensor], name: str, dtype=None) -> _vp:
    if t is None:
        return _vp(0)
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return _vp(t.data_ptr())


def make_config(*, num_layers, num_requests, max_slots, block_size=64, num_heads=64, head_dim=128, topk=2048,
                max_rows=1, key_fp8=True, q_bf16=True, alpha=0.9, gamma=0.05, target_sparsity=0.5,
                seed=0, pooling=SPIN_POOL_MAX, mtp_policy=SPIN_MTP_UNION_PREFIX) -> SpinConfig:
    return SpinConfig(num_layers, num_requests, max_slots, block_size, num_heads, head_dim, topk, max_rows,
                      SPIN_FP8_E4M3 if key_fp8 else SPIN_F32, SPIN_BF16 if q_bf16 else SPIN_F32,
                      alpha, gamma, target_sparsity, seed, pooling, mtp_policy)


def spin_state_bytes(cfg: SpinConfig) -> int:
    return int(load().spin_state_bytes(ctypes.byref(cfg)))


class SpinState:
    """A state (EMA V and D of every layer and request, plus scratch) living
    in one device buffer allocated with PyTorch and handed to
    ``spin_state_create``."""

    def __init__(self, cfg: SpinConfig, device="cuda", stream=None):
        lib = load()
        self.cfg = cfg
        nbytes = lib.spin_state_bytes(ctypes.byref(cfg))
        if nbytes == 0:
            raise SpinError(1, "spin_state_bytes (invalid config)")
        self.nbytes = nbytes
        self.mem = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.mem.data_ptr()) % 256
        self.base = self.mem[off:off + nbytes]
        h = _vp()
        _check(lib.spin_state_create(ctypes.byref(cfg), _vp(self.base.data_ptr()), nbytes, _stream(stream),
                                     ctypes.byref(h)), "spin_state_create")
        self.handle = h
        self.score_stride = int(lib.spin_score_stride(h))
        self.mask_stride = int(lib.spin_mask_stride(h))

    # device views into the state block (for tests and inspection)
    def _view(self, ptr: int, count: int, dtype, shape):
        off = ptr - self.base.data_ptr()
        nb = count * torch.tensor([], dtype=dtype).element_size()
        return self.base[off:off + nb].view(dtype).view(shape)

    def ema(self, layer: int):
        V, D, st = _vp(), _vp(), _i64()
        _check(load().spin_state_ema(self.handle, layer, ctypes.byref(V), ctypes.byref(D), ctypes.byref(st)),
               "spin_state_ema")
        Q = self.cfg.num_requests
        return (self._view(V.value, Q * st.value, torch.float32, (Q, st.value)),
                self._view(D.value, Q * st.value, torch.float32, (Q, st.value)))

    def vmax(self, layer: int):
        """V's 32-slot group maxima of a layer, [Q][slot_stride / 32], or None."""
        p, st = _vp(), _i64()
        _check(load().spin_state_vmax(self.handle, layer, ctypes.byref(p), ctypes.byref(st)), "spin_state_vmax")
        if not p.value:
            return None
        Q = self.cfg.num_requests
        return self._view(p.value, Q * st.value, torch.float32, (Q, st.value))

    def refresh(self, layer: int = -1, stream=None):
        """After writing V or D through ema(): brings the state's derived data up to date."""
        _check(load().spin_state_refresh(self.handle, layer, _stream(stream)), "spin_state_refresh")

    def block_scores(self):
        S, st = _vp(), _i64()
        _check(load().spin_state_block_scores(self.handle, ctypes.byref(S), ctypes.byref(st)), "block_scores")
        Q, R = self.cfg.num_requests, self.cfg.max_rows
        return self._view(S.value, Q * R * st.value, torch.float32, (Q, R, st.value))

    def qquant(self, rows: int):
        q8, wq = _vp(), _vp()
        _check(load().spin_state_qquant(self.handle, ctypes.byref(q8), ctypes.byref(wq)), "qquant")
        Q, H, d = self.cfg.num_requests, self.cfg.num_heads, self.cfg.head_dim
        return (self._view(q8.value, Q * rows * H * d, torch.uint8, (Q, rows, H, d)),
                self._view(wq.value, Q * rows * H, torch.float32, (Q, rows, H)))

    def new_scores(self):
        return torch.empty((self.cfg.num_requests, self.cfg.max_rows, self.score_stride), dtype=torch.float32,
                           device=self.base.device)

    def new_mask(self):
        return torch.zeros((self.cfg.num_requests, self.mask_stride), dtype=torch.uint8, device=self.base.device)

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            load().spin_state_destroy(self.handle)
            self.handle = _vp(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# --------------------------------------------------------------------------
# entry points (same names as the C ABI)
# --------------------------------------------------------------------------
def spin_set_layer_sparsity(st: SpinState, sparsity) -> None:
    arr = (ctypes.c_float * st.cfg.num_layers)(*[float(x) for x in sparsity])
    _check(load().spin_set_layer_sparsity(st.handle, ctypes.cast(arr, _vp)), "spin_set_layer_sparsity")


def spin_set_score_kernel(st: SpinState, kind: int) -> None:
    _check(load().spin_set_score_kernel(st.handle, kind), "spin_set_score_kernel")


def spin_set_fault_injection(st: SpinState, mode: int) -> None:
    _check(load().spin_set_fault_injection(st.handle, mode), "spin_set_fault_injection")


STAGES = ["predict", "select", "quantize", "score", "topk", "ema", "compact", "miss"]


def spin_set_kernel_timing(st: SpinState, enable: bool) -> None:
    _check(load().spin_set_kernel_timing(st.handle, int(bool(enable))), "spin_set_kernel_timing")


def spin_set_step(st: SpinState, step: int, stream=None) -> None:
    _check(load().spin_set_step(st.handle, int(step), _stream(stream)), "spin_set_step")


def spin_set_lookahead(st: SpinState, enable: bool = True) -> None:
    """Pipelined one-row decode steps: each step prepares the next step's
    selection, whose select kernel runs beside the step's top-k on a second
    stream (see include/spin.h)."""
    _check(load().spin_set_lookahead(st.handle, 1 if enable else 0), "spin_set_lookahead")


def spin_advance_step(st: SpinState, stream=None) -> None:
    _check(load().spin_advance_step(st.handle, _stream(stream)), "spin_advance_step")


def spin_set_kernel_timing_mask(st: SpinState, stages) -> None:
    """Time only the named stages (see STAGES); the others run without events."""
    mask = 0
    for name in stages:
        if name not in STAGES:
            raise ValueError(f"unknown stage {name!r}; stages are {STAGES}")
        mask |= 1 << STAGES.index(name)
    _check(load().spin_set_kernel_timing_mask(st.handle, mask), "spin_set_kernel_timing_mask")


def spin_kernel_times(st: SpinState):
    """{stage: (milliseconds, launches)} since the last call (synchronises)."""
    n = len(STAGES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(load().spin_kernel_times(st.handle, ctypes.cast(ms, _vp), ctypes.cast(cnt, _vp), n),
           "spin_kernel_times")
    return {STAGES[i]: (float(ms[i]), int(cnt[i])) for i in range(n)}


def spin_reset_requests(st: SpinState, layer: int, requests, stream=None) -> None:
    req = (ctypes.c_int32 * len(requests))(*[int(r) for r in requests])
    _check(load().spin_reset_requests(st.handle, layer, ctypes.cast(req, _vp), len(requests), _stream(stream)),
           "spin_reset_requests")


def spin_prepare_selections(st: SpinState, step: int, ctx_len: torch.Tensor, stream=None) -> None:
    """Every layer's one-row selection of `step`, made at once on the state's
    prepare streams; each layer's next pipelined decode step scores it (see
    include/spin.h)."""
    _check(load().spin_prepare_selections(st.handle, step, _dev(ctx_len, "ctx_len", torch.int32), _stream(stream)),
           "spin_prepare_selections")


def spin_predict_select(st: SpinState, layer: int, rows: int, step: int, ctx_len: torch.Tensor,
                        mask: torch.Tensor, stream=None) -> None:
    _check(load().spin_predict_select(st.handle, layer, rows, step, _dev(ctx_len, "ctx_len", torch.int32),
                                      _dev(mask, "mask", torch.uint8), _stream(stream)), "spin_predict_select")


def spin_indexer_score(st: SpinState, layer: int, rows: int, keys: torch.Tensor, key_scale, block_table,
                       q, w, ctx_len, mask, scores, stream=None) -> None:
    _check(load().spin_indexer_score(
        st.handle, layer, rows, _dev(keys, "keys"), _dev(key_scale, "key_scale", torch.float32), keys.shape[0],
        _dev(block_table, "block_table", torch.int32), block_table.shape[-1], _dev(q, "q"),
        _dev(w, "w", torch.float32), _dev(ctx_len, "ctx_len", torch.int32), _dev(mask, "mask", torch.uint8),
        _dev(scores, "scores", torch.float32), _stream(stream)), "spin_indexer_score")


def spin_topk(st: SpinState, rows: int, scores, mask, ctx_len, topk, stream=None) -> None:
    _check(load().spin_topk(st.handle, rows, _dev(scores, "scores", torch.float32), _dev(mask, "mask", torch.uint8),
                            _dev(ctx_len, "ctx_len", torch.int32), _dev(topk, "topk", torch.int32),
                            _stream(stream)), "spin_topk")


def spin_topk_noalloc(num_requests: int, rows: int, max_rows: int, max_slots: int, block_size: int, k: int,
                      scores, mask, ctx_len, topk, stream=None) -> None:
    """Stateless top-k with the library's fixed scratch (no device allocation
    anywhere); see include/spin.h for its size limit and sharing rules."""
    _check(load().spin_topk_noalloc(num_requests, rows, max_rows, max_slots, block_size, k,
                                    _dev(scores, "scores", torch.float32), _dev(mask, "mask", torch.uint8),
                                    _dev(ctx_len, "ctx_len", torch.int32), _dev(topk, "topk", torch.int32),
                                    _stream(stream)), "spin_topk_noalloc")


def spin_topk_noalloc_error(stream=None):
    """Returns (status, raw device error word) of the last spin_topk_noalloc
    call on the current device; synchronises the stream."""
    word = _u32()
    status = load().spin_topk_noalloc_error(_stream(stream), ctypes.byref(word))
    return int(status), int(word.value)


def spin_ema_update(st: SpinState, layer: int, rows: int, scores, mask, ctx_len, accepted=None,
                    stream=None) -> None:
    _check(load().spin_ema_update(st.handle, layer, rows, _dev(scores, "scores", torch.float32),
                                  _dev(mask, "mask", torch.uint8), _dev(ctx_len, "ctx_len", torch.int32),
                                  _dev(accepted, "accepted", torch.int32), _stream(stream)), "spin_ema_update")


def spin_decode_step(st: SpinState, layer: int, rows: int, step: int, keys, key_scale, block_table, q, w,
                     ctx_len, defer_update: bool, mask, topk, scores=None, stream=None) -> None:
    _check(load().spin_decode_step(
        st.handle, layer, rows, step, _dev(keys, "keys"), _dev(key_scale, "key_scale", torch.float32),
        keys.shape[0], _dev(block_table, "block_table", torch.int32), block_table.shape[-1], _dev(q, "q"),
        _dev(w, "w", torch.float32), _dev(ctx_len, "ctx_len", torch.int32), int(bool(defer_update)),
        _dev(mask, "mask", torch.uint8), _dev(topk, "topk", torch.int32), _dev(scores, "scores", torch.float32),
        _stream(stream)), "spin_decode_step")


def spin_miss_count(st: SpinState, rows: int, full_topk, mask, missed, total, stream=None) -> None:
    _check(load().spin_miss_count(st.handle, rows, _dev(full_topk, "full_topk", torch.int32),
                                  _dev(mask, "mask", torch.uint8), _dev(missed, "missed", torch.int32),
                                  _dev(total, "total", torch.int32), _stream(stream)), "spin_miss_count")


def spin_slot_prediction(st: SpinState, layer: int, rows: int, kind: int, step: int, ctx_len, pred,
                         stream=None) -> None:
    _check(load().spin_slot_prediction(st.handle, layer, rows, kind, step, _dev(ctx_len, "ctx_len", torch.int32),
                                       _dev(pred, "pred", torch.float32), _stream(stream)), "spin_slot_prediction")


def spin_pearson(st: SpinState, rows: int, x, y, ctx_len, out, stream=None) -> None:
    _check(load().spin_pearson(st.handle, rows, _dev(x, "x", torch.float32), _dev(y, "y", torch.float32),
                               _dev(ctx_len, "ctx_len", torch.int32), _dev(out, "out", torch.float64),
                               _stream(stream)), "spin_pearson")


def spin_topk_overlap(st: SpinState, rows: int, a, b, out, stream=None) -> None:
    _check(load().spin_topk_overlap(st.handle, rows, _dev(a, "a", torch.int32), _dev(b, "b", torch.int32),
                                    _dev(out, "out", torch.int32), _stream(stream)), "spin_topk_overlap")


def spin_allocate_layer_sparsity(miss, blocks, lo, s_glob: float):
    n = len(miss)
    arr = lambda xs: (ctypes.c_double * n)(*[float(x) for x in xs])
    out = (ctypes.c_float * n)()
    _check(load().spin_allocate_layer_sparsity(n, ctypes.cast(arr(miss), _vp), ctypes.cast(arr(blocks), _vp),
                                               ctypes.cast(arr(lo), _vp), float(s_glob), ctypes.cast(out, _vp)),
           "spin_allocate_layer_sparsity")
    return [float(x) for x in out]


def spin_get_error(st: SpinState, stream=None):
    """Returns (status, raw device error word); synchronises the stream."""
    word = _u32()
    status = load().spin_get_error(st.handle, _stream(stream), ctypes.byref(word))
    return int(status), int(word.value)


def spin_state_export(st: SpinState, stream=None) -> bytes:
    n = load().spin_state_export_bytes(st.handle)
    buf = ctypes.create_string_buffer(n)
    _check(load().spin_state_export(st.handle, ctypes.cast(buf, _vp), n, _stream(stream)), "spin_state_export")
    return buf.raw


def spin_state_import(st: SpinState, blob: bytes, stream=None) -> None:
    buf = ctypes.create_string_buffer(blob, len(blob))
    _check(load().spin_state_import(st.handle, ctypes.cast(buf, _vp), len(blob), _stream(stream)),
           "spin_state_import")


def spin_status_string(status: int) -> str:
    return load().spin_status_string(status).decode()
