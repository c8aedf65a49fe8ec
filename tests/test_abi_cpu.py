"""CPU-only checks of the C-ABI library: it builds for sm_100a, loads, exports
every entry point include/spin.h declares, and its host-only logic (state
sizing, argument validation, the per-layer budget allocator) behaves.  No
call here touches a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import indexer_sparse_attention_b200 as isa
from indexer_sparse_attention_b200 import build as isa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    isa_build.build()
    return isa.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "spin.h")).read()
    return sorted(set(re.findall(r"SPIN_API\s+[\w\s\*]+?\b(spin_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["spin_state_bytes", "spin_state_create", "spin_state_destroy", "spin_predict_select",
                     "spin_indexer_score", "spin_topk", "spin_ema_update", "spin_decode_step", "spin_get_error",
                     "spin_status_string", "spin_state_export", "spin_state_import", "spin_set_layer_sparsity"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(isa.LIB_PATH)
    for name in declared_functions():
        assert hasattr(so, name), name


def _cfg(**over):
    base = dict(num_layers=1, num_requests=96, max_slots=524288 + 64, block_size=64, num_heads=64, head_dim=128,
                topk=2048, max_rows=1, key_fp8=True, q_bf16=True, alpha=0.9, gamma=0.05, target_sparsity=0.5,
                seed=2)
    base.update(over)
    return isa.make_config(**base)


def _expected_bytes(L, Q, R, H, d, b, max_slots, pooling=0):
    a = lambda x: (x + 255) // 256 * 256
    mb = -(-max_slots // b)
    slot = mb * b
    blk = -(-mb // 16) * 16
    vg = slot // 32 if (b >= 32 and pooling == isa.SPIN_POOL_MAX) else 0  # V's 32-slot group maxima
    parts = [16, L * Q * slot * 4, L * Q * slot * 4, L * Q * vg * 4, Q * R * blk * 4, Q * blk * 4, Q * 4, Q * R * H * d,
             Q * R * H * 4, Q * R * slot * 4, Q * R * blk * max(1, b // 32) * 4, 8,
             # the selection a pipelined step prepares for the next one, per layer, and ctx_len + 1
             L * Q * blk * 4, L * Q * 4, L * Q * mb, L * Q * 4, Q * 4,
             Q * blk * 4, Q * 4, Q * 4,  # and the top-k's copy of the kept lists
             min(L, 8) * Q * R * blk * 4]  # block scores of the streams of spin_prepare_selections
    return sum(a(p) for p in parts)


@pytest.mark.parametrize("over", [{}, {"max_rows": 4, "num_requests": 32, "max_slots": 131072 + 128},
                                  {"num_layers": 8, "num_requests": 8, "max_slots": 1048576 + 64},
                                  {"key_fp8": False, "q_bf16": False, "num_heads": 8, "head_dim": 64,
                                   "num_requests": 1, "max_slots": 4096 + 32, "topk": 256},
                                  {"block_size": 16, "max_slots": 4096 + 16}, {"block_size": 32},
                                  {"pooling": 1}, {"pooling": 2, "block_size": 256}])
def test_state_bytes_matches_documented_layout(lib, over):
    cfg = _cfg(**over)
    got = isa.spin_state_bytes(cfg)
    exp = _expected_bytes(cfg.num_layers, cfg.num_requests, cfg.max_rows, cfg.num_heads, cfg.head_dim,
                          cfg.block_size, cfg.max_slots, cfg.pooling)
    assert got == exp


@pytest.mark.parametrize("over", [{"block_size": 48}, {"block_size": 8}, {"max_rows": 5}, {"max_rows": 0},
                                  {"target_sparsity": 1.0}, {"target_sparsity": -0.1}, {"gamma": 1.5},
                                  {"num_requests": 0}, {"key_fp8": False, "q_bf16": True}, {"pooling": 3},
                                  {"mtp_policy": 2}, {"mtp_policy": -1},
                                  {"max_slots": 64 * 50000}, {"alpha": float("nan")}])
def test_invalid_configs_rejected(lib, over):
    assert isa.spin_state_bytes(_cfg(**over)) == 0


def test_create_rejects_bad_arguments_without_a_device(lib):
    cfg = _cfg(num_requests=1, max_slots=4096)
    h = ctypes.c_void_p()
    st = lib.spin_state_create(ctypes.byref(cfg), ctypes.c_void_p(0), 1 << 30, ctypes.c_void_p(0), ctypes.byref(h))
    assert st == 1 and not h.value                      # SPIN_EINVAL: NULL device block
    st = lib.spin_state_create(ctypes.byref(cfg), ctypes.c_void_p(4096 + 8), 1 << 30, ctypes.c_void_p(0),
                               ctypes.byref(h))
    assert st == 1                                      # misaligned block
    st = lib.spin_state_create(ctypes.byref(cfg), ctypes.c_void_p(4096), 16, ctypes.c_void_p(0), ctypes.byref(h))
    assert st == 2                                      # SPIN_ENOMEM
    args = [None, 0, 1, 0, None, None, 1, None, 1, None, None, None, 0, None, None, None, None]
    assert lib.spin_decode_step(*args) == 4             # SPIN_ESTATE


def test_status_strings(lib):
    for code in range(8):
        assert isinstance(isa.spin_status_string(code), str) and isa.spin_status_string(code)


def test_layer_allocator_matches_oracle(lib, oracle_lib):
    rng = np.random.default_rng(0)
    for trial in range(20):
        L = int(rng.integers(1, 12))
        miss = rng.uniform(0, 0.4, L) * (rng.uniform(size=L) < 0.8)
        blocks = rng.integers(2000, 20000, L).astype(np.float64)
        lo = np.maximum(0.05, 32.0 / blocks)
        s_glob = float(rng.choice([0.0, 0.3, 0.5, 0.7, 0.95]))
        got = np.array(isa.spin_allocate_layer_sparsity(miss, blocks, lo, s_glob))
        ref = oracle_lib.layer_sparsity(miss, blocks, lo, s_glob)
        assert np.allclose(got, ref, atol=2e-6), (trial, got, ref)


def test_layer_allocator_rejects_bad_input(lib):
    with pytest.raises(isa.SpinError):
        isa.spin_allocate_layer_sparsity([0.1], [100.0], [0.05], 1.0)
    with pytest.raises(isa.SpinError):
        isa.spin_allocate_layer_sparsity([-0.1], [100.0], [0.05], 0.5)


def test_null_state_rejected_by_every_entry_point(lib):
    """Every call that takes a state answers SPIN_ESTATE for a NULL handle,
    before it touches the device (no GPU needed)."""
    isa.load()
    skip = {"spin_state_bytes", "spin_state_create", "spin_topk_noalloc", "spin_topk_noalloc_error",
            "spin_allocate_layer_sparsity",
            "spin_status_string", "spin_state_export_bytes", "spin_score_stride", "spin_mask_stride",
            "spin_state_destroy"}
    names = [n for n in isa.__all__ if n.startswith("spin_") and n not in skip]
    checked = 0
    for name in names:
        fn = getattr(lib, name, None)
        if fn is None or fn.restype is not ctypes.c_int or not fn.argtypes:
            continue
        ptr = lambda t: t in (ctypes.c_void_p, ctypes.c_char_p) or issubclass(t, ctypes._Pointer)
        args = [None] + [None if ptr(t) else 0 for t in fn.argtypes[1:]]
        assert fn(*args) == 4, name                      # SPIN_ESTATE
        checked += 1
    for name in ("spin_slot_prediction", "spin_pearson", "spin_topk_overlap", "spin_decode_step"):
        assert name in names
    assert checked >= 20
