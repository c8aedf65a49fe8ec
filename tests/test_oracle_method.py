"""Pins for the oracle's SPIN steps.  Each check comes from outside the oracle:
what the pages fix (the gamma share of exploration, skipped slots keep their
state, union of row masks, prefix-valid replay, all-keep at 0% sparsity),
closed forms, library routines (numpy reductions and sorts, torch fp64
matmul) and brute force on tiny inputs."""
import itertools
import json
import math
import os

from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_printed.json")


# ----------------------------------------------------------------------------
# predict + block max-pool
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("ctx_len,rows,b", [(1, 1, 4), (37, 1, 8), (64, 3, 8), (130, 4, 16), (5, 4, 4)])
def test_pool_without_diagonal_is_blockwise_max_of_V(oracle_lib, ctx_len, rows, b):
    rng = np.random.default_rng(ctx_len)
    n_stride = (ctx_len + rows + b) // b + 1
    V = rng.standard_normal(n_stride * b).astype(np.float32)
    D = np.full(n_stride * b, -np.inf, np.float32)
    S = oracle_lib.predict_pool(V, D, ctx_len, rows, b, n_stride)
    for r in range(rows):
        vis = ctx_len + r                     # slots 0..p_r
        n = -(-vis // b)
        padded = np.full(n * b, -np.inf, np.float32)
        padded[:vis] = V[:vis]
        ref = padded.reshape(n, b).max(axis=1)
        assert np.array_equal(S[r, :n], ref)
        assert np.all(np.isnan(S[r, n:]))


@pytest.mark.parametrize("delta0", [0, 1, 5, 17, 63])
def test_pool_diagonal_one_hot_lands_in_block_of_p_minus_delta(oracle_lib, delta0):
    b, ctx_len, rows = 8, 70, 4
    n_stride = 12
    V = np.full(n_stride * b, -np.inf, np.float32)
    D = np.full(n_stride * b, -np.inf, np.float32)
    D[delta0] = 1.0
    S = oracle_lib.predict_pool(V, D, ctx_len, rows, b, n_stride)
    for r in range(rows):
        p = ctx_len - 1 + r
        n = -(-(p + 1) // b)
        expect = np.full(n, -np.inf, np.float32)
        if p - delta0 >= 0:
            expect[(p - delta0) // b] = 1.0
        assert np.array_equal(S[r, :n], expect), (r, S[r, :n])


def test_pool_bounds_and_attains(oracle_lib):
    rng = np.random.default_rng(3)
    b, ctx_len, rows = 16, 203, 2
    n_stride = 16
    V = rng.standard_normal(n_stride * b).astype(np.float32)
    D = rng.standard_normal(n_stride * b).astype(np.float32)
    S = oracle_lib.predict_pool(V, D, ctx_len, rows, b, n_stride)
    for r in range(rows):
        p = ctx_len - 1 + r
        z = np.maximum(V[: p + 1], D[p - np.arange(p + 1)])
        for j in range(-(-(p + 1) // b)):
            blk = z[j * b: min((j + 1) * b, p + 1)]
            assert S[r, j] >= blk.max() and S[r, j] in blk


# ----------------------------------------------------------------------------
# budget, predicted top, exploration, union
# ----------------------------------------------------------------------------
def _select(oracle_lib, S, ctx_len, rows, b, s, g, seed=11, req=2, layer=1, step=5):
    return oracle_lib.select(S, ctx_len, rows, b, s, g, seed, req, layer, step)


@pytest.mark.parametrize("n,s,g", [(100, 0.5, 0.05), (8193, 0.5, 0.05), (8193, 0.4, 0.05), (65, 0.3, 0.05),
                                   (33, 0.5, 0.10), (7, 0.9, 0.5), (1, 0.5, 0.05), (50, 0.2, 0.0)])
def test_single_row_budget_and_gamma_share(oracle_lib, n, s, g):
    b = 64
    ctx_len = (n - 1) * b + 13
    rng = np.random.default_rng(n)
    S = rng.standard_normal((1, n)).astype(np.float32)
    mask = _select(oracle_lib, S, ctx_len, 1, b, s, g)
    B = n - math.floor(np.float64(np.float32(s)) * n)
    n_exp = math.floor(np.float64(np.float32(g)) * B)
    assert np.count_nonzero(mask) == B                  # |kept| = budget
    assert np.count_nonzero(mask == 2) == n_exp         # gamma share of the same budget
    assert np.count_nonzero(mask == 1) == B - n_exp


def test_zero_sparsity_is_all_keep(oracle_lib):
    S = np.random.default_rng(0).standard_normal((3, 20)).astype(np.float32)
    mask = _select(oracle_lib, S, 64 * 17 + 5, 3, 64, 0.0, 0.05)
    n_last = -(-(64 * 17 + 5 + 2) // 64)
    assert np.all(mask[:n_last] == 1) and np.all(mask[n_last:] == 0)


def _brute_force_predicted(S, n_pred):
    """All subsets of size n_pred; exactly one has every member ranked above
    every non-member by (higher score, then lower index)."""
    n = S.size
    found = []
    for sub in itertools.combinations(range(n), n_pred):
        inside = set(sub)
        ok = all((S[x] > S[y]) or (S[x] == S[y] and x < y)
                 for x in inside for y in range(n) if y not in inside)
        if ok:
            found.append(inside)
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("trial", range(12))
def test_predicted_set_brute_force_with_ties(oracle_lib, trial):
    rng = np.random.default_rng(100 + trial)
    n = int(rng.integers(3, 11))
    S = rng.integers(0, 4, n).astype(np.float32)           # many ties
    if trial % 3 == 0:
        S[rng.integers(0, n)] = np.inf                      # never-observed block
    b = 4
    ctx_len = (n - 1) * b + 1
    s = float(rng.choice([0.2, 0.3, 0.5, 0.7]))
    mask = _select(oracle_lib, S[None, :], ctx_len, 1, b, s, 0.0)
    B = n - math.floor(np.float64(np.float32(s)) * n)
    assert set(np.nonzero(mask == 1)[0]) == _brute_force_predicted(S, B)


def test_exploration_takes_smallest_philox_keys_among_candidates(oracle_lib):
    rng = np.random.default_rng(5)
    n, b, s, g = 500, 64, 0.5, 0.2
    S = rng.standard_normal((1, n)).astype(np.float32)
    seed, req, layer, step = 99, 3, 2, 41
    mask = oracle_lib.select(S, (n - 1) * b + 1, 1, b, s, g, seed, req, layer, step)
    cand = [j for j in range(n) if mask[j] != 1]
    keys = {j: oracle_lib.explore_key(seed, j, req, layer, step) for j in cand}
    explored = [j for j in cand if mask[j] == 2]
    rest = [j for j in cand if mask[j] == 0]
    assert max(keys[j] for j in explored) <= min(keys[j] for j in rest)


def test_exploration_is_uniform_over_candidates(oracle_lib):
    # Predicted blocks fixed by S; over many steps each remaining block must be
    # explored equally often (uniformly random unkept blocks).
    n, b, s, g = 40, 64, 0.5, 0.2
    S = np.arange(n, 0, -1, dtype=np.float32)[None, :]      # predicted = lowest indices
    counts = np.zeros(n)
    T = 3000
    for t in range(T):
        m = oracle_lib.select(S, (n - 1) * b + 1, 1, b, s, g, 7, 0, 0, t)
        counts += (m == 2)
    B = n - math.floor(np.float64(np.float32(s)) * n)
    n_exp = math.floor(np.float64(np.float32(g)) * B)
    n_pred = B - n_exp
    cand = counts[n_pred:]
    assert np.all(counts[:n_pred] == 0)
    expected = T * n_exp / (n - n_pred)
    chi2 = float(((cand - expected) ** 2 / expected).sum())
    assert chi2 < 3 * (n - n_pred), chi2                  # dof = 23


@pytest.mark.parametrize("ctx_len", [64 * 30 + 1, 64 * 30 + 62, 64 * 31])
def test_union_of_row_masks(oracle_lib, ctx_len):
    rng = np.random.default_rng(ctx_len)
    rows, b, s, g = 4, 64, 0.4, 0.05
    n_stride = 40
    S = rng.standard_normal((rows, n_stride)).astype(np.float32)
    mask = oracle_lib.select(S, ctx_len, rows, b, s, g, 1, 0, 0, 3)
    n0 = -(-ctx_len // b)
    B0 = n0 - math.floor(np.float64(np.float32(s)) * n0)
    n_exp = math.floor(np.float64(np.float32(g)) * B0)
    union = set()
    for r in range(rows):
        n = -(-(ctx_len + r) // b)
        Br = n - math.floor(np.float64(np.float32(s)) * n)
        order = np.lexsort((np.arange(n), -S[r, :n].astype(np.float64)))
        own = set(order[: Br - n_exp].tolist())
        assert own <= set(np.nonzero(mask == 1)[0])       # union is a superset of each row's mask
        union |= own
    assert union == set(np.nonzero(mask == 1)[0])
    n_last = -(-(ctx_len + rows - 1) // b)
    assert np.count_nonzero(mask == 2) == min(n_exp, n_last - len(union))
    assert np.all(mask[n_last:] == 0)


def test_union_realized_sparsity_not_above_target(oracle_lib):
    # The pages report realized sparsity below the 40% target under the row
    # union (thelatestinai listing, Table 7); the union can only add blocks.
    pages = json.load(open(GOLDEN))["table7_realized_sparsity"]
    assert pages["row_local_union_prefix_valid"] <= pages["target"]
    rng = np.random.default_rng(9)
    realized = []
    for t in range(50):
        ctx_len = int(rng.integers(2000, 4000))
        S = rng.standard_normal((4, 70)).astype(np.float32)
        mask = oracle_lib.select(S, ctx_len, 4, 64, pages["target"], 0.05, 1, 0, 0, t)
        n_last = -(-(ctx_len + 3) // 64)
        realized.append(1 - np.count_nonzero(mask[:n_last]) / n_last)
    assert max(realized) <= pages["target"] + 1e-12


# ----------------------------------------------------------------------------
# MTP baseline policy: row-0 sharing (SPIN listing, Table 7 and Figure 2)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("trial", range(10))
def test_row0_sharing_brute_force(oracle_lib, trial):
    # Row 0's own budget and predicted set (brute force over subsets), every
    # block past row 0's range kept, exploration = the n_exp smallest
    # (Philox key, block) among row 0's unkept blocks.
    rng = np.random.default_rng(300 + trial)
    b, rows = 4, int(rng.integers(2, 5))
    n0 = int(rng.integers(3, 10))
    ctx_len = (n0 - 1) * b + int(rng.integers(1, b + 1))
    n_last = -(-(ctx_len + rows - 1) // b)
    S = rng.integers(0, 4, (rows, n_last + 2)).astype(np.float32)
    s, g = float(rng.choice([0.3, 0.5, 0.7])), float(rng.choice([0.0, 0.25, 0.5]))
    seed, req, layer, step = 21, trial, 2, 8
    mask = oracle_lib.select(S, ctx_len, rows, b, s, g, seed, req, layer, step, oracle_lib.MTP_ROW0)
    B0 = n0 - math.floor(np.float64(np.float32(s)) * n0)
    n_exp = math.floor(np.float64(np.float32(g)) * B0)
    pred = _brute_force_predicted(S[0, :n0], B0 - n_exp) if B0 - n_exp > 0 else set()
    rest = sorted((oracle_lib.explore_key(seed, j, req, layer, step), j) for j in range(n0) if j not in pred)
    expect = np.zeros(S.shape[1], np.uint8)
    expect[list(pred)] = 1
    expect[n0:n_last] = 1
    for _, j in rest[:n_exp]:
        expect[j] = 2
    assert np.array_equal(mask, expect)


def test_row0_sharing_ignores_draft_rows_and_equals_union_for_one_row(oracle_lib):
    rng = np.random.default_rng(31)
    b, rows, ctx_len, s, g = 64, 4, 64 * 40 + 62, 0.5, 0.05
    S = rng.standard_normal((rows, 44)).astype(np.float32)
    m1 = oracle_lib.select(S, ctx_len, rows, b, s, g, 3, 1, 0, 9, oracle_lib.MTP_ROW0)
    S2 = S.copy()
    S2[1:] = rng.standard_normal((rows - 1, 44)).astype(np.float32)
    m2 = oracle_lib.select(S2, ctx_len, rows, b, s, g, 3, 1, 0, 9, oracle_lib.MTP_ROW0)
    assert np.array_equal(m1, m2)
    for pol in (oracle_lib.MTP_ROW0, oracle_lib.MTP_UNION_PREFIX):   # one row: the policies agree
        assert np.array_equal(oracle_lib.select(S[:1], ctx_len, 1, b, s, g, 3, 1, 0, 9, pol),
                              oracle_lib.select(S[:1], ctx_len, 1, b, s, g, 3, 1, 0, 9))
    z = oracle_lib.select(S, ctx_len, rows, b, 0.0, g, 3, 1, 0, 9, oracle_lib.MTP_ROW0)
    n_last = -(-(ctx_len + rows - 1) // b)
    assert np.all(z[:n_last] == 1) and np.all(z[n_last:] == 0)   # all-keep control


def test_row0_sharing_realized_sparsity_at_least_union(oracle_lib):
    # The pages print a higher realized sparsity for row-0 sharing than for
    # the row-local union at the same target (thelatestinai listing, Table 7).
    # With the drafts' new blocks unobserved (+inf block score), the union
    # holds row 0's predicted set and every new block, so it keeps at least as
    # many blocks; both stay at or under the target.
    pages = json.load(open(GOLDEN))["table7_realized_sparsity"]
    assert pages["row0_sharing_row0_update"] >= pages["row_local_union_prefix_valid"]
    rng = np.random.default_rng(33)
    for t in range(40):
        ctx_len = int(rng.integers(2000, 4000))
        n0, n_last = -(-ctx_len // 64), -(-(ctx_len + 3) // 64)
        S = rng.standard_normal((4, 70)).astype(np.float32)
        S[:, n0:n_last] = np.inf
        real = {}
        for pol in (oracle_lib.MTP_ROW0, oracle_lib.MTP_UNION_PREFIX):
            m = oracle_lib.select(S, ctx_len, 4, 64, pages["target"], 0.05, 1, 0, 0, t, pol)
            assert np.all(m[n0:n_last] != 0)
            real[pol] = 1 - np.count_nonzero(m[:n_last]) / n_last
            assert real[pol] <= pages["target"] + 1e-12
        assert real[oracle_lib.MTP_ROW0] >= real[oracle_lib.MTP_UNION_PREFIX]


def test_row0_update_uses_row0_scores_only(oracle_lib):
    # Row-0 update: whatever the accepted length, only row 0's scores move the
    # state.  From the never-observed sentinels the first observation is the
    # score itself, so V_s = I_{0,s} and D_{p0-s} = I_{0,s} on row 0's kept
    # slots, and nothing a draft row alone sees changes.
    rng = np.random.default_rng(34)
    b, n_stride, ctx_len, rows = 8, 12, 61, 4
    p0 = ctx_len - 1
    mask = (rng.uniform(size=n_stride) < 0.6).astype(np.uint8)
    mask[-(-(ctx_len + rows - 1) // b) - 1] = 1
    scores = rng.uniform(0, 3, (rows, n_stride * b)).astype(np.float32)
    assert oracle_lib.update_rows(oracle_lib.MTP_ROW0, 3) == 1
    assert oracle_lib.update_rows(oracle_lib.MTP_UNION_PREFIX, 3) == 3
    V, D = _state(n_stride * b, fill=(np.inf, -np.inf))
    oracle_lib.ema_update(V, D, scores, mask, ctx_len, oracle_lib.update_rows(oracle_lib.MTP_ROW0, 3), b, 0.9)
    kept = np.array([mask[s // b] != 0 for s in range(n_stride * b)])
    slots = np.arange(n_stride * b)
    seen = kept & (slots <= p0)
    assert np.array_equal(V[seen], scores[0, seen])
    assert np.all(np.isposinf(V[~seen]))
    assert np.array_equal(D[p0 - slots[seen]], scores[0, seen])
    d_seen = np.zeros(n_stride * b, bool)
    d_seen[p0 - slots[seen]] = True
    assert np.all(np.isneginf(D[~d_seen]))


# ----------------------------------------------------------------------------
# indexer scores
# ----------------------------------------------------------------------------
def _decode_table(oracle_lib):
    return np.array([oracle_lib.e4m3_decode(c) for c in range(256)])


def test_fp8_scores_vs_torch_matmul_through_permuted_block_table(oracle_lib):
    rng = np.random.default_rng(4)
    b, d, H, rows = 8, 32, 6, 3
    n_blocks, pages = 9, 14
    ctx_len = (n_blocks - 1) * b + 3
    keys8 = rng.integers(0, 256, (pages, b, d), dtype=np.uint8)
    keys8[(keys8 & 0x7F) == 0x7F] = 0x11                        # no NaN codes
    kscale = rng.uniform(0.01, 2.0, (pages, b)).astype(np.float32)
    bt = rng.permutation(pages)[:n_blocks].astype(np.int32)
    q8 = rng.integers(0, 256, (rows, H, d), dtype=np.uint8)
    q8[(q8 & 0x7F) == 0x7F] = 0x22
    wq = rng.uniform(-1, 1, (rows, H)).astype(np.float32)
    mask = np.zeros(n_blocks + 2, np.uint8)
    mask[[0, 2, 3, 8]] = [1, 2, 1, 1]
    slot_stride = (n_blocks + 2) * b
    got = oracle_lib.score_fp8(keys8, kscale, bt, q8, wq, ctx_len, mask, slot_stride)
    dec = _decode_table(oracle_lib)
    K = torch.from_numpy(dec[keys8[bt]].reshape(n_blocks * b, d) * kscale[bt].reshape(-1, 1))
    Qm = torch.from_numpy(dec[q8])                                # [rows,H,d]
    dots = torch.einsum("rhd,sd->rsh", Qm, K)
    ref = (torch.relu(dots) * torch.from_numpy(wq.astype(np.float64))[:, None, :]).sum(-1).numpy()
    for r in range(rows):
        p = ctx_len - 1 + r
        for s in range(slot_stride):
            scored = s <= p and s // b < n_blocks and mask[s // b] != 0
            if scored:
                assert abs(got[r, s] - ref[r, s]) <= 1e-12 * max(1.0, abs(ref[r, s])), (r, s)
            else:
                assert np.isnan(got[r, s])


def test_score_closed_form_relu_and_weights(oracle_lib):
    # One-dimensional structure: k_s = c_s e_0, q_h = a_h e_0, so
    # I_s = sum_h w_h max(0, a_h c_s) in closed form (ReLU clips negatives).
    b, d, H = 4, 16, 5
    c = np.array([1.0, -2.0, 0.5, 3.0, -0.25, 2.0, 1.5, -1.0])
    keys = np.zeros((2, b, d), np.float32)
    keys.reshape(-1, d)[:, 0] = c
    a = np.array([1.0, -1.0, 2.0, 0.0, -3.0])
    w = np.array([[0.5, 2.0, 0.25, 7.0, 1.0]], np.float32)
    q = np.zeros((1, H, d), np.float32)
    q[0, :, 0] = a
    mask = np.array([1, 1], np.uint8)
    got = oracle_lib.score_f32(keys, np.array([0, 1], np.int32), q, w, 8, mask, 8)
    ref = [sum(w[0, h] * max(0.0, a[h] * cs) for h in range(H)) for cs in c]
    assert np.allclose(got[0], ref, rtol=0, atol=1e-12)


def test_score_fp8_power_of_two_query_scale_folds_into_weight(oracle_lib):
    # ReLU(c x) = c ReLU(x) for c > 0: scaling a head's query by 2^m and its
    # weight by 2^-m leaves the score unchanged (the reason the query scale
    # can live in the head weight).
    rng = np.random.default_rng(8)
    b, d, H = 4, 64, 4
    q = rng.standard_normal((1, H, d))
    w = rng.uniform(0, 1, (1, H)).astype(np.float32)
    keys8 = rng.integers(0, 0x70, (3, b, d), dtype=np.uint8)
    ks = np.ones((3, b), np.float32)
    bt = np.arange(3, dtype=np.int32)
    mask = np.ones(3, np.uint8)
    q8a, wqa, _ = oracle_lib.quantize_q(q, w)
    q8b, wqb, eb = oracle_lib.quantize_q(q * 2.0 ** 7, w)
    assert np.array_equal(q8a, q8b)
    sa = oracle_lib.score_fp8(keys8, ks, bt, q8a, wqa, 12, mask, 12)
    sb = oracle_lib.score_fp8(keys8, ks, bt, q8b, (wqb * 2.0 ** -7).astype(np.float32), 12, mask, 12)
    assert np.array_equal(sa, sb)


# ----------------------------------------------------------------------------
# token top-k
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("trial", range(10))
def test_topk_vs_lexsort_with_ties_and_padding(oracle_lib, trial):
    rng = np.random.default_rng(200 + trial)
    b = 4
    n = int(rng.integers(1, 12))
    ctx_len = int(rng.integers((n - 1) * b + 1, n * b + 1))
    row = int(rng.integers(0, 2))
    n_stride = n + 1
    scores = rng.integers(0, 5, n_stride * b).astype(np.float64)
    mask = (rng.uniform(size=n_stride) < 0.6).astype(np.uint8)
    k = int(rng.integers(1, 20))
    got = oracle_lib.topk_row(scores, mask, ctx_len, row, b, k)
    p = ctx_len - 1 + row
    cand = np.array([s for s in range(p + 1) if mask[s // b]], np.int64)
    if cand.size:
        order = np.lexsort((cand, -scores[cand]))             # by score desc, then slot asc
        chosen = np.sort(cand[order[:k]])
    else:
        chosen = np.array([], np.int64)
    ref = np.full(k, -1, np.int64)
    ref[: chosen.size] = chosen
    assert np.array_equal(got, ref)


def test_topk_at_zero_sparsity_is_full_topk(oracle_lib):
    rng = np.random.default_rng(6)
    b, n, k = 64, 50, 256
    ctx_len = n * b - 7
    S = rng.standard_normal((1, n + 1)).astype(np.float32)
    mask = oracle_lib.select(S, ctx_len, 1, b, 0.0, 0.05, 0, 0, 0, 0)
    scores = rng.standard_normal((n + 1) * b)
    got = oracle_lib.topk_row(scores, mask, ctx_len, 0, b, k)
    full = torch.topk(torch.from_numpy(scores[:ctx_len]), k).indices.numpy()
    assert np.array_equal(got, np.sort(full))


# ----------------------------------------------------------------------------
# EMA update
# ----------------------------------------------------------------------------
def _state(n_slots, rng=None, fill=None):
    if fill is not None:
        return np.full(n_slots, fill[0], np.float32), np.full(n_slots, fill[1], np.float32)
    return (rng.uniform(0, 10, n_slots).astype(np.float32),
            rng.uniform(0, 10, n_slots).astype(np.float32))


def test_ema_skipped_slots_unchanged_and_first_observation_replaces_sentinel(oracle_lib):
    rng = np.random.default_rng(10)
    b, n_stride, ctx_len = 8, 10, 75
    V, D = _state(n_stride * b, fill=(np.inf, -np.inf))
    V[:40] = rng.uniform(0, 5, 40)
    V0, D0 = V.copy(), D.copy()
    mask = np.zeros(n_stride, np.uint8)
    mask[[1, 4, 9]] = [1, 2, 1]
    scores = rng.uniform(0, 3, (1, n_stride * b)).astype(np.float32)
    oracle_lib.ema_update(V, D, scores, mask, ctx_len, 1, b, 0.9)
    p = ctx_len - 1
    scored = [s for s in range(p + 1) if mask[s // b]]
    unscored = [s for s in range(n_stride * b) if s not in scored]
    assert np.array_equal(V[unscored].view(np.uint32), V0[unscored].view(np.uint32))
    touched_d = {p - s for s in scored}
    untouched_d = [x for x in range(n_stride * b) if x not in touched_d]
    assert np.array_equal(D[untouched_d].view(np.uint32), D0[untouched_d].view(np.uint32))
    for s in scored:
        if np.isinf(V0[s]):
            assert V[s] == scores[0, s]
        assert D[p - s] == scores[0, s]                       # D started at the -inf sentinel


def test_ema_alpha_zero_is_previous_iteration_predictor(oracle_lib):
    # alpha = 0 turns the vertical state into the last observed score: the
    # "Prev-iter" predictor of the thelatestinai listing, Table 1.
    rng = np.random.default_rng(11)
    b, n_stride, ctx_len = 4, 6, 22
    V, D = _state(n_stride * b, rng)
    mask = np.ones(n_stride, np.uint8)
    scores = rng.uniform(0, 3, (1, n_stride * b)).astype(np.float32)
    oracle_lib.ema_update(V, D, scores, mask, ctx_len, 1, b, 0.0)
    assert np.array_equal(V[:ctx_len], scores[0, :ctx_len])


@pytest.mark.parametrize("alpha", [0.9, 0.5, 0.99])
def test_ema_constant_input_closed_form(oracle_lib, alpha):
    # x_n = alpha^n x_0 + (1 - alpha^n) y for a constant observation y.
    b, n_stride, ctx_len = 4, 2, 8
    V, D = _state(n_stride * b, fill=(5.0, 5.0))
    y = np.full((1, n_stride * b), 1.25, np.float32)
    mask = np.ones(n_stride, np.uint8)
    steps = 40
    for _ in range(steps):
        oracle_lib.ema_update(V, D, y, mask, ctx_len, 1, b, alpha)
    a32 = float(np.float32(alpha))
    expect = a32 ** steps * 5.0 + (1 - a32 ** steps) * 1.25
    assert np.allclose(V[:ctx_len], expect, rtol=steps * 2e-7, atol=0)
    assert np.allclose(D[:ctx_len], expect, rtol=steps * 2e-7, atol=0)


@pytest.mark.parametrize("accepted", [1, 2, 3, 4])
def test_prefix_valid_replay_equals_sequential_rows(oracle_lib, accepted):
    # Replaying the accepted rows at once equals applying them one at a time,
    # each as a single-row update at its own position.
    rng = np.random.default_rng(12 + accepted)
    b, n_stride, ctx_len, rows = 8, 12, 61, 4
    V, D = _state(n_stride * b, rng)
    V[rng.integers(0, 96, 10)] = np.inf
    D[rng.integers(0, 96, 10)] = -np.inf
    mask = (rng.uniform(size=n_stride) < 0.5).astype(np.uint8)
    scores = rng.uniform(0, 3, (rows, n_stride * b)).astype(np.float32)
    Va, Da = V.copy(), D.copy()
    oracle_lib.ema_update(Va, Da, scores, mask, ctx_len, accepted, b, 0.9)
    Vb, Db = V.copy(), D.copy()
    for r in range(accepted):
        oracle_lib.ema_update(Vb, Db, scores[r:r + 1], mask, ctx_len + r, 1, b, 0.9)
    assert np.array_equal(Va.view(np.uint32), Vb.view(np.uint32))
    assert np.array_equal(Da.view(np.uint32), Db.view(np.uint32))


def test_ema_rejected_draft_slots_keep_sentinel(oracle_lib):
    b, n_stride, ctx_len, rows = 8, 6, 30, 4
    V, D = _state(n_stride * b, fill=(np.inf, -np.inf))
    mask = np.ones(n_stride, np.uint8)
    scores = np.ones((rows, n_stride * b), np.float32)
    oracle_lib.ema_update(V, D, scores, mask, ctx_len, 2, b, 0.9)
    p_last_valid = ctx_len - 1 + 1
    assert np.all(np.isfinite(V[: p_last_valid + 1]))
    assert np.all(np.isposinf(V[p_last_valid + 1:]))


# ----------------------------------------------------------------------------
# per-layer budget and miss metric
# ----------------------------------------------------------------------------
def test_layer_sparsity_meets_global_budget_and_is_proportional(oracle_lib):
    miss = np.array([0.02, 0.10, 0.30, 0.05, 0.0, 0.2, 0.15, 0.01])
    N = np.array([4000, 8000, 12000, 16000, 4096, 9000, 7000, 5000], np.float64)
    lo = np.full(8, 0.05)
    s = oracle_lib.layer_sparsity(miss, N, lo, 0.5)
    f = 1 - s
    assert abs((f * N).sum() - 0.5 * N.sum()) <= 1e-9 * N.sum()
    assert np.all(f >= lo - 1e-15) and np.all(f <= 1 + 1e-15)
    free = (f > lo + 1e-12) & (f < 1 - 1e-12)
    ratio = f[free] / (miss[free] + 1e-3)
    assert np.allclose(ratio, ratio[0], rtol=1e-9)
    assert np.all(np.diff(f[np.argsort(miss)]) >= -1e-15)   # more misses -> more kept


def test_layer_sparsity_infeasible_floor_and_all_keep(oracle_lib):
    N = np.array([10.0, 10.0])
    s = oracle_lib.layer_sparsity(np.array([0.1, 0.2]), N, np.array([0.6, 0.7]), 0.5)
    assert np.allclose(1 - s, [0.6, 0.7])
    s0 = oracle_lib.layer_sparsity(np.array([0.1, 0.2]), N, np.array([0.05, 0.05]), 0.0)
    assert np.allclose(s0, 0.0)


def test_random_predictor_recall_matches_table1(oracle_lib):
    # A predictor that keeps k random tokens recalls k / L of the true top-k in
    # expectation.  With block size 1 the miss metric is 1 - recall; the pages
    # print 0.022 for the random baseline at 94k context (thelatestinai
    # listing, Table 1, AA-LCR columns).
    pages = json.load(open(GOLDEN))["table1_random_recall"]
    L, k = pages["aa_lcr"]["context_tokens"], pages["k_reading"]
    rng = np.random.default_rng(13)
    recalls = []
    for _ in range(200):
        full = np.sort(rng.choice(L, k, replace=False)).astype(np.int32)
        keep = np.zeros(L, np.uint8)
        keep[rng.choice(L, k, replace=False)] = 1
        recalls.append(1 - oracle_lib.miss_fraction(full, keep, 1))
    assert round(float(np.mean(recalls)), 3) == pages["aa_lcr"]["recall"]


def test_p99_nearest_rank(oracle_lib):
    assert oracle_lib.p99(np.arange(1, 101)) == 99
    assert oracle_lib.p99(np.arange(1, 1001)) == 990
    assert oracle_lib.p99([3.0]) == 3.0


# --------------------------------------------------------------------------
# Block-reduction variants (SPIN listing, Figure 3: Mean and Top-4 against
# Max pooling; the pages define neither, the oracle takes the plain readings)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("b", [16, 64, 256])
def test_pool_mean_and_top4_on_exact_integers(oracle_lib, b):
    """Integer-valued z: every partial sum is exact, so the mean and the top-4
    mean must equal the brute-force values whatever the summation order."""
    rng = np.random.default_rng(b)
    n_slots = 5 * b + 7                                   # a ragged last block
    V = rng.integers(0, 1000, n_slots + 8).astype(np.float32)
    D = np.where(rng.random(n_slots + 8) < 0.5, -np.inf, rng.integers(0, 1000, n_slots + 8)).astype(np.float32)
    ctx = n_slots
    for rows in (1, 3):
        S_mean = oracle_lib.predict_pool(V, D, ctx, rows, b, 8, oracle_lib.POOL_MEAN)
        S_top4 = oracle_lib.predict_pool(V, D, ctx, rows, b, 8, oracle_lib.POOL_TOP4)
        S_max = oracle_lib.predict_pool(V, D, ctx, rows, b, 8, oracle_lib.POOL_MAX)
        for r in range(rows):
            p = ctx - 1 + r
            for j in range(oracle_lib.num_blocks(ctx, r, b)):
                i = np.arange(j * b, min((j + 1) * b, p + 1))
                z = np.maximum(V[i], D[p - i]).astype(np.float64)
                assert S_mean[r, j] == np.float32(z.mean())
                top = np.sort(z)[::-1][:4]
                assert S_top4[r, j] == np.float32(top.mean())
                assert S_max[r, j] == np.float32(z.max())


def test_pool_variants_order_and_sentinels(oracle_lib):
    """Mean <= Top-4 <= Max on real-valued z; a never-observed slot (V = +inf)
    makes every variant +inf; a block with fewer than 4 visible slots averages
    them all."""
    rng = np.random.default_rng(3)
    n = 64 * 40 + 3
    V = rng.standard_normal(n + 4).astype(np.float32) * 10
    D = rng.standard_normal(n + 4).astype(np.float32) * 10
    V[64 * 7 + 5] = np.inf
    S = {m: oracle_lib.predict_pool(V, D, n, 1, 64, 48, m)[0] for m in (0, 1, 2)}
    nb = oracle_lib.num_blocks(n, 0, 64)
    assert np.all(S[1][:nb] <= S[2][:nb]) and np.all(S[2][:nb] <= S[0][:nb])
    assert all(np.isinf(S[m][7]) for m in (0, 1, 2))
    # the last block holds 3 visible slots
    p = n - 1
    i = np.arange(64 * (nb - 1), n)
    z = np.maximum(V[i], D[p - i]).astype(np.float64)
    assert len(i) == 3 and S[2][nb - 1] == _exact_mean(z)


def _f32_nearest(fr):
    """A rational rounded to the nearest float32, ties to even, by integer
    arithmetic on the exact value (no float operation rounds on the way)."""
    if fr == 0:
        return np.float32(0.0)
    sign = -1.0 if fr < 0 else 1.0
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()   # 2^e <= a < 2^(e+2)
    if a < Fraction(2) ** e:
        e -= 1
    while a >= Fraction(2) ** (e + 1):
        e += 1
    ulp_exp = max(e, -126) - 23                                   # spacing of floats at a
    n = a / Fraction(2) ** ulp_exp
    k = n.numerator // n.denominator
    rest = n - k
    if rest > Fraction(1, 2) or (rest == Fraction(1, 2) and k % 2 == 1):
        k += 1
    return np.float32(sign * float(k) * 2.0 ** ulp_exp)        # exact: k <= 2^24


def _exact_mean(z):
    z = [float(np.float32(v)) for v in z]
    return _f32_nearest(sum((Fraction(v) for v in z), Fraction(0)) / len(z))


def test_f32_nearest_reference_on_known_values():
    # the reference rounding itself, on values whose float is known
    assert _f32_nearest(Fraction(1, 3)) == np.float32(1.0 / 3.0)
    mid = Fraction(1) + Fraction(1, 2 ** 24)                    # halfway between 1 and 1 + 2^-23
    assert _f32_nearest(mid) == np.float32(1.0)                 # ties to even
    assert _f32_nearest(mid + Fraction(1, 2 ** 60)) == np.nextafter(np.float32(1), np.float32(2))
    assert _f32_nearest(Fraction(3, 2 ** 150)) == np.float32(2.0 ** -148)   # 1.5 units -> 2 (even)
    assert _f32_nearest(Fraction(1, 2 ** 150)) == np.float32(0.0)          # half a unit -> 0 (even)


def test_mean_exact_against_rational_arithmetic(oracle_lib):
    """The pools' mean is the exact sum over the count rounded once: checked
    against exact rational arithmetic on values spanning the float range
    (2^-149 .. 2^120, mixed signs, up to 256 values), where any fixed double
    summation order would lose bits."""
    rng = np.random.default_rng(77)
    for trial in range(400):
        n = int(rng.integers(1, 257))
        kind = trial % 4
        if kind == 0:    # one exponent band: a sum in double would be exact
            z = rng.uniform(0, 50, n)
        elif kind == 1:  # wide spread, both signs
            z = rng.standard_normal(n) * 2.0 ** rng.integers(-140, 120, n)
        elif kind == 2:  # subnormals and tiny values
            z = rng.integers(-2 ** 20, 2 ** 20, n) * 2.0 ** -149
        else:            # large values that cancel, plus small ones
            z = np.concatenate([[2.0 ** 100, -(2.0 ** 100)], rng.uniform(-1, 1, n - 2)]) if n > 2 else [1.0] * n
        z = np.asarray(z, np.float32)
        got = oracle_lib.mean_exact(z)
        ref = _exact_mean(z)
        assert got.view(np.uint32) == ref.view(np.uint32), (trial, got, ref)
        perm = rng.permutation(z.size)
        assert oracle_lib.mean_exact(z[perm]).view(np.uint32) == got.view(np.uint32)   # no order enters


def test_pool_mean_and_top4_exact_on_wide_values(oracle_lib):
    """The block Mean and Top-4 on z spanning 2^60 equal the exact rational
    values: with z = (2^60, 1, -2^60, 1, 0, ...) over 16 slots the mean is
    2/16 exactly (a left-to-right double sum would absorb the first 1)."""
    b = 16
    D = np.full(b, -np.inf, np.float32)
    V = np.zeros(b, np.float32)
    V[0], V[1], V[8], V[9] = 2.0 ** 60, 1.0, -(2.0 ** 60), 1.0
    assert oracle_lib.predict_pool(V, D, b, 1, b, 1, oracle_lib.POOL_MEAN)[0, 0] == np.float32(2.0 / 16)
    # top-4 of the same block: 2^60, 1, 1, 0 -> (2^60 + 2) / 4 rounds to 2^58
    assert oracle_lib.predict_pool(V, D, b, 1, b, 1, oracle_lib.POOL_TOP4)[0, 0] == np.float32(2.0 ** 58)
    rng = np.random.default_rng(9)
    n = 64 * 9 + 5
    V = (rng.standard_normal(n + 4) * 2.0 ** rng.integers(-60, 60, n + 4)).astype(np.float32)
    D = (rng.standard_normal(n + 4) * 2.0 ** rng.integers(-60, 60, n + 4)).astype(np.float32)
    for rows in (1, 3):
        Sm = oracle_lib.predict_pool(V, D, n, rows, 64, 16, oracle_lib.POOL_MEAN)
        St = oracle_lib.predict_pool(V, D, n, rows, 64, 16, oracle_lib.POOL_TOP4)
        for r in range(rows):
            p = n - 1 + r
            for j in range(oracle_lib.num_blocks(n, r, 64)):
                i = np.arange(j * 64, min((j + 1) * 64, p + 1))
                z = np.maximum(V[i], D[p - i])
                assert Sm[r, j].view(np.uint32) == _exact_mean(z).view(np.uint32), (r, j)
                assert St[r, j].view(np.uint32) == _exact_mean(np.sort(z)[::-1][:4]).view(np.uint32), (r, j)


# ----------------------------------------------------------------------------
# predictor quality (SPIN listing, Table 1)
# ----------------------------------------------------------------------------
def test_pearson_matches_numpy_corrcoef_on_finite_pairs(oracle_lib):
    rng = np.random.default_rng(40)
    x = rng.standard_normal(5000).astype(np.float32)
    y = (0.3 * x + rng.standard_normal(5000)).astype(np.float32)
    x[rng.integers(0, 5000, 40)] = -np.inf
    y[rng.integers(0, 5000, 40)] = np.nan
    ok = np.isfinite(x) & np.isfinite(y)
    ref = np.corrcoef(x[ok].astype(np.float64), y[ok].astype(np.float64))[0, 1]
    assert abs(oracle_lib.pearson(x, y) - ref) < 1e-12


def test_pearson_affine_constant_and_short(oracle_lib):
    x = np.arange(100, dtype=np.float32)
    assert abs(oracle_lib.pearson(x, 3 * x + 1) - 1.0) < 1e-12
    assert abs(oracle_lib.pearson(x, -0.5 * x + 7) + 1.0) < 1e-12
    assert oracle_lib.pearson(x, np.full(100, 2.0, np.float32)) == 0.0
    one = np.full(100, -np.inf, np.float32)
    one[5] = 1.0
    assert oracle_lib.pearson(one, x) == 0.0                  # a single finite pair


@pytest.mark.parametrize("ctx_len,rows,b", [(37, 1, 8), (130, 4, 16), (64 * 9 + 1, 3, 64)])
def test_slot_prediction_pools_to_block_scores(oracle_lib, ctx_len, rows, b):
    # The block max-pool of the slot prediction is the predicted block score
    # (pinned above against V's blockwise maximum and the diagonal one-hot);
    # a slot no step has scored has no prediction.
    rng = np.random.default_rng(ctx_len)
    n_stride = -(-(ctx_len + rows) // b) + 1
    V = rng.standard_normal(n_stride * b).astype(np.float32)
    D = rng.standard_normal(n_stride * b).astype(np.float32)
    D[rng.random(D.size) < 0.3] = -np.inf
    V[ctx_len - 1] = np.inf                                   # the newest slot: never scored
    z = oracle_lib.slot_prediction(V, D, ctx_len, rows, n_stride * b)
    S = oracle_lib.predict_pool(V, D, ctx_len, rows, b, n_stride)
    for r in range(rows):
        p = ctx_len - 1 + r
        assert z[r, ctx_len - 1] == -np.inf
        assert np.all(np.isfinite(np.delete(z[r, : p + 1], ctx_len - 1)))   # V finite elsewhere
        for j in range(-(-(p + 1) // b)):
            blk = z[r, j * b: min((j + 1) * b, p + 1)]
            if ctx_len - 1 in range(j * b, min((j + 1) * b, p + 1)):
                assert S[r, j] == np.inf                      # the sentinel keeps the block
            else:
                assert S[r, j] == blk.max()


def test_random_prediction_uniform_uncorrelated_and_table1_recall(oracle_lib):
    # The random baseline of Table 1 (thelatestinai listing): correlation 0 and
    # top-k recall k / L in expectation; the pages print 0.022 at AA-LCR's 94k.
    pages = json.load(open(GOLDEN))["table1_random_recall"]
    L, k = pages["aa_lcr"]["context_tokens"], pages["k_reading"]
    assert round(k / L, 3) == pages["aa_lcr"]["recall"]
    rng = np.random.default_rng(41)
    scores = rng.standard_normal(L).astype(np.float32)
    true_top = set(oracle_lib.topk_visible(scores, L, 0, k).tolist())
    recalls, corr = [], []
    for step in range(60):
        u = oracle_lib.random_prediction(5, 1, 2, step, L, 1, L)[0]
        assert np.all((u >= 0) & (u < 1))
        corr.append(oracle_lib.pearson(u, scores))
        recalls.append(len(true_top & set(oracle_lib.topk_visible(u, L, 0, k).tolist())) / k)
    sigma = math.sqrt(k * (1 - k / L) * (1 - k / L)) / k / math.sqrt(len(recalls))
    assert abs(np.mean(recalls) - k / L) < 4 * sigma
    assert abs(np.mean(corr)) < 4 / math.sqrt(L * len(corr))
    hist = np.histogram(oracle_lib.random_prediction(5, 1, 2, 0, L, 1, L)[0], bins=50, range=(0, 1))[0]
    e = L / 50
    assert float(((hist - e) ** 2 / e).sum()) < 3 * 49       # chi-square, 49 dof
