"""Predictor-quality profile on the GPU (SPIN listing, Table 1), through the
C ABI, against the oracle: slot predictions bit for bit, Pearson correlation
within 1e-9 of the oracle's double two-pass value, top-k lists and their
overlaps exactly."""
import numpy as np
import pytest
import torch

import indexer_sparse_attention_b200 as isa
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from indexer_sparse_attention_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def make_state(Q, max_slots, R, k=256, b=64, seed=7):
    cfg = isa.make_config(num_layers=2, num_requests=Q, max_slots=max_slots, block_size=b, topk=k, max_rows=R,
                          gamma=0.05, target_sparsity=0.5, seed=seed)
    return isa.SpinState(cfg)


@pytest.mark.parametrize("R", [1, 3])
def test_slot_predictions_bit_exact(R):
    rng = np.random.default_rng(R)
    max_slots = 64 * 300 + 64
    st = make_state(Q=3, max_slots=max_slots, R=R)
    V, D = st.ema(1)
    v = (rng.standard_normal(V.shape) * 5).astype(np.float32)
    v[rng.random(V.shape) < 0.05] = np.inf                   # never-scored slots
    V.copy_(torch.from_numpy(v))
    d = (rng.standard_normal(D.shape) * 5).astype(np.float32)
    d[rng.random(D.shape) < 0.3] = -np.inf
    D.copy_(torch.from_numpy(d))
    st.refresh()  # V and D were written through the views
    ctx = np.array([1, 64 * 137 + 29, max_slots - R + 1], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    stride = st.score_stride
    for kind in (isa.SPIN_PRED_EMA, isa.SPIN_PRED_RANDOM):
        pred = st.new_scores()
        pred.fill_(float("nan"))
        isa.spin_slot_prediction(st, 1, R, kind, 12, ctx_t, pred)
        assert isa.spin_get_error(st)[0] == 0
        got = pred.cpu().numpy()
        for q in range(3):
            if kind == isa.SPIN_PRED_EMA:
                ref = oracle.slot_prediction(V[q].cpu().numpy(), D[q].cpu().numpy(), int(ctx[q]), R, stride)
            else:
                ref = oracle.random_prediction(7, q, 1, 12, int(ctx[q]), R, stride)
            for r in range(R):
                p = int(ctx[q]) + r
                assert np.array_equal(got[q, r, :p].view(np.uint32), ref[r, :p].view(np.uint32)), (kind, q, r)


def test_pearson_matches_oracle():
    rng = np.random.default_rng(5)
    R, max_slots = 2, 300_000
    st = make_state(Q=4, max_slots=max_slots, R=R)
    ctx = np.array([1, 2, 123_457, max_slots - 1], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    x = st.new_scores()
    y = st.new_scores()
    xs = (rng.standard_normal(x.shape) * 3 + 1).astype(np.float32)
    ys = (0.6 * xs + rng.standard_normal(y.shape)).astype(np.float32)
    xs[rng.random(xs.shape) < 0.01] = -np.inf
    ys[rng.random(ys.shape) < 0.01] = np.nan
    ys[2, 1] = 4.0                                            # constant row -> 0
    x.copy_(torch.from_numpy(xs))
    y.copy_(torch.from_numpy(ys))
    out = torch.zeros((4, R), dtype=torch.float64, device="cuda")
    isa.spin_pearson(st, R, x, y, ctx_t, out)
    assert isa.spin_get_error(st)[0] == 0
    got = out.cpu().numpy()
    for q in range(4):
        for r in range(R):
            n = int(ctx[q]) + r
            ref = oracle.pearson(xs[q, r, :n], ys[q, r, :n])
            assert abs(got[q, r] - ref) <= 1e-9, (q, r, got[q, r], ref)
    assert got[2, 1] == 0.0
    isa.spin_pearson(st, R, x, x, ctx_t, out)                 # a series with itself
    got = out.cpu().numpy()
    assert np.all(np.abs(got[2:] - 1.0) < 1e-12)


def test_topk_overlap_matches_set_intersection():
    rng = np.random.default_rng(6)
    Q, R, k = 5, 2, 256
    st = make_state(Q=Q, max_slots=70_000, R=R, k=k)
    a = np.full((Q, R, k), -1, np.int32)
    b = np.full((Q, R, k), -1, np.int32)
    for q in range(Q):
        for r in range(R):
            na, nb = (k, k) if q < 3 else (int(rng.integers(0, k)), int(rng.integers(0, k)))
            a[q, r, :na] = np.sort(rng.choice(1000, na, replace=False))
            b[q, r, :nb] = np.sort(rng.choice(1000, nb, replace=False))
    a[0, 0] = b[0, 0]                                         # identical lists
    out = torch.zeros((Q, R), dtype=torch.int32, device="cuda")
    isa.spin_topk_overlap(st, R, torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), out)
    got = out.cpu().numpy()
    for q in range(Q):
        for r in range(R):
            ref = len(set(a[q, r][a[q, r] >= 0].tolist()) & set(b[q, r][b[q, r] >= 0].tolist()))
            assert got[q, r] == ref, (q, r)
    assert got[0, 0] == k


def test_predictor_topk_and_recall_end_to_end():
    """The recall pipeline a profile runs: predictions, the top-k of each with
    every block kept (-inf predictions rank last), the overlap with the top-k
    of the indexer scores.  Top-k lists equal the oracle's over the visible
    slots, and so do the recalls."""
    rng = np.random.default_rng(8)
    R, k, max_slots = 2, 512, 64 * 800 + 64
    st = make_state(Q=2, max_slots=max_slots, R=R, k=k)
    V, D = st.ema(0)
    v = rng.standard_normal(V.shape).astype(np.float32)
    v[:, 40_000:] = np.inf
    V.copy_(torch.from_numpy(v))
    D.copy_(torch.from_numpy(rng.standard_normal(D.shape).astype(np.float32)))
    st.refresh()  # V and D were written through the views
    ctx = np.array([64 * 700 + 5, 30_001], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    scores = st.new_scores()
    sc = rng.standard_normal(scores.shape).astype(np.float32)
    scores.copy_(torch.from_numpy(sc))
    allk = torch.ones_like(st.new_mask())
    true_top = torch.empty((2, R, k), dtype=torch.int32, device="cuda")
    isa.spin_topk(st, R, scores, allk, ctx_t, true_top)
    pred = st.new_scores()
    isa.spin_slot_prediction(st, 0, R, isa.SPIN_PRED_EMA, 0, ctx_t, pred)
    pred_top = torch.empty_like(true_top)
    isa.spin_topk(st, R, pred, allk, ctx_t, pred_top)
    ov = torch.zeros((2, R), dtype=torch.int32, device="cuda")
    isa.spin_topk_overlap(st, R, pred_top, true_top, ov)
    assert isa.spin_get_error(st)[0] == 0
    for q in range(2):
        z = oracle.slot_prediction(V[q].cpu().numpy(), D[q].cpu().numpy(), int(ctx[q]), R, st.score_stride)
        for r in range(R):
            t_ref = oracle.topk_visible(sc[q, r], int(ctx[q]), r, k)
            p_ref = oracle.topk_visible(z[r], int(ctx[q]), r, k)
            assert np.array_equal(true_top[q, r].cpu().numpy(), t_ref), (q, r)
            assert np.array_equal(pred_top[q, r].cpu().numpy(), p_ref), (q, r)
            assert ov[q, r].item() == len(set(t_ref.tolist()) & set(p_ref.tolist()))
