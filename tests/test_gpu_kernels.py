"""Kernel-level parity on the GPU, through the C ABI, against the oracle.

Every case uses seeded synthetic inputs at sizes the oracle finishes in
seconds that still span several tiles and a ragged tail.  Integer and
selection results must match bit for bit; scores within
|gpu - ref| <= 1e-4 + 1e-3 |ref| of the fp64 oracle."""
import numpy as np
import pytest
import torch

import indexer_sparse_attention_b200 as isa
import oracle
import workloads
from lockstep import pool_close, score_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from indexer_sparse_attention_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def make_state(Q=3, max_slots=8192 + 64, R=1, H=64, d=128, k=256, fp8=True, s=0.5, g=0.05, seed=7, layers=1, b=64,
               mtp_policy=isa.SPIN_MTP_UNION_PREFIX):
    cfg = isa.make_config(num_layers=layers, num_requests=Q, max_slots=max_slots, block_size=b, num_heads=H,
                          head_dim=d, topk=k, max_rows=R, key_fp8=fp8, q_bf16=fp8, alpha=0.9, gamma=g,
                          target_sparsity=s, seed=seed, mtp_policy=mtp_policy)
    return isa.SpinState(cfg)


def random_state(st, layer, rng, frac_sentinel=0.1):
    V, D = st.ema(layer)
    v = rng.uniform(0, 50, V.shape).astype(np.float32)
    dd = rng.uniform(0, 50, D.shape).astype(np.float32)
    v[rng.uniform(size=v.shape) < frac_sentinel] = np.inf
    dd[rng.uniform(size=dd.shape) < frac_sentinel] = -np.inf
    # coarse values create ties in the block scores
    v = np.round(v / 4) * 4
    V.copy_(torch.from_numpy(v))
    D.copy_(torch.from_numpy(dd))
    st.refresh()  # V and D were written through the views
    torch.cuda.synchronize()


@pytest.mark.parametrize("R", [1, 2, 4])
@pytest.mark.parametrize("s,g", [(0.5, 0.05), (0.4, 0.1), (0.9, 0.3), (0.0, 0.05), (0.3, 0.0)])
def test_predict_select_bit_exact(R, s, g):
    rng = np.random.default_rng(int(R * 100 + s * 10 + g * 1000))
    st = make_state(Q=5, max_slots=8192 + 64, R=R, s=s, g=g)
    random_state(st, 0, rng)
    ctx = np.array([1, 63, 64 * 37 + 5, 8192 - R + 1, 4096], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    mask = st.new_mask()
    for step in [0, 3, 1 << 33]:
        isa.spin_predict_select(st, 0, R, step, ctx_t, mask)
        assert isa.spin_get_error(st)[0] == 0
        V, D = st.ema(0)
        S_gpu = st.block_scores().cpu().numpy()
        for q in range(5):
            S_ref = oracle.predict_pool(V[q].cpu().numpy(), D[q].cpu().numpy(), int(ctx[q]), R, 64, st.mask_stride)
            if s > 0:
                for r in range(R):
                    n = oracle.num_blocks(int(ctx[q]), r, 64)
                    assert np.array_equal(S_gpu[q, r, :n], S_ref[r, :n])
            m_ref = oracle.select(S_ref, int(ctx[q]), R, 64, s, g, 7, q, 0, step)
            assert np.array_equal(mask[q].cpu().numpy(), m_ref), (q, step)


@pytest.mark.parametrize("R", [1, 2, 3, 4])
@pytest.mark.parametrize("b", [16, 32, 128, 256])
def test_max_pooling_block_sizes_bit_exact(R, b):
    """Max pooling at every block size: b = 16 keeps no group maxima (V is
    read slot by slot), b >= 32 takes V's part from the 32-slot group maxima
    except in the group of the newest slots.  Contexts end on, just before
    and just after 32-slot and block boundaries; the block scores and the
    mask equal the oracle's bit for bit."""
    rng = np.random.default_rng(R * 31 + b)
    max_slots = 300 * b + 64
    st = make_state(Q=6, max_slots=max_slots, R=R, H=16, s=0.5, g=0.1, b=b)  # H: a valid config at b = 256
    random_state(st, 0, rng)
    top = max_slots - R + 1
    ctx = np.array([1, 31, 32 * 7 + 1, b * 40, b * 97 + 33, top], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    mask = st.new_mask()
    isa.spin_predict_select(st, 0, R, 4, ctx_t, mask)
    assert isa.spin_get_error(st)[0] == 0
    V, D = st.ema(0)
    S_gpu = st.block_scores().cpu().numpy()
    for q in range(len(ctx)):
        S_ref = oracle.predict_pool(V[q].cpu().numpy(), D[q].cpu().numpy(), int(ctx[q]), R, b, st.mask_stride)
        for r in range(R):
            n = oracle.num_blocks(int(ctx[q]), r, b)
            assert np.array_equal(S_gpu[q, r, :n].view(np.uint32), S_ref[r, :n].view(np.uint32)), (q, r)
        m_ref = oracle.select(S_ref, int(ctx[q]), R, b, 0.5, 0.1, 7, q, 0, 4)
        assert np.array_equal(mask[q].cpu().numpy(), m_ref), q


@pytest.mark.parametrize("g", [0.1, 0.3])
def test_select_large_request_with_infinite_and_tied_scores(g):
    # one 1M-slot request: 16,385 blocks, many equal block scores.  The
    # exploration draw of ~820 blocks (g = 0.1) goes through the sorted short
    # list, ~2,460 (g = 0.3) overflow it and take the radix select; the
    # 300K-slot request's draw is ranked by counting.
    rng = np.random.default_rng(1)
    st = make_state(Q=2, max_slots=1024 * 1024 + 64, R=1, s=0.5, g=g, k=2048)
    V, D = st.ema(0)
    v = rng.integers(0, 3, V.shape).astype(np.float32)
    v[:, -5000:] = np.inf
    V.copy_(torch.from_numpy(v))
    D.fill_(-np.inf)
    st.refresh()  # V and D were written through the views
    ctx = np.array([1024 * 1024 + 1, 300000], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    mask = st.new_mask()
    isa.spin_predict_select(st, 0, 1, 11, ctx_t, mask)
    assert isa.spin_get_error(st)[0] == 0
    for q in range(2):
        S_ref = oracle.predict_pool(V[q].cpu().numpy(), D[q].cpu().numpy(), int(ctx[q]), 1, 64, st.mask_stride)
        m_ref = oracle.select(S_ref, int(ctx[q]), 1, 64, 0.5, g, 7, q, 0, 11)
        assert np.array_equal(mask[q].cpu().numpy(), m_ref)


def fp8_inputs(Q, R, H, d, max_slots, rng, device="cuda", permute=True):
    wl = workloads.config(1, requests=Q, ctx0=(max_slots - 8,) * Q, steps=1, H=H, d=d, rows=R,
                          permute_pages=permute, spare_slots=8)
    cache = workloads.make_key_cache(wl, 0, device)
    q = (torch.randn((Q, R, H, d), generator=torch.Generator(device).manual_seed(int(rng.integers(1 << 30))),
                     device=device) * torch.exp(torch.randn((Q, R, H, 1), device=device) * 2)).to(torch.bfloat16)
    q[0, 0, 3] = 0                                            # an all-zero head
    w = torch.rand((Q, R, H), device=device)
    return wl, cache, q.contiguous(), w.contiguous()


def run_score(st, kind, R, cache, q, w, ctx_t, mask, fp8=True):
    isa.spin_set_score_kernel(st, kind)
    scores = st.new_scores()
    scores.fill_(float("nan"))
    isa.spin_indexer_score(st, 0, R, cache.keys, cache.kscale if fp8 else None, cache.block_table, q, w, ctx_t,
                           mask, scores)
    assert isa.spin_get_error(st)[0] == 0
    return scores


@pytest.mark.parametrize("R", [1, 2, 4])
@pytest.mark.parametrize("kind", [isa.SPIN_SCORE_SIMT, isa.SPIN_SCORE_TCGEN05])
def test_fp8_scores_vs_oracle(R, kind):
    check_fp8_scores(R, 64, kind, R)


@pytest.mark.parametrize("R,H", [(1, 32), (1, 128), (2, 128), (3, 48)])
def test_tcgen05_other_head_counts(R, H):
    """Head counts other than 64 take the tcgen05 kernel's generic column
    loop: N = 32, 128 (two CTAs per SM), 256 and 144 (one CTA per SM, rows
    split over two epilogue groups; 48 heads end on a 16-column load)."""
    check_fp8_scores(R, H, isa.SPIN_SCORE_TCGEN05, 100 + H + R)


@pytest.mark.parametrize("R", [1, 2, 4])
def test_tcgen05_short_requests_between_long_ones(R):
    """One-tile requests between long ones, so that CTAs meet request changes
    every few tiles: N = 64 (two CTAs per SM, one query buffer, side data two
    tiles ahead), N = 128 (two CTAs per SM, one query buffer, one tile ahead)
    and N = 256 (one CTA per SM, two query buffers).  The epilogue's side-data prefetch
    must never wait on its own hand-back (a stalled wait would end in
    ERR_TIMEOUT); scores match the oracle on the short requests and on a
    sample of the long ones."""
    rng = np.random.default_rng(40 + R)
    Q, H, d, max_slots = 5, 64, 128, 64 * 1501
    st = make_state(Q=Q, max_slots=max_slots, R=R, H=H, d=d)
    wl, cache, q, w = fp8_inputs(Q, R, H, d, max_slots, rng, permute=False)
    ctx = np.array([64 * 1500, 100, 64 * 1500, 100, 64 * 1500 - 37], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    m = np.zeros((Q, st.mask_stride), np.uint8)
    for qq in range(Q):
        m[qq, : oracle.num_blocks(int(ctx[qq]), R - 1, 64)] = 1
    scores = run_score(st, isa.SPIN_SCORE_TCGEN05, R, cache, q, w, ctx_t, torch.from_numpy(m).cuda())
    for qq in range(Q):
        q8, wq, _ = oracle.quantize_q(q[qq].float().cpu().numpy().astype(np.float64), w[qq].cpu().numpy())
        keys, ks, ident = workloads.request_pages(cache, qq)
        n_last = oracle.num_blocks(int(ctx[qq]), R - 1, 64)
        sub = m[qq].copy()
        if n_last > 8:                                       # a sample of a long request's blocks
            sub[:] = 0
            sub[rng.choice(n_last, 12, replace=False)] = 1
            sub[n_last - 1] = 1
        ref = oracle.score_fp8(keys.numpy(), ks.numpy(), ident.numpy(), q8, wq, int(ctx[qq]), sub, st.score_stride)
        got = scores[qq, :R].cpu().numpy()
        sc = ~np.isnan(ref)
        assert sc.sum() > 0
        assert score_close(got[sc], ref[sc]).all(), qq


def check_fp8_scores(R, H, kind, seed):
    rng = np.random.default_rng(seed)
    Q, d, max_slots = 3, 128, 64 * 41
    st = make_state(Q=Q, max_slots=max_slots, R=R, H=H, d=d)
    wl, cache, q, w = fp8_inputs(Q, R, H, d, max_slots, rng)
    ctx = np.array([64 * 40 + 7 - R + 1, 130, 64 * 23], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    m = (rng.uniform(size=(Q, st.mask_stride)) < 0.6).astype(np.uint8)
    for qq in range(Q):
        m[qq, oracle.num_blocks(int(ctx[qq]), R - 1, 64):] = 0
        m[qq, 0] = 2                                         # odd kept counts -> half-filled tiles
    mask = torch.from_numpy(m).cuda()
    scores = run_score(st, kind, R, cache, q, w, ctx_t, mask)
    q8g, wqg = st.qquant(R)
    for qq in range(Q):
        q8, wq, _ = oracle.quantize_q(q[qq].float().cpu().numpy().astype(np.float64), w[qq].cpu().numpy())
        assert np.array_equal(q8g[qq].cpu().numpy(), q8)
        assert np.array_equal(wqg[qq].cpu().numpy(), wq)
        keys, ks, ident = workloads.request_pages(cache, qq)
        ref = oracle.score_fp8(keys.numpy(), ks.numpy(), ident.numpy(), q8, wq, int(ctx[qq]), m[qq], st.score_stride)
        got = scores[qq, :R].cpu().numpy()
        sc = ~np.isnan(ref)
        assert sc.sum() > 0
        assert score_close(got[sc], ref[sc]).all()
        assert np.all(np.isnan(got[~sc]))                    # nothing written outside kept, visible slots


def test_tcgen05_agrees_with_simt_at_serving_shape():
    rng = np.random.default_rng(5)
    Q, R, H, d, max_slots = 8, 1, 64, 128, 64 * 300
    st = make_state(Q=Q, max_slots=max_slots, R=R)
    wl, cache, q, w = fp8_inputs(Q, R, H, d, max_slots, rng)
    ctx_t = torch.full((Q,), max_slots - 3, dtype=torch.int32).cuda()
    mask = torch.from_numpy((rng.uniform(size=(Q, st.mask_stride)) < 0.5).astype(np.uint8)).cuda()
    a = run_score(st, isa.SPIN_SCORE_SIMT, R, cache, q, w, ctx_t, mask)
    b = run_score(st, isa.SPIN_SCORE_TCGEN05, R, cache, q, w, ctx_t, mask)
    fin = ~torch.isnan(a)
    assert torch.equal(fin, ~torch.isnan(b))
    assert score_close(b[fin].cpu().numpy(), a[fin].cpu().numpy()).all()


def test_fp32_scores_vs_oracle():
    rng = np.random.default_rng(9)
    wl = workloads.config(0, ctx0=(4096,), steps=4)
    cache = workloads.make_key_cache(wl, 0, "cuda")
    st = make_state(Q=1, max_slots=wl.max_slots, R=1, H=8, d=64, fp8=False, k=256)
    q = torch.randn((1, 1, 8, 64), device="cuda")
    w = torch.rand((1, 1, 8), device="cuda")
    ctx = 4097
    m = (rng.uniform(size=(1, st.mask_stride)) < 0.7).astype(np.uint8)
    scores = run_score(st, isa.SPIN_SCORE_AUTO, 1, cache, q, w, torch.tensor([ctx], dtype=torch.int32).cuda(),
                       torch.from_numpy(m).cuda(), fp8=False)
    ref = oracle.score_f32(cache.keys.cpu().numpy(), cache.block_table[0].cpu().numpy(), q[0].cpu().numpy(),
                           w[0].cpu().numpy(), ctx, m[0], st.score_stride)
    got = scores[0, :1].cpu().numpy()
    sc = ~np.isnan(ref)
    assert score_close(got[sc], ref[sc]).all()


@pytest.mark.parametrize("R", [1, 4])
@pytest.mark.parametrize("kind", ["random", "ties", "few"])
def test_topk_bit_exact(R, kind):
    rng = np.random.default_rng(R + len(kind))
    Q, k = 4, 256
    st = make_state(Q=Q, max_slots=64 * 200, R=R, k=k)
    ctx = np.array([64 * 200 - R + 1, 64 * 37 + 11, 3, 64 * 5], np.int64)
    m = (rng.uniform(size=(Q, st.mask_stride)) < 0.5).astype(np.uint8)
    if kind == "few":
        m[:] = 0
        m[:, 1] = 1                                         # fewer than k scored slots: padding
    for qq in range(Q):
        m[qq, oracle.num_blocks(int(ctx[qq]), R - 1, 64):] = 0
    scores = st.new_scores()
    if kind == "ties":
        vals = rng.integers(0, 6, scores.shape).astype(np.float32)
        vals[rng.uniform(size=vals.shape) < 0.01] = -0.0
    else:
        vals = rng.standard_normal(scores.shape).astype(np.float32) * 10
    scores.copy_(torch.from_numpy(vals))
    topk = torch.empty((Q, R, k), dtype=torch.int32, device="cuda")
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    isa.spin_topk(st, R, scores, torch.from_numpy(m).cuda(), ctx_t, topk)
    assert isa.spin_get_error(st)[0] == 0
    got = topk.cpu().numpy()
    for qq in range(Q):
        for r in range(R):
            ref = oracle.topk_row(vals[qq, r].astype(np.float64), m[qq], int(ctx[qq]), r, 64, k)
            assert np.array_equal(got[qq, r], ref), (qq, r)


@pytest.mark.parametrize("R", [1, 2, 3, 4])
@pytest.mark.parametrize("kept", [0.5, 0.9])
def test_ema_update_prefix_valid_bit_exact(R, kept):
    # at 90% most blocks are kept with a kept successor: the replay's path
    # for those blocks (only r < a tested) against the general one
    rng = np.random.default_rng(40 + R + int(100 * kept))
    Q = 6
    st = make_state(Q=Q, max_slots=64 * 60, R=R)
    random_state(st, 0, rng, frac_sentinel=0.3)
    ctx = np.array([64 * 60 - R + 1, 64 * 10 + 1, 64 * 10, 1, 65, 64 * 33 + 17], np.int64)
    m = (rng.uniform(size=(Q, st.mask_stride)) < kept).astype(np.uint8)
    for qq in range(Q):
        m[qq, oracle.num_blocks(int(ctx[qq]), R - 1, 64):] = 0
    acc = rng.integers(1, R + 1, Q).astype(np.int32)
    scores = st.new_scores()
    vals = rng.uniform(0, 30, scores.shape).astype(np.float32)
    scores.copy_(torch.from_numpy(vals))
    V, D = st.ema(0)
    V0, D0 = V.cpu().numpy().copy(), D.cpu().numpy().copy()
    isa.spin_ema_update(st, 0, R, scores, torch.from_numpy(m).cuda(), torch.from_numpy(ctx).to(torch.int32).cuda(),
                        torch.from_numpy(acc).cuda())
    assert isa.spin_get_error(st)[0] == 0
    for qq in range(Q):
        v, d = V0[qq].copy(), D0[qq].copy()
        oracle.ema_update(v, d, vals[qq, :R], m[qq], int(ctx[qq]), int(acc[qq]), 64, 0.9)
        assert np.array_equal(V[qq].cpu().numpy().view(np.uint32), v.view(np.uint32)), qq
        assert np.array_equal(D[qq].cpu().numpy().view(np.uint32), d.view(np.uint32)), qq


def test_miss_count():
    rng = np.random.default_rng(3)
    Q, R, k = 3, 2, 128
    st = make_state(Q=Q, max_slots=64 * 50, R=R, k=k)
    m = (rng.uniform(size=(Q, st.mask_stride)) < 0.5).astype(np.uint8)
    full = rng.integers(0, 64 * 50, (Q, R, k)).astype(np.int32)
    full[:, :, -7:] = -1
    missed = torch.zeros((Q, R), dtype=torch.int32, device="cuda")
    total = torch.zeros((Q, R), dtype=torch.int32, device="cuda")
    isa.spin_miss_count(st, R, torch.from_numpy(full).cuda(), torch.from_numpy(m).cuda(), missed, total)
    for qq in range(Q):
        for r in range(R):
            frac = oracle.miss_fraction(full[qq, r], m[qq], 64)
            assert total[qq, r].item() == k - 7
            assert abs(missed[qq, r].item() / (k - 7) - frac) < 1e-12


@pytest.mark.parametrize("pattern", ["hidden_from_sample", "only_in_sample", "all_equal", "heavy_ties"])
def test_topk_fallback_paths_bit_exact(pattern):
    """Score patterns that defeat the sampled threshold estimate (the sample
    reads 4 of every 64 kept-slot positions) or overflow the on-chip
    candidate list, so each exact fallback of the top-k kernel runs."""
    rng = np.random.default_rng(len(pattern))
    Q, R, k = 2, 1, 2048
    st = make_state(Q=Q, max_slots=64 * 600, R=R, k=k)
    ctx = np.array([64 * 600, 64 * 431 + 9], np.int64)
    m = (rng.uniform(size=(Q, st.mask_stride)) < 0.8).astype(np.uint8)
    for qq in range(Q):
        m[qq, oracle.num_blocks(int(ctx[qq]), R - 1, 64):] = 0
    scores = st.new_scores()
    vals = rng.uniform(0, 1, scores.shape).astype(np.float32)
    pos = np.zeros(scores.shape, np.int64)
    for qq in range(Q):       # position of each slot in the ascending kept-slot order
        kept = np.nonzero(m[qq])[0]
        slots = (kept[:, None] * 64 + np.arange(64)[None, :]).ravel()
        pos[qq, 0, slots[slots < st.score_stride]] = np.arange(slots.size)[slots < st.score_stride]
    sampled = (pos % 64) < 4
    if pattern == "hidden_from_sample":
        vals[~sampled] += 100.0
    elif pattern == "only_in_sample":
        vals[sampled] += 100.0
    elif pattern == "all_equal":
        vals[:] = 3.0
    else:
        vals = rng.integers(0, 3, scores.shape).astype(np.float32)
    scores.copy_(torch.from_numpy(vals))
    topk = torch.empty((Q, R, k), dtype=torch.int32, device="cuda")
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    isa.spin_topk(st, R, scores, torch.from_numpy(m).cuda(), ctx_t, topk)
    assert isa.spin_get_error(st)[0] == 0
    got = topk.cpu().numpy()
    for qq in range(Q):
        ref = oracle.topk_row(vals[qq, 0].astype(np.float64), m[qq], int(ctx[qq]), 0, 64, k)
        assert np.array_equal(got[qq, 0], ref), (pattern, qq)


def test_kernel_timing_mask_times_only_named_stages():
    """spin_set_kernel_timing_mask brackets only the named stages with events;
    every launch is still counted."""
    wl = workloads.config(1, requests=2, ctx0=(9000, 20000), steps=2, spare_slots=8)
    cache = workloads.make_key_cache(wl, 0, "cuda")
    q, w = workloads.make_queries(wl, 0, 1, "cuda")
    st = make_state(Q=2, max_slots=wl.max_slots, k=wl.topk, s=0.4)
    ctx = torch.tensor([9001, 20001], dtype=torch.int32, device="cuda")
    mask = st.new_mask()
    topk = torch.empty((2, 1, wl.topk), dtype=torch.int32, device="cuda")
    isa.spin_kernel_times(st)
    isa.spin_set_kernel_timing_mask(st, ["score"])
    for step in range(2):
        isa.spin_decode_step(st, 0, 1, step, cache.keys, cache.kscale, cache.block_table, q[:, :1].contiguous(),
                             w[:, :1].contiguous(), ctx, False, mask, topk)
    isa.spin_set_kernel_timing(st, False)
    times = isa.spin_kernel_times(st)
    assert times["score"][1] == 2 and times["score"][0] > 0
    for stage in ("predict", "select", "topk"):
        assert times[stage][1] == 2 and times[stage][0] == 0
    assert isa.spin_get_error(st)[0] == 0
    with pytest.raises(ValueError):
        isa.spin_set_kernel_timing_mask(st, ["no such stage"])


@pytest.mark.parametrize("R", [2, 4])
def test_select_rows_long_context_bit_exact(R):
    """640K slots with too many requests for clusters (74), so one CTA per
    request: two rows' block keys still fit on chip together and their radix
    passes run together; four rows' do not, and the rows' selects run one
    after another.  The union masks equal the oracle's bit for bit."""
    rng = np.random.default_rng(R + 40)
    max_slots = 640 * 1024 + 64
    st = make_state(Q=74, max_slots=max_slots, R=R, H=16, s=0.5, g=0.1, k=2048)
    V, D = st.ema(0)
    v = rng.integers(0, 6, V.shape).astype(np.float32)    # many equal block scores
    v[:, -3000:] = np.inf
    V.copy_(torch.from_numpy(v))
    d = rng.standard_normal(D.shape).astype(np.float32)
    d[rng.random(D.shape) < 0.5] = -np.inf
    D.copy_(torch.from_numpy(d))
    st.refresh()  # V and D were written through the views
    ctx = np.full(74, max_slots - 64 - R + 1, np.int64)
    ctx[1], ctx[2], ctx[3] = 1, 300_000 + 37, 64 * 5000
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    mask = st.new_mask()
    isa.spin_predict_select(st, 0, R, 6, ctx_t, mask)
    assert isa.spin_get_error(st)[0] == 0
    for q in range(4):
        S_ref = oracle.predict_pool(V[q].cpu().numpy(), D[q].cpu().numpy(), int(ctx[q]), R, 64, st.mask_stride)
        m_ref = oracle.select(S_ref, int(ctx[q]), R, 64, 0.5, 0.1, 7, q, 0, 6)
        assert np.array_equal(mask[q].cpu().numpy(), m_ref), q


@pytest.mark.parametrize("R", [1, 2, 4])
@pytest.mark.parametrize("s,g", [(0.5, 0.05), (0.4, 0.3), (0.0, 0.05), (0.3, 0.0), (0.999, 0.5)])
def test_select_cluster_paths_bit_exact(R, s, g):
    """Long contexts take the cluster select (8 CTAs per request): the rows'
    radix selects across ranks, ties in block order across ranks, the
    exploration draw by list and by radix, all-keep, and empty requests."""
    rng = np.random.default_rng(int(R * 1000 + s * 100 + g * 10))
    st = make_state(Q=4, max_slots=1024 * 1024 + 64, R=R, s=s, g=g, k=2048)
    V, D = st.ema(0)
    v = rng.integers(0, 4, V.shape).astype(np.float32)    # many equal block scores
    v[:, -3000:] = np.inf
    V.copy_(torch.from_numpy(v))
    d = rng.standard_normal(D.shape).astype(np.float32)
    d[rng.random(D.shape) < 0.5] = -np.inf
    D.copy_(torch.from_numpy(d))
    st.refresh()  # V and D were written through the views
    ctx = np.array([1, 1024 * 1024 - R + 1, 300_000 + 37, 64 * 5000], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    mask = st.new_mask()
    for step in [0, 5]:
        isa.spin_predict_select(st, 0, R, step, ctx_t, mask)
        assert isa.spin_get_error(st)[0] == 0
        for q in range(4):
            S_ref = oracle.predict_pool(V[q].cpu().numpy(), D[q].cpu().numpy(), int(ctx[q]), R, 64, st.mask_stride)
            m_ref = oracle.select(S_ref, int(ctx[q]), R, 64, s, g, 7, q, 0, step)
            assert np.array_equal(mask[q].cpu().numpy(), m_ref), (q, step)


@pytest.mark.parametrize("R", [2, 4])
@pytest.mark.parametrize("max_slots", [8192 + 64, 1024 * 1024 + 64])
def test_mtp_row0_select_bit_exact(R, max_slots):
    """Row-0 sharing: row 0's block scores, its predicted set, the drafts'
    new blocks kept and the exploration among row 0's unkept blocks, bit
    for bit, in the one-CTA select and (1M slots) the cluster select."""
    rng = np.random.default_rng(R * 7 + max_slots % 97)
    st = make_state(Q=4, max_slots=max_slots, R=R, s=0.5, g=0.1, k=2048, mtp_policy=isa.SPIN_MTP_ROW0)
    V, D = st.ema(0)
    v = rng.integers(0, 4, V.shape).astype(np.float32)    # many equal block scores
    v[:, -3000:] = np.inf
    V.copy_(torch.from_numpy(v))
    d = rng.standard_normal(D.shape).astype(np.float32)
    d[rng.random(D.shape) < 0.5] = -np.inf
    D.copy_(torch.from_numpy(d))
    st.refresh()  # V and D were written through the views
    top = max_slots - 64 - R + 1
    ctx = np.array([1, top, top // 3 + 37, 64 * (top // 200)], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    mask = st.new_mask()
    for step in [0, 5]:
        isa.spin_predict_select(st, 0, R, step, ctx_t, mask)
        assert isa.spin_get_error(st)[0] == 0
        S_gpu = st.block_scores().cpu().numpy()
        for q in range(4):
            S_ref = oracle.predict_pool(V[q].cpu().numpy(), D[q].cpu().numpy(), int(ctx[q]), R, 64, st.mask_stride)
            n0 = oracle.num_blocks(int(ctx[q]), 0, 64)
            assert np.array_equal(S_gpu[q, 0, :n0].view(np.uint32), S_ref[0, :n0].view(np.uint32)), (q, step)
            m_ref = oracle.select(S_ref, int(ctx[q]), R, 64, 0.5, 0.1, 7, q, 0, step, oracle.MTP_ROW0)
            assert np.array_equal(mask[q].cpu().numpy(), m_ref), (q, step)


@pytest.mark.parametrize("pooling", [isa.SPIN_POOL_MEAN, isa.SPIN_POOL_TOP4])
@pytest.mark.parametrize("R,b", [(1, 64), (4, 64), (2, 16), (1, 256)])
@pytest.mark.parametrize("spread", [False, True])
def test_pooling_variants_vs_exact_mean(pooling, R, b, spread):
    """Mean and Top-4 block pooling: the kernel's block scores are within one
    float ulp (plus the double sum's bound where z takes both signs) of the
    oracle's exact mean rounded once, and nearly always equal to it; the mask
    equals the oracle's selection from the GPU's block scores bit for bit.
    With `spread` the values span 2^-60 .. 2^60, where the double sum is not
    exact."""
    rng = np.random.default_rng(pooling * 100 + R * 10 + b + 1000 * spread)
    max_slots = 200 * b + 64
    cfg = isa.make_config(num_layers=1, num_requests=3, max_slots=max_slots, block_size=b, topk=256, max_rows=R,
                          gamma=0.05, target_sparsity=0.5, seed=7, pooling=pooling)
    st = isa.SpinState(cfg)
    V, D = st.ema(0)
    scale = 2.0 ** rng.integers(-60, 60, V.shape) if spread else 10.0
    v = (rng.standard_normal(V.shape) * scale).astype(np.float32)
    v[rng.random(V.shape) < 0.02] = np.inf                # never-observed slots
    V.copy_(torch.from_numpy(v))
    d = (rng.standard_normal(D.shape) * scale).astype(np.float32)
    d[rng.random(D.shape) < 0.3] = -np.inf
    D.copy_(torch.from_numpy(d))
    st.refresh()  # V and D were written through the views
    ctx = np.array([1, 37 * b + 5, max_slots - R + 1], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    mask = st.new_mask()
    isa.spin_predict_select(st, 0, R, 3, ctx_t, mask)
    assert isa.spin_get_error(st)[0] == 0
    S_gpu = st.block_scores().cpu().numpy()
    n_same = n_all = 0
    for q in range(3):
        Vq, Dq = V[q].cpu().numpy(), D[q].cpu().numpy()
        S_ref = oracle.predict_pool(Vq, Dq, int(ctx[q]), R, b, st.mask_stride, pooling)
        for r in range(R):
            n = oracle.num_blocks(int(ctx[q]), r, b)
            p = int(ctx[q]) - 1 + r
            zabs = np.zeros(n)
            for j in range(n):
                i = np.arange(j * b, min((j + 1) * b, p + 1))
                z = np.abs(np.maximum(Vq[i], Dq[p - i]).astype(np.float64))
                zabs[j] = z[np.isfinite(z)].mean() if np.isfinite(z).any() else 0.0
            assert pool_close(S_gpu[q, r, :n], S_ref[r, :n], zabs).all(), (q, r)
            n_same += int((S_gpu[q, r, :n].view(np.uint32) == S_ref[r, :n].view(np.uint32)).sum())
            n_all += n
        m_ref = oracle.select(S_gpu[q, :R, :st.mask_stride], int(ctx[q]), R, b, 0.5, 0.05, 7, q, 0, 3)
        assert np.array_equal(mask[q].cpu().numpy(), m_ref), q
    if not spread:
        # a narrow exponent band: the double sum is exact, one rounding remains
        assert n_same >= 0.999 * n_all, (n_same, n_all)
