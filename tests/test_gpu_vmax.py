"""V's 32-slot group maxima.  With max pooling the prediction takes V's part
of a block score from them for every block below the newest one (the max over
a block of max(V_i, D_{p-i}) is the larger of V's maximum over the block and
D's), so each writer of V must leave every group maximum equal to the maximum
of its 32 values: state creation, fused one-row steps (tensor-core and SIMT
score kernels), the MTP prefix-valid replay and the row-0 update, request
resets, a checkpoint import, and direct writes followed by
spin_state_refresh.  The masks these states lead to are checked against the
oracle here on the last step and by the lock-step tests throughout."""
import numpy as np
import pytest
import torch

import indexer_sparse_attention_b200 as isa
import oracle
import workloads
from lockstep import Harness

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from indexer_sparse_attention_b200 import build
    build.build()
    oracle.build()


def assert_groups_exact(st, layers=(0,)):
    torch.cuda.synchronize()
    for layer in layers:
        V, _ = st.ema(layer)
        g = st.vmax(layer)
        assert g is not None
        ref = V.view(V.shape[0], -1, 32).amax(-1)
        bad = (g != ref).nonzero()
        assert bad.numel() == 0, (layer, bad[:5].tolist())


@pytest.mark.parametrize("kernel", [isa.SPIN_SCORE_AUTO, isa.SPIN_SCORE_SIMT])
def test_one_row_steps_keep_groups(kernel):
    # contexts that cross a 32-slot group and a block boundary during the steps
    wl = workloads.config(2, requests=4, ctx0=(4096 - 4, 6000 - 3, 64 * 50, 1000), steps=8)
    h = Harness(wl, score_kernel=kernel)
    assert_groups_exact(h.st)                      # all +inf at creation
    h.set_sparsity([0.0])
    h.run_step(0)
    assert_groups_exact(h.st)
    h.set_sparsity([wl.sparsity])
    for t in range(1, wl.steps):
        h.run_step(0, check=[0, 1] if t == wl.steps - 1 else ())
        assert_groups_exact(h.st)


@pytest.mark.parametrize("policy", [isa.SPIN_MTP_UNION_PREFIX, isa.SPIN_MTP_ROW0])
def test_mtp_replay_keeps_groups(policy):
    wl = workloads.config(3, requests=4, ctx0=(4096 - 6, 2000, 64 * 20, 777), steps=6, mtp_policy=policy)
    h = Harness(wl)
    acc = workloads.accepted_lengths(wl, wl.steps).numpy()
    h.set_sparsity([0.0])
    h.run_step(0)
    assert_groups_exact(h.st)
    h.set_sparsity([wl.sparsity])
    for t in range(1, wl.steps):
        h.run_step(0, accepted=acc[t], check=[0] if t == wl.steps - 1 else ())
        assert_groups_exact(h.st)


def test_reset_import_and_direct_writes_keep_groups():
    wl = workloads.config(2, requests=3, ctx0=(3000, 2000, 1500), steps=4, layers=2)
    h = Harness(wl)
    h.set_sparsity([0.0, 0.0])
    for layer in (0, 1):
        h.run_step(layer)
    h.set_sparsity([0.5, 0.5])
    for layer in (0, 1):
        h.run_step(layer)
    assert_groups_exact(h.st, (0, 1))
    blob = isa.spin_state_export(h.st)
    isa.spin_reset_requests(h.st, 1, [0, 2])       # one layer's rows back to +inf
    assert_groups_exact(h.st, (0, 1))
    assert torch.isinf(h.st.vmax(1)[[0, 2]]).all() and not torch.isinf(h.st.vmax(1)[1]).all()
    isa.spin_state_import(h.st, blob)              # the checkpoint's groups come back
    assert_groups_exact(h.st, (0, 1))
    V, D = h.st.ema(0)
    rng = np.random.default_rng(5)
    v = rng.standard_normal(V.shape).astype(np.float32)
    v[rng.random(V.shape) < 0.05] = np.inf
    V.copy_(torch.from_numpy(v))
    before = h.st.vmax(1).clone()
    h.st.refresh(0)
    assert_groups_exact(h.st, (0, 1))
    assert torch.equal(before, h.st.vmax(1))       # the other layer untouched
    # the prediction from the written state equals the oracle's selection
    ctx = np.array([3000, 2000, 1500], np.int64)
    ctx_t = torch.from_numpy(ctx).to(torch.int32).cuda()
    mask = h.st.new_mask()
    isa.spin_predict_select(h.st, 0, 1, 9, ctx_t, mask)
    assert isa.spin_get_error(h.st)[0] == 0
    for q in range(3):
        S_ref = oracle.predict_pool(V[q].cpu().numpy(), D[q].cpu().numpy(), int(ctx[q]), 1, 64, h.st.mask_stride)
        m_ref = oracle.select(S_ref, int(ctx[q]), 1, 64, 0.5, wl.gamma, wl.seed, q, 0, 9)
        assert np.array_equal(mask[q].cpu().numpy(), m_ref), q


@pytest.mark.parametrize("b,pooling", [(16, isa.SPIN_POOL_MAX), (64, isa.SPIN_POOL_MEAN), (64, isa.SPIN_POOL_TOP4)])
def test_no_groups_without_max_pooling_or_with_small_blocks(b, pooling):
    cfg = isa.make_config(num_layers=1, num_requests=2, max_slots=64 * 40, block_size=b, topk=256, pooling=pooling)
    st = isa.SpinState(cfg)
    assert st.vmax(0) is None
    st.refresh()                                   # nothing to bring up to date, no error
