"""Decode-step trajectories through spin_decode_step, checked in lock step
against the oracle on every step (mask, top-k, V, D bit for bit; scores
within rel 1e-3 / abs 1e-4 of fp64), for each of the five workloads (scaled
to oracle-friendly sizes except where stated) and the per-layer budget."""
import numpy as np
import pytest
import torch

import indexer_sparse_attention_b200 as isa
import oracle
import workloads
from lockstep import Harness, run_multilayer, score_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from indexer_sparse_attention_b200 import build
    build.build()
    oracle.build()


def bootstrap(h, layer=0, sample_blocks=None):
    """Step 0: all-keep history bootstrap."""
    keep = list(h.sparsity)
    h.set_sparsity([0.0] * h.wl.layers)
    h.run_step(layer, check=range(min(2, h.wl.requests)), sample_blocks=sample_blocks)
    h.set_sparsity(keep)


def test_tiny_fp32_workload_all_steps():
    wl = workloads.config(0)
    h = Harness(wl)
    bootstrap(h)
    kept_fracs = []
    for _ in range(wl.steps - 1):
        res = h.run_step(0, check=[0])
        kept_fracs.append(res[0]["kept"] / res[0]["n"])
    assert all(abs(f - 0.7) < 0.02 for f in kept_fracs)


@pytest.mark.parametrize("kind", [isa.SPIN_SCORE_TCGEN05, isa.SPIN_SCORE_SIMT])
def test_dsa_single_request(kind):
    wl = workloads.config(1, steps=8, ctx0=(16384 + 37,))
    h = Harness(wl, score_kernel=kind)
    bootstrap(h)
    for _ in range(wl.steps - 1):
        h.run_step(0, check=[0])


def test_dsa_single_request_full_context():
    # 65,536-slot context as specified, 6 steps, tensor-core path
    wl = workloads.config(1, steps=6)
    h = Harness(wl)
    bootstrap(h)
    for _ in range(wl.steps - 1):
        h.run_step(0, check=[0], sample_blocks=64)


def test_serving_batch_scaled():
    wl = workloads.config(2, requests=6, ctx0=(20000, 8192, 65536, 1000, 33333, 64 * 64), steps=5)
    h = Harness(wl)
    bootstrap(h)
    for s in [0.4, 0.5, 0.5, 0.0]:
        h.set_sparsity([s])
        h.run_step(0, check=range(6))


def test_mtp_rows_union_and_prefix_valid_replay():
    wl = workloads.config(3, requests=5, ctx0=(8192, 8190, 64 * 30 + 62, 4000, 129), steps=8)
    h = Harness(wl)
    bootstrap(h)
    acc = workloads.accepted_lengths(wl, wl.steps).numpy()
    realized = []
    for t in range(1, wl.steps):
        res = h.run_step(0, accepted=acc[t], check=range(5))
        realized += [1 - r["kept"] / r["n"] for r in res.values()]
    assert max(realized) <= 0.4 + 1e-9                      # union only adds blocks


def test_mtp_rows_small_topk_takes_the_group_path():
    """Four MTP rows with a top-k small enough (k = 64) that rows of the longer
    requests take the top-k's group-maxima path, which reads the score
    maxima of each 32 slots, while the short request's rows fit on chip and
    its maxima are skipped: every row's top-k equals the oracle's."""
    wl = workloads.config(3, requests=4, ctx0=(30_000, 20_000, 64 * 40 + 5, 1500), steps=5, topk=64)
    h = Harness(wl)
    bootstrap(h)
    acc = workloads.accepted_lengths(wl, wl.steps).numpy()
    for t in range(1, wl.steps):
        h.run_step(0, accepted=acc[t], check=range(4))


@pytest.mark.parametrize("defer", [True, False])
def test_mtp_row0_sharing_and_row0_update(defer):
    """The baseline MTP policy in lock step: row 0's mask for every row and
    the EMA update from row 0's scores alone, with deferred accepted lengths
    and with the update inside the decode step."""
    wl = workloads.config(3, requests=5, ctx0=(8192, 8190, 64 * 30 + 62, 4000, 129), steps=6,
                          mtp_policy=isa.SPIN_MTP_ROW0)
    h = Harness(wl)
    bootstrap(h)
    acc = workloads.accepted_lengths(wl, wl.steps).numpy()
    realized = []
    for t in range(1, wl.steps):
        res = h.run_step(0, accepted=acc[t] if defer else None, check=range(5), defer=defer)
        realized += [1 - r["kept"] / r["n"] for r in res.values()]
    assert max(realized) <= 0.4 + 1e-9


def test_multilayer_per_layer_budget():
    """Ragged long-context workload, scaled: warm-up at uniform 50% with a
    shadow full indexer measuring miss on the GPU, then per-layer budgets."""
    wl = workloads.config(4, layers=2, requests=3, ctx0=(70000, 40000, 100000), steps=6, warmup_steps=2)
    run_multilayer(Harness(wl), check=range(wl.requests), check_warmup=[1])


def test_serving_full_size_sampled():
    """96 requests x 512K slots, the configuration the benchmark times:
    all-keep bootstrap, then 50% and 40% steps; three sampled requests are
    replayed in the oracle (mask, top-k and state bit for bit; scores on 48
    random kept blocks plus the ragged last block)."""
    wl = workloads.config(2, steps=3)
    h = Harness(wl)
    check = [0, 47, 95]
    bootstrap(h, sample_blocks=48)
    h.run_step(0, check=check, sample_blocks=48)
    h.set_sparsity([0.4])
    h.run_step(0, check=check, sample_blocks=48)


def test_export_import_resumes_bit_identically():
    wl = workloads.config(2, requests=3, ctx0=(5000, 9000, 300), steps=6)
    h = Harness(wl)
    bootstrap(h)
    h.run_step(0)
    blob = isa.spin_state_export(h.st)
    saved = (h.committed.copy(), h.step_index)
    outs = []
    for _ in range(2):
        h.run_step(0)
        outs.append((h.mask.clone(), h.topk.clone()))
    V1 = [x.clone() for x in h.st.ema(0)]
    isa.spin_state_import(h.st, blob)
    h.committed, h.step_index = saved
    for i in range(2):
        h.run_step(0)
        assert torch.equal(h.mask, outs[i][0]) and torch.equal(h.topk, outs[i][1])
    V2 = h.st.ema(0)
    assert torch.equal(V1[0].view(torch.int32), V2[0].view(torch.int32))
    assert torch.equal(V1[1].view(torch.int32), V2[1].view(torch.int32))


def test_device_argument_errors_set_error_word():
    wl = workloads.config(2, requests=3, ctx0=(5000, 9000, 300), steps=2)
    h = Harness(wl)
    qstep, wstep, ctx = h.step_inputs(0, 1)
    bad_ctx = ctx.clone()
    bad_ctx[1] = wl.max_slots + 5                           # past the capacity
    cache = h.caches[0]
    topk = torch.empty((3, 1, wl.topk), dtype=torch.int32, device="cuda")
    isa.spin_decode_step(h.st, 0, 1, 0, cache.keys, cache.kscale, cache.block_table, qstep, wstep, bad_ctx,
                         False, h.mask, topk, None)
    status, word = isa.spin_get_error(h.st)
    assert status == 6 and word & 1                          # SPIN_EDEVICE, ERR_CTX_LEN
    assert torch.all(topk[1] == -1)
    bt = cache.block_table.clone()
    bt[2, :] = cache.keys.shape[0] + 10                      # every page of request 2 outside the cache
    isa.spin_decode_step(h.st, 0, 1, 0, cache.keys, cache.kscale, bt, qstep, wstep, ctx, False, h.mask, topk, None)
    status, word = isa.spin_get_error(h.st)
    assert status == 6 and word & 2
    with pytest.raises(isa.SpinError):
        isa.spin_decode_step(h.st, 0, 2, 0, cache.keys, cache.kscale, cache.block_table, qstep, wstep, ctx,
                             False, h.mask, topk, None)     # rows > max_rows: SPIN_EINVAL
    assert isa.spin_get_error(h.st)[0] == 0


def test_scores_jumping_between_steps():
    """Head weights scaled by 4 and then by 1/16 between steps move every
    score (and so the top-k threshold and the EMA state) far from the last
    step's values; every step still matches the oracle bit for bit."""
    wl = workloads.config(2, requests=3, ctx0=(200_000, 150_000, 90_011), steps=8)
    h = Harness(wl)
    bootstrap(h, sample_blocks=48)
    _, wall = h.queries[0]
    for factor in (1.0, 1.0, 4.0, 4.0, 0.25, 1.0, 1.0):
        pos = h.committed - np.array(wl.ctx0, np.int64)    # each request's next query position
        for qi in range(wl.requests):
            wall[qi, int(pos[qi])] *= factor               # head weights scale every score
        h.run_step(0, check=range(wl.requests), sample_blocks=48)


@pytest.mark.parametrize("b", [16, 32, 128, 256])
def test_block_sizes_other_than_64(b):
    """Paged blocks of 16..256 slots (the CUDA-core indexer takes them; the
    tensor-core tile is built for 64): predict, select, score, top-k and EMA
    in lock step."""
    wl = workloads.config(1, b=b, steps=4, ctx0=(12_000 + 37,), sparsity=0.5)
    h = Harness(wl)
    bootstrap(h)
    for _ in range(wl.steps - 1):
        h.run_step(0, check=[0], sample_blocks=max(8, 3072 // b))


def test_maximum_context():
    """One request at the largest context a state accepts (the top-k keeps a
    1.31M-slot bitmap on chip): 20,480 blocks, sampled lock-step checks."""
    limit = 160 * 1024 * 8                                  # slots the on-chip top-k bitmap holds
    wl = workloads.config(2, requests=1, ctx0=(limit - 8,), steps=3, spare_slots=0)
    assert wl.max_slots <= limit
    h = Harness(wl)
    bootstrap(h, sample_blocks=32)
    for _ in range(wl.steps - 1):
        h.run_step(0, check=[0], sample_blocks=32)


@pytest.mark.parametrize("pooling", [isa.SPIN_POOL_MEAN, isa.SPIN_POOL_TOP4])
def test_decode_steps_with_pooling_variants(pooling):
    """Serving-shaped steps with Mean and Top-4 block pooling, in lock step."""
    wl = workloads.config(2, requests=2, ctx0=(120_000, 64 * 900 + 11), steps=4, pooling=pooling)
    h = Harness(wl)
    bootstrap(h, sample_blocks=32)
    for _ in range(wl.steps - 1):
        h.run_step(0, check=range(wl.requests), sample_blocks=32)
