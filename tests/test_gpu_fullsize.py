"""Lock-step parity at the specified sizes of the MTP and the multi-layer
ragged workloads, on sampled requests: the GPU runs the whole batch, and
each checked request is replayed in the oracle from the GPU's state before
the step (mask, top-k and the next V, D bit for bit; scores within rel 1e-3 /
abs 1e-4 of fp64 on a sample of kept blocks plus the ragged last block)."""
import numpy as np
import pytest

import oracle
import workloads
from lockstep import Harness, run_multilayer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from indexer_sparse_attention_b200 import build
    build.build()
    oracle.build()


def test_mtp_full_size_sampled():
    """32 requests x 128K slots, 4 query rows (1 verify + 3 drafts): the kept
    mask is the union of the rows' predicted sets plus one exploration draw,
    and the EMA update replays the accepted prefix, with accepted lengths drawn
    from P(a = 1..4) = (0.30, 0.25, 0.20, 0.25) (SPIN digest, arXiv深度剖析;
    SPIN listing, Table 7)."""
    wl = workloads.config(3, steps=4)
    assert wl.requests == 32 and wl.ctx0[0] == 128 * 1024 and wl.rows == 4
    h = Harness(wl)
    check = [0, 13, 31]
    keep = list(h.sparsity)
    h.set_sparsity([0.0])
    h.run_step(0, check=check, sample_blocks=48)            # all-keep bootstrap
    h.set_sparsity(keep)
    acc = workloads.accepted_lengths(wl, wl.steps).numpy()
    realized = []
    for t in range(1, wl.steps):
        res = h.run_step(0, accepted=acc[t], check=check, sample_blocks=48)
        realized += [1 - r["kept"] / r["n"] for r in res.values()]
    assert max(realized) <= wl.sparsity + 1e-9              # the union only adds blocks


def test_ragged_multilayer_full_size_sampled():
    """8 layers x 8 requests with contexts drawn in [256K, 1M], per-layer
    budgets allocated from the warm-up miss rates at a 50% global target
    (SPIN v3 record, 摘要): an all-keep step, two warm-up steps, two steps with
    the allocated sparsities; the shortest and the longest request are
    checked on every layer."""
    wl = workloads.config(4, steps=5, warmup_steps=2)
    assert wl.layers == 8 and wl.requests == 8 and min(wl.ctx0) >= 256 * 1024 and max(wl.ctx0) <= 1024 * 1024
    h = Harness(wl)
    ctx = np.array(wl.ctx0)
    check = [int(np.argmin(ctx)), int(np.argmax(ctx))]
    s, miss = run_multilayer(h, check=check, check_warmup=check[:1], sample_blocks=32)
    s = np.asarray(s)
    assert np.all((s >= 0) & (s < 1))
