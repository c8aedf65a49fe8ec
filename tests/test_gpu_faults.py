"""Device-side failure detection without a GPU fault: the tensor-core score
kernel's bounded waits.  A test hook makes CTA 0 withhold the copy of its
first key stage, so a wait that nothing will satisfy runs out after its 2 s
limit; the kernel must report SPIN_ETIMEOUT through the device error word,
drain its copies, free its tensor memory and return -- and the context must
stay usable for the next, correct step."""
import time

import pytest
import torch

import indexer_sparse_attention_b200 as isa
import oracle
import workloads
from lockstep import Harness

pytestmark = pytest.mark.gpu


def test_withheld_stage_times_out_and_context_survives():
    from indexer_sparse_attention_b200 import build
    build.build()
    oracle.build()
    wl = workloads.config(2, requests=4, ctx0=(30000, 20000, 9000, 64 * 300), steps=4)
    h = Harness(wl, score_kernel=isa.SPIN_SCORE_TCGEN05)
    h.set_sparsity([0.0])
    h.run_step(0, check=[0])
    h.set_sparsity([0.5])
    qstep, wstep, ctx = h.step_inputs(0, 1)
    cache = h.caches[0]
    topk = torch.empty((wl.requests, 1, wl.topk), dtype=torch.int32, device="cuda")
    isa.spin_set_fault_injection(h.st, 1)
    t0 = time.time()
    isa.spin_decode_step(h.st, 0, 1, 1, cache.keys, cache.kscale, cache.block_table, qstep, wstep, ctx, False,
                         h.mask, topk, h.scores)
    status, word = isa.spin_get_error(h.st)
    elapsed = time.time() - t0
    assert status == 5 and word & 8, (status, hex(word))     # SPIN_ETIMEOUT, ERR_TIMEOUT
    assert elapsed < 30
    # the hook fires once; the next steps run normally and match the oracle
    h.committed += 1
    h.step_index = 2
    for _ in range(2):
        h.run_step(0, check=[0, 1, 2, 3])
