"""Context-sharded SPIN (indexer_sparse_attention_b200.sharded) on gloo ranks
on the CPU: each request's slots are split over 2 or 3 ranks, the block scores
and top-k candidates are all-gathered, and the score and D-offset halos cross
rank boundaries.  The per-shard arithmetic is the oracle's, applied to what
each rank owns; every step's mask and top-k, and the final V and D, must equal
the unsharded oracle's bit for bit (one row per step, MTP rows with the
row-local union and prefix-valid replay over drawn accepted lengths, and the
row-0 policy)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleShardBackend:
    """Shard arithmetic from the oracle's functions."""

    def __init__(self, wl, pages, qw, sparsity, policy):
        import oracle
        self.o, self.wl, self.pages, self.qw, self.s, self.policy = oracle, wl, pages, qw, sparsity, policy
        self.nmax = wl.max_blocks
        self.cur = None  # (step inputs per request) set before each step

    def predict(self, q, V, D, ctx, rows):
        return self.o.predict_pool(V, D, ctx, rows, self.wl.b, self.nmax)

    def select(self, q, S, ctx, rows, step):
        return self.o.select(S, ctx, rows, self.wl.b, self.s, self.wl.gamma, self.wl.seed, q, 0, step, self.policy)

    def score(self, q, mask, ctx, rows):
        qs, ws = self.cur[q]
        q8, wq, _ = self.o.quantize_q(qs, ws)
        keys, ks, ident = self.pages[q]
        return self.o.score_fp8(keys, ks, ident, q8, wq, ctx, mask, self.nmax * self.wl.b)

    def ema(self, V, D, s32, mask, ctx, n_upd):
        self.o.ema_update(V, D, s32, mask, ctx, n_upd, self.wl.b, self.wl.alpha)


def _scenarios():
    import workloads
    base = dict(requests=2, ctx0=(3000 - 40, 1777), spare_slots=8, sparsity=0.5)
    return [
        ("one row", workloads.config(2, steps=6, **base), None, 0),
        ("MTP union + prefix-valid", workloads.config(3, steps=6, **base), "drawn", 0),
        ("MTP row 0", workloads.config(3, steps=5, mtp_policy=1, **base), "drawn", 1),
    ]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads
        from indexer_sparse_attention_b200.sharded import ShardLayout, ShardedSpin
        oracle.build()
        res = {}
        for name, wl, acc_kind, policy in _scenarios():
            Q, R, b, nmax = wl.requests, wl.rows, wl.b, wl.max_blocks
            cache = workloads.make_key_cache(wl, 0, "cpu")
            pages = [tuple(x.numpy() for x in workloads.request_pages(cache, q)) for q in range(Q)]
            qall, wall = workloads.make_queries(wl, 0, wl.steps * R + R, "cpu")
            acc = (workloads.accepted_lengths(wl, wl.steps).numpy() if acc_kind else
                   np.full((wl.steps, Q), R, np.int32))
            # unsharded oracle (fp64 scores drive top-k and state)
            slot_stride = nmax * b
            Vr = [np.full(slot_stride, np.inf, np.float32) for _ in range(Q)]
            Dr = [np.full(slot_stride, -np.inf, np.float32) for _ in range(Q)]
            committed = np.array(wl.ctx0, np.int64)
            backend = OracleShardBackend(wl, pages, None, 0.0, policy)
            shard = ShardedSpin(backend, ShardLayout(wl.max_slots, b, world), R, wl.topk, wl.ctx0, mtp_row0=bool(policy))
            same_mask = same_topk = 0
            for t in range(wl.steps):
                s = 0.0 if t == 0 else wl.sparsity
                a_t = acc[t] if t > 0 else np.full(Q, R, np.int32)
                cur = []
                for q in range(Q):
                    pos0 = int(committed[q] - wl.ctx0[q])
                    cur.append((qall[q, pos0:pos0 + R].float().numpy().astype(np.float64),
                                wall[q, pos0:pos0 + R].numpy()))
                ref_masks, ref_topk = [], []
                for q in range(Q):
                    keys, ks, ident = pages[q]
                    o = oracle.decode_step_request(
                        V=Vr[q], D=Dr[q], ctx_len=int(committed[q] + 1), rows=R, b=b, sparsity=np.float32(s),
                        gamma=wl.gamma, alpha=wl.alpha, seed=wl.seed, request=q, layer=0, step=t, topk=wl.topk,
                        q=cur[q][0], w=cur[q][1], keys=keys, kscale=ks, block_table=ident, key_fp8=True,
                        accepted=int(a_t[q]), n_stride=nmax, mtp_policy=policy)
                    ref_masks.append(o["mask"])
                    ref_topk.append(o["topk"])
                committed = committed + a_t
                backend.s = np.float32(s)
                backend.cur = cur
                masks, topk = shard.step(R, t, accepted=a_t)
                same_mask += all(np.array_equal(masks[q], ref_masks[q]) for q in range(Q))
                same_topk += all(np.array_equal(topk[q], ref_topk[q]) for q in range(Q))
            V, D = shard.gather_state()
            vis = [int(c) for c in committed]           # slots 0..C-1 exist after the last step
            v_ok = all(np.array_equal(V[q, :vis[q]].view(np.uint32), Vr[q][:vis[q]].view(np.uint32))
                       for q in range(Q))
            d_ok = all(np.array_equal(D[q, :vis[q]].view(np.uint32), Dr[q][:vis[q]].view(np.uint32))
                       for q in range(Q))
            res[name] = (same_mask, same_topk, wl.steps, v_ok, d_ok)
        out[rank] = res
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_steps_equal_the_unsharded_oracle(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert set(res) == set(range(world))
    for rank, per in res.items():
        for name, (same_mask, same_topk, steps, v_ok, d_ok) in per.items():
            assert same_mask == steps, (rank, name, "masks", same_mask, steps)
            assert same_topk == steps, (rank, name, "top-k", same_topk, steps)
            assert v_ok and d_ok, (rank, name, "state", v_ok, d_ok)
