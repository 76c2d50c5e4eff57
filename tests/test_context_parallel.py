"""Context-parallel prefill: the zig-zag row plan, the sequence all-gather and
the per-chunk composition.

CPU tests run the host logic on gloo ranks (world size 2) with the oracle
standing in for the kernels, and compare the gathered result with one oracle
call over the whole sequence: the selections, outputs and log-sum-exps must be
identical, since each row's arithmetic does not depend on how rows are split.
The GPU test runs the library's kernels on one rank (two chunks) against one
call over the whole sequence, bit for bit.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_10_b200 import context_parallel as cp
from block_sparse_long_10_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BF = torch.bfloat16
W_SMALL = synth.Workload("cp-small", "prefill", 1, 240, 4, 2, 64, 2, 32, 4, 64, 5, 4)  # 2·W·r | 240 for W = 1, 2, 3


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class OracleOps:
    """The per-chunk steps done by the oracle, writing into the given tensors."""

    def __init__(self, r, budget, scale):
        self.r, self.budget, self.scale = r, budget, scale

    @staticmethod
    def _bits(t):
        return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    def pool(self, k_idx, kp):
        import oracle
        out = oracle.pool(self._bits(k_idx), self.r)
        kp.copy_(torch.from_numpy(out.view(np.int16)).view(BF))

    def index_topk(self, q_idx, w, kp, sel, pos0):
        import oracle
        s, _, _, _ = oracle.index_topk(self._bits(q_idx), w.numpy(), self._bits(kp), self.r,
                                       self.budget, q_pos0=np.array([pos0], np.int64))
        sel.copy_(torch.from_numpy(s).view(sel.shape))

    def attn(self, q, k, v, sel, o, lse, pos0):
        import oracle
        kb = self.budget // self.r
        oo, ll = oracle.attn(self._bits(q), self._bits(k), self._bits(v), self.r, self.scale,
                             sel=sel.reshape(-1, kb).numpy(), q_pos0=np.array([pos0], np.int64))
        o.copy_(torch.from_numpy(oo).view(o.shape).to(BF))
        lse.copy_(torch.from_numpy(ll).view(lse.shape).float())

    def finish(self):
        pass


def _one_shot(x, w):
    """The whole sequence in one oracle call per step."""
    ops = OracleOps(w.r, w.budget, w.scale)
    kp = torch.empty(1, w.T // w.r, w.Di, dtype=BF)
    ops.pool(x["k_idx"], kp)
    sel = torch.empty(1, w.T, w.kb, dtype=torch.int32)
    ops.index_topk(x["q_idx"], x["w"], kp, sel, 0)
    o = torch.empty_like(x["q"])
    lse = torch.empty(1, w.T, w.Hq, dtype=torch.float32)
    ops.attn(x["q"], x["k"], x["v"], sel, o, lse, 0)
    return sel, o, lse


def _local(x, world, rank, r):
    return {n: cp.shard_rows(x[n], world, rank, r) for n in ("q", "k", "v", "q_idx", "w", "k_idx")}


# ------------------------------------------------------------------ plan --

@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_zigzag_plan_covers_every_row_once_with_equal_indexer_work(world):
    r, T = 4, 2 * 4 * 8 * 12                        # a multiple of 2·W·r for every W here
    if T % (2 * world * r):
        T = 2 * world * r * 7
    plan = cp.zigzag_chunks(T, world, r)
    rows = sorted(p for chunks in plan for s, e in chunks for p in range(s, e))
    assert rows == list(range(T))
    for chunks in plan:
        assert all(s % r == 0 and e % r == 0 for s, e in chunks)
    # indexer pairs per rank: each row p scores floor(p / r) candidate blocks
    pairs = [sum(p // r for s, e in chunks for p in range(s, e)) for chunks in plan]
    assert len(set(pairs)) == 1
    assert sum(pairs) == sum(p // r for p in range(T))


def test_zigzag_plan_rejects_unaligned_lengths():
    with pytest.raises(ValueError):
        cp.zigzag_chunks(100, 2, 4)                 # not a multiple of 16
    with pytest.raises(ValueError):
        cp.zigzag_chunks(64, 0, 4)


def test_shard_rows_and_single_rank_gather_round_trip():
    x = torch.arange(1 * 64 * 3).view(1, 64, 3)
    parts = [cp.shard_rows(x, 2, i, 4) for i in range(2)]
    assert parts[0][0, :16].equal(x[0, 0:16]) and parts[0][0, 16:].equal(x[0, 48:64])
    assert parts[1][0, :16].equal(x[0, 16:32]) and parts[1][0, 16:].equal(x[0, 32:48])
    assert cp.gather_sequence(cp.shard_rows(x, 1, 0, 4)).equal(x)


def test_single_rank_context_parallel_equals_one_shot_oracle():
    w = W_SMALL
    x = synth.make_prefill(w, "cpu")
    ref = _one_shot(x, w)
    got = cp.prefill_context_parallel(**_local(x, 1, 0, w.r), r=w.r, budget=w.budget,
                                      scale=w.scale, ops=OracleOps(w.r, w.budget, w.scale))
    assert torch.equal(got["sel"], ref[0])
    assert torch.equal(got["o"].view(torch.int16), ref[1].view(torch.int16))
    assert torch.equal(got["lse"], ref[2])


def test_context_parallel_rejects_batches_and_ragged_rows():
    w = W_SMALL
    x = synth.make_prefill(w, "cpu")
    loc = _local(x, 1, 0, w.r)
    bad = dict(loc, q=torch.cat([loc["q"], loc["q"]], 0))
    with pytest.raises(ValueError):
        cp.prefill_context_parallel(**bad, ops=OracleOps(w.r, w.budget, w.scale))
    bad = dict(loc, k=loc["k"][:, :-4])
    with pytest.raises(ValueError):
        cp.prefill_context_parallel(**bad, ops=OracleOps(w.r, w.budget, w.scale))


# ------------------------------------------------------------ two ranks --

def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="2")
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W_SMALL
        x = synth.make_prefill(w, "cpu")              # same seed: same inputs on every rank
        loc = _local(x, world, rank, w.r)
        k_back = cp.gather_sequence(loc["k"])
        kp_rows = torch.empty(1, loc["k_idx"].shape[1] // w.r, w.Di, dtype=BF)
        OracleOps(w.r, w.budget, w.scale).pool(loc["k_idx"], kp_rows)
        kp_back = cp.gather_sequence(kp_rows)
        kp_full = torch.empty(1, w.n_blocks, w.Di, dtype=BF)
        OracleOps(w.r, w.budget, w.scale).pool(x["k_idx"], kp_full)
        got = cp.prefill_context_parallel(**loc, r=w.r, budget=w.budget, scale=w.scale,
                                          ops=OracleOps(w.r, w.budget, w.scale))
        full = {n: cp.gather_sequence(t) for n, t in got.items()}
        res = {"k_round_trip": bool(torch.equal(k_back, x["k"])),
               "pooled_in_place": bool(torch.equal(kp_back.view(torch.int16),
                                                   kp_full.view(torch.int16)))}
        if rank == 0:
            sel, o, lse = _one_shot(x, w)
            res.update(sel=bool(torch.equal(full["sel"], sel)),
                       o=bool(torch.equal(full["o"].view(torch.int16), o.view(torch.int16))),
                       lse=bool(torch.equal(full["lse"], lse)),
                       needles=all(j in full["sel"][0, t].tolist() for _, t, j in x["needles"]))
        q.put((rank, res))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_multi_rank_context_parallel_equals_one_shot_oracle_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    for r in range(1, world):
        assert res[r] == {"k_round_trip": True, "pooled_in_place": True}
    assert res[0] == {"k_round_trip": True, "pooled_in_place": True, "sel": True, "o": True,
                      "lse": True, "needles": True}


# ------------------------------------------------------------------- GPU --

@pytest.mark.gpu
def test_context_parallel_kernels_equal_one_call_gpu():
    """One rank, two zig-zag chunks (rows 0..C-1 and C..2C-1) through the
    library's kernels: identical to one call over the whole sequence."""
    import block_sparse_long_10_b200 as qsa
    dev = "cuda"
    w = synth.Workload("cp-gpu", "prefill", 1, 4096, 8, 2, 128, 4, 64, 4, 512, 21, 8)
    x = synth.make_prefill(w, dev)
    kp = torch.empty(1, w.n_blocks, w.Di, dtype=BF, device=dev)
    qsa.qsa_pool(x["k_idx"], kp, w.r)
    sel = torch.empty(1, w.T, w.kb, dtype=torch.int32, device=dev)
    ws = qsa.workspace(qsa.qsa_index_topk_workspace_size(1, w.T, w.n_blocks, w.Hi, w.Di, w.r, w.budget))
    qsa.qsa_index_topk(x["q_idx"], x["w"], kp, sel, ws, w.r, w.budget)
    o = torch.empty_like(x["q"])
    lse = torch.empty(1, w.T, w.Hq, dtype=torch.float32, device=dev)
    qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, o, w.r, w.budget, w.scale, lse=lse)
    assert qsa.qsa_check_device_status(ws) == 0
    got = cp.prefill_context_parallel(**_local(x, 1, 0, w.r), r=w.r, budget=w.budget,
                                      scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(got["sel"], sel)
    assert torch.equal(got["o"].view(torch.int16), o.view(torch.int16))
    assert torch.equal(got["lse"], lse)


# ------------------------------------------------------ a rank that dies --

def _dying_worker(rank, world, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="1")
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    dist.barrier()  # both ranks are up
    if rank == 1:
        os._exit(0)  # leaves between steps, before the all-gather, without a word
    w = W_SMALL
    x = synth.make_prefill(w, "cpu")
    try:
        cp.prefill_context_parallel(**_local(x, world, rank, w.r), r=w.r, budget=w.budget,
                                    scale=w.scale, ops=OracleOps(w.r, w.budget, w.scale))
        q.put((rank, "completed"))
    except Exception as exc:  # the collective reports the missing rank
        q.put((rank, type(exc).__name__))
    q.close()
    q.join_thread()  # the result reaches the parent before this process ends
    os._exit(0)


def test_a_rank_that_leaves_fails_the_survivors_collective_instead_of_hanging():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:  # only processes this test started
        p.kill()
    assert not alive
    rank, outcome = q.get(timeout=10)
    assert rank == 0 and outcome != "completed"
