"""Context-parallel QSA prefill: one long sequence's query rows split across GPUs.

Once the whole causal prefix of K, V and the pooled indexer keys is in memory,
every query row of the QSA layer is independent of every other: its indexer
scores, its top-k selection and its attention over the expanded tokens read
nothing another row writes ("On the Design of Qwen3.8-Next Architecture",
token-mixing paragraph: the indexer scores micro-blocks, the kept blocks are
expanded for the attention; article "用125亿分之6的参数，打平3970亿的旗舰模型",
section "稀疏注意力：给检索建索引，也得先学会省纸").  So a sequence too long
for one GPU's time budget is split by query rows, one process per GPU:

* Row assignment.  The indexer's work on row p grows with p (it scores every
  complete block before p), while the attention's is flat once the prefix
  passes the token budget.  The sequence is cut into 2W equal chunks of C rows
  and rank i owns chunks i and 2W-1-i (zig-zag), so every rank scores the same
  number of (row, block) pairs.  C is a multiple of the micro-block size r, so
  no micro-block straddles two ranks.
* Each rank holds, for its own rows only, every per-token input: q, k, v,
  q_idx, w, k_idx (what a sequence-sharded projection leaves behind), laid out
  as chunk i followed by chunk 2W-1-i.
* Step 1 pools the rank's own indexer keys (``qsa_pool``).
* Step 2 is the one data-path collective: an all-gather of K, V and the pooled
  keys into whole-sequence buffers (NCCL over NVLink on GPUs).  The pooled keys
  are gathered rather than the raw indexer keys: r times fewer bytes.
* Step 3 runs, per owned chunk, ``qsa_index_topk`` and
  ``qsa_sparse_attn_prefill`` with ``q_pos0`` = the chunk's first position.
  Outputs stay sharded, in the rank's row order.

Only batch 1 is split this way: a batch of sequences shards by sequence, with
no collective at all.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (qsa_index_topk, qsa_index_topk_workspace_size, qsa_pool,
               qsa_sparse_attn_prefill, qsa_check_device_status, workspace, QSAError)

__all__ = ["zigzag_chunks", "shard_rows", "gather_sequence", "prefill_context_parallel",
           "LibraryOps"]


def _world(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


def zigzag_chunks(T: int, world: int, r: int = 4) -> list:
    """Row ranges owned by each rank: ``[[(s, e), (s, e)], ...]`` (rank i owns
    chunks i and 2W-1-i of 2W equal chunks).  T must be a multiple of 2·W·r."""
    if world < 1 or r < 1 or T < 0 or T % (2 * world * r):
        raise ValueError(f"T={T} must be a multiple of 2 * world * r = {2 * world * r}")
    C = T // (2 * world)
    return [[(i * C, (i + 1) * C), ((2 * world - 1 - i) * C, (2 * world - i) * C)]
            for i in range(world)]


def shard_rows(x: torch.Tensor, world: int, rank: int, r: int = 4) -> torch.Tensor:
    """The rows of a whole-sequence tensor [1, T, ...] that ``rank`` owns, as
    one contiguous tensor [1, 2C, ...] (its first chunk, then its second)."""
    (a0, a1), (b0, b1) = zigzag_chunks(x.shape[1], world, r)[rank]
    return torch.cat([x[:, a0:a1], x[:, b0:b1]], dim=1).contiguous()


def gather_sequence(local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's rows [1, 2C, ...] back into sequence order
    [1, 2·W·C, ...].

    The ranks' first chunks are chunks 0..W-1 in rank order, so they land in
    place in one all-gather.  Their second chunks are chunks 2W-1..W, the
    reverse of rank order: they are gathered into a staging buffer and copied
    into place.  Without an initialised process group (one rank) the local
    rows already are the whole sequence.
    """
    if local.dim() < 2 or local.shape[0] != 1 or local.shape[1] % 2:
        raise ValueError("local rows must be [1, 2C, ...]")
    world, _ = _world(group)
    if world == 1:
        return local.contiguous()
    C = local.shape[1] // 2
    tail = tuple(local.shape[2:])
    full = local.new_empty((1, 2 * world * C) + tail)
    front = full[:, : world * C]                       # contiguous: batch 1
    dist.all_gather_into_tensor(front.reshape(-1), local[:, :C].contiguous().reshape(-1),
                                group=group)
    stage = local.new_empty((world, C) + tail)
    dist.all_gather_into_tensor(stage.reshape(-1), local[:, C:].contiguous().reshape(-1),
                                group=group)
    for i in range(world):
        c = 2 * world - 1 - i
        full[0, c * C:(c + 1) * C].copy_(stage[i])
    return full


class LibraryOps:
    """The per-chunk steps on the library's CUDA kernels (the product path).

    Each call writes into the output tensors it is given.  One indexer
    workspace is kept and grown as needed; ``finish`` reads its device status
    word and raises ``QSAError`` on a recorded device error.
    """

    def __init__(self, r: int, budget: int, scale: float):
        self.r, self.budget, self.scale = r, budget, scale
        self._ws = None

    def pool(self, k_idx, kp):
        qsa_pool(k_idx, kp, self.r)

    def index_topk(self, q_idx, w, kp, sel, pos0: int):
        B, Tq, Hi, Di = q_idx.shape
        need = qsa_index_topk_workspace_size(B, Tq, kp.shape[1], Hi, Di, self.r, self.budget)
        if self._ws is None or self._ws.numel() < need:
            if self._ws is not None:
                self.finish()
            self._ws = workspace(need, q_idx.device)
        p0 = torch.full((B,), pos0, dtype=torch.int64, device=q_idx.device)
        qsa_index_topk(q_idx, w, kp, sel, self._ws, self.r, self.budget, q_pos0=p0)

    def attn(self, q, k, v, sel, o, lse, pos0: int):
        p0 = torch.full((q.shape[0],), pos0, dtype=torch.int64, device=q.device)
        qsa_sparse_attn_prefill(q, k, v, sel, o, self.r, self.budget, self.scale, q_pos0=p0,
                                lse=lse)

    def finish(self):
        if self._ws is not None:
            rc = qsa_check_device_status(self._ws)
            if rc != 0:
                raise QSAError(rc, "context-parallel prefill")


def prefill_context_parallel(q, k, v, q_idx, w, k_idx, r: int = 4, budget: int = 2048,
                             scale: float | None = None, group=None, ops=None) -> dict:
    """QSA prefill of this rank's rows of one sequence split across the group.

    Inputs are this rank's rows (``shard_rows`` order): q [1, 2C, Hq, D],
    k/v [1, 2C, Hkv, D], q_idx [1, 2C, Hi, Di], w [1, 2C, Hi], k_idx [1, 2C, Di];
    the whole sequence is T = 2·W·C tokens with C a multiple of r.  Returns
    ``{"sel", "o", "lse"}`` for the same rows: sel [1, 2C, budget/r] int32,
    o [1, 2C, Hq, D] bf16, lse [1, 2C, Hq] fp32.  ``ops`` carries out the
    per-chunk steps (``LibraryOps``, the library's kernels, unless given).
    """
    world, rank = _world(group)
    if q.dim() != 4 or q.shape[0] != 1:
        raise ValueError("context-parallel prefill splits one sequence: q must be [1, 2C, Hq, D]")
    n_local = q.shape[1]
    for t, name in ((k, "k"), (v, "v"), (q_idx, "q_idx"), (w, "w"), (k_idx, "k_idx")):
        if t.shape[0] != 1 or t.shape[1] != n_local:
            raise ValueError(f"{name} must hold the same {n_local} rows as q")
    T = world * n_local
    plan = zigzag_chunks(T, world, r)[rank]
    C = n_local // 2
    D = q.shape[-1]
    if scale is None:
        scale = D ** -0.5
    ops = LibraryOps(r, budget, scale) if ops is None else ops

    # Step 1: pool this rank's own indexer keys (each chunk is whole blocks).
    kp_local = k_idx.new_empty((1, n_local // r, k_idx.shape[-1]))
    ops.pool(k_idx, kp_local)

    # Step 2: the whole causal prefix of K, V and the pooled keys, in sequence order.
    k_full = gather_sequence(k, group)
    v_full = gather_sequence(v, group)
    kp_full = gather_sequence(kp_local, group)

    # Step 3: selection and attention per owned chunk, at its absolute position.
    kb = budget // r
    sel = torch.empty((1, n_local, kb), dtype=torch.int32, device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((1, n_local, q.shape[2]), dtype=torch.float32, device=q.device)
    for slot, (s, e) in enumerate(plan):
        rows = slice(slot * C, (slot + 1) * C)
        ops.index_topk(q_idx[:, rows], w[:, rows], kp_full[:, : e // r], sel[:, rows], s)
        ops.attn(q[:, rows], k_full[:, :e], v_full[:, :e], sel[:, rows], o[:, rows],
                 lse[:, rows], s)
    ops.finish()
    return {"sel": sel, "o": o, "lse": lse}
