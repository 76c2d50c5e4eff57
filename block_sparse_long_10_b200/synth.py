"""Seeded synthetic inputs for the QSA layer (shared by tests, smoke and bench).

This module holds input construction only -- shapes, value distributions and
needle planting -- and none of the layer's arithmetic.  Random draws use a
seeded ``torch.Generator`` on the device the tensors are made on; the same
seed on another device gives different (equally distributed) values, so a
test always generates on one device and copies to the other.

Workloads follow the deployed QSA configuration (token budget 2048, micro
block r = 4: "On the Design of Qwen3.8-Next Architecture", token-mixing
paragraph) at 2K (tiny), 32K, 128K and 1M prefill and a 64 x 256K decode
batch.  The pages measure retrieval quality on long-context suites that are
not available here; planted "needle" blocks stand in for them: a block whose
indexer keys are a scaled copy of one query's weighted indexer query, whose
attention keys are a scaled copy of that query's first head in each KV group,
and whose values are a constant pattern.
"""
from __future__ import annotations

import dataclasses
import math

import torch

NEEDLE_ALPHA = 16.0  # indexer-key scale of a planted block
NEEDLE_BETA = 24.0   # attention-key scale of a planted block
NEEDLE_VALUE = 2.0   # constant value pattern of a planted block


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "prefill" or "decode"
    B: int
    T: int             # prefill sequence length, or decode cache length L
    Hq: int
    Hkv: int
    D: int
    Hi: int
    Di: int
    r: int
    budget: int
    seed: int
    needles: int       # prefill: per batch row; decode: per sequence

    @property
    def kb(self) -> int:
        return self.budget // self.r

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def n_blocks(self) -> int:
        return self.T // self.r


WORKLOADS = {
    w.name: w for w in [
        Workload("prefill-2k-tiny", "prefill", 1, 2048, 4, 1, 64, 2, 32, 4, 512, 0, 8),
        Workload("prefill-32k", "prefill", 1, 32768, 16, 2, 128, 4, 64, 4, 2048, 1, 64),
        Workload("prefill-128k", "prefill", 1, 131072, 16, 2, 128, 4, 64, 4, 2048, 2, 256),
        Workload("prefill-1m", "prefill", 1, 1048576, 16, 2, 128, 4, 64, 4, 2048, 3, 1024),
        Workload("decode-256k-b64", "decode", 64, 262144, 16, 2, 128, 4, 64, 4, 2048, 4, 16),
    ]
}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields changed (smaller parity cases)."""
    return dataclasses.replace(w, **changes)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_bf16(shape, g, device) -> torch.Tensor:
    return torch.empty(shape, dtype=torch.bfloat16, device=device).normal_(generator=g)


def _head_weights(shape, g, device) -> torch.Tensor:
    """Per-token indexer head weights: softmax over heads of N(0,1) logits."""
    logits = torch.empty(shape, dtype=torch.float32, device=device).normal_(generator=g)
    return torch.softmax(logits, dim=-1)


def _unit(x: torch.Tensor) -> torch.Tensor:
    x = x.float()
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def _distinct(draw, n: int, taken: set) -> list:
    out = []
    while len(out) < n:
        v = draw()
        if v not in taken:
            taken.add(v)
            out.append(v)
    return out


def make_prefill(w: Workload, device="cpu", seed: int | None = None) -> dict:
    """Q, K, V, indexer q/k, head weights, with needles planted.

    Layouts: q [B,T,Hq,D], k/v [B,T,Hkv,D], q_idx [B,T,Hi,Di], k_idx [B,T,Di]
    (bf16); w [B,T,Hi] fp32.  ``needles`` is a list of (b, t, j) with j the
    planted block for query row t.
    """
    seed = w.seed if seed is None else seed
    g = _gen(seed, device)
    B, T = w.B, w.T
    x = {
        "q": _normal_bf16((B, T, w.Hq, w.D), g, device),
        "k": _normal_bf16((B, T, w.Hkv, w.D), g, device),
        "v": _normal_bf16((B, T, w.Hkv, w.D), g, device),
        "q_idx": _normal_bf16((B, T, w.Hi, w.Di), g, device),
        "k_idx": _normal_bf16((B, T, w.Di), g, device),
        "w": _head_weights((B, T, w.Hi), g, device),
    }
    # Needle rows and blocks: drawn on the host from the same seed.
    hg = torch.Generator().manual_seed(seed + 7919)
    lo = w.r * w.kb
    needles = []
    if w.needles and T > lo:
        for b in range(B):
            rows = _distinct(lambda: int(torch.randint(lo, T, (1,), generator=hg)),
                             min(w.needles, T - lo), set())
            taken: set = set()
            for t in rows:
                c = t // w.r

                def draw_block(c=c):
                    d = float(torch.rand((1,), generator=hg))
                    return min(int(d * c), c - 1)

                if len(taken) >= c:
                    continue
                j = _distinct(draw_block, 1, taken)[0]
                needles.append((b, t, j))
        plant_needles(x, needles, w)
    x["needles"] = needles
    return x


def plant_needles(x: dict, needles, w: Workload) -> None:
    """Overwrite the r tokens of each needle block (see module docstring)."""
    if not needles:
        return
    b = torch.tensor([n[0] for n in needles], device=x["q"].device)
    t = torch.tensor([n[1] for n in needles], device=x["q"].device)
    j = torch.tensor([n[2] for n in needles], device=x["q"].device)
    wq = (x["w"][b, t][..., None] * x["q_idx"][b, t].float()).sum(dim=1)
    key_idx = (NEEDLE_ALPHA * _unit(wq)).to(torch.bfloat16)           # [n, Di]
    qh = x["q"][b, t][:, :: w.G]                                       # [n, Hkv, D]
    key_att = (NEEDLE_BETA * _unit(qh)).to(torch.bfloat16)            # [n, Hkv, D]
    for i in range(w.r):
        tok = j * w.r + i
        x["k_idx"][b, tok] = key_idx
        x["k"][b, tok] = key_att
        x["v"][b, tok] = NEEDLE_VALUE


def make_decode(w: Workload, device="cpu", seed: int | None = None,
                seqlens=None) -> dict:
    """Caches and one new query per sequence, needles planted for that query.

    Layouts: q [B,Hq,D], q_idx [B,Hi,Di] (bf16), w [B,Hi] fp32,
    k_cache/v_cache [B,L,Hkv,D], k_idx_cache [B,L,Di] (bf16), seqlens [B]
    int32 (default: all L).  The new token's K/V are already in the caches.
    """
    seed = w.seed if seed is None else seed
    g = _gen(seed, device)
    B, L = w.B, w.T
    x = {
        "q": _normal_bf16((B, w.Hq, w.D), g, device),
        "q_idx": _normal_bf16((B, w.Hi, w.Di), g, device),
        "w": _head_weights((B, w.Hi), g, device),
    }
    k = torch.empty((B, L, w.Hkv, w.D), dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    ki = torch.empty((B, L, w.Di), dtype=torch.bfloat16, device=device)
    for bb in range(B):  # per sequence: bounded temporaries
        k[bb].normal_(generator=g)
        v[bb].normal_(generator=g)
        ki[bb].normal_(generator=g)
    x["k_cache"], x["v_cache"], x["k_idx_cache"] = k, v, ki
    if seqlens is None:
        seqlens = [L] * B
    x["seqlens"] = torch.tensor(seqlens, dtype=torch.int32, device=device)
    hg = torch.Generator().manual_seed(seed + 7919)
    needles = []
    for bb in range(B):
        c = (int(seqlens[bb]) - 1) // w.r
        if c <= 0 or not w.needles:
            continue
        js = _distinct(lambda: int(torch.randint(0, c, (1,), generator=hg)),
                       min(w.needles, c), set())
        needles += [(bb, j) for j in js]
    if needles:
        b = torch.tensor([n[0] for n in needles], device=device)
        j = torch.tensor([n[1] for n in needles], device=device)
        wq = (x["w"][b][..., None] * x["q_idx"][b].float()).sum(dim=1)
        key_idx = (NEEDLE_ALPHA * _unit(wq)).to(torch.bfloat16)
        key_att = (NEEDLE_BETA * _unit(x["q"][b][:, :: w.G])).to(torch.bfloat16)
        for i in range(w.r):
            tok = j * w.r + i
            k[b, tok] = key_att
            ki[b, tok] = key_idx
            v[b, tok] = NEEDLE_VALUE
    x["needles"] = needles
    return x


def bf16_bits(t: torch.Tensor):
    """A bf16 tensor's raw bit patterns as a host numpy uint16 array."""
    import numpy as np
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
