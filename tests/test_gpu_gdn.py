"""GPU parity of the gated delta rule kernels (qsa_gdn_prefill / decode)
against the oracle's recurrence (oracle/gdn.py), through the C ABI.

The kernels run the recurrence in fp32 on exact bf16 inputs; over T tokens the
rounding of each step's rank-1 update adds up to a relative error of order
T * 1e-7 (unit keys and gates <= 1 keep the state bounded).  The bar:
|gpu - ref| <= 1e-3 * max(|ref|, 1e-3 * max|ref|) per tensor.
"""
import numpy as np
import pytest
import torch

import block_sparse_long_10_b200 as qsa
from oracle import gdn

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _close(name, gpu, ref):
    assert gpu.shape == ref.shape and np.isfinite(gpu).all(), name
    floor = 1e-3 * max(np.abs(ref).max(), 1e-30)
    bad = np.abs(gpu - ref) > 1e-3 * np.maximum(np.abs(ref), floor)
    assert not bad.any(), (name, int(bad.sum()), float(np.abs(gpu - ref).max()))


def _inputs(B, T, H, dk, dv, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    q = torch.randn(B, T, H, dk, generator=g, device=DEV).bfloat16()
    k = torch.randn(B, T, H, dk, generator=g, device=DEV)
    k = (k / k.norm(dim=-1, keepdim=True)).bfloat16()
    v = torch.randn(B, T, H, dv, generator=g, device=DEV).bfloat16()
    alpha = 0.9 + 0.1 * torch.rand(B, T, H, generator=g, device=DEV)
    beta = torch.rand(B, T, H, generator=g, device=DEV)
    s0 = torch.randn(B, H, dv, dk, generator=g, device=DEV) * 0.1
    return q, k, v, alpha, beta, s0


@pytest.mark.parametrize("B,T,H,dk,dv", [(2, 300, 3, 128, 128), (1, 1000, 2, 64, 64),
                                         (1, 77, 4, 128, 64), (2, 1, 2, 64, 128)])
def test_gdn_prefill_matches_recurrence(B, T, H, dk, dv):
    q, k, v, a, b, s0 = _inputs(B, T, H, dk, dv, seed=T)
    o = torch.full((B, T, H, dv), float("nan"), device=DEV)
    s1 = torch.full((B, H, dv, dk), float("nan"), device=DEV)
    qsa.qsa_gdn_prefill(q, k, v, a, b, o, s1, state_in=s0)
    torch.cuda.synchronize()
    o_ref, s_ref = gdn.gdn_recurrent(_bits(q), _bits(k), _bits(v), a.cpu().numpy(),
                                     b.cpu().numpy(), s0.cpu().numpy())
    _close("o", o.cpu().numpy().astype(np.float64), o_ref)
    _close("state", s1.cpu().numpy().astype(np.float64), s_ref)


def test_gdn_zero_initial_state_and_empty_prefill():
    q, k, v, a, b, _ = _inputs(1, 50, 2, 64, 64, seed=3)
    o = torch.empty(1, 50, 2, 64, device=DEV)
    s1 = torch.full((1, 2, 64, 64), float("nan"), device=DEV)
    qsa.qsa_gdn_prefill(q, k, v, a, b, o, s1)
    o_ref, s_ref = gdn.gdn_recurrent(_bits(q), _bits(k), _bits(v), a.cpu().numpy(), b.cpu().numpy())
    _close("o", o.cpu().numpy().astype(np.float64), o_ref)
    s2 = torch.full_like(s1, float("nan"))
    qsa.qsa_gdn_prefill(q[:, :0], k[:, :0], v[:, :0], a[:, :0], b[:, :0], o[:, :0], s2, state_in=s1)
    torch.cuda.synchronize()
    assert torch.equal(s2, s1)


def test_gdn_decode_continues_the_prefill():
    B, T, H, dk, dv = 3, 40, 2, 128, 128
    q, k, v, a, b, s0 = _inputs(B, T, H, dk, dv, seed=9)
    st = torch.empty(B, H, dv, dk, device=DEV)
    o = torch.empty(B, 30, H, dv, device=DEV)
    qsa.qsa_gdn_prefill(q[:, :30].contiguous(), k[:, :30].contiguous(), v[:, :30].contiguous(),
                        a[:, :30].contiguous(), b[:, :30].contiguous(), o, st, state_in=s0)
    outs = []
    for t in range(30, T):
        od = torch.empty(B, H, dv, device=DEV)
        qsa.qsa_gdn_decode(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(),
                           a[:, t].contiguous(), b[:, t].contiguous(), st, od)
        outs.append(od)
    torch.cuda.synchronize()
    o_ref, s_ref = gdn.gdn_recurrent(_bits(q), _bits(k), _bits(v), a.cpu().numpy(),
                                     b.cpu().numpy(), s0.cpu().numpy())
    _close("decode o", torch.stack(outs, 1).cpu().numpy().astype(np.float64), o_ref[:, 30:])
    _close("state", st.cpu().numpy().astype(np.float64), s_ref)


def _close_chunked(name, gpu, ref):
    """The chunked form runs its state products on the tensor cores with each fp32
    operand split into bf16 high and low parts (hi.hi + hi.lo + lo.hi): every
    product carries a relative error of about 2^-16, so an element that is a sum
    of such products with cancellation is off by up to about 1e-5 of the largest
    output, not 1e-6 as the fp32 recurrence.  Same relative bar, that floor."""
    assert gpu.shape == ref.shape and np.isfinite(gpu).all(), name
    floor = 1e-2 * max(np.abs(ref).max(), 1e-30)
    bad = np.abs(gpu - ref) > 1e-3 * np.maximum(np.abs(ref), floor)
    assert not bad.any(), (name, int(bad.sum()), float(np.abs(gpu - ref).max()))


def _chunked(q, k, v, a, b, s0=None):
    B, T, H, dk = k.shape
    dv = v.shape[3]
    o = torch.full((B, T, H, dv), float("nan"), device=DEV)
    s1 = torch.full((B, H, dv, dk), float("nan"), device=DEV)
    ws = qsa.workspace(qsa.qsa_gdn_prefill_chunked_workspace_size(B, T, H, dk, dv))
    qsa.qsa_gdn_prefill_chunked(q, k, v, a, b, o, s1, ws, state_in=s0)
    torch.cuda.synchronize()
    return o, s1


@pytest.mark.parametrize("B,T,H,dk,dv", [(2, 300, 3, 128, 128), (1, 1000, 2, 64, 64),
                                         (1, 77, 4, 128, 64), (2, 1, 2, 64, 128),
                                         (1, 128, 2, 128, 128), (2, 640, 1, 64, 128)])
def test_gdn_prefill_chunked_matches_recurrence(B, T, H, dk, dv):
    """The chunked form (64-token chunks: full chunks, a partial last chunk, a
    single token) against the oracle's token-by-token recurrence."""
    q, k, v, a, b, s0 = _inputs(B, T, H, dk, dv, seed=T + 1)
    o, s1 = _chunked(q, k, v, a, b, s0)
    o_ref, s_ref = gdn.gdn_recurrent(_bits(q), _bits(k), _bits(v), a.cpu().numpy(),
                                     b.cpu().numpy(), s0.cpu().numpy())
    _close_chunked("o", o.cpu().numpy().astype(np.float64), o_ref)
    _close_chunked("state", s1.cpu().numpy().astype(np.float64), s_ref)


def test_gdn_prefill_chunked_gates_at_their_ends():
    """Decay gates of exactly 0 (the memory is wiped inside a chunk) and 1, write
    gates of 0 and 1, no initial state; then an empty prefill copies the state."""
    B, T, H, dk, dv = 1, 200, 2, 64, 64
    q, k, v, a, b, _ = _inputs(B, T, H, dk, dv, seed=11)
    a[:, 70] = 0.0
    a[:, 130:140] = 1.0
    b[:, 20:30] = 0.0
    b[:, 150] = 1.0
    o, s1 = _chunked(q, k, v, a, b)
    o_ref, s_ref = gdn.gdn_recurrent(_bits(q), _bits(k), _bits(v), a.cpu().numpy(),
                                     b.cpu().numpy())
    _close_chunked("o", o.cpu().numpy().astype(np.float64), o_ref)
    _close_chunked("state", s1.cpu().numpy().astype(np.float64), s_ref)
    s2 = torch.full_like(s1, float("nan"))
    ws = qsa.workspace(qsa.qsa_gdn_prefill_chunked_workspace_size(B, 0, H, dk, dv))
    qsa.qsa_gdn_prefill_chunked(q[:, :0], k[:, :0], v[:, :0], a[:, :0], b[:, :0], o[:, :0], s2,
                                ws, state_in=s1)
    torch.cuda.synchronize()
    assert torch.equal(s2, s1)
