// Backward of the sparse prefill attention, for the second training stage
// ("用125亿分之6的参数，打平3970亿的旗舰模型", section
// "稀疏注意力：给检索建索引，也得先学会省纸": after the dense distillation the
// indexer and the backbone are trained together on the sparse pattern).
//
// Forward (qsa_sparse_attn_prefill): query t at position p = t, head h of KV
// group g = h / G, attends to S(t) = { 4j + i <= p : j in sel[t] }:
//   o = sum_u P(u) v_g(u),   P = softmax_u(scale q_h . k_g(u)).
// With the selection held fixed, for an output gradient do_h:
//   D_h   = do_h . o_h = sum_u P(u) (do_h . v_g(u))
//   dS(u) = P(u) (do_h . v_g(u) - D_h)
//   dq_h  = scale sum_u dS(u) k_g(u)
//   dk_g(u) += scale dS(u) q_h,   dv_g(u) += P(u) do_h     (over every row and head)
//
// First version, on the CUDA cores: one CTA per (sequence, query, KV group),
// 4 warps over the selected blocks, lanes over the head dimension.  Sweep 1
// gives each head's softmax normaliser and D_h (online, fp32); sweep 2 forms
// dS and accumulates dq in registers (merged across warps through shared
// memory, one writer per element) and adds each key's dk and dv contributions,
// summed over the group's heads, with vector atomics.  The row's q and do sit
// in shared memory as fp32.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {
namespace sbw {

constexpr int R = 4;
constexpr int WARPS = 4;
constexpr unsigned FULL = 0xffffffffu;

QSA_DEVICE float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
    return x;
}

template <int DPL>
QSA_DEVICE void load_bf16(const uint16_t *p, float (&x)[DPL]) {
    if constexpr (DPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        x[0] = bf16_lo(u.x);
        x[1] = bf16_hi(u.x);
        x[2] = bf16_lo(u.y);
        x[3] = bf16_hi(u.y);
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
        x[0] = bf16_lo(u);
        x[1] = bf16_hi(u);
    }
}

template <int DPL>
QSA_DEVICE void atomic_add_vec(float *p, const float (&x)[DPL]) {
    if constexpr (DPL == 4)
        atomicAdd(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
    else
        atomicAdd(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
}

template <int D, int G>
__global__ void __launch_bounds__(WARPS * 32)
    sparse_bwd_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                      const uint16_t *__restrict__ v, const int32_t *__restrict__ sel,
                      const uint16_t *__restrict__ dout, int64_t T, int Hkv, int kb,
                      float scale, float *__restrict__ dq, float *__restrict__ dk,
                      float *__restrict__ dv) {
    constexpr int DPL = D / 32;  // head dims per lane: 2 or 4
    __shared__ __align__(16) float qs[G][D];
    __shared__ __align__(16) float ds_[G][D];
    __shared__ float red[WARPS][G][3];
    __shared__ float stat[G][2];
    __shared__ __align__(16) float dqp[WARPS][G][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t item = blockIdx.x;
    const int g = (int)(item % Hkv);
    const int64_t bt = item / Hkv;
    const int64_t b = bt / T, t = bt % T;
    const int Hq = Hkv * G;
    const int64_t p = t, c = p / R;

    // the row's queries and output gradients of this group's heads, as fp32
    for (int i = threadIdx.x; i < G * D; i += WARPS * 32) {
        const int hh = i / D, d = i % D;
        const int64_t off = ((b * T + t) * Hq + g * G + hh) * D + d;
        qs[hh][d] = __uint_as_float((uint32_t)q[off] << 16);
        ds_[hh][d] = __uint_as_float((uint32_t)dout[off] << 16);
    }
    __syncthreads();

    const int32_t *srow = sel + (b * T + t) * kb;
    const uint16_t *kg = k + b * T * Hkv * D + g * D + lane * DPL;
    const uint16_t *vg = v + b * T * Hkv * D + g * D + lane * DPL;
    float *dkg = dk + b * T * Hkv * D + g * D + lane * DPL;
    float *dvg = dv + b * T * Hkv * D + g * D + lane * DPL;

    // sweep 1: per head, online max / sum of exp(scale q.k) and sum of its
    // weights times do.v
    float m[G], l[G], acc[G];
#pragma unroll
    for (int i = 0; i < G; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
        acc[i] = 0.f;
    }
    for (int e = warp; e < kb; e += WARPS) {
        const int64_t j = srow[e];
        if (j < 0 || j > c) continue;
        for (int ii = 0; ii < R; ++ii) {
            const int64_t u = j * R + ii;
            if (u > p) break;
            float kk[DPL], vv[DPL];
            load_bf16<DPL>(kg + u * Hkv * D, kk);
            load_bf16<DPL>(vg + u * Hkv * D, vv);
#pragma unroll
            for (int i = 0; i < G; ++i) {
                float sq = 0.f, sd = 0.f;
#pragma unroll
                for (int e2 = 0; e2 < DPL; ++e2) {
                    sq = fmaf(qs[i][lane * DPL + e2], kk[e2], sq);
                    sd = fmaf(ds_[i][lane * DPL + e2], vv[e2], sd);
                }
                const float s = warp_sum(sq) * scale;
                const float dp = warp_sum(sd);
                if (s > m[i]) {
                    const float a = expf(m[i] - s);
                    l[i] = l[i] * a + 1.f;
                    acc[i] = acc[i] * a + dp;
                    m[i] = s;
                } else {
                    const float pe = expf(s - m[i]);
                    l[i] += pe;
                    acc[i] = fmaf(pe, dp, acc[i]);
                }
            }
        }
    }
    if (lane == 0)
#pragma unroll
        for (int i = 0; i < G; ++i) {
            red[warp][i][0] = m[i];
            red[warp][i][1] = l[i];
            red[warp][i][2] = acc[i];
        }
    __syncthreads();
    if (threadIdx.x < G) {
        const int i = threadIdx.x;
        float mm = -INFINITY;
        for (int w = 0; w < WARPS; ++w) mm = fmaxf(mm, red[w][i][0]);
        float ll = 0.f, aa = 0.f;
        for (int w = 0; w < WARPS; ++w)
            if (red[w][i][1] > 0.f) {
                const float f = expf(red[w][i][0] - mm);
                ll = fmaf(red[w][i][1], f, ll);
                aa = fmaf(red[w][i][2], f, aa);
            }
        stat[i][0] = ll > 0.f ? mm + logf(ll) : INFINITY;  // log-normaliser (empty: P = 0)
        stat[i][1] = ll > 0.f ? aa / ll : 0.f;             // D_h
    }
    __syncthreads();

    // sweep 2: dS, dq (registers), dk and dv (atomics, summed over the heads)
    float dqa[G][DPL];
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int e2 = 0; e2 < DPL; ++e2) dqa[i][e2] = 0.f;
    for (int e = warp; e < kb; e += WARPS) {
        const int64_t j = srow[e];
        if (j < 0 || j > c) continue;
        for (int ii = 0; ii < R; ++ii) {
            const int64_t u = j * R + ii;
            if (u > p) break;
            float kk[DPL], vv[DPL], dka[DPL], dva[DPL];
            load_bf16<DPL>(kg + u * Hkv * D, kk);
            load_bf16<DPL>(vg + u * Hkv * D, vv);
#pragma unroll
            for (int e2 = 0; e2 < DPL; ++e2) {
                dka[e2] = 0.f;
                dva[e2] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < G; ++i) {
                float sq = 0.f, sd = 0.f;
#pragma unroll
                for (int e2 = 0; e2 < DPL; ++e2) {
                    sq = fmaf(qs[i][lane * DPL + e2], kk[e2], sq);
                    sd = fmaf(ds_[i][lane * DPL + e2], vv[e2], sd);
                }
                const float s = warp_sum(sq) * scale;
                const float dp = warp_sum(sd);
                const float pr = expf(s - stat[i][0]);
                const float dsc = pr * (dp - stat[i][1]);
#pragma unroll
                for (int e2 = 0; e2 < DPL; ++e2) {
                    dqa[i][e2] = fmaf(dsc, kk[e2], dqa[i][e2]);
                    dka[e2] = fmaf(dsc, qs[i][lane * DPL + e2], dka[e2]);
                    dva[e2] = fmaf(pr, ds_[i][lane * DPL + e2], dva[e2]);
                }
            }
#pragma unroll
            for (int e2 = 0; e2 < DPL; ++e2) dka[e2] *= scale;
            atomic_add_vec<DPL>(dkg + u * Hkv * D, dka);
            atomic_add_vec<DPL>(dvg + u * Hkv * D, dva);
        }
    }
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int e2 = 0; e2 < DPL; ++e2) dqp[warp][i][lane * DPL + e2] = dqa[i][e2];
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += WARPS * 32) {
        const int hh = i / D, d = i % D;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) sum += dqp[w][hh][d];
        dq[((b * T + t) * Hq + g * G + hh) * D + d] = scale * sum;
    }
}

template <int D, int G>
static cudaError_t launch(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const int32_t *sel, const uint16_t *dout, int B, int64_t T, int Hkv,
                          int kb, float scale, float *dq, float *dk, float *dv, cudaStream_t s) {
    const int64_t grid = (int64_t)B * T * Hkv;
    sparse_bwd_kernel<D, G><<<(unsigned)grid, WARPS * 32, 0, s>>>(q, k, v, sel, dout, T, Hkv, kb,
                                                                  scale, dq, dk, dv);
    return cudaGetLastError();
}

}  // namespace sbw

cudaError_t launch_sparse_attn_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                        const int32_t *sel, const uint16_t *dout, int B,
                                        int64_t T, int Hq, int Hkv, int D, int kb, float scale,
                                        float *dq, float *dk, float *dv, cudaStream_t s) {
    const size_t kv_bytes = (size_t)B * T * Hkv * D * sizeof(float);
    cudaError_t e = cudaMemsetAsync(dk, 0, kv_bytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, kv_bytes, s);
    if (e != cudaSuccess || B == 0 || T == 0) return e;
    const int G = Hq / Hkv;
#define QSA_SBW(D_, G_) \
    if (D == D_ && G == G_) return sbw::launch<D_, G_>(q, k, v, sel, dout, B, T, Hkv, kb, scale, dq, dk, dv, s);
    QSA_SBW(64, 1) QSA_SBW(64, 2) QSA_SBW(64, 4) QSA_SBW(64, 8)
    QSA_SBW(128, 1) QSA_SBW(128, 2) QSA_SBW(128, 4) QSA_SBW(128, 8)
#undef QSA_SBW
    return cudaErrorInvalidValue;
}

}  // namespace qsa
