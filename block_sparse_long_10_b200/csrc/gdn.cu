// Gated DeltaNet token mixing: the gated delta rule, prefill and decode
// ("用125亿分之6的参数，打平3970亿的旗舰模型", hybrid token-mixing section: three
// GDN layers for every global-attention layer; GDN keeps a matrix state, writes
// the error between the token's information and what the memory holds for it,
// under a decay gate and a write gate.  "On the Design of Qwen3.8-Next
// Architecture", token-mixing paragraph: a fixed-size recurrent state with a
// decay gate and delta writes, so decoding needs no growing cache).
//
// Per (sequence, head), state S in R^{DV x DK} (fp32), per token t:
//   S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T,   o_t = S_t q_t.
//
// First version: one CTA per (sequence, head) holds the whole state in
// registers (256 threads, DV rows, 256 / DV threads per row, DK * DV / 256
// columns per thread) and walks the tokens in order; a token's k, q, v are
// staged in shared memory (double-buffered, one barrier per token), the row
// dot products S k and S q are reduced over the row's threads by shuffles.
// Decode is the same step for one token with the state read from and written
// back to memory.  (The chunked tensor-core form of the rule is the next
// version; this one is the exact recurrence.)
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {
namespace gdn {

constexpr int THREADS = 256;
constexpr unsigned FULL = 0xffffffffu;

template <int DK, int DV>
struct Cfg {
    static constexpr int TPR = THREADS / DV;     // threads per state row
    static constexpr int COLS = DK / TPR;        // state columns per thread
    static_assert(TPR >= 1 && TPR <= 32 && (TPR & (TPR - 1)) == 0, "row split");
    static_assert(COLS % 4 == 0, "vector columns");
};

template <int TPR>
QSA_DEVICE float row_sum(float x) {
#pragma unroll
    for (int off = 1; off < TPR; off <<= 1) x += __shfl_xor_sync(FULL, x, off);
    return x;
}

// One token's update of this thread's slice of the state, and its share of o.
template <int DK, int DV>
QSA_DEVICE float step(float (&S)[Cfg<DK, DV>::COLS], const float *ks, const float *qs,
                      float v_row, float alpha, float beta, int c0) {
    using C = Cfg<DK, DV>;
    float sk = 0.f;
#pragma unroll
    for (int c = 0; c < C::COLS; ++c) sk = fmaf(S[c], ks[c0 + c], sk);
    sk = row_sum<C::TPR>(sk);
    const float coef = beta * (v_row - alpha * sk);
    float so = 0.f;
#pragma unroll
    for (int c = 0; c < C::COLS; ++c) {
        S[c] = fmaf(alpha, S[c], coef * ks[c0 + c]);
        so = fmaf(S[c], qs[c0 + c], so);
    }
    return row_sum<C::TPR>(so);
}

template <int DK, int DV>
__global__ void __launch_bounds__(THREADS)
    gdn_prefill_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                       const uint16_t *__restrict__ v, const float *__restrict__ alpha,
                       const float *__restrict__ beta, const float *__restrict__ state_in,
                       int64_t T, int H, float *__restrict__ o, float *__restrict__ state_out) {
    using C = Cfg<DK, DV>;
    __shared__ __align__(16) float ks[2][DK];
    __shared__ __align__(16) float qs[2][DK];
    __shared__ float vs[2][DV];
    __shared__ float gs[2][2];
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;  // b * H + h
    const int64_t b = bh / H;
    const int h = (int)(bh % H);
    const int row = tid / C::TPR, c0 = (tid % C::TPR) * C::COLS;

    float S[C::COLS];
    const float *sin = state_in ? state_in + (bh * DV + row) * DK + c0 : nullptr;
#pragma unroll
    for (int c = 0; c < C::COLS; ++c) S[c] = sin ? sin[c] : 0.f;

    auto stage = [&](int64_t t, int buf) {
        const int64_t tok = (b * T + t) * H + h;
        for (int i = tid; i < DK; i += THREADS) {
            ks[buf][i] = __uint_as_float((uint32_t)k[tok * DK + i] << 16);
            qs[buf][i] = __uint_as_float((uint32_t)q[tok * DK + i] << 16);
        }
        for (int i = tid; i < DV; i += THREADS) vs[buf][i] = __uint_as_float((uint32_t)v[tok * DV + i] << 16);
        if (tid == 0) {
            gs[buf][0] = alpha[tok];
            gs[buf][1] = beta[tok];
        }
    };
    if (T > 0) stage(0, 0);
    __syncthreads();
    for (int64_t t = 0; t < T; ++t) {
        const int buf = (int)(t & 1);
        if (t + 1 < T) stage(t + 1, buf ^ 1);  // the other buffer was last read at t - 1
        const float ot = step<DK, DV>(S, ks[buf], qs[buf], vs[buf][row], gs[buf][0],
                                      gs[buf][1], c0);
        if (tid % C::TPR == 0) o[((b * T + t) * H + h) * DV + row] = ot;
        __syncthreads();
    }
    float *sout = state_out + (bh * DV + row) * DK + c0;
#pragma unroll
    for (int c = 0; c < C::COLS; ++c) sout[c] = S[c];
}

template <int DK, int DV>
__global__ void __launch_bounds__(THREADS)
    gdn_decode_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                      const uint16_t *__restrict__ v, const float *__restrict__ alpha,
                      const float *__restrict__ beta, float *__restrict__ state,
                      float *__restrict__ o) {
    using C = Cfg<DK, DV>;
    __shared__ __align__(16) float ks[DK];
    __shared__ __align__(16) float qs[DK];
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int row = tid / C::TPR, c0 = (tid % C::TPR) * C::COLS;
    for (int i = tid; i < DK; i += THREADS) {
        ks[i] = __uint_as_float((uint32_t)k[bh * DK + i] << 16);
        qs[i] = __uint_as_float((uint32_t)q[bh * DK + i] << 16);
    }
    __syncthreads();
    float *srow = state + (bh * DV + row) * DK + c0;
    float S[C::COLS];
#pragma unroll
    for (int c = 0; c < C::COLS; c += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(srow + c);
        S[c] = x.x;
        S[c + 1] = x.y;
        S[c + 2] = x.z;
        S[c + 3] = x.w;
    }
    const float vr = __uint_as_float((uint32_t)v[bh * DV + row] << 16);
    const float ot = step<DK, DV>(S, ks, qs, vr, alpha[bh], beta[bh], c0);
#pragma unroll
    for (int c = 0; c < C::COLS; c += 4)
        *reinterpret_cast<float4 *>(srow + c) = make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
    if (tid % C::TPR == 0) o[bh * DV + row] = ot;
}

}  // namespace gdn

cudaError_t launch_gdn_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                               const float *alpha, const float *beta, const float *state_in,
                               int B, int64_t T, int H, int dk, int dv, float *o,
                               float *state_out, cudaStream_t s) {
    const int64_t grid = (int64_t)B * H;
    if (grid == 0) return cudaSuccess;
#define QSA_GDN(DK_, DV_)                                                                   \
    if (dk == DK_ && dv == DV_) {                                                           \
        gdn::gdn_prefill_kernel<DK_, DV_><<<(unsigned)grid, gdn::THREADS, 0, s>>>(           \
            q, k, v, alpha, beta, state_in, T, H, o, state_out);                             \
        return cudaGetLastError();                                                          \
    }
    QSA_GDN(64, 64) QSA_GDN(128, 128) QSA_GDN(128, 64) QSA_GDN(64, 128)
#undef QSA_GDN
    return cudaErrorInvalidValue;
}

cudaError_t launch_gdn_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              const float *alpha, const float *beta, float *state, int B, int H,
                              int dk, int dv, float *o, cudaStream_t s) {
    const int64_t grid = (int64_t)B * H;
    if (grid == 0) return cudaSuccess;
#define QSA_GDN(DK_, DV_)                                                                      \
    if (dk == DK_ && dv == DV_) {                                                              \
        gdn::gdn_decode_kernel<DK_, DV_><<<(unsigned)grid, gdn::THREADS, 0, s>>>(q, k, v, alpha, \
                                                                                beta, state, o); \
        return cudaGetLastError();                                                             \
    }
    QSA_GDN(64, 64) QSA_GDN(128, 128) QSA_GDN(128, 64) QSA_GDN(64, 128)
#undef QSA_GDN
    return cudaErrorInvalidValue;
}

}  // namespace qsa
