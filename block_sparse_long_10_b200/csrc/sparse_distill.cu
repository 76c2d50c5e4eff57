// Stage-2 indexer loss: the KL between the sparse attention's mass on each
// selected block and the indexer's softmax over the same blocks, and its
// gradients with respect to the indexer's inputs
// ("用125亿分之6的参数，打平3970亿的旗舰模型", section
// "稀疏注意力：给检索建索引，也得先学会省纸": after the dense distillation,
// the second stage trains the indexer together with the backbone on the
// sparse pattern).
//
// Definitions, for query t at position p = t, c = floor(p / 4), and the
// selected candidate blocks J(t) = {j in sel[t] : 0 <= j < c} (the forced own
// block is never scored, so it takes no part):
//   a(t, j)  = sum_h sum_{i<4} exp(scale q_h(t) . k_g(4j + i) - lse_h(t))
//              (the sparse attention's probabilities over S(t); lse from the
//              sparse forward, which normalises over the whole token set)
//   pi(t, j) = a(t, j) / Z(t),   Z(t) = sum_{j in J(t)} a(t, j)
//   s(t, j)  = sum_h w_h(t) max(0, d_h(t, j)),   d_h = q_idx_h(t) . Kp(j)
//   KL(t)    = A / Z - ln Z + LSE,  A = sum_J a (ln a - s),  LSE = ln sum_J exp s
//              (0 when |J(t)| < 2)
//   g(t, j)  = exp(s - LSE) - pi
//   dq_idx_h(t) = sum_J g w_h 1[d_h > 0] Kp(j),   dw_h(t) = sum_J g max(0, d_h)
//   dKp(j)   = sum_t sum_h g w_h 1[d_h > 0] q_idx_h(t),   dk_idx(4j + i) = dKp(j) / 4
//
// First version, on the CUDA cores:
//   1. teacher_kernel: one warp per (query row, KV group); lane (i, n) takes
//      token i of a selected block and query head n of the group, so one
//      block's 4 x G probabilities come from one pass of dot products and a
//      warp sum; the mass per (group, row, selection entry) goes to the
//      workspace.
//   2. rows_kernel: one warp per query row; pass 1 (lanes over the selected
//      candidates) gives the scores, Z, A and LSE, pass 2 (lanes over the
//      indexer dims, blocks in turn) the gradients; dKp by atomics.
//   3. dk_idx_kernel: the pooled-key gradient spread back over the tokens.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {
namespace sds {

constexpr int R = 4;
constexpr float LOG2E = 1.4426950408889634f;
constexpr unsigned FULL = 0xffffffffu;
constexpr int MAXE = 1024;  // selection entries per row

QSA_DEVICE float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
    return x;
}

// ------------------------------------------------------------ teacher --
constexpr int TW = 4;  // warps per CTA

// mass[(g * rows + row) * kb + e]: the group's probability mass on selection
// entry e of the row (0 for entries that are not candidates).
template <int D, int G>
__global__ void __launch_bounds__(TW * 32)
    teacher_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                   const float *__restrict__ lse, const int32_t *__restrict__ sel, int64_t T,
                   int64_t rows, int Hkv, int kb, float scale_log2, float *__restrict__ mass) {
    constexpr int QS = D + 4;  // padded rows: the heads' float4 reads hit distinct banks
    __shared__ __align__(16) float qs_all[TW][8 * QS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t unit = (int64_t)blockIdx.x * TW + warp;  // (row, group)
    if (unit >= rows * Hkv) return;
    const int g = (int)(unit % Hkv);
    const int64_t row = unit / Hkv;  // b * T + t
    const int64_t b = row / T, t = row % T;
    const int64_t c = t / R;
    const int Hq = Hkv * G;
    float *qs = qs_all[warp];
    for (int i = lane; i < 8 * D; i += 32) {
        const int n = i / D, d = i % D;
        qs[n * QS + d] =
            n < G ? __uint_as_float((uint32_t)q[(row * Hq + g * G + n) * D + d] << 16) : 0.f;
    }
    __syncwarp();
    const int ti = lane >> 3, n = lane & 7;  // token of the block, head of the group
    const float lse2 = n < G ? lse[row * Hq + g * G + n] * LOG2E : 0.f;
    const float *qn = qs + n * QS;
    const int32_t *srow = sel + row * kb;
    float *mrow = mass + ((int64_t)g * rows + row) * kb;
    for (int e = 0; e < kb; ++e) {
        const int j = srow[e];
        float pv = 0.f;
        if (j >= 0 && j < c) {  // uniform across the warp
            const uint16_t *kr = k + ((b * T + (int64_t)j * R + ti) * Hkv + g) * D;
            float acc = 0.f;
#pragma unroll 4
            for (int d8 = 0; d8 < D / 8; ++d8) {
                const uint4 v = *reinterpret_cast<const uint4 *>(kr + d8 * 8);
                const float4 qa = *reinterpret_cast<const float4 *>(qn + d8 * 8);
                const float4 qb = *reinterpret_cast<const float4 *>(qn + d8 * 8 + 4);
                acc = fmaf(qa.x, bf16_lo(v.x), acc);
                acc = fmaf(qa.y, bf16_hi(v.x), acc);
                acc = fmaf(qa.z, bf16_lo(v.y), acc);
                acc = fmaf(qa.w, bf16_hi(v.y), acc);
                acc = fmaf(qb.x, bf16_lo(v.z), acc);
                acc = fmaf(qb.y, bf16_hi(v.z), acc);
                acc = fmaf(qb.z, bf16_lo(v.w), acc);
                acc = fmaf(qb.w, bf16_hi(v.w), acc);
            }
            if (n < G) pv = exp2f(acc * scale_log2 - lse2);
        }
        const float a = warp_sum(pv);
        if (lane == 0) mrow[e] = a;
    }
}

// --------------------------------------------------------------- rows --
constexpr int RW = 2;  // rows (warps) per CTA

template <int HI, int DI>
__global__ void __launch_bounds__(RW * 32)
    rows_kernel(const uint16_t *__restrict__ q_idx, const float *__restrict__ w,
                const uint16_t *__restrict__ kp, const int32_t *__restrict__ sel,
                const float *__restrict__ mass, int64_t T, int64_t rows, int64_t N, int Hkv,
                int kb, float *__restrict__ kl, float *__restrict__ dq, float *__restrict__ dw,
                float *__restrict__ dkp, void *status) {
    constexpr int DPL = DI / 32;  // dims per lane in pass 2
    __shared__ __align__(16) float qs_all[RW][HI * DI];
    __shared__ int blk_all[RW][MAXE];
    __shared__ float s_all[RW][MAXE];
    __shared__ float a_all[RW][MAXE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * RW + warp;
    if (row >= rows) return;
    const int64_t b = row / T, t = row % T;
    const int64_t c = t / R;
    float *qs = qs_all[warp];
    int *blk = blk_all[warp];
    float *sv = s_all[warp];
    float *av = a_all[warp];

    // the row's selected candidates, in selection order
    const int32_t *srow = sel + row * kb;
    int m = 0;
    for (int e0 = 0; e0 < kb; e0 += 32) {
        const int e = e0 + lane;
        const int j = e < kb ? srow[e] : -1;
        const bool cand = j >= 0 && j < c;
        const uint32_t bal = __ballot_sync(FULL, cand);
        if (cand) {
            const int pos = m + __popc(bal & ((1u << lane) - 1u));
            blk[pos] = j;
            float a = 0.f;
            for (int gg = 0; gg < Hkv; ++gg) a += mass[((int64_t)gg * rows + row) * kb + e];
            av[pos] = a;
        }
        m += __popc(bal);
    }
    auto zero_row = [&]() {
        for (int i = lane; i < HI * DI; i += 32) dq[row * HI * DI + i] = 0.f;
        if (lane < HI) dw[row * HI + lane] = 0.f;
        if (lane == 0) kl[row] = 0.f;
    };
    if (m < 2) {
        zero_row();
        return;
    }
    const uint32_t *qrow = reinterpret_cast<const uint32_t *>(q_idx + row * HI * DI);
    for (int i = lane; i < HI * DI / 2; i += 32) {
        const uint32_t v = qrow[i];
        qs[2 * i] = bf16_lo(v);
        qs[2 * i + 1] = bf16_hi(v);
    }
    __syncwarp();
    float wv[HI];
#pragma unroll
    for (int h = 0; h < HI; ++h) wv[h] = w[row * HI + h];
    const uint16_t *kpb = kp + b * N * DI;

    // pass 1: scores, their log-sum-exp, Z and A
    float mx = -INFINITY, l = 0.f, Z = 0.f, A = 0.f;
    for (int e = lane; e < m; e += 32) {
        const uint4 *kr = reinterpret_cast<const uint4 *>(kpb + (int64_t)blk[e] * DI);
        float d[HI];
#pragma unroll
        for (int h = 0; h < HI; ++h) d[h] = 0.f;
#pragma unroll 1
        for (int c8 = 0; c8 < DI / 8; ++c8) {
            const uint4 v = kr[c8];
            const float x[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                                bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
            for (int h = 0; h < HI; ++h)
#pragma unroll
                for (int u = 0; u < 8; ++u) d[h] = fmaf(qs[h * DI + c8 * 8 + u], x[u], d[h]);
        }
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < HI; ++h) s = fmaf(wv[h], fmaxf(d[h], 0.f), s);
        sv[e] = s;
        if (s > mx) {
            l = l * expf(mx - s) + 1.f;
            mx = s;
        } else {
            l += expf(s - mx);
        }
        const float a = av[e];
        Z += a;
        if (a > 0.f) A += a * (logf(a) - s);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
        const float m2 = __shfl_xor_sync(FULL, mx, off);
        const float l2 = __shfl_xor_sync(FULL, l, off);
        const float mn = fmaxf(mx, m2);
        l = (mn == -INFINITY) ? 0.f : l * expf(mx - mn) + l2 * expf(m2 - mn);
        mx = mn;
        Z += __shfl_xor_sync(FULL, Z, off);
        A += __shfl_xor_sync(FULL, A, off);
    }
    __syncwarp();
    if (!(Z > 0.f)) {  // the teacher's mass on the selected candidates vanished in fp32
        if (lane == 0) record_status(status, QSA_ERR_DEVICE);
        zero_row();
        return;
    }
    const float lse_s = mx + logf(l);
    const float inv_z = 1.f / Z;
    if (lane == 0) kl[row] = A * inv_z - logf(Z) + lse_s;

    // pass 2: lanes over the indexer dims, selected blocks in turn
    float qd[HI][DPL], dqa[HI][DPL], dwa[HI];
#pragma unroll
    for (int h = 0; h < HI; ++h) {
        dwa[h] = 0.f;
#pragma unroll
        for (int u = 0; u < DPL; ++u) {
            qd[h][u] = qs[h * DI + lane * DPL + u];
            dqa[h][u] = 0.f;
        }
    }
    for (int e = 0; e < m; ++e) {
        const int64_t j = blk[e];
        const float gsc = expf(sv[e] - lse_s) - av[e] * inv_z;
        float kx[DPL];
        const uint16_t *kr = kpb + j * DI + lane * DPL;
#pragma unroll
        for (int u = 0; u < DPL; ++u) kx[u] = __uint_as_float((uint32_t)kr[u] << 16);
        float contrib[DPL];
#pragma unroll
        for (int u = 0; u < DPL; ++u) contrib[u] = 0.f;
#pragma unroll
        for (int h = 0; h < HI; ++h) {
            float dp = 0.f;
#pragma unroll
            for (int u = 0; u < DPL; ++u) dp = fmaf(qd[h][u], kx[u], dp);
            dp = warp_sum(dp);
            dwa[h] = fmaf(gsc, fmaxf(dp, 0.f), dwa[h]);
            const float coef = dp > 0.f ? gsc * wv[h] : 0.f;
#pragma unroll
            for (int u = 0; u < DPL; ++u) {
                dqa[h][u] = fmaf(coef, kx[u], dqa[h][u]);
                contrib[u] = fmaf(coef, qd[h][u], contrib[u]);
            }
        }
        float *dk = dkp + (b * N + j) * DI + lane * DPL;
#pragma unroll
        for (int u = 0; u < DPL; ++u) atomicAdd(dk + u, contrib[u]);
    }
#pragma unroll
    for (int h = 0; h < HI; ++h) {
#pragma unroll
        for (int u = 0; u < DPL; ++u) dq[(row * HI + h) * DI + lane * DPL + u] = dqa[h][u];
        if (lane == 0) dw[row * HI + h] = dwa[h];
    }
}

// dk_idx[b, u, :] = dKp[b, u / 4, :] / 4 for tokens of complete blocks, else 0.
__global__ void dk_idx_kernel(const float *__restrict__ dkp, int64_t T, int64_t N, int Di,
                              int64_t total, float *__restrict__ dk_idx) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= total) return;
    const int d = (int)(i % Di);
    const int64_t bt = i / Di;
    const int64_t b = bt / T, u = bt % T;
    dk_idx[i] = u < N * R ? dkp[(b * N + u / R) * Di + d] * 0.25f : 0.f;
}

template <int D, int G>
static cudaError_t launch_teacher(const uint16_t *q, const uint16_t *k, const float *lse,
                                  const int32_t *sel, int64_t T, int64_t rows, int Hkv, int kb,
                                  float scale, float *mass, cudaStream_t s) {
    const int64_t units = rows * Hkv;
    teacher_kernel<D, G><<<(unsigned)((units + TW - 1) / TW), TW * 32, 0, s>>>(
        q, k, lse, sel, T, rows, Hkv, kb, scale * LOG2E, mass);
    return cudaGetLastError();
}

template <int HI, int DI>
static cudaError_t launch_rows(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                               const int32_t *sel, const float *mass, int64_t T, int64_t rows,
                               int64_t N, int Hkv, int kb, float *kl, float *dq, float *dw,
                               float *dkp, void *status, cudaStream_t s) {
    rows_kernel<HI, DI><<<(unsigned)((rows + RW - 1) / RW), RW * 32, 0, s>>>(
        q_idx, w, kp, sel, mass, T, rows, N, Hkv, kb, kl, dq, dw, dkp, status);
    return cudaGetLastError();
}

}  // namespace sds

size_t index_distill_sparse_ws_bytes(int B, int64_t T, int Hkv, int kb) {
    return kWsHeader + (size_t)Hkv * B * T * kb * sizeof(float);
}

int index_distill_sparse_max_entries() { return sds::MAXE; }

cudaError_t launch_index_distill_sparse(const uint16_t *q, const uint16_t *k, const float *lse,
                                        const int32_t *sel, const uint16_t *q_idx,
                                        const float *w, const uint16_t *kp, int B, int64_t T,
                                        int Hq, int Hkv, int D, int Hi, int Di, int kb,
                                        float scale, float *kl, float *dq_idx, float *dw,
                                        float *dkp, float *dk_idx, void *ws, cudaStream_t s) {
    const int64_t rows = (int64_t)B * T;
    const int64_t N = T / sds::R;
    float *mass = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kWsHeader);
    cudaError_t e = cudaSuccess;
    if (N > 0) e = cudaMemsetAsync(dkp, 0, (size_t)B * N * Di * sizeof(float), s);
    if (e != cudaSuccess || rows == 0) return e;
    const int G = Hq / Hkv;
    e = cudaErrorInvalidValue;
#define QSA_SDT(D_, G_) \
    if (D == D_ && G == G_) e = sds::launch_teacher<D_, G_>(q, k, lse, sel, T, rows, Hkv, kb, scale, mass, s);
    QSA_SDT(64, 1) QSA_SDT(64, 2) QSA_SDT(64, 4) QSA_SDT(64, 8)
    QSA_SDT(128, 1) QSA_SDT(128, 2) QSA_SDT(128, 4) QSA_SDT(128, 8)
#undef QSA_SDT
    if (e != cudaSuccess) return e;
    e = cudaErrorInvalidValue;
#define QSA_SDR(HI_, DI_)                                                                        \
    if (Hi == HI_ && Di == DI_)                                                                  \
        e = sds::launch_rows<HI_, DI_>(q_idx, w, kp, sel, mass, T, rows, N, Hkv, kb, kl, dq_idx, \
                                       dw, dkp, ws, s);
    QSA_SDR(1, 32) QSA_SDR(2, 32) QSA_SDR(4, 32) QSA_SDR(1, 64) QSA_SDR(2, 64) QSA_SDR(4, 64)
#undef QSA_SDR
    if (e != cudaSuccess || !dk_idx) return e;
    const int64_t total = rows * Di;
    sds::dk_idx_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(dkp, T, N, Di, total,
                                                                       dk_idx);
    return cudaGetLastError();
}

}  // namespace qsa
