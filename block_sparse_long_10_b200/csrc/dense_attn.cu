// Dense causal GQA attention, prefill: the full-attention layer that QSA
// replaces ("用125亿分之6的参数，打平3970亿的旗舰模型", section
// "稀疏注意力：给检索建索引，也得先学会省纸": QSA against grouped-query
// attention), kept as the speed-up baseline on the same tensors.
//
// Flash-attention tiling with GQA row packing: a CTA owns 128 rows = the G
// query heads of one KV head for 128 / G consecutive tokens, so each 64-key
// K/V tile loaded into shared memory (cp.async, 2-stage ring, XOR swizzle)
// serves 128 rows.  8 warps x 16 rows; S = Q K^T and O += P V on mma.sync
// with fp32 accumulation; the online softmax stays in registers and P is
// reused in registers as the A operand of P V.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {

namespace dat {

constexpr int WARPS = 8;
constexpr int THREADS = WARPS * 32;
constexpr int ROWS = 128;
constexpr int KT = 64;  // keys per tile
constexpr int STAGES = 2;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

template <int D>
struct Cfg {
    static constexpr int ROWB = D * 2;
    static constexpr int CH = D / 8;
    static constexpr int TILE = KT * ROWB;
    static constexpr int STAGE_BYTES = 2 * TILE;
    static constexpr int BYTES = STAGES * STAGE_BYTES;
};

template <int D, int G>
__global__ void __launch_bounds__(THREADS, 1)
    dense_prefill_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                         const uint16_t *__restrict__ v, int64_t T, int Hkv,
                         float scale_log2, uint16_t *__restrict__ o, float *__restrict__ lse,
                         int n_qt) {
    using C = Cfg<D>;
    constexpr int TOK = ROWS / G;
    constexpr int KSTEP = D / 16;
    constexpr int NT_O = D / 8;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;
    const int Hq = Hkv * G;

    // longest query tiles first
    const int qt = n_qt - 1 - (int)(blockIdx.x % n_qt);
    const int bg = blockIdx.x / n_qt;
    const int g = bg % Hkv;
    const int64_t b = bg / Hkv;
    const int64_t t0 = (int64_t)qt * TOK;

    // rows lr and lr + 8 of this warp
    int64_t tok[2];
    int head[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int r = warp * 16 + lr + e * 8;
        tok[e] = t0 + r / G;
        head[e] = g * G + r % G;
    }
    uint32_t qa[KSTEP][4];
#pragma unroll
    for (int ks = 0; ks < KSTEP; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int rr = e & 1, dof = (e >> 1) * 8;
            uint32_t val = 0;
            if (tok[rr] < T)
                val = *reinterpret_cast<const uint32_t *>(
                    q + ((b * T + tok[rr]) * Hq + head[rr]) * D + ks * 16 + dof + 2 * lc);
            qa[ks][e] = val;
        }

    const int64_t t_last = (t0 + TOK - 1 < T) ? t0 + TOK - 1 : T - 1;
    const int n_kt = (int)((t_last + KT) / KT);
    const uint16_t *kbase = k + (b * T) * Hkv * D + g * D;
    const uint16_t *vbase = v + (b * T) * Hkv * D + g * D;

    auto load_tile = [&](int kt) {
        if (kt < n_kt) {
            uint8_t *dk = smem + (kt % STAGES) * C::STAGE_BYTES;
            uint8_t *dv = dk + C::TILE;
            for (int i = tid; i < KT * C::CH; i += THREADS) {
                const int kr = i / C::CH, ch = i % C::CH;
                const int64_t u = (int64_t)kt * KT + kr;
                const bool ok = u <= t_last;
                const int64_t off = ok ? u * Hkv * D + ch * 8 : 0;
                const int dst = kr * C::ROWB + ((ch ^ (kr & 7)) * 16);
                cp_async16(smem_u32(dk + dst), kbase + off, ok ? 16 : 0);
                cp_async16(smem_u32(dv + dst), vbase + off, ok ? 16 : 0);
            }
        }
        cp_async_commit();
    };
    load_tile(0);

    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    float oacc[NT_O][4];
#pragma unroll
    for (int nt = 0; nt < NT_O; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[nt][e] = 0.f;

#pragma unroll 1
    for (int kt = 0; kt < n_kt; ++kt) {
        cp_async_wait<0>();
        __syncthreads();
        load_tile(kt + 1);
        const uint8_t *sk = smem + (kt % STAGES) * C::STAGE_BYTES;
        const uint8_t *sv = sk + C::TILE;
        float sacc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KSTEP; ++ks) {
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                const int mi = lane >> 3;
                const int kr = pp * 16 + (mi >> 1) * 8 + (lane & 7);
                const int dc = ks * 2 + (mi & 1);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(smem_u32(sk + kr * C::ROWB + ((dc ^ (kr & 7)) * 16)), b0, b1, b2, b3);
                mma_bf16_16816(sacc[2 * pp], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
                mma_bf16_16816(sacc[2 * pp + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2,
                               b3);
            }
        }
        const bool need_mask = (int64_t)kt * KT + KT - 1 > t0;
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {  // row lr (e2 = 0) or lr + 8 (e2 = 1)
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float x = sacc[nt][e2 * 2 + c] * scale_log2;
                    if (need_mask) {
                        const int64_t u = (int64_t)kt * KT + nt * 8 + 2 * lc + c;
                        if (u > tok[e2]) x = -INFINITY;
                    }
                    sacc[nt][e2 * 2 + c] = x;
                    mx = fmaxf(mx, x);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run[e2], mx);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = fast_exp2(m_run[e2] - m_use);
            float ls = 0.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const float pv = fast_exp2(sacc[nt][e2 * 2 + c] - m_use);
                    sacc[nt][e2 * 2 + c] = pv;
                    ls += pv;
                }
            l_run[e2] = l_run[e2] * alpha + ls;
            m_run[e2] = m_new;
#pragma unroll
            for (int nt = 0; nt < NT_O; ++nt) {
                oacc[nt][e2 * 2] *= alpha;
                oacc[nt][e2 * 2 + 1] *= alpha;
            }
        }
        // O += P V
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
            const uint32_t a0 = pack_bf16x2(sacc[2 * kk][0], sacc[2 * kk][1]);
            const uint32_t a1 = pack_bf16x2(sacc[2 * kk][2], sacc[2 * kk][3]);
            const uint32_t a2 = pack_bf16x2(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]);
            const uint32_t a3 = pack_bf16x2(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3]);
#pragma unroll
            for (int dp = 0; dp < NT_O / 2; ++dp) {
                const int mi = lane >> 3;
                const int kr = kk * 16 + (mi & 1) * 8 + (lane & 7);
                const int dc = dp * 2 + (mi >> 1);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(smem_u32(sv + kr * C::ROWB + ((dc ^ (kr & 7)) * 16)), b0, b1,
                                  b2, b3);
                mma_bf16_16816(oacc[2 * dp], a0, a1, a2, a3, b0, b1);
                mma_bf16_16816(oacc[2 * dp + 1], a0, a1, a2, a3, b2, b3);
            }
        }
    }
    cp_async_wait<0>();

#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
        float l = l_run[e2];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (tok[e2] >= T) continue;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint16_t *orow = o + ((b * T + tok[e2]) * Hq + head[e2]) * D;
#pragma unroll
        for (int nt = 0; nt < NT_O; ++nt) {
            const uint32_t pk = pack_bf16x2(oacc[nt][e2 * 2] * inv, oacc[nt][e2 * 2 + 1] * inv);
            *reinterpret_cast<uint32_t *>(orow + nt * 8 + 2 * lc) = pk;
        }
        if (lse && lc == 0)
            lse[(b * T + tok[e2]) * Hq + head[e2]] =
                l > 0.f ? (m_run[e2] + __log2f(l)) * LN2 : -INFINITY;
    }
}

template <int D, int G>
static cudaError_t launch_dense(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B,
                                int64_t T, int Hkv, float scale, uint16_t *o, float *lse,
                                cudaStream_t s) {
    using C = Cfg<D>;
    auto kern = dense_prefill_kernel<D, G>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), C::BYTES);
    if (e != cudaSuccess) return e;
    constexpr int TOK = ROWS / G;
    const int n_qt = (int)((T + TOK - 1) / TOK);
    const int64_t grid = (int64_t)n_qt * B * Hkv;
    if (grid == 0) return cudaSuccess;
    kern<<<(unsigned)grid, THREADS, C::BYTES, s>>>(q, k, v, T, Hkv, scale * LOG2E, o, lse, n_qt);
    return cudaGetLastError();
}

}  // namespace dat

cudaError_t launch_dense_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B,
                                 int64_t T, int Hq, int Hkv, int D, float scale, uint16_t *o,
                                 float *lse, cudaStream_t s) {
    const int G = Hq / Hkv;
#define QSA_DENSE(D_, G_) \
    if (D == D_ && G == G_) return dat::launch_dense<D_, G_>(q, k, v, B, T, Hkv, scale, o, lse, s);
    QSA_DENSE(64, 1) QSA_DENSE(64, 2) QSA_DENSE(64, 4) QSA_DENSE(64, 8)
    QSA_DENSE(128, 1) QSA_DENSE(128, 2) QSA_DENSE(128, 4) QSA_DENSE(128, 8)
#undef QSA_DENSE
    return cudaErrorInvalidValue;
}

}  // namespace qsa
