// Gated DeltaNet prefill in chunks: the gated delta rule of gdn.cu
// ("用125亿分之6的参数，打平3970亿的旗舰模型", hybrid token-mixing section;
// "On the Design of Qwen3.8-Next Architecture", token-mixing paragraph),
//   S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T,   o_t = S_t q_t,
// rewritten over chunks of C tokens so that all work inside a chunk is matrix
// products.  With gamma_t = prod_{i<=t} alpha_i inside the chunk (i, t from 0)
// and S0 the state entering it, u_t = beta_t (v_t - alpha_t S_{t-1} k_t) obeys
//   (I + A) U = diag(beta) V - diag(beta gamma) K S0^T,
//   A_tj = beta_t (gamma_t / gamma_j) k_t . k_j  (j < t),
// so U = Ut - W S0^T with Ut = (I + A)^-1 diag(beta) V and
// W = (I + A)^-1 diag(beta gamma) K, and
//   O  = diag(gamma) Q S0^T + P U,   P_tj = (gamma_t / gamma_j) q_t . k_j  (j <= t),
//   S_C = gamma_{C-1} S0 + U^T diag(g) K,   g_j = gamma_{C-1} / gamma_j.
// Two kernels:
//   gdn_chunk_prep  one CTA per (sequence, head, chunk), all in parallel: the
//                   gates' log prefix sums, A and P from the chunk's dot
//                   products K K^T and Q K^T (mma.sync: bf16 products, fp32
//                   sums), the triangular solve for [Ut | W] by forward
//                   substitution in fp32 (one column per thread, held in
//                   registers: columns do not depend on one another), written
//                   to the workspace (W and P as bf16 high + low parts);
//   gdn_chunk_scan  per (sequence, head), VS = 16 rows of the state per CTA
//                   (the rows are independent: U, O and the state update of a
//                   row slice need only that slice), each CTA walking its chunks
//                   in order with its rows of the state in registers; the state
//                   products (W S0^T, Q S0^T, U^T diag(g) K) and P U run on
//                   mma.sync with every fp32 operand split into bf16 high and
//                   low parts (hi.hi + hi.lo + lo.hi, about 2^-16 relative).
// Tokens past the end of the sequence enter the last chunk as alpha = 1,
// beta = 0 and zero vectors: they change nothing.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {
namespace gdc {

constexpr int C = 64;          // tokens per chunk
constexpr int THREADS = 256;   // both kernels
constexpr float LOG_FLOOR = -80.f;

template <int DK, int DV>
struct Ws {  // per (sequence, head, chunk) record in the workspace, bytes
    static constexpr size_t W = (size_t)C * DK * 2;   // each of hi, lo (bf16)
    static constexpr size_t U = (size_t)C * DV * 4;   // Ut (fp32)
    static constexpr size_t P = (size_t)C * C * 2;    // each of hi, lo (bf16)
    static constexpr size_t OFF_WH = 0, OFF_WL = W, OFF_U = 2 * W, OFF_PH = 2 * W + U,
                            OFF_PL = OFF_PH + P, OFF_G = OFF_PL + P,   // gamma[C], g[C]
                            OFF_KH = OFF_G + 2 * C * 4, OFF_KL = OFF_KH + W;  // g_t k_t hi, lo
    static constexpr size_t BYTES = (OFF_KL + W + 255) / 256 * 256;
};

QSA_DEVICE void split_bf16(float x, uint16_t &hi, uint16_t &lo) {
    hi = to_bf16_bits(x);
    lo = to_bf16_bits(x - __uint_as_float((uint32_t)hi << 16));
}

// ---------------------------------------------------------------- prep --
template <int DK, int DV>
struct PrepCfg {
    static constexpr int NX = DV + DK;                  // columns of [Ut | W]
    static constexpr int KSTR = DK * 2 + 16;            // K, Q rows (bf16), padded: bytes
    static constexpr int ASTR = C + 4;                  // A rows (fp32), 16-byte aligned
    static constexpr int OFF_K = 0;                     // [C][KSTR] bytes
    static constexpr int OFF_Q = OFF_K + C * KSTR;      // [C][KSTR] bytes
    static constexpr int OFF_A = OFF_Q + C * KSTR;      // [C][ASTR] fp32
    static constexpr int OFF_L = OFF_A + C * ASTR * 4;  // log prefix, beta, gamma, g: [C] each
    static constexpr int BYTES = OFF_L + 4 * C * 4;
    static_assert(NX <= THREADS, "one column of [Ut | W] per thread");
    static_assert(KSTR % 16 == 0 && OFF_A % 16 == 0, "16-byte rows");
};

template <int DK, int DV>
__global__ void __launch_bounds__(THREADS, 2)
    gdn_chunk_prep(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                   const uint16_t *__restrict__ v, const float *__restrict__ alpha,
                   const float *__restrict__ beta, int64_t T, int H, int n_ch,
                   uint8_t *__restrict__ ws) {
    using P = PrepCfg<DK, DV>;
    using W = Ws<DK, DV>;
    extern __shared__ __align__(128) uint8_t smp[];
    float *As = reinterpret_cast<float *>(smp + P::OFF_A);
    float *ell = reinterpret_cast<float *>(smp + P::OFF_L), *bet = ell + C;
    float *gam = bet + C, *gl = gam + C;  // gamma_t, gamma_{C-1} / gamma_t
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;
    const int ch = blockIdx.x % n_ch;
    const int64_t bh = blockIdx.x / n_ch;  // b * H + h
    const int64_t b = bh / H, h = bh % H;
    const int64_t t0 = (int64_t)ch * C;
    uint8_t *rec = ws + (size_t)blockIdx.x * W::BYTES;
    auto kval = [&](int t, int d) {  // the chunk's key t, dimension d
        return __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t *>(
                                   smp + P::OFF_K + t * P::KSTR + d * 2)
                               << 16);
    };

    // the chunk's keys and queries as bf16 rows (zeros past the sequence)
    constexpr int CPR = DK / 8;  // 16-byte pieces per row
    for (int i = tid; i < C * CPR; i += THREADS) {
        const int t = i / CPR, c = i % CPR;
        const int64_t tok = t0 + t;
        uint4 kv = make_uint4(0u, 0u, 0u, 0u), qv = kv;
        if (tok < T) {
            const int64_t off = ((b * T + tok) * H + h) * DK + c * 8;
            kv = *reinterpret_cast<const uint4 *>(k + off);
            qv = *reinterpret_cast<const uint4 *>(q + off);
        }
        *reinterpret_cast<uint4 *>(smp + P::OFF_K + t * P::KSTR + c * 16) = kv;
        *reinterpret_cast<uint4 *>(smp + P::OFF_Q + t * P::KSTR + c * 16) = qv;
    }
    if (tid < 32) {  // gates: the log prefix of alpha (two tokens per lane), beta
        float la[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int t = lane * 2 + e;
            const int64_t tok = t0 + t;
            const float a = tok < T ? alpha[(b * T + tok) * H + h] : 1.f;
            la[e] = fmaxf(logf(a), LOG_FLOOR);
            bet[t] = tok < T ? beta[(b * T + tok) * H + h] : 0.f;
        }
        float run = la[0] + la[1];  // inclusive scan of the lane pairs
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, run, off);
            if (lane >= off) run += y;
        }
        const float excl = run - (la[0] + la[1]);
        ell[lane * 2] = excl + la[0];
        ell[lane * 2 + 1] = excl + la[0] + la[1];
        __syncwarp();
        const float last = ell[C - 1];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int t = lane * 2 + e;
            gam[t] = expf(ell[t]);
            gl[t] = expf(last - ell[t]);
        }
    }
    __syncthreads();

    // A (strictly lower) and P (lower, with the diagonal) from the chunk's dot
    // products K K^T and Q K^T on mma.sync (bf16 products, fp32 sums).  Warp
    // pair mt = warp / 2 takes rows 16 mt .. 16 mt + 15 and the 2 (mt + 1)
    // eight-column tiles of the lower triangle there, mt + 1 per warp.
    {
        const int mt = warp >> 1, half = warp & 1, ntn = mt + 1;
        float accA[4][4], accP[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) accA[n][e] = accP[n][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
            const int ar = mt * 16 + (lane & 15), acol = ks * 32 + (lane >> 4) * 16;
            uint32_t ak[4], aq[4];
            ldmatrix_x4(smem_u32(smp + P::OFF_K + ar * P::KSTR + acol), ak[0], ak[1], ak[2], ak[3]);
            ldmatrix_x4(smem_u32(smp + P::OFF_Q + ar * P::KSTR + acol), aq[0], aq[1], aq[2], aq[3]);
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                if (n < ntn) {
                    const int nt = half * ntn + n;
                    const int br = nt * 8 + (lane & 7), bcol = ks * 32 + ((lane >> 3) & 1) * 16;
                    uint32_t b0, b1;
                    ldmatrix_x2(smem_u32(smp + P::OFF_K + br * P::KSTR + bcol), b0, b1);
                    mma_bf16_16816(accA[n], ak[0], ak[1], ak[2], ak[3], b0, b1);
                    mma_bf16_16816(accP[n], aq[0], aq[1], aq[2], aq[3], b0, b1);
                }
            }
        }
        uint32_t *ph2 = reinterpret_cast<uint32_t *>(rec + W::OFF_PH);
        uint32_t *pl2 = reinterpret_cast<uint32_t *>(rec + W::OFF_PL);
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            if (n < ntn) {
                const int nt = half * ntn + n;
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {  // rows lr, lr + 8 of the tile
                    const int t = mt * 16 + lr + hr * 8;
                    uint16_t phv[2], plv[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j = nt * 8 + 2 * lc + e;
                        float a = 0.f, pv = 0.f;
                        if (j <= t) {
                            const float gr = expf(ell[t] - ell[j]);
                            if (j < t) a = bet[t] * gr * accA[n][hr * 2 + e];
                            pv = gr * accP[n][hr * 2 + e];
                        }
                        As[t * P::ASTR + j] = a;
                        split_bf16(pv, phv[e], plv[e]);
                    }
                    // P goes straight to the workspace as hi + lo
                    ph2[(t * C + nt * 8 + 2 * lc) >> 1] = (uint32_t)phv[0] | ((uint32_t)phv[1] << 16);
                    pl2[(t * C + nt * 8 + 2 * lc) >> 1] = (uint32_t)plv[0] | ((uint32_t)plv[1] << 16);
                }
            }
        }
        // P above the diagonal blocks (no tile computed there) is zero
        for (int i = tid; i < C * C / 2; i += THREADS) {
            const int t = i / (C / 2), j = (i % (C / 2)) * 2;
            if (j >= (t / 16) * 16 + 16) {
                ph2[i] = 0u;
                pl2[i] = 0u;
            }
        }
    }
    __syncthreads();

    // forward substitution, one column of [Ut | W] per thread, held in
    // registers (a column depends only on itself and A): row t minus the
    // earlier rows it depends on, in the order j = 0 .. t - 1
    if (tid < P::NX) {
        const int col = tid;
        float x[C];
        if (col < DV) {  // beta v
#pragma unroll
            for (int t = 0; t < C; ++t) {
                const int64_t tok = t0 + t;
                const float vv =
                    tok < T ? __uint_as_float((uint32_t)v[((b * T + tok) * H + h) * DV + col] << 16)
                            : 0.f;
                x[t] = bet[t] * vv;
            }
        } else {  // beta gamma k
#pragma unroll
            for (int t = 0; t < C; ++t) x[t] = bet[t] * gam[t] * kval(t, col - DV);
        }
#pragma unroll
        for (int t = 1; t < C; ++t) {
            float acc = x[t];
            const float4 *arow = reinterpret_cast<const float4 *>(As + t * P::ASTR);
#pragma unroll
            for (int j4 = 0; j4 < (t + 3) / 4; ++j4) {
                const float4 a4 = arow[j4];
                acc = fmaf(-a4.x, x[4 * j4], acc);
                if (4 * j4 + 1 < t) acc = fmaf(-a4.y, x[4 * j4 + 1], acc);
                if (4 * j4 + 2 < t) acc = fmaf(-a4.z, x[4 * j4 + 2], acc);
                if (4 * j4 + 3 < t) acc = fmaf(-a4.w, x[4 * j4 + 3], acc);
            }
            x[t] = acc;
        }
        if (col < DV) {
            float *u = reinterpret_cast<float *>(rec + W::OFF_U);
#pragma unroll
            for (int t = 0; t < C; ++t) u[t * DV + col] = x[t];
        } else {
            uint16_t *wh = reinterpret_cast<uint16_t *>(rec + W::OFF_WH);
            uint16_t *wl = reinterpret_cast<uint16_t *>(rec + W::OFF_WL);
#pragma unroll
            for (int t = 0; t < C; ++t) split_bf16(x[t], wh[t * DK + col - DV], wl[t * DK + col - DV]);
        }
    }
    if (tid < C) {
        float *g = reinterpret_cast<float *>(rec + W::OFF_G);
        g[tid] = gam[tid];
        g[C + tid] = gl[tid];
    }
    for (int i = tid; i < C * DK; i += THREADS) {  // g_t k_t, the state update's operand
        const int t = i / DK, d = i % DK;
        uint16_t kh, kl;
        split_bf16(gl[t] * kval(t, d), kh, kl);
        reinterpret_cast<uint16_t *>(rec + W::OFF_KH)[t * DK + d] = kh;
        reinterpret_cast<uint16_t *>(rec + W::OFF_KL)[t * DK + d] = kl;
    }
}

// ---------------------------------------------------------------- scan --
constexpr int VS = 16;  // state rows (value dims) per scan CTA

template <int DK, int DV>
struct ScanCfg {
    static constexpr int SSTR = DK * 2 + 16;  // state hi/lo [VS][DK] bf16, padded rows
    static constexpr int WSTR = DK * 2 + 16;  // W hi/lo, Q, gK hi/lo [C][DK] bf16
    static constexpr int PSTR = C * 2 + 16;   // P hi/lo [C][C] bf16
    static constexpr int USTR = VS * 2 + 16;  // U hi/lo [C][VS] bf16
    static constexpr int NSL = DV / VS;       // CTAs per (sequence, head)
    static constexpr int OFF_SH = 0;
    static constexpr int OFF_SL = OFF_SH + VS * SSTR;
    static constexpr int OFF_UH = OFF_SL + VS * SSTR;
    static constexpr int OFF_UL = OFF_UH + C * USTR;
    static constexpr int OFF_ST = OFF_UL + C * USTR;   // two stages of a chunk's operands
    // within a stage
    static constexpr int WH = 0, WL = WH + C * WSTR, Q = WL + C * WSTR, KH = Q + C * WSTR,
                         KL = KH + C * WSTR, PH = KL + C * WSTR, PL = PH + C * PSTR,
                         GM = PL + C * PSTR;            // gamma [C] fp32
    static constexpr int STAGE = GM + C * 4;
    static constexpr int BYTES = OFF_ST + 2 * STAGE;
    // state tiles (rows v, columns k): MT x NTS tiles of 16 x 8 over 8 warps
    static constexpr int MT = VS / 16, NTS = DK / 8, WPM = 8 / MT, NPW = NTS / WPM;
    // U / O tiles (rows t, columns v): 4 x VS/8 tiles, VS/16 per warp
    static constexpr int NU = VS / 16;
    static_assert(8 % MT == 0 && NTS % WPM == 0, "state tiles over 8 warps");
    static_assert(STAGE % 16 == 0 && OFF_ST % 16 == 0, "16-byte copies");
};

template <int DK, int DV>
__global__ void __launch_bounds__(THREADS, 1)
    gdn_chunk_scan(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                   const float *__restrict__ state_in, int64_t T, int H, int n_ch,
                   const uint8_t *__restrict__ ws, float *__restrict__ o,
                   float *__restrict__ state_out) {
    using S = ScanCfg<DK, DV>;
    using W = Ws<DK, DV>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;
    const int64_t bh = blockIdx.x / S::NSL, b = bh / H, h = bh % H;
    const int v0 = (int)(blockIdx.x % S::NSL) * VS;  // this CTA's rows of the state

    // state tiles of this warp: rows 16 ms + (lr, lr + 8), columns 8 (ns0 + n) + 2 lc (+1)
    const int ms = warp % S::MT, ns0 = (warp / S::MT) * S::NPW;
    float st[S::NPW][4];
    const float *sin = state_in ? state_in + bh * DV * DK : nullptr;
#pragma unroll
    for (int n = 0; n < S::NPW; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = ms * 16 + lr + (e >> 1) * 8, c = (ns0 + n) * 8 + 2 * lc + (e & 1);
            st[n][e] = sin ? sin[(v0 + r) * DK + c] : 0.f;
        }
    // U / O tiles of this warp: rows 16 mu + (lr, lr + 8), columns 8 (nu0 + n) + 2 lc (+1)
    const int mu = warp & 3, nu0 = (warp >> 2) * S::NU;

    // a chunk's operands into stage stg: W, P and g K from its workspace record,
    // Q from the queries, gamma
    auto prefetch = [&](int chn, int stg) {
        const uint8_t *rec = ws + (size_t)(bh * n_ch + chn) * W::BYTES;
        const int64_t t0 = (int64_t)chn * C;
        uint8_t *sb = smem + S::OFF_ST + stg * S::STAGE;
        for (int i = tid; i < C * (DK / 8); i += THREADS) {
            const int t = i / (DK / 8), c8 = i % (DK / 8);
            const int64_t tok = t0 + t;
            const size_t ro = (size_t)(t * DK + c8 * 8) * 2;
            const int so = t * S::WSTR + c8 * 16;
            cp_async16(smem_u32(sb + S::WH + so), rec + W::OFF_WH + ro, 16);
            cp_async16(smem_u32(sb + S::WL + so), rec + W::OFF_WL + ro, 16);
            cp_async16(smem_u32(sb + S::KH + so), rec + W::OFF_KH + ro, 16);
            cp_async16(smem_u32(sb + S::KL + so), rec + W::OFF_KL + ro, 16);
            cp_async16(smem_u32(sb + S::Q + so),
                       q + ((b * T + (tok < T ? tok : 0)) * H + h) * DK + c8 * 8,
                       tok < T ? 16 : 0);
        }
        for (int i = tid; i < C * (C / 8); i += THREADS) {
            const int t = i / (C / 8), c8 = i % (C / 8);
            const size_t ro = (size_t)(t * C + c8 * 8) * 2;
            cp_async16(smem_u32(sb + S::PH + t * S::PSTR + c8 * 16), rec + W::OFF_PH + ro, 16);
            cp_async16(smem_u32(sb + S::PL + t * S::PSTR + c8 * 16), rec + W::OFF_PL + ro, 16);
        }
        for (int i = tid; i < C / 4; i += THREADS)
            cp_async16(smem_u32(sb + S::GM + i * 16), rec + W::OFF_G + i * 16, 16);
        cp_async_commit();
    };
    if (n_ch > 0) prefetch(0, 0);

#pragma unroll 1
    for (int ch = 0; ch < n_ch; ++ch) {
        const int64_t t0 = (int64_t)ch * C;
        const uint8_t *rec = ws + (size_t)(bh * n_ch + ch) * W::BYTES;
        const uint8_t *sb = smem + S::OFF_ST + (ch & 1) * S::STAGE;
        const float *gm = reinterpret_cast<const float *>(sb + S::GM);
        // the next chunk's operands go into the other stage, free since the
        // previous chunk ended
        if (ch + 1 < n_ch) prefetch(ch + 1, (ch + 1) & 1);
        // ---- the state as bf16 hi + lo --------------------------------------
#pragma unroll
        for (int n = 0; n < S::NPW; ++n)
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                const int r = ms * 16 + lr + (e >> 1) * 8, c = (ns0 + n) * 8 + 2 * lc;
                uint16_t h0, l0, h1, l1;
                split_bf16(st[n][e], h0, l0);
                split_bf16(st[n][e + 1], h1, l1);
                *reinterpret_cast<uint32_t *>(smem + S::OFF_SH + r * S::SSTR + c * 2) =
                    (uint32_t)h0 | ((uint32_t)h1 << 16);
                *reinterpret_cast<uint32_t *>(smem + S::OFF_SL + r * S::SSTR + c * 2) =
                    (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
        if (ch + 1 < n_ch)
            cp_async_wait<1>();  // this chunk's group; the next one may stay in flight
        else
            cp_async_wait<0>();
        __syncthreads();

        // ---- U = Ut - W S0^T and O1 = Q S0^T (rows t, columns v; K = DK) ------
        float u[S::NU][4], ov[S::NU][4];
#pragma unroll
        for (int n = 0; n < S::NU; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                u[n][e] = 0.f;
                ov[n][e] = 0.f;
            }
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
            uint32_t wh[4], wl[4], qa[4];
            const int ar = mu * 16 + (lane & 15);
            const int acol = (ks * 16) * 2 + (lane >> 4) * 16;
            ldmatrix_x4(smem_u32(sb + S::WH + ar * S::WSTR + acol), wh[0], wh[1], wh[2], wh[3]);
            ldmatrix_x4(smem_u32(sb + S::WL + ar * S::WSTR + acol), wl[0], wl[1], wl[2], wl[3]);
            ldmatrix_x4(smem_u32(sb + S::Q + ar * S::WSTR + acol), qa[0], qa[1], qa[2], qa[3]);
#pragma unroll
            for (int n = 0; n < S::NU; ++n) {
                // B = S0^T (k x v) from the state rows v (k contiguous): no transpose
                const int br = (nu0 + n) * 8 + (lane & 7);
                const int bcol = ks * 32 + ((lane >> 3) & 1) * 16;
                uint32_t sh0, sh1, sl0, sl1;
                ldmatrix_x2(smem_u32(smem + S::OFF_SH + br * S::SSTR + bcol), sh0, sh1);
                ldmatrix_x2(smem_u32(smem + S::OFF_SL + br * S::SSTR + bcol), sl0, sl1);
                mma_bf16_16816(u[n], wh[0], wh[1], wh[2], wh[3], sh0, sh1);
                mma_bf16_16816(u[n], wh[0], wh[1], wh[2], wh[3], sl0, sl1);
                mma_bf16_16816(u[n], wl[0], wl[1], wl[2], wl[3], sh0, sh1);
                mma_bf16_16816(ov[n], qa[0], qa[1], qa[2], qa[3], sh0, sh1);
                mma_bf16_16816(ov[n], qa[0], qa[1], qa[2], qa[3], sl0, sl1);
            }
        }
        const float *ut = reinterpret_cast<const float *>(rec + W::OFF_U);
#pragma unroll
        for (int n = 0; n < S::NU; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = mu * 16 + lr + (e >> 1) * 8, c = (nu0 + n) * 8 + 2 * lc + (e & 1);
                u[n][e] = ut[t * DV + v0 + c] - u[n][e];
                ov[n][e] *= gm[t];
            }
        // U to shared memory as hi + lo, rows t
#pragma unroll
        for (int n = 0; n < S::NU; ++n)
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                const int t = mu * 16 + lr + (e >> 1) * 8, c = (nu0 + n) * 8 + 2 * lc;
                uint16_t h0, l0, h1, l1;
                split_bf16(u[n][e], h0, l0);
                split_bf16(u[n][e + 1], h1, l1);
                *reinterpret_cast<uint32_t *>(smem + S::OFF_UH + t * S::USTR + c * 2) =
                    (uint32_t)h0 | ((uint32_t)h1 << 16);
                *reinterpret_cast<uint32_t *>(smem + S::OFF_UL + t * S::USTR + c * 2) =
                    (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
        __syncthreads();

        // ---- O += P U (rows t, columns v; K = the chunk's tokens) ------------
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
            uint32_t ph[4], pl[4];
            const int ar = mu * 16 + (lane & 15);
            const int acol = (ks * 16) * 2 + (lane >> 4) * 16;
            ldmatrix_x4(smem_u32(sb + S::PH + ar * S::PSTR + acol), ph[0], ph[1], ph[2], ph[3]);
            ldmatrix_x4(smem_u32(sb + S::PL + ar * S::PSTR + acol), pl[0], pl[1], pl[2], pl[3]);
#pragma unroll
            for (int n = 0; n < S::NU; ++n) {
                // B = U (tokens x v), rows t (v contiguous): transposed load
                const int kr = ks * 16 + (lane & 15);
                const int bcol = (nu0 + n) * 16;
                uint32_t uh0, uh1, ul0, ul1;
                ldmatrix_x2_trans(smem_u32(smem + S::OFF_UH + kr * S::USTR + bcol), uh0, uh1);
                ldmatrix_x2_trans(smem_u32(smem + S::OFF_UL + kr * S::USTR + bcol), ul0, ul1);
                mma_bf16_16816(ov[n], ph[0], ph[1], ph[2], ph[3], uh0, uh1);
                mma_bf16_16816(ov[n], ph[0], ph[1], ph[2], ph[3], ul0, ul1);
                mma_bf16_16816(ov[n], pl[0], pl[1], pl[2], pl[3], uh0, uh1);
            }
        }
#pragma unroll
        for (int n = 0; n < S::NU; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = mu * 16 + lr + (e >> 1) * 8, c = (nu0 + n) * 8 + 2 * lc + (e & 1);
                const int64_t tok = t0 + t;
                if (tok < T) o[((b * T + tok) * H + h) * DV + v0 + c] = ov[n][e];
            }

        // ---- S = gamma_{C-1} S0 + U^T (g K) (rows v, columns k; K = tokens) ---
        const float glast = gm[C - 1];
#pragma unroll
        for (int n = 0; n < S::NPW; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) st[n][e] *= glast;
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
            // A = U^T (v x tokens) from U's rows t (v contiguous): transposed load
            uint32_t ah[4], al[4];
            const int kr = ks * 16 + (lane & 7) + ((lane >> 4) << 3);
            const int mcol = (ms * 16 + ((lane >> 3) & 1) * 8) * 2;
            ldmatrix_x4_trans(smem_u32(smem + S::OFF_UH + kr * S::USTR + mcol), ah[0], ah[1], ah[2], ah[3]);
            ldmatrix_x4_trans(smem_u32(smem + S::OFF_UL + kr * S::USTR + mcol), al[0], al[1], al[2], al[3]);
#pragma unroll
            for (int n = 0; n < S::NPW; ++n) {
                // B = g K (tokens x k), rows t (k contiguous): transposed load
                const int br = ks * 16 + (lane & 15);
                const int bcol = (ns0 + n) * 16;
                uint32_t kh0, kh1, kl0, kl1;
                ldmatrix_x2_trans(smem_u32(sb + S::KH + br * S::WSTR + bcol), kh0, kh1);
                ldmatrix_x2_trans(smem_u32(sb + S::KL + br * S::WSTR + bcol), kl0, kl1);
                mma_bf16_16816(st[n], ah[0], ah[1], ah[2], ah[3], kh0, kh1);
                mma_bf16_16816(st[n], ah[0], ah[1], ah[2], ah[3], kl0, kl1);
                mma_bf16_16816(st[n], al[0], al[1], al[2], al[3], kh0, kh1);
            }
        }
        __syncthreads();  // the chunk's shared operands are consumed
    }
    float *sout = state_out + bh * DV * DK;
#pragma unroll
    for (int n = 0; n < S::NPW; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = ms * 16 + lr + (e >> 1) * 8, c = (ns0 + n) * 8 + 2 * lc + (e & 1);
            sout[(v0 + r) * DK + c] = st[n][e];
        }
}

template <int DK, int DV>
static cudaError_t launch(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const float *alpha, const float *beta, const float *state_in, int B,
                          int64_t T, int H, float *o, float *state_out, uint8_t *ws,
                          cudaStream_t s) {
    const int n_ch = (int)((T + C - 1) / C);
    const int64_t bhs = (int64_t)B * H;
    if (n_ch > 0) {
        auto k1 = gdn_chunk_prep<DK, DV>;
        cudaError_t e = ensure_smem(reinterpret_cast<const void *>(k1), PrepCfg<DK, DV>::BYTES);
        if (e != cudaSuccess) return e;
        k1<<<(unsigned)(bhs * n_ch), THREADS, PrepCfg<DK, DV>::BYTES, s>>>(q, k, v, alpha, beta,
                                                                            T, H, n_ch, ws);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    auto k2 = gdn_chunk_scan<DK, DV>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(k2), ScanCfg<DK, DV>::BYTES);
    if (e != cudaSuccess) return e;
    k2<<<(unsigned)(bhs * ScanCfg<DK, DV>::NSL), THREADS, ScanCfg<DK, DV>::BYTES, s>>>(
        q, k, state_in, T, H, n_ch, ws, o, state_out);
    return cudaGetLastError();
}

}  // namespace gdc

size_t gdn_chunked_ws_bytes(int B, int64_t T, int H, int dk, int dv) {
    const int64_t n_ch = (T + gdc::C - 1) / gdc::C;
    size_t rec = 0;
    if (dk == 64 && dv == 64) rec = gdc::Ws<64, 64>::BYTES;
    if (dk == 128 && dv == 128) rec = gdc::Ws<128, 128>::BYTES;
    if (dk == 128 && dv == 64) rec = gdc::Ws<128, 64>::BYTES;
    if (dk == 64 && dv == 128) rec = gdc::Ws<64, 128>::BYTES;
    return kWsHeader + (size_t)B * H * n_ch * rec;
}

cudaError_t launch_gdn_prefill_chunked(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                       const float *alpha, const float *beta,
                                       const float *state_in, int B, int64_t T, int H, int dk,
                                       int dv, float *o, float *state_out, void *ws,
                                       cudaStream_t s) {
    if ((int64_t)B * H == 0) return cudaSuccess;
    uint8_t *rec = static_cast<uint8_t *>(ws) + kWsHeader;
#define QSA_GDC(DK_, DV_)                                                                   \
    if (dk == DK_ && dv == DV_)                                                             \
        return gdc::launch<DK_, DV_>(q, k, v, alpha, beta, state_in, B, T, H, o, state_out, \
                                     rec, s);
    QSA_GDC(64, 64) QSA_GDC(128, 128) QSA_GDC(128, 64) QSA_GDC(64, 128)
#undef QSA_GDC
    return cudaErrorInvalidValue;
}

}  // namespace qsa
