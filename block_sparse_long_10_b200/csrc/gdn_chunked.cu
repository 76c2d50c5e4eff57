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
//                   products, the triangular solve for [Ut | W] by forward
//                   substitution (fp32 on CUDA cores), written to the
//                   workspace (W and P as bf16 high + low parts);
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
    static constexpr int OFF_K = 0;                     // [C][DK + 1] fp32
    static constexpr int OFF_Q = OFF_K + C * (DK + 1);  // [C][DK + 1] fp32
    static constexpr int OFF_X = OFF_Q + C * (DK + 1);  // [C][NX] fp32
    static constexpr int OFF_A = OFF_X + C * NX;        // [C][C + 1] fp32
    static constexpr int OFF_L = OFF_A + C * (C + 1);   // log prefix [C], beta [C]
    static constexpr int FLOATS = OFF_L + 2 * C;
    static constexpr int BYTES = FLOATS * 4;
};

template <int DK, int DV>
__global__ void __launch_bounds__(THREADS)
    gdn_chunk_prep(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                   const uint16_t *__restrict__ v, const float *__restrict__ alpha,
                   const float *__restrict__ beta, int64_t T, int H, int n_ch,
                   uint8_t *__restrict__ ws) {
    using P = PrepCfg<DK, DV>;
    using W = Ws<DK, DV>;
    extern __shared__ __align__(16) float sm[];
    float *Ks = sm + P::OFF_K, *Qs = sm + P::OFF_Q, *X = sm + P::OFF_X, *Am = sm + P::OFF_A;
    float *ell = sm + P::OFF_L, *bet = ell + C;
    const int tid = threadIdx.x, lane = tid & 31;
    const int ch = blockIdx.x % n_ch;
    const int64_t bh = blockIdx.x / n_ch;  // b * H + h
    const int64_t b = bh / H, h = bh % H;
    const int64_t t0 = (int64_t)ch * C;
    uint8_t *rec = ws + (size_t)blockIdx.x * W::BYTES;

    // the chunk's keys, queries, values (v scaled by beta into X's first DV columns)
    for (int i = tid; i < C * DK; i += THREADS) {
        const int t = i / DK, d = i % DK;
        const int64_t tok = t0 + t;
        const int64_t off = ((b * T + tok) * H + h) * DK + d;
        Ks[t * (DK + 1) + d] = tok < T ? __uint_as_float((uint32_t)k[off] << 16) : 0.f;
        Qs[t * (DK + 1) + d] = tok < T ? __uint_as_float((uint32_t)q[off] << 16) : 0.f;
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
    }
    __syncthreads();
    for (int i = tid; i < C * DV; i += THREADS) {
        const int t = i / DV, d = i % DV;
        const int64_t tok = t0 + t;
        const float vv =
            tok < T ? __uint_as_float((uint32_t)v[((b * T + tok) * H + h) * DV + d] << 16) : 0.f;
        X[t * P::NX + d] = bet[t] * vv;
    }
    for (int i = tid; i < C * DK; i += THREADS) {
        const int t = i / DK, d = i % DK;
        X[t * P::NX + DV + d] = bet[t] * expf(ell[t]) * Ks[t * (DK + 1) + d];
    }
    // A (strictly lower) and P (lower, with the diagonal): dot products
    for (int i = tid; i < C * C; i += THREADS) {
        const int t = i / C, j = i % C;
        float a = 0.f, p = 0.f;
        if (j <= t) {
            float dk_ = 0.f, dq_ = 0.f;
#pragma unroll 8
            for (int d = 0; d < DK; ++d) {
                const float kj = Ks[j * (DK + 1) + d];
                dk_ = fmaf(Ks[t * (DK + 1) + d], kj, dk_);
                dq_ = fmaf(Qs[t * (DK + 1) + d], kj, dq_);
            }
            const float gr = expf(ell[t] - ell[j]);
            if (j < t) a = bet[t] * gr * dk_;
            p = gr * dq_;
        }
        Am[t * (C + 1) + j] = a;
        // P goes straight to the workspace as hi + lo
        uint16_t ph, pl;
        split_bf16(p, ph, pl);
        reinterpret_cast<uint16_t *>(rec + W::OFF_PH)[t * C + j] = ph;
        reinterpret_cast<uint16_t *>(rec + W::OFF_PL)[t * C + j] = pl;
    }
    __syncthreads();
    // forward substitution: row t of [Ut | W] minus the earlier rows it depends on
    for (int t = 1; t < C; ++t) {
        for (int col = tid; col < P::NX; col += THREADS) {
            float acc = X[t * P::NX + col];
            for (int j = 0; j < t; ++j) acc = fmaf(-Am[t * (C + 1) + j], X[j * P::NX + col], acc);
            X[t * P::NX + col] = acc;
        }
        __syncthreads();
    }
    for (int i = tid; i < C * DV; i += THREADS) {
        const int t = i / DV, d = i % DV;
        reinterpret_cast<float *>(rec + W::OFF_U)[t * DV + d] = X[t * P::NX + d];
    }
    for (int i = tid; i < C * DK; i += THREADS) {
        const int t = i / DK, d = i % DK;
        uint16_t wh, wl;
        split_bf16(X[t * P::NX + DV + d], wh, wl);
        reinterpret_cast<uint16_t *>(rec + W::OFF_WH)[t * DK + d] = wh;
        reinterpret_cast<uint16_t *>(rec + W::OFF_WL)[t * DK + d] = wl;
    }
    if (tid < C) {
        float *g = reinterpret_cast<float *>(rec + W::OFF_G);
        g[tid] = expf(ell[tid]);                  // gamma_t
        g[C + tid] = expf(ell[C - 1] - ell[tid]); // gamma_{C-1} / gamma_t
    }
    for (int i = tid; i < C * DK; i += THREADS) {  // g_t k_t, the state update's operand
        const int t = i / DK, d = i % DK;
        uint16_t kh, kl;
        split_bf16(expf(ell[C - 1] - ell[t]) * Ks[t * (DK + 1) + d], kh, kl);
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
