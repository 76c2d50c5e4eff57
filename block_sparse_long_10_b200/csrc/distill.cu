// Stage-1 indexer distillation: the KL loss between the dense attention's mass
// on each micro-block and the indexer's softmax over the same blocks, and the
// gradients of that loss with respect to the indexer's inputs
// ("用125亿分之6的参数，打平3970亿的旗舰模型", section
// "稀疏注意力：给检索建索引，也得先学会省纸": the first training stage trains
// only the indexer, to imitate the full-attention model's distribution, under a
// KL-divergence loss).
//
// Definitions, for query t at position p with candidates j < c = floor(p / 4):
//   a(t, j)   = sum_h sum_{i<4} exp(scale q_h(t) . k_g(4j + i) - lse_h(t))
//               (dense causal attention mass of all Hq heads; lse from the main
//               layer's dense forward)
//   pi(t, j)  = a(t, j) / Z(t),   Z(t) = sum_{j<c} a(t, j)
//   s(t, j)   = sum_h w_h(t) max(0, d_h(t, j)),   d_h = q_idx_h(t) . Kp(j)
//   KL(t)     = sum_j pi (ln pi - s + LSE(t)) = A / Z - ln Z + LSE,
//               A = sum_j a (ln a - s),  LSE = ln sum_j exp s    (0 when c < 2)
//   dL/ds     = exp(s - LSE) - pi
//   dq_idx_h(t) = sum_j dL/ds w_h 1[d_h > 0] Kp(j);   dw_h(t) = sum_j dL/ds max(0, d_h)
//   dKp(j)    = sum_t sum_h dL/ds w_h 1[d_h > 0] q_idx_h(t);  dk_idx(4j + i) = dKp(j) / 4
//
// Three kernels, in stream order:
//   1. teacher_kernel: the dense Q K^T tiles of the dense prefill kernel
//      (mma.sync, GQA row packing, cp.async ring) restricted to the candidate
//      blocks' keys; each probability exp2(S log2e scale - lse log2e) is summed
//      over the block's 4 keys and the KV group's G heads in registers and
//      shuffles, and written once per (group, query, block) to the workspace.
//   2. rows_tc_kernel: 32 query rows per CTA; pass 1 over their candidates
//      (head dot products on mma.sync) gives Z, A and LSE (the rows' loss),
//      pass 2 forms dL/ds, accumulates dw and dq_idx = sum G Kp on mma.sync.
//      Writes (Z, LSE) per row for kernel 3.
//   3. dkp_tc_kernel: one CTA per 32 blocks; streams the rows that see those
//      blocks in tiles of 32, recomputes the head dot products on the tensor
//      cores (mma.sync), forms dL/ds, and accumulates dKp = sum G^T Q_idx on
//      the tensor cores with G split into bf16 high and low parts: a fixed
//      summation order, no atomics.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {

namespace dst {

constexpr int R = 4;
constexpr float LOG2E = 1.4426950408889634f;
constexpr unsigned FULL = 0xffffffffu;

// ------------------------------------------------------------ teacher --
constexpr int TW = 8;
constexpr int TTHREADS = TW * 32;
constexpr int TROWS = 128;
constexpr int KT = 64;  // keys per tile (16 blocks)
constexpr int TSTAGES = 2;

template <int D>
struct TCfg {
    static constexpr int ROWB = D * 2;
    static constexpr int CH = D / 8;
    static constexpr int TILE = KT * ROWB;
    static constexpr int BYTES = TSTAGES * TILE;
};

template <int D, int G>
__global__ void __launch_bounds__(TTHREADS, 2)
    teacher_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                   const float *__restrict__ lse, int B, int64_t T, int Hkv, int64_t N,
                   float scale_log2, float *__restrict__ apart, int n_qt) {
    using C = TCfg<D>;
    constexpr int TOK = TROWS / G;
    constexpr int KSTEP = D / 16;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;
    const int Hq = Hkv * G;

    const int qt = n_qt - 1 - (int)(blockIdx.x % n_qt);  // longest query tiles first
    const int bg = blockIdx.x / n_qt;
    const int g = bg % Hkv;
    const int64_t b = bg / Hkv;
    const int64_t t0 = (int64_t)qt * TOK;

    // rows lr and lr + 8 of this warp: (token, head) pairs, G heads per token
    int64_t tok[2], cand[2];
    int head[2];
    float lse2[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int r = warp * 16 + lr + e * 8;
        tok[e] = t0 + r / G;
        head[e] = g * G + r % G;
        const bool in = tok[e] < T;
        cand[e] = in ? tok[e] / R : 0;
        lse2[e] = in ? lse[(b * T + tok[e]) * Hq + head[e]] * LOG2E : 0.f;
    }
    const int64_t t_last = (t0 + TOK - 1 < T) ? t0 + TOK - 1 : T - 1;
    const int64_t n_keys = (t_last / R) * R;  // keys of the last row's candidate blocks
    const int n_kt = (int)((n_keys + KT - 1) / KT);
    if (n_kt == 0) return;

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

    const uint16_t *kbase = k + (b * T) * Hkv * D + g * D;
    auto load_tile = [&](int kt) {
        if (kt < n_kt) {
            uint8_t *dk = smem + (kt % TSTAGES) * C::TILE;
            for (int i = tid; i < KT * C::CH; i += TTHREADS) {
                const int kr = i / C::CH, ch = i % C::CH;
                const int64_t u = (int64_t)kt * KT + kr;
                const bool ok = u < n_keys;
                const int64_t off = ok ? u * Hkv * D + ch * 8 : 0;
                cp_async16(smem_u32(dk + kr * C::ROWB + ((ch ^ (kr & 7)) * 16)), kbase + off,
                           ok ? 16 : 0);
            }
        }
        cp_async_commit();
    };
    load_tile(0);

    float *ag = apart + ((int64_t)g * B + b) * T * N;
#pragma unroll 1
    for (int kt = 0; kt < n_kt; ++kt) {
        cp_async_wait<0>();
        __syncthreads();
        load_tile(kt + 1);
        const uint8_t *sk = smem + (kt % TSTAGES) * C::TILE;
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
        // Columns nt*8 + 2lc, +1 of this lane belong to block kt*16 + 2nt + (lc >> 1).
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int64_t j = (int64_t)kt * (KT / R) + nt * 2 + (lc >> 1);
                const bool ok = j < cand[e2];
                float pr = 0.f;
                if (ok)
                    pr = fast_exp2(sacc[nt][e2 * 2] * scale_log2 - lse2[e2]) +
                         fast_exp2(sacc[nt][e2 * 2 + 1] * scale_log2 - lse2[e2]);
                pr += __shfl_xor_sync(FULL, pr, 1);  // the block's other two keys
#pragma unroll
                for (int off = 4; off < 4 * G; off <<= 1)  // the token's G heads
                    pr += __shfl_xor_sync(FULL, pr, off);
                if (ok && (lr % G) == 0 && (lc & 1) == 0) ag[tok[e2] * N + j] = pr;
            }
        }
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------- dKp --
constexpr int JB = 32;  // blocks per CTA
constexpr int RT = 32;  // rows per tile

// dKp on the tensor cores.  Per CTA: JB pooled blocks; per tile of RT rows:
//   A  d_h(t, j) = q_idx_h(t) . Kp(j) for the tile's 32 x 32 (row, block)
//      pairs: one 16 x 8 tile per warp, mma.sync over Di (bf16 in, fp32 sum);
//   B  per pair s, dL/ds and G_h = dL/ds w_h 1[d_h > 0] as in the rows
//      kernel, written to shared memory as bf16 high and low parts
//      (G = hi + lo to about 2^-17 relative);
//   C  dKp[blocks x Di] += sum_h (G_h^hi + G_h^lo)^T Q_h, mma.sync with the
//      rows as K; two 16 x 8 accumulator tiles per warp, in registers across
//      all row tiles (a fixed summation order, no atomics).
// Shared operand rows are padded by 16 bytes so that ldmatrix is free of bank
// conflicts.
constexpr int TCW = 8;  // warps
template <int HI, int DI>
struct TcCfg {
    static constexpr int KPSTR = DI * 2 + 16;       // [block][dim] bf16
    static constexpr int QSTR = HI * DI * 2 + 16;   // [row][head][dim] bf16
    static constexpr int GSTR = RT * 2 + 16;        // [head][hi/lo][block][row] bf16
    static constexpr int OFF_KP = 0;
    static constexpr int OFF_Q = OFF_KP + JB * KPSTR;
    static constexpr int OFF_G = OFF_Q + RT * QSTR;
    static constexpr int OFF_A = OFF_G + HI * 2 * JB * GSTR;   // [row][block] fp32
    static constexpr int OFF_W = OFF_A + RT * JB * 4;          // [row][head] fp32
    static constexpr int OFF_Z = OFF_W + RT * HI * 4;
    static constexpr int OFF_L = OFF_Z + RT * 4;
    static constexpr int BYTES = OFF_L + RT * 4;
    static_assert(JB == 32 && RT == 32, "tile shape");
    static_assert((DI / 8) % 2 == 0, "dims in pairs of n-tiles");
};

template <int HI, int DI>
__global__ void __launch_bounds__(TCW * 32)
    dkp_tc_kernel(const uint16_t *__restrict__ q_idx, const float *__restrict__ w,
                  const uint16_t *__restrict__ kp, const float *__restrict__ apart,
                  const float2 *__restrict__ stats, int B, int64_t T, int64_t N, int Hkv,
                  int n_jt, float *__restrict__ dkp, float *__restrict__ dk_idx) {
    using C = TcCfg<HI, DI>;
    constexpr int KS = DI / 16;
    constexpr int NT = DI / 8;  // dim n-tiles of the dKp tile
    extern __shared__ __align__(128) uint8_t smem[];
    float *sa = reinterpret_cast<float *>(smem + C::OFF_A);
    float *sw = reinterpret_cast<float *>(smem + C::OFF_W);
    float *sz = reinterpret_cast<float *>(smem + C::OFF_Z);
    float *sl = reinterpret_cast<float *>(smem + C::OFF_L);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;
    const int jt = blockIdx.x % n_jt;
    const int64_t b = blockIdx.x / n_jt;
    const int64_t j0 = (int64_t)jt * JB;
    const int nj = (int)((N - j0) < JB ? (N - j0) : JB);
    const int64_t gstride = (int64_t)B * T * N;

    // the CTA's pooled keys (rows past nj zero)
    for (int i = tid; i < JB * (DI / 8); i += TCW * 32) {
        const int jj = i / (DI / 8), ch = i % (DI / 8);
        cp_async16(smem_u32(smem + C::OFF_KP + jj * C::KPSTR + ch * 16),
                   kp + (b * N + j0 + (jj < nj ? jj : 0)) * DI + ch * 8, jj < nj ? 16 : 0);
    }
    cp_async_commit();

    // phase A/B: this warp's (row, block) tile; phase C: its two dKp tiles
    const int am = warp >> 2, an = warp & 3;          // rows 16 am.., blocks 8 an..
    const int cm = warp & 1, cn = (warp >> 1) * 2;    // blocks 16 cm.., dims 8 cn.. (2 tiles)
    const bool cwork = cn < NT;  // Di = 32 has work for four warps only
    float acc[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[u][e] = 0.f;

    int64_t t_begin = (j0 + 1) * R;  // rows that see block j0 and have two candidates
    if (t_begin < 2 * R) t_begin = 2 * R;
#pragma unroll 1
    for (int64_t t0 = t_begin; t0 < T; t0 += RT) {
        __syncthreads();  // the previous tile's operands are consumed
        for (int i = tid; i < RT * (HI * DI / 8); i += TCW * 32) {
            const int tt = i / (HI * DI / 8), ch = i % (HI * DI / 8);
            const int64_t t = t0 + tt;
            cp_async16(smem_u32(smem + C::OFF_Q + tt * C::QSTR + ch * 16),
                       q_idx + (b * T + (t < T ? t : 0)) * HI * DI + ch * 8, t < T ? 16 : 0);
        }
        cp_async_commit();
        for (int i = tid; i < RT * HI; i += TCW * 32) {
            const int64_t t = t0 + i / HI;
            sw[i] = t < T ? w[(b * T + t) * HI + i % HI] : 0.f;
        }
        for (int i = tid; i < RT; i += TCW * 32) {
            const int64_t t = t0 + i;
            const float2 st = t < T ? stats[b * T + t] : make_float2(0.f, 0.f);
            sz[i] = st.x;
            sl[i] = st.y;
        }
        for (int i = tid; i < RT * JB; i += TCW * 32) {
            const int tt = i / JB, jj = i % JB;
            const int64_t t = t0 + tt, j = j0 + jj;
            float a = 0.f;
            if (t < T && jj < nj && j < t / R)
                for (int gg = 0; gg < Hkv; ++gg) a += apart[gg * gstride + (b * T + t) * N + j];
            sa[i] = a;
        }
        cp_async_wait<0>();
        __syncthreads();

        // ---- A: d_h for rows 16 am + (lr, lr + 8), blocks 8 an + (2 lc, 2 lc + 1)
        float d[HI][4];
#pragma unroll
        for (int h = 0; h < HI; ++h) {
#pragma unroll
            for (int e = 0; e < 4; ++e) d[h][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t a0, a1, a2, a3, b0, b1;
                const int ar = am * 16 + (lane & 15);
                ldmatrix_x4(smem_u32(smem + C::OFF_Q + ar * C::QSTR + (h * DI + ks * 16) * 2 +
                                     (lane >> 4) * 16),
                            a0, a1, a2, a3);
                const int br = an * 8 + (lane & 7);
                ldmatrix_x2(smem_u32(smem + C::OFF_KP + br * C::KPSTR + ks * 32 +
                                     ((lane >> 3) & 1) * 16),
                            b0, b1);
                mma_bf16_16816(d[h], a0, a1, a2, a3, b0, b1);
            }
        }
        // ---- B: dL/ds and G_h per pair, to shared memory as bf16 hi + lo
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int rr = am * 16 + lr + (e >> 1) * 8;
            const int jl = an * 8 + 2 * lc + (e & 1);
            const int64_t t = t0 + rr, j = j0 + jl;
            const int64_t ct = t < T ? t / R : 0;
            const float Zt = sz[rr];
            float s = 0.f;
#pragma unroll
            for (int h = 0; h < HI; ++h) s = fmaf(sw[rr * HI + h], fmaxf(d[h][e], 0.f), s);
            const bool valid = jl < nj && ct > j && ct >= 2 && Zt > 0.f;
            const float gs = valid ? expf(s - sl[rr]) - sa[rr * JB + jl] * (1.f / Zt) : 0.f;
#pragma unroll
            for (int h = 0; h < HI; ++h) {
                const float g = d[h][e] > 0.f ? gs * sw[rr * HI + h] : 0.f;
                const uint16_t hi = to_bf16_bits(g);
                const uint16_t lo = to_bf16_bits(g - __uint_as_float((uint32_t)hi << 16));
                uint16_t *gp = reinterpret_cast<uint16_t *>(smem + C::OFF_G) +
                               ((h * 2) * JB + jl) * (C::GSTR / 2) + rr;
                gp[0] = hi;
                gp[JB * (C::GSTR / 2)] = lo;
            }
        }
        __syncthreads();
        // ---- C: dKp tiles (blocks 16 cm.., dims 8 (cn + u)..) += G^T Q
        if (!cwork) continue;
#pragma unroll
        for (int h = 0; h < HI; ++h)
#pragma unroll
            for (int hl = 0; hl < 2; ++hl)
#pragma unroll
                for (int ks = 0; ks < RT / 16; ++ks) {
                    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                    const int gr = cm * 16 + (lane & 15);
                    ldmatrix_x4(smem_u32(smem + C::OFF_G + ((h * 2 + hl) * JB + gr) * C::GSTR +
                                         ks * 32 + (lane >> 4) * 16),
                                a0, a1, a2, a3);
                    const int qr = ks * 16 + (lane & 15);
                    ldmatrix_x4_trans(smem_u32(smem + C::OFF_Q + qr * C::QSTR +
                                               (h * DI + cn * 8) * 2 + (lane >> 4) * 16),
                                      b0, b1, b2, b3);
                    mma_bf16_16816(acc[0], a0, a1, a2, a3, b0, b1);
                    mma_bf16_16816(acc[1], a0, a1, a2, a3, b2, b3);
                }
    }

    // rows 16 cm + lr (+8) are blocks, columns 8 (cn + u) + 2 lc (+1) are dims
    if (!cwork) return;
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int jl = cm * 16 + lr + (e >> 1) * 8;
            const int kk = (cn + u) * 8 + 2 * lc + (e & 1);
            if (jl >= nj) continue;
            const int64_t j = j0 + jl;
            dkp[(b * N + j) * DI + kk] = acc[u][e];
            if (dk_idx)
#pragma unroll
                for (int i = 0; i < R; ++i) dk_idx[(b * T + j * R + i) * DI + kk] = acc[u][e] * (1.f / R);
        }
}

// The rows' loss, dw and dq_idx on the tensor cores.  Per CTA: RT rows (one
// sequence), swept twice over their candidate blocks in tiles of JB:
//   pass 1  d_h on mma.sync (one 16 x 8 tile per warp, as in dkp_tc_kernel),
//           s, the teacher mass a, and per row the scores' running log-sum-exp,
//           Z and A, merged over lanes and warps at the end -> KL, (Z, LSE);
//   pass 2  d_h again, dL/ds, dw_h += dL/ds max(0, d_h) per row, and
//           G_h = dL/ds w_h 1[d_h > 0] to shared memory as bf16 high and low
//           parts; dq_h[rows x Di] += G_h Kp on mma.sync, the accumulators of
//           one (head, 16 rows, range of dims) per warp in registers.
// Rows with fewer than two candidates get zeros, as in the definition.
template <int HI, int DI>
struct RtCfg {
    static constexpr int NT = DI / 8;
    static constexpr int TPW = HI * 2 * NT / TCW;   // dq n-tiles per warp
    static_assert(TPW >= 1 && NT % TPW == 0, "dq tiles split evenly over the warps");
    static constexpr int KPSTR = DI * 2 + 16;       // [block][dim] bf16
    static constexpr int QSTR = HI * DI * 2 + 16;   // [row][head][dim] bf16
    static constexpr int GSTR = JB * 2 + 16;        // [head][hi/lo][row][block] bf16
    static constexpr int OFF_KP = 0;
    static constexpr int OFF_Q = OFF_KP + JB * KPSTR;
    static constexpr int OFF_G = OFF_Q + RT * QSTR;
    static constexpr int OFF_A = OFF_G + HI * 2 * RT * GSTR;   // [row][block] fp32
    static constexpr int OFF_W = OFF_A + RT * JB * 4;          // [row][head] fp32
    static constexpr int OFF_R = OFF_W + RT * HI * 4;          // 4 warps x RT rows x 4 partials
    static constexpr int OFF_S = OFF_R + 4 * RT * 4 * 4;       // per row: LSE, 1/Z, live flag
    static constexpr int OFF_DW = OFF_S + RT * 4 * 4;          // 4 warps x RT rows x HI
    static constexpr int BYTES = OFF_DW + 4 * RT * HI * 4;
};

template <int HI, int DI>
__global__ void __launch_bounds__(TCW * 32)
    rows_tc_kernel(const uint16_t *__restrict__ q_idx, const float *__restrict__ w,
                   const uint16_t *__restrict__ kp, const float *__restrict__ apart, int B,
                   int64_t T, int64_t N, int Hkv, int n_rt, float *__restrict__ kl,
                   float *__restrict__ dq, float *__restrict__ dw, float *__restrict__ dk_idx,
                   float2 *__restrict__ stats, void *status) {
    using C = RtCfg<HI, DI>;
    constexpr int KS = DI / 16;
    extern __shared__ __align__(128) uint8_t smem[];
    float *sa = reinterpret_cast<float *>(smem + C::OFF_A);
    float *sw = reinterpret_cast<float *>(smem + C::OFF_W);
    float *sred = reinterpret_cast<float *>(smem + C::OFF_R);
    float *srow = reinterpret_cast<float *>(smem + C::OFF_S);
    float *sdw = reinterpret_cast<float *>(smem + C::OFF_DW);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;
    const int rt = n_rt - 1 - (int)(blockIdx.x % n_rt);  // longest rows first
    const int64_t b = blockIdx.x / n_rt;
    const int64_t t0 = (int64_t)rt * RT;
    const int64_t t_end = t0 + RT < T ? t0 + RT : T;
    const int64_t c_max = (t_end - 1) / R;  // candidates of the tile's last row
    const int n_jt = (int)((c_max + JB - 1) / JB);
    const int64_t gstride = (int64_t)B * T * N;

    if (dk_idx)  // tokens of the trailing partial block: no pooled key
        for (int i = tid; i < RT * DI; i += TCW * 32) {
            const int64_t t = t0 + i / DI;
            if (t < T && t >= N * R) dk_idx[(b * T + t) * DI + i % DI] = 0.f;
        }
    for (int i = tid; i < RT * (HI * DI / 8); i += TCW * 32) {
        const int tt = i / (HI * DI / 8), ch = i % (HI * DI / 8);
        const int64_t t = t0 + tt;
        cp_async16(smem_u32(smem + C::OFF_Q + tt * C::QSTR + ch * 16),
                   q_idx + (b * T + (t < T ? t : 0)) * HI * DI + ch * 8, t < T ? 16 : 0);
    }
    cp_async_commit();
    for (int i = tid; i < RT * HI; i += TCW * 32) {
        const int64_t t = t0 + i / HI;
        sw[i] = t < T ? w[(b * T + t) * HI + i % HI] : 0.f;
    }

    const int am = warp >> 2, an = warp & 3;  // d tile: rows 16 am.., blocks 8 an..
    // the candidate-block tile: pooled keys and the teacher mass
    auto load_tile = [&](int jt) {
        const int64_t jb0 = (int64_t)jt * JB;
        for (int i = tid; i < JB * (DI / 8); i += TCW * 32) {
            const int jj = i / (DI / 8), ch = i % (DI / 8);
            const bool ok = jb0 + jj < c_max;
            cp_async16(smem_u32(smem + C::OFF_KP + jj * C::KPSTR + ch * 16),
                       kp + (b * N + (ok ? jb0 + jj : 0)) * DI + ch * 8, ok ? 16 : 0);
        }
        cp_async_commit();
        for (int i = tid; i < RT * JB; i += TCW * 32) {
            const int tt = i / JB, jj = i % JB;
            const int64_t t = t0 + tt, j = jb0 + jj;
            float a = 0.f;
            if (t < T && j < t / R)
                for (int gg = 0; gg < Hkv; ++gg) a += apart[gg * gstride + (b * T + t) * N + j];
            sa[i] = a;
        }
        cp_async_wait<0>();
    };
    auto dots = [&](float (&d)[HI][4]) {
#pragma unroll
        for (int h = 0; h < HI; ++h) {
#pragma unroll
            for (int e = 0; e < 4; ++e) d[h][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t a0, a1, a2, a3, b0, b1;
                const int ar = am * 16 + (lane & 15);
                ldmatrix_x4(smem_u32(smem + C::OFF_Q + ar * C::QSTR + (h * DI + ks * 16) * 2 +
                                     (lane >> 4) * 16),
                            a0, a1, a2, a3);
                const int br = an * 8 + (lane & 7);
                ldmatrix_x2(smem_u32(smem + C::OFF_KP + br * C::KPSTR + ks * 32 +
                                     ((lane >> 3) & 1) * 16),
                            b0, b1);
                mma_bf16_16816(d[h], a0, a1, a2, a3, b0, b1);
            }
        }
    };
    auto score = [&](const float (&d)[HI][4], int e, int rr) {
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < HI; ++h) s = fmaf(sw[rr * HI + h], fmaxf(d[h][e], 0.f), s);
        return s;
    };

    // ---- pass 1: the scores' log-sum-exp, Z and A per row ------------------
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, Zp[2] = {0.f, 0.f},
          Ap[2] = {0.f, 0.f};
#pragma unroll 1
    for (int jt = 0; jt < n_jt; ++jt) {
        __syncthreads();
        load_tile(jt);
        __syncthreads();
        float d[HI][4];
        dots(d);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int rr = am * 16 + lr + (e >> 1) * 8;
            const int64_t t = t0 + rr, j = (int64_t)jt * JB + an * 8 + 2 * lc + (e & 1);
            if (t >= T || j >= t / R) continue;
            const float s = score(d, e, rr);
            const float a = sa[rr * JB + an * 8 + 2 * lc + (e & 1)];
            const int k = e >> 1;
            if (s > m[k]) {
                l[k] = l[k] * expf(m[k] - s) + 1.f;
                m[k] = s;
            } else {
                l[k] += expf(s - m[k]);
            }
            Zp[k] += a;
            if (a > 0.f) Ap[k] += a * (logf(a) - s);
        }
    }
    // merge over the quad's lanes, then over the four warps of each row half
#pragma unroll
    for (int k = 0; k < 2; ++k) {
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            const float m2 = __shfl_xor_sync(FULL, m[k], off);
            const float l2 = __shfl_xor_sync(FULL, l[k], off);
            const float mn = fmaxf(m[k], m2);
            l[k] = (mn == -INFINITY) ? 0.f : l[k] * expf(m[k] - mn) + l2 * expf(m2 - mn);
            m[k] = mn;
            Zp[k] += __shfl_xor_sync(FULL, Zp[k], off);
            Ap[k] += __shfl_xor_sync(FULL, Ap[k], off);
        }
        if (lc == 0) {
            float *r4 = sred + ((an * RT) + am * 16 + lr + k * 8) * 4;
            r4[0] = m[k];
            r4[1] = l[k];
            r4[2] = Zp[k];
            r4[3] = Ap[k];
        }
    }
    __syncthreads();
    if (tid < RT) {
        const int rr = tid;
        const int64_t t = t0 + rr, row = b * T + t;
        float M = -INFINITY, Lsum = 0.f, Z = 0.f, A = 0.f;
        for (int wn = 0; wn < 4; ++wn) {
            const float *r4 = sred + (wn * RT + rr) * 4;
            const float mn = fmaxf(M, r4[0]);
            Lsum = (mn == -INFINITY) ? 0.f : Lsum * expf(M - mn) + r4[1] * expf(r4[0] - mn);
            M = mn;
            Z += r4[2];
            A += r4[3];
        }
        float live = 0.f, lse_s = 0.f, inv_z = 0.f;
        if (t < T) {
            if (t / R < 2) {
                kl[row] = 0.f;
                stats[row] = make_float2(1.f, 0.f);
            } else if (!(Z > 0.f)) {  // the teacher's candidate mass vanished in fp32
                record_status(status, QSA_ERR_DEVICE);
                kl[row] = 0.f;
                stats[row] = make_float2(0.f, 0.f);
            } else {
                lse_s = M + logf(Lsum);
                inv_z = 1.f / Z;
                live = 1.f;
                kl[row] = A * inv_z - logf(Z) + lse_s;
                stats[row] = make_float2(Z, lse_s);
            }
        }
        srow[rr * 4 + 0] = lse_s;
        srow[rr * 4 + 1] = inv_z;
        srow[rr * 4 + 2] = live;
    }

    // ---- pass 2: dL/ds, dw and dq_idx --------------------------------------
    // dq tiles of this warp: head qh, rows 16 qm.., dims 8 (qn0 + u)..
    const int tile0 = warp * C::TPW;
    const int qh = tile0 / (2 * C::NT), qm = (tile0 / C::NT) % 2, qn0 = tile0 % C::NT;
    float acc[C::TPW][4];
#pragma unroll
    for (int u = 0; u < C::TPW; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[u][e] = 0.f;
    float dwa[2][HI];
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int h = 0; h < HI; ++h) dwa[k][h] = 0.f;
#pragma unroll 1
    for (int jt = 0; jt < n_jt; ++jt) {
        __syncthreads();
        load_tile(jt);
        __syncthreads();
        float d[HI][4];
        dots(d);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int rr = am * 16 + lr + (e >> 1) * 8;
            const int jl = an * 8 + 2 * lc + (e & 1);
            const int64_t t = t0 + rr, j = (int64_t)jt * JB + jl;
            const bool valid = t < T && j < t / R && srow[rr * 4 + 2] > 0.f;
            const float gs = valid ? expf(score(d, e, rr) - srow[rr * 4]) -
                                         sa[rr * JB + jl] * srow[rr * 4 + 1]
                                   : 0.f;
#pragma unroll
            for (int h = 0; h < HI; ++h) {
                dwa[e >> 1][h] = fmaf(gs, fmaxf(d[h][e], 0.f), dwa[e >> 1][h]);
                const float g = d[h][e] > 0.f ? gs * sw[rr * HI + h] : 0.f;
                const uint16_t hi = to_bf16_bits(g);
                const uint16_t lo = to_bf16_bits(g - __uint_as_float((uint32_t)hi << 16));
                uint16_t *gp = reinterpret_cast<uint16_t *>(smem + C::OFF_G) +
                               ((h * 2) * RT + rr) * (C::GSTR / 2) + jl;
                gp[0] = hi;
                gp[RT * (C::GSTR / 2)] = lo;
            }
        }
        __syncthreads();
        // dq_qh[rows 16 qm.., dims] += (G^hi + G^lo)[rows, blocks] Kp[blocks, dims]
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
            for (int ks = 0; ks < JB / 16; ++ks) {
                uint32_t a0, a1, a2, a3;
                const int gr = qm * 16 + (lane & 15);
                ldmatrix_x4(smem_u32(smem + C::OFF_G + ((qh * 2 + hl) * RT + gr) * C::GSTR +
                                     ks * 32 + (lane >> 4) * 16),
                            a0, a1, a2, a3);
                const int kr = ks * 16 + (lane & 15);
                if constexpr (C::TPW == 1) {
                    uint32_t b0, b1;
                    ldmatrix_x2_trans(smem_u32(smem + C::OFF_KP + kr * C::KPSTR + qn0 * 16),
                                      b0, b1);
                    mma_bf16_16816(acc[0], a0, a1, a2, a3, b0, b1);
                } else {
#pragma unroll
                    for (int u = 0; u < C::TPW; u += 2) {
                        uint32_t b0, b1, b2, b3;
                        ldmatrix_x4_trans(smem_u32(smem + C::OFF_KP + kr * C::KPSTR +
                                                   (qn0 + u) * 16 + (lane >> 4) * 16),
                                          b0, b1, b2, b3);
                        mma_bf16_16816(acc[u], a0, a1, a2, a3, b0, b1);
                        mma_bf16_16816(acc[u + 1], a0, a1, a2, a3, b2, b3);
                    }
                }
            }
    }

    // dq: rows 16 qm + lr (+8), dims 8 (qn0 + u) + 2 lc (+1); rows with fewer
    // than two candidates get zeros (G was zero for them)
#pragma unroll
    for (int u = 0; u < C::TPW; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t t = t0 + qm * 16 + lr + (e >> 1) * 8;
            if (t >= T) continue;
            dq[((b * T + t) * HI + qh) * DI + (qn0 + u) * 8 + 2 * lc + (e & 1)] = acc[u][e];
        }
    // dw: over the quad's lanes, then the four warps of each row half
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int h = 0; h < HI; ++h) {
            float v = dwa[k][h];
            v += __shfl_xor_sync(FULL, v, 1);
            v += __shfl_xor_sync(FULL, v, 2);
            if (lc == 0) sdw[(an * RT + am * 16 + lr + k * 8) * HI + h] = v;
        }
    __syncthreads();
    for (int i = tid; i < RT * HI; i += TCW * 32) {
        const int rr = i / HI, h = i % HI;
        const int64_t t = t0 + rr;
        if (t >= T) continue;
        float v = 0.f;
        for (int wn = 0; wn < 4; ++wn) v += sdw[(wn * RT + rr) * HI + h];
        dw[(b * T + t) * HI + h] = v;
    }
}

template <int D, int G>
static cudaError_t launch_teacher(const uint16_t *q, const uint16_t *k, const float *lse, int B,
                                  int64_t T, int Hkv, int64_t N, float scale, float *apart,
                                  cudaStream_t s) {
    using C = TCfg<D>;
    auto kern = teacher_kernel<D, G>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), C::BYTES);
    if (e != cudaSuccess) return e;
    constexpr int TOK = TROWS / G;
    const int n_qt = (int)((T + TOK - 1) / TOK);
    const int64_t grid = (int64_t)n_qt * B * Hkv;
    if (grid == 0) return cudaSuccess;
    kern<<<(unsigned)grid, TTHREADS, C::BYTES, s>>>(q, k, lse, B, T, Hkv, N, scale * LOG2E, apart,
                                                   n_qt);
    return cudaGetLastError();
}

template <int HI, int DI>
static cudaError_t launch_indexer_side(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                                       const float *apart, int B, int64_t T, int64_t N, int Hkv,
                                       float *kl, float *dq, float *dw, float *dkp, float *dk_idx,
                                       float2 *stats, void *status, cudaStream_t s) {
    const int64_t rows = (int64_t)B * T;
    if (rows > 0) {
        using C = RtCfg<HI, DI>;
        auto kern = rows_tc_kernel<HI, DI>;
        cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), C::BYTES);
        if (e != cudaSuccess) return e;
        const int n_rt = (int)((T + RT - 1) / RT);
        kern<<<(unsigned)((int64_t)n_rt * B), TCW * 32, C::BYTES, s>>>(
            q_idx, w, kp, apart, B, T, N, Hkv, n_rt, kl, dq, dw, dk_idx, stats, status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (N > 0) {
        using C = TcCfg<HI, DI>;
        auto kern = dkp_tc_kernel<HI, DI>;
        cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), C::BYTES);
        if (e != cudaSuccess) return e;
        const int n_jt = (int)((N + JB - 1) / JB);
        kern<<<(unsigned)((int64_t)n_jt * B), TCW * 32, C::BYTES, s>>>(
            q_idx, w, kp, apart, stats, B, T, N, Hkv, n_jt, dkp, dk_idx);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace dst

size_t index_distill_ws_bytes(int B, int64_t T, int Hkv) {
    const int64_t N = T / dst::R;
    const size_t apart = (size_t)Hkv * B * T * N * sizeof(float);
    const size_t stats = (size_t)B * T * sizeof(float2);
    return kWsHeader + ((apart + 15) & ~(size_t)15) + stats;
}

cudaError_t launch_index_distill(const uint16_t *q, const uint16_t *k, const float *lse,
                                 const uint16_t *q_idx, const float *w, const uint16_t *kp, int B,
                                 int64_t T, int Hq, int Hkv, int D, int Hi, int Di, float scale,
                                 float *kl, float *dq, float *dw, float *dkp, float *dk_idx,
                                 void *ws, cudaStream_t s) {
    const int64_t N = T / dst::R;
    const size_t apart_bytes = (size_t)Hkv * B * T * N * sizeof(float);
    float *apart = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kWsHeader);
    float2 *stats = reinterpret_cast<float2 *>(static_cast<uint8_t *>(ws) + kWsHeader +
                                               ((apart_bytes + 15) & ~(size_t)15));
    const int G = Hq / Hkv;
    cudaError_t e = cudaErrorInvalidValue;
    if (N > 0) {
#define QSA_TEACHER(D_, G_) \
    if (D == D_ && G == G_) e = dst::launch_teacher<D_, G_>(q, k, lse, B, T, Hkv, N, scale, apart, s);
        QSA_TEACHER(64, 1) QSA_TEACHER(64, 2) QSA_TEACHER(64, 4) QSA_TEACHER(64, 8)
        QSA_TEACHER(128, 1) QSA_TEACHER(128, 2) QSA_TEACHER(128, 4) QSA_TEACHER(128, 8)
#undef QSA_TEACHER
        if (e != cudaSuccess) return e;
    }
    e = cudaErrorInvalidValue;
#define QSA_IDX_SIDE(HI_, DI_)                                                                   \
    if (Hi == HI_ && Di == DI_)                                                                  \
        e = dst::launch_indexer_side<HI_, DI_>(q_idx, w, kp, apart, B, T, N, Hkv, kl, dq, dw, dkp, \
                                               dk_idx, stats, ws, s);
    QSA_IDX_SIDE(1, 32) QSA_IDX_SIDE(2, 32) QSA_IDX_SIDE(4, 32)
    QSA_IDX_SIDE(1, 64) QSA_IDX_SIDE(2, 64) QSA_IDX_SIDE(4, 64)
#undef QSA_IDX_SIDE
    return e;
}

}  // namespace qsa
