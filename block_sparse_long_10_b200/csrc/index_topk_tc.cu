// Lightweight MQA indexer on tcgen05: fused block scores + exact top-k.
//
// "用125亿分之6的参数，打平3970亿的旗舰模型", section
// "稀疏注意力：给检索建索引，也得先学会省纸": a lightweight MQA indexer (several
// query heads, one shared pooled key head) scores every micro-block and the
// highest-scoring blocks are kept, following DSA's lightweight indexer;
// "On the Design of Qwen3.8-Next Architecture" (token-mixing paragraph):
// indexing O(n^2 / r), token budget 2048.
//
//   s(t, j) = sum_h w[t, h] * max(0, q_idx[t, h, :] . Kp[j, :])   (fp32)
//   keep the kb - 1 best j < floor(p / r) by (s desc, j asc) + own block.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0      TMA producer: the CTA's query tile (NCOL (query, head) rows,
//               double-buffered) and a 4-stage ring of 128-block pooled-key
//               tiles, 128/64-byte swizzled;
//   warp 1      TMEM owner and MMA issuer: per pooled-key tile one thread
//               issues D[128 blocks, NCOL columns] = Kp_tile x Q_tile^T as
//               Di/16 tcgen05.mma (bf16 in, fp32 in TMEM), double-buffered;
//   warps 2-17  epilogue: TMEM lane = block, so each thread reads one block's
//               scores for a quarter of the columns (32x32b loads, 16 columns
//               at a time) and forms the ReLU-weighted head sum in registers,
//               two heads per packed f32x2 multiply-add.
// Each query tile is swept twice (the pooled keys stay in L2):
//   pass 1  every thread keeps, per query, the maximum of a lower bound of
//           the score over its block lane and groups of R consecutive tiles
//           (at most 16 groups, so at most 2048 group maxima per query, kept
//           as 16-bit keys: the score rounded down to bf16 precision).  The
//           group maxima belong to distinct candidates, so the (kb-1)-th
//           largest of them, theta, is at most the true (kb-1)-th best score.
//           With Hi >= 2 the bound is linear: max(0, x) >= x and w >= 0 give
//             s(t, j) >= u_t . Kp[j] - c_t,  u_t = sum_h max(w_h, 0) q_idx[t, h],
//           (c_t = sum over negative weights of |w_h| |q_h|_1 max|Kp|), so
//           the MMA folds the head weights in: u_t enters as two bf16 rows
//           (u = hi + lo to ~2^-17) and the epilogue does one add and one max
//           per pair instead of the ReLU-weighted head sum.  theta is lowered
//           by a margin that covers the rounding of both passes (bounded by
//           |u|_1, sum_h |w_h| |q_h|_1 and max|Kp|).  With Hi = 1 pass 1 keeps
//           the exact score.  The bound is looser than the exact score (about
//           1.3-3x the survivors on random data) but costs a fraction of it.
//   pass 2  the exact scores (with Hi = 1 bit-identical to pass 1's) are
//           filtered by s >= theta and appended (64-bit key: order-preserving score bits
//           above the complemented block index) to the query's list in the
//           workspace.  Every top-(kb-1) candidate has s >= theta.  The test
//           is branch-free (a bit mask per thread, the survivor's score parked
//           in shared memory); survivors are staged per warp in shared memory
//           and moved to the lists in batches, and the lists are checked for
//           capacity every CHECK_EVERY tiles.
// Finalisation (per query): exact radix select of the list's kb - 1 best
// keys in shared memory, stable radix sort by block id, own block appended.
// A list that would overflow (only with heavily tied scores) is cut to its
// kb - 1 best keys on the spot and the filter becomes strict, which is exact
// because blocks are swept in ascending order.  Scores never reach HBM.
#include <stdlib.h>

#include "qsa_common.cuh"
#include "qsa_launch.h"
#include "sm100.cuh"
#include "topk_warp.cuh"


namespace qsa {
namespace itc {

constexpr int MB = 128;          // pooled blocks per tile = MMA M = TMEM lanes
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 16;    // 4 per TMEM lane quarter
constexpr int SEL_WARPS = 8;     // epilogue warps that also run the selections
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr int CAP = 4096;        // candidate-list capacity per query (workspace)
constexpr int SELBUF = 1024;     // per selecting warp, u64 keys in shared memory
constexpr int CHECK_EVERY = 16;  // pass-2 tiles between list-capacity checks (even)
static_assert(CHECK_EVERY % 2 == 0, "checks fall on the second tile of a pair");
constexpr int MAX_GROUPS = 16;   // group maxima per block lane and query
constexpr int MAX_KEEP = 511;    // the final sort network takes up to 512 keys
constexpr int MAX_GRID = 160;
constexpr int STG_ENT = 128;     // staged pass-2 survivors per epilogue warp

constexpr int KMAX_PARTS = 128;  // CTAs of the bound pre-pass that reduce max|Kp|
// The linear bound costs a fraction of the exact score in pass 1 but lets
// ~1.5x the survivors through to the selection; it pays from about this many
// pooled-key tiles per query tile on (measured: 1M context wins, 128K loses).
// QSA_INDEX_LB_MIN_KT overrides it (tests use 0 to run the bound at any size).
constexpr int LB_MIN_KT = 384;

template <int HI, int DI>
struct L {
    static constexpr int NCOL = HI == 1 ? 128 : 256;  // MMA N
    // two accumulator buffers; TMEM is allocated in powers of two columns
    static constexpr int TMEM_COLS = 2 * NCOL <= 128 ? 128 : 2 * NCOL <= 256 ? 256 : 512;
    static_assert(2 * NCOL <= 512, "TMEM");
    static constexpr int QT = NCOL / HI;              // queries per tile
    static constexpr int QPT = NCOL / 4 / HI;         // queries per epilogue thread
    static constexpr bool LB = HI >= 2;               // pass 1 on the linear bound
    static constexpr int UCOL = 2 * QT;               // pass-1 MMA N: (query, hi/lo) rows
    static_assert(!LB || UCOL <= NCOL, "pass-1 columns fit the buffer");
    static constexpr int ROWB = DI * 2;               // 64 or 128 bytes (= swizzle width)
    static constexpr int KP_TILE = MB * ROWB;
    static constexpr int Q_TILE = NCOL * ROWB;
    static constexpr int U_TILE = UCOL * ROWB;        // loaded into the query buffer first
    static constexpr int OFF_KP = 0;
    static constexpr int OFF_Q = OFF_KP + STAGES * KP_TILE;
    static constexpr int OFF_BUF = OFF_Q + 2 * Q_TILE;
    static constexpr int OFF_HIST = OFF_BUF + SEL_WARPS * SELBUF * 8;
    static_assert(EPI_WARPS * QPT * 32 * 4 <= SEL_WARPS * SELBUF * 8, "pass-2 score park");
    static_assert(EPI_WARPS * MAX_GROUPS * MB * 2 <= SEL_WARPS * SELBUF * 8, "bound keys");
    static_assert((EPI_WARPS - SEL_WARPS) * 256 * 4 <= EPI_WARPS * STG_ENT * 8, "bound hists");
    static_assert(SEL_WARPS * 512 * 4 <= EPI_WARPS * STG_ENT * 8, "sort hists");
    static constexpr int OFF_W = OFF_HIST + SEL_WARPS * 256 * 4;
    static constexpr int OFF_THR = OFF_W + QT * 16;
    static constexpr int OFF_C = OFF_THR + QT * 4;
    static constexpr int OFF_CNT = OFF_C + QT * 4;
    static constexpr int OFF_STGK = OFF_CNT + QT * 4;           // staged keys, per warp
    static constexpr int OFF_STGX = OFF_STGK + EPI_WARPS * STG_ENT * 8;  // their query
    static constexpr int OFF_BAR = OFF_STGX + EPI_WARPS * STG_ENT;
    static constexpr int NBAR = 2 * STAGES + 13;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;  // room to align the base to 1 KiB
};

struct Args {
    const float *w;
    const float2 *aux;        // per query (|u|_1 + sum_h |w_h| |q_h|_1, c_t / max|Kp|)
    const float *kmax_part;   // KMAX_PARTS partial maxima of |Kp|
    const int64_t *q_pos0;
    int B;
    int64_t Tq, n_blocks;
    int kb;
    int32_t *sel;
    float *sel_score;
    uint8_t *ws;
    int n_qt, total_tiles;
    uint64_t wait_limit;  // ns
    int grid;
    int lb_min_kt;        // pass 1 on the linear bound from this many key tiles
};

QSA_DEVICE void epi_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(EPI_WARPS * 32) : "memory"); }

QSA_DEVICE int64_t causal_blocks(int64_t pos, int64_t n_blocks, void *status) {
    if (pos < 0) return 0;
    int64_t c = pos / 4;
    if (c > n_blocks) {
        record_status(status, QSA_ERR_DEVICE);
        c = n_blocks;
    }
    return c;
}

// Per query tile geometry, identical in every role.
struct TileGeo {
    int b;
    int64_t t0, pb, c_min, c_max;
    int n_kt, R;
    bool lb;  // pass 1 on the linear bound (Hi >= 2 and enough key tiles)
};

template <int QT, bool LB>
QSA_DEVICE TileGeo tile_geo(const Args &a, int tile) {
    TileGeo g;
    g.b = tile % a.B;
    const int qt = a.n_qt - 1 - tile / a.B;  // longest query tiles first
    g.t0 = (int64_t)qt * QT;
    g.pb = a.q_pos0 ? a.q_pos0[g.b] : 0;
    const int64_t t_last = (g.t0 + QT < a.Tq ? g.t0 + QT : a.Tq) - 1;
    g.c_max = causal_blocks(g.pb + t_last, a.n_blocks, nullptr);
    g.c_min = causal_blocks(g.pb + g.t0, a.n_blocks, nullptr);
    g.n_kt = (int)((g.c_max + MB - 1) / MB);
    g.R = (g.n_kt + MAX_GROUPS - 1) / MAX_GROUPS;
    if (g.R < 1) g.R = 1;
    g.lb = LB && g.n_kt >= a.lb_min_kt;
    return g;
}

QSA_DEVICE uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
QSA_DEVICE float f2_sum(uint64_t p) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
    return lo + hi;
}

// s = sum_h w_h * max(x_h, 0) in fp32, heads paired on the packed f32x2 pipe:
// (w0 r0 + w2 r2) + (w1 r1 + w3 r3).  The ReLU is taken on the FMA pipe as
// x + |x| = 2 max(x, 0) (exact below half the float range), against halved
// weights, so every product w_h max(x_h, 0) is the same fp32 value as with a
// max instruction, which would run on the half-rate ALU pipe.  Both passes
// call this same function, so a block's score is bit-identical in them.
QSA_DEVICE float relu2(uint32_t v) {
    const float x = __uint_as_float(v);
    return x + fabsf(x);
}
template <int HI>
QSA_DEVICE float score_of(const uint32_t *v, const float4 wh) {
    const float r0 = relu2(v[0]);
    if constexpr (HI == 1) {
        return wh.x * r0;
    } else {
        const float r1 = relu2(v[1]);
        uint64_t acc;
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(acc) : "l"(f2_pack(wh.x, wh.y)), "l"(f2_pack(r0, r1)));
        if constexpr (HI == 4) {
            const float r2 = relu2(v[2]);
            const float r3 = relu2(v[3]);
            asm("fma.rn.f32x2 %0, %1, %2, %0;"
                : "+l"(acc)
                : "l"(f2_pack(wh.z, wh.w)), "l"(f2_pack(r2, r3)));
        }
        return f2_sum(acc);
    }
}

// Pass-1 operands.  One warp per query row: u = sum_h max(w_h, 0) q_idx[h]
// in fp32, stored as two bf16 rows hi = bf16(u), lo = bf16(u - hi);
// aux = (|u|_1 + sum_h |w_h| |q_h|_1, sum_h max(-w_h, 0) |q_h|_1).  CTAs from
// n_qcta on reduce max|Kp| over the pooled keys into KMAX_PARTS partials.
template <int HI, int DI>
__global__ void __launch_bounds__(256) ubound_kernel(const uint16_t *__restrict__ q_idx,
                                                     const float *__restrict__ w, int64_t rows,
                                                     const uint16_t *__restrict__ kp,
                                                     int64_t kp_vec16, uint16_t *__restrict__ uu,
                                                     float2 *__restrict__ aux,
                                                     float *__restrict__ kmax_part, int n_qcta) {
    constexpr int DPL = DI / 32;  // dims per lane: 1 or 2
    const int lane = threadIdx.x & 31;
    if ((int)blockIdx.x < n_qcta) {
        const int64_t nw = (int64_t)n_qcta * 8;
        for (int64_t row = blockIdx.x * 8 + (threadIdx.x >> 5); row < rows; row += nw) {
            float u[DPL], qn[HI], wv[HI];
#pragma unroll
            for (int e = 0; e < DPL; ++e) u[e] = 0.f;
#pragma unroll
            for (int h = 0; h < HI; ++h) {
                wv[h] = w[row * HI + h];
                const uint16_t *qh = q_idx + (row * HI + h) * DI + lane * DPL;
                float x[DPL];
                if constexpr (DPL == 2) {
                    const uint32_t b = *reinterpret_cast<const uint32_t *>(qh);
                    x[0] = bf16_lo(b);
                    x[1] = bf16_hi(b);
                } else {
                    x[0] = __uint_as_float((uint32_t)qh[0] << 16);
                }
                float a1 = 0.f;
#pragma unroll
                for (int e = 0; e < DPL; ++e) {
                    u[e] = fmaf(fmaxf(wv[h], 0.f), x[e], u[e]);
                    a1 += fabsf(x[e]);
                }
                qn[h] = a1;
            }
            float un = 0.f;
            uint16_t hi[DPL], lo[DPL];
#pragma unroll
            for (int e = 0; e < DPL; ++e) {
                un += fabsf(u[e]);
                hi[e] = to_bf16_bits(u[e]);
                lo[e] = to_bf16_bits(u[e] - __uint_as_float((uint32_t)hi[e] << 16));
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) {
                un += __shfl_xor_sync(0xffffffffu, un, off);
#pragma unroll
                for (int h = 0; h < HI; ++h) qn[h] += __shfl_xor_sync(0xffffffffu, qn[h], off);
            }
            uint16_t *uh = uu + row * 2 * DI + lane * DPL;
#pragma unroll
            for (int e = 0; e < DPL; ++e) {
                uh[e] = hi[e];
                uh[DI + e] = lo[e];
            }
            if (lane == 0) {
                float A = un, C = 0.f;
#pragma unroll
                for (int h = 0; h < HI; ++h) {
                    A = fmaf(fabsf(wv[h]), qn[h], A);
                    C = fmaf(fmaxf(-wv[h], 0.f), qn[h], C);
                }
                aux[row] = make_float2(A, C);
            }
        }
    } else {
        // max|Kp|: 16-byte loads, bf16 magnitudes compared as integers
        __shared__ uint32_t red[8];
        const int part = blockIdx.x - n_qcta;
        uint32_t m = 0;
        for (int64_t i = (int64_t)part * 256 + threadIdx.x; i < kp_vec16; i += KMAX_PARTS * 256) {
            const uint4 v = ldg_stream(kp + i * 8);
            const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                m = max(m, wd[c] & 0x7FFFu);
                m = max(m, (wd[c] >> 16) & 0x7FFFu);
            }
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) red[threadIdx.x >> 5] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t mm = 0;
            for (int i = 0; i < 8; ++i) mm = max(mm, red[i]);
            // magnitude bits of a finite bf16; an inf/NaN pattern maps to +inf
            kmax_part[part] = mm >= 0x7F80u ? INFINITY : __uint_as_float(mm << 16);
        }
    }
}

template <int HI, int DI>
__global__ void __launch_bounds__(THREADS, 1)
    idx_tc_kernel(const __grid_constant__ CUtensorMap tm_kp,
                  const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_u, const Args a) {
    using Lx = L<HI, DI>;
    constexpr int NCOL = Lx::NCOL;
    constexpr int QT = Lx::QT;
    constexpr int QPT = Lx::QPT;
    constexpr int KSTEPS = DI / 16;
    constexpr uint32_t IDESC = sm100::idesc_bf16_f32(MB, NCOL);
    constexpr uint32_t IDESC_U = sm100::idesc_bf16_f32(MB, Lx::LB ? Lx::UCOL : NCOL);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float4 *s_w = reinterpret_cast<float4 *>(sm + Lx::OFF_W);
    float *s_thr = reinterpret_cast<float *>(sm + Lx::OFF_THR);
    int *s_c = reinterpret_cast<int *>(sm + Lx::OFF_C);
    int *s_cnt = reinterpret_cast<int *>(sm + Lx::OFF_CNT);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + Lx::OFF_BAR);
    uint64_t *full = bar, *empty = bar + STAGES;
    uint64_t *tfull = bar + 2 * STAGES, *tempty = tfull + 2;
    uint64_t *qfull = tfull + 4, *qempty = tfull + 6;
    uint64_t *mma_done = tfull + 8;
    uint64_t *ufull = tfull + 9, *p1done = tfull + 11;  // pass-1 operand in, pass-1 MMAs done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Lx::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Lx::OFF_MISC + 8);
    volatile int *overflow = reinterpret_cast<volatile int *>(sm + Lx::OFF_MISC + 16);
    float *s_kmax = reinterpret_cast<float *>(sm + Lx::OFF_MISC + 24);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = a.kb - 1;
    // workspace: candidate lists, then group maxima, per CTA
    uint64_t *lists = reinterpret_cast<uint64_t *>(a.ws + kWsHeader) + (size_t)blockIdx.x * QT * CAP;
    // group maxima as 16-bit keys: the top half of the order-preserving score
    // key, i.e. the score rounded down, so theta stays a lower bound
    uint16_t *gmax_g = reinterpret_cast<uint16_t *>(reinterpret_cast<uint64_t *>(a.ws + kWsHeader) +
                                                    (size_t)a.grid * QT * CAP) +
                       (size_t)blockIdx.x * QT * (MAX_GROUPS * MB);

    if (tid == 0) {
        for (int i = 0; i < STAGES; ++i) {
            sm100::mbar_init(&full[i], 1);
            sm100::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            sm100::mbar_init(&tfull[i], 1);
            sm100::mbar_init(&tempty[i], EPI_WARPS);
            sm100::mbar_init(&qfull[i], 1);
            sm100::mbar_init(&qempty[i], 1);
        }
        sm100::mbar_init(mma_done, 1);
        for (int i = 0; i < 2; ++i) {
            sm100::mbar_init(&ufull[i], 1);
            sm100::mbar_init(&p1done[i], 1);
        }
        *abort_flag = 0;
        *overflow = 0;
        sm100::fence_mbar_init();
    }
    if (Lx::LB && warp == 2) {  // max|Kp| from the pre-pass partials
        float m = 0.f;
        for (int i = lane; i < KMAX_PARTS; i += 32) m = fmaxf(m, a.kmax_part[i]);
#pragma unroll
        for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) *s_kmax = m;
    }
    if (warp == 1) sm100::tmem_alloc(tmem_slot, Lx::TMEM_COLS);
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane == 0) {
            sm100::prefetch_tensormap(&tm_kp);
            sm100::prefetch_tensormap(&tm_q);
            if (Lx::LB) sm100::prefetch_tensormap(&tm_u);
            uint32_t it = 0;
            int last_kp[STAGES], last_q[2] = {-1, -1}, last_u[2] = {-1, -1};  // latest loads
            for (int s2 = 0; s2 < STAGES; ++s2) last_kp[s2] = -1;
            for (int i = 0;; ++i) {
                const int tile = blockIdx.x + i * gridDim.x;
                if (tile >= a.total_tiles) break;
                const TileGeo g = tile_geo<QT, Lx::LB>(a, tile);
                const int qb = i & 1;
                uint8_t *qbuf = sm + Lx::OFF_Q + qb * Lx::Q_TILE;
                const int64_t qrow = (int64_t)g.b * a.Tq + g.t0;
                const bool q_free = sm100::mbar_wait(&qempty[qb], ((i >> 1) & 1) ^ 1, abort_flag,
                                                     a.wait_limit, a.ws);
                bool q_issued = false;
                // With the linear bound the buffer first holds the pass-1 operand
                // (u as hi/lo rows); the query tile replaces it once the pass-1
                // MMAs have read it.
                auto load_q = [&]() {
                    q_issued = true;
                    if (g.lb && !sm100::mbar_wait(&p1done[qb], (i >> 1) & 1, abort_flag,
                                                    a.wait_limit, a.ws))
                        return;
                    sm100::mbar_arrive_expect_tx(&qfull[qb], Lx::Q_TILE);
                    sm100::tma_load_2d(qbuf, &tm_q, 0, (int32_t)(qrow * HI), &qfull[qb]);
                    last_q[qb] = i;
                };
                if (q_free) {
                    if (g.lb) {
                        sm100::mbar_arrive_expect_tx(&ufull[qb], Lx::U_TILE);
                        sm100::tma_load_2d(qbuf, &tm_u, 0, (int32_t)(qrow * 2), &ufull[qb]);
                        last_u[qb] = i;
                    } else {
                        load_q();
                    }
                } else {
                    q_issued = true;  // aborted: nothing more goes into this buffer
                }
                const int q_at = (STAGES - 1 < g.n_kt - 1 ? STAGES - 1 : g.n_kt - 1);
                for (int pass = 0; pass < 2; ++pass)
                    for (int kt = 0; kt < g.n_kt; ++kt, ++it) {
                        const int s = it % STAGES;
                        if (sm100::mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag,
                                             a.wait_limit, a.ws)) {
                            sm100::mbar_arrive_expect_tx(&full[s], Lx::KP_TILE);
                            sm100::tma_load_2d(sm + Lx::OFF_KP + s * Lx::KP_TILE, &tm_kp, 0,
                                               (int32_t)((int64_t)g.b * a.n_blocks + (int64_t)kt * MB),
                                               &full[s]);
                            last_kp[s] = (int)it;
                        }
                        // the pass-2 query tile goes in after the first few pass-2 key tiles
                        if (pass == 1 && kt == q_at && !q_issued) load_q();
                    }
                if (!q_issued) load_q();  // a tile without candidates still takes both
            }
            if (*abort_flag) {
                // let this CTA's own copies in flight land before it exits (bounded)
                for (int s2 = 0; s2 < STAGES; ++s2)
                    if (last_kp[s2] >= 0)
                        sm100::mbar_wait_for(&full[s2], (last_kp[s2] / STAGES) & 1, 100000000ull);
                for (int qb = 0; qb < 2; ++qb) {
                    if (last_q[qb] >= 0)
                        sm100::mbar_wait_for(&qfull[qb], (last_q[qb] >> 1) & 1, 100000000ull);
                    if (last_u[qb] >= 0)
                        sm100::mbar_wait_for(&ufull[qb], (last_u[qb] >> 1) & 1, 100000000ull);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer --
        if (lane == 0) {
            uint32_t it = 0;
            // This thread shares its SM sub-partition with four epilogue warps,
            // so the issue loop is kept short: the operand descriptors differ
            // only in their start-address field (address >> 4, low 14 bits), so
            // they are one constant high part and a 32-bit low part that the
            // k-steps advance by 32 bytes (2 units) each.
            const uint64_t desc_hi = sm100::smem_desc_kmajor(0, Lx::ROWB);
            const uint32_t kp_lo = (smem_u32(sm + Lx::OFF_KP) >> 4) & 0x3FFFu;
            const uint32_t q_lo = (smem_u32(sm + Lx::OFF_Q) >> 4) & 0x3FFFu;
            for (int i = 0;; ++i) {
                const int tile = blockIdx.x + i * gridDim.x;
                if (tile >= a.total_tiles) break;
                const TileGeo g = tile_geo<QT, Lx::LB>(a, tile);
                const int qb = i & 1;
                const uint32_t b_lo = q_lo + qb * (Lx::Q_TILE >> 4);
                // one sweep of the pooled-key tiles against the buffer's operand
                auto sweep = [&](bool op_ok, uint32_t idesc) {
                    for (int kt = 0; kt < g.n_kt; ++kt, ++it) {
                        const int s = it % STAGES;
                        const int tb = it & 1;
                        const bool ok = op_ok &&
                                        sm100::mbar_wait(&full[s], (it / STAGES) & 1, abort_flag,
                                                         a.wait_limit, a.ws) &&
                                        sm100::mbar_wait(&tempty[tb], ((it >> 1) & 1) ^ 1,
                                                         abort_flag, a.wait_limit, a.ws);
                        if (!ok) continue;
                        sm100::tc_fence_after();
                        const uint32_t a_lo = kp_lo + s * (Lx::KP_TILE >> 4);
#pragma unroll
                        for (int k = 0; k < KSTEPS; ++k)
                            sm100::mma_bf16(tmem_base + tb * NCOL, desc_hi | (a_lo + 2 * k),
                                            desc_hi | (b_lo + 2 * k), idesc, k > 0);
                        sm100::mma_commit(&empty[s]);
                        sm100::mma_commit(&tfull[tb]);
                    }
                };
                bool q_ok;
                if (g.lb) {
                    const bool u_ok =
                        sm100::mbar_wait(&ufull[qb], (i >> 1) & 1, abort_flag, a.wait_limit, a.ws);
                    sm100::tc_fence_after();
                    sweep(u_ok, IDESC_U);
                    sm100::mma_commit(&p1done[qb]);  // the buffer may take the query tile
                    q_ok = sm100::mbar_wait(&qfull[qb], (i >> 1) & 1, abort_flag, a.wait_limit, a.ws);
                    sm100::tc_fence_after();
                    sweep(q_ok, IDESC);
                } else {
                    q_ok = sm100::mbar_wait(&qfull[qb], (i >> 1) & 1, abort_flag, a.wait_limit, a.ws);
                    sm100::tc_fence_after();
                    sweep(q_ok, IDESC);
                    sweep(q_ok, IDESC);
                }
                if (q_ok) sm100::mma_commit(&qempty[qb]);
            }
            // every MMA this thread issued has retired before TMEM is freed (bounded)
            sm100::mma_commit(mma_done);
            sm100::mbar_wait_for(mma_done, 0, 1000000000ull);
        }
    } else {
        // ------------------------------------------------------ epilogue --
        const int e = warp - 2;                 // 0..15
        const int etid = tid - 64;
        const int lq = warp & 3;                // TMEM lane quarter this warp may read
        const int cq = e >> 2;                  // column quarter
        const int q0 = cq * QPT;                // first query of this thread
        const int p = lq * 32 + lane;           // block position within the tile
        const bool selw = e < SEL_WARPS;
        // 9-bit digits of the largest block id
        int sort_passes = 1;
        while (sort_passes < 4 && ((a.n_blocks - 1) >> (9 * sort_passes)) > 0) ++sort_passes;
        // the final sort's 512-bin histograms use the staging area, idle by then
        uint32_t *hist9 = reinterpret_cast<uint32_t *>(sm + Lx::OFF_STGK) + (selw ? e : 0) * 512;
        uint32_t *hist = reinterpret_cast<uint32_t *>(sm + Lx::OFF_HIST) + (selw ? e : 0) * 256;
        uint64_t *buf = reinterpret_cast<uint64_t *>(sm + Lx::OFF_BUF) + (size_t)(selw ? e : 0) * SELBUF;
        uint32_t it = 0;
        for (int i = 0;; ++i) {
            const int tile = blockIdx.x + i * gridDim.x;
            if (tile >= a.total_tiles) break;
            const TileGeo g = tile_geo<QT, Lx::LB>(a, tile);
            const int n_groups = (g.n_kt + g.R - 1) / g.R;

            for (int q = etid; q < QT; q += EPI_WARPS * 32) {
                const int64_t t = g.t0 + q;
                float wv[4] = {0.f, 0.f, 0.f, 0.f};
                int c = 0;
                if (t < a.Tq) {
                    c = (int)causal_blocks(g.pb + t, a.n_blocks, a.ws);
                    const float *wr = a.w + ((int64_t)g.b * a.Tq + t) * HI;
#pragma unroll
                    for (int h = 0; h < HI; ++h) wv[h] = wr[h];
                }
                // halved: the scoring doubles the ReLU (exact both ways)
                s_w[q] = make_float4(0.5f * wv[0], 0.5f * wv[1], 0.5f * wv[2], 0.5f * wv[3]);
                s_c[q] = c;
                s_cnt[q] = 0;
            }
            epi_sync();

            // ---- pass 1: group maxima -----------------------------------
            float gm[QPT];
#pragma unroll
            for (int x = 0; x < QPT; ++x) gm[x] = -INFINITY;
            int r_in = 0, grp = 0;  // tiles into the current group, group index
            for (int kt = 0; kt < g.n_kt; ++kt, ++it) {
                const int tb = it & 1;
                sm100::mbar_wait(&tfull[tb], (it >> 1) & 1, abort_flag, a.wait_limit, a.ws);
                sm100::tc_fence_after();
                const int j = kt * MB + p;
                const bool tail = (int64_t)kt * MB + MB > g.c_min;
                if (g.lb) {
                    // columns (query, hi/lo): the bound is hi + lo, one max per pair
                    const uint32_t taddr = tmem_base + ((uint32_t)(lq * 32) << 16) + tb * NCOL +
                                           cq * (Lx::UCOL / 4);
                    constexpr int CW = 16;
                    constexpr int NCH = Lx::UCOL / 4 / CW;
#pragma unroll
                    for (int ch = 0; ch < NCH; ++ch) {
                        uint32_t v[CW];
                        sm100::tmem_ld16(taddr + CW * ch, v);
                        if (!tail) {
#pragma unroll
                            for (int qq = 0; qq < CW / 2; ++qq) {
                                const int x = ch * (CW / 2) + qq;
                                gm[x] = fmaxf(gm[x], __uint_as_float(v[2 * qq]) +
                                                         __uint_as_float(v[2 * qq + 1]));
                            }
                        } else {
#pragma unroll
                            for (int qq = 0; qq < CW / 2; ++qq) {
                                const int x = ch * (CW / 2) + qq;
                                const float lb =
                                    __uint_as_float(v[2 * qq]) + __uint_as_float(v[2 * qq + 1]);
                                if (j < s_c[q0 + x]) gm[x] = fmaxf(gm[x], lb);
                            }
                        }
                    }
                } else {
                    const uint32_t taddr =
                        tmem_base + ((uint32_t)(lq * 32) << 16) + tb * NCOL + cq * (NCOL / 4);
                    constexpr int CW = 16;  // columns per load: 16 values live at a time
                    constexpr int NCH = NCOL / 4 / CW;
#pragma unroll
                    for (int ch = 0; ch < NCH; ++ch) {
                        uint32_t v[CW];
                        sm100::tmem_ld16(taddr + CW * ch, v);
                        if (!tail) {
#pragma unroll
                            for (int qq = 0; qq < CW / HI; ++qq) {
                                const int x = ch * (CW / HI) + qq;
                                gm[x] = fmaxf(gm[x], score_of<HI>(v + qq * HI, s_w[q0 + x]));
                            }
                        } else {
#pragma unroll
                            for (int qq = 0; qq < CW / HI; ++qq) {
                                const int x = ch * (CW / HI) + qq;
                                const float s = score_of<HI>(v + qq * HI, s_w[q0 + x]);
                                if (j < s_c[q0 + x]) gm[x] = fmaxf(gm[x], s);
                            }
                        }
                    }
                }
                sm100::tc_fence_before();
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&tempty[tb]);
                if (++r_in == g.R || kt + 1 == g.n_kt) {
#pragma unroll
                    for (int x = 0; x < QPT; ++x) {
                        gmax_g[(size_t)(q0 + x) * (MAX_GROUPS * MB) + grp * MB + p] =
                            (uint16_t)(score_key(gm[x]) >> 16);
                        gm[x] = -INFINITY;
                    }
                    r_in = 0;
                    ++grp;
                }
            }
            epi_sync();

            // ---- theta: the (kb-1)-th largest group maximum --------------
            // every epilogue warp takes queries; the bound needs the score value
            // only, so the keys are the 32-bit score keys (the selection
            // buffers hold 16 x 1024 of them; warps past the selecting ones
            // keep their histograms in the idle staging area)
            {
                uint16_t *kbuf = reinterpret_cast<uint16_t *>(sm + Lx::OFF_BUF) + e * (MAX_GROUPS * MB);
                uint32_t *th_hist = selw ? hist
                                         : reinterpret_cast<uint32_t *>(sm + Lx::OFF_STGK) +
                                               (e - SEL_WARPS) * 256;
#pragma unroll 1
                for (int q = e; q < QT; q += EPI_WARPS) {
                    float th = K > 0 ? -INFINITY : INFINITY;
                    const int G = n_groups * MB;
                    if (K > 0 && G >= K && g.t0 + q < a.Tq) {
                        const uint16_t *src = gmax_g + (size_t)q * (MAX_GROUPS * MB);
                        for (int x = 8 * lane; x < G; x += 256)  // G is a multiple of 128
                            cp_async16(smem_u32(kbuf + x), src + x, 16);
                        cp_async_commit();
                        cp_async_wait<0>();
                        __syncwarp();
                        // widen with zero low bits (rounds down); below the key of
                        // -inf lie only NaN patterns, so clamp there
                        const uint32_t k32 =
                            idx::warp_kth_largest_narrow<uint16_t>(kbuf, G, K, th_hist, lane) << 16;
                        th = k32 <= score_key(-INFINITY) ? -INFINITY : key_score(k32);
                        if (g.lb && lane == 0 && th > -INFINITY) {
                            // from the bound back to the score: subtract c_t and a
                            // margin for the rounding of u (hi + lo), of both MMAs'
                            // fp32 sums and of the epilogue arithmetic
                            const float2 ax = a.aux[(int64_t)g.b * a.Tq + g.t0 + q];
                            const float km = *s_kmax;
                            const float c = ax.y * km;
                            const float margin =
                                c + km * ax.x * 0x1p-14f + (fabsf(th) + c) * 0x1p-20f;
                            th = margin < INFINITY ? th - margin : -INFINITY;
                        }
                    }
                    if (g.t0 + q >= a.Tq) th = INFINITY;   // padding queries keep nothing
                    if (lane == 0) s_thr[q] = th;
                    __syncwarp();
                }
            }
            epi_sync();

            // ---- pass 2: keep every candidate with s >= theta ------------
            // s >= theta  <=>  s > below(theta), the next float down
            float thp[QPT];
#pragma unroll
            for (int x = 0; x < QPT; ++x) thp[x] = nextafterf(s_thr[q0 + x], -INFINITY);
            // this warp's survivor scores, [query x][lane]: the selection buffers
            // are idle during pass 2.  Where two tiles' worth fit (16 warps x 2 x
            // QPT x 32 floats), the survivors of a pair of tiles are staged
            // together, halving the per-tile votes and their latency.
            constexpr bool PAIR = 2 * EPI_WARPS * QPT * 32 * 4 <= SEL_WARPS * SELBUF * 8;
            float *scw0 = reinterpret_cast<float *>(sm + Lx::OFF_BUF) + e * (QPT * 32);
            float *scw1 = scw0 + (PAIR ? EPI_WARPS * QPT * 32 : 0);
            uint32_t hit_p = 0;  // survivors of the pair's first tile, not yet staged
            // survivors are staged per warp in shared memory (no atomic on the
            // way) and moved to the query lists in batches, one entry per lane
            uint64_t *stg_key = reinterpret_cast<uint64_t *>(sm + Lx::OFF_STGK) + e * STG_ENT;
            uint8_t *stg_x = sm + Lx::OFF_STGX + e * STG_ENT;
            int stg_n = 0;  // warp-uniform
            auto append = [&](int x, uint64_t key) {
                const int pos = atomicAdd(&s_cnt[q0 + x], 1);
                if (pos < CAP) lists[(size_t)(q0 + x) * CAP + pos] = key;
                if (pos == CAP - CHECK_EVERY * MB) *overflow = 1;
            };
            auto flush = [&]() {
                __syncwarp();
                for (int i = lane; i < stg_n; i += 32) append(stg_x[i], stg_key[i]);
                __syncwarp();
                stg_n = 0;
            };
            for (int kt = 0; kt < g.n_kt; ++kt, ++it) {
                const int tb = it & 1;
                sm100::mbar_wait(&tfull[tb], (it >> 1) & 1, abort_flag, a.wait_limit, a.ws);
                sm100::tc_fence_after();
                const int j = kt * MB + p;
                const bool tail = (int64_t)kt * MB + MB > g.c_min;
                const uint32_t taddr =
                    tmem_base + ((uint32_t)(lq * 32) << 16) + tb * NCOL + cq * (NCOL / 4);
                uint32_t hit = 0;
                float *scw = (kt & 1) ? scw1 : scw0;
                {
                    constexpr int CW = 16;  // columns per load: 16 values live at a time
                    constexpr int NCH = NCOL / 4 / CW;
#pragma unroll
                    for (int ch = 0; ch < NCH; ++ch) {
                        uint32_t v[CW];
                        sm100::tmem_ld16(taddr + CW * ch, v);
#pragma unroll
                        for (int qq = 0; qq < CW / HI; ++qq) {
                            const int x = ch * (CW / HI) + qq;
                            const float s = score_of<HI>(v + qq * HI, s_w[q0 + x]);
                            if (s > thp[x]) {
                                hit |= 1u << (QPT - 1 - x);
                                scw[x * 32 + lane] = s;
                            }
                        }
                    }
                }
                // the TMEM buffer is free before the appends: they only need the
                // mask and the parked scores
                sm100::tc_fence_before();
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&tempty[tb]);
                if (tail) {  // blocks past a query's causal limit drop out
                    uint32_t vm = 0;
#pragma unroll
                    for (int x = 0; x < QPT; ++x) vm = (vm << 1) | (uint32_t)(j < s_c[q0 + x]);
                    hit &= vm;
                }
                // the pair's first tile waits for its second (list checks fall on
                // second tiles: CHECK_EVERY is even)
                if (PAIR && !(kt & 1) && kt + 1 != g.n_kt) {
                    hit_p = hit;
                    continue;
                }
                if (__any_sync(0xffffffffu, (hit | hit_p) != 0)) {  // most tiles at long range
                    // this lane's offset among the warp's survivors: the count's
                    // bit planes by ballot (independent votes, no shuffle chain)
                    const int nl = __popc(hit) + __popc(hit_p);
                    const uint32_t lt = (1u << lane) - 1u;
                    int excl, tot;
                    if (g.lb && !__any_sync(0xffffffffu, nl > 1)) {  // long rows: one per lane
                        const uint32_t bal = __ballot_sync(0xffffffffu, nl);
                        excl = __popc(bal & lt);
                        tot = __popc(bal);
                    } else {
                        excl = 0;
                        tot = 0;
#pragma unroll
                        for (int bb = 0; (1 << bb) <= (PAIR ? 2 * QPT : QPT); ++bb) {
                            const uint32_t bal = __ballot_sync(0xffffffffu, (nl >> bb) & 1);
                            excl += __popc(bal & lt) << bb;
                            tot += __popc(bal) << bb;
                        }
                    }
                    const int incl = excl + nl;
                    if (stg_n + tot > STG_ENT) flush();
                    if (tot > STG_ENT) {  // only with heavy ties: append directly
                        while (hit_p) {
                            const int b = 31 - __clz(hit_p);
                            hit_p &= ~(1u << b);
                            const int x = QPT - 1 - b;
                            append(x, idx::make_key(scw0[x * 32 + lane], j - MB));
                        }
                        while (hit) {
                            const int b = 31 - __clz(hit);
                            hit &= ~(1u << b);
                            const int x = QPT - 1 - b;
                            append(x, idx::make_key(scw[x * 32 + lane], j));
                        }
                    } else {
                        int o = stg_n + incl - nl;
                        while (hit_p) {  // the pair's first tile: parked in scw0
                            const int b = 31 - __clz(hit_p);
                            hit_p &= ~(1u << b);
                            const int x = QPT - 1 - b;
                            stg_key[o] = idx::make_key(scw0[x * 32 + lane], j - MB);
                            stg_x[o] = (uint8_t)x;
                            ++o;
                        }
                        while (hit) {
                            const int b = 31 - __clz(hit);
                            hit &= ~(1u << b);
                            const int x = QPT - 1 - b;
                            stg_key[o] = idx::make_key(scw[x * 32 + lane], j);
                            stg_x[o] = (uint8_t)x;
                            ++o;
                        }
                        stg_n += tot;
                    }
                }
                hit_p = 0;
                // lists are checked every CHECK_EVERY tiles: a list below
                // CAP - CHECK_EVERY * MB at a check cannot overflow before the next
                if ((kt + 1) % CHECK_EVERY != 0 && kt + 1 != g.n_kt) continue;
                flush();
                epi_sync();
                if (*overflow) {  // uniform: read after the barrier, set only before it
                    if (selw) {
#pragma unroll 1
                        for (int q = e; q < QT; q += SEL_WARPS) {
                            const int n = s_cnt[q];
                            if (n > CAP - CHECK_EVERY * MB) {
                                const int nn = n < CAP ? n : CAP;
                                uint64_t *lst = lists + (size_t)q * CAP;
                                const uint64_t kth = idx::warp_kth_largest(lst, nn, K, hist, lane);
                                const int m = idx::warp_compact_ge(lst, nn, kth, lane);
                                if (lane == 0) {
                                    s_cnt[q] = m;
                                    // strict from now on: later blocks lose equal-score ties
                                    s_thr[q] = nextafterf(key_score((uint32_t)(kth >> 32)),
                                                          INFINITY);
                                }
                                __syncwarp();
                            }
                        }
                    }
                    epi_sync();
                    if (etid == 0) *overflow = 0;
#pragma unroll
                    for (int x = 0; x < QPT; ++x) thp[x] = nextafterf(s_thr[q0 + x], -INFINITY);
                    epi_sync();
                }
            }

            // ---- finalise: kb - 1 best, ascending by block, own block last
            const bool aborted = *abort_flag != 0;
            if (selw) {
#pragma unroll 1
                for (int q = e; q < QT; q += SEL_WARPS) {
                    const int64_t t = g.t0 + q;
                    if (t >= a.Tq) break;
                    const int c = s_c[q];
                    int n = s_cnt[q] < CAP ? s_cnt[q] : CAP;
                    uint64_t *lst = lists + (size_t)q * CAP;
                    if (n > SELBUF) {  // rare: cut the list in place first
                        const uint64_t kth = idx::warp_kth_largest(lst, n, K, hist, lane);
                        n = idx::warp_compact_ge(lst, n, kth, lane);
                    }
                    // one asynchronous copy of the list (16-byte pieces, all in flight)
                    for (int x = 2 * lane; x < n; x += 64)
                        cp_async16(smem_u32(buf + x), lst + x, 16);
                    cp_async_commit();
                    cp_async_wait<0>();
                    __syncwarp();
                    int m = n;
                    if (n > K) {
                        const uint64_t kth =
                            idx::warp_kth_largest_bisect<SELBUF / 32>(buf, n, K, hist, lane);
                        m = idx::warp_compact_ge(buf, n, kth, lane);
                    }
                    // re-key as (block << 32 | score key) and sort by block
                    for (int x = lane; x < m; x += 32) {
                        const uint64_t k = buf[x];
                        buf[x] = ((uint64_t)(uint32_t)idx::key_block(k) << 32) | (k >> 32);
                    }
                    __syncwarp();
                    const uint64_t *sorted = idx::warp_radix_sort_hi32(
                        buf, buf + SELBUF / 2, m, sort_passes, hist9, lane);
                    if (!aborted) {
                        int32_t *srow = a.sel + ((int64_t)g.b * a.Tq + t) * a.kb;
                        float *sc = a.sel_score ? a.sel_score + ((int64_t)g.b * a.Tq + t) * a.kb
                                                : nullptr;
                        for (int x = lane; x < a.kb; x += 32) {
                            int32_t id;
                            float v;
                            if (x < m) {
                                id = (int32_t)(sorted[x] >> 32);
                                v = key_score((uint32_t)sorted[x]);
                            } else if (x == m) {
                                id = c;
                                v = INFINITY;
                            } else {
                                id = -1;
                                v = -INFINITY;
                            }
                            srow[x] = id;
                            if (sc) sc[x] = v;
                        }
                    }
                    __syncwarp();
                }
            }
            epi_sync();
        }
    }

    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem_base, L<HI, DI>::TMEM_COLS);
    }
}

// ------------------------------------------------------------------- host --
// Bound on any single wait inside the kernel (ns); QSA_DEBUG_WAIT_NS overrides
// it so tests can make a wait run out on purpose.
static uint64_t wait_limit() {
    static uint64_t lim = [] {
        const char *s = getenv("QSA_DEBUG_WAIT_NS");
        return s ? (uint64_t)strtoull(s, nullptr, 10) : 2000000000ull;
    }();
    return lim;
}

static int lb_min_kt() {
    static int v = [] {
        const char *s = getenv("QSA_INDEX_LB_MIN_KT");
        return s ? atoi(s) : LB_MIN_KT;
    }();
    return v;
}

template <int HI>
static int grid_for(int B, int64_t Tq) {
    const int64_t qt = L<HI, 64>::QT;
    const int64_t tiles = (int64_t)B * ((Tq + qt - 1) / qt);
    return (int)(tiles < MAX_GRID ? (tiles > 0 ? tiles : 1) : MAX_GRID);
}

// Workspace after the status header: per CTA the candidate lists and group
// maxima, then (Hi >= 2) the pass-1 operand u as hi/lo bf16 rows
// [B * Tq * 2, Di], the per-query aux pairs and the max|Kp| partials.
template <int HI>
static size_t lists_bytes(int B, int64_t Tq) {
    const size_t per_cta = (size_t)L<HI, 64>::QT * (CAP * 8 + MAX_GROUPS * MB * 2);
    return (size_t)grid_for<HI>(B, Tq) * per_cta;
}
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

template <int HI>
static size_t ws_bytes(int B, int64_t Tq) {
    size_t n = kWsHeader + lists_bytes<HI>(B, Tq);
    if (HI >= 2) {
        n = align256(n) + align256((size_t)B * Tq * 2 * 64 * 2);   // u (Di <= 64)
        n += align256((size_t)B * Tq * sizeof(float2)) + KMAX_PARTS * sizeof(float);
    }
    return n;
}

template <int HI, int DI>
static cudaError_t launch(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                          const int64_t *q_pos0, int B, int64_t Tq, int64_t n_blocks, int kb,
                          int32_t *sel, float *sel_score, void *ws, int num_sms,
                          cudaStream_t s) {
    using Lx = L<HI, DI>;
    auto kern = idx_tc_kernel<HI, DI>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), Lx::ALLOC);
    if (e != cudaSuccess) return e;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    const int64_t rows = (int64_t)B * Tq;
    size_t off = align256(kWsHeader + lists_bytes<HI>(B, Tq));
    uint16_t *uu = reinterpret_cast<uint16_t *>(wsb + off);
    off += align256((size_t)rows * 2 * 64 * 2);
    float2 *aux = reinterpret_cast<float2 *>(wsb + off);
    off += align256((size_t)rows * sizeof(float2));
    float *kmax_part = reinterpret_cast<float *>(wsb + off);
    CUtensorMap tm_kp, tm_q, tm_u;
    if (!tensor_map_2d_bf16(&tm_kp, kp, (uint64_t)B * (uint64_t)n_blocks, DI, MB) ||
        !tensor_map_2d_bf16(&tm_q, q_idx, (uint64_t)rows * HI, DI, Lx::NCOL))
        return cudaErrorInvalidValue;
    if (Lx::LB) {
        if (!tensor_map_2d_bf16(&tm_u, uu, (uint64_t)rows * 2, DI, Lx::UCOL))
            return cudaErrorInvalidValue;
        const int n_qcta = (int)(rows < 8 * 4 * num_sms ? (rows + 7) / 8 : 4 * num_sms);
        ubound_kernel<HI, DI><<<n_qcta + KMAX_PARTS, 256, 0, s>>>(
            q_idx, w, rows, kp, (int64_t)B * n_blocks * DI / 8, uu, aux, kmax_part, n_qcta);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    } else {
        tm_u = tm_q;  // unused
    }
    Args a;
    a.w = w;
    a.aux = aux;
    a.kmax_part = kmax_part;
    a.q_pos0 = q_pos0;
    a.B = B;
    a.Tq = Tq;
    a.n_blocks = n_blocks;
    a.kb = kb;
    a.sel = sel;
    a.sel_score = sel_score;
    a.ws = wsb;
    a.n_qt = (int)((Tq + Lx::QT - 1) / Lx::QT);
    a.total_tiles = a.n_qt * B;
    a.wait_limit = wait_limit();
    a.lb_min_kt = lb_min_kt();
    a.grid = grid_for<HI>(B, Tq);  // the workspace is laid out for this many CTAs
    int grid = a.grid < num_sms ? a.grid : num_sms;
    kern<<<grid, THREADS, Lx::ALLOC, s>>>(tm_kp, tm_q, tm_u, a);
    return cudaGetLastError();
}

}  // namespace itc

size_t index_tc_ws_bytes(int B, int64_t Tq, int Hi) {
    if (Hi == 1) return itc::ws_bytes<1>(B, Tq);
    if (Hi == 2) return itc::ws_bytes<2>(B, Tq);
    return itc::ws_bytes<4>(B, Tq);
}

int index_tc_max_keep() { return itc::MAX_KEEP; }

cudaError_t launch_index_topk_tc(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                                 const int64_t *q_pos0, int B, int64_t Tq, int64_t n_blocks,
                                 int Hi, int Di, int kb, int32_t *sel, float *sel_score, void *ws,
                                 int num_sms, cudaStream_t s) {
    if (Tq == 0) return cudaSuccess;
    if (n_blocks == 0)  // no complete block: nothing to score
        return launch_own_block_only(q_pos0, nullptr, B, Tq, 0, kb, sel, sel_score, ws, s);
#define QSA_ITC(HI_, DI_)        \
    if (Hi == HI_ && Di == DI_)  \
        return itc::launch<HI_, DI_>(q_idx, w, kp, q_pos0, B, Tq, n_blocks, kb, sel, sel_score, \
                                     ws, num_sms, s);
    QSA_ITC(1, 32) QSA_ITC(2, 32) QSA_ITC(4, 32) QSA_ITC(1, 64) QSA_ITC(2, 64) QSA_ITC(4, 64)
#undef QSA_ITC
    return cudaErrorInvalidValue;
}

}  // namespace qsa
