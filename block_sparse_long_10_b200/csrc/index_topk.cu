// Lightweight MQA indexer: fused block scores + exact top-k selection.
//
// "用125亿分之6的参数，打平3970亿的旗舰模型", section
// "稀疏注意力：给检索建索引，也得先学会省纸": a lightweight MQA indexer (several
// query heads, one shared pooled key head) gives every micro-block a score and
// the highest-scoring blocks are kept; it follows DSA's lightweight indexer.
// "On the Design of Qwen3.8-Next Architecture" (token-mixing paragraph):
// indexing O(n^2 / r), token budget 2048.
//
//   s(t, j) = sum_h w[t, h] * max(0, q_idx[t, h, :] . Kp[j, :])   (fp32)
//   keep the kb - 1 best j < floor(p / r) by (s desc, j asc) + own block.
//
// Scores are never written to memory.  One CTA owns a tile of 64 consecutive
// queries (16 per warp) and sweeps the pooled keys in ascending 64-block
// tiles (cp.async ring in shared memory, L2-resident source).  Each warp keeps
// its queries' indexer vectors as mma.sync A fragments in registers and gets
// s(t, j) for 2 queries x 2 blocks x all heads per thread per 8-block slice,
// so the ReLU-weighted head sum happens in registers.
//
// Selection is exact.  Per query, candidates whose score beats a running
// threshold are appended to a list in the workspace (64-bit keys: order-
// preserving score bits above the complemented block index).  When a list
// could overflow it is compacted to its kb - 1 best keys by a warp-wide radix
// select, and the threshold rises to the smallest kept score.  Because blocks
// are swept in ascending order, a later candidate with a score equal to the
// threshold always loses the index tie-break, so "score > threshold" is an
// exact filter.  At the end the list is reduced to its kb - 1 best keys,
// sorted by block index (bitonic), and written out with the own block.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {

namespace idx {

constexpr int QT = 64;       // queries per CTA tile
constexpr int WARPS = 4;     // 16 queries per warp
constexpr int THREADS = WARPS * 32;
constexpr int NB = 64;       // pooled blocks per shared-memory tile
constexpr int STAGES = 3;
constexpr int CAP = 1024;    // candidate-list capacity per query
constexpr int MAX_KEEP = 511;  // kb - 1 <= 511 (CAP >= 2 * (MAX_KEEP + NB) - ...)

template <int DI>
struct Smem {
    static constexpr int ROWB = DI * 2;
    static constexpr int CH = ROWB / 16;
    static constexpr int STAGE_BYTES = NB * ROWB;
    static constexpr int OFF_STAGE = 0;
    static constexpr int OFF_THR = STAGES * STAGE_BYTES;
    static constexpr int OFF_CNT = OFF_THR + QT * 4;
    static constexpr int OFF_HIST = OFF_CNT + QT * 4;
    static constexpr int OFF_BUF = OFF_HIST + WARPS * 256 * 4;
    static constexpr int BYTES = OFF_BUF + WARPS * CAP * 8;
};

// XOR swizzle of 16-byte chunks so 8 consecutive rows read by ldmatrix hit 8
// distinct bank groups.
template <int DI>
QSA_DEVICE int swz(int row, int chunk) {
    constexpr int CH = DI / 8;
    return chunk ^ ((row / (8 / CH)) & (CH - 1));
}

// ---- warp-level radix select: the K-th largest of n unique u64 keys ------
QSA_DEVICE uint64_t warp_kth_largest(const uint64_t *buf, int n, int K, uint32_t *hist,
                                     int lane) {
    uint64_t prefix = 0;
    int want = K;
#pragma unroll 1
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        const uint64_t hi_mask = (shift == 56) ? 0ull : (~0ull << (shift + 8));
        for (int i = lane; i < n; i += 32) {
            const uint64_t k = buf[i];
            if ((k & hi_mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
        __syncwarp();
        uint32_t local[8];
        uint32_t sum = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            local[b] = hist[lane * 8 + b];
            sum += local[b];
        }
        uint32_t incl = sum;  // sum over lanes >= this lane
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
            if (lane + off < 32) incl += y;
        }
        uint32_t cum = incl - sum;  // keys in higher digits than this lane's bins
        int found = -1, new_want = 0;
#pragma unroll
        for (int b = 7; b >= 0; --b) {
            if (found < 0 && (int)cum < want && want <= (int)(cum + local[b])) {
                found = lane * 8 + b;
                new_want = want - (int)cum;
            }
            cum += local[b];
        }
        const uint32_t ball = __ballot_sync(0xffffffffu, found >= 0);
        const int src = __ffs(ball) - 1;
        const uint32_t bucket = __shfl_sync(0xffffffffu, found >= 0 ? hist[found] : 0u, src);
        found = __shfl_sync(0xffffffffu, found, src);
        want = __shfl_sync(0xffffffffu, new_want, src);
        prefix |= (uint64_t)(uint32_t)found << shift;
        __syncwarp();
        if (shift > 0 && (int)bucket == want) {
            // every key of this bucket is kept: the K-th largest is its minimum
            const uint64_t m = ~0ull << shift;
            uint64_t mn = ~0ull;
            for (int i = lane; i < n; i += 32) {
                const uint64_t k = buf[i];
                if ((k & m) == prefix && k < mn) mn = k;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const uint64_t o = __shfl_xor_sync(0xffffffffu, mn, off);
                mn = o < mn ? o : mn;
            }
            return mn;
        }
    }
    return prefix;
}

// Keep the keys >= kth (exactly K of them) at the front of buf; returns count.
QSA_DEVICE int warp_compact_ge(uint64_t *buf, int n, uint64_t kth, int lane) {
    int base = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const uint64_t k = (i < n) ? buf[i] : 0ull;
        const bool keep = (i < n) && (k >= kth);
        const uint32_t m = __ballot_sync(0xffffffffu, keep);
        if (keep) buf[base + __popc(m & ((1u << lane) - 1u))] = k;
        base += __popc(m);
    }
    __syncwarp();
    return base;
}

QSA_DEVICE void warp_bitonic_sort(uint64_t *buf, int P, int lane) {
    for (int k = 2; k <= P; k <<= 1) {
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            for (int pr = lane; pr < P / 2; pr += 32) {
                const int i = (pr / jj) * 2 * jj + (pr % jj);
                const int ixj = i + jj;
                const uint64_t a = buf[i], b = buf[ixj];
                const bool up = (i & k) == 0;
                if ((a > b) == up) {
                    buf[i] = b;
                    buf[ixj] = a;
                }
            }
            __syncwarp();
        }
    }
}

QSA_DEVICE uint64_t make_key(float s, int j) {
    return ((uint64_t)score_key(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
}
QSA_DEVICE int key_block(uint64_t k) { return (int)(0xFFFFFFFFu - (uint32_t)k); }

template <int HI, int DI>
__global__ void __launch_bounds__(THREADS, 2)
    index_topk_kernel(const uint16_t *__restrict__ q_idx, const float *__restrict__ w,
                      const uint16_t *__restrict__ kp, const int64_t *__restrict__ q_pos0,
                      int B, int64_t Tq, int64_t n_blocks, int kb,
                      int32_t *__restrict__ sel, float *__restrict__ sel_score,
                      uint8_t *__restrict__ ws, int n_qt, int total_tiles) {
    using S = Smem<DI>;
    constexpr int KSTEPS = DI / 16;
    constexpr int CH = S::CH;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *stage_base = smem + S::OFF_STAGE;
    float *thr = reinterpret_cast<float *>(smem + S::OFF_THR);
    int *cnt = reinterpret_cast<int *>(smem + S::OFF_CNT);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem + S::OFF_HIST) + warp * 256;
    uint64_t *buf = reinterpret_cast<uint64_t *>(smem + S::OFF_BUF) + (size_t)warp * CAP;
    __shared__ int s_tile;

    int *tile_counter = reinterpret_cast<int *>(ws + kWsCounters);
    uint64_t *lists = reinterpret_cast<uint64_t *>(ws + kWsHeader) +
                      (size_t)blockIdx.x * QT * CAP;
    const int K = kb - 1;

    for (;;) {
        if (tid == 0) s_tile = atomicAdd(tile_counter, 1);
        __syncthreads();
        const int tile = s_tile;
        if (tile >= total_tiles) break;
        const int b = tile % B;
        const int qt = n_qt - 1 - tile / B;  // longest query tiles first
        const int64_t t0 = (int64_t)qt * QT;
        const int64_t pos_base = q_pos0 ? q_pos0[b] : 0;

        if (tid < QT) {
            thr[tid] = K > 0 ? -INFINITY : INFINITY;  // kb == 1: own block only
            cnt[tid] = 0;
        }

        // this thread's two queries: rows lr and lr + 8 of the warp's 16
        int64_t tq[2];
        int64_t cq[2];
        float wv[2][HI];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            tq[e] = t0 + warp * 16 + lr + e * 8;
            cq[e] = 0;
#pragma unroll
            for (int h = 0; h < HI; ++h) wv[e][h] = 0.f;
            if (tq[e] < Tq) {
                int64_t c = (pos_base + tq[e]) / 4;
                if (pos_base + tq[e] < 0) c = 0;
                if (c > n_blocks) {
                    record_status(ws, QSA_ERR_DEVICE);
                    c = n_blocks;
                }
                cq[e] = c;
                const float *wr = w + ((int64_t)b * Tq + tq[e]) * HI;
#pragma unroll
                for (int h = 0; h < HI; ++h) wv[e][h] = wr[h];
            }
        }
        // A fragments of the warp's 16 queries for every head and k-step
        uint32_t afr[HI][KSTEPS][4];
#pragma unroll
        for (int h = 0; h < HI; ++h)
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int row = e & 1;        // a0: lr, a1: lr+8, a2: lr, a3: lr+8
                    const int dof = (e >> 1) * 8; // a2/a3: dims + 8
                    const int64_t t = tq[row];
                    uint32_t v = 0;
                    if (t < Tq)
                        v = *reinterpret_cast<const uint32_t *>(
                            q_idx + (((int64_t)b * Tq + t) * HI + h) * DI + ks * 16 + dof +
                            2 * lc);
                    afr[h][ks][e] = v;
                }
        // candidate range of the whole tile
        const int64_t t_last = (t0 + QT - 1 < Tq) ? t0 + QT - 1 : Tq - 1;
        int64_t c_max = (pos_base + t_last) / 4;
        if (pos_base + t_last < 0) c_max = 0;
        if (c_max > n_blocks) c_max = n_blocks;
        const int n_tiles = (int)((c_max + NB - 1) / NB);
        __syncthreads();

        auto load_tile = [&](int kt) {
            if (kt < n_tiles) {
                uint8_t *dst = stage_base + (kt % STAGES) * S::STAGE_BYTES;
                for (int i = tid; i < NB * CH; i += THREADS) {
                    const int row = i / CH, ch = i % CH;
                    const int64_t j = (int64_t)kt * NB + row;
                    const bool ok = j < c_max;
                    const uint16_t *src = ok ? kp + ((int64_t)b * n_blocks + j) * DI + ch * 8 : kp;
                    cp_async16(smem_u32(dst + row * S::ROWB + swz<DI>(row, ch) * 16), src,
                               ok ? 16 : 0);
                }
            }
            cp_async_commit();
        };
#pragma unroll
        for (int s = 0; s < STAGES - 1; ++s) load_tile(s);

#pragma unroll 1
        for (int kt = 0; kt < n_tiles; ++kt) {
            cp_async_wait<STAGES - 2>();
            __syncthreads();
            load_tile(kt + STAGES - 1);

            // keep every list of this warp below CAP - NB before the tile
#pragma unroll 1
            for (int qq = 0; qq < 16; ++qq) {
                const int q = warp * 16 + qq;
                const int n = cnt[q];
                if (n > CAP - NB) {
                    uint64_t *lst = lists + (size_t)q * CAP;
                    for (int i = lane; i < n; i += 32) buf[i] = lst[i];
                    __syncwarp();
                    const uint64_t kth = warp_kth_largest(buf, n, K, hist, lane);
                    const int m = warp_compact_ge(buf, n, kth, lane);
                    for (int i = lane; i < m; i += 32) lst[i] = buf[i];
                    __syncwarp();
                    if (lane == 0) {
                        cnt[q] = m;
                        thr[q] = key_score((uint32_t)(kth >> 32));
                    }
                    __syncwarp();
                }
            }
            const float th0 = thr[warp * 16 + lr], th1 = thr[warp * 16 + lr + 8];

            const uint8_t *st = stage_base + (kt % STAGES) * S::STAGE_BYTES;
#pragma unroll 1
            for (int pass = 0; pass < NB / 16; ++pass) {
                float acc[2][HI][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int h = 0; h < HI; ++h)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[nt][h][e] = 0.f;
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const int mi = lane >> 3, rr = lane & 7;
                    const int row = pass * 16 + (mi >> 1) * 8 + rr;
                    const int ch = ks * 2 + (mi & 1);
                    uint32_t b00, b01, b10, b11;
                    ldmatrix_x4(smem_u32(st + row * S::ROWB + swz<DI>(row, ch) * 16), b00, b01,
                                b10, b11);
#pragma unroll
                    for (int h = 0; h < HI; ++h) {
                        mma_bf16_16816(acc[0][h], afr[h][ks][0], afr[h][ks][1], afr[h][ks][2],
                                       afr[h][ks][3], b00, b01);
                        mma_bf16_16816(acc[1][h], afr[h][ks][0], afr[h][ks][1], afr[h][ks][2],
                                       afr[h][ks][3], b10, b11);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int qi = e >> 1;
                        const int64_t j = (int64_t)kt * NB + pass * 16 + nt * 8 + 2 * lc + (e & 1);
                        float s = 0.f;
#pragma unroll
                        for (int h = 0; h < HI; ++h) s = fmaf(wv[qi][h], fmaxf(acc[nt][h][e], 0.f), s);
                        if (j < cq[qi] && s > (qi ? th1 : th0)) {
                            const int q = warp * 16 + lr + qi * 8;
                            const int pos = atomicAdd(&cnt[q], 1);
                            lists[(size_t)q * CAP + pos] = make_key(s, (int)j);
                        }
                    }
                }
            }
        }
        cp_async_wait<0>();
        __syncthreads();

        // ---- finalise this warp's 16 queries -------------------------------
#pragma unroll 1
        for (int qq = 0; qq < 16; ++qq) {
            const int q = warp * 16 + qq;
            const int64_t t = t0 + q;
            if (t >= Tq) break;
            int64_t c = (pos_base + t) / 4;
            if (pos_base + t < 0) c = 0;
            if (c > n_blocks) c = n_blocks;
            const int n = cnt[q];
            const uint64_t *lst = lists + (size_t)q * CAP;
            for (int i = lane; i < n; i += 32) buf[i] = lst[i];
            __syncwarp();
            int m = n;
            if (n > K) {
                const uint64_t kth = warp_kth_largest(buf, n, K, hist, lane);
                m = warp_compact_ge(buf, n, kth, lane);
            }
            // re-key by block index for the ascending sort
            int P = 1;
            while (P < m) P <<= 1;
            for (int i = lane; i < P; i += 32) {
                uint64_t v = ~0ull;
                if (i < m) {
                    const uint64_t k = buf[i];
                    v = ((uint64_t)(uint32_t)key_block(k) << 32) | (k >> 32);
                }
                buf[i] = v;
            }
            __syncwarp();
            if (P > 1) warp_bitonic_sort(buf, P, lane);
            int32_t *srow = sel + ((int64_t)b * Tq + t) * kb;
            float *sc = sel_score ? sel_score + ((int64_t)b * Tq + t) * kb : nullptr;
            for (int i = lane; i < kb; i += 32) {
                int32_t id;
                float v;
                if (i < m) {
                    const uint64_t e = buf[i];
                    id = (int32_t)(e >> 32);
                    v = key_score((uint32_t)e);
                } else if (i == m) {
                    id = (int32_t)c;
                    v = INFINITY;
                } else {
                    id = -1;
                    v = -INFINITY;
                }
                srow[i] = id;
                if (sc) sc[i] = v;
            }
            __syncwarp();
        }
        __syncthreads();
    }
}

}  // namespace idx

size_t index_topk_ws_bytes(int grid) {
    return kWsHeader + (size_t)grid * idx::QT * idx::CAP * sizeof(uint64_t);
}

int index_topk_max_keep() { return idx::MAX_KEEP; }

template <int HI, int DI>
static cudaError_t launch_idx(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                              const int64_t *q_pos0, int B, int64_t Tq, int64_t n_blocks,
                              int kb, int32_t *sel, float *sel_score, uint8_t *ws, int grid,
                              cudaStream_t s) {
    using S = idx::Smem<DI>;
    auto kern = idx::index_topk_kernel<HI, DI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         S::BYTES);
    if (e != cudaSuccess) return e;
    const int n_qt = (int)((Tq + idx::QT - 1) / idx::QT);
    const int total = n_qt * B;
    e = cudaMemsetAsync(ws + kWsCounters, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
    kern<<<grid, idx::THREADS, S::BYTES, s>>>(q_idx, w, kp, q_pos0, B, Tq, n_blocks, kb, sel,
                                              sel_score, ws, n_qt, total);
    return cudaGetLastError();
}

int index_topk_grid(int num_sms) { return num_sms * 2; }

cudaError_t launch_index_topk(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                              const int64_t *q_pos0, int B, int64_t Tq, int64_t n_blocks,
                              int Hi, int Di, int kb, int32_t *sel, float *sel_score,
                              void *ws, int grid, cudaStream_t s) {
    uint8_t *wsb = static_cast<uint8_t *>(ws);
#define QSA_IDX_CASE(HI_, DI_)                                                              \
    if (Hi == HI_ && Di == DI_)                                                             \
        return launch_idx<HI_, DI_>(q_idx, w, kp, q_pos0, B, Tq, n_blocks, kb, sel, sel_score, \
                                    wsb, grid, s);
    QSA_IDX_CASE(1, 32)
    QSA_IDX_CASE(2, 32)
    QSA_IDX_CASE(4, 32)
    QSA_IDX_CASE(1, 64)
    QSA_IDX_CASE(2, 64)
    QSA_IDX_CASE(4, 64)
#undef QSA_IDX_CASE
    return cudaErrorInvalidValue;
}

}  // namespace qsa
