// Decode-step indexer: one query per sequence against all of its pooled keys.
//
// Same definition as the prefill indexer ("用125亿分之6的参数，打平3970亿的旗舰
// 模型", section "稀疏注意力：给检索建索引，也得先学会省纸"; "On the Design of
// Qwen3.8-Next Architecture", token-mixing paragraph):
//   s(j) = sum_h w[h] * max(0, q_idx[h, :] . Kp[j, :]),  j < floor(p / r),
//   keep the kb - 1 best (s desc, j asc) + own block, ascending, -1 padded.
//
// The step streams every pooled key of every sequence once (8 MiB per 256K
// sequence) and is HBM-bound; the scores themselves are small (256 KiB per
// sequence), so they are written out and selected in a second, L2-resident
// pass:
//   A  split CTAs stream 128-block tiles of pooled keys (TMA, 128-byte
//      swizzle, 4-stage ring); each warp takes 16 blocks per tile through
//      mma.sync (A = pooled keys, B = the query's heads as 8 zero-padded
//      columns), finishes the ReLU-weighted head sum with two lane shuffles,
//      writes the scores and keeps a running maximum per thread.  The
//      per-thread maxima are distinct candidates' scores, so the (kb-1)-th
//      largest of them is a lower bound theta of the (kb-1)-th best score.
//   B  one CTA per sequence computes theta, gathers the candidates with
//      score >= theta into shared memory (a few hundred on random data; an
//      exact radix select over all scores handles overflow), selects the
//      kb - 1 best exactly and sorts them by block index.
#include <stdlib.h>

#include "qsa_common.cuh"
#include "qsa_launch.h"
#include "sm100.cuh"
#include "topk_warp.cuh"

namespace qsa {

namespace idd {

constexpr int WARPS = 8;
constexpr int THREADS = WARPS * 32;
constexpr int NB = 128;            // blocks per tile (16 per warp)
constexpr int STAGES = 4;
constexpr int CHB = 2048;          // candidate blocks per split CTA
constexpr int GROUPS_PER_CTA = THREADS / 4;  // one running maximum per (warp, quad)
constexpr int SEL_THREADS = 1024;
constexpr int LIST_CAP = 8192;     // survivors held in shared memory
constexpr uint64_t WAIT_NS = 2000000000ull;

QSA_DEVICE uint64_t make_key(float s, int j) {
    return ((uint64_t)score_key(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
}

// Work item = (sequence, split).  Candidate range of one item.
struct DecItem {
    int b, n, n_tiles;
    int64_t row0;
};

QSA_DEVICE DecItem dec_item(int item, int nsplit, const int32_t *seqlens, int64_t n_blocks,
                            void *ws, bool report) {
    DecItem d;
    d.b = item / nsplit;
    const int split = item % nsplit;
    const int64_t p = (int64_t)seqlens[d.b] - 1;
    int64_t c = p >= 0 ? p / 4 : 0;
    if (p < 0 || c > n_blocks) {
        if (report && split == 0) record_status(ws, QSA_ERR_DEVICE);
        c = c > n_blocks ? n_blocks : c;
    }
    const int64_t j0 = (int64_t)split * CHB;
    int64_t j1 = j0 + CHB;
    if (j1 > c) j1 = c;
    d.n = j1 > j0 ? (int)(j1 - j0) : 0;
    d.n_tiles = (d.n + NB - 1) / NB;
    d.row0 = (int64_t)d.b * n_blocks + j0;
    return d;
}

// Persistent: CTA k takes items k, k + gridDim.x, ...; one TMA ring runs
// across item boundaries so the stream never drains.
template <int HI, int DI>
__global__ void __launch_bounds__(THREADS, 3)
    decode_score_kernel(const __grid_constant__ CUtensorMap tm_kp, const uint16_t *__restrict__ q_idx,
                        const float *__restrict__ w, const int32_t *__restrict__ seqlens,
                        int64_t n_blocks, int nsplit, int n_items, float *__restrict__ scores,
                        uint32_t *__restrict__ gmax, void *ws) {
    griddep_wait();  // inputs (pooled keys, queries, lengths) of earlier kernels
    constexpr int ROWB = DI * 2, CH = DI / 8, KSTEPS = DI / 16;
    constexpr int TILE = NB * ROWB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + STAGES * TILE);
    __shared__ int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) sm100::mbar_init(&full[s], 1);
        s_abort = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();

    // producer cursor (thread 0): next (item, tile) to load
    int p_item = blockIdx.x, p_kt = 0;
    DecItem pd;
    if (tid == 0 && p_item < n_items) pd = dec_item(p_item, nsplit, seqlens, n_blocks, ws, false);
    uint32_t issued = 0;
    auto issue_next = [&]() {
        if (tid != 0) return;
        while (p_item < n_items && p_kt >= pd.n_tiles) {  // skip to an item with tiles left
            p_item += gridDim.x;
            p_kt = 0;
            if (p_item < n_items) pd = dec_item(p_item, nsplit, seqlens, n_blocks, ws, false);
        }
        if (p_item >= n_items || s_abort) return;
        const int s = issued % STAGES;
        sm100::mbar_arrive_expect_tx(&full[s], TILE);
        sm100::tma_load_2d(sm + s * TILE, &tm_kp, 0, (int32_t)(pd.row0 + (int64_t)p_kt * NB),
                           &full[s]);
        ++issued;
        ++p_kt;
    };
    for (int k = 0; k < STAGES; ++k) issue_next();

    uint32_t consumed = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const DecItem d = dec_item(item, nsplit, seqlens, n_blocks, ws, tid == 0);
        // query heads as B fragments (N = 8 columns, heads >= HI are zero)
        uint32_t bq[KSTEPS][2];
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
            uint32_t v0 = 0, v1 = 0;
            if (lr < HI) {
                const uint16_t *qh = q_idx + ((int64_t)d.b * HI + lr) * DI + ks * 16 + 2 * lc;
                v0 = *reinterpret_cast<const uint32_t *>(qh);
                v1 = *reinterpret_cast<const uint32_t *>(qh + 8);
            }
            bq[ks][0] = v0;
            bq[ks][1] = v1;
        }
        float w0 = 0.f, w1 = 0.f;  // weights of heads 2*lc and 2*lc + 1
        if (2 * lc < HI) w0 = w[(int64_t)d.b * HI + 2 * lc];
        if (2 * lc + 1 < HI) w1 = w[(int64_t)d.b * HI + 2 * lc + 1];

        float run_max = -INFINITY;
        for (int kt = 0; kt < d.n_tiles; ++kt, ++consumed) {
            const int s = consumed % STAGES;
            sm100::mbar_wait(&full[s], (consumed / STAGES) & 1, (volatile int *)&s_abort,
                             WAIT_NS, ws);
            const uint8_t *st = sm + s * TILE;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                const int mi = lane >> 3;
                const int row = warp * 16 + (mi & 1) * 8 + (lane & 7);
                const int ch = ks * 2 + (mi >> 1);
                const int sw = ch ^ ((row / (8 / CH)) & (CH - 1));
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(smem_u32(st + row * ROWB + sw * 16), a0, a1, a2, a3);
                mma_bf16_16816(acc, a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
            }
            // rows (blocks) lr and lr + 8; columns (heads) 2lc, 2lc + 1
            float s0 = w0 * fmaxf(acc[0], 0.f) + w1 * fmaxf(acc[1], 0.f);
            float s1 = w0 * fmaxf(acc[2], 0.f) + w1 * fmaxf(acc[3], 0.f);
            s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
            s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
            const int r0 = kt * NB + warp * 16 + lr, r1 = r0 + 8;
            if (r0 < d.n) run_max = fmaxf(run_max, s0);
            if (r1 < d.n) run_max = fmaxf(run_max, s1);
            if (lc == 0) {
                if (r0 < d.n) scores[d.row0 + r0] = s0;
                if (r1 < d.n) scores[d.row0 + r1] = s1;
            }
            __syncthreads();  // every warp is done with this stage
            issue_next();
        }
        // one maximum per (warp, lr): the four lanes of a quad hold the same value
        if (lc == 0) gmax[(int64_t)item * GROUPS_PER_CTA + warp * 8 + lr] = score_key(run_max);
    }
    if (tid == 0 && s_abort) {
        // after a timed-out wait, let this CTA's own copies in flight land (bounded)
        for (uint32_t k = consumed; k < issued; ++k)
            sm100::mbar_wait_for(&full[k % STAGES], (k / STAGES) & 1, 100000000ull);
    }
}

// ---- block-wide selection helpers (SEL_THREADS threads) -------------------
QSA_DEVICE void block_hist_add(uint32_t *hist, uint32_t digit, bool active, int lane) {
    (void)lane;
    if (active) atomicAdd(&hist[digit], 1u);
}

// K-th largest of n unique u64 keys produced by key_at(i); all threads call.
template <class KeyAt>
QSA_DEVICE uint64_t block_kth_largest(KeyAt key_at, int n, int K, uint32_t *hist, int *sh,
                                      uint64_t *red) {
    const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31, warp = tid >> 5;
    uint64_t mn = ~0ull, mx = 0ull;  // the highest bit on which the keys differ
    for (int i = tid; i < n; i += nth) {
        const uint64_t k = key_at(i);
        mn = k < mn ? k : mn;
        mx = k > mx ? k : mx;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t a = __shfl_xor_sync(0xffffffffu, mn, off);
        const uint64_t c = __shfl_xor_sync(0xffffffffu, mx, off);
        mn = a < mn ? a : mn;
        mx = c > mx ? c : mx;
    }
    if (lane == 0) {
        red[warp] = mn;
        red[32 + warp] = mx;
    }
    __syncthreads();
    mn = ~0ull;
    mx = 0ull;
    for (int i = 0; i < nth / 32; ++i) {
        mn = red[i] < mn ? red[i] : mn;
        mx = red[32 + i] > mx ? red[32 + i] : mx;
    }
    __syncthreads();
    if (mn == mx || K >= n) return mn;
    if (K == 1) return mx;
    int top = 63 - __clzll((long long)(mn ^ mx));
    uint64_t prefix = top >= 63 ? 0ull : (mn & (~0ull << (top + 1)));
    int want = K;
    for (;;) {
        const int shift = top - 7;
        const uint64_t hm = top >= 63 ? 0ull : (~0ull << (top + 1));
        for (int i = tid; i < 256; i += nth) hist[i] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < n; i0 += nth) {
            const int i = i0 + tid;
            const uint64_t k = i < n ? key_at(i) : 0ull;
            const bool m = i < n && (k & hm) == prefix;
            const uint32_t d = (uint32_t)((shift >= 0 ? (k >> shift) : (k << -shift)) & 255u);
            block_hist_add(hist, d, m, lane);
        }
        __syncthreads();
        if (tid < 32) {
            uint32_t local[8], sum = 0;
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) {
                local[bb] = hist[lane * 8 + bb];
                sum += local[bb];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
                if (lane + off < 32) incl += y;
            }
            uint32_t cum = incl - sum;
#pragma unroll
            for (int bb = 7; bb >= 0; --bb) {
                if ((int)cum < want && want <= (int)(cum + local[bb])) {
                    sh[0] = lane * 8 + bb;
                    sh[1] = want - (int)cum;
                    sh[2] = (int)local[bb];
                }
                cum += local[bb];
            }
        }
        __syncthreads();
        const int found = sh[0];
        want = sh[1];
        const int cnt = sh[2];
        __syncthreads();
        prefix |= shift >= 0 ? ((uint64_t)(uint32_t)found << shift)
                             : ((uint64_t)(uint32_t)found >> -shift);
        if (shift <= 0) return prefix;
        if (cnt == want) {  // bucket kept whole: its minimum is the answer
            const uint64_t m2 = ~0ull << shift;
            uint64_t bmin = ~0ull;
            for (int i = tid; i < n; i += nth) {
                const uint64_t k = key_at(i);
                if ((k & m2) == prefix && k < bmin) bmin = k;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const uint64_t a = __shfl_xor_sync(0xffffffffu, bmin, off);
                bmin = a < bmin ? a : bmin;
            }
            if (lane == 0) red[warp] = bmin;
            __syncthreads();
            bmin = ~0ull;
            for (int i = 0; i < nth / 32; ++i) bmin = red[i] < bmin ? red[i] : bmin;
            __syncthreads();
            return bmin;
        }
        top = shift - 1;
    }
}

// One CTA per sequence: block-wide radix selects, a parallel survivor scan,
// and a rank sort (each thread counts the kept blocks below its own).
__global__ void __launch_bounds__(SEL_THREADS)
    decode_select_kernel(const float *__restrict__ scores, const uint32_t *__restrict__ gmax,
                         const int32_t *__restrict__ seqlens, int64_t n_blocks, int kb,
                         int nsplit, int32_t *__restrict__ sel, float *__restrict__ sel_score) {
    griddep_wait();  // the scores and maxima of the scoring kernel
    extern __shared__ __align__(16) uint8_t smem[];
    uint64_t *list = reinterpret_cast<uint64_t *>(smem);  // [LIST_CAP] survivors
    uint64_t *kept = list + LIST_CAP;                      // [1024] kept keys
    uint64_t *sorted = kept + 1024;                        // [512] by block, then scratch
    __shared__ uint32_t hist[256];
    __shared__ int sh[4];
    __shared__ uint64_t red[64];
    __shared__ int s_cnt;
    const int tid = threadIdx.x;
    const int b = blockIdx.x;
    const int K = kb - 1;
    int64_t p = (int64_t)seqlens[b] - 1;
    int64_t c = p >= 0 ? p / 4 : 0;
    if (c > n_blocks) c = n_blocks;
    const int n = (int)c;
    const float *sc = scores + (int64_t)b * n_blocks;
    // any subset of the group maxima still bounds the (kb-1)-th best score
    const int G = nsplit * GROUPS_PER_CTA < LIST_CAP ? nsplit * GROUPS_PER_CTA : LIST_CAP;
    const uint32_t *gm = gmax + (int64_t)b * nsplit * GROUPS_PER_CTA;

    int m = 0;
    if (K > 0 && n > 0) {
        // theta: the (kb-1)-th largest group maximum
        __shared__ float s_theta;
        if (tid == 0) s_theta = -INFINITY;
        if (n > K && G >= K) {
            for (int i = tid; i < G; i += SEL_THREADS) list[i] = ((uint64_t)gm[i] << 32) | (uint32_t)i;
            __syncthreads();
            const uint64_t kth =
                block_kth_largest([&](int i) { return list[i]; }, G, K, hist, sh, red);
            if (tid == 0) s_theta = key_score((uint32_t)(kth >> 32));
        }
        if (tid == 0) s_cnt = 0;
        __syncthreads();
        const float theta = s_theta;
        // survivors: score >= theta; 16 independent loads in flight per thread
        constexpr int U = 16;
        for (int j0 = 0; j0 < n; j0 += U * SEL_THREADS) {
            float v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + u * SEL_THREADS + tid;
                v[u] = j < n ? sc[j] : -INFINITY;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + u * SEL_THREADS + tid;
                if (j < n && v[u] >= theta) {
                    const int pos = atomicAdd(&s_cnt, 1);
                    if (pos < LIST_CAP) list[pos] = make_key(v[u], j);
                }
            }
        }
        __syncthreads();
        const int cnt = s_cnt;
        __syncthreads();
        uint64_t kth = 0;
        if (cnt <= LIST_CAP) {
            if (cnt > K) kth = block_kth_largest([&](int i) { return list[i]; }, cnt, K, hist, sh, red);
        } else {  // many ties at theta: exact select over every score
            kth = block_kth_largest([&](int i) { return make_key(sc[i], i); }, n, K, hist, sh,
                                    red);
        }
        if (tid == 0) s_cnt = 0;
        __syncthreads();
        if (cnt <= LIST_CAP) {
            for (int i = tid; i < cnt; i += SEL_THREADS) {
                const uint64_t k = list[i];
                if (k >= kth) kept[atomicAdd(&s_cnt, 1)] = k;
            }
        } else {
            for (int j = tid; j < n; j += SEL_THREADS) {
                const uint64_t k = make_key(sc[j], j);
                if (k >= kth) kept[atomicAdd(&s_cnt, 1)] = k;
            }
        }
        __syncthreads();
        m = s_cnt;  // <= K
        const int words = (n + 31) / 32;
        if (words <= LIST_CAP * 2) {
            // counting sort by block id: one bit per kept block, rank = number of
            // set bits below it (chunk prefix per thread + popcounts in the chunk)
            uint32_t *bm = reinterpret_cast<uint32_t *>(list);
            uint32_t *chunk_pre = reinterpret_cast<uint32_t *>(sorted + 512);  // [SEL_THREADS]
            const int per = (words + SEL_THREADS - 1) / SEL_THREADS;
            for (int i = tid; i < words; i += SEL_THREADS) bm[i] = 0;
            __syncthreads();
            if (tid < m) {
                const uint32_t jb = 0xFFFFFFFFu - (uint32_t)kept[tid];
                atomicOr(&bm[jb >> 5], 1u << (jb & 31));
            }
            __syncthreads();
            uint32_t cnt_t = 0;
            for (int wv = tid * per; wv < (tid + 1) * per && wv < words; ++wv) cnt_t += __popc(bm[wv]);
            chunk_pre[tid] = cnt_t;
            __syncthreads();
            if (tid < 32) {  // exclusive scan of the SEL_THREADS chunk counts
                uint32_t run = 0;
                for (int base = 0; base < SEL_THREADS; base += 32) {
                    const uint32_t x = chunk_pre[base + tid];
                    uint32_t incl = x;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
                        if (tid >= off) incl += y;
                    }
                    chunk_pre[base + tid] = run + incl - x;
                    run += __shfl_sync(0xffffffffu, incl, 31);
                }
            }
            __syncthreads();
            if (tid < m) {
                const uint64_t k = kept[tid];
                const uint32_t jb = 0xFFFFFFFFu - (uint32_t)k;
                const int wd = (int)(jb >> 5), ck = wd / per;
                uint32_t rank = chunk_pre[ck];
                for (int wv = ck * per; wv < wd; ++wv) rank += __popc(bm[wv]);
                rank += __popc(bm[wd] & ((1u << (jb & 31)) - 1u));
                sorted[rank] = k;
            }
        } else if (tid < m) {  // very long caches: rank by direct counting
            const uint64_t k = kept[tid];
            const uint32_t jb = 0xFFFFFFFFu - (uint32_t)k;
            int rank = 0;
            for (int i = 0; i < m; ++i) rank += (0xFFFFFFFFu - (uint32_t)kept[i]) < jb;
            sorted[rank] = k;
        }
        __syncthreads();
    }
    for (int i = tid; i < kb; i += SEL_THREADS) {
        int32_t id;
        float v;
        if (i < m) {
            id = (int32_t)(0xFFFFFFFFu - (uint32_t)sorted[i]);
            v = key_score((uint32_t)(sorted[i] >> 32));
        } else if (i == m) {
            id = (int32_t)c;
            v = INFINITY;
        } else {
            id = -1;
            v = -INFINITY;
        }
        sel[(int64_t)b * kb + i] = id;
        if (sel_score) sel_score[(int64_t)b * kb + i] = v;
    }
}

}  // namespace idd

static int decode_nsplit(int64_t n_blocks) {
    int64_t ns = (n_blocks + idd::CHB - 1) / idd::CHB;
    return (int)(ns < 1 ? 1 : ns);
}

// The selection kernel's shared list is fixed-size; only the block count's
// range limits the decode indexer.
int index_decode_merge_cap(int64_t n_blocks, int kb) {
    (void)kb;
    return n_blocks <= ((int64_t)1 << 30) ? 1 : -1;
}

size_t index_decode_ws_bytes(int B, int64_t n_blocks, int kb, int /*num_sms*/) {
    (void)kb;
    const int ns = decode_nsplit(n_blocks);
    const size_t scores = (((size_t)B * (size_t)n_blocks * 4) + 255) / 256 * 256;
    const size_t gm = (size_t)B * ns * idd::GROUPS_PER_CTA * 4;
    return kWsHeader + scores + gm;
}

template <int HI, int DI>
static cudaError_t launch_dec(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                              const int32_t *seqlens, int B, int64_t n_blocks, int kb,
                              int32_t *sel, float *sel_score, void *ws, int sms, cudaStream_t s) {
    const int ns = decode_nsplit(n_blocks);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    const size_t scores_bytes = (((size_t)B * (size_t)n_blocks * 4) + 255) / 256 * 256;
    float *scores = reinterpret_cast<float *>(wsb + kWsHeader);
    uint32_t *gmax = reinterpret_cast<uint32_t *>(wsb + kWsHeader + scores_bytes);
    CUtensorMap tm;
    if (!tensor_map_2d_bf16(&tm, kp, (uint64_t)B * (uint64_t)(n_blocks > 0 ? n_blocks : 1), DI,
                            idd::NB))
        return cudaErrorInvalidValue;
    constexpr int smem1 = idd::STAGES * idd::NB * DI * 2 + idd::STAGES * 8 + 1024;
    auto k1 = idd::decode_score_kernel<HI, DI>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(k1), smem1);
    if (e != cudaSuccess) return e;
    const int n_items = B * ns;
    const int grid = n_items < 3 * sms ? n_items : 3 * sms;
    e = launch_dependent(k1, dim3(grid), dim3(idd::THREADS), (size_t)smem1, s, tm, q_idx, w,
                         seqlens, n_blocks, ns, n_items, scores, gmax, ws);
    if (e != cudaSuccess) return e;
    const int smem2 = (idd::LIST_CAP + 2048) * 8;
    e = ensure_smem(reinterpret_cast<const void *>(idd::decode_select_kernel), smem2);
    if (e != cudaSuccess) return e;
    return launch_dependent(idd::decode_select_kernel, dim3(B), dim3(idd::SEL_THREADS),
                            (size_t)smem2, s, scores, (const uint32_t *)gmax, seqlens, n_blocks,
                            kb, ns, sel, sel_score);
}

cudaError_t launch_index_topk_decode(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                                     const int32_t *seqlens, int B, int64_t n_blocks, int Hi,
                                     int Di, int kb, int32_t *sel, float *sel_score, void *ws,
                                     int num_sms, cudaStream_t s) {
    if (n_blocks == 0)  // every cache shorter than one block: nothing to score
        return launch_own_block_only(nullptr, seqlens, B, 1, 0, kb, sel, sel_score, ws, s);
#define QSA_DEC(HI_, DI_)          \
    if (Hi == HI_ && Di == DI_)    \
        return launch_dec<HI_, DI_>(q_idx, w, kp, seqlens, B, n_blocks, kb, sel, sel_score, ws, \
                                    num_sms, s);
    QSA_DEC(1, 32) QSA_DEC(2, 32) QSA_DEC(4, 32) QSA_DEC(1, 64) QSA_DEC(2, 64) QSA_DEC(4, 64)
#undef QSA_DEC
    return cudaErrorInvalidValue;
}

}  // namespace qsa
