// Decode-step indexer: one query per sequence against all of its pooled keys.
//
// Same definition as the prefill indexer ("用125亿分之6的参数，打平3970亿的旗舰
// 模型", section "稀疏注意力：给检索建索引，也得先学会省纸"; "On the Design of
// Qwen3.8-Next Architecture", token-mixing paragraph):
//   s(j) = sum_h w[h] * max(0, q_idx[h, :] . Kp[j, :]),  j < floor(p / r),
//   keep the kb - 1 best (s desc, j asc) + own block, ascending, -1 padded.
//
// The step streams every pooled key of every sequence once (8 MiB per 256K
// sequence) and is HBM-bound.  Pass 1 splits each sequence's candidates
// across CTAs: 64-block tiles are staged with cp.async, each warp scores 16
// blocks per tile with mma.sync (A = pooled keys, B = the query's heads as
// N = 8 columns, zero-padded), the ReLU-weighted head sum is finished with two
// lane shuffles, and the CTA keeps its split's kb - 1 best keys with a radix
// select.  Pass 2 merges the splits of each sequence exactly (radix select,
// then a bitonic sort by block index).
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {

namespace idd {

constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr int NB = 64;            // blocks per stage
constexpr int STAGES = 3;
constexpr int CHB = 4096;         // candidate blocks per split CTA
constexpr int MERGE_THREADS = 512;

QSA_DEVICE uint64_t make_key(float s, int j) {
    return ((uint64_t)score_key(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
}

// Block-wide radix select: the K-th largest of n unique keys (1 <= K <= n).
// `hist` holds 256 counters, `sh` four ints, `red` one u64 per warp; all threads
// must call.
QSA_DEVICE uint64_t block_kth_largest(const uint64_t *keys, int n, int K, uint32_t *hist,
                                      int *sh, uint64_t *red) {
    const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31;
    uint64_t prefix = 0;
    int want = K;
#pragma unroll 1
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += nth) hist[i] = 0;
        __syncthreads();
        const uint64_t hi_mask = (shift == 56) ? 0ull : (~0ull << (shift + 8));
        for (int i = tid; i < n; i += nth) {
            const uint64_t k = keys[i];
            if ((k & hi_mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            uint32_t local[8], sum = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                local[b] = hist[lane * 8 + b];
                sum += local[b];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
                if (lane + off < 32) incl += y;
            }
            uint32_t cum = incl - sum;
            int found = -1, nw = 0;
#pragma unroll
            for (int b = 7; b >= 0; --b) {
                if (found < 0 && (int)cum < want && want <= (int)(cum + local[b])) {
                    found = lane * 8 + b;
                    nw = want - (int)cum;
                }
                cum += local[b];
            }
            if (found >= 0) {
                sh[0] = found;
                sh[1] = nw;
                sh[3] = (int)local[found - lane * 8];
            }
        }
        __syncthreads();
        prefix |= (uint64_t)(uint32_t)sh[0] << shift;
        want = sh[1];
        const int bucket = sh[3];
        __syncthreads();
        if (shift > 0 && bucket == want) {
            // every key of this bucket is kept: the K-th largest is its minimum
            const uint64_t m = ~0ull << shift;
            uint64_t mn = ~0ull;
            for (int i = tid; i < n; i += nth) {
                const uint64_t k = keys[i];
                if ((k & m) == prefix && k < mn) mn = k;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const uint64_t o = __shfl_xor_sync(0xffffffffu, mn, off);
                mn = o < mn ? o : mn;
            }
            if (lane == 0) red[tid >> 5] = mn;
            __syncthreads();
            mn = ~0ull;
            for (int i = 0; i < nth / 32; ++i) mn = red[i] < mn ? red[i] : mn;
            __syncthreads();
            return mn;
        }
    }
    return prefix;
}

template <int HI, int DI>
__global__ void __launch_bounds__(THREADS, 3)
    decode_split_kernel(const uint16_t *__restrict__ q_idx, const float *__restrict__ w,
                        const uint16_t *__restrict__ kp, const int32_t *__restrict__ seqlens,
                        int64_t n_blocks, int kb, int nsplit, uint64_t *__restrict__ part_keys,
                        int *__restrict__ part_cnt, void *ws) {
    constexpr int ROWB = DI * 2, CH = DI / 8, KSTEPS = DI / 16;
    constexpr int STAGE_BYTES = NB * ROWB;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    __shared__ uint32_t hist[256];
    __shared__ int sh[4];
    __shared__ uint64_t red[THREADS / 32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;
    const int b = blockIdx.x / nsplit, split = blockIdx.x % nsplit;
    const int K = kb - 1;

    int64_t p = (int64_t)seqlens[b] - 1;
    int64_t c = p >= 0 ? p / 4 : 0;
    if (p < 0 || c > n_blocks) {
        if (tid == 0) record_status(ws, QSA_ERR_DEVICE);
        c = c > n_blocks ? n_blocks : c;
    }
    const int64_t j0 = (int64_t)split * CHB;
    int64_t j1 = j0 + CHB;
    if (j1 > c) j1 = c;
    const int n = j1 > j0 ? (int)(j1 - j0) : 0;

    // query heads as B fragments (N = 8 columns, heads >= HI are zero)
    uint32_t bq[KSTEPS][2];
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
        uint32_t v0 = 0, v1 = 0;
        if (lr < HI) {
            const uint16_t *qh = q_idx + ((int64_t)b * HI + lr) * DI + ks * 16 + 2 * lc;
            v0 = *reinterpret_cast<const uint32_t *>(qh);
            v1 = *reinterpret_cast<const uint32_t *>(qh + 8);
        }
        bq[ks][0] = v0;
        bq[ks][1] = v1;
    }
    float w0 = 0.f, w1 = 0.f;  // weights of heads 2*lc and 2*lc + 1
    if (2 * lc < HI) w0 = w[(int64_t)b * HI + 2 * lc];
    if (2 * lc + 1 < HI) w1 = w[(int64_t)b * HI + 2 * lc + 1];

    const int n_tiles = (n + NB - 1) / NB;
    const uint16_t *kpb = kp + ((int64_t)b * n_blocks + j0) * DI;
    auto load_tile = [&](int kt) {
        if (kt < n_tiles) {
            uint8_t *dst = smem + (kt % STAGES) * STAGE_BYTES;
            for (int i = tid; i < NB * CH; i += THREADS) {
                const int row = i / CH, ch = i % CH;
                const int jj = kt * NB + row;
                const bool ok = jj < n;
                const int sw = ch ^ ((row / (8 / CH)) & (CH - 1));
                cp_async16(smem_u32(dst + row * ROWB + sw * 16),
                           ok ? kpb + (int64_t)jj * DI + ch * 8 : kp, ok ? 16 : 0);
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
        const uint8_t *st = smem + (kt % STAGES) * STAGE_BYTES;
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
        if (lc == 0) {
            const int r0 = kt * NB + warp * 16 + lr, r1 = r0 + 8;
            if (r0 < n) keys[r0] = make_key(s0, (int)(j0 + r0));
            if (r1 < n) keys[r1] = make_key(s1, (int)(j0 + r1));
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // keep the split's K best
    uint64_t *out = part_keys + ((int64_t)b * nsplit + split) * K;
    if (n <= K) {
        for (int i = tid; i < n; i += THREADS) out[i] = keys[i];
        if (tid == 0) part_cnt[b * nsplit + split] = n;
        return;
    }
    const uint64_t kth = block_kth_largest(keys, n, K, hist, sh, red);
    if (tid == 0) sh[2] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += THREADS) {
        const uint64_t k = keys[i];
        if (k >= kth) out[atomicAdd(&sh[2], 1)] = k;
    }
    if (tid == 0) part_cnt[b * nsplit + split] = K;
}

__global__ void __launch_bounds__(MERGE_THREADS)
    decode_merge_kernel(const uint64_t *__restrict__ part_keys, const int *__restrict__ part_cnt,
                        const int32_t *__restrict__ seqlens, int64_t n_blocks, int kb,
                        int nsplit, int cap_n, int32_t *__restrict__ sel,
                        float *__restrict__ sel_score) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem);   // [cap_n] gathered split keys
    uint64_t *sorted = keys + cap_n;                        // [<= 1024] kept keys
    __shared__ uint32_t hist[256];
    __shared__ int sh[4];
    __shared__ uint64_t red[MERGE_THREADS / 32];
    const int tid = threadIdx.x;
    const int b = blockIdx.x;
    const int K = kb - 1;
    int64_t p = (int64_t)seqlens[b] - 1;
    int64_t c = p >= 0 ? p / 4 : 0;
    if (c > n_blocks) c = n_blocks;

    int n = 0;
    for (int s = 0; s < nsplit; ++s) {
        const int cnt = part_cnt[b * nsplit + s];
        const uint64_t *src = part_keys + ((int64_t)b * nsplit + s) * K;
        for (int i = tid; i < cnt; i += MERGE_THREADS) keys[n + i] = src[i];
        n += cnt;
    }
    __syncthreads();
    if (n > K) {
        const uint64_t kth = block_kth_largest(keys, n, K, hist, sh, red);
        if (tid == 0) sh[2] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += MERGE_THREADS) {
            const uint64_t k = keys[i];
            if (k >= kth) sorted[atomicAdd(&sh[2], 1)] = k;
        }
        n = K;
    } else {
        for (int i = tid; i < n; i += MERGE_THREADS) sorted[i] = keys[i];
    }
    __syncthreads();
    // re-key by block index and sort ascending
    int P = 1;
    while (P < n) P <<= 1;
    for (int i = tid; i < P; i += MERGE_THREADS) {
        uint64_t v = ~0ull;
        if (i < n) {
            const uint64_t k = sorted[i];
            v = ((uint64_t)(0xFFFFFFFFu - (uint32_t)k) << 32) | (k >> 32);
        }
        sorted[i] = v;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1)
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            for (int pr = tid; pr < P / 2; pr += MERGE_THREADS) {
                const int i = (pr / jj) * 2 * jj + (pr % jj), ixj = i + jj;
                const uint64_t a = sorted[i], bb = sorted[ixj];
                if ((a > bb) == ((i & k) == 0)) {
                    sorted[i] = bb;
                    sorted[ixj] = a;
                }
            }
            __syncthreads();
        }
    for (int i = tid; i < kb; i += MERGE_THREADS) {
        int32_t id;
        float v;
        if (i < n) {
            id = (int32_t)(sorted[i] >> 32);
            v = key_score((uint32_t)sorted[i]);
        } else if (i == n) {
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

// Gathered split keys the merge CTA holds in shared memory (<= 25600).
int index_decode_merge_cap(int64_t n_blocks, int kb) {
    const int64_t n = (int64_t)decode_nsplit(n_blocks) * (kb > 1 ? kb - 1 : 1);
    return n > 25600 ? -1 : (int)n;
}

size_t index_decode_ws_bytes(int B, int64_t n_blocks, int kb, int /*num_sms*/) {
    const int ns = decode_nsplit(n_blocks);
    size_t keys = (size_t)B * ns * (size_t)(kb > 1 ? kb - 1 : 1) * sizeof(uint64_t);
    size_t cnts = (size_t)B * ns * sizeof(int);
    return kWsHeader + ((keys + 255) / 256) * 256 + cnts;
}

template <int HI, int DI>
static cudaError_t launch_dec(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                              const int32_t *seqlens, int B, int64_t n_blocks, int kb,
                              int32_t *sel, float *sel_score, void *ws, cudaStream_t s) {
    const int ns = decode_nsplit(n_blocks);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    const size_t keys_bytes = (size_t)B * ns * (size_t)(kb > 1 ? kb - 1 : 1) * sizeof(uint64_t);
    uint64_t *part_keys = reinterpret_cast<uint64_t *>(wsb + kWsHeader);
    int *part_cnt = reinterpret_cast<int *>(wsb + kWsHeader + ((keys_bytes + 255) / 256) * 256);
    constexpr int smem1 = idd::STAGES * idd::NB * DI * 2 + idd::CHB * 8;
    auto k1 = idd::decode_split_kernel<HI, DI>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
    if (e != cudaSuccess) return e;
    if (kb == 1) {  // own block only: no candidate is kept
        e = cudaMemsetAsync(part_cnt, 0, (size_t)B * ns * sizeof(int), s);
        if (e != cudaSuccess) return e;
    } else {
        k1<<<B * ns, idd::THREADS, smem1, s>>>(q_idx, w, kp, seqlens, n_blocks, kb, ns, part_keys,
                                                part_cnt, ws);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int cap_n = index_decode_merge_cap(n_blocks, kb);
    const int smem2 = (cap_n + 1024) * 8;
    e = cudaFuncSetAttribute(idd::decode_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem2);
    if (e != cudaSuccess) return e;
    idd::decode_merge_kernel<<<B, idd::MERGE_THREADS, smem2, s>>>(part_keys, part_cnt, seqlens,
                                                                   n_blocks, kb, ns, cap_n, sel,
                                                                   sel_score);
    return cudaGetLastError();
}


cudaError_t launch_index_topk_decode(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                                     const int32_t *seqlens, int B, int64_t n_blocks, int Hi,
                                     int Di, int kb, int32_t *sel, float *sel_score, void *ws,
                                     int /*num_sms*/, cudaStream_t s) {
#define QSA_DEC(HI_, DI_)          \
    if (Hi == HI_ && Di == DI_)    \
        return launch_dec<HI_, DI_>(q_idx, w, kp, seqlens, B, n_blocks, kb, sel, sel_score, ws, s);
    QSA_DEC(1, 32) QSA_DEC(2, 32) QSA_DEC(4, 32) QSA_DEC(1, 64) QSA_DEC(2, 64) QSA_DEC(4, 64)
#undef QSA_DEC
    return cudaErrorInvalidValue;
}

}  // namespace qsa
