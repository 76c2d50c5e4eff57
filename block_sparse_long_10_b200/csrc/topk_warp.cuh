// Warp-level exact top-k helpers over unique 64-bit keys (order-preserving
// score bits above the complemented block index), shared by the indexers.
#pragma once

#include "qsa_common.cuh"

namespace qsa {
namespace idx {

// Histogram increment.  The radix passes start at the highest bit on which
// the keys differ, so digits spread over the bins and plain shared atomics
// see little contention.
QSA_DEVICE void hist_add(uint32_t *hist, uint32_t digit, bool active, int lane) {
    (void)lane;
    if (active) atomicAdd(&hist[digit], 1u);
}

QSA_DEVICE uint64_t warp_min_u64(uint64_t v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, v, off);
        v = o < v ? o : v;
    }
    return v;
}
QSA_DEVICE uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, v, off);
        v = o > v ? o : v;
    }
    return v;
}

// Radix select: the K-th largest of n unique keys (1 <= K <= n) in `buf`
// (shared or global memory).  The first 8-bit digit sits just below the
// highest bit on which the keys differ; later digits follow; the search stops
// as soon as the bucket holding the K-th key is kept whole (its minimum is
// then the answer).
QSA_DEVICE uint64_t warp_kth_largest(const uint64_t *buf, int n, int K, uint32_t *hist,
                                     int lane) {
    constexpr int U = 4;  // keys per lane loaded together (buf may be in global memory)
    uint64_t mn = ~0ull, mx = 0ull;
    for (int i0 = 0; i0 < n; i0 += 32 * U) {
        uint64_t kk[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * 32 + lane;
            kk[u] = i < n ? buf[i] : 0ull;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (i0 + u * 32 + lane < n) {
                mn = kk[u] < mn ? kk[u] : mn;
                mx = kk[u] > mx ? kk[u] : mx;
            }
        }
    }
    mn = warp_min_u64(mn);
    mx = warp_max_u64(mx);
    if (mn == mx || K >= n) return mn;
    if (K == 1) return mx;
    int top = 63 - __clzll((long long)(mn ^ mx));      // highest differing bit
    uint64_t prefix = top >= 63 ? 0ull : (mn & (~0ull << (top + 1)));
    int want = K;
#pragma unroll 1
    for (;;) {
        const int shift = top - 7;                       // window [shift, top]
        const uint64_t hm = top >= 63 ? 0ull : (~0ull << (top + 1));
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        for (int i0 = 0; i0 < n; i0 += 32 * U) {
            uint64_t kk[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u * 32 + lane;
                kk[u] = i < n ? buf[i] : 0ull;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u * 32 + lane;
                const uint64_t k = kk[u];
                const bool m = i < n && (k & hm) == prefix;
                const uint32_t d =
                    (uint32_t)((shift >= 0 ? (k >> shift) : (k << -shift)) & 255u);
                hist_add(hist, d, m, lane);
            }
        }
        __syncwarp();
        uint32_t local[8];
        uint32_t sum = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            local[b] = hist[lane * 8 + b];
            sum += local[b];
        }
        uint32_t incl = sum;  // keys in this lane's bins and above
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
            if (lane + off < 32) incl += y;
        }
        uint32_t cum = incl - sum;
        int found = -1, new_want = 0;
        uint32_t cnt = 0;
#pragma unroll
        for (int b = 7; b >= 0; --b) {
            if (found < 0 && (int)cum < want && want <= (int)(cum + local[b])) {
                found = lane * 8 + b;
                new_want = want - (int)cum;
                cnt = local[b];
            }
            cum += local[b];
        }
        const uint32_t ball = __ballot_sync(0xffffffffu, found >= 0);
        const int src = __ffs(ball) - 1;
        found = __shfl_sync(0xffffffffu, found, src);
        want = __shfl_sync(0xffffffffu, new_want, src);
        cnt = __shfl_sync(0xffffffffu, cnt, src);
        prefix |= shift >= 0 ? ((uint64_t)(uint32_t)found << shift)
                             : ((uint64_t)(uint32_t)found >> -shift);
        __syncwarp();
        if (shift <= 0) return prefix;                   // every bit decided
        if ((int)cnt == want) {                          // bucket kept whole
            const uint64_t m2 = ~0ull << shift;
            uint64_t bmin = ~0ull;
            for (int i0 = 0; i0 < n; i0 += 32 * U) {
                uint64_t kk[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = i0 + u * 32 + lane;
                    kk[u] = i < n ? buf[i] : ~0ull;
                }
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if ((kk[u] & m2) == prefix && kk[u] < bmin) bmin = kk[u];
            }
            return warp_min_u64(bmin);
        }
        top = shift - 1;
    }
}

// The K-th largest of n 32-bit (or 16-bit) keys (1 <= K <= n; equal keys
// allowed: the result is the K-th value counting multiplicity), same digit
// scheme.
template <typename KeyT>
QSA_DEVICE uint32_t warp_kth_largest_narrow(const KeyT *buf, int n, int K, uint32_t *hist,
                                            int lane) {
    uint32_t mn = ~0u, mx = 0u;
    for (int i = lane; i < n; i += 32) {
        const uint32_t k = buf[i];
        mn = k < mn ? k : mn;
        mx = k > mx ? k : mx;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    if (mn == mx || K >= n) return mn;
    if (K == 1) return mx;
    int top = 31 - __clz((int)(mn ^ mx));
    uint32_t prefix = top >= 31 ? 0u : (mn & (~0u << (top + 1)));
    int want = K;
#pragma unroll 1
    for (;;) {
        const int shift = top - 7;
        const uint32_t hm = top >= 31 ? 0u : (~0u << (top + 1));
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        for (int i0 = 0; i0 < n; i0 += 32) {
            const int i = i0 + lane;
            const uint32_t k = i < n ? buf[i] : 0u;
            const bool m = i < n && (k & hm) == prefix;
            const uint32_t d = (shift >= 0 ? (k >> shift) : (k << -shift)) & 255u;
            hist_add(hist, d, m, lane);
        }
        __syncwarp();
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
        int found = -1, new_want = 0;
        uint32_t cnt = 0;
#pragma unroll
        for (int b = 7; b >= 0; --b) {
            if (found < 0 && (int)cum < want && want <= (int)(cum + local[b])) {
                found = lane * 8 + b;
                new_want = want - (int)cum;
                cnt = local[b];
            }
            cum += local[b];
        }
        const uint32_t ball = __ballot_sync(0xffffffffu, found >= 0);
        const int src = __ffs(ball) - 1;
        found = __shfl_sync(0xffffffffu, found, src);
        want = __shfl_sync(0xffffffffu, new_want, src);
        cnt = __shfl_sync(0xffffffffu, cnt, src);
        prefix |= shift >= 0 ? ((uint32_t)found << shift) : ((uint32_t)found >> -shift);
        __syncwarp();
        if (shift <= 0) return prefix;
        if ((int)cnt == want) {  // bucket kept whole: its minimum is the answer
            const uint32_t m2 = ~0u << shift;
            uint32_t bmin = ~0u;
            for (int i = lane; i < n; i += 32) {
                const uint32_t k = buf[i];
                if ((k & m2) == prefix && k < bmin) bmin = k;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) bmin = min(bmin, __shfl_xor_sync(0xffffffffu, bmin, off));
            return bmin;
        }
        top = shift - 1;
    }
}

// The K-th largest of n <= 32 R unique 64-bit keys in shared memory
// (1 <= K <= n) with the high words held in registers: the K-th largest high
// word t is built bit by bit from the top (keep a bit when at least K high
// words are >= the prefix with it set), each step one predicated count per
// register and one warp sum, with no shared-memory atomics.  High words above
// t are all in; when the keys with high word t are exactly the rest, the K-th
// key is the smallest of them; otherwise (equal scores across the cut) the
// radix select above settles it.  Real keys have a nonzero high word (the
// score key of any score >= -inf), so the zero padding never counts.
template <int R>
QSA_DEVICE uint64_t warp_kth_largest_bisect(const uint64_t *buf, int n, int K, uint32_t *hist,
                                            int lane) {
    uint32_t hi[R];
    uint32_t mn = ~0u, mx = 0u;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int i = r * 32 + lane;
        hi[r] = i < n ? (uint32_t)(buf[i] >> 32) : 0u;
        if (i < n) {
            mn = min(mn, hi[r]);
            mx = max(mx, hi[r]);
        }
    }
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
    uint32_t t;
    if (mn == mx) {
        t = mn;
    } else {
        const int top = 31 - __clz((int)(mn ^ mx));
        t = top == 31 ? 0u : (mn & (~0u << (top + 1)));  // the bits every key shares
#pragma unroll 1
        for (int b = top; b >= 0; --b) {
            const uint32_t c = t | (1u << b);
            uint32_t cnt = 0;
#pragma unroll
            for (int r = 0; r < R; ++r) cnt += hi[r] >= c ? 1u : 0u;
            if ((int)__reduce_add_sync(0xffffffffu, cnt) >= K) t = c;
        }
    }
    uint32_t gt = 0, eq = 0, lo_min = ~0u;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        gt += hi[r] > t ? 1u : 0u;
        if (hi[r] == t) {
            ++eq;
            lo_min = min(lo_min, (uint32_t)buf[r * 32 + lane]);
        }
    }
    gt = __reduce_add_sync(0xffffffffu, gt);
    eq = __reduce_add_sync(0xffffffffu, eq);
    lo_min = __reduce_min_sync(0xffffffffu, lo_min);
    if ((int)(gt + eq) == K) return ((uint64_t)t << 32) | lo_min;
    return warp_kth_largest(buf, n, K, hist, lane);
}

// Keep the keys >= kth (exactly K of them) at the front of buf; returns count.
QSA_DEVICE int warp_compact_ge(uint64_t *buf, int n, uint64_t kth, int lane) {
    constexpr int U = 4;  // keys per lane loaded together (buf may be in global memory)
    int base = 0;
    for (int i0 = 0; i0 < n; i0 += 32 * U) {
        uint64_t kk[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * 32 + lane;
            kk[u] = i < n ? buf[i] : 0ull;
        }
        // every lane holds its batch before any lane writes (the writes only
        // move keys to lower positions, which this batch has already read)
        __syncwarp();
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * 32 + lane;
            const bool keep = (i < n) && (kk[u] >= kth);
            const uint32_t m = __ballot_sync(0xffffffffu, keep);
            if (keep) buf[base + __popc(m & ((1u << lane) - 1u))] = kk[u];
            base += __popc(m);
        }
    }
    __syncwarp();
    return base;
}

// Stable LSD radix sort (9-bit digits, 512-bin histogram: two passes cover
// block ids below 2^18) of m <= 1024 keys by their high 32 bits, which hold
// values below 2^(9*passes).  Ping-pongs between buf and tmp; returns the
// buffer that holds the result.
QSA_DEVICE uint64_t *warp_radix_sort_hi32(uint64_t *buf, uint64_t *tmp, int m, int passes,
                                            uint32_t *hist, int lane) {
    constexpr int NB = 512, PER = NB / 32;
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll 1
    for (int p = 0; p < passes; ++p) {
        const int sh = 32 + 9 * p;
        for (int i = lane; i < NB; i += 32) hist[i] = 0;
        __syncwarp();
        for (int i0 = 0; i0 < m; i0 += 32) {
            const int i = i0 + lane;
            const bool v = i < m;
            const uint64_t k = v ? buf[i] : 0ull;
            const uint32_t d = (uint32_t)(k >> sh) & (NB - 1);
            hist_add(hist, d, v, lane);
        }
        __syncwarp();
        uint32_t local[PER], sum = 0;
#pragma unroll
        for (int b = 0; b < PER; ++b) {
            local[b] = hist[lane * PER + b];
            sum += local[b];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        uint32_t run = incl - sum;
        __syncwarp();
#pragma unroll
        for (int b = 0; b < PER; ++b) {
            hist[lane * PER + b] = run;
            run += local[b];
        }
        __syncwarp();
        for (int i0 = 0; i0 < m; i0 += 32) {
            const int i = i0 + lane;
            const bool v = i < m;
            const uint64_t k = v ? buf[i] : 0ull;
            const uint32_t d = (uint32_t)(k >> sh) & (NB - 1);
            // lanes holding the same digit: one ballot per digit bit
            uint32_t peers = __ballot_sync(0xffffffffu, v);
#pragma unroll
            for (int b = 0; b < 9; ++b) {
                const uint32_t bal = __ballot_sync(0xffffffffu, (d >> b) & 1u);
                peers &= ((d >> b) & 1u) ? bal : ~bal;
            }
            uint32_t base = 0;
            if (v) {
                base = hist[d];
                tmp[base + __popc(peers & lt)] = k;
            }
            __syncwarp();
            if (v && __ffs(peers) - 1 == lane) hist[d] = base + __popc(peers);
            __syncwarp();
        }
        uint64_t *x = buf;
        buf = tmp;
        tmp = x;
    }
    return buf;
}

QSA_DEVICE uint64_t make_key(float s, int j) {
    return ((uint64_t)score_key(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
}
QSA_DEVICE int key_block(uint64_t k) { return (int)(0xFFFFFFFFu - (uint32_t)k); }

}  // namespace idx
}  // namespace qsa
