// Micro-block mean pooling of the indexer keys.
//
// "用125亿分之6的参数，打平3970亿的旗舰模型", section
// "稀疏注意力：给检索建索引，也得先学会省纸": consecutive tokens are packed into
// a micro-block and mean-pooled into one representative key; the paper
// summary "On the Design of Qwen3.8-Next Architecture" (token-mixing
// paragraph) fixes the compression ratio at 4.
//
// HBM-bound streaming kernel: one thread owns 8 dims (16 bytes) of one block,
// reads the four token rows with 16-byte non-allocating loads (consecutive
// threads read consecutive 16-byte chunks), sums in fp32 as
// ((k0 + k1) + (k2 + k3)), scales by 0.25 and rounds to bf16 nearest-even.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {

__global__ void __launch_bounds__(256) pool_r4_kernel(const uint16_t *__restrict__ k_idx,
                                                      int64_t T, int Di, int64_t j0,
                                                      int64_t nblk, int64_t N,
                                                      int64_t total,
                                                      uint16_t *__restrict__ kp) {
    const int chunks = Di >> 3;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(idx % chunks);
        const int64_t rest = idx / chunks;
        const int64_t j = j0 + rest % nblk;
        const int64_t b = rest / nblk;
        const uint16_t *src = k_idx + ((b * T + j * 4) * Di) + c * 8;
        uint4 x[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = ldg_stream(src + (int64_t)i * Di);
        const uint32_t *w0 = &x[0].x, *w1 = &x[1].x, *w2 = &x[2].x, *w3 = &x[3].x;
        uint32_t out[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __fmul_rn(__fadd_rn(__fadd_rn(bf16_lo(w0[e]), bf16_lo(w1[e])),
                                                 __fadd_rn(bf16_lo(w2[e]), bf16_lo(w3[e]))),
                                       0.25f);
            const float hi = __fmul_rn(__fadd_rn(__fadd_rn(bf16_hi(w0[e]), bf16_hi(w1[e])),
                                                 __fadd_rn(bf16_hi(w2[e]), bf16_hi(w3[e]))),
                                       0.25f);
            out[e] = pack_bf16x2(lo, hi);
        }
        *reinterpret_cast<uint4 *>(kp + (b * N + j) * Di + c * 8) =
            make_uint4(out[0], out[1], out[2], out[3]);
    }
}

cudaError_t launch_pool(const uint16_t *k_idx, int B, int64_t T, int Di, int64_t j0,
                        int64_t j1, uint16_t *kp, cudaStream_t s, int num_sms) {
    const int64_t nblk = j1 - j0;
    const int64_t total = (int64_t)B * nblk * (Di / 8);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    pool_r4_kernel<<<(unsigned)blocks, threads, 0, s>>>(k_idx, T, Di, j0, nblk, T / 4,
                                                          total, kp);
    return cudaGetLastError();
}

}  // namespace qsa
