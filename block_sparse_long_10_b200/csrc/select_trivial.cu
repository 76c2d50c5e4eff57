// Selection when there is nothing to rank: no complete micro-block exists
// (n_blocks == 0, every position below r = 4), so every query keeps its own
// block and nothing else ("用125亿分之6的参数，打平3970亿的旗舰模型", section
// "稀疏注意力：给检索建索引，也得先学会省纸": the own block is always kept).
// Same row format as the indexers: own block first, -1 padding; scores +inf
// for the own block, -inf for padding.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {

namespace {

__global__ void own_block_only_kernel(const int64_t *__restrict__ q_pos0,
                                      const int32_t *__restrict__ seqlens, int B, int64_t Tq,
                                      int64_t n_blocks, int kb, int32_t *__restrict__ sel,
                                      float *__restrict__ sel_score, void *status) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= (int64_t)B * Tq * kb) return;
    const int x = (int)(i % kb);
    const int64_t row = i / kb;
    const int64_t b = row / Tq;
    int64_t p;
    if (seqlens) {  // decode: one query per sequence at position seqlens[b] - 1
        p = (int64_t)seqlens[b] - 1;
        if (p < 0 && x == 0) record_status(status, QSA_ERR_DEVICE);
    } else {
        p = (q_pos0 ? q_pos0[b] : 0) + (row - b * Tq);
    }
    int64_t c = p >= 0 ? p / 4 : 0;
    if (c > n_blocks) {
        if (x == 0) record_status(status, QSA_ERR_DEVICE);
        c = n_blocks;
    }
    sel[i] = x == 0 ? (int32_t)c : -1;
    if (sel_score) sel_score[i] = x == 0 ? INFINITY : -INFINITY;
}

}  // namespace

cudaError_t launch_own_block_only(const int64_t *q_pos0, const int32_t *seqlens, int B, int64_t Tq,
                                  int64_t n_blocks, int kb, int32_t *sel, float *sel_score,
                                  void *status, cudaStream_t s) {
    const int64_t n = (int64_t)B * Tq * kb;
    if (n == 0) return cudaSuccess;
    own_block_only_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        q_pos0, seqlens, B, Tq, n_blocks, kb, sel, sel_score, status);
    return cudaGetLastError();
}

}  // namespace qsa
