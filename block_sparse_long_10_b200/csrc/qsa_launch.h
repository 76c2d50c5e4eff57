// Internal launch functions behind the C ABI (host side, not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

struct CUtensorMap_st;

namespace qsa {

// Host caches (host_util.cu).
cudaError_t ensure_smem(const void *kern, int bytes);

// Launch `kern` as a programmatic dependent of the previous kernel in `s`:
// its launch overlaps that kernel's tail; the kernel itself must call
// griddep_wait() before it reads anything the previous kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
bool tensor_map_2d_bf16(CUtensorMap_st *out, const void *base, uint64_t rows, uint32_t cols,
                        uint32_t box_rows);

cudaError_t launch_pool(const uint16_t *k_idx, int B, int64_t T, int Di, int64_t j0,
                        int64_t j1, uint16_t *kp, cudaStream_t s, int num_sms);

size_t index_tc_ws_bytes(int B, int64_t Tq, int Hi);
int index_tc_max_keep();
// Every query keeps only its own block (n_blocks == 0: no complete block yet).
// q_pos0/seqlens as in the indexers (seqlens != nullptr: decode, Tq = 1).
cudaError_t launch_own_block_only(const int64_t *q_pos0, const int32_t *seqlens, int B, int64_t Tq,
                                  int64_t n_blocks, int kb, int32_t *sel, float *sel_score,
                                  void *status, cudaStream_t s);
cudaError_t launch_index_topk_tc(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                                 const int64_t *q_pos0, int B, int64_t Tq, int64_t n_blocks,
                                 int Hi, int Di, int kb, int32_t *sel, float *sel_score, void *ws,
                                 int num_sms, cudaStream_t s);

size_t index_decode_ws_bytes(int B, int64_t n_blocks, int kb, int num_sms);
int index_decode_merge_cap(int64_t n_blocks, int kb);  // -1: too many splits
cudaError_t launch_index_topk_decode(const uint16_t *q_idx, const float *w, const uint16_t *kp,
                                     const int32_t *seqlens, int B, int64_t n_blocks, int Hi,
                                     int Di, int kb, int32_t *sel, float *sel_score, void *ws,
                                     int num_sms, cudaStream_t s);

int sparse_attn_blocks_per_stage(int Hkv);
cudaError_t launch_sparse_attn_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                       const int32_t *sel, const int64_t *q_pos0, int B,
                                       int64_t Tq, int64_t Tk, int Hq, int Hkv, int D, int kb,
                                       float scale, uint16_t *o, float *lse, int num_sms,
                                       cudaStream_t s);
cudaError_t launch_split_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                const int32_t *seqlens, int64_t L_max, const int32_t *sel,
                                int n_entries, int nsplit, int B, int Hq, int Hkv, int D,
                                float scale, uint16_t *o, float *lse, float *part,
                                void *status, int num_sms, cudaStream_t s);

// Stage-1 indexer distillation (distill.cu); the workspace holds the teacher's
// block mass per KV group and the per-row (Z, LSE) after the 256-byte header.
size_t index_distill_ws_bytes(int B, int64_t T, int Hkv);
cudaError_t launch_index_distill(const uint16_t *q, const uint16_t *k, const float *lse,
                                 const uint16_t *q_idx, const float *w, const uint16_t *kp, int B,
                                 int64_t T, int Hq, int Hkv, int D, int Hi, int Di, float scale,
                                 float *kl, float *dq, float *dw, float *dkp, float *dk_idx,
                                 void *ws, cudaStream_t s);

// Stage-2 indexer loss over the selection (sparse_distill.cu); the workspace holds
// the sparse attention's mass per (KV group, row, selection entry) after the header.
size_t index_distill_sparse_ws_bytes(int B, int64_t T, int Hkv, int kb);
int index_distill_sparse_max_entries();
cudaError_t launch_index_distill_sparse(const uint16_t *q, const uint16_t *k, const float *lse,
                                        const int32_t *sel, const uint16_t *q_idx,
                                        const float *w, const uint16_t *kp, int B, int64_t T,
                                        int Hq, int Hkv, int D, int Hi, int Di, int kb,
                                        float scale, float *kl, float *dq_idx, float *dw,
                                        float *dkp, float *dk_idx, void *ws, cudaStream_t s);

// Backward of the sparse prefill attention (sparse_bwd.cu); zeroes dk and dv first.
cudaError_t launch_sparse_attn_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                        const int32_t *sel, const uint16_t *dout, int B,
                                        int64_t T, int Hq, int Hkv, int D, int kb, float scale,
                                        float *dq, float *dk, float *dv, cudaStream_t s);

// Measurement aid (probe.cu): reads `bytes` of `buf` `reps` times through L2.
cudaError_t launch_l2_read_probe(const void *buf, size_t bytes, int reps, uint32_t *sink,
                                 int num_sms, cudaStream_t s);
// Gated delta rule in chunks of 64 tokens (gdn_chunked.cu): chunk-parallel
// triangular solves, then one CTA per (sequence, head) over its chunks.
size_t gdn_chunked_ws_bytes(int B, int64_t T, int H, int dk, int dv);
cudaError_t launch_gdn_prefill_chunked(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                       const float *alpha, const float *beta,
                                       const float *state_in, int B, int64_t T, int H, int dk,
                                       int dv, float *o, float *state_out, void *ws,
                                       cudaStream_t s);
// Gated delta rule (gdn.cu): exact recurrence, one CTA per (sequence, head).
cudaError_t launch_gdn_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                               const float *alpha, const float *beta, const float *state_in,
                               int B, int64_t T, int H, int dk, int dv, float *o,
                               float *state_out, cudaStream_t s);
cudaError_t launch_gdn_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              const float *alpha, const float *beta, float *state, int B, int H,
                              int dk, int dv, float *o, cudaStream_t s);

cudaError_t launch_dense_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B,
                                 int64_t T, int Hq, int Hkv, int D, float scale, uint16_t *o,
                                 float *lse, cudaStream_t s);

}  // namespace qsa
