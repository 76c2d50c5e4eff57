// libqsa C ABI: argument validation, device checks, workspace layout and
// launches.  Every entry point validates on the host first and returns before
// touching the CUDA runtime when an argument is wrong, so argument errors are
// reported identically with or without a GPU.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/qsa.h"
#include "qsa_launch.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kHeader = 256;

struct DeviceInfo {
    std::atomic<int> state{0};  // 0 unknown, 1 sm_100, 2 other arch
    int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// QSA_OK and the SM count of the current device, or an error.
qsa_status_t current_device(int *num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return QSA_ERR_CUDA;
    }
    DeviceInfo &d = g_dev[dev];
    int st = d.state.load(std::memory_order_acquire);
    if (st == 0) {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        st = d.state.load(std::memory_order_relaxed);
        if (st == 0) {
            int major = 0, minor = 0, sms = 0;
            if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
                    cudaSuccess ||
                cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) !=
                    cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                    cudaSuccess) {
                cudaGetLastError();
                return QSA_ERR_CUDA;
            }
            d.num_sms = sms;
            st = (major == 10 && minor == 0) ? 1 : 2;
            d.state.store(st, std::memory_order_release);
        }
    }
    if (st != 1) return QSA_ERR_ARCH;
    *num_sms = d.num_sms;
    return QSA_OK;
}

qsa_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_attn(int Hq, int Hkv, int D) {
    if (D != 64 && D != 128) return false;
    if (Hkv != 1 && Hkv != 2 && Hkv != 4) return false;
    const int G = Hq / Hkv;
    return G == 1 || G == 2 || G == 4 || G == 8;
}

bool supported_indexer(int Hi, int Di) {
    return (Hi == 1 || Hi == 2 || Hi == 4) && (Di == 32 || Di == 64);
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// About one wave of slices (2 CTAs per SM on 148 SMs ~ 296 slots): at 64
// sequences, 4 slices of 128 blocks each.
int sparse_decode_nsplit(int B, int kb) {
    int ns = (int)cdiv(256, B > 0 ? B : 1);
    int max_ns = kb / 16 > 1 ? kb / 16 : 1;
    if (ns > max_ns) ns = max_ns;
    return ns < 1 ? 1 : ns;
}

constexpr int kDenseDecodeChunk = 512;  // blocks (2048 tokens) per split

int dense_decode_nsplit(int64_t L_max) {
    const int64_t n = cdiv(cdiv(L_max, 4), kDenseDecodeChunk);
    return (int)(n < 1 ? 1 : n);
}

size_t partial_bytes(int B, int ns, int Hq, int D) {
    return (size_t)B * ns * Hq * (D + 2) * sizeof(float);
}

}  // namespace

extern "C" {

const char *qsa_version(void) { return "0.1.0"; }

const char *qsa_status_string(qsa_status_t s) {
    switch (s) {
        case QSA_OK: return "ok";
        case QSA_ERR_INVALID_ARG: return "invalid argument";
        case QSA_ERR_UNSUPPORTED_SHAPE: return "shape not supported by the GPU kernels";
        case QSA_ERR_WORKSPACE: return "workspace missing or too small";
        case QSA_ERR_ARCH: return "current device is not sm_100 (B200)";
        case QSA_ERR_CUDA: return "CUDA runtime error";
        case QSA_ERR_TIMEOUT: return "bounded device-side wait timed out";
        case QSA_ERR_DEVICE: return "kernel met an out-of-range input value";
    }
    return "unknown status";
}

// ------------------------------------------------------------------ pool --
qsa_status_t qsa_pool(const qsa_bf16_t *k_idx, int B, int64_t T, int Di, int r,
                      int64_t blk_begin, int64_t blk_end, qsa_bf16_t *k_pooled, void *stream) {
    if (B < 0 || T < 0 || Di <= 0 || r <= 0) return QSA_ERR_INVALID_ARG;
    if (blk_begin < 0 || blk_end < blk_begin || blk_end > T / r) return QSA_ERR_INVALID_ARG;
    if (r != 4 || Di % 8 != 0) return QSA_ERR_UNSUPPORTED_SHAPE;
    if (B == 0 || blk_end == blk_begin) return QSA_OK;
    if (!k_idx || !k_pooled || !aligned16(k_idx) || !aligned16(k_pooled))
        return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_pool(k_idx, B, T, Di, blk_begin, blk_end, k_pooled,
                                      static_cast<cudaStream_t>(stream), sms));
}

// --------------------------------------------------------- index top-k --
size_t qsa_index_topk_workspace_size(int B, int64_t Tq, int64_t n_blocks, int Hi, int Di, int r,
                                     int budget) {
    if (B < 1 || Tq < 0 || n_blocks < 0 || Hi < 1 || Di < 1 || r < 1 || budget < r ||
        budget % r != 0)
        return SIZE_MAX;
    (void)Di;
    return qsa::index_tc_ws_bytes(B, Tq, Hi);
}

qsa_status_t qsa_index_topk(const qsa_bf16_t *q_idx, const float *w, const qsa_bf16_t *k_pooled,
                            const int64_t *q_pos0, int B, int64_t Tq, int64_t n_blocks, int Hi,
                            int Di, int r, int budget, int32_t *sel, float *sel_score, void *ws,
                            size_t ws_bytes, void *stream) {
    if (B < 1 || Tq < 0 || n_blocks < 0 || Hi < 1 || Di < 1 || r < 1 || budget < r ||
        budget % r != 0)
        return QSA_ERR_INVALID_ARG;
    if (Tq == 0) return QSA_OK;
    if (!q_idx || !w || (!k_pooled && n_blocks > 0) || !sel) return QSA_ERR_INVALID_ARG;
    if (!q_pos0 && (Tq - 1) / r > n_blocks) return QSA_ERR_INVALID_ARG;
    const int kb = budget / r;
    if (r != 4 || !supported_indexer(Hi, Di) || kb - 1 > qsa::index_tc_max_keep())
        return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!ws || ws_bytes < qsa::index_tc_ws_bytes(B, Tq, Hi) || !aligned16(ws))
        return QSA_ERR_WORKSPACE;
    if (!aligned16(q_idx) || !aligned16(k_pooled)) return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_index_topk_tc(q_idx, w, k_pooled, q_pos0, B, Tq, n_blocks, Hi,
                                               Di, kb, sel, sel_score, ws, sms,
                                               static_cast<cudaStream_t>(stream)));
}

size_t qsa_index_topk_decode_workspace_size(int B, int64_t n_blocks, int r, int budget) {
    if (B < 1 || n_blocks < 0 || r < 1 || budget < r || budget % r != 0) return SIZE_MAX;
    return qsa::index_decode_ws_bytes(B, n_blocks, budget / r, 0);
}

qsa_status_t qsa_index_topk_decode(const qsa_bf16_t *q_idx, const float *w,
                                   const qsa_bf16_t *k_pooled, const int32_t *seqlens, int B,
                                   int64_t n_blocks, int Hi, int Di, int r, int budget,
                                   int32_t *sel, float *sel_score, void *ws, size_t ws_bytes,
                                   void *stream) {
    if (B < 1 || n_blocks < 0 || Hi < 1 || Di < 1 || r < 1 || budget < r || budget % r != 0)
        return QSA_ERR_INVALID_ARG;
    if (!q_idx || !w || (!k_pooled && n_blocks > 0) || !seqlens || !sel)
        return QSA_ERR_INVALID_ARG;
    const int kb = budget / r;
    if (r != 4 || !supported_indexer(Hi, Di) || kb - 1 > qsa::index_tc_max_keep() ||
        qsa::index_decode_merge_cap(n_blocks, kb) < 0)
        return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!ws || ws_bytes < qsa::index_decode_ws_bytes(B, n_blocks, kb, 0) || !aligned16(ws))
        return QSA_ERR_WORKSPACE;
    if (!aligned16(q_idx) || !aligned16(k_pooled)) return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_index_topk_decode(q_idx, w, k_pooled, seqlens, B, n_blocks, Hi,
                                                   Di, kb, sel, sel_score, ws, sms,
                                                   static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------ sparse attention --
qsa_status_t qsa_sparse_attn_prefill(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                     const qsa_bf16_t *v, const int32_t *sel,
                                     const int64_t *q_pos0, int B, int64_t Tq, int64_t Tk,
                                     int Hq, int Hkv, int D, int r, int budget, float scale,
                                     qsa_bf16_t *o, float *lse, void *stream) {
    if (B < 1 || Tq < 0 || Tk < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 1 || r < 1 ||
        budget < r || budget % r != 0 || !(scale == scale))
        return QSA_ERR_INVALID_ARG;
    if (Tq == 0) return QSA_OK;
    if (Tk < 1 || !q || !k || !v || !sel || !o) return QSA_ERR_INVALID_ARG;
    if (!q_pos0 && Tq > Tk) return QSA_ERR_INVALID_ARG;
    const int kb = budget / r;
    if (r != 4 || !supported_attn(Hq, Hkv, D) || kb > 1024) return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_sparse_attn_prefill(q, k, v, sel, q_pos0, B, Tq, Tk, Hq, Hkv, D,
                                                     kb, scale, o, lse, sms,
                                                     static_cast<cudaStream_t>(stream)));
}

size_t qsa_sparse_attn_decode_workspace_size(int B, int Hq, int D, int r, int budget) {
    if (B < 1 || Hq < 1 || D < 1 || r < 1 || budget < r || budget % r != 0) return SIZE_MAX;
    return kHeader + partial_bytes(B, sparse_decode_nsplit(B, budget / r), Hq, D);
}

qsa_status_t qsa_sparse_attn_decode(const qsa_bf16_t *q, const qsa_bf16_t *k_cache,
                                    const qsa_bf16_t *v_cache, const int32_t *seqlens,
                                    int64_t L_max, const int32_t *sel, int B, int Hq, int Hkv,
                                    int D, int r, int budget, float scale, qsa_bf16_t *o,
                                    float *lse, void *ws, size_t ws_bytes, void *stream) {
    if (B < 1 || L_max < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 1 || r < 1 ||
        budget < r || budget % r != 0 || !(scale == scale))
        return QSA_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !seqlens || !sel || !o) return QSA_ERR_INVALID_ARG;
    const int kb = budget / r;
    if (r != 4 || !supported_attn(Hq, Hkv, D) || kb > 1024) return QSA_ERR_UNSUPPORTED_SHAPE;
    const int ns = sparse_decode_nsplit(B, kb);
    if (!ws || ws_bytes < kHeader + partial_bytes(B, ns, Hq, D) || !aligned16(ws))
        return QSA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    float *part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kHeader);
    return from_cuda(qsa::launch_split_decode(q, k_cache, v_cache, seqlens, L_max, sel, kb, ns, B,
                                              Hq, Hkv, D, scale, o, lse, part, ws, sms,
                                              static_cast<cudaStream_t>(stream)));
}

// -------------------------------------------------------- dense baseline --
qsa_status_t qsa_dense_gqa_prefill(const qsa_bf16_t *q, const qsa_bf16_t *k, const qsa_bf16_t *v,
                                   int B, int64_t T, int Hq, int Hkv, int D, float scale,
                                   qsa_bf16_t *o, float *lse, void *stream) {
    if (B < 1 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 1 || !(scale == scale))
        return QSA_ERR_INVALID_ARG;
    if (T == 0) return QSA_OK;
    if (!q || !k || !v || !o) return QSA_ERR_INVALID_ARG;
    if (!supported_attn(Hq, Hkv, D)) return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_dense_prefill(q, k, v, B, T, Hq, Hkv, D, scale, o, lse,
                                               static_cast<cudaStream_t>(stream)));
}

size_t qsa_dense_gqa_decode_workspace_size(int B, int64_t L_max, int Hq, int D) {
    if (B < 1 || L_max < 1 || Hq < 1 || D < 1) return SIZE_MAX;
    return kHeader + partial_bytes(B, dense_decode_nsplit(L_max), Hq, D);
}

qsa_status_t qsa_dense_gqa_decode(const qsa_bf16_t *q, const qsa_bf16_t *k_cache,
                                  const qsa_bf16_t *v_cache, const int32_t *seqlens,
                                  int64_t L_max, int B, int Hq, int Hkv, int D, float scale,
                                  qsa_bf16_t *o, float *lse, void *ws, size_t ws_bytes,
                                  void *stream) {
    if (B < 1 || L_max < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 1 || !(scale == scale))
        return QSA_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !seqlens || !o) return QSA_ERR_INVALID_ARG;
    if (!supported_attn(Hq, Hkv, D)) return QSA_ERR_UNSUPPORTED_SHAPE;
    const int ns = dense_decode_nsplit(L_max);
    if (!ws || ws_bytes < kHeader + partial_bytes(B, ns, Hq, D) || !aligned16(ws))
        return QSA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    float *part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kHeader);
    const int n_entries = (int)cdiv(L_max, 4);
    return from_cuda(qsa::launch_split_decode(q, k_cache, v_cache, seqlens, L_max, nullptr,
                                              n_entries, ns, B, Hq, Hkv, D, scale, o, lse, part,
                                              ws, sms, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------- sparse attention backward --
qsa_status_t qsa_sparse_attn_backward(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                      const qsa_bf16_t *v, const int32_t *sel,
                                      const qsa_bf16_t *d_o, int B, int64_t T, int Hq, int Hkv,
                                      int D, int r, int budget, float scale, float *dq,
                                      float *dk, float *dv, void *stream) {
    if (B < 1 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 1 || r < 1 ||
        budget < r || budget % r != 0 || !(scale == scale))
        return QSA_ERR_INVALID_ARG;
    if (T == 0) return QSA_OK;
    if (!q || !k || !v || !sel || !d_o || !dq || !dk || !dv) return QSA_ERR_INVALID_ARG;
    const int kb = budget / r;
    if (r != 4 || !supported_attn(Hq, Hkv, D) || kb > 1024) return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_o) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv))
        return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_sparse_attn_backward(q, k, v, sel, d_o, B, T, Hq, Hkv, D, kb,
                                                      scale, dq, dk, dv,
                                                      static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------- measurement aid --
qsa_status_t qsa_probe_l2_read(const void *buf, size_t bytes, int reps, void *sink,
                               void *stream) {
    if (!buf || !sink || reps < 1 || bytes < 16) return QSA_ERR_INVALID_ARG;
    if (!aligned16(buf) || (reinterpret_cast<uintptr_t>(sink) & 3u) != 0) return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_l2_read_probe(buf, bytes, reps, static_cast<uint32_t *>(sink),
                                               sms, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------- Gated DeltaNet --
static bool supported_gdn(int dk, int dv) {
    return (dk == 64 || dk == 128) && (dv == 64 || dv == 128);
}

qsa_status_t qsa_gdn_prefill(const qsa_bf16_t *q, const qsa_bf16_t *k, const qsa_bf16_t *v,
                             const float *alpha, const float *beta, const float *state_in, int B,
                             int64_t T, int H, int dk, int dv, float *o, float *state_out,
                             void *stream) {
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return QSA_ERR_INVALID_ARG;
    if (!state_out || (T > 0 && (!q || !k || !v || !alpha || !beta || !o)))
        return QSA_ERR_INVALID_ARG;
    if (!supported_gdn(dk, dv)) return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(state_out) || (state_in && !aligned16(state_in))) return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_gdn_prefill(q, k, v, alpha, beta, state_in, B, T, H, dk, dv, o,
                                             state_out, static_cast<cudaStream_t>(stream)));
}

size_t qsa_gdn_prefill_chunked_workspace_size(int B, int64_t T, int H, int dk, int dv) {
    if (B < 1 || T < 0 || H < 1 || !supported_gdn(dk, dv)) return SIZE_MAX;
    return qsa::gdn_chunked_ws_bytes(B, T, H, dk, dv);
}

qsa_status_t qsa_gdn_prefill_chunked(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                     const qsa_bf16_t *v, const float *alpha, const float *beta,
                                     const float *state_in, int B, int64_t T, int H, int dk,
                                     int dv, float *o, float *state_out, void *ws,
                                     size_t ws_bytes, void *stream) {
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return QSA_ERR_INVALID_ARG;
    if (!state_out || (T > 0 && (!q || !k || !v || !alpha || !beta || !o)))
        return QSA_ERR_INVALID_ARG;
    if (!supported_gdn(dk, dv)) return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(state_out) || (state_in && !aligned16(state_in)) ||
        (T > 0 && (!aligned16(q) || !aligned16(k))))
        return QSA_ERR_INVALID_ARG;
    if (!ws || ws_bytes < qsa::gdn_chunked_ws_bytes(B, T, H, dk, dv) ||
        (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return QSA_ERR_WORKSPACE;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_gdn_prefill_chunked(q, k, v, alpha, beta, state_in, B, T, H, dk,
                                                     dv, o, state_out, ws,
                                                     static_cast<cudaStream_t>(stream)));
}

qsa_status_t qsa_gdn_decode(const qsa_bf16_t *q, const qsa_bf16_t *k, const qsa_bf16_t *v,
                            const float *alpha, const float *beta, float *state, int B, int H,
                            int dk, int dv, float *o, void *stream) {
    if (B < 1 || H < 1 || dk < 1 || dv < 1) return QSA_ERR_INVALID_ARG;
    if (!q || !k || !v || !alpha || !beta || !state || !o) return QSA_ERR_INVALID_ARG;
    if (!supported_gdn(dk, dv)) return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(state)) return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_gdn_decode(q, k, v, alpha, beta, state, B, H, dk, dv, o,
                                            static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------- indexer distillation --
size_t qsa_index_distill_workspace_size(int B, int64_t T, int Hkv, int r) {
    if (B < 1 || T < 0 || Hkv < 1 || r != 4) return SIZE_MAX;
    return qsa::index_distill_ws_bytes(B, T, Hkv);
}

qsa_status_t qsa_index_distill(const qsa_bf16_t *q, const qsa_bf16_t *k, const float *lse,
                               const qsa_bf16_t *q_idx, const float *w,
                               const qsa_bf16_t *k_pooled, int B, int64_t T, int Hq, int Hkv,
                               int D, int Hi, int Di, int r, float scale, float *kl,
                               float *dq_idx, float *dw, float *dk_pooled, float *dk_idx,
                               void *ws, size_t ws_bytes, void *stream) {
    if (B < 1 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 1 || Hi < 1 || Di < 1 ||
        r < 1 || !(scale == scale))
        return QSA_ERR_INVALID_ARG;
    if (T == 0) return QSA_OK;
    const int64_t N = T / r;
    if (!q || !k || !lse || !q_idx || !w || !kl || !dq_idx || !dw ||
        (N > 0 && (!k_pooled || !dk_pooled)))
        return QSA_ERR_INVALID_ARG;
    if (r != 4 || !supported_attn(Hq, Hkv, D) || !supported_indexer(Hi, Di))
        return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!ws || ws_bytes < qsa::index_distill_ws_bytes(B, T, Hkv) || !aligned16(ws))
        return QSA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_idx) || !aligned16(k_pooled))
        return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_index_distill(q, k, lse, q_idx, w, k_pooled, B, T, Hq, Hkv, D,
                                               Hi, Di, scale, kl, dq_idx, dw, dk_pooled, dk_idx,
                                               ws, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------- stage-2 indexer loss --
size_t qsa_index_distill_sparse_workspace_size(int B, int64_t T, int Hkv, int r, int budget) {
    if (B < 1 || T < 0 || Hkv < 1 || r != 4 || budget < r || budget % r != 0) return SIZE_MAX;
    return qsa::index_distill_sparse_ws_bytes(B, T, Hkv, budget / r);
}

qsa_status_t qsa_index_distill_sparse(const qsa_bf16_t *q, const qsa_bf16_t *k,
                                      const float *lse, const int32_t *sel,
                                      const qsa_bf16_t *q_idx, const float *w,
                                      const qsa_bf16_t *k_pooled, int B, int64_t T, int Hq,
                                      int Hkv, int D, int Hi, int Di, int r, int budget,
                                      float scale, float *kl, float *dq_idx, float *dw,
                                      float *dk_pooled, float *dk_idx, void *ws, size_t ws_bytes,
                                      void *stream) {
    if (B < 1 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 1 || Hi < 1 || Di < 1 ||
        r < 1 || budget < r || budget % r != 0 || !(scale == scale))
        return QSA_ERR_INVALID_ARG;
    if (T == 0) return QSA_OK;
    const int64_t N = T / r;
    if (!q || !k || !lse || !sel || !q_idx || !w || !kl || !dq_idx || !dw ||
        (N > 0 && (!k_pooled || !dk_pooled)))
        return QSA_ERR_INVALID_ARG;
    const int kb = budget / r;
    if (r != 4 || !supported_attn(Hq, Hkv, D) || !supported_indexer(Hi, Di) ||
        kb > qsa::index_distill_sparse_max_entries())
        return QSA_ERR_UNSUPPORTED_SHAPE;
    if (!ws || ws_bytes < qsa::index_distill_sparse_ws_bytes(B, T, Hkv, kb) || !aligned16(ws))
        return QSA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_idx) || !aligned16(k_pooled))
        return QSA_ERR_INVALID_ARG;
    int sms = 0;
    qsa_status_t st = current_device(&sms);
    if (st != QSA_OK) return st;
    return from_cuda(qsa::launch_index_distill_sparse(
        q, k, lse, sel, q_idx, w, k_pooled, B, T, Hq, Hkv, D, Hi, Di, kb, scale, kl, dq_idx, dw,
        dk_pooled, dk_idx, ws, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- status --
qsa_status_t qsa_check_device_status(void *ws, void *stream) {
    if (!ws) return QSA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return QSA_ERR_CUDA;
    }
    int word = 0;
    if (cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return QSA_ERR_CUDA;
    }
    if (word != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return QSA_ERR_CUDA;
    }
    return static_cast<qsa_status_t>(word);
}

}  // extern "C"
