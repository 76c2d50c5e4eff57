// qsa_sparse_attn_decode_noalloc: the split-K sparse decode attention with its
// scratch in a fixed, library-owned device array instead of a caller workspace.
//
// Who needs it: callers that cannot allocate device memory at the point where
// they run a decode step -- for example an inference engine's plugin or op
// whose enqueue function must not allocate, or a serving process that fixes
// its device memory budget at start-up and forbids later allocations -- and
// that therefore cannot obtain the workspace qsa_sparse_attn_decode needs.
//
// The array below is file-scope device memory: every GPU that loads this
// library holds QSA_NOALLOC_SCRATCH_BYTES of it until the process exits.
// Host code must not use the array's name as an address (on the host it is a
// stand-in symbol, not device memory), so the device address is looked up
// once per device with cudaGetSymbolAddress and cached.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/qsa.h"
#include "qsa_launch.h"

namespace {

static __device__ __align__(256) unsigned char qsa_noalloc_scratch[QSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch[kMaxDevices];  // device address of the array, per device
int g_sms[kMaxDevices];
std::mutex g_mu;

// Set-up on the current device (first call on each device): check the
// architecture and resolve the array's device address.
qsa_status_t scratch_for_current_device(void **ptr, int *num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return QSA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch[dev]) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return QSA_ERR_CUDA;
        }
        if (major != 10 || minor != 0) return QSA_ERR_ARCH;
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, qsa_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return QSA_ERR_CUDA;
        }
        g_sms[dev] = sms;
        g_scratch[dev] = p;
    }
    *ptr = g_scratch[dev];
    *num_sms = g_sms[dev];
    return QSA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" qsa_status_t qsa_sparse_attn_decode_noalloc(
    const qsa_bf16_t *q, const qsa_bf16_t *k_cache, const qsa_bf16_t *v_cache,
    const int32_t *seqlens, int64_t L_max, const int32_t *sel, int B, int Hq, int Hkv, int D,
    int r, int budget, float scale, qsa_bf16_t *o, float *lse, void *stream) {
    if (B < 1 || L_max < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 1 || r < 1 ||
        budget < r || budget % r != 0 || !(scale == scale))
        return QSA_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !seqlens || !sel || !o) return QSA_ERR_INVALID_ARG;
    const int kb = budget / r;
    const int G = Hq / Hkv;
    if (r != 4 || (D != 64 && D != 128) || (Hkv != 1 && Hkv != 2 && Hkv != 4) ||
        (G != 1 && G != 2 && G != 4 && G != 8) || kb > 1024)
        return QSA_ERR_UNSUPPORTED_SHAPE;
    // split the selection so that about 512 slices keep the GPU busy
    int ns = (512 + B - 1) / B;
    const int max_ns = kb / 16 > 1 ? kb / 16 : 1;
    if (ns > max_ns) ns = max_ns;
    const size_t need = (size_t)B * ns * Hq * (D + 2) * sizeof(float);
    if (need > QSA_NOALLOC_SCRATCH_BYTES) return QSA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return QSA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    int sms = 0;
    qsa_status_t st = scratch_for_current_device(&scratch, &sms);
    if (st != QSA_OK) return st;
    // Every (sequence, slice) partial that the combine step reads is written by
    // this call first, so the shared array needs no clearing between calls.
    const cudaError_t e = qsa::launch_split_decode(
        q, k_cache, v_cache, seqlens, L_max, sel, kb, ns, B, Hq, Hkv, D, scale, o, lse,
        static_cast<float *>(scratch), nullptr, sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
