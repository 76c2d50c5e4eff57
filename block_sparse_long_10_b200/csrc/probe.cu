// L2 read-bandwidth probe: the denominator for kernels whose source stays in
// L2 (the sparse attention at 128K and below, whose 128 MiB of K/V fit in the
// 126 MB L2).  Every thread streams 16-byte L2 loads (cached at L2, not L1)
// over a buffer small enough to stay L2-resident, eight loads in flight per
// thread, and folds them into one word so that no load is dead.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {

__global__ void __launch_bounds__(256) l2_read_kernel(const uint4 *__restrict__ buf, int64_t n16,
                                                      int reps, uint32_t *__restrict__ sink) {
    constexpr int U = 8;
    uint32_t acc = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int r = 0; r < reps; ++r) {
        for (int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i0 < n16;
             i0 += stride * U) {
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t i = i0 + u * stride;
                if (i < n16) {
                    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                                 : "=r"(v[u].x), "=r"(v[u].y), "=r"(v[u].z), "=r"(v[u].w)
                                 : "l"(buf + i));
                } else {
                    v[u] = make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
        }
    }
    if (acc == 0x9E3779B9u) sink[0] = acc;  // practically never: keeps the loads live
}

cudaError_t launch_l2_read_probe(const void *buf, size_t bytes, int reps, uint32_t *sink,
                                 int num_sms, cudaStream_t s) {
    const int64_t n16 = (int64_t)(bytes / 16);
    if (n16 == 0 || reps <= 0) return cudaSuccess;
    l2_read_kernel<<<num_sms * 8, 256, 0, s>>>(static_cast<const uint4 *>(buf), n16, reps, sink);
    return cudaGetLastError();
}

}  // namespace qsa
