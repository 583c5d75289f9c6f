// Read-only HBM calibration: a streaming read of a large buffer, to set beside the
// decode kernels the best rate at which this GPU's memory delivers bytes when
// nothing is written back (a copy measurement counts a read and a write per byte
// and does not show the read ceiling that the decode kernels stream against).
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvdecode.h"

namespace {

// 16-byte loads that do not allocate in L1 (the buffer is many times L2); every
// block folds what it read into one word so that the loads are not dead.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__global__ void __launch_bounds__(512) read_stream_kernel(const uint4 *__restrict__ buf, size_t n16,
                                                         unsigned long long *sink) {
    constexpr int U = 8;  // loads in flight per thread
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t acc = 0;
    for (; i + (U - 1) * stride < n16; i += U * stride) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) v[u] = ld_stream(buf + i + u * stride);
#pragma unroll
        for (int u = 0; u < U; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n16; i += stride) {
        const uint4 v = ld_stream(buf + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0 && acc == 0x9e3779b9u) atomicAdd(sink, 1ull);  // practically never taken
}

}  // namespace

extern "C" int kvd_read_stream(const void *buf, size_t bytes, unsigned long long *sink, int blocks_per_sm,
                               kvd_stream_t stream) {
    if (!buf || !sink || bytes == 0 || bytes % 16 != 0 || ((uintptr_t)buf & 15u) != 0 || blocks_per_sm <= 0)
        return KVD_ERR_INVALID_ARG;
    const int sms = kvd_num_sms();
    if (sms <= 0) return KVD_ERR_CUDA;
    read_stream_kernel<<<sms * blocks_per_sm, 512, 0, (cudaStream_t)stream>>>((const uint4 *)buf, bytes / 16, sink);
    return cudaGetLastError() == cudaSuccess ? KVD_OK : KVD_ERR_CUDA;
}
