// pkv_probe.cu -- a read-only HBM streaming kernel that measures the ceiling
// the decode kernels are held against.
//
// The decode path only reads its large inputs (K and V rows) and writes a
// small output, so the copy bandwidth (read + write) is not its true upper
// bound: a stream of reads alone keeps the DRAM bus in one direction.  This
// kernel reads a buffer once with 16-byte loads that bypass L1, keeps eight
// loads in flight per thread, and folds what it read into one word so that
// no load can be dropped.  It is part of the measurement, not of the method.

#include <cuda_runtime.h>

#include <cstdint>

#include "pagedkv.h"

void pkv_set_last_error(const char *msg);   // pagedkv.cu

namespace {

constexpr int kProbeThreads = 512;
constexpr int kProbeUnroll = 8;

__device__ __forceinline__ uint4 load_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__global__ void __launch_bounds__(kProbeThreads)
hbm_read_probe_kernel(const uint4 *__restrict__ buf, int64_t n_vec, uint32_t *__restrict__ sink)
{
    const int64_t stride = (int64_t)gridDim.x * kProbeThreads;
    int64_t i = (int64_t)blockIdx.x * kProbeThreads + threadIdx.x;
    uint32_t acc = 0;
    for (; i + (kProbeUnroll - 1) * stride < n_vec; i += kProbeUnroll * stride) {
        uint4 v[kProbeUnroll];
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u)
            v[u] = load_stream(buf + i + u * stride);
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u)
            acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n_vec; i += stride) {
        const uint4 v = load_stream(buf + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
    // one word per CTA: the fold of everything its threads read
    acc = __reduce_xor_sync(0xffffffffu, acc);
    if ((threadIdx.x & 31) == 0)
        atomicXor(sink, acc);
}

}  // namespace

extern "C" pkv_status pkv_hbm_read_probe(const void *buf, size_t bytes, unsigned int *sink,
                                         int grid, void *stream)
{
    if (!buf || !sink || bytes == 0 || bytes % 16 != 0 || grid <= 0 || grid > (1 << 20)) {
        pkv_set_last_error("hbm_read_probe: null pointer, size not a positive multiple of 16, "
                           "or grid outside 1 .. 2^20");
        return PKV_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(buf) & 15u) || (reinterpret_cast<uintptr_t>(sink) & 3u)) {
        pkv_set_last_error("hbm_read_probe: buf must be 16-byte and sink 4-byte aligned");
        return PKV_ERR_MISALIGNED;
    }
    hbm_read_probe_kernel<<<(unsigned)grid, kProbeThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(buf), (int64_t)(bytes / 16), sink);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        pkv_set_last_error(cudaGetErrorString(e));
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}
