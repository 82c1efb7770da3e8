// pkv_probe.cu -- read-only HBM kernels that measure the ceilings the decode
// kernels are held against: a sequential stream, and whole chunks read in a
// given (random) order.
//
// The decode path only reads its large inputs (K and V rows) and writes a
// small output, so the copy bandwidth (read + write) is not its true upper
// bound: a stream of reads alone keeps the DRAM bus in one direction.  This
// kernel reads a buffer once with 16-byte loads that bypass L1, keeps eight
// loads in flight per thread, and folds what it read into one word so that
// no load can be dropped.  It is part of the measurement, not of the method.

#include <cuda_runtime.h>

#include <climits>
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

// Launched like the decode kernels (programmatic dependent launch), so that
// back-to-back launches overlap one launch's start with the previous one's
// end exactly as the decode's do.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kern, unsigned grid, void *stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kProbeThreads);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

__global__ void __launch_bounds__(kProbeThreads)
hbm_read_probe_kernel(const uint4 *__restrict__ buf, int64_t n_vec, uint32_t *__restrict__ sink)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
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

// The same reads, as whole chunks taken in the order `order` lists them: a
// warp reads one chunk at a time (its lanes' 16-byte loads across it, eight
// in flight each), warps walking the list with a grid stride.  With a random
// order of 4 KiB chunks this is the access a paged cache sees: blocks
// scattered over the pool, each read whole once.
__global__ void __launch_bounds__(kProbeThreads)
hbm_gather_probe_kernel(const uint4 *__restrict__ buf, const int32_t *__restrict__ order,
                        int64_t n_chunks, int64_t vec_per_chunk, uint32_t *__restrict__ sink)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * (kProbeThreads / 32);
    uint32_t acc = 0;
    for (int64_t c = ((int64_t)blockIdx.x * kProbeThreads + threadIdx.x) >> 5; c < n_chunks; c += nw) {
        const int64_t ch = __ldg(order + c);
        if (ch < 0 || ch >= n_chunks)
            continue;                               // not a chunk of the buffer
        const uint4 *src = buf + ch * vec_per_chunk;
        for (int64_t v0 = lane; v0 < vec_per_chunk; v0 += 32 * kProbeUnroll) {
            uint4 v[kProbeUnroll];
#pragma unroll
            for (int u = 0; u < kProbeUnroll; ++u)
                v[u] = v0 + u * 32 < vec_per_chunk ? load_stream(src + v0 + u * 32) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int u = 0; u < kProbeUnroll; ++u)
                acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
        }
    }
    acc = __reduce_xor_sync(0xffffffffu, acc);
    if (lane == 0)
        atomicXor(sink, acc);
}

}  // namespace

extern "C" pkv_status pkv_hbm_gather_probe(const void *buf, size_t chunk_bytes, const int32_t *order,
                                           int64_t n_chunks, unsigned int *sink, int grid, void *stream)
{
    if (!buf || !order || !sink || chunk_bytes == 0 || chunk_bytes % 16 != 0 || n_chunks <= 0 ||
        n_chunks > INT32_MAX || grid <= 0 || grid > (1 << 20)) {
        pkv_set_last_error("hbm_gather_probe: null pointer, chunk size not a positive multiple of 16, "
                           "chunk count outside 1 .. 2^31-1, or grid outside 1 .. 2^20");
        return PKV_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(buf) & 15u) || (reinterpret_cast<uintptr_t>(order) & 3u) ||
        (reinterpret_cast<uintptr_t>(sink) & 3u)) {
        pkv_set_last_error("hbm_gather_probe: buf must be 16-byte, order and sink 4-byte aligned");
        return PKV_ERR_MISALIGNED;
    }
    const cudaError_t e = launch_pdl(hbm_gather_probe_kernel, (unsigned)grid, stream, static_cast<const uint4 *>(buf),
                                     order, n_chunks, (int64_t)(chunk_bytes / 16), sink);
    if (e != cudaSuccess) {
        pkv_set_last_error(cudaGetErrorString(e));
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

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
    const cudaError_t e = launch_pdl(hbm_read_probe_kernel, (unsigned)grid, stream, static_cast<const uint4 *>(buf),
                                     (int64_t)(bytes / 16), sink);
    if (e != cudaSuccess) {
        pkv_set_last_error(cudaGetErrorString(e));
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}
