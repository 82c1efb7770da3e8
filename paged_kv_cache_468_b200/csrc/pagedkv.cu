// pagedkv.cu -- C-ABI entry points of libpagedkv.so (see include/pagedkv.h).
//
// Host-side work only: argument validation, the partition plan, TMA tensor
// maps, launches.  Every computation of the hot path runs in the kernels of
// pkv_kernels.cuh.  The library allocates no device memory.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "pagedkv.h"
#include "pkv_kernels.cuh"
#include "pkv_prefill.cuh"

namespace {

thread_local std::string g_last_error;

pkv_status fail(pkv_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
pkv_status fail(pkv_status s, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

pkv_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(PKV_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kPlanSmCount = 148;        // B200 SM count used by the automatic plan
// A prefill CTA takes up to this many row tiles (of 128/G query tokens) of one
// (sequence, kv head) in turn: fewer CTAs amortise their set-up over more
// tiles, but each CTA's work grows, and the hardware's balancing of CTAs over
// the SMs needs the largest CTA to stay small next to the average work per SM.
constexpr int kPrefillMaxTilesPerCta = 4;

int prefill_tiles_per_cta(int batch, int Hkv, int row_tiles, int sms)
{
    // at most 1/8 of the average work per CTA slot (2 per SM) in one CTA,
    // counting a row tile's work at half the largest one's
    const int64_t per_slot_share = (int64_t)batch * Hkv * row_tiles / (2 * 2 * 8 * (int64_t)sms);
    int t = 1;
    while (t * 2 <= kPrefillMaxTilesPerCta && t * 2 <= per_slot_share)
        t *= 2;
    return t;
}
constexpr int kAutoPartitionTokens = 512;

// ---- TMA tensor maps ------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// The cache [num_blocks, bs, Hkv, D] seen as a 3-D tensor
// (innermost first) {D, Hkv, num_blocks*bs}; a box is 64 columns x 1 head x
// bs token rows, written to shared memory with the 128-byte swizzle.
pkv_status make_cache_map(CUtensorMap *map, const void *base, int64_t num_blocks, int bs,
                          int Hkv, int D, pkv_dtype dt)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)(num_blocks * bs)};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)bs};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = enc(map, dt == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                     3, const_cast<void *>(base), dims, strides, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return PKV_OK;
}

// The cache as a 4-D tensor {D, Hkv, bs, num_blocks}: a box is 64 columns x
// 1 head x bs rows x 1 block.  Unlike the 3-D view, rows before a block's
// first row are outside the tensor, so a load that starts at a negative row
// reads zeros there (the one-pass cascade loads a partly filled block that
// way, its valid rows at the end of the box).
pkv_status make_cache_map_4d(CUtensorMap *map, const void *base, int64_t num_blocks, int bs,
                             int Hkv, int D, pkv_dtype dt)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)bs, (cuuint64_t)num_blocks};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2, (cuuint64_t)bs * Hkv * D * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)bs, 1};
    cuuint32_t estride[4] = {1, 1, 1, 1};
    CUresult r = enc(map, dt == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                     4, const_cast<void *>(base), dims, strides, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled (4-D cache) failed (CUresult %d)", (int)r);
    return PKV_OK;
}

// K and V caches, each as the 3-D view (whole blocks) and the 4-D view
// (shifted partly filled blocks) the tensor-core kernels load through.
struct CacheMaps {
    CUtensorMap k, v, k4, v4;
};

pkv_status make_cache_maps(CacheMaps *m, const void *key_cache, const void *value_cache,
                           int64_t num_blocks, int bs, int Hkv, int D, pkv_dtype dt)
{
    pkv_status s;
    if ((s = make_cache_map(&m->k, key_cache, num_blocks, bs, Hkv, D, dt)) != PKV_OK ||
        (s = make_cache_map(&m->v, value_cache, num_blocks, bs, Hkv, D, dt)) != PKV_OK ||
        (s = make_cache_map_4d(&m->k4, key_cache, num_blocks, bs, Hkv, D, dt)) != PKV_OK ||
        (s = make_cache_map_4d(&m->v4, value_cache, num_blocks, bs, Hkv, D, dt)) != PKV_OK)
        return s;
    return PKV_OK;
}

// The query [T, Hq, D] seen as {D, Hq, T}; a box is 64 columns x the G heads
// of one kv head x `tokens` query tokens: rows (token, head) of 128 bytes,
// 128-byte swizzle, the prefill CTA's Q tile.  Rows past T read as zero.
pkv_status make_query_map(CUtensorMap *map, const void *base, int64_t T, int Hq, int D, int G,
                          int tokens, pkv_dtype dt)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)tokens};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = enc(map, dt == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                     3, const_cast<void *>(base), dims, strides, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled (query) failed (CUresult %d)", (int)r);
    return PKV_OK;
}

// ---- launch configurations ------------------------------------------------

// Warps per CTA and pipeline depth (stages per warp), chosen by sweeping on
// B200: several small CTAs per SM hide each CTA's start-up (table lookup ->
// TMA -> first data) behind the others' streaming.  PKV_TUNE_NW / PKV_TUNE_S
// override every shape at build time (used for tuning sweeps).
template <int D, int BS>
struct Tuning;
#if defined(PKV_TUNE_NW) && defined(PKV_TUNE_S)
template <int D, int BS>
struct Tuning { static constexpr int NW = PKV_TUNE_NW, S = PKV_TUNE_S; };
#else
template <> struct Tuning<64, 16>  { static constexpr int NW = 4, S = 2; };   // 33 KB, 6 CTAs/SM
template <> struct Tuning<64, 32>  { static constexpr int NW = 2, S = 3; };   // 49 KB
template <> struct Tuning<128, 16> { static constexpr int NW = 2, S = 2; };   // 33 KB, 6 CTAs/SM
template <> struct Tuning<128, 32> { static constexpr int NW = 2, S = 2; };   // 65 KB, 3 CTAs/SM
#endif

int current_device()
{
    int dev = 0;
    cudaGetDevice(&dev);
    return dev;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel on the stream finishes; it waits (griddepcontrol.wait)
// before it reads any memory.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Merge launch: 512 threads per CTA; with at most 8 partitions per row each
// 128/64-thread group merges its own row, otherwise the groups split a row.
template <bool BF16, int D>
cudaError_t launch_merge_d(const pkv::DecodeArgs &a, const int32_t *context_lens, int rows,
                           int Hq, int np, int pt, int span, cudaStream_t st)
{
    constexpr int NT = 512, NG = NT / D;
    if (np <= 8)
        return launch_pdl(pkv::lse_merge_kernel<BF16, D, NT>, dim3((unsigned)((rows + NG - 1) / NG)),
                          dim3(NT), 0, st, a.ws_m, a.ws_l, a.ws_o, context_lens, Hq, rows, np, pt,
                          span, a.out);
    return launch_pdl(pkv::lse_merge_wide_kernel<BF16, D, NT>, dim3((unsigned)rows), dim3(NT), 0, st,
                      a.ws_m, a.ws_l, a.ws_o, context_lens, Hq, rows, np, pt, span, a.out);
}

template <bool BF16>
cudaError_t launch_merge(int D, const pkv::DecodeArgs &a, const int32_t *context_lens, int batch,
                         int Hq, int np, int pt, int span, cudaStream_t st)
{
    const int rows = batch * Hq;
    return D == 64 ? launch_merge_d<BF16, 64>(a, context_lens, rows, Hq, np, pt, span, st)
                   : launch_merge_d<BF16, 128>(a, context_lens, rows, Hq, np, pt, span, st);
}

template <int D, int BS, bool BF16>
pkv_status launch_decode(const CUtensorMap &mk, const CUtensorMap &mv, const pkv::DecodeArgs &a,
                         int batch, int Hkv, cudaStream_t st)
{
    constexpr int NW = Tuning<D, BS>::NW;
    constexpr int S = Tuning<D, BS>::S;
    using Shape = pkv::DecodeShape<D, BS, NW, S>;
    auto kern = pkv::paged_decode_kernel<D, BS, BF16, NW, S>;
    static bool configured[64] = {};
    static std::mutex mu;
    const int dev = current_device();
    {
        std::lock_guard<std::mutex> lk(mu);
        if (dev < 0 || dev >= 64 || !configured[dev]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 Shape::kSmemBytes);
            if (e != cudaSuccess)
                return cuda_fail(e, "cudaFuncSetAttribute(decode)");
            if (dev >= 0 && dev < 64)
                configured[dev] = true;
        }
    }
    dim3 grid((unsigned)a.num_parts, (unsigned)Hkv, (unsigned)batch);
    cudaError_t e = launch_pdl(kern, grid, dim3(NW * 32), Shape::kSmemBytes, st, mk, mv, a);
    if (e != cudaSuccess)
        return cuda_fail(e, "paged_decode_kernel launch");
    return PKV_OK;
}

template <bool BF16>
pkv_status dispatch_decode(int D, int bs, const CUtensorMap &mk, const CUtensorMap &mv,
                           const pkv::DecodeArgs &a, int batch, int Hkv, cudaStream_t st)
{
    if (D == 64 && bs == 16) return launch_decode<64, 16, BF16>(mk, mv, a, batch, Hkv, st);
    if (D == 64 && bs == 32) return launch_decode<64, 32, BF16>(mk, mv, a, batch, Hkv, st);
    if (D == 128 && bs == 16) return launch_decode<128, 16, BF16>(mk, mv, a, batch, Hkv, st);
    if (D == 128 && bs == 32) return launch_decode<128, 32, BF16>(mk, mv, a, batch, Hkv, st);
    return fail(PKV_ERR_UNSUPPORTED, "head_dim %d / block_size %d not compiled", D, bs);
}

pkv_status check_shapes(int batch, int Hq, int Hkv, int D, int max_blocks, int bs)
{
    if (batch < 0 || Hq <= 0 || Hkv <= 0 || max_blocks <= 0)
        return fail(PKV_ERR_INVALID_ARG, "batch=%d num_heads=%d num_kv_heads=%d max_blocks=%d",
                    batch, Hq, Hkv, max_blocks);
    if (Hq % Hkv != 0 || Hq / Hkv > 8)
        return fail(PKV_ERR_UNSUPPORTED, "group size num_heads/num_kv_heads must be an integer 1..8 "
                    "(num_heads=%d, num_kv_heads=%d)", Hq, Hkv);
    if (D != 64 && D != 128)
        return fail(PKV_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", D);
    if (bs != 16 && bs != 32)
        return fail(PKV_ERR_UNSUPPORTED, "block_size %d (supported: 16, 32)", bs);
    if ((int64_t)max_blocks * bs >= (int64_t)1 << 30)
        return fail(PKV_ERR_INVALID_ARG, "max_blocks * block_size too large");
    if (batch > 65535 || Hkv > 65535)
        return fail(PKV_ERR_UNSUPPORTED, "batch and num_kv_heads must be <= 65535");
    return PKV_OK;
}

void plan(int batch, int Hkv, int max_blocks, int bs, int requested, int *pt, int *np)
{
    const int span = max_blocks * bs;
    int t = span;
    if (requested > 0) {
        t = (requested + bs - 1) / bs * bs;
    } else if (requested == 0) {
        const bool long_ctx = span >= 2048;
        const bool few_items = (int64_t)batch * Hkv < kPlanSmCount;
        if (long_ctx || few_items)
            t = kAutoPartitionTokens;
    }
    int parts = (span + t - 1) / t;
    if (parts <= 1) {
        t = span;
        parts = 1;
    }
    *pt = t;
    *np = parts;
}

}  // namespace

// Shared with the allocator's translation unit (not part of the public ABI).
__attribute__((visibility("hidden"))) void pkv_set_last_error(const char *msg)
{
    g_last_error = msg ? msg : "";
}

extern "C" {

const char *pkv_status_str(pkv_status s)
{
    switch (s) {
    case PKV_OK: return "PKV_OK";
    case PKV_ERR_INVALID_ARG: return "PKV_ERR_INVALID_ARG";
    case PKV_ERR_UNSUPPORTED: return "PKV_ERR_UNSUPPORTED";
    case PKV_ERR_OUT_OF_RANGE: return "PKV_ERR_OUT_OF_RANGE";
    case PKV_ERR_OOM: return "PKV_ERR_OOM";
    case PKV_ERR_CUDA: return "PKV_ERR_CUDA";
    case PKV_ERR_WORKSPACE: return "PKV_ERR_WORKSPACE";
    case PKV_ERR_MISALIGNED: return "PKV_ERR_MISALIGNED";
    }
    return "PKV_ERR_UNKNOWN";
}

const char *pkv_last_error(void) { return g_last_error.c_str(); }

const char *pkv_version(void) { return "pagedkv 0.1.0 sm_100a"; }

pkv_status pkv_device_flags(int device, unsigned int *flags, int clear)
{
    if (!flags)
        return fail(PKV_ERR_INVALID_ARG, "flags is NULL");
    int prev = 0;
    cudaError_t e = cudaGetDevice(&prev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    if (device != prev && (e = cudaSetDevice(device)) != cudaSuccess)
        return cuda_fail(e, "cudaSetDevice");
    pkv_status st = PKV_OK;
    e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpyFromSymbol(flags, pkv::g_device_flags, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(pkv::g_device_flags, &zero, sizeof zero);
    }
    if (e != cudaSuccess)
        st = cuda_fail(e, "reading the device flag word");
    if (device != prev)
        cudaSetDevice(prev);
    return st;
}

pkv_status pkv_copy_blocks(const void *src_key_cache, const void *src_value_cache,
                           void *dst_key_cache, void *dst_value_cache, const int32_t *block_mapping,
                           int num_pairs, int64_t src_num_blocks, int64_t dst_num_blocks,
                           int64_t block_bytes, void *stream)
{
    if (num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0 || block_bytes <= 0)
        return fail(PKV_ERR_INVALID_ARG, "num_pairs=%d src_num_blocks=%lld dst_num_blocks=%lld "
                    "block_bytes=%lld", num_pairs, (long long)src_num_blocks,
                    (long long)dst_num_blocks, (long long)block_bytes);
    if (block_bytes % 16 != 0)
        return fail(PKV_ERR_UNSUPPORTED, "block_bytes %lld is not a multiple of 16",
                    (long long)block_bytes);
    if (num_pairs >= (1 << 30))   // 2 CTAs per pair must fit gridDim.x (< 2^31)
        return fail(PKV_ERR_UNSUPPORTED, "num_pairs %d >= 2^30", num_pairs);
    if (num_pairs == 0)
        return PKV_OK;
    if (!src_key_cache || !src_value_cache || !dst_key_cache || !dst_value_cache || !block_mapping)
        return fail(PKV_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(src_key_cache) || !aligned16(src_value_cache) || !aligned16(dst_key_cache) ||
        !aligned16(dst_value_cache))
        return fail(PKV_ERR_MISALIGNED, "cache pointers must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(block_mapping) & 7u)
        return fail(PKV_ERR_MISALIGNED, "block_mapping must be 8-byte aligned");
    const int64_t vec_per_block = block_bytes / 16;
    const int64_t blocks = 2 * (int64_t)num_pairs;   // one CTA per (pair, K or V)
    cudaError_t e = launch_pdl(pkv::copy_blocks_kernel, dim3((unsigned)blocks), dim3(pkv::kCopyThreads), 0,
                               static_cast<cudaStream_t>(stream),
                               static_cast<const uint4 *>(src_key_cache), static_cast<const uint4 *>(src_value_cache),
                               static_cast<uint4 *>(dst_key_cache), static_cast<uint4 *>(dst_value_cache),
                               block_mapping, num_pairs, src_num_blocks, dst_num_blocks, vec_per_block);
    if (e != cudaSuccess)
        return cuda_fail(e, "copy_blocks_kernel launch");
    return PKV_OK;
}

pkv_status pkv_selftest_bounded_wait(int64_t limit_ns, void *stream)
{
    if (limit_ns <= 0 || limit_ns > 10000000000ll)
        return fail(PKV_ERR_INVALID_ARG, "limit_ns must be in (0, 1e10]");
    pkv::bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        (uint64_t)limit_ns);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e, "bounded_wait_selftest_kernel launch");
    return PKV_OK;
}

pkv_status pkv_kv_cache_write(const void *key, const void *value, const int64_t *slot_mapping,
                              int64_t num_tokens, int num_kv_heads, int head_dim, void *key_cache,
                              void *value_cache, int64_t num_blocks, int block_size,
                              pkv_dtype dtype, void *stream)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 || block_size <= 0)
        return fail(PKV_ERR_INVALID_ARG, "num_tokens=%lld num_kv_heads=%d head_dim=%d "
                    "num_blocks=%lld block_size=%d", (long long)num_tokens, num_kv_heads, head_dim,
                    (long long)num_blocks, block_size);
    if (dtype != PKV_F16 && dtype != PKV_BF16)
        return fail(PKV_ERR_INVALID_ARG, "dtype %d", (int)dtype);
    if ((head_dim * 2) % 16 != 0)
        return fail(PKV_ERR_UNSUPPORTED, "head_dim %d: rows must be a multiple of 16 bytes", head_dim);
    if (num_tokens == 0)
        return PKV_OK;
    if (!key || !value || !slot_mapping || !key_cache || !value_cache)
        return fail(PKV_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return fail(PKV_ERR_MISALIGNED, "key/value/cache pointers must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(slot_mapping) & 7u) != 0)
        return fail(PKV_ERR_MISALIGNED, "slot_mapping must be 8-byte aligned");
    const int64_t vec_per_token = (int64_t)num_kv_heads * head_dim / 8;
    const int64_t n_vec = num_tokens * vec_per_token;
    const int threads = 256;
    int64_t blocks = (n_vec + threads - 1) / threads;
    if (blocks > 148 * 16)
        blocks = 148 * 16;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_pdl(pkv::kv_write_kernel, dim3((unsigned)blocks), dim3(threads), 0, st,
                               static_cast<const uint4 *>(key), static_cast<const uint4 *>(value),
                               slot_mapping, n_vec, vec_per_token, num_blocks * block_size,
                               static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache));
    if (e != cudaSuccess)
        return cuda_fail(e, "kv_write_kernel launch");
    return PKV_OK;
}

pkv_status pkv_decode_plan(int batch, int num_heads, int num_kv_heads, int head_dim, int max_blocks,
                           int block_size, int partition_tokens, int *plan_partition_tokens,
                           int *plan_num_partitions)
{
    pkv_status s = check_shapes(batch, num_heads, num_kv_heads, head_dim, max_blocks, block_size);
    if (s != PKV_OK)
        return s;
    int pt, np;
    plan(batch, num_kv_heads, max_blocks, block_size, partition_tokens, &pt, &np);
    if (plan_partition_tokens)
        *plan_partition_tokens = pt;
    if (plan_num_partitions)
        *plan_num_partitions = np;
    return PKV_OK;
}

size_t pkv_decode_workspace_bytes(int batch, int num_heads, int num_kv_heads, int head_dim,
                                  int max_blocks, int block_size, int partition_tokens)
{
    if (check_shapes(batch, num_heads, num_kv_heads, head_dim, max_blocks, block_size) != PKV_OK)
        return 0;
    int pt, np;
    plan(batch, num_kv_heads, max_blocks, block_size, partition_tokens, &pt, &np);
    if (np <= 1)
        return 0;
    return (size_t)batch * num_heads * np * (size_t)(head_dim + 2) * sizeof(float);
}

pkv_status pkv_paged_attention_decode(const void *query, const void *key_cache,
                                      const void *value_cache, const int32_t *block_tables,
                                      int max_blocks, const int32_t *context_lens, int batch,
                                      int num_heads, int num_kv_heads, int head_dim, int block_size,
                                      int64_t num_blocks, float scale, int partition_tokens,
                                      void *workspace, size_t workspace_bytes, void *out,
                                      pkv_dtype dtype, void *stream)
{
    pkv_status s = check_shapes(batch, num_heads, num_kv_heads, head_dim, max_blocks, block_size);
    if (s != PKV_OK)
        return s;
    if (dtype != PKV_F16 && dtype != PKV_BF16)
        return fail(PKV_ERR_INVALID_ARG, "dtype %d", (int)dtype);
    if (num_blocks <= 0 || num_blocks * block_size >= ((int64_t)1 << 31))
        return fail(PKV_ERR_INVALID_ARG, "num_blocks %lld: need 0 < num_blocks*block_size < 2^31",
                    (long long)num_blocks);
    if (!std::isfinite(scale))
        return fail(PKV_ERR_INVALID_ARG, "scale is not finite");
    if (batch == 0)
        return PKV_OK;
    if (!query || !key_cache || !value_cache || !block_tables || !context_lens || !out)
        return fail(PKV_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out))
        return fail(PKV_ERR_MISALIGNED, "query/cache/out pointers must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u))
        return fail(PKV_ERR_MISALIGNED, "block_tables/context_lens must be 4-byte aligned");

    int pt, np;
    plan(batch, num_kv_heads, max_blocks, block_size, partition_tokens, &pt, &np);
    const size_t need = pkv_decode_workspace_bytes(batch, num_heads, num_kv_heads, head_dim,
                                                   max_blocks, block_size, partition_tokens);
    if (np > 1) {
        if (!workspace || workspace_bytes < need)
            return fail(PKV_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                        workspace ? workspace_bytes : (size_t)0);
        if (!aligned16(workspace))
            return fail(PKV_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    }

    CUtensorMap mk, mv;
    if ((s = make_cache_map(&mk, key_cache, num_blocks, block_size, num_kv_heads, head_dim, dtype)) != PKV_OK)
        return s;
    if ((s = make_cache_map(&mv, value_cache, num_blocks, block_size, num_kv_heads, head_dim, dtype)) != PKV_OK)
        return s;

    pkv::DecodeArgs a;
    a.query = static_cast<const uint16_t *>(query);
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.out = static_cast<uint16_t *>(out);
    const size_t rows = (size_t)batch * num_heads * np;
    float *ws = static_cast<float *>(workspace);
    a.ws_m = np > 1 ? ws : nullptr;
    a.ws_l = np > 1 ? ws + rows : nullptr;
    a.ws_o = np > 1 ? ws + 2 * rows : nullptr;
    a.max_blocks = max_blocks;
    a.num_heads = num_heads;
    a.group = num_heads / num_kv_heads;
    a.num_blocks = (int)num_blocks;
    a.part_tokens = pt;
    a.num_parts = np;
    a.records_only = 0;
    a.scale_log2 = (float)((double)scale * 1.4426950408889634);

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = dtype == PKV_BF16 ? dispatch_decode<true>(head_dim, block_size, mk, mv, a, batch, num_kv_heads, st)
                          : dispatch_decode<false>(head_dim, block_size, mk, mv, a, batch, num_kv_heads, st);
    if (s != PKV_OK)
        return s;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e, "paged_decode_kernel launch");
    if (np > 1) {
        e = dtype == PKV_BF16 ? launch_merge<true>(head_dim, a, context_lens, batch, num_heads, np, pt,
                                                   max_blocks * block_size, st)
                              : launch_merge<false>(head_dim, a, context_lens, batch, num_heads, np,
                                                    pt, max_blocks * block_size, st);
        if (e != cudaSuccess)
            return cuda_fail(e, "lse_merge_kernel launch");
    }
    return PKV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Cascade decode (shared prefixes)
// ---------------------------------------------------------------------------
namespace {

struct CascadePlan {
    int pt;        // partition length in tokens (prefix and suffix)
    int pp;        // prefix partitions
    int ps;        // suffix partitions
    int chunks;    // member chunks per group (128 query rows per prefix CTA)
    size_t m_p, l_p, o_p, m_s, l_s, o_s, total;   // workspace offsets
};

pkv_status cascade_plan(int batch, int Hq, int Hkv, int D, int max_prefix_blocks,
                        int max_suffix_blocks, int max_group_size, int bs, int partition_tokens,
                        CascadePlan *c)
{
    pkv_status s = check_shapes(batch, Hq, Hkv, D, std::max(1, max_suffix_blocks), bs);
    if (s != PKV_OK)
        return s;
    if (max_prefix_blocks <= 0 || max_suffix_blocks <= 0 || max_group_size <= 0)
        return fail(PKV_ERR_INVALID_ARG, "max_prefix_blocks, max_suffix_blocks and max_group_size "
                    "must be positive");
    if ((int64_t)max_prefix_blocks * bs >= ((int64_t)1 << 30))
        return fail(PKV_ERR_INVALID_ARG, "max_prefix_blocks * block_size too large");
    c->pt = partition_tokens > 0 ? (partition_tokens + bs - 1) / bs * bs : kAutoPartitionTokens;
    c->pp = (max_prefix_blocks * bs + c->pt - 1) / c->pt;
    c->ps = (max_suffix_blocks * bs + c->pt - 1) / c->pt;
    const int members_per_cta = pkv::kPfRows / (Hq / Hkv);
    c->chunks = (max_group_size + members_per_cta - 1) / members_per_cta;
    const size_t rp = (size_t)batch * Hq * c->pp, rs = (size_t)batch * Hq * c->ps;
    c->m_p = 0;
    c->l_p = align256(c->m_p + rp * 4);
    c->o_p = align256(c->l_p + rp * 4);
    c->m_s = align256(c->o_p + rp * (size_t)D * 4);
    c->l_s = align256(c->m_s + rs * 4);
    c->o_s = align256(c->l_s + rs * 4);
    c->total = align256(c->o_s + rs * (size_t)D * 4);
    return PKV_OK;
}

template <int D, int BS, bool BF16>
cudaError_t launch_prefix(const CUtensorMap &mq, const CacheMaps &cm,
                          const pkv::CascadeArgs &c, cudaStream_t st)
{
    constexpr int smem = pkv::PfShape<D>::kSmemBytes;
    auto kern = pkv::prefix_tc_kernel<D, BS, BF16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)   // two CTAs (and their TMEM) per SM
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    const dim3 grid((unsigned)c.num_parts, (unsigned)c.num_kv_heads,
                    (unsigned)((size_t)c.num_groups * c.chunks));
    return launch_pdl(kern, grid, dim3(pkv::kPfThreads), smem, st, mq, cm.k, cm.v, cm.k4, cm.v4, c);
}

template <bool BF16>
cudaError_t dispatch_prefix(int D, int bs, const CUtensorMap &mq, const CacheMaps &cm,
                            const pkv::CascadeArgs &c, cudaStream_t st)
{
    if (D == 64 && bs == 16) return launch_prefix<64, 16, BF16>(mq, cm, c, st);
    if (D == 64 && bs == 32) return launch_prefix<64, 32, BF16>(mq, cm, c, st);
    if (D == 128 && bs == 16) return launch_prefix<128, 16, BF16>(mq, cm, c, st);
    return launch_prefix<128, 32, BF16>(mq, cm, c, st);
}

// One-pass cascade: a CTA per (kv head, chunk of 32/G members of a group),
// then free_chunks CTAs per kv head for the sequences outside every group.
template <int D, int BS, bool BF16>
cudaError_t launch_cascade_one_pass(const CUtensorMap &mq, const CacheMaps &cm,
                                    const pkv::CascadeArgs &c, int free_chunks, cudaStream_t st)
{
    constexpr int smem = pkv::PfShape<D>::kSmemBytes;
    auto kern = pkv::cascade_tc_kernel<D, BS, BF16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)   // two CTAs (and their TMEM) per SM
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    const dim3 grid(1u, (unsigned)c.num_kv_heads,
                    (unsigned)((size_t)c.num_groups * c.chunks + (size_t)free_chunks));
    return launch_pdl(kern, grid, dim3(pkv::kPfThreads), smem, st, mq, cm.k, cm.v, cm.k4, cm.v4, c);
}

template <bool BF16>
cudaError_t dispatch_cascade_one_pass(int D, int bs, const CUtensorMap &mq, const CacheMaps &cm,
                                      const pkv::CascadeArgs &c, int free_chunks, cudaStream_t st)
{
    if (D == 64 && bs == 16) return launch_cascade_one_pass<64, 16, BF16>(mq, cm, c, free_chunks, st);
    if (D == 64 && bs == 32) return launch_cascade_one_pass<64, 32, BF16>(mq, cm, c, free_chunks, st);
    if (D == 128 && bs == 16) return launch_cascade_one_pass<128, 16, BF16>(mq, cm, c, free_chunks, st);
    return launch_cascade_one_pass<128, 32, BF16>(mq, cm, c, free_chunks, st);
}

}  // namespace

extern "C" size_t pkv_decode_cascade_workspace_bytes(int batch, int num_heads, int num_kv_heads,
                                                     int head_dim, int max_prefix_blocks,
                                                     int max_suffix_blocks, int max_group_size,
                                                     int block_size, int partition_tokens)
{
    CascadePlan c;
    if (cascade_plan(batch, num_heads, num_kv_heads, head_dim, max_prefix_blocks, max_suffix_blocks,
                     max_group_size, block_size, partition_tokens, &c) != PKV_OK)
        return 0;
    return c.total;
}

namespace {

// The one pass takes 32 query rows per CTA (32/G members): chunks of a group
// and CTAs for the sequences outside every group, per kv head.
constexpr int kOnePassRows = pkv::kCasRows;
struct OnePassGrid {
    int64_t group_chunks;   // member chunks of all groups
    int chunks;             // member chunks per group
    int free_chunks;        // chunks over the whole batch for ungrouped sequences
};
OnePassGrid one_pass_grid(int batch, int G, int max_group_size, int num_groups)
{
    const int per_cta = kOnePassRows / G;
    OnePassGrid g;
    g.chunks = (max_group_size + per_cta - 1) / per_cta;
    g.group_chunks = (int64_t)num_groups * g.chunks;
    g.free_chunks = (batch + per_cta - 1) / per_cta;
    return g;
}

// The one-pass choice of pkv_paged_attention_decode_cascade (see the header).
bool cascade_one_pass(int batch, int G, int num_kv_heads, int max_group_size, int num_groups,
                      int partition_tokens)
{
    const OnePassGrid g = one_pass_grid(batch, G, max_group_size, num_groups);
    return num_groups > 0 && g.group_chunks + g.free_chunks <= 65535 &&
           (partition_tokens < 0 ||
            (partition_tokens == 0 && g.group_chunks * num_kv_heads >= kPlanSmCount));
}

}  // namespace

extern "C" pkv_status pkv_decode_cascade_plan(int batch, int num_heads, int num_kv_heads, int head_dim,
                                              int max_prefix_blocks, int max_suffix_blocks,
                                              int max_group_size, int num_groups, int block_size,
                                              int partition_tokens, int *one_pass,
                                              int *prefix_partitions)
{
    CascadePlan plan;
    pkv_status s = cascade_plan(batch, num_heads, num_kv_heads, head_dim, max_prefix_blocks,
                                max_suffix_blocks, max_group_size, block_size, partition_tokens, &plan);
    if (s != PKV_OK)
        return s;
    if (num_groups < 0 || num_groups > batch)
        return fail(PKV_ERR_INVALID_ARG, "num_groups %d (0 .. batch)", num_groups);
    const bool op = cascade_one_pass(batch, num_heads / num_kv_heads, num_kv_heads, max_group_size,
                                     num_groups, partition_tokens);
    if (one_pass)
        *one_pass = op ? 1 : 0;
    if (prefix_partitions)
        *prefix_partitions = op ? 1 : plan.pp;
    return PKV_OK;
}

extern "C" pkv_status pkv_paged_attention_decode_cascade(
    const void *query, const void *key_cache, const void *value_cache, const int32_t *prefix_tables,
    int max_prefix_blocks, const int32_t *prefix_lens, const int32_t *group_start, int num_groups,
    int max_group_size, const int32_t *suffix_tables, int max_suffix_blocks,
    const int32_t *suffix_lens, int batch, int num_heads, int num_kv_heads, int head_dim,
    int block_size, int64_t num_blocks, float scale, int partition_tokens, void *workspace,
    size_t workspace_bytes, void *out, pkv_dtype dtype, void *stream)
{
    CascadePlan plan;
    pkv_status s = cascade_plan(batch, num_heads, num_kv_heads, head_dim, max_prefix_blocks,
                                max_suffix_blocks, max_group_size, block_size, partition_tokens, &plan);
    if (s != PKV_OK)
        return s;
    if (dtype != PKV_F16 && dtype != PKV_BF16)
        return fail(PKV_ERR_INVALID_ARG, "dtype %d", (int)dtype);
    if (num_groups < 0 || num_groups > batch)
        return fail(PKV_ERR_INVALID_ARG, "num_groups %d (0 .. batch)", num_groups);
    if (num_blocks <= 0 || num_blocks * block_size >= ((int64_t)1 << 31))
        return fail(PKV_ERR_INVALID_ARG, "num_blocks %lld: need 0 < num_blocks*block_size < 2^31",
                    (long long)num_blocks);
    if (!std::isfinite(scale))
        return fail(PKV_ERR_INVALID_ARG, "scale is not finite");
    if (batch == 0)
        return PKV_OK;
    if (!query || !key_cache || !value_cache || !suffix_tables || !suffix_lens || !out ||
        (num_groups > 0 && (!prefix_tables || !prefix_lens || !group_start)))
        return fail(PKV_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out))
        return fail(PKV_ERR_MISALIGNED, "query/cache/out pointers must be 16-byte aligned");
    if (!workspace || workspace_bytes < plan.total)
        return fail(PKV_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", plan.total,
                    workspace ? workspace_bytes : (size_t)0);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(PKV_ERR_MISALIGNED, "workspace must be 256-byte aligned");

    CUtensorMap mk, mv;
    if ((s = make_cache_map(&mk, key_cache, num_blocks, block_size, num_kv_heads, head_dim, dtype)) != PKV_OK)
        return s;
    if ((s = make_cache_map(&mv, value_cache, num_blocks, block_size, num_kv_heads, head_dim, dtype)) != PKV_OK)
        return s;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const float scale_log2 = (float)((double)scale * 1.4426950408889634);

    // One pass (prefix and own blocks in one CTA, no records, no merge) when
    // asked for (partition_tokens < 0) or, automatically, when the groups'
    // CTAs alone fill the GPU; else the prefix is split into partitions.
    const int G = num_heads / num_kv_heads;
    const bool one_pass =
        cascade_one_pass(batch, G, num_kv_heads, max_group_size, num_groups, partition_tokens);
    if (!one_pass && (int64_t)num_groups * plan.chunks > 65535)
        return fail(PKV_ERR_UNSUPPORTED, "num_groups x member chunks (%lld) above 65535",
                    (long long)num_groups * plan.chunks);
    if (one_pass) {
        const OnePassGrid og = one_pass_grid(batch, G, max_group_size, num_groups);
        CUtensorMap mq;
        CacheMaps cm;
        if ((s = make_query_map(&mq, query, batch, num_heads, head_dim, G, kOnePassRows / G, dtype)) != PKV_OK ||
            (s = make_cache_maps(&cm, key_cache, value_cache, num_blocks, block_size, num_kv_heads,
                                 head_dim, dtype)) != PKV_OK)
            return s;
        pkv::CascadeArgs c{};
        c.query = static_cast<const uint16_t *>(query);
        c.prefix_tables = prefix_tables;
        c.prefix_lens = prefix_lens;
        c.group_start = group_start;
        c.batch = batch;
        c.max_prefix_blocks = max_prefix_blocks;
        c.num_groups = num_groups;
        c.max_group_size = max_group_size;
        c.num_heads = num_heads;
        c.num_kv_heads = num_kv_heads;
        c.group = G;
        c.num_blocks = (int)num_blocks;
        c.chunks = og.chunks;
        c.scale_log2 = scale_log2;
        c.suffix_tables = suffix_tables;
        c.suffix_lens = suffix_lens;
        c.out = static_cast<uint16_t *>(out);
        c.max_suffix_blocks = max_suffix_blocks;
        cudaError_t e = dtype == PKV_BF16
                            ? dispatch_cascade_one_pass<true>(head_dim, block_size, mq, cm, c, og.free_chunks, st)
                            : dispatch_cascade_one_pass<false>(head_dim, block_size, mq, cm, c, og.free_chunks, st);
        if (e != cudaSuccess)
            return cuda_fail(e, "cascade_tc_kernel launch");
        return PKV_OK;
    }

    // level 1: shared prefixes, one pass per group
    pkv::CascadeArgs c{};
    c.query = static_cast<const uint16_t *>(query);
    c.prefix_tables = prefix_tables;
    c.prefix_lens = prefix_lens;
    c.group_start = group_start;
    c.rec_m = reinterpret_cast<float *>(ws + plan.m_p);
    c.rec_l = reinterpret_cast<float *>(ws + plan.l_p);
    c.rec_o = reinterpret_cast<float *>(ws + plan.o_p);
    c.batch = batch;
    c.max_prefix_blocks = max_prefix_blocks;
    c.num_groups = num_groups;
    c.max_group_size = max_group_size;
    c.num_heads = num_heads;
    c.num_kv_heads = num_kv_heads;
    c.group = num_heads / num_kv_heads;
    c.num_blocks = (int)num_blocks;
    c.part_tokens = plan.pt;
    c.num_parts = plan.pp;
    c.chunks = plan.chunks;
    c.scale_log2 = scale_log2;
    cudaError_t e = cudaSuccess;
    if (num_groups > 0) {
        // the members of a group are consecutive query rows: a Q tile is
        // 128/G members x the G heads of one kv head
        CUtensorMap mq;
        if ((s = make_query_map(&mq, query, batch, num_heads, head_dim, c.group,
                                pkv::kPfRows / c.group, dtype)) != PKV_OK)
            return s;
        CacheMaps cm;
        if ((s = make_cache_maps(&cm, key_cache, value_cache, num_blocks, block_size, num_kv_heads,
                                 head_dim, dtype)) != PKV_OK)
            return s;
        e = dtype == PKV_BF16 ? dispatch_prefix<true>(head_dim, block_size, mq, cm, c, st)
                              : dispatch_prefix<false>(head_dim, block_size, mq, cm, c, st);
        if (e != cudaSuccess)
            return cuda_fail(e, "prefix_tc_kernel launch");
    }

    // level 2: each sequence's own blocks, as partition records
    pkv::DecodeArgs a;
    a.query = c.query;
    a.block_tables = suffix_tables;
    a.context_lens = suffix_lens;
    a.out = static_cast<uint16_t *>(out);
    a.ws_m = reinterpret_cast<float *>(ws + plan.m_s);
    a.ws_l = reinterpret_cast<float *>(ws + plan.l_s);
    a.ws_o = reinterpret_cast<float *>(ws + plan.o_s);
    a.max_blocks = max_suffix_blocks;
    a.num_heads = num_heads;
    a.group = num_heads / num_kv_heads;
    a.num_blocks = (int)num_blocks;
    a.part_tokens = plan.ps > 1 ? plan.pt : max_suffix_blocks * block_size;
    a.num_parts = plan.ps;
    a.records_only = 1;
    a.scale_log2 = scale_log2;
    s = dtype == PKV_BF16 ? dispatch_decode<true>(head_dim, block_size, mk, mv, a, batch, num_kv_heads, st)
                          : dispatch_decode<false>(head_dim, block_size, mk, mv, a, batch, num_kv_heads, st);
    if (s != PKV_OK)
        return s;

    // merge prefix and suffix records of every (sequence, query head) row:
    // one warp per row
    constexpr int NT = 256;
    const int rows = batch * num_heads;
    const int suffix_span = max_suffix_blocks * block_size;
    auto go = [&](auto kern) {
        constexpr int rows_per_cta = NT / 32;
        return launch_pdl(kern, dim3((unsigned)((rows + rows_per_cta - 1) / rows_per_cta)), dim3(NT), 0,
                          st, c, a.ws_m, a.ws_l, a.ws_o, suffix_lens, plan.ps, a.part_tokens,
                          suffix_span, a.out);
    };
    if (dtype == PKV_BF16)
        e = head_dim == 64 ? go(pkv::lse_merge_cascade_kernel<true, 64, NT>)
                           : go(pkv::lse_merge_cascade_kernel<true, 128, NT>);
    else
        e = head_dim == 64 ? go(pkv::lse_merge_cascade_kernel<false, 64, NT>)
                           : go(pkv::lse_merge_cascade_kernel<false, 128, NT>);
    if (e != cudaSuccess)
        return cuda_fail(e, "lse_merge_cascade_kernel launch");
    return PKV_OK;
}

// ---------------------------------------------------------------------------
// Chunked prefill
// ---------------------------------------------------------------------------
namespace {

template <int D, int BS, bool BF16>
cudaError_t launch_prefill(const CUtensorMap &mq, const CacheMaps &cm,
                           const pkv::PrefillArgs &p, int max_query_len, cudaStream_t st)
{
    constexpr int smem = pkv::PfShape<D>::kSmemBytes;
    auto kern = pkv::prefill_tc_kernel<D, BS, BF16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)   // two CTAs (and their TMEM) per SM
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    // a CTA per (tiles_per_cta row tiles, kv head, sequence)
    const int tokens_per_cta = pkv::kPfRows / p.group;
    const int row_tiles = (max_query_len + tokens_per_cta - 1) / tokens_per_cta;
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, current_device());
    if (e != cudaSuccess)
        return e;
    pkv::PrefillArgs q = p;
    q.tiles_per_cta = prefill_tiles_per_cta(p.batch, p.num_kv_heads, row_tiles, std::max(sms, 1));
    const dim3 grid((unsigned)((row_tiles + q.tiles_per_cta - 1) / q.tiles_per_cta),
                    (unsigned)p.num_kv_heads, (unsigned)p.batch);
    return launch_pdl(kern, grid, dim3(pkv::kPfThreads), smem, st, mq, cm.k, cm.v, cm.k4, cm.v4, q);
}

template <bool BF16>
cudaError_t dispatch_prefill(int D, int bs, const CUtensorMap &mq, const CacheMaps &cm,
                             const pkv::PrefillArgs &p, int max_query_len, cudaStream_t st)
{
    if (D == 64 && bs == 16) return launch_prefill<64, 16, BF16>(mq, cm, p, max_query_len, st);
    if (D == 64 && bs == 32) return launch_prefill<64, 32, BF16>(mq, cm, p, max_query_len, st);
    if (D == 128 && bs == 16) return launch_prefill<128, 16, BF16>(mq, cm, p, max_query_len, st);
    return launch_prefill<128, 32, BF16>(mq, cm, p, max_query_len, st);
}

}  // namespace

extern "C" pkv_status pkv_paged_attention_prefill(
    const void *query, int num_tokens, const int32_t *query_start, int max_query_len,
    const void *key_cache,
    const void *value_cache, const int32_t *block_tables, int max_blocks,
    const int32_t *context_lens, int batch, int num_heads, int num_kv_heads, int head_dim,
    int block_size, int64_t num_blocks, float scale, void *out, pkv_dtype dtype, void *stream)
{
    pkv_status s = check_shapes(batch, num_heads, num_kv_heads, head_dim, max_blocks, block_size);
    if (s != PKV_OK)
        return s;
    if (dtype != PKV_F16 && dtype != PKV_BF16)
        return fail(PKV_ERR_INVALID_ARG, "dtype %d", (int)dtype);
    if (num_tokens < 0)
        return fail(PKV_ERR_INVALID_ARG, "num_tokens %d", num_tokens);
    if (max_query_len < 0 || max_query_len > max_blocks * block_size)
        return fail(PKV_ERR_INVALID_ARG, "max_query_len %d (0 .. max_blocks*block_size)", max_query_len);
    if ((int64_t)max_query_len * (num_heads / num_kv_heads) > ((int64_t)1 << 30))
        return fail(PKV_ERR_UNSUPPORTED, "max_query_len too large");
    if (num_blocks <= 0 || num_blocks * block_size >= ((int64_t)1 << 31))
        return fail(PKV_ERR_INVALID_ARG, "num_blocks %lld: need 0 < num_blocks*block_size < 2^31",
                    (long long)num_blocks);
    if (!std::isfinite(scale))
        return fail(PKV_ERR_INVALID_ARG, "scale is not finite");
    if (batch == 0 || max_query_len == 0 || num_tokens == 0)
        return PKV_OK;
    if (!query || !query_start || !key_cache || !value_cache || !block_tables || !context_lens || !out)
        return fail(PKV_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out))
        return fail(PKV_ERR_MISALIGNED, "query/cache/out pointers must be 16-byte aligned");
    CUtensorMap mq;
    CacheMaps cm;
    const int group = num_heads / num_kv_heads;
    if ((s = make_query_map(&mq, query, num_tokens, num_heads, head_dim, group, pkv::kPfRows / group,
                            dtype)) != PKV_OK ||
        (s = make_cache_maps(&cm, key_cache, value_cache, num_blocks, block_size, num_kv_heads, head_dim,
                             dtype)) != PKV_OK)
        return s;
    pkv::PrefillArgs p;
    p.query = static_cast<const uint16_t *>(query);
    p.query_start = query_start;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.out = static_cast<uint16_t *>(out);
    p.batch = batch;
    p.num_tokens = num_tokens;
    p.max_query_len = max_query_len;
    p.max_blocks = max_blocks;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = num_heads / num_kv_heads;
    p.num_blocks = (int)num_blocks;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = dtype == PKV_BF16
                        ? dispatch_prefill<true>(head_dim, block_size, mq, cm, p, max_query_len, st)
                        : dispatch_prefill<false>(head_dim, block_size, mq, cm, p, max_query_len, st);
    if (e != cudaSuccess)
        return cuda_fail(e, "prefill_tc_kernel launch");
    return PKV_OK;
}

// ---------------------------------------------------------------------------
// Decode with a library-owned workspace (no allocation by anyone at call time)
// ---------------------------------------------------------------------------
// Some callers cannot allocate device memory when they decode: a custom
// allocator that owns the whole pool, a runtime that forbids cudaMalloc on its
// serving path, or plain C code with no allocator at all.  For them the split
// plan's workspace lives in this fixed array, reserved in device memory on
// every GPU that loads the library and kept until the process exits.  Calls
// share it, so two calls whose kernels overlap on the GPU (different streams,
// or different host threads) race on it and must be serialised by the caller.
// The array keeps whatever the last call left; nothing in it has to start at
// zero, because every partition record the merge reads is written earlier in
// the same call.
namespace {

constexpr size_t kStaticWorkspaceBytes = PKV_STATIC_WORKSPACE_BYTES;
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// The current context's unique id (cuCtxGetId), or 0 when there is no
// current context or the driver does not offer the call.  Ids are never
// reused within a process, unlike context handles.
unsigned long long current_context_id()
{
    using GetCurrentFn = CUresult (*)(CUcontext *);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long *);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_static_workspace in the current context of `dev`.  In
// host code the symbol is only a stand-in for the device array, so its
// address comes from cudaGetSymbolAddress, called with that device current.
// The address is kept per device together with the id of the context it was
// looked up in: a new context on the device (after cudaDeviceReset, say)
// reloads the module, and the next call looks the address up again.
pkv_status static_workspace_ptr(int dev, void **ptr)
{
    struct Entry {
        unsigned long long ctx;
        void *addr;
    };
    static Entry cache[64] = {};
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    const bool slot = dev >= 0 && dev < 64;
    const unsigned long long id = current_context_id();
    if (slot && id != 0 && cache[dev].addr && cache[dev].ctx == id) {
        *ptr = cache[dev].addr;
        return PKV_OK;
    }
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
    // the lookup made the device's primary context current if none was
    const unsigned long long now = current_context_id();
    if (slot && now != 0)
        cache[dev] = Entry{now, p};
    *ptr = p;
    return PKV_OK;
}

}  // namespace

extern "C" pkv_status pkv_paged_attention_decode_static_workspace(
    const void *query, const void *key_cache, const void *value_cache, const int32_t *block_tables,
    int max_blocks, const int32_t *context_lens, int batch, int num_heads, int num_kv_heads,
    int head_dim, int block_size, int64_t num_blocks, float scale, int partition_tokens, void *out,
    pkv_dtype dtype, void *stream)
{
    pkv_status s = check_shapes(batch, num_heads, num_kv_heads, head_dim, max_blocks, block_size);
    if (s != PKV_OK)
        return s;
    const size_t need = pkv_decode_workspace_bytes(batch, num_heads, num_kv_heads, head_dim,
                                                   max_blocks, block_size, partition_tokens);
    if (need > kStaticWorkspaceBytes)
        return fail(PKV_ERR_WORKSPACE,
                    "this call needs %zu bytes of workspace but the library's static workspace "
                    "holds %zu (PKV_STATIC_WORKSPACE_BYTES); use pkv_paged_attention_decode with a "
                    "caller-provided workspace, fewer partitions or a smaller batch",
                    need, kStaticWorkspaceBytes);
    void *ws = nullptr;
    if (need > 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaGetDevice");
        if ((s = static_workspace_ptr(dev, &ws)) != PKV_OK)
            return s;
    }
    return pkv_paged_attention_decode(query, key_cache, value_cache, block_tables, max_blocks,
                                      context_lens, batch, num_heads, num_kv_heads, head_dim,
                                      block_size, num_blocks, scale, partition_tokens, ws,
                                      need > 0 ? kStaticWorkspaceBytes : 0, out, dtype, stream);
}
