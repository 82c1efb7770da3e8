// pkv_kernels.cuh -- sm_100a kernels of the paged KV-cache hot path.
//
// Sources (web pages describing vLLM's paged KV cache):
//   [YK] "大模型推理框架 vLLM 源码解析 一" (ai.yueke.cloud), section 三: caches
//        of shape [num_blocks, block_size, num_heads, head_dim]; for token j of
//        sequence i the physical block is block_tables[i][j // block_size] and
//        the offset j % block_size.
//   [FC] "23.1 vLLM：高吞吐推理框架原理与部署" (r.flycode100.com), section 二.2
//        step 3: the kernel finds the blocks scattered in memory through the
//        block table and computes attention piece by piece.
//   [MH] "大模型推理框架VLLM-0.7.3源码" (mhpq.cn), sections 2.1 / 3.3:
//        slot_mapping names the cell each current token's K/V is written to.
//
// Design (B200):
//   kv_write_kernel    one 16-byte vector per thread: coalesced reads of the
//                      new rows, 16-byte stores into the slot's row.
//   paged_decode_kernel one CTA per (partition, kv head, sequence).  Each of
//                      its NW warps streams every NW-th block of the partition
//                      through its own S-deep ring of shared-memory stages,
//                      filled by TMA (3-D tensor map over the cache viewed as
//                      [num_blocks*block_size, num_kv_heads, head_dim], 128-byte
//                      swizzle, evict-first L2 policy).  The whole GQA group of
//                      query heads is one mma tile, so each K/V block is read
//                      from HBM once per group:
//                        S^T[tokens x heads] = K[tokens x D] * Q^T[D x heads]
//                        O^T[D x heads]     += V^T[D x tokens] * P^T[tokens x heads]
//                      with mma.sync m16n8k16 (fp32 accumulate), ldmatrix from
//                      the swizzled stages, and P^T formed in registers with
//                      movmatrix.  P is split into a 16-bit high part and a
//                      16-bit remainder, each multiplied by V, so the weights
//                      keep ~16 extra bits.  Online softmax (running max/sum
//                      per head, base-2 exponent) is per warp; warps merge by
//                      log-sum-exp in shared memory at the end.
//   lse_merge_kernel   split-context plans: merges the partitions' (max,
//                      normaliser, normalised output) into the final row.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "pagedkv.h"
#include "pkv_ptx.cuh"

namespace pkv {

// Per-device error word (see PKV_DEVFLAG_* in pagedkv.h).
__device__ unsigned int g_device_flags;

constexpr float kNegInf = -__builtin_huge_valf();
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per pipeline wait

__device__ __forceinline__ void raise_flag(unsigned int bit) { atomicOr(&g_device_flags, bit); }

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    if constexpr (BF16) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    } else {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
}

template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t x)
{
    if constexpr (BF16) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&x);
        return __bfloat1622float2(v);
    } else {
        __half2 v = *reinterpret_cast<__half2 *>(&x);
        return __half22float2(v);
    }
}

template <bool BF16>
__device__ __forceinline__ uint16_t to_storage(float x)
{
    if constexpr (BF16) {
        __nv_bfloat16 v = __float2bfloat16_rn(x);
        return *reinterpret_cast<uint16_t *>(&v);
    } else {
        __half v = __float2half_rn(x);
        return *reinterpret_cast<uint16_t *>(&v);
    }
}

// D/32 consecutive floats of a record, one lane's share
template <int D>
__device__ __forceinline__ void load_slice(const float *p, float (&v)[D / 32])
{
    if constexpr (D == 128) {
        const float4 x = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    } else {
        const float2 x = __ldg(reinterpret_cast<const float2 *>(p));
        v[0] = x.x; v[1] = x.y;
    }
}

// ---------------------------------------------------------------------------
// KV write through slot_mapping ([MH] 2.1, 3.3)
// ---------------------------------------------------------------------------
// n_vec = num_tokens * num_kv_heads * vec_per_row 16-byte vectors; vector i of
// the input lives at row i / vec_per_row = t * Hkv + h, and goes to the cache
// row slot * Hkv + h at the same vector offset.
__global__ void kv_write_kernel(const uint4 *__restrict__ key, const uint4 *__restrict__ value,
                                const int64_t *__restrict__ slot_mapping, int64_t n_vec,
                                int64_t vec_per_token, int64_t total_slots,
                                uint4 *__restrict__ key_cache, uint4 *__restrict__ value_cache)
{
    // Launched with programmatic dependent launch, this grid may become
    // resident while the previous kernel on the stream finishes (its launch
    // latency is then hidden): it waits for that kernel before it touches
    // memory, which may have read these cells or written these inputs.  A
    // decode launched after this kernel may start its own set-up now; it waits
    // for this grid to finish before it reads any memory.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec; i += stride) {
        const int64_t t = i / vec_per_token;
        const int64_t within = i - t * vec_per_token;   // h * vec_per_row + v
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0)
            continue;                                    // padding token
        if (slot >= total_slots) {
            if (within == 0)
                raise_flag(PKV_DEVFLAG_SLOT_RANGE);
            continue;
        }
        const int64_t dst = slot * vec_per_token + within;
        const uint4 k = __ldg(key + i);
        const uint4 v = __ldg(value + i);
        key_cache[dst] = k;
        value_cache[dst] = v;
    }
}

// ---------------------------------------------------------------------------
// One K/V block of the group tile, for one warp
// ---------------------------------------------------------------------------
// sk / sv: shared addresses of the swizzled K and V tiles of one block (BS
// token rows of D columns, 64-column halves of BS*128 bytes, 128-byte
// swizzle); valid: rows holding tokens (later rows are masked; their V rows
// must be zero).  qf: Q^T fragments of this warp's 8 query columns.  Updates
// the running max m_run / lane-partial normaliser l_run of the lane's columns
// 2c, 2c+1 (base-2 units) and the O^T accumulators (high part and remainder of
// P, each times V):
//   S^T[t, n] = sum_d K[t, d] Q[n, d]            (mma.sync m16n8k16, fp32)
//   online softmax per column n
//   O^T[d, n] += sum_t V[t, d] P[t, n]
template <int D, int BS, bool BF16>
__device__ __forceinline__ void attend_block(uint32_t sk, uint32_t sv, int valid,
                                             const uint32_t (&qf)[D / 16][2], float scale_log2,
                                             float (&m_run)[2], float (&l_run)[2],
                                             float (&acc_hi)[D / 16][4], float (&acc_lo)[D / 16][4],
                                             int lane)
{
    constexpr int MT = BS / 16;
    constexpr int KS = D / 16;
    constexpr int kHalfBytes = BS * 128;
    // ---- scores: S^T[t, n] = sum_d K[t, d] Q[n, d] ----
    float sc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        float s0[4] = {0.f, 0.f, 0.f, 0.f};   // two accumulation chains (even / odd k)
        float s1[4] = {0.f, 0.f, 0.f, 0.f};
        const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int chunk = (ks & 3) * 2 + (lane >> 4);
            const uint32_t addr = sk + (uint32_t)((ks >> 2) * kHalfBytes + row * 128 +
                                                  ((chunk ^ (row & 7)) << 4));
            uint32_t af[4];
            ldsm_x4(addr, af);
            if (ks & 1)
                mma_16816<BF16>(s1, af, qf[ks][0], qf[ks][1]);
            else
                mma_16816<BF16>(s0, af, qf[ks][0], qf[ks][1]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
            sc[mt][i] = s0[i] + s1[i];
    }

    // ---- online softmax (base 2), per column n = 2c + j ----
    float mx[2] = {kNegInf, kNegInf};
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = mt * 16 + (lane >> 2) + (i >= 2 ? 8 : 0);
            const float v = t < valid ? sc[mt][i] * scale_log2 : kNegInf;
            sc[mt][i] = v;
            mx[i & 1] = fmaxf(mx[i & 1], v);
        }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 4));
        mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 8));
        mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 16));
    }
    // The running maximum moves only when a block's maximum exceeds it by
    // more than 8 (base 2), so the weights stay <= 2^8 and O and the
    // normaliser are rescaled only then, not on every block that raises the
    // maximum a little.  alpha is 0 on a column's first scored block
    // (m_run = -inf) and 1 while a column has seen no token at all.
    float alpha[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const bool move = mx[j] > m_run[j] + 8.f;
        const float mnew = move ? mx[j] : m_run[j];
        alpha[j] = move ? ex2(m_run[j] - mnew) : 1.f;
        m_run[j] = mnew;
    }
    float ls[2] = {0.f, 0.f};
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float p = m_run[i & 1] == kNegInf ? 0.f : ex2(sc[mt][i] - m_run[i & 1]);
            sc[mt][i] = p;
            ls[i & 1] += p;
        }
#pragma unroll
    for (int j = 0; j < 2; ++j)
        l_run[j] = l_run[j] * alpha[j] + ls[j];
    if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
        for (int dt = 0; dt < KS; ++dt) {
            acc_hi[dt][0] *= alpha[0];
            acc_hi[dt][1] *= alpha[1];
            acc_hi[dt][2] *= alpha[0];
            acc_hi[dt][3] *= alpha[1];
            acc_lo[dt][0] *= alpha[0];
            acc_lo[dt][1] *= alpha[1];
            acc_lo[dt][2] *= alpha[0];
            acc_lo[dt][3] *= alpha[1];
        }
    }

    // ---- O^T[d, n] += sum_t V[t, d] P[t, n] ----
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const uint32_t h01 = pack2<BF16>(sc[mt][0], sc[mt][1]);
        const uint32_t h23 = pack2<BF16>(sc[mt][2], sc[mt][3]);
        const float2 f01 = unpack2<BF16>(h01);
        const float2 f23 = unpack2<BF16>(h23);
        const uint32_t l01 = pack2<BF16>(sc[mt][0] - f01.x, sc[mt][1] - f01.y);
        const uint32_t l23 = pack2<BF16>(sc[mt][2] - f23.x, sc[mt][3] - f23.y);
        const uint32_t bh0 = movmatrix_trans(h01);
        const uint32_t bh1 = movmatrix_trans(h23);
        const uint32_t bl0 = movmatrix_trans(l01);
        const uint32_t bl1 = movmatrix_trans(l23);
        const int t = mt * 16 + (lane & 7) + (lane >> 4) * 8;
#pragma unroll
        for (int dt = 0; dt < KS; ++dt) {
            const int d = dt * 16 + ((lane >> 3) & 1) * 8;
            const int chunk = (d & 63) >> 3;
            const uint32_t addr = sv + (uint32_t)((d >> 6) * kHalfBytes + t * 128 +
                                                  ((chunk ^ (t & 7)) << 4));
            uint32_t af[4];
            ldsm_x4_trans(addr, af);
            mma_16816<BF16>(acc_hi[dt], af, bh0, bh1);
            mma_16816<BF16>(acc_lo[dt], af, bl0, bl1);
        }
    }

}

// ---------------------------------------------------------------------------
// Decode
// ---------------------------------------------------------------------------
struct DecodeArgs {
    const uint16_t *query;        // [B, Hq, D]
    const int32_t *block_tables;  // [B, max_blocks]
    const int32_t *context_lens;  // [B]
    uint16_t *out;                // [B, Hq, D]        (single-pass plans)
    float *ws_m;                  // [B*Hq, P]          (split plans)
    float *ws_l;                  // [B*Hq, P]
    float *ws_o;                  // [B*Hq, P, D]
    int max_blocks;
    int num_heads;
    int group;                    // Hq / Hkv, 1..8
    int num_blocks;
    int part_tokens;              // tokens per partition (multiple of block size)
    int num_parts;                // partitions per sequence (1 = single pass)
    int records_only;             // 1: write partition records even for one partition
    float scale_log2;             // scale * log2(e)
};

template <int D, int BS, int NW, int S>
struct DecodeShape {
    static constexpr int kHalves = D / 64;             // 64-element (128-byte) column halves
    static constexpr int kHalfBytes = BS * 128;        // one half of one tile
    static constexpr int kTileBytes = kHalves * kHalfBytes;   // BS x D x 2 bytes
    static constexpr int kStageBytes = 2 * kTileBytes;        // K tile + V tile
    static constexpr int kRingBytes = NW * S * kStageBytes;
    static constexpr int kScratchBytes = NW * 8 * D * 4 + NW * 16 * 4;
    static constexpr int kSmemBytes =
        (kRingBytes > kScratchBytes ? kRingBytes : kScratchBytes) + 1024;   // + alignment slack
};

template <int D, int BS, bool BF16, int NW, int S>
__global__ void __launch_bounds__(NW * 32)
paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const DecodeArgs a)
{
    using Shape = DecodeShape<D, BS, NW, S>;
    constexpr int kHalfBytes = Shape::kHalfBytes;
    constexpr int kTileBytes = Shape::kTileBytes;
    constexpr int kStageBytes = Shape::kStageBytes;
    constexpr int KS = D / 16;    // 16-wide column tiles of the head dimension
    static_assert(BS % 16 == 0 && D % 64 == 0, "tile shape");

    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[NW * S];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int part = blockIdx.x;
    const int kvh = blockIdx.y;
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int Hq = a.num_heads;
    const int G = a.group;
    const bool split = a.num_parts > 1 || a.records_only;

    // Set-up that touches no global memory, then wait for the previous kernel
    // on the stream (programmatic dependent launch lets this CTA start while
    // it finishes; it may have written the caches or this call's inputs).
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < S; ++s)
            mbar_init(smem_addr(&bars[warp * S + s]), 1);
    }
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    fence_mbar_init();
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    // The context length, this warp's first 32 table entries and the query are
    // loaded together: the table window is bounded by the partition and the
    // row, not by the length, so it does not wait for it.
    const int blk0 = (part * a.part_tokens) / BS;
    const int part_blocks = a.part_tokens / BS;
    const int32_t *trow = a.block_tables + (size_t)b * a.max_blocks + blk0 + warp;
    int ids;   // lane j holds the physical id of this warp's block (window*32 + j)
    {
        const int lb = warp + lane * NW;   // block of window 0 within the partition
        ids = (lb < part_blocks && blk0 + lb < a.max_blocks) ? __ldg(trow + (size_t)lane * NW) : 0;
    }
    int L = __ldg(a.context_lens + b);

    // Q^T as the B operand of S^T = K Q^T: column n = query head kvh*G + n of
    // the group (n >= G are zero columns), row k = head-dim index.
    uint32_t qf[KS][2];
    {
        const int n = lane >> 2;
        const int c = lane & 3;
        const uint32_t *q32 = reinterpret_cast<const uint32_t *>(
            a.query + ((size_t)b * Hq + (size_t)kvh * G + (n < G ? n : 0)) * D);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qf[ks][0] = n < G ? __ldg(q32 + ks * 8 + c) : 0u;
            qf[ks][1] = n < G ? __ldg(q32 + ks * 8 + 4 + c) : 0u;
        }
    }

    const int span = a.max_blocks * BS;
    if (L < 0 || L > span) {
        if (threadIdx.x == 0 && part == 0 && kvh == 0)
            raise_flag(PKV_DEVFLAG_CONTEXT_RANGE);
        L = L < 0 ? 0 : span;
    }
    const int tok0 = part * a.part_tokens;
    const int tok1 = min(L, tok0 + a.part_tokens);
    if (tok1 <= tok0) {
        // Nothing to attend to.  Single pass: a zero row (empty context).
        // Split: the merge never reads partitions past the end.
        if (!split) {
            for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
                const size_t row = (size_t)b * Hq + (size_t)kvh * G + idx / D;
                a.out[row * D + idx % D] = 0;
            }
        }
        return;
    }
    const int nblk = (tok1 - tok0 + BS - 1) / BS;

    // This warp's blocks: logical blocks blk0 + warp + k*NW, k = 0 .. nk-1.
    const int nk = nblk > warp ? (nblk - warp + NW - 1) / NW : 0;
    uint8_t *ring = smem + (size_t)warp * S * kStageBytes;
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bar0 = smem_addr(&bars[warp * S]);
    const uint64_t policy = policy_evict_first();

    auto issue = [&](int k) {
        if ((k & 31) == 0 && k > 0) {
            const int kk = k + lane;
            ids = kk < nk ? __ldg(trow + (size_t)kk * NW) : 0;
        }
        int blk = __shfl_sync(0xffffffffu, ids, k & 31);
        if ((unsigned)blk >= (unsigned)a.num_blocks) {
            if (lane == 0)
                raise_flag(PKV_DEVFLAG_BLOCK_RANGE);
            blk = 0;
        }
        if (lane == 0) {
            const int s = k % S;
            const uint32_t bar = bar0 + 8u * s;
            const uint32_t dk = ring_s + (uint32_t)(s * kStageBytes);
            const uint32_t dv = dk + kTileBytes;
            mbar_arrive_expect_tx(bar, kStageBytes);
#pragma unroll
            for (int h = 0; h < Shape::kHalves; ++h) {
                tma_load_3d(dk + h * kHalfBytes, &tm_k, bar, h * 64, kvh, blk * BS, policy);
                tma_load_3d(dv + h * kHalfBytes, &tm_v, bar, h * 64, kvh, blk * BS, policy);
            }
        }
    };

    float m_run[2] = {kNegInf, kNegInf};   // running max (base-2 units) of columns 2c, 2c+1
    float l_run[2] = {0.f, 0.f};           // this lane's share of the running normaliser
    float acc_hi[KS][4];
    float acc_lo[KS][4];
#pragma unroll
    for (int dt = 0; dt < KS; ++dt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc_hi[dt][i] = 0.f;
            acc_lo[dt][i] = 0.f;
        }

    const int pre = nk < S ? nk : S;
    for (int k = 0; k < pre; ++k)
        issue(k);
    int issued = pre;
    int consumed = 0;

    for (int k = 0; k < nk; ++k) {
        const int s = k % S;
        const bool got = mbar_wait_bounded(bar0 + 8u * s, (uint32_t)((k / S) & 1), kWaitLimitNs);
        if (!__all_sync(0xffffffffu, got)) {
            if (lane == 0)
                raise_flag(PKV_DEVFLAG_WAIT_TIMEOUT);
            break;
        }
        consumed = k + 1;
        const uint32_t sk = ring_s + (uint32_t)(s * kStageBytes);
        const uint32_t sv = sk + kTileBytes;
        const int lb = blk0 + warp + k * NW;
        const int valid = min(BS, tok1 - lb * BS);   // >= 1

        if (valid < BS) {
            // Rows past the context end may hold anything (even NaN): zero
            // them in V so that 0-weight * row stays 0.  Whole 128-byte rows,
            // so the swizzle does not matter.
            uint8_t *vt = ring + (size_t)s * kStageBytes + kTileBytes;
            const int per_half = (BS - valid) * 8;
            for (int i = lane; i < Shape::kHalves * per_half; i += 32) {
                const int h = i / per_half;
                const int r = i - h * per_half;
                *reinterpret_cast<uint4 *>(vt + h * kHalfBytes + (valid + (r >> 3)) * 128 +
                                           (r & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
            // order these generic stores before any later TMA (async proxy) write
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        }

        attend_block<D, BS, BF16>(sk, sv, valid, qf, a.scale_log2, m_run, l_run, acc_hi, acc_lo,
                                  lane);

        __syncwarp();
        if (k + S < nk) {
            issue(k + S);
            issued = k + S + 1;
        }
    }

    // A wait gave up: let this warp's copies in flight land (bounded) before
    // the shared memory is reused.
    for (int k = consumed; k < issued; ++k)
        mbar_wait_bounded(bar0 + 8u * (k % S), (uint32_t)((k / S) & 1), kWaitLimitNs / 8);

#pragma unroll
    for (int j = 0; j < 2; ++j) {
        l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], 4);
        l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], 8);
        l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], 16);
    }

    // ---- merge the NW warps (log-sum-exp) through shared memory ----
    __syncthreads();   // all stages consumed: the ring becomes scratch
    float *so = reinterpret_cast<float *>(smem);   // [NW][8][D]
    float *sm = so + NW * 8 * D;                     // [NW][8]
    float *sl = sm + NW * 8;                         // [NW][8]
    {
        const int c = lane & 3;
        const int r = lane >> 2;
#pragma unroll
        for (int dt = 0; dt < KS; ++dt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int n = 2 * c + (i & 1);
                const int d = dt * 16 + r + (i >= 2 ? 8 : 0);
                so[(warp * 8 + n) * D + d] = acc_hi[dt][i] + acc_lo[dt][i];
            }
        if (r == 0) {
            sm[warp * 8 + 2 * c] = m_run[0];
            sm[warp * 8 + 2 * c + 1] = m_run[1];
            sl[warp * 8 + 2 * c] = l_run[0];
            sl[warp * 8 + 2 * c + 1] = l_run[1];
        }
    }
    __syncthreads();

    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
        const int g = idx / D;
        const int d = idx - g * D;
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            M = fmaxf(M, sm[w * 8 + g]);
        float den = 0.f, num = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float e = ex2(sm[w * 8 + g] - M);   // 0 for warps without blocks
            den += e * sl[w * 8 + g];
            num += e * so[(w * 8 + g) * D + d];
        }
        const float o = den > 0.f ? num / den : 0.f;
        const size_t row = (size_t)b * Hq + (size_t)kvh * G + g;
        if (!split) {
            a.out[row * D + d] = to_storage<BF16>(o);
        } else {
            const size_t pr = row * a.num_parts + part;
            a.ws_o[pr * D + d] = o;
            if (d == 0) {
                a.ws_m[pr] = M;
                a.ws_l[pr] = den;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Cascade decode, level 1: a shared prefix read once for a whole group
// ---------------------------------------------------------------------------
// Parallel samples of one prompt share the prompt's blocks ("23.1 vLLM：高吞吐
// 推理框架原理与部署", section 二.3).  Sequences group_start[g] ..
// group_start[g+1]-1 share the prefix_lens[g] tokens (a multiple of the block
// size) listed in prefix_tables[g].  Level 1 (prefix_tc_kernel, in
// pkv_prefill.cuh) runs one CTA per (prefix partition, kv head, chunk of
// 128 / G members) on the tensor cores, so each prefix block is read from HBM
// once per group instead of once per sequence, and writes per query row the
// partition's record (max, normaliser, normalised row); level 2 (the decode
// kernel over each sequence's own suffix, records only) and the cascade merge
// below complete the result, which equals the decode over the concatenated
// table.  When there are enough groups to fill the GPU, one kernel does it all
// instead (cascade_tc_kernel, pkv_prefill.cuh): a CTA per (kv head, chunk of
// 32/G members) reads the group's whole prefix once and then each member's
// own blocks, and writes the output rows; no records, no merge kernel.
struct CascadeArgs {
    const uint16_t *query;           // [B, Hq, D]
    const int32_t *prefix_tables;    // [num_groups, max_prefix_blocks]
    const int32_t *prefix_lens;      // [num_groups]
    const int32_t *group_start;      // [num_groups + 1]
    float *rec_m;                    // prefix records [B*Hq, num_parts]
    float *rec_l;
    float *rec_o;                    // [B*Hq, num_parts, D]
    int batch;
    int max_prefix_blocks;
    int num_groups;
    int max_group_size;
    int num_heads;
    int num_kv_heads;
    int group;                       // Hq / Hkv
    int num_blocks;
    int part_tokens;                 // prefix partition length (multiple of BS)
    int num_parts;                   // prefix partitions
    int chunks;                      // member chunks per group
    float scale_log2;
    // one-pass cascade (prefix and every member's own blocks in one CTA)
    const int32_t *suffix_tables;    // [batch, max_suffix_blocks]
    const int32_t *suffix_lens;      // [batch]
    uint16_t *out;                   // [B, Hq, D]
    int max_suffix_blocks;
};

// Cascade merge: row (b, h) = its group's prefix records (partitions of the
// prefix) and its own suffix records (partitions of the suffix), folded by
// log-sum-exp.  One warp per row, lane = D/32 consecutive columns.  The
// warp finds the row's group with a 32-way search of group_start (one or two
// load rounds), spreads the records' (m, l) over its lanes to take the
// maximum and the weights, then loads every record's O slice independently.
template <bool BF16, int D, int NT>
__global__ void __launch_bounds__(NT)
lse_merge_cascade_kernel(const CascadeArgs c, const float *__restrict__ sm, const float *__restrict__ sl,
                         const float *__restrict__ so, const int32_t *__restrict__ suffix_lens,
                         int suffix_parts, int suffix_part_tokens, int suffix_span,
                         uint16_t *__restrict__ out)
{
    constexpr int VPT = D / 32;
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const size_t row = (size_t)blockIdx.x * (NT / 32) + threadIdx.x / 32;
    if (row >= (size_t)c.batch * c.num_heads)
        return;                                  // whole warp
    const int b = (int)(row / c.num_heads);

    // group of sequence b: the last g with group_start[g] <= b (starts ascend)
    int lo = 0, n = c.num_groups;                // candidates lo .. lo + n - 1
    while (n > 32) {
        const int step = (n + 31) / 32;
        const int idx = lo + lane * step;
        const unsigned le = __ballot_sync(0xffffffffu, idx < lo + n && __ldg(c.group_start + idx) <= b);
        if (le == 0u) {
            n = 0;                               // every candidate starts after b
            break;
        }
        const int nlo = lo + (31 - __clz(le)) * step;
        n = min(step, lo + n - nlo);
        lo = nlo;
    }
    int g = lo - 1;
    if (n > 0) {
        const unsigned le =
            __ballot_sync(0xffffffffu, lane < n && __ldg(c.group_start + lo + lane) <= b);
        if (le != 0u)
            g = lo + 31 - __clz(le);
    }
    int np_p = 0;
    if (g >= 0 && b < __ldg(c.group_start + g + 1)) {
        int Lp = __ldg(c.prefix_lens + g);
        Lp = Lp < 0 ? 0 : Lp;
        np_p = min(c.num_parts, (Lp + c.part_tokens - 1) / c.part_tokens);
    }
    int Ls = __ldg(suffix_lens + b);
    Ls = Ls < 0 ? 0 : (Ls > suffix_span ? suffix_span : Ls);
    const int np_s = (Ls + suffix_part_tokens - 1) / suffix_part_tokens;
    const int nrec = np_p + np_s;               // record k: prefix k, then suffix k - np_p

    // record k's (m, l) and O slice
    auto rec_ml = [&](int k, float &m, float &l) {
        const size_t r = k < np_p ? row * c.num_parts + k : row * suffix_parts + (k - np_p);
        m = __ldg((k < np_p ? c.rec_m : sm) + r);
        l = __ldg((k < np_p ? c.rec_l : sl) + r);
    };
    auto rec_o = [&](int k) {
        return k < np_p ? c.rec_o + (row * c.num_parts + k) * D : so + (row * suffix_parts + (k - np_p)) * D;
    };

    // the maximum over records that hold keys (l > 0)
    float M = kNegInf;
    for (int k0 = 0; k0 < nrec; k0 += 32) {
        float m = kNegInf, l = 0.f;
        if (k0 + lane < nrec)
            rec_ml(k0 + lane, m, l);
        if (l > 0.f)
            M = fmaxf(M, m);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    // weights w_k = 2^(m_k - M) l_k, spread over the lanes; den = sum w_k
    float den = 0.f, acc[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i)
        acc[i] = 0.f;
    for (int k0 = 0; k0 < nrec; k0 += 32) {
        float m = kNegInf, l = 0.f;
        if (k0 + lane < nrec)
            rec_ml(k0 + lane, m, l);
        const float w = l > 0.f ? ex2(m - M) * l : 0.f;
        den += w;
        const int nk = min(32, nrec - k0);
        for (int k = 0; k < nk; ++k) {
            const float wk = __shfl_sync(0xffffffffu, w, k);
            if (wk > 0.f) {                      // warp-uniform
                float v[VPT];
                load_slice<D>(rec_o(k0 + k) + lane * VPT, v);
#pragma unroll
                for (int i = 0; i < VPT; ++i)
                    acc[i] += wk * v[i];
            }
        }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1)
        den += __shfl_xor_sync(0xffffffffu, den, off);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint16_t *o = out + row * D + lane * VPT;
    if constexpr (VPT == 4) {
        *reinterpret_cast<uint2 *>(o) = make_uint2(pack2<BF16>(acc[0] * inv, acc[1] * inv),
                                                   pack2<BF16>(acc[2] * inv, acc[3] * inv));
    } else {
        *reinterpret_cast<uint32_t *>(o) = pack2<BF16>(acc[0] * inv, acc[1] * inv);
    }
}

// ---------------------------------------------------------------------------
// Whole-block copies: copy-on-write and swap
// ---------------------------------------------------------------------------
// A shared block is copied before a sequence writes into it ("23.1 vLLM：高吞吐
// 推理框架原理与部署", section 二.3), and blocks move between the device pool
// and host memory when the scheduler swaps a sequence out and back in ("大模型
// 推理框架 vLLM 源码解析 一", section 三).  Pair i copies block mapping[2i] of
// the source caches to block mapping[2i+1] of the destination caches, K and
// V, as 16-byte vectors; either side may be pinned host memory (reached
// through unified addressing).  Pairs naming a block outside its pool are
// skipped and set PKV_DEVFLAG_BLOCK_RANGE.
// One CTA per (pair, K or V): 256 threads move the block's 16-byte vectors,
// kCopyUnroll loads in flight per thread before their stores.
constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 8;
__global__ void __launch_bounds__(kCopyThreads)
copy_blocks_kernel(const uint4 *__restrict__ src_k, const uint4 *__restrict__ src_v,
                   uint4 *__restrict__ dst_k, uint4 *__restrict__ dst_v,
                   const int32_t *__restrict__ mapping, int num_pairs, int64_t src_blocks,
                   int64_t dst_blocks, int64_t vec_per_block)
{
    // Launched with programmatic dependent launch: wait for the previous
    // kernel on the stream before touching memory, then let the next start.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int64_t pair = blockIdx.x >> 1;
    const bool is_v = blockIdx.x & 1;
    if (pair >= num_pairs)
        return;
    const int64_t s = __ldg(mapping + 2 * pair);
    const int64_t d = __ldg(mapping + 2 * pair + 1);
    if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) {
        if (threadIdx.x == 0 && !is_v)
            raise_flag(PKV_DEVFLAG_BLOCK_RANGE);
        return;                                  // the pair is skipped
    }
    const uint4 *src = (is_v ? src_v : src_k) + s * vec_per_block;
    uint4 *dst = (is_v ? dst_v : dst_k) + d * vec_per_block;
    for (int64_t v0 = threadIdx.x; v0 < vec_per_block; v0 += kCopyThreads * kCopyUnroll) {
        uint4 r[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t v = v0 + u * kCopyThreads;
            if (v < vec_per_block)
                r[u] = src[v];
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t v = v0 + u * kCopyThreads;
            if (v < vec_per_block)
                dst[v] = r[u];
        }
    }
}

// ---------------------------------------------------------------------------
// Self-test of the bounded pipeline wait
// ---------------------------------------------------------------------------
// One warp waits, through the same bounded wait the decode kernel uses, on an
// mbarrier phase that nothing completes; after limit_ns it must give up, set
// PKV_DEVFLAG_WAIT_TIMEOUT and return, leaving the context usable.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0)
        mbar_init(smem_addr(&bar), 1);
    fence_mbar_init();
    __syncwarp();
    const bool got = mbar_wait_bounded(smem_addr(&bar), 0u, limit_ns);
    if (!__all_sync(0xffffffffu, got) && threadIdx.x == 0)
        raise_flag(PKV_DEVFLAG_WAIT_TIMEOUT);
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of split partitions
// ---------------------------------------------------------------------------
// out = sum_p w_p o_p / sum_p w_p, w_p = 2^(m_p - M) l_p, M = max_p m_p, over
// the partitions of a (sequence, query head) row that hold tokens, with an
// online log-sum-exp.  Two launch shapes: lse_merge_kernel for plans with few
// partitions (several rows per CTA, a thread per column), lse_merge_wide_kernel
// for many (a CTA per row, its warps folding interleaved partitions, then
// combined).  Launched with programmatic dependent launch: they wait for the
// decode first.

template <bool BF16, int D, int NT>
__global__ void __launch_bounds__(NT)
lse_merge_kernel(const float *__restrict__ ws_m, const float *__restrict__ ws_l,
                 const float *__restrict__ ws_o, const int32_t *__restrict__ context_lens,
                 int num_heads, int num_rows, int num_parts, int part_tokens, int span,
                 uint16_t *__restrict__ out)
{
    // few partitions: NT / D rows per CTA, thread = one column of one row
    constexpr int NG = NT / D;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int d = threadIdx.x % D;
    const size_t row = (size_t)blockIdx.x * NG + threadIdx.x / D;
    if (row >= (size_t)num_rows)
        return;
    const int b = (int)(row / num_heads);
    int L = __ldg(context_lens + b);
    L = L < 0 ? 0 : (L > span ? span : L);
    const int np = (L + part_tokens - 1) / part_tokens;
    const float *m = ws_m + row * num_parts;
    const float *l = ws_l + row * num_parts;
    const float *o = ws_o + row * num_parts * D + d;
    float M = kNegInf, den = 0.f, num = 0.f;
#pragma unroll 4
    for (int p = 0; p < np; ++p) {
        const float mp = __ldg(m + p);
        const float lp = __ldg(l + p);
        const float op = __ldg(o + (size_t)p * D);
        if (mp > M) {
            const float sc = ex2(M - mp);   // 0 while M is -inf
            den *= sc;
            num *= sc;
            M = mp;
        }
        const float w = ex2(mp - M) * lp;
        den += w;
        num += w * op;
    }
    out[row * D + d] = to_storage<BF16>(den > 0.f ? num / den : 0.f);
}

// Many partitions: one CTA per row; NG groups of 32 threads, group g folds the
// partitions p = g, g + NG, ... (a thread holds D/32 consecutive columns, so a
// group's loads of one partition are independent of its other partitions'),
// then group 0 folds the NG partial results.
template <bool BF16, int D, int NT>
__global__ void __launch_bounds__(NT)
lse_merge_wide_kernel(const float *__restrict__ ws_m, const float *__restrict__ ws_l,
                      const float *__restrict__ ws_o, const int32_t *__restrict__ context_lens,
                      int num_heads, int num_rows, int num_parts, int part_tokens, int span,
                      uint16_t *__restrict__ out)
{
    constexpr int VPT = D / 32;
    constexpr int NG = NT / 32;
    __shared__ float s_M[NG], s_den[NG];
    __shared__ __align__(16) float s_num[NG][D];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int grp = threadIdx.x >> 5;
    const size_t row = blockIdx.x;
    if (row >= (size_t)num_rows)
        return;                                  // whole CTA
    const int b = (int)(row / num_heads);
    int L = __ldg(context_lens + b);
    L = L < 0 ? 0 : (L > span ? span : L);
    const int np = (L + part_tokens - 1) / part_tokens;
    const float *m = ws_m + row * num_parts;
    const float *l = ws_l + row * num_parts;
    const float *o = ws_o + row * num_parts * D + lane * VPT;
    float M = kNegInf, den = 0.f, num[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i)
        num[i] = 0.f;
#pragma unroll 4
    for (int p = grp; p < np; p += NG) {
        const float mp = __ldg(m + p);
        const float lp = __ldg(l + p);
        float v[VPT];
        load_slice<D>(o + (size_t)p * D, v);
        if (mp > M) {
            const float sc = ex2(M - mp);       // 0 while M is -inf
            den *= sc;
#pragma unroll
            for (int i = 0; i < VPT; ++i)
                num[i] *= sc;
            M = mp;
        }
        const float w = ex2(mp - M) * lp;
        den += w;
#pragma unroll
        for (int i = 0; i < VPT; ++i)
            num[i] += w * v[i];
    }
    if (lane == 0) {
        s_M[grp] = M;
        s_den[grp] = den;
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i)
        s_num[grp][lane * VPT + i] = num[i];
    __syncthreads();
    if (grp == 0) {
        float Mt = kNegInf;
#pragma unroll
        for (int q = 0; q < NG; ++q)
            Mt = fmaxf(Mt, s_M[q]);
        float dt = 0.f, nt[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i)
            nt[i] = 0.f;
#pragma unroll
        for (int q = 0; q < NG; ++q) {
            // 0 for groups that held no partition (also when none did: no NaN)
            const float e = s_M[q] == kNegInf ? 0.f : ex2(s_M[q] - Mt);
            dt += e * s_den[q];
#pragma unroll
            for (int i = 0; i < VPT; ++i)
                nt[i] += e * s_num[q][lane * VPT + i];
        }
        const float inv = dt > 0.f ? 1.f / dt : 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i)
            nt[i] = dt > 0.f ? nt[i] * inv : 0.f;
        uint16_t *op = out + row * D + lane * VPT;
        if constexpr (VPT == 4) {
            *reinterpret_cast<uint2 *>(op) =
                make_uint2(pack2<BF16>(nt[0], nt[1]), pack2<BF16>(nt[2], nt[3]));
        } else {
            *reinterpret_cast<uint32_t *>(op) = pack2<BF16>(nt[0], nt[1]);
        }
    }
}

}  // namespace pkv
