// pkv_prefill.cuh -- many query rows over the paged KV cache on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory):
// chunked prefill (prefill_tc_kernel), the shared-prefix pass of cascade
// decode (prefix_tc_kernel, which differs only in its work map, no causal
// mask, and its output: partition records for the cascade merge), and the
// one-pass cascade decode (cascade_tc_kernel: a group's prefix and then each
// member's own blocks, output rows).
//
// Sequence b brings C_b = query_start[b+1] - query_start[b] new tokens, the
// last C_b of its L_b = context_lens[b] cached tokens (their K/V were written
// through slot_mapping beforehand, "大模型推理框架 vLLM 源码解析 一",
// section 三); query token i sits at position L_b - C_b + i and attends
// causally over tokens 0 .. L_b - C_b + i of its paged cache.
//
// A prefill CTA takes 1-4 consecutive row tiles of one (kv head, sequence);
// the prefix pass one CTA per (prefix partition, kv head, chunk of 128/G group
// members).  A row is a (query token or group member, head of the kv head's
// GQA group) pair, 128 rows per tile (the M of every MMA).
// Keys are taken 64 at a time (a "key tile": 64 / block_size cache blocks
// located through the block table, exactly as the decode kernels do):
//
//   S_j  = Q K_j^T        tcgen05.mma, Q and K_j in shared memory, S in TMEM
//   P_j  = 2^(S_j*scale*log2e - m)    one row per softmax thread, bf16/f16,
//                                      stored over S_j in TMEM
//   O   += P_j V_j         tcgen05.mma, P from TMEM, V from shared memory
//                          (read MN-major), O in TMEM
//
// The running row maximum m is only moved when a tile's maximum exceeds it
// by more than 2^8 (P then stays <= 256); O and the row sum are rescaled by
// the softmax warps at that point, so the result equals the one-pass softmax
// up to rounding.  S (and P over it) is double-buffered in TMEM: the
// tensor core computes S_{j+1} while the softmax warps work on tile j.
//
// Ordering (tcgen05 keeps back-to-back MMAs in issue order only when they
// share the accumulator and the shape; S and O differ in both):
//   * S_{j+1} overwrites the buffer that holds P_{j-1}, the A operand of
//     P_{j-1} V_{j-1}: the MMA thread issues S_{j+1} only after that MMA has
//     completed (O_DONE of tile j-1).
//   * The softmax warps store P_j only after P_{j-1} V_{j-1} has completed:
//     O is then stable for a rescale, and O_DONE (one barrier, one phase per
//     tile) is never more than one phase ahead of any wait on it.  Without
//     this wait the softmax could finish its last tile while two P V phases
//     were still open, and the epilogue's parity wait for the last phase then
//     matched the phase two back and read O early (wrong rows in 10-40% of
//     runs of a 7-token chunk over 520 keys).
//   * While P_j is stored, the only MMA that can be running is S_{j+1}, which
//     writes the other buffer.
// Warp roles: 0-3 softmax + epilogue (warp w owns TMEM lanes 32w..32w+31),
// 4 loads the K ring (3 stages), 5 allocates TMEM and issues every MMA, 6
// loads the V ring (2 stages), 7 loads Q.  Whole blocks come through a 3-D
// view of the cache; a sequence's partly filled last block comes through a
// 4-D view {head_dim, kv heads, block rows, blocks} at a negative row offset,
// so that the cells past its end are never read (the rows before it read as
// zero) and a masked key always meets a finite V row.  A prefill CTA takes a few
// consecutive row tiles of one (sequence, kv head) in turn; the other modes
// run one work tile per CTA.  Every wait is bounded; on a time-out the CTA
// records PKV_DEVFLAG_WAIT_TIMEOUT, lets in-flight copies and MMAs finish and
// frees its TMEM.
#pragma once

#include "pkv_kernels.cuh"

namespace pkv {

struct PrefillArgs {
    const uint16_t *query;           // [T, Hq, D], T = query_start[batch]
    const int32_t *query_start;      // [batch + 1]
    const int32_t *block_tables;     // [batch, max_blocks]
    const int32_t *context_lens;     // [batch]
    uint16_t *out;                   // [T, Hq, D]
    int batch;
    int num_tokens;                  // T: rows of query / out
    int max_query_len;               // chunks longer than this are not covered by the grid
    int max_blocks;
    int num_heads;
    int num_kv_heads;
    int group;
    int num_blocks;
    int tiles_per_cta;               // consecutive row tiles (of 128/G query tokens) a CTA takes
    float scale_log2;
};

constexpr int kPfRows = 128;             // query rows per CTA (MMA M)
constexpr int kPfKeys = 64;              // keys per tile (N of Q K^T, K of P V)
constexpr int kPfThreads = 256;          // 8 warps
constexpr uint32_t kPfTmemCols = 256;    // S/P: 2 x 64 columns, O: D columns at 128
constexpr int kPfKStages = 3;
constexpr int kPfVStages = 2;
constexpr int kCasRows = 32;             // one-pass cascade: query rows per CTA (held 4 times)

template <int D>
struct PfShape {
    static constexpr int kHalves = D / 64;                  // 128-byte column halves
    static constexpr int kQHalf = kPfRows * 128;            // one half of Q: 128 rows x 128 B
    static constexpr int kKVHalf = kPfKeys * 128;           // one half of a K or V tile
    static constexpr int kQBytes = kHalves * kQHalf;
    static constexpr int kKVBytes = kHalves * kKVHalf;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kQBytes;
    static constexpr int kVOff = kKOff + kPfKStages * kKVBytes;
    static constexpr int kDataBytes = kVOff + kPfVStages * kKVBytes;
    // + 1024 so that the data can start on a 1024-byte boundary; the barriers
    // sit in whichever end of that slack has room
    // two CTAs per SM, never three: a third would wait for TMEM (2 x 256
    // columns fill the SM's 512) instead of working
    static constexpr int kSmemBytes = (kDataBytes + 1024 > 80 * 1024) ? kDataBytes + 1024 : 80 * 1024;
};

// mbarrier slots
enum PfBar {
    kBarQFull = 0,
    kBarKFull = 1,     // kPfKStages
    kBarKEmpty = 4,    // kPfKStages
    kBarVFull = 7,     // kPfVStages
    kBarVEmpty = 9,    // kPfVStages
    kBarSFull = 11,    // 2, one per S/P buffer
    kBarPFull = 13,    // 2, one per S/P buffer
    kBarODone = 15,
    kBarDrain = 16,
    kBarTmemSlot = 17,   // not a barrier: the TMEM base address
    kBarEpi0 = 18,       // one-pass cascade: the softmax warps' partial results
    kBarEpi1 = 19,
    kBarQEmpty = 20,     // the Q buffer is free: the work tile's last S has completed
    kNumPfBars = 22
};
// A barrier per S/P buffer completes once per two tiles, and buffer j & 1 is
// refilled (S_{j+2}) only after P_j V_j has completed: no barrier can run two
// phases ahead of its waiter.

// Transpose a 4 x 4 array of 16-byte chunks over the four lanes of a quad
// (q = lane & 3): lane h enters with chunk v of its row in c[v] and leaves
// with chunk q of quad row h in c[h].  Two exchange stages, with the partner
// two lanes away and then one lane away; each moves half of the chunks.
__device__ __forceinline__ uint4 shfl_xor4(const uint4 &x, int m)
{
    return make_uint4(__shfl_xor_sync(0xffffffffu, x.x, m), __shfl_xor_sync(0xffffffffu, x.y, m),
                      __shfl_xor_sync(0xffffffffu, x.z, m), __shfl_xor_sync(0xffffffffu, x.w, m));
}
__device__ __forceinline__ void quad_transpose(uint4 (&c)[4], int q)
{
    const bool hi = (q & 2) != 0, lo = (q & 1) != 0;
    uint4 r0 = shfl_xor4(hi ? c[0] : c[2], 2), r1 = shfl_xor4(hi ? c[1] : c[3], 2);
    if (hi) {
        c[0] = r0;
        c[1] = r1;
    } else {
        c[2] = r0;
        c[3] = r1;
    }
    r0 = shfl_xor4(lo ? c[0] : c[1], 1);
    r1 = shfl_xor4(lo ? c[2] : c[3], 1);
    if (lo) {
        c[0] = r0;
        c[2] = r1;
    } else {
        c[1] = r0;
        c[3] = r1;
    }
}

// Bits lo .. hi-1 of a 64-column mask (clamped to 0 .. 64; empty when hi <= lo).
__device__ __forceinline__ uint64_t col_range(int lo, int hi)
{
    lo = max(lo, 0);
    hi = min(hi, 64);
    if (hi <= lo)
        return 0ull;
    const uint64_t upto = hi >= 64 ? ~0ull : (1ull << hi) - 1ull;
    return upto & ~((1ull << lo) - 1ull);
}

// What a CTA of the shared body computes.
enum TcMode : int {
    // causal rows of one sequence's chunk; output rows
    kTcPrefill = 0,
    // the query rows of a group's members over one partition of their shared
    // prefix; partition records for the cascade merge
    kTcPrefix = 1,
    // the query rows of a group's members over the group's whole prefix, then
    // each member's rows over that member's own blocks (the other rows see
    // none of them); output rows.  Extra CTAs at the end of the grid take the
    // sequences outside every group (own blocks only).  A CTA takes 32 query
    // rows (32/G members) and holds them in all four softmax warps' lanes (Q
    // is loaded four times): warp w weighs key columns 16w .. 16w+15 of every
    // tile with its own running maximum and sum, so the four share the
    // exponentials of a tile; their partial rows are merged by log-sum-exp in
    // the epilogue.  The tensor core does the padding (M = 128 for 32 rows);
    // the softmax, which bounds a tile's time, does none.
    kTcCascade = 2,
};

// One-pass cascade: the keys of a member's own blocks are taken in the order
// (last block, block 0, block 1, ...), and the last block, when partly
// filled, is loaded shifted so that its valid rows end the block's 16 or 32
// rows (the rows before them lie outside the block and read as zero).  The
// valid keys of every key tile are then one contiguous range of its columns.
// Attention does not depend on the order of the keys.

// The body shared by the three modes.
template <int D, int BS, bool BF16, int MODE>
__device__ __forceinline__ void tc_attend(const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                          const CUtensorMap *tm_v, const CUtensorMap *tm_k4,
                                          const CUtensorMap *tm_v4, const PrefillArgs &a,
                                          const CascadeArgs &c)
{
    using Sh = PfShape<D>;
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static_assert(kPfKeys % BS == 0, "whole blocks per key tile");
    static_assert(kPfKeys + D <= (int)kPfTmemCols, "TMEM columns");
    constexpr int KS = D / 16;               // k-steps of Q K^T
    constexpr int KV_STEPS = kPfKeys / 16;   // k-steps of P V
    constexpr int BPT = kPfKeys / BS;        // cache blocks per key tile
    static_assert(32 % BPT == 0, "a key tile's block ids lie in one 32-id window");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t data_s = (raw_s + 1023u) & ~1023u;
    uint8_t *data = smem_raw + (data_s - raw_s);
    const uint32_t bars_s = data_s - raw_s >= kNumPfBars * 8 ? raw_s : data_s + Sh::kDataBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + (bars_s - raw_s));
    auto bar = [&](int i) { return bars_s + 8u * (uint32_t)i; };

    const int kvh = blockIdx.y;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr bool kCas = MODE != kTcPrefill;   // a cascade mode: c, not a
    const int G = kCas ? c.group : a.group;
    // query tokens (cascade: group members) per CTA; the one-pass cascade takes
    // 32 query rows and holds them four times, once in each softmax warp's lanes
    const int TT = (MODE == kTcCascade ? kCasRows : kPfRows) / G;
    const int R = TT * G;         // rows in use (128, or 32 in the one pass, when G divides them)
    const int num_heads = kCas ? c.num_heads : a.num_heads;
    const int num_blocks = kCas ? c.num_blocks : a.num_blocks;
    const float scale_log2 = kCas ? c.scale_log2 : a.scale_log2;

    if (threadIdx.x == 0) {
        mbar_init(bar(kBarQFull), 1);
#pragma unroll
        for (int s = 0; s < kPfKStages; ++s) {
            mbar_init(bar(kBarKFull + s), 1);
            mbar_init(bar(kBarKEmpty + s), 1);
        }
#pragma unroll
        for (int s = 0; s < kPfVStages; ++s) {
            mbar_init(bar(kBarVFull + s), 1);
            mbar_init(bar(kBarVEmpty + s), 1);
        }
        mbar_init(bar(kBarSFull + 0), 1);
        mbar_init(bar(kBarSFull + 1), 1);
        mbar_init(bar(kBarPFull + 0), 4);       // one arrive per softmax warp
        mbar_init(bar(kBarPFull + 1), 4);
        mbar_init(bar(kBarODone), 1);
        mbar_init(bar(kBarQEmpty), 1);
        mbar_init(bar(kBarDrain), 1);
        mbar_init(bar(kBarEpi0), 4);            // one arrive per softmax warp
        mbar_init(bar(kBarEpi1), 4);
        prefetch_tensormap(tm_q);
        prefetch_tensormap(tm_k);
        prefetch_tensormap(tm_v);
        prefetch_tensormap(tm_k4);
        prefetch_tensormap(tm_v4);
    }
    fence_mbar_init();
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    // The CTA's work: query rows row0 .. row0+127 of a row space of `rows`
    // real rows ((token or member) x head of the group), whose first query
    // row is query row q_tok0; keys 0 .. p_max of a key range that starts at
    // block trow[0]; row r sees keys up to pos0 + r / G (prefill, causal) or
    // all of them (prefix).
    int rows, row0, q_tok0, p_max, pos0, rec_part = 0;
    const int32_t *trow;
    // one-pass cascade: members first .. first + n_mem - 1 (the CTA's query
    // rows, G per member); prefix of Lp tokens; lane l of every warp holds the
    // key counts of members l, l + 32, l + 64, l + 96 (0 for a member another
    // CTA covers); sequences outside every group are those before gs0 or
    // from gsN on
    int n_mem = 0, Lp = 0, gs0 = 0, gsN = 0, nt_cas = 0;
    bool grouped = false;
    int mlen[4] = {0, 0, 0, 0};
    if constexpr (MODE == kTcPrefill) {
        rows = row0 = q_tok0 = p_max = pos0 = 0;   // per work tile: next_work below
        trow = a.block_tables;
    } else if constexpr (MODE == kTcPrefix) {
        const int pp = blockIdx.x;
        const int g = blockIdx.z / c.chunks;
        const int mc = blockIdx.z - g * c.chunks;
        int first = __ldg(c.group_start + g);
        int count = __ldg(c.group_start + g + 1) - first;
        if (first < 0 || count < 0 || first + count > c.batch || count > c.max_group_size) {
            if (threadIdx.x == 0 && pp == 0 && kvh == 0 && mc == 0)
                raise_flag(PKV_DEVFLAG_CONTEXT_RANGE);
            first = first < 0 ? 0 : (first > c.batch ? c.batch : first);
            count = count < 0 ? 0 : count;
            count = min(count, min(c.max_group_size, c.batch - first));
        }
        int Lp = __ldg(c.prefix_lens + g);
        const int span = c.max_prefix_blocks * BS;
        if (Lp < 0 || Lp > span || Lp % BS != 0) {
            if (threadIdx.x == 0 && pp == 0 && kvh == 0 && mc == 0)
                raise_flag(PKV_DEVFLAG_CONTEXT_RANGE);
            Lp = Lp < 0 ? 0 : (Lp > span ? span : Lp - Lp % BS);
        }
        const int tok0 = pp * c.part_tokens;
        const int tok1 = min(Lp, tok0 + c.part_tokens);
        rows = count * G;
        row0 = mc * R;
        if (row0 >= rows || tok1 <= tok0)
            return;                                 // nothing here (the merge skips it)
        q_tok0 = first + mc * TT;
        p_max = tok1 - tok0 - 1;
        pos0 = p_max;
        trow = c.prefix_tables + (size_t)g * c.max_prefix_blocks + tok0 / BS;
        rec_part = pp;
    } else {
        const int gz = c.num_groups * c.chunks;
        int first;
        const int z = blockIdx.z;
        if (c.num_groups > 0) {
            gs0 = min(max(__ldg(c.group_start), 0), c.batch);
            gsN = min(max(__ldg(c.group_start + c.num_groups), gs0), c.batch);
        }
        if (z < gz) {
            const int g = z / c.chunks;
            const int mc = z - g * c.chunks;
            first = __ldg(c.group_start + g);
            int count = __ldg(c.group_start + g + 1) - first;
            if (first < 0 || count < 0 || first + count > c.batch || count > c.max_group_size) {
                if (threadIdx.x == 0 && kvh == 0 && mc == 0)
                    raise_flag(PKV_DEVFLAG_CONTEXT_RANGE);
                first = first < 0 ? 0 : (first > c.batch ? c.batch : first);
                count = count < 0 ? 0 : count;
                count = min(count, min(c.max_group_size, c.batch - first));
            }
            Lp = __ldg(c.prefix_lens + g);
            const int span = c.max_prefix_blocks * BS;
            if (Lp < 0 || Lp > span || Lp % BS != 0) {
                if (threadIdx.x == 0 && kvh == 0 && mc == 0)
                    raise_flag(PKV_DEVFLAG_CONTEXT_RANGE);
                Lp = Lp < 0 ? 0 : (Lp > span ? span : Lp - Lp % BS);
            }
            first += mc * TT;
            n_mem = min(TT, count - mc * TT);
            trow = c.prefix_tables + (size_t)g * c.max_prefix_blocks;
            grouped = true;
        } else {
            first = (z - gz) * TT;
            n_mem = min(TT, c.batch - first);
            trow = c.prefix_tables;                 // not read: Lp = 0
            if (n_mem > 0 && first >= gs0 && first + n_mem <= gsN)
                n_mem = 0;                          // every sequence here is in a group
        }
        if (n_mem <= 0)
            return;                                 // whole CTA, before TMEM is touched
        const int sspan = c.max_suffix_blocks * BS;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = lane + 32 * i;
            if (m < n_mem) {
                const int b = first + m;
                if (grouped || b < gs0 || b >= gsN) {
                    int Ls = __ldg(c.suffix_lens + b);
                    if (Ls < 0 || Ls > sspan) {
                        raise_flag(PKV_DEVFLAG_CONTEXT_RANGE);
                        Ls = Ls < 0 ? 0 : sspan;
                    }
                    mlen[i] = Ls;
                }
            }
        }
        int tiles = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            tiles += (mlen[i] + kPfKeys - 1) / kPfKeys;
        nt_cas = (Lp + kPfKeys - 1) / kPfKeys + __reduce_add_sync(0xffffffffu, tiles);
        rows = n_mem * G;
        row0 = 0;
        q_tok0 = first;
        pos0 = p_max = 0;                           // unused: the walk gives each tile's keys
        if (nt_cas == 0) {
            // no keys for any row: zero output rows (the rows this CTA owns)
            for (int idx = threadIdx.x; idx < rows * D; idx += kPfThreads) {
                const int r = idx / D;
                const int b = first + r / G;
                if (grouped || b < gs0 || b >= gsN)
                    c.out[((size_t)b * num_heads + (size_t)kvh * G + r % G) * D + idx % D] = 0;
            }
            return;
        }
    }
    // key count of member m (warp-uniform m), from the lanes' registers
    auto member_len = [&](int m) -> int {
        const int v = m < 32 ? mlen[0] : (m < 64 ? mlen[1] : (m < 96 ? mlen[2] : mlen[3]));
        return __shfl_sync(0xffffffffu, v, m & 31);
    };
    // the next member after m with keys (n_mem if none)
    auto next_member = [&](int m) -> int {
        for (++m; m < n_mem; ++m)
            if (member_len(m) > 0)
                break;
        return m;
    };
    // one-pass cascade: the key tiles in order -- segment m = -1 is the
    // prefix, m >= 0 member m's own blocks; tile k of the segment, whose
    // keys number len
    struct Walk {
        int m, k, len;
    };
    auto walk_start = [&]() -> Walk {
        Walk w{-1, 0, Lp};
        if (w.len == 0) {
            w.m = next_member(-1);
            w.len = w.m < n_mem ? member_len(w.m) : 0;
        }
        return w;
    };
    auto walk_next = [&](Walk &w) -> bool {         // true: a new segment starts
        if (++w.k * kPfKeys < w.len)
            return false;
        w.m = next_member(w.m);
        w.len = w.m < n_mem ? member_len(w.m) : 0;
        w.k = 0;
        return true;
    };
    const int nt = MODE == kTcCascade ? nt_cas : p_max / kPfKeys + 1;   // key tiles
    const int nblk = p_max / BS + 1;                // cache blocks read (other modes)

    // Work tiles.  A prefill CTA takes tiles_per_cta consecutive row tiles of
    // one (sequence, kv head), the last (longest: most keys) first.  Its
    // tensor memory, rings and barrier phases carry over from tile to tile,
    // and the next tile's Q and first keys load while the current one
    // finishes; the CTAs of one (sequence, kv head) run side by side, so their
    // common keys come from L2.  The other modes run the one tile set up above.
    struct Wk {
        int rows, row0, q_tok0, p_max, pos0, kvh, nt, nblk;
        int tail;    // valid rows of block nblk-1 when it is the sequence's partly filled last block, else 0
        const int32_t *trow;
    };
    // prefill: the sequence's chunk, read once per CTA
    int pf_rt = 0, pf_q0 = 0, pf_C = 0, pf_L = 0;
    if constexpr (MODE == kTcPrefill) {
        const int b = blockIdx.z;
        pf_q0 = __ldg(a.query_start + b);
        pf_C = __ldg(a.query_start + b + 1) - pf_q0;
        pf_L = __ldg(a.context_lens + b);
        const int span = a.max_blocks * BS;
        if (pf_q0 < 0 || pf_C < 0 || pf_q0 + pf_C > a.num_tokens || pf_C > a.max_query_len || pf_L < 0 ||
            pf_L > span || pf_C > pf_L) {
            if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0)
                raise_flag(PKV_DEVFLAG_CONTEXT_RANGE);
            pf_L = pf_L < 0 ? 0 : (pf_L > span ? span : pf_L);
            if (pf_q0 < 0 || pf_C < 0 || pf_q0 + pf_C > a.num_tokens)
                pf_C = 0;                           // rows outside query/out: skip the sequence
            pf_C = min(pf_C, min(pf_L, a.max_query_len));
        }
        // the CTA's row tiles that hold query tokens, last first
        const int rt_lo = blockIdx.x * a.tiles_per_cta;
        pf_rt = min((pf_C + TT - 1) / TT, rt_lo + a.tiles_per_cta) - 1;
        if (pf_rt < rt_lo)
            return;                                 // the chunk ends before this CTA's tiles
    }
    bool single_done = false;
    auto next_work = [&](Wk &wk) -> bool {
        if constexpr (MODE == kTcPrefill) {
            if (pf_rt < (int)blockIdx.x * a.tiles_per_cta)
                return false;
            const int rt = pf_rt--;
            const int i0 = rt * TT;                 // first query token of the tile
            wk.rows = pf_C * G;
            wk.row0 = rt * R;
            wk.q_tok0 = pf_q0 + i0;
            wk.pos0 = pf_L - pf_C + i0;             // the first row's last key
            wk.p_max = pf_L - pf_C + min(pf_C, i0 + TT) - 1;   // last key any row of the tile sees
            wk.kvh = blockIdx.y;
            wk.nt = wk.p_max / kPfKeys + 1;
            wk.nblk = wk.p_max / BS + 1;
            wk.tail = (pf_L % BS != 0 && (pf_L - 1) / BS == wk.nblk - 1) ? pf_L % BS : 0;
            wk.trow = a.block_tables + (size_t)blockIdx.z * a.max_blocks;
            return true;
        } else {
            if (single_done)
                return false;
            single_done = true;
            // prefix partitions are whole blocks
            wk = Wk{rows, row0, q_tok0, p_max, pos0, kvh, nt, nblk, 0, trow};
            return true;
        }
    };

    // Keys outside a tile's valid range meet V rows with weight 0, so those
    // rows must be finite: the V ring starts at zero and then only ever holds
    // loaded rows -- never a cell past a sequence's end (a partly filled last
    // block is loaded shifted, the rows before it read as zero) -- or zero fill.
    {
        uint4 *vr = reinterpret_cast<uint4 *>(data + Sh::kVOff);
        for (int i = threadIdx.x; i < kPfVStages * Sh::kKVBytes / 16; i += kPfThreads)
            vr[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();   // before any TMA write of the ring (ordered by the barrier below)
    }

    // ---- tensor memory ----
    if (warp == 5) {
        tmem_alloc(bar(kBarTmemSlot), kPfTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(&bars[kBarTmemSlot]);
    const uint32_t tO = tmem + 2 * kPfKeys;         // O columns

    const uint32_t sQ = data_s + Sh::kQOff;
    const uint32_t sK = data_s + Sh::kKOff;
    const uint32_t sV = data_s + Sh::kVOff;

    if (warp == 4 || warp == 6) {
        // ---- loads: warp 4 Q and the K ring, warp 6 the V ring ----
        const bool is_k = warp == 4;
        const CUtensorMap *tm = is_k ? tm_k : tm_v;        // 3-D view: whole blocks
        const CUtensorMap *tm4 = is_k ? tm_k4 : tm_v4;     // 4-D view: shifted last blocks
        const int full0 = is_k ? kBarKFull : kBarVFull;
        const int empty0 = is_k ? kBarKEmpty : kBarVEmpty;
        const uint32_t ring = is_k ? sK : sV;
        const int NS = is_k ? kPfKStages : kPfVStages;
        int issued = 0;
        {
            // the whole warp walks the tiles: block ids are read 32 at a time,
            // one per lane, and lane 0 issues the copies
            // prefill: the sequence's other CTAs reread these blocks; cascade:
            // each is read once per group and kv head
            const uint64_t policy = kCas ? policy_evict_first() : policy_evict_normal();
            if constexpr (MODE == kTcCascade) {
                // block ids of window w of a segment, lane l: entry w + l of the
                // segment's block order (the prefix in table order; a member's
                // last block first, then its blocks from 0)
                auto load_ids = [&](const Walk &g, int w) -> int {
                    const int nb = (g.len + BS - 1) / BS;
                    const int r = w + lane;
                    if (g.m >= n_mem || r >= nb)
                        return 0;
                    if (g.m < 0)
                        return __ldg(trow + r);
                    const int32_t *t = c.suffix_tables + (size_t)(q_tok0 + g.m) * c.max_suffix_blocks;
                    return __ldg(t + (r == 0 ? nb - 1 : r - 1));
                };
                Walk wk = walk_start();
                int ids = load_ids(wk, 0);
                // the next segment's first ids are read one segment ahead
                Walk nx = wk;
                nx.k = (nx.len + kPfKeys - 1) / kPfKeys - 1;
                walk_next(nx);
                int ids_next = load_ids(nx, 0);
                for (int j = 0; j < nt; ++j) {
                    const int s = j % NS;
                    if (j >= NS) {
                        const bool free_ = mbar_wait_bounded(bar(empty0 + s), (uint32_t)((j / NS - 1) & 1),
                                                             kWaitLimitNs);
                        if (!__all_sync(0xffffffffu, free_)) {
                            if (lane == 0)
                                raise_flag(PKV_DEVFLAG_WAIT_TIMEOUT);
                            break;
                        }
                    }
                    const int nb_seg = (wk.len + BS - 1) / BS;
                    const int kb0 = wk.k * BPT;            // a tile never straddles 32 ids
                    const int nb = min(BPT, nb_seg - kb0);
                    if (kb0 > 0 && (kb0 & 31) == 0)
                        ids = load_ids(wk, kb0);
                    if (lane == 0)
                        mbar_arrive_expect_tx(bar(full0 + s), (uint32_t)(nb * BS * D * 2));
                    __syncwarp();
                    const int i = lane / Sh::kHalves;
                    const int h = lane - i * Sh::kHalves;
                    int blk = __shfl_sync(0xffffffffu, ids, (kb0 + min(i, BPT - 1)) & 31);
                    if (i < nb) {
                        if ((unsigned)blk >= (unsigned)num_blocks) {
                            if (h == 0)
                                raise_flag(PKV_DEVFLAG_BLOCK_RANGE);
                            blk = 0;
                        }
                        // a member's partly filled last block is shifted to end at
                        // its slot's last row; the rows before it read as zero
                        const int shift = (wk.m >= 0 && kb0 + i == 0) ? wk.len - nb_seg * BS : 0;
                        const uint32_t dst = ring + s * Sh::kKVBytes + h * Sh::kKVHalf + i * BS * 128;
                        if (shift)
                            tma_load_4d(dst, tm4, bar(full0 + s), h * 64, kvh, shift, blk, policy);
                        else
                            tma_load_3d(dst, tm, bar(full0 + s), h * 64, kvh, blk * BS, policy);
                    }
                    issued = j + 1;
                    if (walk_next(wk)) {
                        ids = ids_next;
                        nx = wk;
                        nx.k = (nx.len + kPfKeys - 1) / kPfKeys - 1;
                        walk_next(nx);
                        ids_next = load_ids(nx, 0);
                    }
                }
            } else {
            // work tiles in order; key tiles numbered across them (J) so the
            // rings and their barriers carry over from one work tile to the next
            Wk cur, nxt;
            bool has_cur = next_work(cur);
            bool has_nxt = has_cur && next_work(nxt);
            // block ids, read 32 at a time (one per lane); the next work tile's
            // first 32 are read while this one streams
            int ids = has_cur && lane < cur.nblk ? __ldg(cur.trow + lane) : 0;
            int ids_nxt = has_nxt && lane < nxt.nblk ? __ldg(nxt.trow + lane) : 0;
            int J = 0;
            bool ok = true;
            while (has_cur && ok) {
                for (int j = 0; j < cur.nt; ++j, ++J) {
                    const int s = J % NS;
                    if (J >= NS) {
                        const bool free_ = mbar_wait_bounded(bar(empty0 + s), (uint32_t)((J / NS - 1) & 1),
                                                             kWaitLimitNs);
                        if (!__all_sync(0xffffffffu, free_)) {
                            if (lane == 0)
                                raise_flag(PKV_DEVFLAG_WAIT_TIMEOUT);
                            ok = false;
                            break;
                        }
                    }
                    const int kb0 = j * BPT;               // a tile never straddles 32 ids
                    const int nb = min(BPT, cur.nblk - kb0);
                    if (kb0 > 0 && (kb0 & 31) == 0)
                        ids = kb0 + lane < cur.nblk ? __ldg(cur.trow + kb0 + lane) : 0;
                    if (lane == 0)
                        mbar_arrive_expect_tx(bar(full0 + s), (uint32_t)(nb * BS * D * 2));
                    __syncwarp();
                    // lane i * kHalves + h copies half h of the tile's block i: the
                    // tile's copies leave in one warp instruction, not one by one
                    const int i = lane / Sh::kHalves;
                    const int h = lane - i * Sh::kHalves;
                    int blk = __shfl_sync(0xffffffffu, ids, (kb0 + min(i, BPT - 1)) & 31);
                    if (i < nb) {
                        if ((unsigned)blk >= (unsigned)num_blocks) {
                            if (h == 0)
                                raise_flag(PKV_DEVFLAG_BLOCK_RANGE);
                            blk = 0;
                        }
                        // the sequence's partly filled last block ends at its
                        // slot's last row; the rows before it read as zero
                        const int shift = (cur.tail && kb0 + i == cur.nblk - 1) ? cur.tail - BS : 0;
                        const uint32_t dst = ring + s * Sh::kKVBytes + h * Sh::kKVHalf + i * BS * 128;
                        if (shift)
                            tma_load_4d(dst, tm4, bar(full0 + s), h * 64, cur.kvh, shift, blk, policy);
                        else
                            tma_load_3d(dst, tm, bar(full0 + s), h * 64, cur.kvh, blk * BS, policy);
                    }
                    issued = J + 1;
                }
                if (!ok)
                    break;
                cur = nxt;
                has_cur = has_nxt;
                ids = ids_nxt;
                if (has_cur) {
                    has_nxt = next_work(nxt);
                    ids_nxt = has_nxt && lane < nxt.nblk ? __ldg(nxt.trow + lane) : 0;
                }
            }
            }
        }
        // copies still in flight land before the CTA can exit
        if (lane == 0) {
            for (int j = issued > NS ? issued - NS : 0; j < issued; ++j)
                mbar_wait_bounded(bar(full0 + j % NS), (uint32_t)((j / NS) & 1), kWaitLimitNs / 8);
        }
    } else if (warp == 7) {
        // ---- Q of each work tile: the buffer is free once the previous work
        // tile's last S = Q K^T has completed (the one-pass cascade holds its
        // 32 rows four times) ----
        if (lane == 0) {
            constexpr int kCopies = MODE == kTcCascade ? 4 : 1;
            const uint64_t policy = policy_evict_normal();
            Wk wk;
            int u = 0;
            while (next_work(wk)) {
                if (u > 0 && !mbar_wait_bounded(bar(kBarQEmpty), (uint32_t)((u - 1) & 1), kWaitLimitNs)) {
                    raise_flag(PKV_DEVFLAG_WAIT_TIMEOUT);
                    break;
                }
                mbar_arrive_expect_tx(bar(kBarQFull), (uint32_t)(kCopies * Sh::kHalves * R * 128));
#pragma unroll
                for (int q = 0; q < kCopies; ++q)
#pragma unroll
                    for (int h = 0; h < Sh::kHalves; ++h)
                        tma_load_3d(sQ + h * Sh::kQHalf + q * 32 * 128, tm_q, bar(kBarQFull), h * 64,
                                    wk.kvh * G, wk.q_tok0, policy);
                ++u;
            }
            // the last Q lands before the CTA can exit
            if (u > 0)
                mbar_wait_bounded(bar(kBarQFull), (uint32_t)((u - 1) & 1), kWaitLimitNs / 8);
        }
    } else if (warp == 5) {
        // ---- MMA issue: one thread ----
        if (lane == 0) {
            constexpr uint32_t idS = f16_idesc<BF16>(kPfRows, kPfKeys, false);
            constexpr uint32_t idO = f16_idesc<BF16>(kPfRows, D, true);
            // S_j = Q K_j^T into S buffer j & 1; Q and K K-major, 128-byte rows.
            // Buffer j & 1 last held P_{j-2}, read by P_{j-2} V_{j-2}: an MMA
            // with another accumulator and shape is not ordered behind it, so
            // the caller waits for it to complete first.
            auto issue_s = [&](int j) -> bool {
                const int ks_ = j % kPfKStages;
                if (!mbar_wait_bounded(bar(kBarKFull + ks_), (uint32_t)((j / kPfKStages) & 1),
                                       kWaitLimitNs))
                    return false;
                tc_fence_after();
                const uint32_t kt = sK + ks_ * Sh::kKVBytes;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const uint32_t koff = (uint32_t)((ks & 3) * 32);   // 16 elements = 32 bytes
                    tc_mma_f16(tmem + (j & 1) * kPfKeys,
                               sw128_desc(sQ + (ks >> 2) * Sh::kQHalf + koff, 16, 1024),
                               sw128_desc(kt + (ks >> 2) * Sh::kKVHalf + koff, 16, 1024), idS,
                               ks > 0 ? 1u : 0u);
                }
                tc_commit(bar(kBarSFull + (j & 1)));
                tc_commit(bar(kBarKEmpty + ks_));
                return true;
            };
            bool ok = true;
            if constexpr (MODE != kTcPrefill) {
                // One work tile (the prefix pass and the one-pass cascade).  This
                // plain loop is kept apart from the prefill's loop over several
                // work tiles below: running the one-pass cascade through that
                // loop made it 5 % slower.
                ok = mbar_wait_bounded(bar(kBarQFull), 0u, kWaitLimitNs) && issue_s(0);
                for (int j = 0; ok && j < nt; ++j) {
                    if (j + 1 < nt) {
                        // P_{j-1} V_{j-1} reads buffer (j+1) & 1.  O_DONE is at most
                        // one phase past j-1 here: P_j V_j is not issued yet.
                        if (j >= 1 &&
                            !(ok = mbar_wait_bounded(bar(kBarODone), (uint32_t)((j - 1) & 1), kWaitLimitNs)))
                            break;
                        if (!(ok = issue_s(j + 1)))
                            break;
                    }
                    const int vs = j % kPfVStages;
                    ok = mbar_wait_bounded(bar(kBarPFull + (j & 1)), (uint32_t)((j >> 1) & 1), kWaitLimitNs) &&
                         mbar_wait_bounded(bar(kBarVFull + vs), (uint32_t)((j / kPfVStages) & 1),
                                           kWaitLimitNs);
                    if (!ok)
                        break;
                    tc_fence_after();
                    // O += P_j V_j, as below
                    const uint32_t vt = sV + vs * Sh::kKVBytes;
                    const uint32_t tp = tmem + (j & 1) * kPfKeys;
#pragma unroll
                    for (int kk = 0; kk < KV_STEPS; ++kk)
                        tc_mma_f16_ts(tO, tp + kk * 8, sw128_desc(vt + kk * 16 * 128, Sh::kKVHalf, 1024),
                                      idO, (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(bar(kBarODone));
                    tc_commit(bar(kBarVEmpty + vs));
                }
            } else {
                // Key tiles are numbered across the CTA's work tiles (J), in one
                // loop; the current work tile holds key tiles Jbeg .. Jend-1.  S
                // of the next key tile, in this work tile or the next, is issued
                // before P V of the current one.  The last S of a work tile is
                // followed by a commit to Q_EMPTY, which lets the loader bring the
                // next work tile's Q.
                Wk nxt;
                int Jend = 0;
                bool has_nxt = false;
                if (next_work(nxt)) {
                    Jend = nxt.nt;
                    has_nxt = next_work(nxt);
                    ok = mbar_wait_bounded(bar(kBarQFull), 0u, kWaitLimitNs) && issue_s(0);
                    if (ok && Jend == 1)
                        tc_commit(bar(kBarQEmpty));
                }
                int Jbeg = 0;
                int u = 0;                              // work tile index
                for (int J = 0; ok && J < Jend; ++J) {
                    if (J + 1 < Jend) {
                        // P_{J-1} V_{J-1} reads buffer (J+1) & 1.  O_DONE is at most
                        // one phase past J-1 here: P_J V_J is not issued yet.
                        if (J >= 1 &&
                            !(ok = mbar_wait_bounded(bar(kBarODone), (uint32_t)((J - 1) & 1), kWaitLimitNs)))
                            break;
                        if (!(ok = issue_s(J + 1)))
                            break;
                        if (J + 2 == Jend)
                            tc_commit(bar(kBarQEmpty));         // that S was the work tile's last
                    }
                    const int vs = J % kPfVStages;
                    ok = mbar_wait_bounded(bar(kBarPFull + (J & 1)), (uint32_t)((J >> 1) & 1), kWaitLimitNs) &&
                         mbar_wait_bounded(bar(kBarVFull + vs), (uint32_t)((J / kPfVStages) & 1), kWaitLimitNs);
                    if (!ok)
                        break;
                    tc_fence_after();
                    // O += P_J V_J: P from TMEM (16 keys = 8 packed columns per
                    // k-step), V MN-major (head dim along the rows: halves LBO
                    // apart, 8-key groups 1024 bytes apart); the work tile's first
                    // P V overwrites O (its previous contents were read by the
                    // softmax warps before they stored this P)
                    const uint32_t vt = sV + vs * Sh::kKVBytes;
                    const uint32_t tp = tmem + (J & 1) * kPfKeys;
#pragma unroll
                    for (int kk = 0; kk < KV_STEPS; ++kk)
                        tc_mma_f16_ts(tO, tp + kk * 8, sw128_desc(vt + kk * 16 * 128, Sh::kKVHalf, 1024),
                                      idO, (J > Jbeg || kk > 0) ? 1u : 0u);
                    tc_commit(bar(kBarODone));
                    tc_commit(bar(kBarVEmpty + vs));
                    if (J + 1 == Jend && has_nxt) {
                        // the next work tile's first S, after this work tile's
                        // last P V (which must not wait for the next Q).  It
                        // overwrites the buffer P_{J-1} V_{J-1} read: wait for
                        // P_J V_J, which completes after it.  O_DONE is at most
                        // one phase past J here: P_FULL of tile J came after the
                        // softmax warps saw tile J-1's phase complete.
                        if (!(ok = mbar_wait_bounded(bar(kBarODone), (uint32_t)(J & 1), kWaitLimitNs) &&
                                   mbar_wait_bounded(bar(kBarQFull), (uint32_t)((u + 1) & 1), kWaitLimitNs) &&
                                   issue_s(J + 1)))
                            break;
                        ++u;
                        Jbeg = J + 1;
                        Jend += nxt.nt;
                        if (nxt.nt == 1)
                            tc_commit(bar(kBarQEmpty));         // that S was its work tile's last
                        has_nxt = next_work(nxt);
                    }
                }
            }
            if (!ok)
                raise_flag(PKV_DEVFLAG_WAIT_TIMEOUT);
            // every MMA issued has finished before the TMEM is released
            tc_commit(bar(kBarDrain));
            mbar_wait_bounded(bar(kBarDrain), 0u, kWaitLimitNs);
        }
    } else if constexpr (MODE == kTcCascade) {
        // ---- one-pass cascade softmax: every softmax warp holds the CTA's
        // query rows (up to 32: member rl / G, head rl % G) in its own lanes,
        // and takes key columns 16w .. 16w+15 of every tile, with its own
        // running maximum, sum and O rows; the four are merged at the end ----
        const int rl = lane;
        const bool real = rl < rows;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int cw0 = warp * 16;                  // this warp's key columns
        float m_used = kNegInf;
        float l = 0.f;
        bool ok = true;
        const float sc = scale_log2;
        const bool fold = sc > 0.f;
        const float sm = fold ? 1.f : sc;
        const float se = fold ? sc : 1.f;
        Walk sw = walk_start();
        for (int j = 0; j < nt; ++j) {
            const int s = j & 1;
            ok = mbar_wait_bounded(bar(kBarSFull + s), (uint32_t)((j >> 1) & 1), kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // valid key columns [clo, chi) and the rows [rlo, rhi) that see them
            int clo = 0, chi, rlo = 0, rhi = rows;
            const int nbs = (sw.len + BS - 1) / BS;
            if (sw.m < 0) {
                chi = min(kPfKeys, sw.len - sw.k * kPfKeys);
            } else {
                clo = sw.k == 0 ? nbs * BS - sw.len : 0;
                chi = BS * min(BPT, nbs - sw.k * BPT);
                rlo = sw.m * G;
                rhi = rlo + G;
            }
            const int lo = max(clo, cw0), hi = min(chi, cw0 + 16);   // this warp's share
            uint32_t pw[8];                         // packed weights of columns cw0 .. cw0+15
            bool resc = false;
            float alpha = 1.f;
            if (lo < hi) {
                uint32_t raw[16];
                tmem_ld16(tmem + lane_base + s * kPfKeys + cw0, raw);
                const bool row_on = rl >= rlo && rl < rhi;
                float x[16];
                float mx[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float v = fold ? __uint_as_float(raw[i]) : __uint_as_float(raw[i]) * sm;
                    x[i] = row_on && cw0 + i >= lo && cw0 + i < hi ? v : kNegInf;
                    mx[i & 3] = fmaxf(mx[i & 3], x[i]);
                }
                const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * se;
                resc = mt > m_used + 8.f;
                const float m_new = resc ? mt : m_used;
                alpha = resc ? ex2(m_used - m_new) : 1.f;
                const float msub = m_new == kNegInf ? 0.f : m_new;
                float rsv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    pw[i] = pack2<BF16>(ex2(fmaf(x[2 * i], se, -msub)), ex2(fmaf(x[2 * i + 1], se, -msub)));
                    const float2 pr = unpack2<BF16>(pw[i]);
                    rsv[i & 3] += pr.x + pr.y;
                }
                l = l * alpha + ((rsv[0] + rsv[1]) + (rsv[2] + rsv[3]));
                m_used = m_new;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    pw[i] = 0u;
            }
            if (j > 0) {
                // as below: P_{j-1} V_{j-1} has completed before P_j is stored
                ok = mbar_wait_bounded(bar(kBarODone), (uint32_t)((j - 1) & 1), kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tO + lane_base + c0, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tO + lane_base + c0, o);
                }
            }
            // P over the first 32 columns of S_j: this warp's 8 packed columns,
            // zero for the other warps' keys
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                pk[i] = (i >> 3) == warp ? pw[i & 7] : 0u;
            tmem_st32(tmem + lane_base + s * kPfKeys, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(kBarPFull + s));
            walk_next(sw);
        }
        if (ok)
            ok = mbar_wait_bounded(bar(kBarODone), (uint32_t)((nt - 1) & 1), kWaitLimitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0)
            raise_flag(PKV_DEVFLAG_WAIT_TIMEOUT);
        // merge the four warps' partial softmaxes of each row by log-sum-exp,
        // through the K/V rings (free: every load has been consumed by an MMA
        // that has completed); a warp that gave up leaves NaN as its maximum
        float *st_m = reinterpret_cast<float *>(data + Sh::kKOff);   // [4][32]
        float *st_l = st_m + 4 * 32;                                  // [4][32]
        float *part = st_l + 4 * 32;                                  // [4][D][32], scaled O rows
        st_m[warp * 32 + lane] = ok ? m_used : __int_as_float(0x7fc00000);
        st_l[warp * 32 + lane] = l;
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bar(kBarEpi0));
        bool go = mbar_wait_bounded(bar(kBarEpi0), 0u, kWaitLimitNs);
        float M = kNegInf;
        bool bad = false;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float mw = st_m[w * 32 + lane];
            bad |= mw != mw;
            M = fmaxf(M, mw);
        }
        go = __all_sync(0xffffffffu, go && !bad);
        if (go) {
            float L = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float mw = st_m[w * 32 + lane];
                L += mw == kNegInf ? 0.f : ex2(mw - M) * st_l[w * 32 + lane];
            }
            const float f = L > 0.f && m_used != kNegInf ? ex2(m_used - M) / L : 0.f;
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(tO + lane_base + c0, o);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    part[(warp * D + c0 + i) * 32 + lane] = __uint_as_float(o[i]) * f;
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bar(kBarEpi1));
        go = __all_sync(0xffffffffu, mbar_wait_bounded(bar(kBarEpi1), 0u, kWaitLimitNs) && go);
        if (!go && lane == 0)
            raise_flag(PKV_DEVFLAG_WAIT_TIMEOUT);
        const int b = q_tok0 + rl / G;
        if (go && real && (grouped || b < gs0 || b >= gsN)) {
            // this warp writes columns D/4 * w .. D/4 * (w+1) - 1 of row rl
            constexpr int CW = D / 4;
            uint4 *orow = reinterpret_cast<uint4 *>(
                c.out + ((size_t)b * num_heads + (size_t)kvh * G + rl % G) * D + warp * CW);
#pragma unroll
            for (int i = 0; i < CW; i += 8) {
                uint32_t wd[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float v0 = 0.f, v1 = 0.f;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        v0 += part[(w * D + warp * CW + i + 2 * e) * 32 + lane];
                        v1 += part[(w * D + warp * CW + i + 2 * e + 1) * 32 + lane];
                    }
                    wd[e] = pack2<BF16>(v0, v1);
                }
                orow[i / 8] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            }
        }
    } else {
        // ---- softmax and epilogue: thread = row r of the tile = TMEM lane r ----
        const int r = warp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        // row r is (token r / G, head r % G) of the tile; so is the first row
        // of its quad, r - q.  Divided once here: an integer division goes
        // through the MUFU unit, which the other softmax warps keep busy.
        const int q = lane & 3;
        const int r_tok = r / G, r_head = r - r_tok * G;
        int rq_tok = r_tok, rq_head = r_head - q;
        while (rq_head < 0) {
            rq_head += G;
            --rq_tok;
        }
        // for a positive scale the maximum is taken on the raw scores and the
        // scale is folded into the exponent, p = 2^(s*scale - m)
        const float sc = scale_log2;
        const bool fold = sc > 0.f;
        const float sm = fold ? 1.f : sc;       // applied before the maximum
        const float se = fold ? sc : 1.f;       // applied in the exponent
        bool ok = true;
        Wk cur;
        int J = 0;                              // the work tile's first key tile
        while (ok && next_work(cur)) {
        const int grow = cur.row0 + r;          // row within the sequence
        const bool real = r < R && grow < cur.rows;
        const int pos = real && MODE == kTcPrefill ? cur.pos0 + r_tok : cur.p_max;
        float m_used = kNegInf;
        float l = 0.f;
        for (int j = 0; j < cur.nt; ++j) {
            const int Jj = J + j;
            const int s = Jj & 1;
            ok = mbar_wait_bounded(bar(kBarSFull + s), (uint32_t)((Jj >> 1) & 1), kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t raw[64];
            tmem_ld64(tmem + lane_base + s * kPfKeys, raw);
            // the scores with the mask applied (-inf where a row sees no key)
            float x[64];
            const int t0 = j * kPfKeys;
            if (t0 + kPfKeys - 1 <= cur.pos0) {     // every key visible to every row
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    x[c] = fold ? __uint_as_float(raw[c]) : __uint_as_float(raw[c]) * sm;
            } else if (!cur.tail || j + 1 < cur.nt) {   // causal mask, no shifted block
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float v = fold ? __uint_as_float(raw[c]) : __uint_as_float(raw[c]) * sm;
                    x[c] = t0 + c <= pos ? v : kNegInf;
                }
            } else {
                // the work tile's last key tile holds the sequence's partly
                // filled last block, loaded shifted: its slot starts with
                // BS - tail rows of zeros (no key), then keys of positions
                // t0 + c - (BS - tail); columns past it are past the context
                const int sh_lo = (cur.nblk - 1 - j * BPT) * BS;
                const int sh = BS - cur.tail;
                const int nv = pos - t0 + 1;        // keys of this row in the tile, were none shifted
                // visible columns: [0, min(nv, sh_lo)) and, in the shifted slot, [sh_lo + sh, nv + sh)
                const uint64_t vm = col_range(0, min(nv, sh_lo)) | col_range(sh_lo + sh, nv + sh);
                const uint32_t vlo = (uint32_t)vm, vhi = (uint32_t)(vm >> 32);
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float v = fold ? __uint_as_float(raw[c]) : __uint_as_float(raw[c]) * sm;
                    x[c] = (((c < 32 ? vlo : vhi) >> (c & 31)) & 1u) ? v : kNegInf;
                }
            }
            // eight independent max chains of three-input maxima, not a 64-long one
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mx[i] = fmaxf(x[2 * i], x[2 * i + 1]);
#pragma unroll
            for (int c = 16; c < 64; c += 2)
                mx[(c >> 1) & 7] = fmax3(mx[(c >> 1) & 7], x[c], x[c + 1]);
            const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * se;
            const bool resc = mt > m_used + 8.f;    // first tile: m_used = -inf
            const float m_new = resc ? mt : m_used;
            const float alpha = resc ? ex2(m_used - m_new) : 1.f;
            const float msub = m_new == kNegInf ? 0.f : m_new;
            // exponents two columns at a time (packed f32x2 fma); the row sum is
            // taken over the rounded weights the MMA multiplies, so the
            // normalised weights sum to one exactly (four packed chains)
            const uint64_t se2 = f2(se, se), nm2 = f2(-msub, -msub);
            uint32_t pk[32];
            uint64_t rsv[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const uint64_t e = fma2(f2(x[2 * c], x[2 * c + 1]), se2, nm2);
                pk[c] = pack2<BF16>(ex2(f2_lo(e)), ex2(f2_hi(e)));
                const float2 pr = unpack2<BF16>(pk[c]);
                rsv[c & 3] = add2(rsv[c & 3], f2(pr.x, pr.y));
            }
            const uint64_t r2 = add2(add2(rsv[0], rsv[1]), add2(rsv[2], rsv[3]));
            const float rs = f2_lo(r2) + f2_hi(r2);
            l = l * alpha + rs;
            m_used = m_new;
            if (j > 0) {
                // Wait for P_{j-1} V_{j-1}: O then holds it (for the rescale),
                // and O_DONE stays within one phase of this warp, so the
                // epilogue's parity wait below names the last tile's phase and
                // no other.  O_DONE cannot be ahead of this wait either: P_j V_j
                // needs this warp's P_j.  The MMA that may still run now is
                // S_{j+1}, into the other S/P buffer.
                ok = mbar_wait_bounded(bar(kBarODone), (uint32_t)((Jj - 1) & 1), kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tO + lane_base + c0, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tO + lane_base + c0, o);
                }
            }
            // P_j over the first 32 columns of S_j (already read into registers)
            tmem_st32(tmem + lane_base + s * kPfKeys, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(kBarPFull + s));
        }
        if (ok)
            ok = mbar_wait_bounded(bar(kBarODone), (uint32_t)((J + cur.nt - 1) & 1), kWaitLimitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            // query row (q_tok0 + r / G, head kvh * G + r % G): row0 is a multiple of G
            const size_t orow_i =
                (size_t)(cur.q_tok0 + r_tok) * num_heads + (size_t)cur.kvh * G + r_head;
            if constexpr (MODE == kTcPrefill) {
                // A row is D * 2 contiguous bytes, and rows of different
                // tokens lie apart.  Each thread normalises its own row, then
                // the four lanes of a quad trade 16-byte chunks so that a store
                // instruction writes 64 contiguous bytes of each of eight rows
                // (one quad per row), not 16 bytes of each of 32 rows.
                uint4 *orow[4];
                int tk = rq_tok, hd = rq_head;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int rr = r - q + h;           // the quad's row h: (token tk, head hd)
                    const bool rr_real = rr < R && cur.row0 + rr < cur.rows;
                    orow[h] = rr_real ? reinterpret_cast<uint4 *>(
                                            a.out + ((size_t)(cur.q_tok0 + tk) * num_heads +
                                                     (size_t)cur.kvh * G + hd) * D)
                                      : nullptr;
                    if (++hd == G) {
                        hd = 0;
                        ++tk;
                    }
                }
                // O in two 64-column loads (one for D = 64)
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 64) {
                    uint32_t o[64];
                    tmem_ld64(tO + lane_base + c0, o);
#pragma unroll
                    for (int g2 = 0; g2 < 2; ++g2) {
                        uint4 ch[4];
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                w[e] = pack2<BF16>(__uint_as_float(o[32 * g2 + 8 * v + 2 * e]) * inv,
                                                   __uint_as_float(o[32 * g2 + 8 * v + 2 * e + 1]) * inv);
                            ch[v] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                        quad_transpose(ch, q);
#pragma unroll
                        for (int h = 0; h < 4; ++h)
                            if (orow[h] != nullptr)
                                orow[h][(c0 + 32 * g2) / 8 + q] = ch[h];
                    }
                }
            } else {
                // partition record: (m, l) with sum_k 2^(s_k) = 2^m * l, and O / l
                const size_t rec = orow_i * c.num_parts + rec_part;
                float4 *orec = reinterpret_cast<float4 *>(c.rec_o + rec * D);
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tO + lane_base + c0, o);
                    if (real) {
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            orec[c0 / 4 + v] = make_float4(__uint_as_float(o[4 * v]) * inv,
                                                           __uint_as_float(o[4 * v + 1]) * inv,
                                                           __uint_as_float(o[4 * v + 2]) * inv,
                                                           __uint_as_float(o[4 * v + 3]) * inv);
                    }
                }
                if (real) {
                    c.rec_m[rec] = m_used;
                    c.rec_l[rec] = l;
                }
            }
            // the next work tile's first P V overwrites O: these reads of O
            // complete (tcgen05.wait::ld) before this warp stores that tile's P
        }
        J += cur.nt;
        }
        if (!ok && lane == 0)
            raise_flag(PKV_DEVFLAG_WAIT_TIMEOUT);
    }

    // ---- release the tensor memory once every warp is done with it ----
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kPfTmemCols);
    }
}

// tm_k / tm_v view the caches as 3-D tensors {head_dim, num_kv_heads,
// num_blocks * block_size} (box 64 x 1 x block_size), tm_k4 / tm_v4 as 4-D
// tensors {head_dim, num_kv_heads, block_size, num_blocks} (box 64 x 1 x
// block_size x 1): whole blocks come through the first, a partly filled last
// block, shifted so that the rows before it read as zero, through the second.
template <int D, int BS, bool BF16>
__global__ void __launch_bounds__(kPfThreads, 2)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k4,
                  const __grid_constant__ CUtensorMap tm_v4, const PrefillArgs a)
{
    tc_attend<D, BS, BF16, kTcPrefill>(&tm_q, &tm_k, &tm_v, &tm_k4, &tm_v4, a, CascadeArgs{});
}

template <int D, int BS, bool BF16>
__global__ void __launch_bounds__(kPfThreads, 2)
prefix_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k4,
                 const __grid_constant__ CUtensorMap tm_v4, const CascadeArgs c)
{
    tc_attend<D, BS, BF16, kTcPrefix>(&tm_q, &tm_k, &tm_v, &tm_k4, &tm_v4, PrefillArgs{}, c);
}

template <int D, int BS, bool BF16>
__global__ void __launch_bounds__(kPfThreads, 2)
cascade_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k4,
                  const __grid_constant__ CUtensorMap tm_v4, const CascadeArgs c)
{
    tc_attend<D, BS, BF16, kTcCascade>(&tm_q, &tm_k, &tm_v, &tm_k4, &tm_v4, PrefillArgs{}, c);
}

}  // namespace pkv
