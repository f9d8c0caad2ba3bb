// Attention on the 5th-generation tensor cores (tcgen05 + TMEM): the varlen causal prefill
// (prefill_tcgen05_kernel, below) and the shared-prefix tiles of the decode step
// (prefix_tiles_kernel, further down, where its own description is).
//
// ("Nano-vLLM inference engine architecture", section "Low-level performance details":
// prefill runs a variable-length attention over cumulative sequence lengths; "Nano-vLLM
// part 1" section 5.2 builds those lengths; section 4.2's prefix caching means the keys
// of a sequence are its cached prefix followed by the suffix stored in this step.)
//
// Query tile: 128 rows = 128/P tokens of one sequence times the P query heads (P = query
// heads per KV head when that is a power of two up to 8, else 1) that share one KV head,
// so each K/V tile fetched serves P heads.  Keys come in tiles of 128 from the
// block-paged cache.  With a causal mask a query tile only visits key tiles up to its
// last token's position (bottom-right alignment: suffix token r is at position
// Lk - Lq + r).
//
// Work unit: a PAIR of query tiles of the same sequence and KV head (A = tile 2w, B = tile
// 2w + 1, which has at least as many key tiles; B may be absent).  Both read the same K/V tiles, so
// each tile is fetched once for 256 query rows, and the two tiles' MMAs and softmaxes
// interleave: while one tile's softmax runs, the tensor core computes the other tile's
// P V and its next S.  One CTA per SM, persistent: the CTAs claim units dynamically from
// the plan kernel's list, which holds the pairs with the most key tiles first.  Warp roles:
//   warp 0      TMA producer: K_0, Q_A, V_0, Q_B, then K_j and V_j tiles into a 4-stage
//               K/V ring (one 3-D tensor-map box per cache block piece; a 128-key tile
//               spans 128 / block_size blocks when the block size is below 128); the Q
//               tiles go into a ring of 3 buffers.  The MMA issuer starts S_A0 before
//               waiting for Q_B;
//   warp 1      allocates all 512 TMEM columns; one lane issues the MMAs in the order
//                 S_A0 S_B0 | O_A += P_A0 V_0, S_A1, O_B += P_B0 V_0, S_B1 | ...
//               where S = Q K_j^T is SS (both operands K-major in shared memory) and
//               O += P V is TS (P from TMEM, V MN-major in shared memory);
//   warps 2, 3  idle (they complete warpgroup 0, which gives registers to the softmax);
//   warps 4..7  softmax of tile A, warps 8..11 softmax of tile B: one thread per query
//               row (each warp on its own 32 TMEM lanes), see the pass comments below.
// TMEM columns: tile A S/P [0, 128), O [128, 256); tile B S/P [256, 384), O [384, 512).
// The MMAs of one thread execute in issue order, so S_{j+1} (issued after O += P_j V_j)
// cannot overwrite P_j early.
//
// Stale rows (freed blocks are not cleared, part 1 section 4.3): the scores of K rows past
// the length are replaced by -inf with a bit mask (never by arithmetic, which would keep a
// NaN), and V rows past the length in the last key tile are zeroed in shared memory
// before their MMAs, so a 0 weight never meets a NaN.
#include <algorithm>
#include <cfloat>
#include <climits>
#include <cmath>
#include <mutex>

#include "attn_warp.cuh"
#include "nvpa_internal.h"
#include "sm100.cuh"

namespace nvpa {

using namespace sm100;

namespace {

constexpr int kQ = 128;          // query rows per tile (MMA M): tokens x packed heads
constexpr int kKV = 128;         // keys per tile (MMA N of QK^T, K of PV)
// Shared memory holds seven 32 KB tiles (of the 227 KB a CTA may have): a ring of K/V
// stages, each one K or one V tile, and a ring of Q tiles.  A tile takes 2 to 5 us from
// the TMA issue to its arrival under load, and the first tiles of a unit are the ones
// most often not in L2; with a third Q buffer the next unit's Q_A can be loaded while both
// Q tiles of the current unit are still in use, which pays more than a fifth K/V stage.
constexpr int kStages = 4;         // K/V ring stages
constexpr int kQBufs = 3;          // Q tile ring: tiles A and B of a unit take the next two
constexpr int kWarps = 12;       // producer, MMA, 2 idle, 2 x 4 softmax
constexpr int kThreads = kWarps * 32;
// Register split (setmaxnreg acts on whole warpgroups): the launch gives every thread
// kLaunchRegs; warpgroup 0 (producer, MMA, idle) gives registers back down to kSmallRegs
// and the two softmax warpgroups take kSoftmaxRegs.  The shares add up to the launch's
// total: 4 * kSmallRegs + 8 * kSoftmaxRegs == 12 * kLaunchRegs (per 32 lanes), and no
// SM sub-partition (warps w, w+4, w+8) exceeds its 16384 registers.
constexpr int kLaunchRegs = 168, kSmallRegs = 104, kSoftmaxRegs = 200;
static_assert(4 * kSmallRegs + 8 * kSoftmaxRegs == 12 * kLaunchRegs, "register split");
static_assert((kSmallRegs + 2 * kSoftmaxRegs) * 32 <= 16384, "sub-partition registers");
constexpr int kTmemCols = 512;   // 2 tiles x (S/P 128 + O up to 128)
constexpr int kMinTokensPerTile = 16;   // 128 rows / at most 8 packed heads
constexpr int kUnitRing = 4;            // claimed unit indices handed from the producer to the others
constexpr int kUnitReaders = 1 + 8;     // MMA warp + the 8 softmax warps

// Bit k set for the first n of 32 columns (n clamped to [0, 32]).
__device__ __forceinline__ uint32_t visible_mask(int n) {
    return n >= 32 ? 0xffffffffu : n <= 0 ? 0u : ((1u << n) - 1u);
}

// bits as a float when bit k of vm is set, else `fill` (shift/and/or, no predicate).
__device__ __forceinline__ float keep_or(uint32_t bits, uint32_t vm, int k, float fill) {
    const uint32_t keep = (uint32_t)((int32_t)(vm << (31 - k)) >> 31);
    return __uint_as_float((bits & keep) | (__float_as_uint(fill) & ~keep));
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// The softmax of one S row (one thread per row, the whole 128-column row in registers) is a
// single code path for every tile and either sign of the scale, kept small on purpose: the
// warps that issue the MMAs and the copies share each SM sub-partition's instruction
// cache with two softmax warps, and the fully unrolled row loops are most of the kernel's
// code.

// Columns at or past lim - key0 (keys the row does not see, including rows past the
// sequence) become -inf by bit mask, whatever they held.
template <int N>
__device__ __forceinline__ void mask_row(uint32_t (&sv)[N], int key0, int lim) {
#pragma unroll
    for (int c = 0; c < N / 32; ++c) {
        const uint32_t vm = visible_mask(lim - key0 - c * 32);
#pragma unroll
        for (int k = 0; k < 32; ++k) sv[c * 32 + k] = __float_as_uint(keep_or(sv[c * 32 + k], vm, k, -INFINITY));
    }
}

// Largest value of the row: two independent accumulators, two new values per three-input
// instruction.
template <int N>
__device__ __forceinline__ float row_max(const uint32_t (&sv)[N]) {
    float e0 = -INFINITY, e1 = -INFINITY;
#pragma unroll
    for (int k = 0; k < N; k += 4) {
        e0 = max3(e0, __uint_as_float(sv[k]), __uint_as_float(sv[k + 1]));
        e1 = max3(e1, __uint_as_float(sv[k + 2]), __uint_as_float(sv[k + 3]));
    }
    return fmaxf(e0, e1);
}

// P = exp2(s * c + nm) of N raw scores of a row (c > 0: the scale in log2 units; one
// packed FMA per pair of scores), packed to bf16 pairs and written to TMEM from column
// p_col on (32 S columns become 16 P columns); returns the sum of the fp32 values.  A -inf
// score or offset gives 0.
template <int N>
__device__ __forceinline__ float exp_row(const uint32_t (&sv)[N], uint32_t p_col, float c, float nm) {
    const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(nm, nm);
    uint64_t l0 = f2_pack(0.f, 0.f), l1 = l0;
#pragma unroll
    for (int cc = 0; cc < N / 32; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
            float a, b;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[cc * 32 + k]), __uint_as_float(sv[cc * 32 + k + 1])), c2, nm2),
                      a, b);
            a = fast_exp2(a);
            b = fast_exp2(b);
            const uint64_t p2 = f2_pack(a, b);
            if ((k / 2) & 1)
                l1 = f2_add(l1, p2);
            else
                l0 = f2_add(l0, p2);
            pk[k / 2] = pack_bf16x2(a, b);
        }
        tmem_st16(p_col + cc * 16, pk);
    }
    float a0, b0, a1, b1;
    f2_unpack(l0, a0, b0);
    f2_unpack(l1, a1, b1);
    return (a0 + b0) + (a1 + b1);
}

// One 32-byte global store (the address must be 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :: "l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]),
                    "r"(w[7])
                 : "memory");
}

struct PrefillParams {
    const int32_t* block_tables;
    const int32_t* cu_q;
    const int32_t* cu_k;
    uint16_t* out;
    float* lse_out;
    int32_t* err;
    const int4* tiles;           // plan: (sequence, query tile A, query tile B or -1, key partition)
    const int32_t* ntiles;       // plan: number of entries
    int32_t* unit_counter;       // next unit to claim (reset by the plan)
    // shared-prefix decode mode: "sequences" are prefix groups whose "queries" are the
    // members' decode query rows; results go to each member's prefix partition slot
    const uint16_t* q_rows;      // decode q [batch, Hq, D]
    const int32_t* members;      // members of all groups, grouped
    const int32_t* group_start;  // [num_groups + 1] into members
    const int32_t* group_len;    // [num_groups] shared prefix length in tokens
    float* o_part;               // partition c of the prefix goes to slot c of each member
    float* lse_part;
    int s_max;
    int pchunk;                  // prefix keys per partition (a multiple of 128)
    int batch, total_q, hq, hkv, group;
    int pack, pack_shift;        // query heads per row group (P) and log2(P)
    int tq;                      // tokens per tile, 128 / P
    int hgroups;                 // head groups, hq / P
    int max_blocks, num_blocks, block_size, block_shift;
    int max_q, max_k, causal;
    float scale_log2;            // |scale| * log2(e) (a negative scale flips the sign of Q K^T)
    int negate_qk;               // scale < 0: S = -Q K^T
    int out_v8;                  // out is 32-byte aligned: 32-byte stores in the epilogue
};

template <int D>
struct Layout {
    static constexpr int REGIONS = D / 64;                  // 64 bf16 = one 128-byte swizzle row
    static constexpr int REGION_BYTES = 128 * 128;          // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = REGIONS * REGION_BYTES;
    static constexpr int Q_OFF = 0;                         // ring of kQBufs Q tiles
    static constexpr int STAGE_OFF = kQBufs * TILE_BYTES;
    static constexpr int BAR_OFF = STAGE_OFF + kStages * TILE_BYTES;
    // barriers (the per-tile ones come in pairs: + 0 for tile A, + 1 for tile B)
    static constexpr int B_QFULL = 0, B_QEMPTY = kQBufs, B_KVFULL = 2 * kQBufs, B_KVEMPTY = B_KVFULL + kStages;
    static constexpr int B_SFULL = B_KVEMPTY + kStages, B_PFULL = B_SFULL + 2, B_ODONE = B_PFULL + 2;
    static constexpr int B_OFINAL = B_ODONE + 2, B_OFREE = B_OFINAL + 2, B_DRAIN = B_OFREE + 2;
    static constexpr int B_UFULL = B_DRAIN + 1, B_UEMPTY = B_UFULL + kUnitRing;
    static constexpr int NBARS = B_UEMPTY + kUnitRing;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;     // tmem base, abort flag
    static constexpr int RING_OFF = (MISC_OFF + 16 + 15) / 16 * 16;   // unit descriptions
    static constexpr int BYTES = RING_OFF + 32 * kUnitRing;
    static constexpr int ALLOC = BYTES + 1024;               // room to align the base to 1024
};
static_assert(Layout<128>::ALLOC <= 227 * 1024, "shared memory per CTA");

// A work unit as the producer hands it to the MMA and softmax warps (32 bytes in shared
// memory): its plan entry, head group and the lengths of its sequence (or prefix group),
// so that no consumer reads global memory at a unit boundary.  e.x < 0 ends the loop.
struct UnitDesc {
    int4 e;              // plan entry: sequence (group), query tile A, tile B or -1, key partition
    int hg;              // head group
    int q0, lq, lk;      // first query row, query rows, keys (shared-prefix tiles: prefix length)
};
static_assert(sizeof(UnitDesc) == 32, "unit description size");

struct TileInfo {
    bool valid;          // false: the pair's B slot is empty
    int seq, qt, head0, hk;
    int q0, lq, lk;      // first query row (global), query rows, keys of the sequence
    int kbeg, chunk;     // shared-prefix tiles: first key and index of the key partition
    int tok0, ntok;      // first token of the tile inside the sequence, tokens in the tile
    int nkv;             // key tiles visited
};

__device__ __forceinline__ int tile_nkv(int causal, int lq, int lk, int tok0, int ntok) {
    const int ktiles = (lk + kKV - 1) / kKV;
    return causal ? min(ktiles, (lk - lq + tok0 + ntok - 1) / kKV + 1) : ktiles;
}

// Tile A (second = false) or B of unit u.
template <bool PREFIX>
__device__ __forceinline__ TileInfo tile_info(const PrefillParams& p, const UnitDesc& u, bool second) {
    TileInfo t;
    const int qt = second ? u.e.z : u.e.y;
    t.valid = qt >= 0;
    t.seq = u.e.x;
    t.qt = max(qt, 0);
    t.head0 = u.hg * p.pack;
    t.hk = t.head0 / p.group;
    t.q0 = u.q0;
    t.lq = u.lq;
    if constexpr (PREFIX) {
        // group e.x: its members are the queries, keys [kbeg, kbeg + lk) of its shared
        // prefix the keys (no mask)
        t.chunk = u.e.w;
        t.kbeg = t.chunk * p.pchunk;
        t.lk = min(p.pchunk, u.lk - t.kbeg);
    } else {
        t.chunk = 0;
        t.kbeg = 0;
        t.lk = u.lk;
    }
    t.tok0 = t.qt * p.tq;
    t.ntok = min(p.tq, t.lq - t.tok0);
    t.nkv = t.valid ? tile_nkv(PREFIX ? 0 : p.causal, t.lq, t.lk, t.tok0, t.ntok) : 0;
    return t;
}

// The lengths of the sequence (group) of plan entry e, from global memory.
template <bool PREFIX>
__device__ __forceinline__ UnitDesc describe_unit(const PrefillParams& p, int4 e, int hg) {
    UnitDesc u;
    u.e = e;
    u.hg = hg;
    if (e.x < 0) {
        u.q0 = u.lq = u.lk = 0;
    } else if constexpr (PREFIX) {
        u.q0 = __ldg(p.group_start + e.x);
        u.lq = __ldg(p.group_start + e.x + 1) - u.q0;
        u.lk = __ldg(p.group_len + e.x);
    } else {
        u.q0 = __ldg(p.cu_q + e.x);
        u.lq = __ldg(p.cu_q + e.x + 1) - u.q0;
        u.lk = __ldg(p.cu_k + e.x + 1) - __ldg(p.cu_k + e.x);
    }
    return u;
}

// ------------------------------------------------------------------------------------
// plan: list the query-tile pairs, the ones with the most key tiles first
// ------------------------------------------------------------------------------------
constexpr int kPlanBuckets = 4096;   // key-tile counts sorted exactly; longer pairs share the top bucket

// Key tiles visited by the pair (2w, 2w + 1) of a sequence with cnt query tiles (tile
// 2w + 1, when it exists, ends later and visits at least as many).
__device__ __forceinline__ int pair_nkv(const PrefillParams& p, int lq, int lk, int cnt, int w) {
    const int qt = 2 * w + 1 < cnt ? 2 * w + 1 : 2 * w;
    return tile_nkv(p.causal, lq, lk, qt * p.tq, min(p.tq, lq - qt * p.tq));
}

// Work units are pairs of query tiles (2w, 2w + 1) of one sequence, counted from its first
// tile, so that both tiles of a pair end in the same 128-key tile when 2 * tokens per tile
// = 128 and the cached prefix is a whole number of 128-key tiles (block sizes 128 and
// 256): they then finish their key loops together; for an odd tile count the last tile
// stands alone.  The list is sorted by key tiles, most first (a counting sort over the
// pairs' key-tile counts), so that the units claimed last are the shortest and the CTAs
// finish close together.  The order inside one count is whatever the atomics give: it
// decides only which CTA runs a unit, never a result.
__global__ void __launch_bounds__(1024) prefill_plan_kernel(const PrefillParams p, int4* tiles,
                                                            int32_t* ntiles) {
    __shared__ int s_hist[kPlanBuckets];
    __shared__ int warp_tot[32];
    // the attention grid may launch now: it sets up, then waits for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const long long cap = (long long)p.max_blocks * p.block_size;
    auto seq_ok = [&](int i, int& lq, int& lk) {
        const int q0 = __ldg(p.cu_q + i), q1 = __ldg(p.cu_q + i + 1);
        const int k0 = __ldg(p.cu_k + i), k1 = __ldg(p.cu_k + i + 1);
        lq = q1 - q0;
        lk = k1 - k0;
        return q0 >= 0 && lq >= 0 && lk >= lq && lq <= p.max_q && lk <= p.max_k && lk <= cap &&
               q1 <= p.total_q;
    };
    auto bucket = [&](int nkv) { return min(nkv, kPlanBuckets - 1); };
    for (int b = tid; b < kPlanBuckets; b += blockDim.x) s_hist[b] = 0;
    __syncthreads();
    // histogram of the pairs' key-tile counts (a malformed sequence gives none and is flagged)
    for (int i = tid; i < p.batch; i += blockDim.x) {
        int lq, lk;
        if (!seq_ok(i, lq, lk)) {
            flag_error(p.err, NVPA_FLAG_BAD_LENGTH);
            continue;
        }
        const int cnt = (lq + p.tq - 1) / p.tq;
        for (int w = 0; 2 * w < cnt; ++w) atomicAdd(&s_hist[bucket(pair_nkv(p, lq, lk, cnt, w))], 1);
    }
    __syncthreads();
    // first position of each count, counts in descending order: thread t takes buckets
    // kPlanBuckets - 1 - 4t - k (k < 4); a block-wide exclusive scan of the thread sums
    constexpr int kPer = kPlanBuckets / 1024;
    int v[kPer];
    int sum = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        v[k] = s_hist[kPlanBuckets - 1 - (kPer * tid + k)];
        sum += v[k];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    int run = incl - sum + (wid ? warp_tot[wid - 1] : 0);
    const int total = warp_tot[31];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        s_hist[kPlanBuckets - 1 - (kPer * tid + k)] = run;
        run += v[k];
    }
    __syncthreads();
    // place each pair at the next free position of its count
    for (int i = tid; i < p.batch; i += blockDim.x) {
        int lq, lk;
        if (!seq_ok(i, lq, lk)) continue;
        const int cnt = (lq + p.tq - 1) / p.tq;
        for (int w = 0; 2 * w < cnt; ++w) {
            const int pos = atomicAdd(&s_hist[bucket(pair_nkv(p, lq, lk, cnt, w))], 1);
            tiles[pos] = make_int4(i, 2 * w, 2 * w + 1 < cnt ? 2 * w + 1 : -1, 0);
        }
    }
    if (tid == 0) {
        *ntiles = total;
        ntiles[1] = 0;   // the attention kernel's unit counter
    }
}

// ------------------------------------------------------------------------------------
// the attention kernel
// ------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tcgen05_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                       const __grid_constant__ CUtensorMap v_map, const PrefillParams p) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(smem);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
    UnitDesc* unit_ring = reinterpret_cast<UnitDesc*>(smem + L::RING_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(bars + L::B_SFULL + x, 1);
            mbar_init(bars + L::B_PFULL + x, 4);
            mbar_init(bars + L::B_ODONE + x, 1);
            mbar_init(bars + L::B_OFINAL + x, 1);
            mbar_init(bars + L::B_OFREE + x, 4);
        }
        for (int q = 0; q < kQBufs; ++q) {
            mbar_init(bars + L::B_QFULL + q, 1);
            mbar_init(bars + L::B_QEMPTY + q, 1);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bars + L::B_KVFULL + s, 1);
            mbar_init(bars + L::B_KVEMPTY + s, 1);
        }
        mbar_init(bars + L::B_DRAIN, 1);
        for (int i = 0; i < kUnitRing; ++i) {
            mbar_init(bars + L::B_UFULL + i, 1);
            mbar_init(bars + L::B_UEMPTY + i, kUnitReaders);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&q_map);
        tma_prefetch_desc(&k_map);
        tma_prefetch_desc(&v_map);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // (broadcast from lane 0: a shuffled value is known to be the same in every lane, which
    // lets the compiler keep what is derived from it, like the MMA operands, warp-uniform)
    const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
    // This grid is launched as a programmatic dependent of its plan kernel: the setup above
    // overlaps the plan, and nothing the plan writes is read before this wait.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // Work units: every plan entry (a pair of query tiles) for every head group.
    const int total = __ldcg(p.ntiles) * p.hgroups;
    auto unit_of = [&](int idx, int4& e, int& hg) {
        hg = idx % p.hgroups;
        e = __ldg(p.tiles + idx / p.hgroups);
    };
    // Units are claimed dynamically (longest first, as the plan orders them): the producer
    // claims them with an atomic, one unit ahead of the one it loads, and hands each one's
    // description to the MMA and softmax warps through a small ring in shared memory.
    // claim(n) returns the n-th unit of this CTA; e.x is -1 at the end, -2 if a wait timed
    // out.
    auto claim = [&](int n) -> UnitDesc {
        const int slot = n % kUnitRing;
        UnitDesc u;
        if (!mbar_wait(bars + L::B_UFULL + slot, (n / kUnitRing) & 1, abort_flag, p.err)) {
            u.e = make_int4(-2, -1, -1, 0);
            u.hg = u.q0 = u.lq = u.lk = 0;
            return u;
        }
        u = unit_ring[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::B_UEMPTY + slot);
        return u;
    };

    if (warp < 4) {
      // warpgroup 0: producer, MMA issuer and two idle warps, with few registers
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kSmallRegs));
      if (warp == 0) {
        // ============================ TMA producer ============================
        // The whole warp walks the units; lane 0 issues the copies and barrier operations,
        // lane c < 8 holds the physical block of piece c of the next key tile, loaded one
        // key tile ahead so that no copy waits on a block-table lookup.
        uint32_t fill = 0;
        uint32_t qfill = 0;
        const int piece = min(p.block_size, kKV);
        // The block id of piece `lane` of key tile j, or kNoPiece for lanes past the tile's
        // pieces.  The load is only issued here; its value is range-checked where it is
        // used (load_kv, one key tile later), so the warp does not stall on it.
        constexpr int kNoPiece = INT_MIN;
        auto load_pieces = [&](const int32_t* bt, int kbeg, int lk, int j) {
            const int key0 = j * kKV;
            const int npieces = (min(kKV, lk - key0) + piece - 1) / piece;
            return lane < npieces ? __ldg(bt + ((kbeg + key0 + lane * piece) >> p.block_shift)) : kNoPiece;
        };
        // Claims run one unit ahead: the index and description of unit n + 1 are fetched
        // while unit n's copies are issued, so that the next unit's first copies do not
        // wait for an atomic and two dependent global loads.
        auto claim_next = [&]() -> int { return lane == 0 ? atomicAdd(p.unit_counter, 1) : 0; };
        auto resolve = [&](int pending) -> int {
            const int i = __shfl_sync(0xffffffffu, pending, 0);
            return i < total ? i : -1;
        };
        auto entry = [&](int idx, int4& e, int& hg) {
            e = make_int4(-1, -1, -1, 0);
            hg = 0;
            if (idx >= 0) unit_of(idx, e, hg);
        };
        UnitDesc cur;
        {
            int4 e;
            int hg;
            entry(resolve(claim_next()), e, hg);
            cur = describe_unit<false>(p, e, hg);
        }
        int pending = claim_next();
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int slot = n % kUnitRing;
            if (!mbar_wait(bars + L::B_UEMPTY + slot, ((n / kUnitRing) & 1) ^ 1, abort_flag, p.err)) break;
            if (lane == 0) {
                unit_ring[slot] = cur;
                mbar_arrive(bars + L::B_UFULL + slot);
            }
            if (cur.e.x < 0) break;
            // the next unit: its index now, its plan entry in flight, and the claim after it
            const int nidx = resolve(pending);
            int4 ne;
            int nhg;
            entry(nidx, ne, nhg);
            pending = nidx >= 0 ? claim_next() : total;
            const TileInfo ta = tile_info<false>(p, cur, false);
            const TileInfo tb = tile_info<false>(p, cur, true);
            const int nkv = max(ta.nkv, tb.nkv);
            const int32_t* bt = p.block_tables + (size_t)ta.seq * p.max_blocks;
            int cur_blk = load_pieces(bt, ta.kbeg, ta.lk, 0);
            int nxt_blk = nkv > 1 ? load_pieces(bt, ta.kbeg, ta.lk, 1) : kNoPiece;
            // Q tile x of this unit into the next buffer of the Q ring (a buffer frees after
            // the last S of the tile that used it, three tiles earlier)
            auto load_q = [&](int x) -> bool {
                const TileInfo& t = x ? tb : ta;
                if (!t.valid) return true;
                const uint32_t qs = qfill % kQBufs;
                if (!mbar_wait(bars + L::B_QEMPTY + qs, ((qfill / kQBufs) & 1) ^ 1, abort_flag, p.err)) return false;
                uint8_t* qdst = smem + L::Q_OFF + qs * L::TILE_BYTES;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bars + L::B_QFULL + qs, L::TILE_BYTES);
                    for (int r = 0; r < L::REGIONS; ++r)
                        tma_load_3d(qdst + r * L::REGION_BYTES, &q_map, bars + L::B_QFULL + qs, r * 64,
                                    t.head0, t.q0 + t.tok0);
                }
                ++qfill;
                return true;
            };
            // K (kv = 0) or V tile j, whose block pieces lane c holds in blk_lane; a block id out
            // of range is flagged (once, with the K tile) and its piece is not loaded
            auto load_kv = [&](int kv, int j, int blk_lane) -> bool {
                const int slot = fill % kStages;
                if (!mbar_wait(bars + L::B_KVEMPTY + slot, ((fill / kStages) & 1) ^ 1, abort_flag, p.err))
                    return false;
                const bool in_range = blk_lane >= 0 && blk_lane < p.num_blocks;
                if (kv == 0 && blk_lane != kNoPiece && !in_range) flag_error(p.err, NVPA_FLAG_BAD_BLOCK_ID);
                const uint32_t valid_mask = __ballot_sync(0xffffffffu, in_range);
                const uint32_t bytes = (uint32_t)__popc(valid_mask) * (uint32_t)(piece * 128 * L::REGIONS);
                uint8_t* dst = smem + L::STAGE_OFF + slot * L::TILE_BYTES;
                // a piece whose block id is out of range is zero-filled instead of loaded (its
                // keys then score 0 and its values add nothing), so the stage never feeds the
                // MMAs what a previous tile left there
                const uint32_t bad_mask = __ballot_sync(0xffffffffu, blk_lane != kNoPiece && !in_range);
                if (bad_mask != 0) {
                    for (uint32_t m = bad_mask; m != 0; m &= m - 1) {
                        const int c = __ffs(m) - 1;
                        for (int r = 0; r < L::REGIONS; ++r) {
                            uint4* rows = reinterpret_cast<uint4*>(dst + r * L::REGION_BYTES + c * piece * 128);
                            for (int k = lane; k < piece * 8; k += 32) rows[k] = make_uint4(0, 0, 0, 0);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                const CUtensorMap* map = kv ? &v_map : &k_map;
                if (lane == 0) mbar_arrive_expect_tx(bars + L::B_KVFULL + slot, bytes);
                for (uint32_t m = valid_mask; m != 0; m &= m - 1) {
                    const int c = __ffs(m) - 1;
                    const int blk = __shfl_sync(0xffffffffu, blk_lane, c);
                    if (lane == 0) {
                        const int kc = ta.kbeg + j * kKV + c * piece;
                        const int z = blk * p.block_size + (kc & (p.block_size - 1));
                        for (int r = 0; r < L::REGIONS; ++r)
                            tma_load_3d(dst + r * L::REGION_BYTES + c * piece * 128, map, bars + L::B_KVFULL + slot,
                                        r * 64, ta.hk, z);
                    }
                }
                ++fill;
                return true;
            };
            // K_0 first (its ring slot frees early), then Q_A, V_0, Q_B, then K_j, V_j.  A Q
            // buffer held the tile three Q loads back: with two tiles per unit, Q_A reuses
            // tile B's of the unit before last (long done) and Q_B tile A's of the previous
            // unit (free once that tile's last S completes)
            if (nkv > 0) ok = load_kv(0, 0, cur_blk);
            if (ok) ok = load_q(0);
            if (ok && nkv > 0) ok = load_kv(1, 0, cur_blk);
            if (ok) ok = load_q(1);
            // the lengths of the next unit's sequence: these loads overlap this unit's waits
            const UnitDesc nxt = describe_unit<false>(p, ne, nhg);
            for (int j = 1; j < nkv && ok; ++j) {
                cur_blk = nxt_blk;
                nxt_blk = j + 1 < nkv ? load_pieces(bt, ta.kbeg, ta.lk, j + 1) : kNoPiece;
                ok = load_kv(0, j, cur_blk);
                if (ok) ok = load_kv(1, j, cur_blk);
            }
            cur = nxt;
        }
        // let every copy this warp started land before the CTA can exit
        if (lane == 0) {
            for (uint32_t s = 0; s < (uint32_t)kStages; ++s) {
                if (fill <= s) continue;
                const uint32_t last = fill - 1 - (fill - 1 - s) % kStages;   // last fill of slot s
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(bars + L::B_KVFULL + s, (last / kStages) & 1) &&
                       global_ns() - t0 < 100000000ull) {
                }
            }
            for (uint32_t q = 0; q < (uint32_t)kQBufs; ++q) {
                if (qfill <= q) continue;
                const uint32_t last = qfill - 1 - (qfill - 1 - q) % kQBufs;
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(bars + L::B_QFULL + q, (last / kQBufs) & 1) && global_ns() - t0 < 100000000ull) {
                }
            }
        }
      } else if (warp == 1) {
        // ============================ MMA issuer ============================
        // Per unit: S_A0, S_B0, then for each key tile j: O_A += P_Aj V_j, S_A(j+1),
        // O_B += P_Bj V_j, S_B(j+1).  Tile A's softmax of key tile j+1 thus overlaps tile
        // B's P V and S MMAs, and the other way round.  K_j's ring slot is released after
        // the last S that reads it, V_j's after the last P V.
        // a negative softmax scale is applied as S = -Q K^T (the descriptor's negate-A bit),
        // so the softmax always multiplies by a positive factor
        const uint32_t IDESC_QK = idesc_bf16_f32(kQ, kKV, false) | (p.negate_qk ? (1u << 13) : 0u);
        constexpr uint32_t IDESC_PV = idesc_bf16_f32(kQ, D, true);
        uint32_t fbase = 0;                    // ring fill index of this unit's K_0
        uint32_t qcons = 0;                    // Q tiles consumed (ring position)
        uint32_t puse[2] = {0, 0};             // P_j waits per tile
        int units[2] = {0, 0};                 // units in which the tile had work
        bool ok = true;
        // Operand descriptors: one low half per buffer (Q tiles and ring stage 0, K-major for
        // S, MN-major for V), offsets added per MMA; every operand of the MMA instructions
        // is derived from warp-uniform values only, so issuing one costs a few instructions.
        constexpr uint32_t DESC_HI = sdesc_sw128_hi(1024);
        constexpr uint32_t TILE16 = L::TILE_BYTES >> 4, REGION16 = L::REGION_BYTES >> 4;
        const uint32_t q_lo = sdesc_sw128_lo(sbase + L::Q_OFF, 16);
        const uint32_t k_lo = sdesc_sw128_lo(sbase + L::STAGE_OFF, 16);
        const uint32_t v_lo = sdesc_sw128_lo(sbase + L::STAGE_OFF, L::REGION_BYTES);
        auto issue_qk = [&](int x, int kslot, uint32_t qs) {
            const uint32_t a = q_lo + qs * TILE16, b = k_lo + (uint32_t)kslot * TILE16;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t o = (kk / 4) * REGION16 + (kk % 4) * 2;   // 64-column region, 32 bytes of K
                umma_ss(tmem + x * 256, sdesc_join(a + o, DESC_HI), sdesc_join(b + o, DESC_HI), IDESC_QK,
                        kk > 0 ? 1u : 0u);
            }
            umma_commit(bars + L::B_SFULL + x);
        };
        auto issue_pv = [&](int x, int vslot, bool accumulate) {
            const uint32_t b = v_lo + (uint32_t)vslot * TILE16;
#pragma unroll
            for (int kk = 0; kk < kKV / 16; ++kk)   // 16 keys = 16 rows of 128 bytes per MMA
                umma_ts(tmem + x * 256 + kKV, tmem + x * 256 + kk * 8, sdesc_join(b + kk * 128, DESC_HI), IDESC_PV,
                        (accumulate || kk > 0) ? 1u : 0u);
            umma_commit(bars + L::B_ODONE + x);
        };
        for (int n = 0; ok; ++n) {
            const UnitDesc u = claim(n);
            if (__shfl_sync(0xffffffffu, u.e.x, 0) < 0) break;
            const TileInfo ta = tile_info<false>(p, u, false);
            const TileInfo tb = tile_info<false>(p, u, true);
            // the ring positions follow from these counts: broadcast them (see tmem above)
            const int nk[2] = {__shfl_sync(0xffffffffu, ta.nkv, 0), __shfl_sync(0xffffffffu, tb.nkv, 0)};
            const bool val[2] = {__shfl_sync(0xffffffffu, (int)ta.valid, 0) != 0,
                                 __shfl_sync(0xffffffffu, (int)tb.valid, 0) != 0};
            const int lk = __shfl_sync(0xffffffffu, ta.lk, 0);
            const int nkv = max(nk[0], nk[1]);
            // S of key tile 0: tile A as soon as Q_A and K_0 are in, then tile B
            if (nkv > 0 && !mbar_wait(bars + L::B_KVFULL + fbase % kStages, (fbase / kStages) & 1, abort_flag, p.err))
                break;
            uint32_t qsl[2] = {0, 0};
            for (int x = 0; x < 2 && ok; ++x) {
                if (!val[x]) continue;
                qsl[x] = qcons % kQBufs;
                if (!mbar_wait(bars + L::B_QFULL + qsl[x], (qcons / kQBufs) & 1, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                ++qcons;
                tc_fence_after();
                if (lane == 0) {
                    if (nk[x] > 0) issue_qk(x, fbase % kStages, qsl[x]);
                    if (nk[x] <= 1) umma_commit(bars + L::B_QEMPTY + qsl[x]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (nkv > 0 && lane == 0) umma_commit(bars + L::B_KVEMPTY + fbase % kStages);
            __syncwarp();
            for (int j = 0; j < nkv && ok; ++j) {
                const uint32_t fv = fbase + 2 * (uint32_t)j + 1, fk = fv + 1;
                const int vslot = fv % kStages, kslot = fk % kStages;
                if (!mbar_wait(bars + L::B_KVFULL + vslot, (fv / kStages) & 1, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                const int valid = min(kKV, lk - j * kKV);
                if (valid < kKV) {
                    // zero the V rows past the sequence (stale cache rows, or never loaded)
                    uint8_t* vt = smem + L::STAGE_OFF + vslot * L::TILE_BYTES;
                    for (int r = 0; r < L::REGIONS; ++r) {
                        uint4* rowp = reinterpret_cast<uint4*>(vt + r * L::REGION_BYTES + valid * 128);
                        const int n16 = (kKV - valid) * 8;
                        for (int k = lane; k < n16; k += 32) rowp[k] = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                bool k_next = false;
                for (int x = 0; x < 2; ++x) {
                    if (j >= nk[x]) continue;
                    if (!mbar_wait(bars + L::B_PFULL + x, puse[x] & 1, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    ++puse[x];
                    if (j == 0 && units[x] > 0 &&
                        !mbar_wait(bars + L::B_OFREE + x, (units[x] - 1) & 1, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // P V first: it does not need K_{j+1}, which may still be in flight
                    if (lane == 0) {
                        issue_pv(x, vslot, j > 0);
                        if (j == nk[x] - 1) umma_commit(bars + L::B_OFINAL + x);
                    }
                    __syncwarp();
                    if (j + 1 < nk[x]) {
                        if (!k_next) {
                            if (!mbar_wait(bars + L::B_KVFULL + kslot, (fk / kStages) & 1, abort_flag, p.err)) {
                                ok = false;
                                break;
                            }
                            k_next = true;
                            tc_fence_after();
                        }
                        if (lane == 0) {
                            issue_qk(x, kslot, qsl[x]);
                            if (j + 2 == nk[x]) umma_commit(bars + L::B_QEMPTY + qsl[x]);
                        }
                        __syncwarp();
                    }
                }
                if (!ok) break;
                if (lane == 0) {
                    umma_commit(bars + L::B_KVEMPTY + vslot);
                    if (k_next) umma_commit(bars + L::B_KVEMPTY + kslot);
                }
                __syncwarp();
            }
            fbase += 2 * (uint32_t)nkv;
            for (int x = 0; x < 2; ++x) {
                if (nk[x] > 0) ++units[x];
            }
        }
        // every MMA this thread issued completes before TMEM is released
        if (lane == 0) umma_commit(bars + L::B_DRAIN);
        __syncwarp();
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(bars + L::B_DRAIN, 0) && global_ns() - t0 < 100000000ull) {
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // ============================ softmax warps ============================
        // warps 4..7: tile A, warps 8..11: tile B
        const int x = (warp - 4) >> 2;
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;            // row of the tile: token r / P, head r % P
        const int rtok = r >> p.pack_shift;
        const int rhead = r & (p.pack - 1);
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_col = tmem + lane_base + x * 256;
        const uint32_t o_col = s_col + kKV;
        uint64_t* b_sfull = bars + L::B_SFULL + x;
        uint64_t* b_pfull = bars + L::B_PFULL + x;
        uint64_t* b_odone = bars + L::B_ODONE + x;
        uint64_t* b_ofinal = bars + L::B_OFINAL + x;
        uint64_t* b_ofree = bars + L::B_OFREE + x;
        uint32_t s_use = 0;
        int tcount = 0;
        uint32_t pv_before = 0;                       // PVs issued for this tile slot before
        for (int n = 0;; ++n) {
            const UnitDesc u = claim(n);
            if (u.e.x < 0) break;
            const TileInfo t = tile_info<false>(p, u, x == 1);
            if (t.nkv == 0) continue;
            const int pos = t.lk - t.lq + t.tok0 + rtok;           // absolute position of this row
            const int lim = p.causal ? min(t.lk, pos + 1) : t.lk;  // keys 0 .. lim-1 visible
            const int lim_min = __reduce_min_sync(0xffffffffu, lim);
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j < t.nkv; ++j) {
                if (!mbar_wait(b_sfull, s_use & 1, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                ++s_use;
                tc_fence_after();
                const int key0 = j * kKV;
                const bool open = key0 + kKV <= lim_min;          // no mask anywhere in the warp
                // the whole S_j row in registers: four loads, one wait
                uint32_t sv[kKV];
#pragma unroll
                for (int c = 0; c < kKV / 32; ++c)
                    tmem_ld32(s_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv + c * 32));
                tmem_wait_ld();
                // keys the row does not see at -inf (diagonal tiles only), then the row's
                // largest value in log2 units (raw scores times a positive factor)
                if (!open) mask_row<kKV>(sv, key0, lim);
                const float mt = row_max<kKV>(sv) * p.scale_log2;
                const bool over = mt > m + kRescaleSlack;
                const bool rescale = __any_sync(0xffffffffu, over);
                float alpha = 1.f;
                if (rescale) {
                    const float m_new = over ? mt : m;
                    alpha = over ? (m == -INFINITY ? 0.f : fast_exp2(m - m_new)) : 1.f;
                    l *= alpha;
                    m = m_new;
                }
                // P_j = exp2(s * scale - m) as bf16 pairs over the first kKV/2 columns of S_j.
                // A row with no visible key yet (m = -inf) gets exp2(-inf) = 0 through its
                // offset.
                l += exp_row<kKV>(sv, s_col, p.scale_log2, m > -INFINITY ? -m : -INFINITY);
                if (rescale && j > 0) {
                    // O holds P_0..P_{j-1} V (all complete once S_j is): rescale it before
                    // P_j is released to the MMA
                    if (!mbar_wait(b_odone, (pv_before + j - 1) & 1, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(o_col + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                        tmem_st32(o_col + c * 32, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_pfull);
            }
            if (!ok) break;
            if (!mbar_wait(b_ofinal, tcount & 1, abort_flag, p.err)) break;
            tc_fence_after();
            const bool row_ok = rtok < t.ntok;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const size_t orow = (size_t)(t.q0 + t.tok0 + rtok) * p.hq + t.head0 + rhead;
            uint4* dst = reinterpret_cast<uint4*>(p.out + orow * D);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(o_col + c * 32, o);
                tmem_wait_ld();
                if (c == D / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b_ofree);
                }
                if (row_ok && p.out_v8) {
                    // 32-byte stores: each fills a whole sector of the output row (a warp's
                    // 32 rows are 32 different lines, so the count of store instructions is
                    // what the epilogue's time goes by)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint32_t w[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            w[k] = pack_bf16x2(__uint_as_float(o[16 * q + 2 * k]) * inv,
                                               __uint_as_float(o[16 * q + 2 * k + 1]) * inv);
                        st_global_v8(dst + c * 4 + 2 * q, w);
                    }
                } else if (row_ok) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
                        dst[c * 4 + q] = w;
                    }
                }
            }
            if (row_ok && p.lse_out != nullptr) p.lse_out[orow] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
            pv_before += (uint32_t)t.nkv;
            ++tcount;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------------------------
// the shared-prefix tiles of the decode step: one query tile per CTA at a time, two S
// buffers and Q in TMEM
// ------------------------------------------------------------------------------------
// A group of sequences that share a cached prefix ("Nano-vLLM part 1" section 4.2) attends
// the prefix once: the query rows of a tile are the members' decode queries (128 / P
// members times the P query heads of one KV head), the keys one partition of the prefix,
// with no mask but the prefix's length, and each member's result goes to that
// partition's slot of its split-KV partials for the decode combine.
//
// Work unit: ONE query tile.  A group has few tiles and each tile few key tiles, so there
// is no second tile to overlap with; instead S = Q K_j^T alternates between two TMEM
// buffers, so S_{j+1} is computed while the softmax still works on S_j: the MMA warp
// issues O += P_j V_j and S_{j+2} as soon as P_j is ready, and the next softmax finds its
// S waiting.  Q is kept in TMEM (the A operand of S = Q K^T, like P for O += P V), so the
// S MMAs read only K from shared memory.  TMEM columns: S buffers [0, 128) and
// [128, 256), O [256, 256 + D), Q [384, 384 + D / 2) (bf16 pairs).  The two query tiles
// of a plan entry are consecutive units (claimed by different CTAs at about the same
// time, so their K/V tiles are read from DRAM once).  Warp roles:
//   warp 0      TMA producer: K_0, K_1, V_0, K_2, V_1, ... (the order the MMAs read them)
//               into a 6-stage K/V ring;
//   warp 1      MMA issuer: S_0, S_1, then O += P_j V_j, S_{j+2} for each key tile j;
//   warps 2, 3  idle (warpgroup 0's register share goes to the softmax);
//   warps 4..11 softmax, two warps per row: warps 4..7 keys 0..63 of each key tile and O
//               columns [0, D/2), warps 8..11 keys 64..127 and O columns [D/2, D); the two
//               warps of a row exchange its largest score and, at the end, its sum through
//               shared memory; each warp also stores its half of the row's Q into TMEM.
constexpr int kStages2 = 6;
// Units (query tiles) per CTA below which the prefix grid leaves CTAs idle: with about
// three units each the tiles of a decode step's shared prefixes take a fifth of the SMs or
// less, and the split-KV worker, which runs beside them, streams on the rest.
constexpr int kPrefixUnitsPerCta = 3;
constexpr uint32_t kS2Cols = 128, kO2Col = 256, kQ2Col = 384;

template <int D>
struct PrefixLayout {
    static constexpr int REGIONS = D / 64;
    static constexpr int REGION_BYTES = 128 * 128;
    static constexpr int TILE_BYTES = REGIONS * REGION_BYTES;
    static constexpr int STAGE_OFF = 0;
    static constexpr int BAR_OFF = kStages2 * TILE_BYTES;
    static constexpr int B_KVFULL = 0, B_KVEMPTY = kStages2, B_SFULL = 2 * kStages2, B_PFULL = B_SFULL + 2;
    static constexpr int B_ODONE = B_PFULL + 2, B_OFINAL = B_ODONE + 1, B_OFREE = B_OFINAL + 1;
    static constexpr int B_QREADY = B_OFREE + 1, B_DRAIN = B_QREADY + 1, B_XCH = B_DRAIN + 1;
    static constexpr int B_UFULL = B_XCH + 4, B_UEMPTY = B_UFULL + kUnitRing;
    static constexpr int NBARS = B_UEMPTY + kUnitRing;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int RING_OFF = (MISC_OFF + 16 + 15) / 16 * 16;
    static constexpr int XCH_OFF = RING_OFF + 32 * kUnitRing;   // [2 slots][2 halves][128 rows] floats
    static constexpr int BYTES = XCH_OFF + 2 * 2 * kQ * 4;
    static constexpr int ALLOC = BYTES + 1024;
};
static_assert(PrefixLayout<128>::ALLOC <= 227 * 1024, "shared memory per CTA");

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
prefix_tiles_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                  const __grid_constant__ CUtensorMap v_map, const PrefillParams p) {
    using L = PrefixLayout<D>;
    (void)q_map;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
    UnitDesc* unit_ring = reinterpret_cast<UnitDesc*>(smem + L::RING_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(bars + L::B_SFULL + b, 1);
            mbar_init(bars + L::B_PFULL + b, 8);
        }
        mbar_init(bars + L::B_ODONE, 1);
        mbar_init(bars + L::B_OFINAL, 1);
        mbar_init(bars + L::B_OFREE, 8);
        mbar_init(bars + L::B_QREADY, 8);
        mbar_init(bars + L::B_DRAIN, 1);
        for (int q = 0; q < 4; ++q) mbar_init(bars + L::B_XCH + q, 2);
        for (int s = 0; s < kStages2; ++s) {
            mbar_init(bars + L::B_KVFULL + s, 1);
            mbar_init(bars + L::B_KVEMPTY + s, 1);
        }
        for (int i = 0; i < kUnitRing; ++i) {
            mbar_init(bars + L::B_UFULL + i, 1);
            mbar_init(bars + L::B_UEMPTY + i, kUnitReaders);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&k_map);
        tma_prefetch_desc(&v_map);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
    // launched as a programmatic dependent of the decode plan: nothing the plan writes is
    // read before this wait
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // The decode worker may launch once every CTA of this grid is past that wait: it reads
    // the plan's tables without a wait of its own and runs on the SMs this grid leaves free
    // (most CTAs find no tile and exit at once), then waits for this grid at its end.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // one unit per query tile: the two tiles of a plan entry, for every head group
    const int total = __ldcg(p.ntiles) * p.hgroups * 2;
    // Only the first ceil(total / kPrefixUnitsPerCta) CTAs take units (every CTA when there
    // are more units than that per CTA); the others exit at once and leave their SMs to the
    // HBM-bound worker running beside this grid.
    const bool idle_cta = (long long)blockIdx.x * kPrefixUnitsPerCta >= (long long)total;
    auto unit_of = [&](int idx, int4& e, int& hg) {
        hg = idx % p.hgroups;
        const int4 pe = __ldg(p.tiles + idx / (2 * p.hgroups));
        e = make_int4(pe.x, ((idx / p.hgroups) & 1) ? pe.z : pe.y, -1, pe.w);
    };
    auto claim = [&](int n) -> UnitDesc {
        const int slot = n % kUnitRing;
        UnitDesc u;
        if (!mbar_wait(bars + L::B_UFULL + slot, (n / kUnitRing) & 1, abort_flag, p.err)) {
            u.e = make_int4(-2, -1, -1, 0);
            u.hg = u.q0 = u.lq = u.lk = 0;
            return u;
        }
        u = unit_ring[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::B_UEMPTY + slot);
        return u;
    };

    if (warp < 4) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kSmallRegs));
      if (warp == 0) {
        // ============================ TMA producer ============================
        uint32_t fill = 0;
        const int piece = min(p.block_size, kKV);
        constexpr int kNoPiece = INT_MIN;
        auto load_pieces = [&](const int32_t* bt, int kbeg, int lk, int j) {
            const int key0 = j * kKV;
            const int npieces = (min(kKV, lk - key0) + piece - 1) / piece;
            return lane < npieces ? __ldg(bt + ((kbeg + key0 + lane * piece) >> p.block_shift)) : kNoPiece;
        };
        auto claim_next = [&]() -> int {
            return lane == 0 ? (idle_cta ? total : atomicAdd(p.unit_counter, 1)) : 0;
        };
        auto resolve = [&](int pending) -> int {
            const int i = __shfl_sync(0xffffffffu, pending, 0);
            return i < total ? i : -1;
        };
        auto entry = [&](int idx, int4& e, int& hg) {
            e = make_int4(-1, -1, -1, 0);
            hg = 0;
            if (idx >= 0) unit_of(idx, e, hg);
        };
        UnitDesc cur;
        {
            int4 e;
            int hg;
            entry(resolve(claim_next()), e, hg);
            cur = describe_unit<true>(p, e, hg);
        }
        int pending = claim_next();
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int slot = n % kUnitRing;
            if (!mbar_wait(bars + L::B_UEMPTY + slot, ((n / kUnitRing) & 1) ^ 1, abort_flag, p.err)) break;
            if (lane == 0) {
                unit_ring[slot] = cur;
                mbar_arrive(bars + L::B_UFULL + slot);
            }
            if (cur.e.x < 0) break;
            const int nidx = resolve(pending);
            int4 ne;
            int nhg;
            entry(nidx, ne, nhg);
            pending = nidx >= 0 ? claim_next() : total;
            const TileInfo ta = tile_info<true>(p, cur, false);
            const int nkv = ta.nkv;
            // the prefix's blocks are the same in every member's table: read the first member's
            const int32_t* bt = p.block_tables + (size_t)__ldg(p.members + ta.q0) * p.max_blocks;
            // K (kv = 0) or V tile j into the next ring stage; lane c holds piece c's block id
            auto load_kv = [&](int kv, int j, int blk_lane) -> bool {
                const int slot = fill % kStages2;
                if (!mbar_wait(bars + L::B_KVEMPTY + slot, ((fill / kStages2) & 1) ^ 1, abort_flag, p.err))
                    return false;
                const bool in_range = blk_lane >= 0 && blk_lane < p.num_blocks;
                if (kv == 0 && blk_lane != kNoPiece && !in_range) flag_error(p.err, NVPA_FLAG_BAD_BLOCK_ID);
                const uint32_t valid_mask = __ballot_sync(0xffffffffu, in_range);
                const uint32_t bytes = (uint32_t)__popc(valid_mask) * (uint32_t)(piece * 128 * L::REGIONS);
                uint8_t* dst = smem + L::STAGE_OFF + slot * L::TILE_BYTES;
                const uint32_t bad_mask = __ballot_sync(0xffffffffu, blk_lane != kNoPiece && !in_range);
                if (bad_mask != 0) {
                    for (uint32_t m = bad_mask; m != 0; m &= m - 1) {
                        const int c = __ffs(m) - 1;
                        for (int r = 0; r < L::REGIONS; ++r) {
                            uint4* rows = reinterpret_cast<uint4*>(dst + r * L::REGION_BYTES + c * piece * 128);
                            for (int k = lane; k < piece * 8; k += 32) rows[k] = make_uint4(0, 0, 0, 0);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                const CUtensorMap* map = kv ? &v_map : &k_map;
                if (lane == 0) mbar_arrive_expect_tx(bars + L::B_KVFULL + slot, bytes);
                for (uint32_t m = valid_mask; m != 0; m &= m - 1) {
                    const int c = __ffs(m) - 1;
                    const int blk = __shfl_sync(0xffffffffu, blk_lane, c);
                    if (lane == 0) {
                        const int kc = ta.kbeg + j * kKV + c * piece;
                        const int z = blk * p.block_size + (kc & (p.block_size - 1));
                        for (int r = 0; r < L::REGIONS; ++r)
                            tma_load_3d(dst + r * L::REGION_BYTES + c * piece * 128, map, bars + L::B_KVFULL + slot,
                                        r * 64, ta.hk, z);
                    }
                }
                ++fill;
                return true;
            };
            if (nkv > 0) {
                int blk0 = load_pieces(bt, ta.kbeg, ta.lk, 0);
                int blk1 = nkv > 1 ? load_pieces(bt, ta.kbeg, ta.lk, 1) : kNoPiece;
                ok = load_kv(0, 0, blk0);
                for (int j = 0; j < nkv && ok; ++j) {
                    const int blk2 = j + 2 < nkv ? load_pieces(bt, ta.kbeg, ta.lk, j + 2) : kNoPiece;
                    if (j + 1 < nkv) ok = load_kv(0, j + 1, blk1);
                    if (ok) ok = load_kv(1, j, blk0);
                    blk0 = blk1;
                    blk1 = blk2;
                }
            }
            cur = describe_unit<true>(p, ne, nhg);
        }
        if (lane == 0) {
            for (uint32_t s = 0; s < (uint32_t)kStages2; ++s) {
                if (fill <= s) continue;
                const uint32_t last = fill - 1 - (fill - 1 - s) % kStages2;
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(bars + L::B_KVFULL + s, (last / kStages2) & 1) &&
                       global_ns() - t0 < 100000000ull) {
                }
            }
        }
      } else if (warp == 1) {
        // ============================ MMA issuer ============================
        const uint32_t IDESC_S = idesc_bf16_f32(kQ, kKV, false) | (p.negate_qk ? (1u << 13) : 0u);
        constexpr uint32_t IDESC_PV = idesc_bf16_f32(kQ, D, true);
        constexpr uint32_t DESC_HI = sdesc_sw128_hi(1024);
        constexpr uint32_t TILE16 = L::TILE_BYTES >> 4, REGION16 = L::REGION_BYTES >> 4;
        const uint32_t k_lo = sdesc_sw128_lo(sbase + L::STAGE_OFF, 16);
        const uint32_t v_lo = sdesc_sw128_lo(sbase + L::STAGE_OFF, L::REGION_BYTES);
        uint32_t fill = 0;     // ring entries consumed, in the producer's order
        uint32_t g = 0;        // key tiles so far (S buffer of key tile j: (g + j) & 1)
        uint32_t qcount = 0;   // units with work
        bool ok = true;
        auto take = [&](uint32_t& slot) -> bool {
            slot = fill % kStages2;
            const bool r = mbar_wait(bars + L::B_KVFULL + slot, (fill / kStages2) & 1, abort_flag, p.err);
            ++fill;
            return r;
        };
        auto issue_s = [&](uint32_t buf, uint32_t kslot) {
            const uint32_t b = k_lo + kslot * TILE16;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t o = (kk / 4) * REGION16 + (kk % 4) * 2;
                umma_ts(tmem + buf * kS2Cols, tmem + kQ2Col + kk * 8, sdesc_join(b + o, DESC_HI), IDESC_S,
                        kk > 0 ? 1u : 0u);
            }
            umma_commit(bars + L::B_SFULL + buf);
            umma_commit(bars + L::B_KVEMPTY + kslot);
        };
        auto issue_pv = [&](uint32_t buf, uint32_t vslot, bool accumulate) {
            const uint32_t b = v_lo + vslot * TILE16;
#pragma unroll
            for (int kk = 0; kk < kKV / 16; ++kk)
                umma_ts(tmem + kO2Col, tmem + buf * kS2Cols + kk * 8, sdesc_join(b + kk * 128, DESC_HI), IDESC_PV,
                        (accumulate || kk > 0) ? 1u : 0u);
            umma_commit(bars + L::B_ODONE);
            umma_commit(bars + L::B_KVEMPTY + vslot);
        };
        for (int n = 0; ok; ++n) {
            const UnitDesc u = claim(n);
            if (__shfl_sync(0xffffffffu, u.e.x, 0) < 0) break;
            const TileInfo t = tile_info<true>(p, u, false);
            const int nk = __shfl_sync(0xffffffffu, t.nkv, 0);
            const int lk = __shfl_sync(0xffffffffu, t.lk, 0);
            if (nk == 0) continue;
            // this unit's Q is in TMEM
            if (!mbar_wait(bars + L::B_QREADY, qcount & 1, abort_flag, p.err)) break;
            uint32_t slot;
            if (!take(slot)) break;
            tc_fence_after();
            if (lane == 0) issue_s(g & 1, slot);
            __syncwarp();
            if (nk > 1) {
                if (!take(slot)) break;
                tc_fence_after();
                if (lane == 0) issue_s((g + 1) & 1, slot);
                __syncwarp();
            }
            for (int j = 0; j < nk && ok; ++j) {
                const uint32_t b = (g + j) & 1;
                if (!mbar_wait(bars + L::B_PFULL + b, ((g + j) >> 1) & 1, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                if (j == 0 && qcount > 0 && !mbar_wait(bars + L::B_OFREE, (qcount - 1) & 1, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                uint32_t vslot;
                if (!take(vslot)) {
                    ok = false;
                    break;
                }
                const int valid = min(kKV, lk - j * kKV);
                if (valid < kKV) {
                    // zero the V rows past the sequence (stale cache rows, or never loaded)
                    uint8_t* vt = smem + L::STAGE_OFF + vslot * L::TILE_BYTES;
                    for (int r = 0; r < L::REGIONS; ++r) {
                        uint4* rowp = reinterpret_cast<uint4*>(vt + r * L::REGION_BYTES + valid * 128);
                        const int n16 = (kKV - valid) * 8;
                        for (int k = lane; k < n16; k += 32) rowp[k] = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                tc_fence_after();
                if (lane == 0) {
                    issue_pv(b, vslot, j > 0);
                    if (j == nk - 1) umma_commit(bars + L::B_OFINAL);
                }
                __syncwarp();
                if (j + 2 < nk) {
                    // S_{j+2} into the buffer whose P_j the P V just issued reads first
                    uint32_t kslot;
                    if (!take(kslot)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) issue_s(b, kslot);
                    __syncwarp();
                }
            }
            g += (uint32_t)nk;
            ++qcount;
        }
        if (lane == 0) umma_commit(bars + L::B_DRAIN);
        __syncwarp();
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(bars + L::B_DRAIN, 0) && global_ns() - t0 < 100000000ull) {
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // ============================ softmax warps ============================
        constexpr int NC = kKV / 2;                    // S columns of this warp
        constexpr int DC = D / 2;                      // O columns of this warp
        const int h = (warp - 4) >> 2;                 // column half
        const int quarter = warp & 3;                  // TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;
        const int rtok = r >> p.pack_shift;
        const int rhead = r & (p.pack - 1);
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_base = tmem + lane_base;
        const uint32_t o_col = tmem + lane_base + kO2Col + h * DC;
        const uint32_t q_col = tmem + lane_base + kQ2Col + h * (D / 4);
        float* xch = reinterpret_cast<float*>(smem + L::XCH_OFF);
        uint64_t* b_xch = bars + L::B_XCH + quarter;
        uint32_t x_use = 0;
        // Publish v, wait for the partner warp of the row, return its value.  Two slots by
        // use parity: a warp can be one exchange ahead of its partner's read, never two.
        auto exchange = [&](float v, float& other) -> bool {
            const int sl = (int)(x_use & 1);
            xch[(sl * 2 + h) * kQ + r] = v;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_xch);
            if (!mbar_wait(b_xch, x_use & 1, abort_flag, p.err)) return false;
            ++x_use;
            tc_fence_after();
            other = xch[(sl * 2 + (h ^ 1)) * kQ + r];
            return true;
        };
        uint32_t g = 0;
        int tcount = 0;
        uint32_t pv_before = 0;
        for (int n = 0;; ++n) {
            const UnitDesc u = claim(n);
            if (u.e.x < 0) break;
            const TileInfo t = tile_info<true>(p, u, false);
            if (t.nkv == 0) continue;
            const bool row_ok = rtok < t.ntok;
            // this warp's half of the row's Q into TMEM (zeros for rows past the tile); the
            // previous unit's S MMAs, which read Q, have all completed (each was waited for)
            {
                // row r: member tok0 + r / P of the group, query head head0 + r % P
                const uint16_t* src = nullptr;
                if (row_ok) {
                    const int b = __ldg(p.members + t.q0 + t.tok0 + rtok);
                    src = p.q_rows + ((size_t)b * p.hq + t.head0 + rhead) * D;
                }
                uint32_t qw[D / 4];   // D / 2 bf16: D / 16 loads of 16 bytes
#pragma unroll
                for (int c = 0; c < D / 16; ++c) {
                    const uint4 v = src != nullptr ? __ldg(reinterpret_cast<const uint4*>(src + h * DC) + c)
                                                   : make_uint4(0, 0, 0, 0);
                    qw[4 * c + 0] = v.x;
                    qw[4 * c + 1] = v.y;
                    qw[4 * c + 2] = v.z;
                    qw[4 * c + 3] = v.w;
                }
                if constexpr (D / 4 == 32) {
                    tmem_st32(q_col, qw);
                } else {
                    tmem_st16(q_col, qw);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + L::B_QREADY);
            }
            // every member sees all of the prefix: only keys past its length are masked
            const int lim = t.lk;
            const int lim_min = lim;
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j < t.nkv; ++j) {
                const uint32_t b = (g + j) & 1;
                if (!mbar_wait(bars + L::B_SFULL + b, ((g + j) >> 1) & 1, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int key0 = j * kKV;
                const bool open = key0 + kKV <= lim_min;
                const uint32_t s_col = s_base + b * kS2Cols;
                uint32_t sv[NC];
#pragma unroll
                for (int c = 0; c < NC / 32; ++c)
                    tmem_ld32(s_col + h * NC + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv + c * 32));
                tmem_wait_ld();
                if (!open) mask_row<NC>(sv, key0 + h * NC, lim);
                float mt = row_max<NC>(sv) * p.scale_log2;
                {
                    float mo;
                    if (!exchange(mt, mo)) {
                        ok = false;
                        break;
                    }
                    mt = fmaxf(mt, mo);
                }
                const bool over = mt > m + kRescaleSlack;
                const bool rescale = __any_sync(0xffffffffu, over);
                float alpha = 1.f;
                if (rescale) {
                    const float m_new = over ? mt : m;
                    alpha = over ? (m == -INFINITY ? 0.f : fast_exp2(m - m_new)) : 1.f;
                    l *= alpha;
                    m = m_new;
                }
                l += exp_row<NC>(sv, s_col + h * (NC / 2), p.scale_log2, m > -INFINITY ? -m : -INFINITY);
                if (rescale && j > 0) {
                    // O holds P_0..P_{j-1} V: wait for the last of those, then rescale this
                    // warp's columns before P_j is released
                    if (!mbar_wait(bars + L::B_ODONE, (pv_before + j - 1) & 1, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < DC / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(o_col + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                        tmem_st32(o_col + c * 32, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + L::B_PFULL + b);
            }
            if (!ok) break;
            if (!mbar_wait(bars + L::B_OFINAL, tcount & 1, abort_flag, p.err)) break;
            tc_fence_after();
            {
                float lo;
                if (!exchange(l, lo)) break;
                l += lo;
            }
            const float inv = l > 0.f ? 1.f / l : 0.f;
            // partition `chunk` of the prefix goes to slot `chunk` of each member's partials
            const int b = row_ok ? __ldg(p.members + t.q0 + t.tok0 + rtok) : 0;
            const size_t orow = ((size_t)b * p.hq + t.head0 + rhead) * p.s_max + t.chunk;
            float* pdst = p.o_part + orow * D;
#pragma unroll
            for (int c = 0; c < DC / 32; ++c) {
                const int cg = h * (DC / 32) + c;   // 32-column chunk of the O row
                uint32_t o[32];
                tmem_ld32(o_col + c * 32, o);
                tmem_wait_ld();
                if (c == DC / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars + L::B_OFREE);
                }
                if (row_ok) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        __stcg(reinterpret_cast<float4*>(pdst + cg * 32 + 4 * q),
                               make_float4(__uint_as_float(o[4 * q + 0]) * inv, __uint_as_float(o[4 * q + 1]) * inv,
                                           __uint_as_float(o[4 * q + 2]) * inv, __uint_as_float(o[4 * q + 3]) * inv));
                }
            }
            if (row_ok && h == 0) __stcg(p.lse_part + orow, l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY);
            pv_before += (uint32_t)t.nkv;
            g += (uint32_t)t.nkv;
            ++tcount;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
// The softmax scale in log2 units.  The kernel multiplies raw scores by a positive factor
// (one packed FMA together with the max subtraction); a negative scale flips the sign of
// Q K^T in the MMA instead, and a zero scale becomes the smallest normal float (every score
// then rounds to 0, the weights are uniform, and a masked -inf score still weighs 0).
void set_scale(PrefillParams& p, float scale) {
    const float a = std::fabs(scale) * kLog2e;
    p.scale_log2 = a > 0.f ? a : FLT_MIN;
    p.negate_qk = scale < 0.f;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 3-D view (dim, heads, rows) of a [rows, heads, dim] bf16 array; box = 64 x box_heads x
// box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int dim, int heads, long long rows, int box_heads,
              int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t gdim[3] = {(cuuint64_t)dim, (cuuint64_t)heads, (cuuint64_t)rows};
    const cuuint64_t gstride[2] = {(cuuint64_t)dim * 2, (cuuint64_t)dim * heads * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
    const cuuint32_t estride[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The varlen prefill runs pairs of query tiles (prefill_tcgen05_kernel); the shared-prefix
// tiles of the decode step run one query tile at a time with two S buffers
// (prefix_tiles_kernel).  Both take the same arguments.
template <int D, bool PREFIX>
constexpr auto prefill_kernel_fn() {
    if constexpr (PREFIX) return prefix_tiles_kernel<D>;
    else return prefill_tcgen05_kernel<D>;
}
template <int D, bool PREFIX>
constexpr int prefill_smem() { return PREFIX ? PrefixLayout<D>::ALLOC : Layout<D>::ALLOC; }

template <int D, bool PREFIX>
cudaError_t launch_prefill(const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm,
                           const PrefillParams& p, int grid, cudaStream_t stream, bool pdl = PREFIX) {
    static std::once_flag once[64];
    static int launch_regs[64];
    int dev = 0;
    cudaGetDevice(&dev);
    std::call_once(once[dev & 63], [dev] {
        cudaFuncSetAttribute(prefill_kernel_fn<D, PREFIX>(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             prefill_smem<D, PREFIX>());
        cudaFuncAttributes fa{};
        launch_regs[dev & 63] =
            cudaFuncGetAttributes(&fa, prefill_kernel_fn<D, PREFIX>()) == cudaSuccess ? fa.numRegs : 0;
    });
    // The warpgroups' setmaxnreg shares add up to kLaunchRegs per thread: with fewer registers
    // at launch the raising warpgroups could never get their share, so do not launch.
    if (launch_regs[dev & 63] != kLaunchRegs) {
        set_error("prefill kernel compiled with %d registers per thread, %d expected", launch_regs[dev & 63],
                  kLaunchRegs);
        return cudaErrorInvalidConfiguration;
    }
    if (!pdl) {
        auto kern = prefill_kernel_fn<D, PREFIX>();
        kern<<<grid, kThreads, prefill_smem<D, PREFIX>(), stream>>>(qm, km, vm, p);
        return cudaGetLastError();
    } else {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = prefill_smem<D, PREFIX>();
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, prefill_kernel_fn<D, PREFIX>(), qm, km, vm, p);
    }
}

}  // namespace

int attention_tile_pack(int hq, int hkv) {
    const int group = hq / hkv;
    return (group & (group - 1)) == 0 ? std::min(group, kQ / kMinTokensPerTile) : 1;
}

cudaError_t launch_decode_prefix_tcgen05(const DecodePrefixArgs& a, cudaStream_t stream) {
    const int pack = attention_tile_pack(a.hq, a.hkv);
    CUtensorMap km, vm;
    const int box_kv = std::min(a.block_size, kKV);
    if (!make_map(&km, a.k_cache, a.head_dim, a.hkv, (long long)a.num_blocks * a.block_size, 1, box_kv) ||
        !make_map(&vm, a.v_cache, a.head_dim, a.hkv, (long long)a.num_blocks * a.block_size, 1, box_kv)) {
        set_error("cuTensorMapEncodeTiled failed (driver entry point missing or bad layout)");
        return cudaErrorInvalidValue;
    }
    PrefillParams p{};
    p.block_tables = a.block_tables;
    p.err = a.err_flag;
    p.tiles = a.tiles;
    p.ntiles = a.ntiles;
    p.unit_counter = a.unit_counter;
    p.q_rows = static_cast<const uint16_t*>(a.q);
    p.members = a.members;
    p.group_start = a.group_start;
    p.group_len = a.group_len;
    p.o_part = a.o_part;
    p.lse_part = a.lse_part;
    p.s_max = a.s_max;
    p.pchunk = a.pchunk;
    p.batch = a.batch;
    p.hq = a.hq;
    p.hkv = a.hkv;
    p.group = a.hq / a.hkv;
    p.pack = pack;
    p.pack_shift = __builtin_ctz((unsigned)pack);
    p.tq = kQ / pack;
    p.hgroups = a.hq / pack;
    p.max_blocks = a.max_blocks_per_seq;
    p.num_blocks = a.num_blocks;
    p.block_size = a.block_size;
    p.block_shift = __builtin_ctz((unsigned)a.block_size);
    set_scale(p, a.scale);
    const long long units = std::max(1LL, a.max_entries) * p.hgroups * 2;   // single-tile units
    const long long cap = a.max_ctas > 0 ? a.max_ctas : (long long)device_sm_count();
    const int grid = (int)std::max(1LL, std::min<long long>(cap, units));
    // the query map is not read in this mode (rows are gathered); any valid map will do
    return a.head_dim == 128 ? launch_prefill<128, true>(km, km, vm, p, grid, stream, a.pdl)
                             : launch_prefill<64, true>(km, km, vm, p, grid, stream, a.pdl);
}

size_t prefill_workspace_bytes(int batch, int total_q) {
    const size_t entries = (size_t)std::max(0, batch) +
                           ((size_t)std::max(0, total_q) + kMinTokensPerTile - 1) / kMinTokensPerTile;
    return 256 + ((entries * sizeof(int4) + 255) & ~size_t(255));
}

nvpa_status_t run_varlen_prefill_tcgen05(const PrefillCall& c, void* workspace, size_t workspace_bytes,
                                         cudaStream_t stream) {
    const size_t need = prefill_workspace_bytes(c.batch, c.total_q);
    if (workspace_bytes < need) {
        set_error("workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
        return NVPA_ERR_WORKSPACE_TOO_SMALL;
    }
    // query heads packed per 128-row tile: the group size when it is a power of two <= 8
    const int group = c.hq / c.hkv;
    const int pack = attention_tile_pack(c.hq, c.hkv);
    CUtensorMap qm, km, vm;
    const int box_kv = std::min(c.block_size, kKV);
    if (!make_map(&qm, c.q, c.head_dim, c.hq, c.total_q, pack, kQ / pack) ||
        !make_map(&km, c.k_cache, c.head_dim, c.hkv, (long long)c.num_blocks * c.block_size, 1, box_kv) ||
        !make_map(&vm, c.v_cache, c.head_dim, c.hkv, (long long)c.num_blocks * c.block_size, 1, box_kv)) {
        set_error("cuTensorMapEncodeTiled failed (driver entry point missing or bad layout)");
        return NVPA_ERR_CUDA;
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    PrefillParams p{};
    p.block_tables = c.block_tables;
    p.cu_q = c.cu_seqlens_q;
    p.cu_k = c.cu_seqlens_k;
    p.out = static_cast<uint16_t*>(c.out);
    p.q_rows = static_cast<const uint16_t*>(c.q);   // the query rows, read directly by one kernel form
    p.lse_out = c.lse_out;
    p.err = c.err_flag;
    p.ntiles = reinterpret_cast<int32_t*>(ws);
    p.unit_counter = reinterpret_cast<int32_t*>(ws) + 1;
    p.tiles = reinterpret_cast<const int4*>(ws + 256);
    p.batch = c.batch;
    p.total_q = c.total_q;
    p.hq = c.hq;
    p.hkv = c.hkv;
    p.group = group;
    p.pack = pack;
    p.pack_shift = __builtin_ctz((unsigned)pack);
    p.tq = kQ / pack;
    p.hgroups = c.hq / pack;
    p.max_blocks = c.max_blocks_per_seq;
    p.num_blocks = c.num_blocks;
    p.block_size = c.block_size;
    p.block_shift = __builtin_ctz((unsigned)c.block_size);
    p.max_q = c.max_seqlen_q;
    p.max_k = c.max_seqlen_k;
    p.causal = c.causal;
    set_scale(p, c.scale);
    p.out_v8 = (reinterpret_cast<uintptr_t>(c.out) & 31u) == 0;

    prefill_plan_kernel<<<1, 1024, 0, stream>>>(p, reinterpret_cast<int4*>(ws + 256), reinterpret_cast<int32_t*>(ws));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_failure(e, "prefill plan launch");
    count_launches(1);
    // one pair per query tile at most, plus one per sequence for a ragged last tile
    const long long max_units = ((long long)c.batch + (c.total_q + p.tq - 1) / p.tq) * p.hgroups;
    const int grid = (int)std::max(1LL, std::min<long long>((long long)device_sm_count(), max_units));
    e = c.head_dim == 128 ? launch_prefill<128, false>(qm, km, vm, p, grid, stream, true)
                          : launch_prefill<64, false>(qm, km, vm, p, grid, stream, true);
    if (e != cudaSuccess) return cuda_failure(e, "prefill tcgen05 launch");
    count_launches(1);
    return NVPA_OK;
}

}  // namespace nvpa
