// Paged decode attention: split-KV partitions merged by log-sum-exp.
//
// The worker kernel is persistent and every warp is an independent worker: it takes
// work items (one KV head of one partition of one sequence's context), streams that
// range's K and V rows from the paged cache into its own ring of shared-memory stages
// with 16-byte cp.async copies (zero-filling rows past the range, never reading them),
// and consumes each 16-key stage with the CUDA-core tile loop of attn_warp.cuh.  The
// issue side runs STAGES-1 tiles ahead of the consume side and crosses item boundaries
// without draining, so a warp keeps its loads in flight from one item to the next.
//
// Work items: sequence b's context is cut into partitions of `chunk` keys ("Nano-vLLM
// part 1" section 5.2: one query token per sequence reading all its cached tokens).  A
// one-CTA plan kernel turns the device-side context lengths into a table of (sequence,
// partition, key range) entries and resets an item counter; warps grab items from the
// counter with atomics, so uneven context lengths balance across the SMs.  Items are
// ordered sequence-major with the KV heads of one partition adjacent, so the warps
// reading one cache row's different heads run at the same time.  A sequence with one
// partition is written straight to `out`; otherwise each partition writes its normalised
// output and log-sum-exp to the workspace and a combine kernel (one warp per sequence
// and query head) merges them with the log-sum-exp weights:
//     lse = log sum_p exp(lse_p),   out = sum_p exp(lse_p - lse) * o_p.
#include <algorithm>
#include <mutex>

#include "decode_params.cuh"

namespace nvpa {

// ------------------------------------------------------------------------------------
// plan: context lengths -> (sequence, partition, key range) table
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) decode_plan_kernel(const AttnParams p) {
    // Items: every full-length partition first, sequence by sequence, then each sequence's
    // last, shorter partition, longest first (a counting sort over kLengthClasses length
    // classes): the items claimed last are the shortest, so the worker's warps finish
    // close together.
    __shared__ int warp_tot[32];
    __shared__ int s_cls[kLengthClasses];
    const int tid = threadIdx.x;
    pdl_launch_dependents();
    for (int i = tid; i < kLengthClasses; i += blockDim.x) s_cls[i] = 0;
    __syncthreads();
    const long long lim_ll = min((long long)p.max_ctx, (long long)p.max_blocks * p.block_size);
    const int lim = (int)lim_ll;
    auto clamp_ctx = [&](int b, bool flag) {
        int ctx = __ldg(p.context_lens + b);
        if (ctx < 0 || ctx > lim) {
            if (flag) flag_error(p.err, NVPA_FLAG_BAD_LENGTH);
            ctx = min(max(ctx, 0), lim);
        }
        return ctx;
    };
    int carry = 0;
    for (int base = 0; base < p.batch; base += blockDim.x) {
        const int b = base + tid;
        int nfull = 0, ns = 0;
        if (b < p.batch) {
            const int ctx = clamp_ctx(b, true);
            ns = max(1, (ctx + p.chunk - 1) / p.chunk);
            p.nsplit[b] = ns;
            const int last = ctx - (ns - 1) * p.chunk;
            nfull = last == p.chunk ? ns : ns - 1;
            if (last < p.chunk) atomicAdd(s_cls + length_class(last, p.chunk), 1);
        }
        int block_tot = 0;
        const int e = carry + block_exclusive_scan(nfull, warp_tot, block_tot);
        for (int s = 0; s < nfull; ++s)
            p.items[e + s] = make_int4(b, s | (ns << 16), s * p.chunk, (s + 1) * p.chunk);
        carry += block_tot;
    }
    __syncthreads();
    // first position of each length class, longest class first, after the full partitions
    const int cls = kLengthClasses - 1 - tid;
    const int v = tid < kLengthClasses ? s_cls[cls] : 0;
    int tot_short = 0;
    const int e = block_exclusive_scan(v, warp_tot, tot_short);
    if (tid < kLengthClasses) s_cls[cls] = carry + e;
    __syncthreads();
    for (int b = tid; b < p.batch; b += blockDim.x) {
        const int ctx = clamp_ctx(b, false);
        const int ns = max(1, (ctx + p.chunk - 1) / p.chunk);
        const int last = ctx - (ns - 1) * p.chunk;
        if (last == p.chunk) continue;
        const int pos = atomicAdd(s_cls + length_class(last, p.chunk), 1);
        p.items[pos] = make_int4(b, (ns - 1) | (ns << 16), (ns - 1) * p.chunk, ctx);
    }
    if (tid == 0) {
        p.counter[0] = 0;
        p.counter[1] = (carry + tot_short) * p.hkv;
        p.counter[2] = p.counter[3] = p.counter[4] = 0;   // no shared-prefix groups
    }
}

// ------------------------------------------------------------------------------------
// the worker kernel
// ------------------------------------------------------------------------------------
template <int D, int GMAX>
__global__ void __launch_bounds__(kAttnWarps * 32)
paged_attention_kernel(const AttnParams p) {
    using State = WarpAttnState<D, GMAX>;
    using Stage = AttnStage<D, GMAX>;
    constexpr int LPR = State::LPR, RPI = State::RPI, ITER = State::ITER;
    constexpr int STAGES = kAttnStages;

    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = lane / LPR, sub = lane % LPR;
    uint8_t* wsm = smem + (size_t)warp * STAGES * Stage::BYTES;

    const size_t row_stride = (size_t)p.hkv * D;   // elements between cache rows (slots)
    const int bmask = p.block_size - 1;

    // ---------------- issue side: the item whose tiles are being loaded ----------------
    bool it_valid = false;
    int it_qrow = 0, it_seq = 0, it_hk = 0, it_s = 0, it_ns = 1, it_k0 = 0, it_k1 = 0;
    int it_ntiles = 0, it_t = 0, it_fb = 0, it_blk = -1;
    const int32_t* it_bt = nullptr;

    // the plan (and everything before it on the stream) has completed after this wait; with
    // wait_at_end the grid before this one only let it launch once that was so
    if (!p.wait_at_end) pdl_wait();
    // A warp's first item is its index in the grid; the counter hands out the items after
    // the first round, and lane 0 holds the next one, requested one item ahead.  (Claiming
    // the first items from the counter as well made the warps that started first take two
    // items each when there are about as many items as warps, and left the others idle.)
    const int total_items = __ldcg(p.counter + 1);
    const int nwarps = gridDim.x * kAttnWarps;
    int nx_item = blockIdx.x * kAttnWarps + warp;

    auto load_blocks = [&]() {
        it_fb = it_k0 >> p.block_shift;
        const int nblk = (it_k1 > it_k0) ? ((it_k1 - 1) >> p.block_shift) - it_fb + 1 : 0;
        it_blk = -1;
        if (lane < nblk) {
            int e = __ldg(it_bt + it_fb + lane);
            if (e < 0 || e >= p.num_blocks) {
                flag_error(p.err, NVPA_FLAG_BAD_BLOCK_ID);
                e = -1;
            }
            it_blk = e;
        }
    };

    auto fetch = [&]() {
        it_t = 0;
        const int idx = __shfl_sync(0xffffffffu, nx_item, 0);
        if (idx >= total_items) {
            it_valid = false;
            return;
        }
        if (lane == 0) nx_item = nwarps + atomicAdd(p.counter, 1);
        const int4 d = __ldcg(reinterpret_cast<const int4*>(p.items) + idx / p.hkv);
        it_valid = true;
        it_seq = d.x;
        it_qrow = d.x;
        it_s = d.y & 0xffff;
        it_ns = d.y >> 16;
        it_k0 = d.z;
        it_k1 = d.w;
        it_hk = idx % p.hkv;
        it_bt = p.block_tables + (size_t)it_seq * p.max_blocks;
        it_ntiles = max(1, (it_k1 - it_k0 + kTileKeys - 1) / kTileKeys);
        load_blocks();
    };

    auto stage_ptrs = [&](int st, uint16_t*& ks, uint16_t*& vs, uint16_t*& qs, int4*& meta) {
        uint8_t* sb = wsm + st * Stage::BYTES;
        ks = reinterpret_cast<uint16_t*>(sb);
        vs = ks + kTileKeys * D;
        qs = vs + kTileKeys * D;
        meta = reinterpret_cast<int4*>(qs + GMAX * D);   // meta[0], meta[1]
    };

    auto issue = [&](int st) {
        uint16_t *ks, *vs, *qs;
        int4* meta;
        stage_ptrs(st, ks, vs, qs, meta);
        if (!it_valid) {
            if (lane == 0) *meta = make_int4(-1, 0, 0, 0);
            cp_async_commit();
            return;
        }
        const int key0 = it_k0 + kTileKeys * it_t;
        int rows = min(kTileKeys, it_k1 - key0);
        const int bi = (key0 >> p.block_shift) - it_fb;
        int blk = __shfl_sync(0xffffffffu, it_blk, bi & 31);
        if (bi >= 32 && rows > 0) {   // partitions longer than 32 blocks: direct lookup
            blk = __ldg(it_bt + it_fb + bi);
            if (blk < 0 || blk >= p.num_blocks) {
                if (lane == 0) flag_error(p.err, NVPA_FLAG_BAD_BLOCK_ID);
                blk = -1;
            }
        }
        if (blk < 0) rows = 0;
        rows = max(rows, 0);
        const size_t slot0 = (size_t)max(blk, 0) * p.block_size + (key0 & bmask);
        const uint16_t* kg = p.k_cache + slot0 * row_stride + (size_t)it_hk * D + sub * 8;
        const uint16_t* vg = p.v_cache + slot0 * row_stride + (size_t)it_hk * D + sub * 8;
        const bool first = it_t == 0;
        const bool last = it_t + 1 == it_ntiles;
        // fused step: the sequence's newest key sits in the last tile of its last partition
        const int new_row = (p.fused && last && it_s + 1 == it_ns && it_k1 > key0) ? it_k1 - 1 - key0 : -1;
#pragma unroll
        for (int i = 0; i < ITER; ++i) {
            const int r = grp + RPI * i;
            const int nb = r < rows ? 16 : 0;
            if (r == new_row) {
                cp_async16(ks + r * D + sub * 8,
                           p.k_new + (size_t)it_seq * p.k_new_stride + (size_t)it_hk * D + sub * 8, 16);
                cp_async16(vs + r * D + sub * 8,
                           p.v_new + (size_t)it_seq * p.v_new_stride + (size_t)it_hk * D + sub * 8, 16);
            } else {
                cp_async16(ks + r * D + sub * 8, kg + (size_t)r * row_stride, nb);
                cp_async16(vs + r * D + sub * 8, vg + (size_t)r * row_stride, nb);
            }
        }
        if (first) {
            const uint16_t* qg = p.q + ((size_t)it_qrow * p.hq + (size_t)it_hk * p.group) * D;
            for (int c = lane; c < p.group * LPR; c += 32) cp_async16(qs + c * 8, qg + c * 8, 16);
        }
        if (lane == 0) {
            meta[0] = make_int4(it_qrow, it_hk, it_s | (it_ns << 16),
                                rows | (first ? 256 : 0) | (last ? 512 : 0));
            meta[1] = make_int4(new_row, new_row >= 0 ? __ldg(p.slot_mapping + it_seq) : -1, 0, 0);
        }
        cp_async_commit();
        if (last) fetch(); else ++it_t;
    };

    State acc;
    auto epilogue = [&](const int4 meta) {
        acc.finish();
        const int qrow = meta.x, hk = meta.y, s = meta.z & 0xffff, ns = meta.z >> 16;
        if (grp == 0) {
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
                if (g >= p.group) break;
                const int h = hk * p.group + g;
                const float inv = acc.l[g] > 0.f ? 1.f / acc.l[g] : 0.f;
                const float lse = acc.lse(g);
                float v[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) acc.out_pair(g, k, v[2 * k], v[2 * k + 1]);
                if (ns == 1 && p.out_f32 != nullptr) {
                    float* op = p.out_f32 + ((size_t)qrow * p.hq + h) * D + sub * 8;
                    *reinterpret_cast<float4*>(op) = make_float4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
                    *reinterpret_cast<float4*>(op + 4) = make_float4(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv);
                    if (sub == 0 && p.lse_out != nullptr) p.lse_out[(size_t)qrow * p.hq + h] = lse;
                } else if (ns == 1) {
                    uint4 w;
                    w.x = pack_bf16x2(v[0] * inv, v[1] * inv);
                    w.y = pack_bf16x2(v[2] * inv, v[3] * inv);
                    w.z = pack_bf16x2(v[4] * inv, v[5] * inv);
                    w.w = pack_bf16x2(v[6] * inv, v[7] * inv);
                    *reinterpret_cast<uint4*>(p.out + ((size_t)qrow * p.hq + h) * D + sub * 8) = w;
                    if (sub == 0 && p.lse_out != nullptr) p.lse_out[(size_t)qrow * p.hq + h] = lse;
                } else {
                    float* op = p.o_part + (((size_t)qrow * p.hq + h) * p.s_max + s) * D + sub * 8;
                    __stcg(reinterpret_cast<float4*>(op), make_float4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv));
                    __stcg(reinterpret_cast<float4*>(op + 4), make_float4(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv));
                    if (sub == 0) __stcg(p.lse_part + ((size_t)qrow * p.hq + h) * p.s_max + s, lse);
                }
            }
        }
    };

    auto consume = [&](int st) -> bool {
        uint16_t *ks, *vs, *qs;
        int4* meta_p;
        stage_ptrs(st, ks, vs, qs, meta_p);
        const int4 meta = *meta_p;
        if (meta.x < 0) return false;
        const int rows = meta.w & 255;
        if (meta.w & 256) {
            acc.reset();
            acc.load_q(qs, p.group, sub, p.scale_log2);
        }
        acc.consume(ks, vs, rows, lane);
        if (p.fused) {
            const int4 m1 = meta_p[1];
            if (m1.x >= 0 && grp == (m1.x % RPI)) {
                const int slot = m1.y;
                if (slot >= 0 && (long long)slot < p.capacity) {
                    const size_t dst = (size_t)slot * row_stride + (size_t)meta.y * D + sub * 8;
                    *reinterpret_cast<uint4*>(p.k_cache_w + dst) =
                        *reinterpret_cast<const uint4*>(ks + m1.x * D + sub * 8);
                    *reinterpret_cast<uint4*>(p.v_cache_w + dst) =
                        *reinterpret_cast<const uint4*>(vs + m1.x * D + sub * 8);
                } else if (slot != -1 && sub == 0) {
                    flag_error(p.err, NVPA_FLAG_BAD_SLOT);
                }
            }
        }
        if (meta.w & 512) epilogue(meta);
        return true;
    };

    fetch();
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) issue(s);
    int cs = 0, is = STAGES - 1;
    while (true) {
        cp_async_wait<STAGES - 2>();
        __syncwarp();
        issue(is);
        is = (is + 1 == STAGES) ? 0 : is + 1;
        if (!consume(cs)) break;
        cs = (cs + 1 == STAGES) ? 0 : cs + 1;
    }
    cp_async_wait<0>();
    pdl_launch_dependents();
    if (p.wait_at_end) pdl_wait();   // the shared-prefix tiles' grid has completed
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
namespace {

template <int D, int GMAX>
int worker_ctas_per_sm() {
    static std::once_flag once[64];
    static int cached[64];
    int dev = 0;
    cudaGetDevice(&dev);
    dev &= 63;
    std::call_once(once[dev], [&] {
        const int smem = kAttnWarps * kAttnStages * AttnStage<D, GMAX>::BYTES;
        auto kern = paged_attention_kernel<D, GMAX>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kAttnWarps * 32, smem) != cudaSuccess)
            n = 1;
        cached[dev] = std::max(1, n);
    });
    return cached[dev];
}

template <int D, int GMAX>
cudaError_t launch_worker(const AttnParams& p, long long max_items, cudaStream_t stream) {
    const int per_sm = worker_ctas_per_sm<D, GMAX>();
    const long long want = (max_items + kAttnWarps - 1) / kAttnWarps;
    const int grid = (int)std::max(1LL, std::min<long long>((long long)device_sm_count() * per_sm, want));
    const int smem = kAttnWarps * kAttnStages * AttnStage<D, GMAX>::BYTES;
    const cudaError_t e = launch_pdl(paged_attention_kernel<D, GMAX>, dim3(grid), dim3(kAttnWarps * 32),
                                     (size_t)smem, stream, p);
    if (e == cudaSuccess) count_launches(1);
    return e;
}

cudaError_t dispatch_worker(const AttnParams& p, int head_dim, long long max_items, cudaStream_t s) {
    const int g = p.group;
    const int gmax = g <= 1 ? 1 : g <= 2 ? 2 : g <= 4 ? 4 : 8;
#define NVPA_CASE(DD, GG) \
    if (head_dim == DD && gmax == GG) return launch_worker<DD, GG>(p, max_items, s);
    NVPA_CASE(128, 1) NVPA_CASE(128, 2) NVPA_CASE(128, 4) NVPA_CASE(128, 8)
    NVPA_CASE(64, 1) NVPA_CASE(64, 2) NVPA_CASE(64, 4) NVPA_CASE(64, 8)
#undef NVPA_CASE
    return cudaErrorInvalidValue;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }


struct DecodeWorkspace {
    size_t counter, nsplit, items, lse_part, o_part, members, group_start, group_len, ptiles, total;
};

// ptile_entries > 0: room for the shared-prefix plan's tables as well
DecodeWorkspace decode_workspace_layout(int batch, int hq, int hkv, int head_dim, int s_max,
                                        long long ptile_entries = 0) {
    (void)hkv;
    DecodeWorkspace w;
    size_t off = 0;
    w.counter = off; off += 256;
    w.nsplit = off; off = align256(off + sizeof(int32_t) * (size_t)batch);
    w.items = off; off = align256(off + sizeof(int4) * (size_t)batch * s_max);
    w.lse_part = off;
    off = align256(off + (s_max > 1 ? sizeof(float) * (size_t)batch * hq * s_max : 0));
    w.o_part = off;
    off = align256(off + (s_max > 1 ? sizeof(float) * (size_t)batch * hq * s_max * head_dim : 0));
    w.members = w.group_start = w.group_len = w.ptiles = off;
    if (ptile_entries > 0) {
        w.members = off; off = align256(off + sizeof(int32_t) * (size_t)batch);
        w.group_start = off; off = align256(off + sizeof(int32_t) * ((size_t)batch + 1));
        w.group_len = off; off = align256(off + sizeof(int32_t) * (size_t)batch);
        w.ptiles = off; off = align256(off + sizeof(int4) * (size_t)ptile_entries);
    }
    w.total = off;
    return w;
}

// Partitioning of a shared-prefix decode; active == false when the batch is too large
// for the plan's table or smaller than the smallest group (the call then runs as a plain
// decode step).
struct SharedGeometry {
    bool active;
    int chunk, s_max, pchunk, ptq, min_members;
    long long entries;   // bound on prefix tile entries
};

SharedGeometry shared_geometry(int batch, int hq, int hkv, int max_context_len, int block_size,
                               int num_splits, int min_group) {
    SharedGeometry g{};
    g.chunk = decode_chunk_keys(batch, hkv, max_context_len, block_size, num_splits);
    const int ctx = std::max(0, max_context_len);
    g.min_members = min_group > 0 ? std::max(2, min_group) : kDefaultMinGroup;
    // a batch smaller than the smallest group cannot form one: no plan table, no prefix launch
    g.active = batch <= kSharedMaxBatch && batch >= g.min_members;
    // one more partition than a plain decode: splitting a context at the prefix boundary
    // adds at most one (pchunk >= chunk)
    g.s_max = std::max(1, (ctx + g.chunk - 1) / g.chunk) + (g.active ? 1 : 0);
    g.pchunk = (g.chunk + 127) / 128 * 128;
    g.ptq = 128 / attention_tile_pack(hq, hkv);
    const long long groups = batch / g.min_members;
    g.entries = g.active ? ((long long)batch / g.ptq + groups + 1) * ((ctx + g.pchunk - 1) / g.pchunk + 1) : 0;
    return g;
}


}  // namespace

// Keys per decode partition.  Depends on host-side values only, so the launch shape and
// the workspace size are fixed for a given batch and bound (CUDA-graph capturable).
// Automatic sizing counts a batch of full-length contexts against kTargetItems, the
// resident worker warps of a 148-SM B200 (3 CTAs of 4 warps per SM):
//  - small batches get partitions of 64 keys or more, enough for one item per warp;
//  - many sequences (more than kTargetItems / 8 sequence-head pairs) get 352-key
//    partitions: many rounds of items, whose varying lengths even the rounds out; longer
//    partitions write and merge fewer partials but lengthen the last round (measured on
//    512 contexts of up to 4 k keys: 352 keys 1 % faster than 256, 688 keys 3 % slower; on
//    64 contexts of 0.5 to 4 k keys: 336 to 368 keys 3 to 5 % faster than 256, although
//    288 and 320 keys were 6 and 2 % slower and 504 keys 15 % slower);
//  - a few long sequences get about two rounds of items, 128 to 1024 keys each and at
//    most 32 cache blocks: fewer, longer partitions mean fewer partials to write and
//    merge, and two rounds keep the warps that idle in the last one a small share; a
//    worker warp holds one block id per lane for its partition, so a partition of more
//    than 32 blocks looks its later blocks up one key tile at a time, on the copy's path
//    (measured on 8 contexts of 32 k keys in blocks of 16: 512-key partitions 0.205 ms per
//    step, 592 keys (37 blocks) 0.217, 464 keys 0.213, 256 keys 0.228; on 16 contexts of
//    4 k keys 160-key partitions beat 256-key ones by 12 %).
int decode_chunk_keys(int batch, int num_kv_heads, int max_context_len, int block_size, int num_splits) {
    const int ctx = std::max(1, max_context_len);
    if (num_splits > 0) {
        const int per = (ctx + num_splits - 1) / num_splits;
        return std::max(kTileKeys, (per + kTileKeys - 1) / kTileKeys * kTileKeys);
    }
    constexpr long long kTargetItems = 148LL * 3 * kAttnWarps;
    constexpr long long kMinChunkKeys = 64, kFillChunkKeys = 256, kManyChunkKeys = 352;
    constexpr long long kMinLongChunk = 128, kMaxLongChunk = 1024;
    auto round16 = [](long long k) { return (k + kTileKeys - 1) / kTileKeys * kTileKeys; };
    const long long per_partition = (long long)std::max(1, batch) * std::max(1, num_kv_heads);
    const long long fill = round16((ctx + (kTargetItems + per_partition - 1) / per_partition - 1) /
                                   ((kTargetItems + per_partition - 1) / per_partition));
    if (fill < kFillChunkKeys) return (int)std::max(kMinChunkKeys, fill);
    if (per_partition * 8 > kTargetItems) return (int)kManyChunkKeys;
    const long long parts = (2 * kTargetItems + per_partition - 1) / per_partition;
    const long long chunk = round16((ctx + parts - 1) / parts);
    const long long cap = std::min(kMaxLongChunk, std::max(kMinLongChunk, 32LL * std::max(1, block_size)));
    return (int)std::min(cap, std::max(kMinLongChunk, chunk));
}

size_t decode_workspace_bytes(int batch, int hq, int hkv, int head_dim, int max_context_len,
                              int block_size, int num_splits) {
    const int chunk = decode_chunk_keys(batch, hkv, max_context_len, block_size, num_splits);
    const int s_max = std::max(1, (std::max(0, max_context_len) + chunk - 1) / chunk);
    return decode_workspace_layout(batch, hq, hkv, head_dim, s_max).total;
}

size_t decode_shared_prefix_workspace_bytes(int batch, int hq, int hkv, int head_dim,
                                            int max_context_len, int block_size, int num_splits,
                                            int min_group) {
    const SharedGeometry g = shared_geometry(batch, hq, hkv, max_context_len, block_size, num_splits, min_group);
    return decode_workspace_layout(batch, hq, hkv, head_dim, g.s_max, g.entries).total;
}

nvpa_status_t run_paged_decode(const DecodeCall& c, cudaStream_t stream) {
    const SharedGeometry sg = c.shared_prefix
        ? shared_geometry(c.batch, c.hq, c.hkv, c.max_context_len, c.block_size, c.num_splits, c.min_group)
        : SharedGeometry{};
    const bool shared = c.shared_prefix && sg.active;
    const int chunk = decode_chunk_keys(c.batch, c.hkv, c.max_context_len, c.block_size, c.num_splits);
    const int s_max = c.shared_prefix ? sg.s_max : std::max(1, (std::max(0, c.max_context_len) + chunk - 1) / chunk);
    const DecodeWorkspace w = decode_workspace_layout(c.batch, c.hq, c.hkv, c.head_dim, s_max, sg.entries);
    if (c.workspace_bytes < w.total) {
        set_error("workspace too small: %zu bytes given, %zu needed", c.workspace_bytes, w.total);
        return NVPA_ERR_WORKSPACE_TOO_SMALL;
    }
    uint8_t* ws = static_cast<uint8_t*>(c.workspace);
    AttnParams p{};
    p.q = static_cast<const uint16_t*>(c.q);
    p.k_cache = static_cast<const uint16_t*>(c.k_cache);
    p.v_cache = static_cast<const uint16_t*>(c.v_cache);
    p.block_tables = c.block_tables;
    p.context_lens = c.context_lens;
    p.out = static_cast<uint16_t*>(c.out);
    p.out_f32 = c.out_f32;
    p.lse_out = c.lse_out;
    p.counter = reinterpret_cast<int32_t*>(ws + w.counter);
    p.nsplit = reinterpret_cast<int32_t*>(ws + w.nsplit);
    p.items = reinterpret_cast<int4*>(ws + w.items);
    p.lse_part = reinterpret_cast<float*>(ws + w.lse_part);
    p.o_part = reinterpret_cast<float*>(ws + w.o_part);
    p.err = c.err_flag;
    p.batch = c.batch;
    p.hq = c.hq;
    p.hkv = c.hkv;
    p.group = c.hq / c.hkv;
    p.max_blocks = c.max_blocks_per_seq;
    p.num_blocks = c.num_blocks;
    p.block_size = c.block_size;
    p.block_shift = __builtin_ctz((unsigned)c.block_size);
    p.max_ctx = c.max_context_len;
    p.chunk = chunk;
    p.s_max = s_max;
    p.scale_log2 = c.scale * kLog2e;
    p.fused = c.k_new != nullptr ? 1 : 0;
    p.k_new = static_cast<const uint16_t*>(c.k_new);
    p.v_new = static_cast<const uint16_t*>(c.v_new);
    p.k_new_stride = c.k_new_stride;
    p.v_new_stride = c.v_new_stride;
    p.slot_mapping = c.slot_mapping;
    p.capacity = (long long)c.num_blocks * c.block_size;
    p.k_cache_w = static_cast<uint16_t*>(const_cast<void*>(c.k_cache));
    p.v_cache_w = static_cast<uint16_t*>(const_cast<void*>(c.v_cache));

    cudaError_t e = cudaSuccess;
    if (shared) {
        p.ptiles = reinterpret_cast<int4*>(ws + w.ptiles);
        p.members = reinterpret_cast<int32_t*>(ws + w.members);
        p.group_start = reinterpret_cast<int32_t*>(ws + w.group_start);
        p.group_len = reinterpret_cast<int32_t*>(ws + w.group_len);
        p.min_members = sg.min_members;
        p.pchunk = sg.pchunk;
        p.ptq = sg.ptq;
        e = launch_decode_plan_shared(p, stream);
        if (e != cudaSuccess) return cuda_failure(e, "decode plan launch");
        count_launches(1);
        DecodePrefixArgs a{};
        a.q = c.q;
        a.k_cache = c.k_cache;
        a.v_cache = c.v_cache;
        a.block_tables = c.block_tables;
        a.max_blocks_per_seq = c.max_blocks_per_seq;
        a.batch = c.batch;
        a.hq = c.hq;
        a.hkv = c.hkv;
        a.head_dim = c.head_dim;
        a.num_blocks = c.num_blocks;
        a.block_size = c.block_size;
        a.scale = c.scale;
        a.err_flag = c.err_flag;
        a.tiles = p.ptiles;
        a.ntiles = p.counter + 4;
        a.unit_counter = p.counter + 5;
        a.members = p.members;
        a.group_start = p.group_start;
        a.group_len = p.group_len;
        a.o_part = p.o_part;
        a.lse_part = p.lse_part;
        a.s_max = s_max;
        a.pchunk = sg.pchunk;
        a.max_entries = sg.entries;
        a.pdl = true;
        e = launch_decode_prefix_tcgen05(a, stream);
        if (e != cudaSuccess) return cuda_failure(e, "decode shared-prefix launch");
        count_launches(1);
        p.wait_at_end = 1;   // the worker runs beside the prefix tiles
    } else {
        decode_plan_kernel<<<1, 1024, 0, stream>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_failure(e, "decode plan launch");
        count_launches(1);
    }
    const long long max_items = (long long)c.batch * c.hkv * s_max;
    e = dispatch_worker(p, c.head_dim, max_items, stream);
    if (e != cudaSuccess) return cuda_failure(e, "decode worker launch");
    if (s_max > 1) {
        e = launch_decode_combine(p, c.head_dim, stream);
        if (e != cudaSuccess) return cuda_failure(e, "decode combine launch");
        count_launches(1);
    }
    return NVPA_OK;
}

}  // namespace nvpa
