// Parameters and launch helpers shared by the paged decode kernels (plan, shared-prefix
// plan, split-KV worker, combine).
#pragma once

#include <climits>

#include "attn_warp.cuh"
#include "nvpa_internal.h"

namespace nvpa {

#ifndef NVPA_DECODE_STAGES
#define NVPA_DECODE_STAGES 2
#endif

constexpr int kAttnWarps = 4;
constexpr int kAttnStages = NVPA_DECODE_STAGES;
constexpr int kSharedMaxBatch = 2048;   // larger batches are decoded without prefix groups
constexpr int kDefaultMinGroup = 8;

struct AttnParams {
    const uint16_t* q;
    const uint16_t* k_cache;
    const uint16_t* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    // fused decode step: sequence b's newest key/value (position context_lens[b]-1) is read
    // from k_new/v_new row b instead of the cache and written to slot_mapping[b]
    const uint16_t* k_new;
    const uint16_t* v_new;
    long long k_new_stride, v_new_stride;   // elements between rows of k_new / v_new
    const int32_t* slot_mapping;
    long long capacity;                     // num_blocks * block_size
    int fused;
    uint16_t* k_cache_w;
    uint16_t* v_cache_w;
    uint16_t* out;
    float* out_f32;                // partial mode: fp32 normalised output instead of bf16 `out`
    float* lse_out;
    float* o_part;
    float* lse_part;
    int4* items;
    int32_t* nsplit;
    int32_t* counter;              // [0] items claimed after the first round, [1] number of items
    int32_t* err;
    int batch, hq, hkv, group;
    int max_blocks, num_blocks, block_size, block_shift;
    int max_ctx;                   // host-side bound of context_lens
    int chunk, s_max;              // keys per partition, partitions of the longest context
    float scale_log2;
    // shared-prefix plan outputs (decode_plan_shared_kernel)
    int4* ptiles;                  // (group, query tile A, query tile B or -1, prefix partition)
    int32_t* members;              // grouped member lists
    int32_t* group_start;          // [groups + 1]
    int32_t* group_len;            // [groups] prefix tokens
    int min_members, pchunk, ptq;  // smallest group, prefix keys per partition, members per tile
    // 1 when the grid launched just before the worker is the shared-prefix tile kernel: that
    // kernel lets the worker launch only once the plan has completed, so the worker starts at
    // once, runs beside the prefix tiles, and waits for their grid at its end (a kernel after
    // the worker then sees both grids' partials)
    int wait_at_end;
};

template <int D, int GMAX>
struct AttnStage {
    static constexpr int KV_BYTES = kTileKeys * D * 2;
    static constexpr int Q_BYTES = GMAX * D * 2;
    static constexpr int BYTES = 2 * KV_BYTES + Q_BYTES + 32;   // + two int4 of metadata
};

// Programmatic dependent launch: wait for the preceding kernel's results / let the next
// kernel's CTAs start launching.  Both are no-ops for a normal launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}


// Worker items are ordered by length, longest first, in this many classes of a partition's
// key count (class c holds lengths with c = length * 256 / chunk).
constexpr int kLengthClasses = 256;
__device__ __forceinline__ int length_class(int len, int chunk) {
    return min(kLengthClasses - 1, (int)(((long long)len * kLengthClasses) / chunk));
}

// Exclusive prefix sum of v over the block (every thread calls it; blockDim a multiple of
// 32, at most 1024); total = the block's sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int w = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    const int excl = incl - v + (wid ? warp_tot[wid - 1] : 0);
    total = warp_tot[31];
    __syncthreads();
    return excl;
}

constexpr int kSharedTable = 2 * kSharedMaxBatch;   // buckets of the shared-prefix plan (a power of two)
constexpr size_t kSharedPlanSmem = sizeof(int) * (6 * (size_t)kSharedTable + 2 * (size_t)kSharedMaxBatch);

// Launch with programmatic stream serialisation: the kernel may start while its
// predecessor finishes and synchronises with it through griddepcontrol.wait.
template <typename Kernel>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       const AttnParams& p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

// Enqueue the shared-prefix plan (one CTA) on `stream`.
cudaError_t launch_decode_plan_shared(const AttnParams& p, cudaStream_t stream);
// Enqueue the split-KV combine (grid CTAs of 8 warps, one warp per sequence and query
// head), as a programmatic dependent of the worker.
// The split-KV combine over every (sequence, query head) of p (see decode_combine.cu).
cudaError_t launch_decode_combine(const AttnParams& p, int head_dim, cudaStream_t stream);
int decode_combine_warps_per_row(long long rows, int s_max);

}  // namespace nvpa
