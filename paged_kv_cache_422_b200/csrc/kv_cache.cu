// store_kvcache: scatter new K/V rows into the block-paged cache through slot_mapping
// ("Nano-vLLM inference engine architecture", section "PagedAttention's lightweight
// implementation": each token's keys and values land at the cache offset its slot gives;
// the cache is one flat [total_slots, num_kv_heads * head_dim] array per K and V).
//
// gather_kv: the inverse read, one sequence's rows copied out contiguously through its
// block table ("Nano-vLLM part 1", section 4.1: a sequence spans several fixed-size
// blocks, the last one partly filled).  It exists to check the paged addressing
// bit-exactly.
//
// Both are pure copies, bound by HBM bandwidth: 16-byte vector loads and stores, one
// group of lanes per token row, loads of the new rows marked streaming (read once).
#include <algorithm>

#include "common.cuh"
#include "nvpa_internal.h"

namespace nvpa {

// One token row = row16 chunks of 16 bytes (num_kv_heads * head_dim * 2 / 16).  A CTA of
// 256 threads copies tpi tokens at a time with tpt threads per token, each thread moving
// the same chunk index of K and of V.
__global__ void __launch_bounds__(256) store_kvcache_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, long long k_stride16,
    long long v_stride16, uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
    const int32_t* __restrict__ slot_mapping, int num_tokens, int row16, long long capacity,
    int tpt, int tpi, int32_t* err_flag) {
    const int which = threadIdx.x / tpt;
    if (which >= tpi) return;
    const int lt = threadIdx.x - which * tpt;
    for (int t = blockIdx.x * tpi + which; t < num_tokens; t += gridDim.x * tpi) {
        const int slot = __ldg(slot_mapping + t);
        if (slot == -1) continue;   // padding token
        if (slot < 0 || (long long)slot >= capacity) {
            if (lt == 0) flag_error(err_flag, NVPA_FLAG_BAD_SLOT);
            continue;
        }
        const uint4* ks = k + (long long)t * k_stride16;
        const uint4* vs = v + (long long)t * v_stride16;
        uint4* kd = k_cache + (long long)slot * row16;
        uint4* vd = v_cache + (long long)slot * row16;
        for (int c = lt; c < row16; c += tpt) {
            const uint4 a = __ldcs(ks + c);
            const uint4 b = __ldcs(vs + c);
            kd[c] = a;
            vd[c] = b;
        }
    }
}

// One warp per destination row; sequence found by binary search over cu_seqlens_k.
__global__ void __launch_bounds__(256) gather_kv_kernel(
    uint4* __restrict__ dst, const uint4* __restrict__ cache, const int32_t* __restrict__ block_tables,
    int max_blocks, const int32_t* __restrict__ cu_seqlens_k, int batch, int total_k, int row16,
    int num_blocks, int block_size, int block_shift, int32_t* err_flag) {
    const int lane = threadIdx.x & 31;
    for (long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); row < total_k;
         row += (long long)gridDim.x * 8) {
        int lo = 0, hi = batch - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(cu_seqlens_k + mid) <= row) lo = mid; else hi = mid - 1;
        }
        const int k0 = __ldg(cu_seqlens_k + lo), k1 = __ldg(cu_seqlens_k + lo + 1);
        const int pos = (int)(row - k0);
        uint4* d = dst + row * row16;
        if (row < k0 || row >= k1 || (long long)pos >= (long long)max_blocks * block_size) {
            if (lane == 0) flag_error(err_flag, NVPA_FLAG_BAD_LENGTH);
            continue;
        }
        const int blk = checked_block(block_tables + (size_t)lo * max_blocks, pos, block_shift,
                                      num_blocks, lane == 0 ? err_flag : nullptr);
        if (blk < 0) {
            for (int c = lane; c < row16; c += 32) d[c] = make_uint4(0, 0, 0, 0);
            continue;
        }
        const uint4* s = cache + ((long long)blk * block_size + (pos & (block_size - 1))) * row16;
        for (int c = lane; c < row16; c += 32) d[c] = __ldg(s + c);
    }
}

nvpa_status_t run_store_kvcache(const void* k, const void* v, int64_t k_stride, int64_t v_stride,
                                void* k_cache, void* v_cache, const int32_t* slot_mapping,
                                int num_tokens, int hkv, int head_dim, int num_blocks,
                                int block_size, int32_t* err_flag, cudaStream_t stream) {
    if (num_tokens == 0) return NVPA_OK;
    const int row16 = hkv * head_dim / 8;
    const int tpt = std::min(256, (row16 + 31) / 32 * 32);
    const int tpi = 256 / tpt;
    const long long ctas_needed = ((long long)num_tokens + tpi - 1) / tpi;
    const int grid = (int)std::max(1LL, std::min<long long>(ctas_needed, (long long)device_sm_count() * 8));
    store_kvcache_kernel<<<grid, 256, 0, stream>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), k_stride / 8, v_stride / 8,
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slot_mapping, num_tokens, row16,
        (long long)num_blocks * block_size, tpt, tpi, err_flag);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_failure(e, "store_kvcache launch");
    count_launches(1);
    return NVPA_OK;
}

nvpa_status_t run_gather_kv(void* dst, const void* cache, const int32_t* block_tables,
                            int max_blocks_per_seq, const int32_t* cu_seqlens_k, int batch,
                            int total_k, int hkv, int head_dim, int num_blocks, int block_size,
                            int32_t* err_flag, cudaStream_t stream) {
    if (total_k == 0 || batch == 0) return NVPA_OK;
    const int row16 = hkv * head_dim / 8;
    const int grid = (int)std::min<long long>(((long long)total_k + 7) / 8, (long long)device_sm_count() * 16);
    gather_kv_kernel<<<grid, 256, 0, stream>>>(
        static_cast<uint4*>(dst), static_cast<const uint4*>(cache), block_tables, max_blocks_per_seq,
        cu_seqlens_k, batch, total_k, row16, num_blocks, block_size, __builtin_ctz((unsigned)block_size),
        err_flag);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_failure(e, "gather_kv launch");
    count_launches(1);
    return NVPA_OK;
}

}  // namespace nvpa
