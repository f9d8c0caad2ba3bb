// nvpa_paged_decode_attention_static_scratch: paged decode attention for callers that
// cannot allocate device memory themselves.
//
// Some callers have no way to obtain the decode workspace: a plugin inside a host
// runtime whose memory manager owns all device memory and offers it no allocation hook,
// or code that runs where an allocation is not allowed (a cudaMalloc there would fail,
// or would synchronise the device and stall the work already queued).  For them this
// entry point keeps the decode's scratch (the partition plan and the split partials) in
// a fixed array that is part of the library's device image.  The caller still passes the
// inputs and outputs.
//
// The array takes kStaticScratchBytes of device memory on every GPU that loads the
// library, until the process exits.  Its device address is resolved with
// cudaGetSymbolAddress once per device, during the first call made with that device
// current; make that first call before any stream capture.  Only a successful resolution
// is kept: a first call that fails (made during a capture, say) returns the error and the
// next call tries again.  cudaDeviceReset unloads the library's device image, so an
// address kept from before a reset is stale: a process that resets a device must not call
// this entry point on that device again.  Every call shares the one
// array, and the array keeps the last call's contents: nothing in it has to start at
// zero (the plan kernel rewrites the counters it needs on every call), but calls whose
// kernels overlap on the GPU (other streams, other threads) race on it and must be
// serialised by the caller.
#include <mutex>

#include "nvpa_internal.h"

namespace nvpa {

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;   // 64 MiB

__device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

// Per device: the resolved address, or null until a resolution succeeds.
struct ScratchAddress {
    std::mutex mu;
    void* ptr = nullptr;
};
ScratchAddress g_scratch_address[64];

// The array's device address on the current device `dev`, resolved on first use.
cudaError_t scratch_address(int dev, void** ptr) {
    ScratchAddress& sa = g_scratch_address[dev];
    std::lock_guard<std::mutex> lock(sa.mu);
    if (sa.ptr == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        if (p == nullptr) return cudaErrorInvalidSymbol;
        sa.ptr = p;
    }
    *ptr = sa.ptr;
    return cudaSuccess;
}

}  // namespace

}  // namespace nvpa

using namespace nvpa;

extern "C" nvpa_status_t nvpa_paged_decode_attention_static_scratch(
    void* out, float* lse_out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens, int batch,
    int num_q_heads, int num_kv_heads, int head_dim, int num_blocks, int block_size,
    int max_context_len, float softmax_scale, int num_splits, int32_t* err_flag,
    cudaStream_t stream) {
    if (batch < 0 || max_context_len < 0 || num_splits < 0 || num_q_heads <= 0 ||
        num_kv_heads <= 0 || head_dim <= 0) {
        set_error("batch, max_context_len and num_splits must be >= 0, head counts and head_dim > 0");
        return NVPA_ERR_INVALID_ARG;
    }
    const size_t need = decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim,
                                               max_context_len, block_size, num_splits);
    if (need > kStaticScratchBytes) {
        set_error("static scratch holds %zu bytes but this call needs %zu: lower num_splits or the "
                  "batch, or pass a workspace to nvpa_paged_decode_attention",
                  kStaticScratchBytes, need);
        return NVPA_ERR_WORKSPACE_TOO_SMALL;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_failure(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) {
        set_error("device ordinal %d outside the supported 0..63", dev);
        return NVPA_ERR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    e = scratch_address(dev, &scratch);
    if (e != cudaSuccess) return cuda_failure(e, "cudaGetSymbolAddress(static decode scratch)");
    return nvpa_paged_decode_attention(out, lse_out, q, k_cache, v_cache, block_tables,
                                       max_blocks_per_seq, context_lens, batch, num_q_heads,
                                       num_kv_heads, head_dim, num_blocks, block_size,
                                       max_context_len, softmax_scale, num_splits, scratch,
                                       kStaticScratchBytes, err_flag, stream);
}
