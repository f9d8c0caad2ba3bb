// The extern "C" entry points of libnvpa: argument checks, then the launches.
// Every check that needs only host-side values happens here, before anything is
// enqueued; device-side values (slots, block ids, lengths) are checked in the kernels.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "nvpa.h"
#include "nvpa_internal.h"

namespace nvpa {

namespace {
thread_local char g_last_error[512] = "";

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
bool attn_block_size_ok(int bs) { return pow2(bs) && bs >= 16 && bs <= 256; }
}  // namespace

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
}

nvpa_status_t cuda_failure(cudaError_t e, const char* what) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    return NVPA_ERR_CUDA;
}

namespace {
std::atomic<uint64_t> g_launches{0};
}

void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

int device_sm_count() {
    static std::once_flag once[64];
    static int cached[64];
    int dev = 0;
    cudaGetDevice(&dev);
    dev &= 63;
    std::call_once(once[dev], [&] {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 1;
        cached[dev] = n;
    });
    return cached[dev];
}

}  // namespace nvpa

using namespace nvpa;

#define NVPA_REQUIRE(cond, status, ...) \
    do {                                \
        if (!(cond)) {                  \
            set_error(__VA_ARGS__);     \
            return status;              \
        }                               \
    } while (0)

static nvpa_status_t check_attention_shapes(int hq, int hkv, int head_dim, int num_blocks,
                                            int block_size, int max_blocks_per_seq) {
    NVPA_REQUIRE(hq > 0 && hkv > 0, NVPA_ERR_INVALID_ARG, "head counts must be positive");
    NVPA_REQUIRE(hq % hkv == 0, NVPA_ERR_INVALID_ARG,
                 "num_q_heads (%d) must be a multiple of num_kv_heads (%d)", hq, hkv);
    NVPA_REQUIRE(hq / hkv <= 8, NVPA_ERR_UNSUPPORTED, "query heads per KV head above 8");
    NVPA_REQUIRE(head_dim == 64 || head_dim == 128, NVPA_ERR_UNSUPPORTED,
                 "head_dim %d not supported (64, 128)", head_dim);
    NVPA_REQUIRE(block_size > 0 && num_blocks > 0 && max_blocks_per_seq > 0, NVPA_ERR_INVALID_ARG,
                 "block_size, num_blocks and max_blocks_per_seq must be positive");
    NVPA_REQUIRE(attn_block_size_ok(block_size), NVPA_ERR_UNSUPPORTED,
                 "block_size %d not supported (16, 32, 64, 128, 256)", block_size);
    NVPA_REQUIRE((long long)num_blocks * block_size <= 0x7fffffffLL, NVPA_ERR_UNSUPPORTED,
                 "pool of more than 2^31-1 slots");
    return NVPA_OK;
}

extern "C" {

int nvpa_version(void) { return 100; }

const char* nvpa_status_string(int status) {
    switch (status) {
        case NVPA_OK: return "NVPA_OK";
        case NVPA_ERR_INVALID_ARG: return "NVPA_ERR_INVALID_ARG";
        case NVPA_ERR_UNSUPPORTED: return "NVPA_ERR_UNSUPPORTED";
        case NVPA_ERR_CUDA: return "NVPA_ERR_CUDA";
        case NVPA_ERR_WORKSPACE_TOO_SMALL: return "NVPA_ERR_WORKSPACE_TOO_SMALL";
        default: return "NVPA_UNKNOWN_STATUS";
    }
}

const char* nvpa_last_error(void) { return g_last_error; }

uint64_t nvpa_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

nvpa_status_t nvpa_store_kvcache(const void* k, const void* v, int64_t k_token_stride,
                                 int64_t v_token_stride, void* k_cache, void* v_cache,
                                 const int32_t* slot_mapping, int num_tokens, int num_kv_heads,
                                 int head_dim, int num_blocks, int block_size, int32_t* err_flag,
                                 cudaStream_t stream) {
    g_last_error[0] = 0;
    NVPA_REQUIRE(num_tokens >= 0, NVPA_ERR_INVALID_ARG, "num_tokens < 0");
    NVPA_REQUIRE(num_kv_heads > 0 && head_dim > 0 && head_dim % 8 == 0, NVPA_ERR_INVALID_ARG,
                 "num_kv_heads must be positive and head_dim a positive multiple of 8");
    NVPA_REQUIRE(num_blocks > 0 && block_size > 0, NVPA_ERR_INVALID_ARG,
                 "num_blocks and block_size must be positive");
    NVPA_REQUIRE((long long)num_blocks * block_size <= 0x7fffffffLL, NVPA_ERR_UNSUPPORTED,
                 "pool of more than 2^31-1 slots");
    if (num_tokens == 0) return NVPA_OK;
    NVPA_REQUIRE(k && v && k_cache && v_cache && slot_mapping, NVPA_ERR_INVALID_ARG, "null pointer");
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    NVPA_REQUIRE(k_token_stride >= row && v_token_stride >= row, NVPA_ERR_INVALID_ARG,
                 "token stride smaller than num_kv_heads*head_dim");
    NVPA_REQUIRE(k_token_stride % 8 == 0 && v_token_stride % 8 == 0, NVPA_ERR_INVALID_ARG,
                 "token strides must be multiples of 8 elements (16 bytes)");
    NVPA_REQUIRE(aligned16(k) && aligned16(v) && aligned16(k_cache) && aligned16(v_cache),
                 NVPA_ERR_INVALID_ARG, "bf16 pointers must be 16-byte aligned");
    return run_store_kvcache(k, v, k_token_stride, v_token_stride, k_cache, v_cache, slot_mapping,
                             num_tokens, num_kv_heads, head_dim, num_blocks, block_size, err_flag,
                             stream);
}

size_t nvpa_paged_decode_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                        int max_context_len, int block_size, int num_splits) {
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
        num_splits < 0)
        return 0;
    return decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                  block_size, num_splits);
}

nvpa_status_t nvpa_paged_decode_attention(void* out, float* lse_out, const void* q,
                                          const void* k_cache, const void* v_cache,
                                          const int32_t* block_tables, int max_blocks_per_seq,
                                          const int32_t* context_lens, int batch, int num_q_heads,
                                          int num_kv_heads, int head_dim, int num_blocks,
                                          int block_size, int max_context_len, float softmax_scale,
                                          int num_splits, void* workspace, size_t workspace_bytes,
                                          int32_t* err_flag, cudaStream_t stream) {
    g_last_error[0] = 0;
    NVPA_REQUIRE(batch >= 0 && max_context_len >= 0 && num_splits >= 0, NVPA_ERR_INVALID_ARG,
                 "batch, max_context_len and num_splits must be >= 0");
    nvpa_status_t st = check_attention_shapes(num_q_heads, num_kv_heads, head_dim, num_blocks,
                                              block_size, max_blocks_per_seq);
    if (st != NVPA_OK) return st;
    NVPA_REQUIRE(std::isfinite(softmax_scale), NVPA_ERR_INVALID_ARG, "softmax_scale not finite");
    if (batch == 0) return NVPA_OK;
    NVPA_REQUIRE(out && q && k_cache && v_cache && block_tables && context_lens && workspace,
                 NVPA_ERR_INVALID_ARG, "null pointer");
    NVPA_REQUIRE(aligned16(out) && aligned16(q) && aligned16(k_cache) && aligned16(v_cache),
                 NVPA_ERR_INVALID_ARG, "bf16 pointers must be 16-byte aligned");
    NVPA_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, NVPA_ERR_INVALID_ARG,
                 "workspace must be 256-byte aligned");
    DecodeCall c{out, lse_out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                 batch, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, max_context_len,
                 softmax_scale, num_splits, workspace, workspace_bytes, err_flag};
    return run_paged_decode(c, stream);
}

static nvpa_status_t decode_step_common(void* out, float* lse_out, const void* q, const void* k_new,
                                        const void* v_new, int64_t k_token_stride, int64_t v_token_stride,
                                        void* k_cache, void* v_cache, const int32_t* slot_mapping,
                                        const int32_t* block_tables, int max_blocks_per_seq,
                                        const int32_t* context_lens, int batch, int num_q_heads,
                                        int num_kv_heads, int head_dim, int num_blocks, int block_size,
                                        int max_context_len, float softmax_scale, int num_splits,
                                        bool store_optional, int shared_prefix, int min_group,
                                        void* workspace, size_t workspace_bytes, int32_t* err_flag,
                                        cudaStream_t stream) {
    g_last_error[0] = 0;
    NVPA_REQUIRE(batch >= 0 && max_context_len >= 0 && num_splits >= 0 && min_group >= 0,
                 NVPA_ERR_INVALID_ARG, "batch, max_context_len, num_splits and min_group_size must be >= 0");
    nvpa_status_t st = check_attention_shapes(num_q_heads, num_kv_heads, head_dim, num_blocks,
                                              block_size, max_blocks_per_seq);
    if (st != NVPA_OK) return st;
    NVPA_REQUIRE(std::isfinite(softmax_scale), NVPA_ERR_INVALID_ARG, "softmax_scale not finite");
    if (batch == 0) return NVPA_OK;
    const bool any_new = k_new || v_new || slot_mapping;
    const bool all_new = k_new && v_new && slot_mapping;
    NVPA_REQUIRE(all_new || (store_optional && !any_new), NVPA_ERR_INVALID_ARG,
                 store_optional ? "k_new, v_new and slot_mapping must be all set or all null"
                                : "null pointer");
    NVPA_REQUIRE(out && q && k_cache && v_cache && block_tables && context_lens && workspace,
                 NVPA_ERR_INVALID_ARG, "null pointer");
    if (all_new) {
        const int64_t row = (int64_t)num_kv_heads * head_dim;
        NVPA_REQUIRE(k_token_stride >= row && v_token_stride >= row && k_token_stride % 8 == 0 &&
                         v_token_stride % 8 == 0,
                     NVPA_ERR_INVALID_ARG, "token strides must be >= num_kv_heads*head_dim and multiples of 8");
        NVPA_REQUIRE(aligned16(k_new) && aligned16(v_new), NVPA_ERR_INVALID_ARG,
                     "bf16 pointers must be 16-byte aligned");
    }
    NVPA_REQUIRE(aligned16(out) && aligned16(q) && aligned16(k_cache) && aligned16(v_cache),
                 NVPA_ERR_INVALID_ARG, "bf16 pointers must be 16-byte aligned");
    NVPA_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, NVPA_ERR_INVALID_ARG,
                 "workspace must be 256-byte aligned");
    DecodeCall c{out, lse_out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                 batch, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, max_context_len,
                 softmax_scale, num_splits, workspace, workspace_bytes, err_flag};
    if (all_new) {
        c.k_new = k_new;
        c.v_new = v_new;
        c.k_new_stride = k_token_stride;
        c.v_new_stride = v_token_stride;
        c.slot_mapping = slot_mapping;
    }
    c.shared_prefix = shared_prefix;
    c.min_group = min_group;
    return run_paged_decode(c, stream);
}

nvpa_status_t nvpa_decode_step(void* out, float* lse_out, const void* q, const void* k_new,
                               const void* v_new, int64_t k_token_stride, int64_t v_token_stride,
                               void* k_cache, void* v_cache, const int32_t* slot_mapping,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* context_lens, int batch, int num_q_heads,
                               int num_kv_heads, int head_dim, int num_blocks, int block_size,
                               int max_context_len, float softmax_scale, int num_splits,
                               void* workspace, size_t workspace_bytes, int32_t* err_flag,
                               cudaStream_t stream) {
    return decode_step_common(out, lse_out, q, k_new, v_new, k_token_stride, v_token_stride, k_cache,
                              v_cache, slot_mapping, block_tables, max_blocks_per_seq, context_lens,
                              batch, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size,
                              max_context_len, softmax_scale, num_splits, false, 0, 0, workspace,
                              workspace_bytes, err_flag, stream);
}

size_t nvpa_decode_shared_prefix_workspace_size(int batch, int num_q_heads, int num_kv_heads,
                                                int head_dim, int max_context_len, int block_size,
                                                int num_splits, int min_group_size) {
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
        num_splits < 0 || min_group_size < 0 || num_q_heads % num_kv_heads != 0)
        return 0;
    return decode_shared_prefix_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim,
                                                max_context_len, block_size, num_splits, min_group_size);
}

nvpa_status_t nvpa_decode_step_shared_prefix(
    void* out, float* lse_out, const void* q, const void* k_new, const void* v_new,
    int64_t k_token_stride, int64_t v_token_stride, void* k_cache, void* v_cache,
    const int32_t* slot_mapping, const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int batch, int num_q_heads, int num_kv_heads, int head_dim,
    int num_blocks, int block_size, int max_context_len, float softmax_scale, int num_splits,
    int min_group_size, void* workspace, size_t workspace_bytes, int32_t* err_flag,
    cudaStream_t stream) {
    return decode_step_common(out, lse_out, q, k_new, v_new, k_token_stride, v_token_stride, k_cache,
                              v_cache, slot_mapping, block_tables, max_blocks_per_seq, context_lens,
                              batch, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size,
                              max_context_len, softmax_scale, num_splits, true, 1, min_group_size,
                              workspace, workspace_bytes, err_flag, stream);
}

nvpa_status_t nvpa_paged_decode_partial(float* o_part, float* lse_part, const void* q,
                                        const void* k_cache, const void* v_cache,
                                        const int32_t* block_tables, int max_blocks_per_seq,
                                        const int32_t* context_lens, int batch, int num_q_heads,
                                        int num_kv_heads, int head_dim, int num_blocks,
                                        int block_size, int max_context_len, float softmax_scale,
                                        int num_splits, void* workspace, size_t workspace_bytes,
                                        int32_t* err_flag, cudaStream_t stream) {
    g_last_error[0] = 0;
    NVPA_REQUIRE(batch >= 0 && max_context_len >= 0 && num_splits >= 0, NVPA_ERR_INVALID_ARG,
                 "batch, max_context_len and num_splits must be >= 0");
    nvpa_status_t st = check_attention_shapes(num_q_heads, num_kv_heads, head_dim, num_blocks,
                                              block_size, max_blocks_per_seq);
    if (st != NVPA_OK) return st;
    NVPA_REQUIRE(std::isfinite(softmax_scale), NVPA_ERR_INVALID_ARG, "softmax_scale not finite");
    if (batch == 0) return NVPA_OK;
    NVPA_REQUIRE(o_part && lse_part && q && k_cache && v_cache && block_tables && context_lens && workspace,
                 NVPA_ERR_INVALID_ARG, "null pointer");
    NVPA_REQUIRE(aligned16(o_part) && aligned16(q) && aligned16(k_cache) && aligned16(v_cache),
                 NVPA_ERR_INVALID_ARG, "o_part and bf16 pointers must be 16-byte aligned");
    NVPA_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, NVPA_ERR_INVALID_ARG,
                 "workspace must be 256-byte aligned");
    DecodeCall c{o_part, lse_part, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                 batch, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, max_context_len,
                 softmax_scale, num_splits, workspace, workspace_bytes, err_flag};
    c.out_f32 = o_part;
    return run_paged_decode(c, stream);
}

nvpa_status_t nvpa_lse_combine(void* out, float* lse_out, const float* o_parts,
                               const float* lse_parts, int num_parts, int batch, int num_q_heads,
                               int head_dim, cudaStream_t stream) {
    g_last_error[0] = 0;
    NVPA_REQUIRE(num_parts >= 1 && batch >= 0 && num_q_heads > 0, NVPA_ERR_INVALID_ARG,
                 "num_parts must be >= 1, batch >= 0 and num_q_heads > 0");
    NVPA_REQUIRE(head_dim == 64 || head_dim == 128, NVPA_ERR_UNSUPPORTED,
                 "head_dim %d not supported (64, 128)", head_dim);
    NVPA_REQUIRE((long long)num_parts * batch * num_q_heads <= 0x7fffffffLL, NVPA_ERR_UNSUPPORTED,
                 "num_parts * batch * num_q_heads above 2^31-1");
    if (batch == 0) return NVPA_OK;
    NVPA_REQUIRE(out && o_parts && lse_parts, NVPA_ERR_INVALID_ARG, "null pointer");
    NVPA_REQUIRE(aligned16(out) && aligned16(o_parts), NVPA_ERR_INVALID_ARG,
                 "out and o_parts must be 16-byte aligned");
    return run_lse_combine(out, lse_out, o_parts, lse_parts, num_parts, batch, num_q_heads, head_dim,
                           stream);
}

size_t nvpa_varlen_prefill_workspace_size(int batch, int total_q) {
    if (batch < 0 || total_q < 0) return 0;
    return prefill_workspace_bytes(batch, total_q);
}

nvpa_status_t nvpa_varlen_prefill_attention(void* out, float* lse_out, const void* q,
                                            const void* k_cache, const void* v_cache,
                                            const int32_t* block_tables, int max_blocks_per_seq,
                                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                            int batch, int total_q, int max_seqlen_q,
                                            int max_seqlen_k, int num_q_heads, int num_kv_heads,
                                            int head_dim, int num_blocks, int block_size,
                                            float softmax_scale, int causal, void* workspace,
                                            size_t workspace_bytes, int32_t* err_flag,
                                            cudaStream_t stream) {
    g_last_error[0] = 0;
    NVPA_REQUIRE(batch >= 0 && total_q >= 0 && max_seqlen_q >= 0 && max_seqlen_k >= 0,
                 NVPA_ERR_INVALID_ARG, "sizes must be >= 0");
    NVPA_REQUIRE(causal == 0 || causal == 1, NVPA_ERR_INVALID_ARG, "causal must be 0 or 1");
    nvpa_status_t st = check_attention_shapes(num_q_heads, num_kv_heads, head_dim, num_blocks,
                                              block_size, max_blocks_per_seq);
    if (st != NVPA_OK) return st;
    NVPA_REQUIRE(std::isfinite(softmax_scale), NVPA_ERR_INVALID_ARG, "softmax_scale not finite");
    NVPA_REQUIRE((long long)total_q * num_kv_heads <= 0x7fffffffLL, NVPA_ERR_UNSUPPORTED,
                 "total_q * num_kv_heads above 2^31-1");
    if (batch == 0 || total_q == 0) return NVPA_OK;
    NVPA_REQUIRE(out && q && k_cache && v_cache && block_tables && cu_seqlens_q && cu_seqlens_k &&
                     workspace,
                 NVPA_ERR_INVALID_ARG, "null pointer");
    NVPA_REQUIRE(aligned16(out) && aligned16(q) && aligned16(k_cache) && aligned16(v_cache),
                 NVPA_ERR_INVALID_ARG, "bf16 pointers must be 16-byte aligned");
    NVPA_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, NVPA_ERR_INVALID_ARG,
                 "workspace must be 256-byte aligned");
    PrefillCall c{out, lse_out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, cu_seqlens_q,
                  cu_seqlens_k, batch, total_q, max_seqlen_q, max_seqlen_k, num_q_heads, num_kv_heads,
                  head_dim, num_blocks, block_size, softmax_scale, causal, err_flag};
    return run_varlen_prefill_tcgen05(c, workspace, workspace_bytes, stream);
}

nvpa_status_t nvpa_gather_kv(void* dst, const void* cache, const int32_t* block_tables,
                             int max_blocks_per_seq, const int32_t* cu_seqlens_k, int batch,
                             int total_k, int num_kv_heads, int head_dim, int num_blocks,
                             int block_size, int32_t* err_flag, cudaStream_t stream) {
    g_last_error[0] = 0;
    NVPA_REQUIRE(batch >= 0 && total_k >= 0, NVPA_ERR_INVALID_ARG, "sizes must be >= 0");
    NVPA_REQUIRE(num_kv_heads > 0 && head_dim > 0 && head_dim % 8 == 0, NVPA_ERR_INVALID_ARG,
                 "num_kv_heads must be positive and head_dim a positive multiple of 8");
    NVPA_REQUIRE(num_blocks > 0 && max_blocks_per_seq > 0, NVPA_ERR_INVALID_ARG,
                 "num_blocks and max_blocks_per_seq must be positive");
    NVPA_REQUIRE(pow2(block_size), NVPA_ERR_UNSUPPORTED, "block_size must be a power of two");
    if (batch == 0 || total_k == 0) return NVPA_OK;
    NVPA_REQUIRE(dst && cache && block_tables && cu_seqlens_k, NVPA_ERR_INVALID_ARG, "null pointer");
    NVPA_REQUIRE(aligned16(dst) && aligned16(cache), NVPA_ERR_INVALID_ARG,
                 "bf16 pointers must be 16-byte aligned");
    return run_gather_kv(dst, cache, block_tables, max_blocks_per_seq, cu_seqlens_k, batch, total_k,
                         num_kv_heads, head_dim, num_blocks, block_size, err_flag, stream);
}

nvpa_status_t nvpa_check_bounded_wait(int32_t* err_flag, cudaStream_t stream) {
    g_last_error[0] = 0;
    NVPA_REQUIRE(err_flag != nullptr, NVPA_ERR_INVALID_ARG, "err_flag must not be null");
    return run_bounded_wait_check(err_flag, stream);
}

}  // extern "C"
