// Host-side declarations shared by the nvpa translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "nvpa.h"

namespace nvpa {

// printf-style message stored for nvpa_last_error() on the calling thread.
void set_error(const char* fmt, ...);
nvpa_status_t cuda_failure(cudaError_t e, const char* what);
int device_sm_count();
// Adds n to the process-wide count of kernels enqueued by the library.
void count_launches(int n);

struct DecodeCall {
    void* out;
    float* lse_out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    int max_blocks_per_seq;
    const int32_t* context_lens;
    int batch, hq, hkv, head_dim, num_blocks, block_size, max_context_len;
    float scale;
    int num_splits;
    void* workspace;
    size_t workspace_bytes;
    int32_t* err_flag;
    // fused decode step (nvpa_decode_step); k_new == nullptr for plain decode
    const void* k_new = nullptr;
    const void* v_new = nullptr;
    long long k_new_stride = 0, v_new_stride = 0;
    const int32_t* slot_mapping = nullptr;
    // shared-prefix decode (nvpa_decode_step_shared_prefix): group sequences whose block
    // tables start with the same blocks and attend each group's prefix once
    int shared_prefix = 0;
    int min_group = 0;
    // partial decode (nvpa_paged_decode_partial): fp32 normalised output here, `out` unused
    float* out_f32 = nullptr;
};

struct PrefillCall {
    void* out;
    float* lse_out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    int max_blocks_per_seq;
    const int32_t* cu_seqlens_q;
    const int32_t* cu_seqlens_k;
    int batch, total_q, max_seqlen_q, max_seqlen_k;
    int hq, hkv, head_dim, num_blocks, block_size;
    float scale;
    int causal;
    int32_t* err_flag;
};

// Shared-prefix part of a decode: every group's members (query rows) against the group's
// prefix keys on the tensor cores; partition c of a prefix lands in slot c of each member's
// split-KV partials.  The tables come from the decode plan (the kernel waits for it).
struct DecodePrefixArgs {
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    int max_blocks_per_seq;
    int batch, hq, hkv, head_dim, num_blocks, block_size;
    float scale;
    int32_t* err_flag;
    const int4* tiles;           // (group, query tile A, query tile B or -1, partition)
    const int32_t* ntiles;
    int32_t* unit_counter;       // zeroed by the plan; the kernel claims work units from it
    const int32_t* members;
    const int32_t* group_start;
    const int32_t* group_len;
    float* o_part;
    float* lse_part;
    int s_max, pchunk;
    long long max_entries;       // host bound on the number of tile entries
    int max_ctas;                // grid cap (0: one per SM)
    bool pdl;                    // launch as a programmatic dependent of the previous kernel
};
// Query heads that share one 128-row tensor-core tile (the group size when it is a power
// of two up to 8, else 1).
int attention_tile_pack(int hq, int hkv);
cudaError_t launch_decode_prefix_tcgen05(const DecodePrefixArgs& a, cudaStream_t stream);

int decode_chunk_keys(int batch, int num_kv_heads, int max_context_len, int block_size, int num_splits);
size_t decode_workspace_bytes(int batch, int hq, int hkv, int head_dim, int max_context_len,
                              int block_size, int num_splits);
size_t decode_shared_prefix_workspace_bytes(int batch, int hq, int hkv, int head_dim,
                                            int max_context_len, int block_size, int num_splits,
                                            int min_group);
nvpa_status_t run_paged_decode(const DecodeCall& c, cudaStream_t stream);
size_t prefill_workspace_bytes(int batch, int total_q);
nvpa_status_t run_varlen_prefill_tcgen05(const PrefillCall& c, void* workspace, size_t workspace_bytes,
                                         cudaStream_t stream);

nvpa_status_t run_lse_combine(void* out, float* lse_out, const float* o_parts, const float* lse_parts,
                              int num_parts, int batch, int hq, int head_dim, cudaStream_t stream);

nvpa_status_t run_store_kvcache(const void* k, const void* v, int64_t k_stride, int64_t v_stride,
                                void* k_cache, void* v_cache, const int32_t* slot_mapping,
                                int num_tokens, int hkv, int head_dim, int num_blocks,
                                int block_size, int32_t* err_flag, cudaStream_t stream);
nvpa_status_t run_gather_kv(void* dst, const void* cache, const int32_t* block_tables,
                            int max_blocks_per_seq, const int32_t* cu_seqlens_k, int batch,
                            int total_k, int hkv, int head_dim, int num_blocks, int block_size,
                            int32_t* err_flag, cudaStream_t stream);
nvpa_status_t run_bounded_wait_check(int32_t* err_flag, cudaStream_t stream);

}  // namespace nvpa
