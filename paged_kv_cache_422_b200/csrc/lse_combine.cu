// Merge of attention partials computed over disjoint key ranges (split-KV across calls or
// devices): for every (sequence, query head) row w with parts r = 0 .. R-1,
//     lse = log sum_r exp(lse_r),   out = sum_r exp(lse_r - lse) * o_r
// where o_r is part r's output normalised over its own keys and lse_r its log-sum-exp
// (-inf for a part with no keys, which then weighs 0).  This is the log-sum-exp merge of
// the split-KV decode ("Nano-vLLM part 1" section 5.2 decode over the cached tokens, cut
// into partitions) applied to partials that another GPU computed.
//
// One warp per row; each lane owns head_dim / 32 consecutive dims.  The parts' lse values
// are read by every lane (R is small: one part per device), the outputs with 8- or
// 16-byte loads.
#include "attn_warp.cuh"
#include "nvpa_internal.h"

namespace nvpa {

namespace {

template <int D>
__global__ void __launch_bounds__(256) lse_combine_kernel(uint16_t* __restrict__ out, float* __restrict__ lse_out,
                                                          const float* __restrict__ o_parts,
                                                          const float* __restrict__ lse_parts, int num_parts,
                                                          int rows) {
    constexpr int DPL = D / 32;
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= rows) return;
    float mx = -INFINITY;
    for (int r = 0; r < num_parts; ++r) mx = fmaxf(mx, __ldg(lse_parts + (size_t)r * rows + w));
    float acc[DPL];
#pragma unroll
    for (int k = 0; k < DPL; ++k) acc[k] = 0.f;
    float tot = 0.f;
    if (mx > -INFINITY) {
        for (int r = 0; r < num_parts; ++r) {
            const float wr = fast_exp2((__ldg(lse_parts + (size_t)r * rows + w) - mx) * kLog2e);
            tot += wr;
            const float* src = o_parts + ((size_t)r * rows + w) * D + lane * DPL;
            float v[DPL];
            if constexpr (DPL == 4) {
                const float4 t = __ldg(reinterpret_cast<const float4*>(src));
                v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
            } else {
                const float2 t = __ldg(reinterpret_cast<const float2*>(src));
                v[0] = t.x; v[1] = t.y;
            }
#pragma unroll
            for (int k = 0; k < DPL; ++k) acc[k] = fmaf(wr, v[k], acc[k]);
        }
    }
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
    uint16_t* dst = out + (size_t)w * D + lane * DPL;
    if constexpr (DPL == 4) {
        uint2 v;
        v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2*>(dst) = v;
    } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
    if (lane == 0 && lse_out != nullptr) lse_out[w] = tot > 0.f ? mx + __logf(tot) : -INFINITY;
}

}  // namespace

nvpa_status_t run_lse_combine(void* out, float* lse_out, const float* o_parts, const float* lse_parts,
                              int num_parts, int batch, int hq, int head_dim, cudaStream_t stream) {
    const long long rows = (long long)batch * hq;
    const int grid = (int)((rows + 7) / 8);
    uint16_t* o = static_cast<uint16_t*>(out);
    if (head_dim == 128)
        lse_combine_kernel<128><<<grid, 256, 0, stream>>>(o, lse_out, o_parts, lse_parts, num_parts, (int)rows);
    else
        lse_combine_kernel<64><<<grid, 256, 0, stream>>>(o, lse_out, o_parts, lse_parts, num_parts, (int)rows);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_failure(e, "lse combine launch");
    count_launches(1);
    return NVPA_OK;
}

}  // namespace nvpa
