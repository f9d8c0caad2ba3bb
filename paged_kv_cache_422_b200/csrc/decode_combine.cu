// Split-KV combine of the paged decode: merge the partitions of every (sequence, query
// head) that has more than one, with their log-sum-exp weights
//     lse = log sum_p exp(lse_p),   out = sum_p exp(lse_p - lse) * o_p
// (o_p normalised over partition p's keys).  One warp per (sequence, query head); each
// lane owns head_dim / 32 consecutive dims; kCombineLoads partitions are read at a time
// so that long contexts (a hundred partitions and more) are not bound by load latency.
#include "decode_params.cuh"

namespace nvpa {

namespace {

constexpr int kCombineLoads = 8;

template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const AttnParams p) {
    constexpr int DPL = D / 32;   // output dims per lane
    pdl_wait();
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= p.batch * p.hq) return;
    const int b = w / p.hq;
    const int ns = __ldcg(p.nsplit + b);
    if (ns <= 1) return;
    const float* lp = p.lse_part + (size_t)w * p.s_max;
    const float* op = p.o_part + (size_t)w * p.s_max * D + lane * DPL;
    float mx = -INFINITY;
    for (int s = lane; s < ns; s += 32) mx = fmaxf(mx, __ldcg(lp + s));
    mx = warp_max(mx);
    float acc[DPL];
#pragma unroll
    for (int k = 0; k < DPL; ++k) acc[k] = 0.f;
    float tot = 0.f;
    if (mx > -INFINITY) {
        for (int s0 = 0; s0 < ns; s0 += 32) {
            const float wl = (s0 + lane < ns) ? fast_exp2((__ldcg(lp + s0 + lane) - mx) * kLog2e) : 0.f;
            tot += wl;
            const int n = min(32, ns - s0);
            int j = 0;
            for (; j + kCombineLoads <= n; j += kCombineLoads) {   // independent loads in flight
                float ws[kCombineLoads];
                float v[kCombineLoads][DPL];
#pragma unroll
                for (int u = 0; u < kCombineLoads; ++u) {
                    ws[u] = __shfl_sync(0xffffffffu, wl, j + u);
                    const float* src = op + (size_t)(s0 + j + u) * D;
                    if constexpr (DPL == 4) {
                        const float4 t = __ldcg(reinterpret_cast<const float4*>(src));
                        v[u][0] = t.x; v[u][1] = t.y; v[u][2] = t.z; v[u][3] = t.w;
                    } else {
                        const float2 t = __ldcg(reinterpret_cast<const float2*>(src));
                        v[u][0] = t.x; v[u][1] = t.y;
                    }
                }
#pragma unroll
                for (int u = 0; u < kCombineLoads; ++u)
#pragma unroll
                    for (int k = 0; k < DPL; ++k) acc[k] = fmaf(ws[u], v[u][k], acc[k]);
            }
            for (; j < n; ++j) {
                const float ws = __shfl_sync(0xffffffffu, wl, j);
                const float* src = op + (size_t)(s0 + j) * D;
#pragma unroll
                for (int k = 0; k < DPL; ++k) acc[k] = fmaf(ws, __ldcg(src + k), acc[k]);
            }
        }
        tot = warp_sum(tot);
    }
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
    if (p.out_f32 != nullptr) {
        float* dst = p.out_f32 + (size_t)w * D + lane * DPL;
#pragma unroll
        for (int k = 0; k < DPL; ++k) dst[k] = acc[k] * inv;
        if (lane == 0 && p.lse_out != nullptr) p.lse_out[w] = tot > 0.f ? mx + __logf(tot) : -INFINITY;
        return;
    }
    uint16_t* dst = p.out + (size_t)w * D + lane * DPL;
    if constexpr (DPL == 4) {
        uint2 v;
        v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2*>(dst) = v;
    } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
    if (lane == 0 && p.lse_out != nullptr) p.lse_out[w] = tot > 0.f ? mx + __logf(tot) : -INFINITY;
}


}  // namespace

cudaError_t launch_decode_combine(const AttnParams& p, int head_dim, int grid, cudaStream_t stream) {
    return head_dim == 128 ? launch_pdl(decode_combine_kernel<128>, dim3(grid), dim3(256), 0, stream, p)
                           : launch_pdl(decode_combine_kernel<64>, dim3(grid), dim3(256), 0, stream, p);
}

}  // namespace nvpa
