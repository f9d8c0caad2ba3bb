// Split-KV combine of the paged decode: merge the partitions of every (sequence, query
// head) that has more than one, with their log-sum-exp weights
//     lse = log sum_p exp(lse_p),   out = sum_p exp(lse_p - lse) * o_p
// (o_p normalised over partition p's keys).  W warps per (sequence, query head), W = 1,
// 2, 4 or 8 chosen on the host so that few rows with many partitions (long contexts,
// small batches) still spread over the whole GPU: every warp of a row finds the row's
// largest lse, sums its own share of the partitions, and the row's first warp adds the
// shares up through shared memory.  Each lane owns head_dim / 32 consecutive dims;
// kCombineLoads partitions are read at a time, so a warp's share is not bound by load
// latency either.
#include "decode_params.cuh"

namespace nvpa {

namespace {

constexpr int kCombineLoads = 8;
constexpr int kCombineWarps = 8;   // warps per CTA

template <int D, int W>
__global__ void __launch_bounds__(kCombineWarps * 32, 4) decode_combine_kernel(const AttnParams p) {
    constexpr int DPL = D / 32;   // output dims per lane
    constexpr int R = kCombineWarps / W;   // rows per CTA
    __shared__ float red[kCombineWarps][D];
    __shared__ float red_tot[kCombineWarps];
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w = blockIdx.x * R + warp / W;   // row: sequence * hq + query head
    const int part = warp % W;                 // this warp's share of the row's partitions
    const bool row_ok = w < p.batch * p.hq;
    const int b = row_ok ? w / p.hq : 0;
    const float* lp = p.lse_part + (size_t)(row_ok ? w : 0) * p.s_max;
    // the row's first 32 lse slots are read together with its partition count (slots past
    // the count hold stale values and are dropped below), saving a dependent round of loads
    const float lse0 = (row_ok && lane < p.s_max) ? __ldcg(lp + lane) : -INFINITY;
    const int ns = row_ok ? __ldcg(p.nsplit + b) : 0;
    // (no early return: the shares of a row meet at the barrier below)
    const bool merge = ns > 1;
    float acc[DPL];
#pragma unroll
    for (int k = 0; k < DPL; ++k) acc[k] = 0.f;
    float tot = 0.f, mx = -INFINITY;
    if (merge) {
        const float* op = p.o_part + (size_t)w * p.s_max * D + lane * DPL;
        mx = lane < ns ? lse0 : -INFINITY;
        for (int s = lane + 32; s < ns; s += 32) mx = fmaxf(mx, __ldcg(lp + s));
        mx = warp_max(mx);
        const int per = (ns + W - 1) / W;
        const int s_begin = min(ns, part * per), s_end = min(ns, s_begin + per);
        if (mx > -INFINITY) {
            for (int s0 = s_begin; s0 < s_end; s0 += 32) {
                // (the shuffle runs in every lane: s0 is the same across the warp)
                const float sh = __shfl_sync(0xffffffffu, lse0, (s0 + lane) & 31);
                const float ls = s0 + lane < s_end ? (s0 + lane < 32 ? sh : __ldcg(lp + s0 + lane)) : -INFINITY;
                const float wl = (s0 + lane < s_end) ? fast_exp2((ls - mx) * kLog2e) : 0.f;
                tot += wl;
                const int n = min(32, s_end - s0);
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
    }
    if constexpr (W > 1) {
        // the row's first warp adds up the W shares
#pragma unroll
        for (int k = 0; k < DPL; ++k) red[warp][lane * DPL + k] = acc[k];
        if (lane == 0) red_tot[warp] = tot;
        __syncthreads();
        if (part != 0) return;
#pragma unroll
        for (int q = 1; q < W; ++q) {
#pragma unroll
            for (int k = 0; k < DPL; ++k) acc[k] += red[warp + q][lane * DPL + k];
            tot += red_tot[warp + q];
        }
    }
    if (!merge) return;
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

template <int D>
cudaError_t launch_combine_d(const AttnParams& p, int w_per_row, cudaStream_t stream) {
    const long long rows = (long long)p.batch * p.hq;
    const int r = kCombineWarps / w_per_row;
    const dim3 grid((unsigned)((rows + r - 1) / r)), block(kCombineWarps * 32);
    switch (w_per_row) {
        case 8: return launch_pdl(decode_combine_kernel<D, 8>, grid, block, 0, stream, p);
        case 4: return launch_pdl(decode_combine_kernel<D, 4>, grid, block, 0, stream, p);
        case 2: return launch_pdl(decode_combine_kernel<D, 2>, grid, block, 0, stream, p);
        default: return launch_pdl(decode_combine_kernel<D, 1>, grid, block, 0, stream, p);
    }
}

}  // namespace

// Warps per (sequence, query head): enough that the combine has about two CTAs of 8
// warps per SM of a 148-SM B200, never more than the partitions a row can have.
int decode_combine_warps_per_row(long long rows, int s_max) {
    constexpr long long kTargetWarps = 148LL * 2 * kCombineWarps;
    int w = 1;
    while (w < kCombineWarps && rows * (2 * w) <= kTargetWarps && 2 * w <= s_max) w *= 2;
    return w;
}

cudaError_t launch_decode_combine(const AttnParams& p, int head_dim, cudaStream_t stream) {
    const int w = decode_combine_warps_per_row((long long)p.batch * p.hq, p.s_max);
    return head_dim == 128 ? launch_combine_d<128>(p, w, stream) : launch_combine_d<64>(p, w, stream);
}

}  // namespace nvpa
