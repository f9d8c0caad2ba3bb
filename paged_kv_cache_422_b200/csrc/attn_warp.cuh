// One warp, one KV head, up to GMAX query heads of the same group, a 16-key tile of K and
// V in shared memory: the CUDA-core inner loop of paged attention.
//
// Decode attention does 2*g flops per byte of K/V it reads (g = query heads per KV
// head, 1..8), far below the tensor-core ridge point, so it runs on the CUDA cores and
// is bound by HBM bandwidth; the job of this loop is to keep the issue cost per key low
// enough that the loads, not the arithmetic, set the pace.
//
// Lane layout.  A key row of head_dim D bf16 values is D/8 chunks of 16 bytes.  LPR = D/8
// lanes hold one row (lane `sub` owns dims 8*sub .. 8*sub+7); RPI = 32/LPR rows are
// covered per warp instruction; a 16-key tile takes ITER = 16/RPI = LPR/2 instructions.
// QK: every lane forms partial dot products over its 8 dims for its ITER rows; a
// transpose-reduction across the LPR lanes of a row group (log2(LPR) shuffle rounds that
// halve the number of live values each round) leaves lane `sub` holding the full score of
// row RPI*(sub>>1) + grp, where grp = lane / LPR.  Softmax statistics are warp-wide; the
// PV step broadcasts each row's weight from its owner lane and accumulates o over the
// lane's 8 dims.  Scores are kept in the log2 domain (q is pre-scaled by
// softmax_scale * log2(e)) so that the exponentials are single ex2 instructions.
#pragma once

#include "common.cuh"

namespace nvpa {

constexpr int kTileKeys = 16;

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int D, int GMAX>
struct WarpAttnState {
    static constexpr int LPR = D / 8;
    static constexpr int RPI = 32 / LPR;
    static constexpr int ITER = kTileKeys / RPI;
    static_assert(ITER * 2 == LPR, "tile shape assumes 16 keys = RPI * LPR / 2");

    float q[GMAX][8];   // this lane's 8 dims of each query head, scaled to log2 units
    float o[GMAX][8];   // running un-normalised output for the same dims
    float m[GMAX];      // running max (log2 units), warp-uniform
    float l[GMAX];      // running sum of weights, this lane's share

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) o[g][k] = 0.f;
        }
    }

    // q_smem: [G][D] bf16 of the group's query heads.
    __device__ __forceinline__ void load_q(const uint16_t* q_smem, int G, int sub, float scale_log2) {
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            float f[8];
            if (g < G) {
                uint4 u = *reinterpret_cast<const uint4*>(q_smem + g * D + sub * 8);
                unpack8(u, f);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) f[k] = 0.f;
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) q[g][k] = f[k] * scale_log2;
        }
    }

    // One halving round of the transpose-reduction: N live values, partner at lane ^ OFF.
    template <int N, int OFF>
    __device__ __forceinline__ static void reduce_round(float (&v)[GMAX][ITER], int sub) {
        const bool upper = (sub & OFF) != 0;
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
#pragma unroll
            for (int j = 0; j < N / 2; ++j) {
                float lo = v[g][j], hi = v[g][j + N / 2];
                float send = upper ? lo : hi;
                float keep = upper ? hi : lo;
                v[g][j] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
            }
        }
    }

    // Consume one tile.  ks/vs: [16][D] bf16 rows in shared memory; rows >= rows_valid
    // are masked out.  Their shared-memory content must be finite (the loaders zero-fill
    // them) because V rows are multiplied by a zero weight.
    __device__ __forceinline__ void consume(const uint16_t* ks, const uint16_t* vs, int rows_valid,
                                            int lane) {
        const int grp = lane / LPR;
        const int sub = lane % LPR;
        float part[GMAX][ITER];
#pragma unroll
        for (int i = 0; i < ITER; ++i) {
            const int row = grp + RPI * i;
            uint4 u = *reinterpret_cast<const uint4*>(ks + row * D + sub * 8);
            float f[8];
            unpack8(u, f);
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
                float acc = q[g][0] * f[0];
#pragma unroll
                for (int k = 1; k < 8; ++k) acc = fmaf(q[g][k], f[k], acc);
                part[g][i] = acc;
            }
        }
        // transpose-reduce: LPR/2 .. 2 halve the live values, the final round (offset 1)
        // completes the sum inside each lane pair.
        if constexpr (ITER >= 8) reduce_round<8, LPR / 2>(part, sub);
        if constexpr (ITER >= 4) reduce_round<4, (ITER >= 8 ? LPR / 4 : LPR / 2)>(part, sub);
        reduce_round<2, 2>(part, sub);
#pragma unroll
        for (int g = 0; g < GMAX; ++g) part[g][0] += __shfl_xor_sync(0xffffffffu, part[g][0], 1);

        const int my_row = grp + RPI * (sub >> 1);
        const bool row_ok = my_row < rows_valid;
        float p[GMAX];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            const float s = row_ok ? part[g][0] : -INFINITY;
            const float m_new = fmaxf(m[g], warp_max(s));
            float alpha, pg;
            if (m_new == -INFINITY) {
                alpha = 1.f;
                pg = 0.f;
            } else {
                alpha = fast_exp2(m[g] - m_new);
                pg = row_ok ? fast_exp2(s - m_new) : 0.f;
            }
            p[g] = pg;
            l[g] = l[g] * alpha + ((sub & 1) ? 0.f : pg);
            m[g] = m_new;
            if (alpha != 1.f) {
#pragma unroll
                for (int k = 0; k < 8; ++k) o[g][k] *= alpha;
            }
        }
#pragma unroll
        for (int i = 0; i < ITER; ++i) {
            const int row = grp + RPI * i;
            const int owner = grp * LPR + 2 * i;
            float w[GMAX];
#pragma unroll
            for (int g = 0; g < GMAX; ++g) w[g] = __shfl_sync(0xffffffffu, p[g], owner);
            uint4 u = *reinterpret_cast<const uint4*>(vs + row * D + sub * 8);
            float f[8];
            unpack8(u, f);
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
#pragma unroll
                for (int k = 0; k < 8; ++k) o[g][k] = fmaf(w[g], f[k], o[g][k]);
            }
        }
    }

    // Fold the RPI row groups together and total l.  Afterwards every lane with the same
    // `sub` holds the full un-normalised o for dims 8*sub..8*sub+7 and every lane holds
    // the warp total of l (per head).
    __device__ __forceinline__ void finish() {
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
#pragma unroll
                for (int k = 0; k < 8; ++k) o[g][k] += __shfl_xor_sync(0xffffffffu, o[g][k], off);
            }
        }
#pragma unroll
        for (int g = 0; g < GMAX; ++g) l[g] = warp_sum(l[g]);
    }

    // Natural-log sum-exp of head g after finish(); -inf when no key was seen.
    __device__ __forceinline__ float lse(int g) const {
        return l[g] > 0.f ? (m[g] + log2f(l[g])) * kLn2 : -INFINITY;
    }
};

}  // namespace nvpa
