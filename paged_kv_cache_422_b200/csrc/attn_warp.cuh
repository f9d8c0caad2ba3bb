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
constexpr float kRescaleSlack = 8.0f;   // log2 units

// Packed pairs of float32 in one 64-bit register pair; sm_100 executes the .f32x2 forms
// of fma/mul as single instructions, halving the FMA count of the inner loops.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// A packed bf16 pair (low half = element 2j, high half = element 2j+1) widened exactly.
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
    return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

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

    uint64_t q[GMAX][4];  // this lane's 8 dims of each query head as 4 packed pairs, in log2 units
    uint64_t o[GMAX][4];  // running un-normalised output for the same dims, packed pairs
    float m[GMAX];        // running max (log2 units), warp-uniform
    float l[GMAX];        // running sum of weights, this lane's share

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) o[g][k] = 0ull;
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
            for (int k = 0; k < 4; ++k) q[g][k] = f2_pack(f[2 * k] * scale_log2, f[2 * k + 1] * scale_log2);
        }
    }

    // Output dims 8*sub + 2k, 8*sub + 2k + 1 of head g.
    __device__ __forceinline__ void out_pair(int g, int k, float& lo, float& hi) const {
        f2_unpack(o[g][k], lo, hi);
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
            const uint4 u = *reinterpret_cast<const uint4*>(ks + row * D + sub * 8);
            const uint64_t kp[4] = {bf16x2_to_f2(u.x), bf16x2_to_f2(u.y), bf16x2_to_f2(u.z),
                                    bf16x2_to_f2(u.w)};
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
                uint64_t acc = f2_mul(q[g][0], kp[0]);
                acc = f2_fma(q[g][1], kp[1], acc);
                acc = f2_fma(q[g][2], kp[2], acc);
                acc = f2_fma(q[g][3], kp[3], acc);
                float lo, hi;
                f2_unpack(acc, lo, hi);
                part[g][i] = lo + hi;
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
        // Lazy rescaling: weights are exp2(s - m) against a reference max m that moves only
        // when some score exceeds it by more than kRescaleSlack (then o and l are rescaled).
        // Weights stay below 2^kRescaleSlack, far from fp32 overflow, and the final o / l
        // does not depend on which reference was used.  One warp vote replaces the per-tile
        // max reduction in the common case.
        float sc[GMAX];
        bool over = false;
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            sc[g] = row_ok ? part[g][0] : -INFINITY;
            over |= sc[g] > m[g] + kRescaleSlack;
        }
        if (__any_sync(0xffffffffu, over)) {
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
                const float m_new = fmaxf(m[g], warp_max(sc[g]));
                if (m_new > m[g]) {
                    const float alpha = fast_exp2(m[g] - m_new);   // 0 when m was -inf
                    l[g] *= alpha;
                    const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[g][k] = f2_mul(o[g][k], a2);
                    m[g] = m_new;
                }
            }
        }
        float p[GMAX];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            // rows past the range and heads that saw no key yet contribute exactly zero
            const float pg = (row_ok && m[g] > -INFINITY) ? fast_exp2(sc[g] - m[g]) : 0.f;
            p[g] = pg;
            l[g] += (sub & 1) ? 0.f : pg;
        }
#pragma unroll
        for (int i = 0; i < ITER; ++i) {
            const int row = grp + RPI * i;
            const int owner = grp * LPR + 2 * i;
            const uint4 u = *reinterpret_cast<const uint4*>(vs + row * D + sub * 8);
            const uint64_t vp[4] = {bf16x2_to_f2(u.x), bf16x2_to_f2(u.y), bf16x2_to_f2(u.z),
                                    bf16x2_to_f2(u.w)};
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
                const float w = __shfl_sync(0xffffffffu, p[g], owner);
                const uint64_t w2 = f2_pack(w, w);
#pragma unroll
                for (int k = 0; k < 4; ++k) o[g][k] = f2_fma(w2, vp[k], o[g][k]);
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
                for (int k = 0; k < 4; ++k) {
                    float lo, hi;
                    f2_unpack(o[g][k], lo, hi);
                    lo += __shfl_xor_sync(0xffffffffu, lo, off);
                    hi += __shfl_xor_sync(0xffffffffu, hi, off);
                    o[g][k] = f2_pack(lo, hi);
                }
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
