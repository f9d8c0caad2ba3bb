// Device helpers shared by the nvpa kernels: bf16 unpacking, cp.async wrappers and the
// paged address computation (slot = block * block_size + row).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nvpa.h"

namespace nvpa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// The high and low bf16 halves of a packed pair, widened to float32 exactly.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
    f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x);
    f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
    f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z);
    f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

// Two float32 values rounded (nearest-even) to bf16 and packed low|high.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global->shared copy; src_bytes = 0 fills the destination with
// zeros without reading the source.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
                 :: "r"(smem_u32(smem_dst)), "l"(gmem_src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" :: "n"(N) : "memory");
}

__device__ __forceinline__ void flag_error(int32_t* err_flag, int bits) {
    if (err_flag != nullptr) atomicOr(err_flag, bits);
}

// Physical block of logical position `pos` of a sequence, or -1 (flagged) when the
// table entry is outside [0, num_blocks).  Table entries past the sequence's last
// block are never passed here.
__device__ __forceinline__ int checked_block(const int32_t* bt_row, int pos, int block_shift,
                                             int num_blocks, int32_t* err_flag) {
    int blk = __ldg(bt_row + (pos >> block_shift));
    if (blk < 0 || blk >= num_blocks) {
        flag_error(err_flag, NVPA_FLAG_BAD_BLOCK_ID);
        return -1;
    }
    return blk;
}

}  // namespace nvpa
