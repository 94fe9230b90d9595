// tq_common.cuh -- record layout and small device helpers shared by the
// TQ4/4 kernels (append, decode, combine, dequantise).
//
// Record of one (physical block, kv head), 16 tokens, head_dim D:
//   [0, 8D)           key codes    [16][D/2] bytes, element 2j in the low nibble of byte j
//   [8D, 8D+32)       key norms    [16] fp16
//   [8D+32, 16D+32)   value codes  8D bytes, same nibble order, placed for the decode
//                     fragments: byte j = 8m + r of token t sits in chunk (D/8 bytes)
//                     8 (t/2) + ((r + 2 (t/2)) mod 8), at byte 4 (m/2) + 2 (t%2) + (m%2)
//                     of it (the rotation of a token pair's 8 chunks by 2 (t/2) puts
//                     the chunks that one quarter warp of the decode reads in 8
//                     different bank groups)
//   [16D+32, 17D+32)  value scales fp16, the one of token t, group G at byte
//                     2 (4 (c (D/32) + G) + u), c = (t%8)/2, u = 2 (t/8) + t%2
//   [17D+32, 18D+32)  value zeros  fp16, same placement
// The cache is [num_blocks][H_kv][record]; every field starts 16-byte aligned.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tq.h"

namespace tq {

constexpr int kBlock = 16;  // tokens per cache block
constexpr int kGroup = 32;  // value elements per scale/zero group
constexpr unsigned kFull = 0xffffffffu;

template <int D>
struct Rec {
    static constexpr int kCodeRow = D / 2;                        // bytes of one token's codes
    static constexpr int kKCodes = 0;
    static constexpr int kKNorm = kBlock * kCodeRow;               // 8D
    static constexpr int kVCodes = kKNorm + 2 * kBlock;            // 8D + 32
    static constexpr int kVScale = kVCodes + kBlock * kCodeRow;    // 16D + 32
    static constexpr int kVZero = kVScale + D;                     // 17D + 32
    static constexpr int kGroups = D / kGroup;
    static constexpr int kBytes = kVZero + D;                      // 18D + 32
    static constexpr int kPairChunk = D / 8;  // value bytes of one (token pair, r) chunk
    // value byte j of token t, relative to kVCodes
    static __host__ __device__ constexpr int vcode_pos(int t, int j) {
        return (8 * (t >> 1) + (((j & 7) + 2 * (t >> 1)) & 7)) * kPairChunk + 4 * ((j >> 3) >> 1) +
               2 * (t & 1) + ((j >> 3) & 1);
    }
    // scale (zero) of token t, group G, relative to kVScale (kVZero)
    static __host__ __device__ constexpr int group_pos(int t, int G) {
        return 2 * (4 * (((t & 7) >> 1) * kGroups + G) + 2 * (t >> 3) + (t & 1));
    }
    static_assert(D % 32 == 0, "head_dim must be a multiple of 32");
    static_assert(kKNorm % 16 == 0 && kVCodes % 16 == 0 && kVScale % 16 == 0 &&
                      kVZero % 16 == 0 && kBytes % 16 == 0,
                  "record fields must stay 16-byte aligned");
};

// bf16 pair (packed in a uint32, element 0 in the low half) -> two floats, exact
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

// streaming 16-byte read-only load (inputs are read once)
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// n / d for n < 2^32 with M = (2^64 - 1) / d + 1 (exact: the error term of
// n * M / 2^64 stays below 2^-32 < 1/d); d == 1 is flagged by M == 0.
__device__ __forceinline__ uint32_t fast_div(uint32_t n, uint64_t M) {
    return M ? (uint32_t)__umul64hi((uint64_t)n, M) : n;
}
// the multiplier of fast_div for divisor d (0 for d == 1)
inline uint64_t div_magic(uint32_t d) { return d <= 1 ? 0 : ~0ull / d + 1; }

// n / d for n < 2^31 with one 32 x 32 -> 64-bit multiply: floor(n m / 2^s),
// s = 31 + ceil(log2 d), m = ceil(2^s / d) < 2^32 (m d - 2^s < d <= 2^(s-31),
// the round-up condition under which the quotient is exact for 31-bit n).
struct Div32 {
    uint32_t m, s;
};
__device__ __forceinline__ uint32_t fast_div32(uint32_t n, Div32 d) {
    return (uint32_t)(((uint64_t)n * d.m) >> d.s);
}
inline Div32 div32_magic(uint32_t d) {
    uint32_t l = 0;
    while ((1ull << l) < d) l++;
    const uint32_t s = 31 + l;
    return Div32{(uint32_t)(((1ull << s) + d - 1) / d), s};
}

__device__ __forceinline__ void flag_status(int32_t* status, int bits) {
    if (status) atomicOr(status, bits);
}

// Correctly rounded double -> fp16 toward +infinity, for x >= 0.
__device__ __forceinline__ uint16_t double_to_half_up_nonneg(double x) {
    __half h = __double2half(x);  // round to nearest even
    uint16_t b = __half_as_ushort(h);
    if ((double)__half2float(h) < x) b = (uint16_t)(b + 1);  // next representable above
    return b;
}

}  // namespace tq
