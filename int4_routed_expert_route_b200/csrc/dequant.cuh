// dequant.cuh -- register-level decoding of packed int4 / int8 / int2 codes
// into exact fp32 values q * 2^e, shared by the CUDA-core GEMV kernels.
//
// A code c of b bits is placed into the mantissa of 2^23 (float bits
// 0x4B000000 | c << e, exact while c << e < 2^23); one packed f32x2
// subtraction of 2^23 + bias * 2^e then leaves q * 2^e exactly.  The matching
// activation is pre-multiplied by 2^-e (exact), so an f32x2 FMA accumulates q*x.
#pragma once

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Per-bit-width decode tables.
// ---------------------------------------------------------------------------
template <int BITS>
struct Dec;

// int4: 8 codes per word; nibbles 0..4 in place, 5..7 after >> 12.
template <>
struct Dec<4> {
    static constexpr int CH = 16;                  // bytes per lane chunk
    static constexpr int NC = CH * 8 / 4;          // codes per lane chunk (32)
    static constexpr int CPW = 8;                  // codes per 32-bit word
    __device__ static __forceinline__ int exp_of(int p) {
        return (p < 5) ? 4 * p : 4 * (p - 3);      // 0 4 8 12 16 8 12 16
    }
    __device__ static __forceinline__ float bias_of() { return 8.0f; }
    // q * 2^e for the 8 codes of word v, as 4 f32x2 pairs
    __device__ static __forceinline__ void decode(uint32_t v, f2 out[4]) {
        const uint32_t v2 = v >> 12;
        const uint32_t M = 0x4B000000u;
        out[0] = f2_sub(f2_make_bits(M | (v & 0xFu), M | (v & 0xF0u)), f2_make(8388616.0f, 8388736.0f));
        out[1] = f2_sub(f2_make_bits(M | (v & 0xF00u), M | (v & 0xF000u)), f2_make(8390656.0f, 8421376.0f));
        out[2] = f2_sub(f2_make_bits(M | (v & 0xF0000u), M | (v2 & 0xF00u)), f2_make(8912896.0f, 8390656.0f));
        out[3] = f2_sub(f2_make_bits(M | (v2 & 0xF000u), M | (v2 & 0xF0000u)), f2_make(8421376.0f, 8912896.0f));
    }
    // acc += decode(v) . x  in one fixed instruction sequence:
    // 1 shift, 8 lop3, 4 packed subtracts, 4 packed FMAs (8 weights).
    // Packed subtrahends 2^23 + 8 * 2^e for the four code pairs of a word
    // (hoist out of loops).
    struct Consts {
        unsigned long long c[4];
    };
    __device__ static __forceinline__ Consts consts() {
        Consts k;
        k.c[0] = 0x4B0000804B000008ull;
        k.c[1] = 0x4B0080004B000800ull;
        k.c[2] = 0x4B0008004B080000ull;
        k.c[3] = 0x4B0800004B008000ull;
        return k;
    }
    // acc += decode(v) . x[0..3] in one fixed sequence: 1 shift, 8 lop3 whose
    // results pair up in registers, 4 packed subtracts, 4 packed FMAs.
    __device__ static __forceinline__ void dot(uint32_t v, const f2 *x, f2 &acc, const Consts &k) {
        asm("{\n\t"
            ".reg .b32 s, a0, a1, a2, a3, a4, a5, a6, a7;\n\t"
            ".reg .b64 p0, p1, p2, p3;\n\t"
            "shr.u32 s, %1, 12;\n\t"
            "lop3.b32 a0, %1, 0x0000000F, 0x4B000000, 0xEA;\n\t"
            "lop3.b32 a1, %1, 0x000000F0, 0x4B000000, 0xEA;\n\t"
            "lop3.b32 a2, %1, 0x00000F00, 0x4B000000, 0xEA;\n\t"
            "lop3.b32 a3, %1, 0x0000F000, 0x4B000000, 0xEA;\n\t"
            "lop3.b32 a4, %1, 0x000F0000, 0x4B000000, 0xEA;\n\t"
            "lop3.b32 a5, s, 0x00000F00, 0x4B000000, 0xEA;\n\t"
            "lop3.b32 a6, s, 0x0000F000, 0x4B000000, 0xEA;\n\t"
            "lop3.b32 a7, s, 0x000F0000, 0x4B000000, 0xEA;\n\t"
            "mov.b64 p0, {a0, a1};\n\t"
            "mov.b64 p1, {a2, a3};\n\t"
            "mov.b64 p2, {a4, a5};\n\t"
            "mov.b64 p3, {a6, a7};\n\t"
            "sub.rn.f32x2 p0, p0, %6;\n\t"
            "sub.rn.f32x2 p1, p1, %7;\n\t"
            "sub.rn.f32x2 p2, p2, %8;\n\t"
            "sub.rn.f32x2 p3, p3, %9;\n\t"
            "fma.rn.f32x2 %0, p0, %2, %0;\n\t"
            "fma.rn.f32x2 %0, p1, %3, %0;\n\t"
            "fma.rn.f32x2 %0, p2, %4, %0;\n\t"
            "fma.rn.f32x2 %0, p3, %5, %0;\n\t"
            "}"
            : "+l"(acc.v)
            : "r"(v), "l"(x[0].v), "l"(x[1].v), "l"(x[2].v), "l"(x[3].v), "l"(k.c[0]), "l"(k.c[1]),
              "l"(k.c[2]), "l"(k.c[3]));
    }
};

// int8: 4 two's-complement bytes per word; bias 128 after xor 0x80.
template <>
struct Dec<8> {
    static constexpr int CH = 16;
    static constexpr int NC = CH;                  // 16
    static constexpr int CPW = 4;
    __device__ static __forceinline__ int exp_of(int p) { return (p & 1) ? 8 : 0; }
    __device__ static __forceinline__ void decode(uint32_t v, f2 out[2]) {
        const uint32_t u = v ^ 0x80808080u;
        const uint32_t u2 = u >> 16;
        const uint32_t M = 0x4B000000u;
        const float c0 = 8388608.0f + 128.0f, c8 = 8388608.0f + 32768.0f;
        out[0] = f2_sub(f2_make(__uint_as_float(M | (u & 0xFFu)), __uint_as_float(M | (u & 0xFF00u))), f2_make(c0, c8));
        out[1] = f2_sub(f2_make(__uint_as_float(M | (u2 & 0xFFu)), __uint_as_float(M | (u2 & 0xFF00u))), f2_make(c0, c8));
    }
};

// int2: 16 crumbs per word; crumbs 0..9 in place, 10..15 after >> 20.
template <>
struct Dec<2> {
    static constexpr int CH = 8;
    static constexpr int NC = CH * 8 / 2;          // 32
    static constexpr int CPW = 16;
    __device__ static __forceinline__ int exp_of(int p) { return (p < 10) ? 2 * p : 2 * (p - 10); }
    __device__ static __forceinline__ void decode(uint32_t v, f2 out[8]) {
        const uint32_t v2 = v >> 20;
        const uint32_t M = 0x4B000000u;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int p0 = 2 * i, p1 = 2 * i + 1;
            const uint32_t w0 = (p0 < 10) ? (v & (3u << (2 * p0))) : (v2 & (3u << (2 * (p0 - 10))));
            const uint32_t w1 = (p1 < 10) ? (v & (3u << (2 * p1))) : (v2 & (3u << (2 * (p1 - 10))));
            const int e0 = (p0 < 10) ? 2 * p0 : 2 * (p0 - 10);
            const int e1 = (p1 < 10) ? 2 * p1 : 2 * (p1 - 10);
            out[i] = f2_sub(f2_make(__uint_as_float(M | w0), __uint_as_float(M | w1)),
                            f2_make(8388608.0f + 2.0f * static_cast<float>(1u << e0),
                                    8388608.0f + 2.0f * static_cast<float>(1u << e1)));
        }
    }
};

template <int BITS>
struct Chunk;
template <>
struct Chunk<4> { using T = uint4; static constexpr int W = 4; };
template <>
struct Chunk<8> { using T = uint4; static constexpr int W = 4; };
template <>
struct Chunk<2> { using T = uint2; static constexpr int W = 2; };

template <int BITS>
__device__ __forceinline__ void load_chunk(const uint8_t *p, uint32_t w[Chunk<BITS>::W]) {
    if constexpr (Chunk<BITS>::W == 4) {
        const uint4 v = ldg_stream(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
        const uint2 v = ldg_stream8(p);
        w[0] = v.x; w[1] = v.y;
    }
}


}  // namespace moe
