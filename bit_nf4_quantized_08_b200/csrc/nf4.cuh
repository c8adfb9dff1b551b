// nf4.cuh -- the NF4 code book and the per-block dequantization used by every
// kernel of the library (standalone dequant, dequant-GEMM producers).
//
// Code book (QLoRA paper digest, sec. 4 "4-bit NormalFloat", quantile
// equation; blog note p19e99 sec. 2: N(0,1) quantiles normalized to [-1, 1];
// digest: asymmetric so that 0 is exact).  With Q the standard normal
// quantile function and d = (1/32 + 1/30) / 2, the 8 positive codes are
// Q(p) / Q(1-d) for p = 1/2 + i (1/2 - d) / 8, i = 1..8, the 7 negative codes
// Q(p) / |Q(d)| for p = d + i (1/2 - d) / 7, i = 0..6, and index 7 is 0;
// every value is rounded to fp32.  The literals below are those fp32 values.
//
// Dequantization of one 64-element block with constant a (digest sec. 4,
// doubleDequant): w' = bf16_rne(fl32(nf4[code] * a)).  A block has only 16
// distinct outputs, so the kernels build them once per block (16 FMUL + 8
// packs) and then expand codes with byte permutes (PRMT) from registers:
// no shared-memory lookups and no per-element multiplies.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace qlora {

#define QLORA_NF4_BITS                                                                       \
    0xbf800000u, 0xbf3239b1u, 0xbf066b2eu, 0xbeca329eu, 0xbe91a24bu, 0xbe3d353du, 0xbdba7869u, \
        0x00000000u, 0x3da2fb01u, 0x3e24cadfu, 0x3e7c04dau, 0x3ead0336u, 0x3ee1a4b5u,       \
        0x3f1007a9u, 0x3f3913b0u, 0x3f800000u

// FP4 code book (the "Float4 (FP4)" data type the QLoRA paper digest, sec. 6,
// compares NF4 with): the 16 values of a 4-bit float with 1 sign, 2
// exponent (bias 1) and 1 mantissa bit -- magnitudes 0, 0.5, 1, 1.5, 2, 3,
// 4, 6 -- divided by 6 and sorted; -0 (index 7) and +0 (index 8) both
// appear, and the nearest-code rule (ties to the lower index) never picks 8.
#define QLORA_FP4_BITS                                                                       \
    0xbf800000u, 0xbf2aaaabu, 0xbf000000u, 0xbeaaaaabu, 0xbe800000u, 0xbe2aaaabu, 0xbdaaaaabu, \
        0x80000000u, 0x00000000u, 0x3daaaaabu, 0x3e2aaaabu, 0x3e800000u, 0x3eaaaaabu,       \
        0x3f000000u, 0x3f2aaaabu, 0x3f800000u

static constexpr uint32_t kNF4Bits[16] = {QLORA_NF4_BITS};          // host copy
static constexpr uint32_t kCodeBits[2][16] = {{QLORA_NF4_BITS}, {QLORA_FP4_BITS}};
__constant__ uint32_t c_code_bits[2][16] = {{QLORA_NF4_BITS}, {QLORA_FP4_BITS}};  // device copy

// Value j of the 4-bit code book of code type ct (0: NF4, 1: FP4).
__device__ __forceinline__ float code_value(int ct, int j) { return __uint_as_float(c_code_bits[ct][j]); }
__device__ __forceinline__ float nf4_value(int j) { return code_value(0, j); }

// Byte planes of the 16 bf16 outputs of one block: L[q] holds the low bytes
// of codes 4q..4q+3, H[q] the high bytes.
struct Nf4BlockTable {
    uint32_t L[4], H[4];
};

__device__ __forceinline__ Nf4BlockTable nf4_block_table(float a, int ct = 0) {
    uint32_t P[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        P[i] = pack_bf16x2(__fmul_rn(code_value(ct, 2 * i), a), __fmul_rn(code_value(ct, 2 * i + 1), a));
    Nf4BlockTable t;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        t.L[q] = prmt(P[2 * q], P[2 * q + 1], 0x6420u);
        t.H[q] = prmt(P[2 * q], P[2 * q + 1], 0x7531u);
    }
    return t;
}

// Expand one 32-bit word of packed codes (8 elements; byte i holds element 2i
// in its high nibble and 2i+1 in its low nibble) into 4 bf16x2 words,
// out[j] = {element 2j (bits 0..15), element 2j+1 (bits 16..31)}.
__device__ __forceinline__ void nf4_expand_word(uint32_t w, const Nf4BlockTable& t,
                                                uint32_t (&out)[4]) {
    const uint32_t s = w & 0x77777777u;  // low 3 bits of every code
    const uint32_t s_hi = s >> 16;
    const uint32_t wo = w << 4;           // bit 3 of each low-nibble code -> byte msb
    // 0xFF per output byte whose code is >= 8 (PRMT sign-replicate mode).
    // Selector order of the four output bytes follows the nibbles of s:
    // [element 1, element 0, element 3, element 2] (and 5, 4, 7, 6 for s_hi).
    const uint32_t m1 = prmt(wo, w, 0xD9C8u);
    const uint32_t m2 = prmt(wo, w, 0xFBEAu);
    {
        uint32_t la = prmt(t.L[0], t.L[1], s), lb = prmt(t.L[2], t.L[3], s);
        uint32_t ha = prmt(t.H[0], t.H[1], s), hb = prmt(t.H[2], t.H[3], s);
        uint32_t lo = (la & ~m1) | (lb & m1);
        uint32_t hi = (ha & ~m1) | (hb & m1);
        out[0] = prmt(lo, hi, 0x4051u);
        out[1] = prmt(lo, hi, 0x6273u);
    }
    {
        uint32_t la = prmt(t.L[0], t.L[1], s_hi), lb = prmt(t.L[2], t.L[3], s_hi);
        uint32_t ha = prmt(t.H[0], t.H[1], s_hi), hb = prmt(t.H[2], t.H[3], s_hi);
        uint32_t lo = (la & ~m2) | (lb & m2);
        uint32_t hi = (ha & ~m2) | (hb & m2);
        out[2] = prmt(lo, hi, 0x4051u);
        out[3] = prmt(lo, hi, 0x6273u);
    }
}

// fp32 value of the 8-bit double-quantization code k: fl32((k - 127) / 127).
__device__ __forceinline__ float t8_value(int k) {
    return __fdiv_rn((float)(k - 127), 127.0f);
}

// fp32 value of the FP8 double-quantization code k (0..252): the k-th of the
// 253 distinct finite E4M3 values (1 sign, 4 exponent bits with bias 7, 3
// mantissa bits; exponent field 0 subnormal; the all-ones pattern is not a
// number, so the largest value is 448) in ascending order, divided by 448:
// fl32(v / 448) with the quotient taken in fp64 (the "c2^FP8" of the digest,
// sec. 4 double quantization).
__device__ __forceinline__ float e4m3_value(int k) {
    const int j = k < 126 ? 125 - k : k - 127;  // rank among the positive values
    if (k == 126) return 0.0f;
    double v;
    if (j < 7) {
        v = (double)(j + 1) * 0.001953125;  // (m / 8) 2^-6, m = 1..7
    } else {
        const int e = 1 + (j - 7) / 8, m = (j - 7) % 8;
        v = ldexp(1.0 + m / 8.0, e - 7);
    }
    const float f = __double2float_rn(__ddiv_rn(v, 448.0));
    return k < 126 ? -f : f;
}

// Value of the 8-bit double-quantization code k of code book dt
// (0: linear t8, 1: FP8 E4M3).
__device__ __forceinline__ float dq_value(int dt, int k) { return dt ? e4m3_value(k) : t8_value(k); }

// Block constant a' (digest sec. 4 doubleDequant, first dequant):
// fl32(fl32(c8[q8] * c1) + offset) with double quantization, else absmax.
__device__ __forceinline__ float block_scale_dq(uint8_t q8, float c1, float offset, int dt = 0) {
    return __fadd_rn(__fmul_rn(dq_value(dt, q8), c1), offset);
}

// Storage format of a quantized weight beyond the NF4 / linear 8-bit /
// 64-element defaults: code book, double-quantization code book, and block
// size 64 << bs_shift.  Block b of size bs covers the flattened elements
// [b bs, (b+1) bs), so the block of the 64-element column kb64 of row n is
// (n * K/64 + kb64) >> bs_shift.
struct QFormat {
    int code_type;  // 0 NF4, 1 FP4
    int dq_type;    // 0 linear 8-bit, 1 FP8 E4M3
    int bs_shift;   // 0, 1, 2: block size 64, 128, 256
};

}  // namespace qlora
