// quantize.cuh -- NF4 blockwise quantizer, double quantization of the block
// constants, standalone dequantization, and the block-constant expansion used
// by the dequant-GEMM producers.  All kernels are HBM-streaming kernels:
// 128-bit loads and stores, warp shuffles for the block reductions.
//
// Definitions (QLoRA blog note p19e99 sec. 2 "NF4" and sec. 3 "double
// quantization"; QLoRA paper digest sec. 4 "NF4", "double quantization",
// doubleDequant; tutorial "11.3 QLoRA" section "double quantization": 64
// parameters share one fp32 constant, the constants go to 8 bits):
//  - block b = elements [64b, 64b+64) of the flattened row-major tensor (the
//    last block may be shorter); a_b = max |w| over the block.
//  - x = fl32((w * p) * fl32(1 / (a_b * p))) with the exact power-of-two
//    prescale p = 2^64 when a_b < 2^-126 (so the reciprocal stays finite),
//    p = 1 otherwise; a zero block uses the factor 0.
//  - code = index of the nearest NF4 value, exact ties to the lower index.
//  - byte i of the packed codes = (code[2i] << 4) | code[2i+1].
//  - double quantization: offset = fl32(S / nb) with S the fp64 pairwise-tree
//    sum of all a_b (zero-padded to a power of two); d_b = fl32(a_b - offset);
//    c1[g] = max |d_b| over blocks [256g, 256g+256); y = fl32((d_b p) *
//    fl32(1/(c1 p))) (same prescale rule, factor 0 when c1 == 0); q8 = index
//    of the nearest t8[k] = fl32((k-127)/127), ties to the lower index.
#pragma once

#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "nf4.cuh"

namespace qlora {

// ---------------------------------------------------------------------------
// fast nearest-code search
// ---------------------------------------------------------------------------
// x in [-1.03, 1.03] falls in bucket key = RN(16 x + 16) in 0..32, i.e. the
// closed interval [(key - 1/2)/16 - 1, (key + 1/2)/16 - 1].  Buckets are
// narrower than the smallest gap between two decision thresholds (0.080), so
// each holds at most one threshold T_key; base_key counts the thresholds at
// or below the bucket's lower edge.  code(x) = base_key + (x >= T_key), where
// threshold j is the smallest fp32 strictly above the exact midpoint of codes
// j and j+1 (so an exact tie stays with the lower code).  The table holds
// P_key, the largest fp32 below T_key: x >= T_key exactly when x > P_key,
// i.e. when fl(P_key - x) is negative (a difference of two finite floats is
// zero only when they are equal), so the compare is one FADD and the sign
// bit.
// t = fl(16 x + 1.5 * 2^23 + 16) holds the key in its low mantissa bits
// (0x4B400000 + key); (P_key, base_key) sit as one 8-byte entry, so one
// shared load per element fetches both.  64 entries and a 6-bit key mask:
// any input (NaN included) reads inside the table.
struct __align__(16) SearchSmem {
    uint2 e[64];   // {P_key bits, base_key}
    int inc[64];
};

__device__ __forceinline__ void load_search_tables(SearchSmem& st, const Nf4SearchTable& tab) {
    for (int i = threadIdx.x; i < 64; i += blockDim.x) {
        st.e[i] = make_uint2(__float_as_uint(i < 33 ? tab.thr[i] : 3.0f), (uint32_t)(i < 33 ? tab.base[i] : 15));
        st.inc[i] = i < 33 ? tab.inc[i] : 0;
    }
}

constexpr float kKeyMagic = 12582928.0f;  // 1.5 * 2^23 + 16

// CT = 1 (FP4): a bucket's threshold may count twice (inc = 2).
template <int CT = 0>
__device__ __forceinline__ uint32_t nf4_lookup(float x, float t, const SearchSmem& st) {
    const uint32_t key = __float_as_uint(t) & 63u;
    const uint2 e = st.e[key];
    const uint32_t above = __float_as_uint(__fsub_rn(__uint_as_float(e.x), x)) >> 31;
    if (CT == 0) return e.y + above;
    return e.y + above * (uint32_t)st.inc[key];
}

template <int CT = 0>
__device__ __forceinline__ uint32_t nf4_search(float x, const SearchSmem& st) {
    return nf4_lookup<CT>(x, fmaf(x, 16.0f, kKeyMagic), st);
}

// Two lanes of fp32x2 arithmetic (sm_100a packed FP32): the same IEEE
// round-to-nearest products and fused multiply-adds as the scalar forms.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Codes of two elements x = fl(w * rcp) in one fp32x2 multiply and FMA.
template <int CT = 0>
__device__ __forceinline__ void nf4_search2(float w0, float w1, uint64_t rcp2, const SearchSmem& st, uint32_t& c0,
                                            uint32_t& c1) {
    const uint64_t x2 = f2_mul(f2_pack(w0, w1), rcp2);
    const uint64_t t2 = f2_fma(x2, f2_pack(16.0f, 16.0f), f2_pack(kKeyMagic, kKeyMagic));
    float x0, x1, t0, t1;
    f2_unpack(x2, x0, x1);
    f2_unpack(t2, t0, t1);
    c0 = nf4_lookup<CT>(x0, t0, st);
    c1 = nf4_lookup<CT>(x1, t1, st);
}

// Pack 8 codes (element order) into one word: byte i = (c[2i] << 4) | c[2i+1].
__device__ __forceinline__ uint32_t pack8(const uint32_t (&c)[8]) {
    uint32_t acc = c[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) acc = acc * 16u + c[i];  // c0 ends in the top nibble
    return __byte_perm(acc, 0u, 0x0123);                 // reverse bytes: (c0,c1) -> byte 0
}

// ---------------------------------------------------------------------------
// K1: quantize.  One CTA (8 warps) per group of 16384 elements; warp w
// handles rows 4w..4w+3 of 512 elements; a lane holds 16 consecutive
// elements, 4 << bs_shift lanes make one block (64, 128 or 256 elements).
// Also writes the group's fp64 pairwise-tree sum of block maxima for the
// double-quantization offset.  CT: code book (0 NF4, 1 FP4).
// ---------------------------------------------------------------------------
template <bool BF16, int CT>
__global__ void __launch_bounds__(256, BF16 ? 4 : 2) k_quantize_blocks(const void* W, int64_t n,
                                                            uint8_t* codes,
                                                            float* absmax,
                                                            double* group_sums,
                                                            Nf4SearchTable tab, int bs_shift) {
    __shared__ SearchSmem st;
    __shared__ double s_wsum[8];
    // dependent launch: resident before the kernel ahead ends, no access to
    // memory before it has.  The kernels that wait this way take no
    // __restrict__ pointers: with them the compiler may move loads of
    // "unchanging" data above griddepcontrol.wait.
    pdl_trigger();
    pdl_wait();
    load_search_tables(st, tab);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bshift = 6 + bs_shift;                  // log2 of the block size
    const int64_t nb = (n + (1 << bshift) - 1) >> bshift;
    const int blanes = 4 << bs_shift;                 // lanes per block
    constexpr int WORDS = BF16 ? 8 : 16;  // 32-bit words per lane per row
    uint32_t raw[4][WORDS];
    int64_t e0[4];

#pragma unroll
    for (int it = 0; it < 4; ++it) {
        e0[it] = (int64_t)blockIdx.x * 16384 + (int64_t)(warp * 4 + it) * 512 + lane * 16;
        if (e0[it] + 16 <= n) {
            const uint4* src = BF16 ? reinterpret_cast<const uint4*>(
                                          static_cast<const uint16_t*>(W) + e0[it])
                                    : reinterpret_cast<const uint4*>(
                                          static_cast<const float*>(W) + e0[it]);
#pragma unroll
            for (int v = 0; v < WORDS / 4; ++v) {
                uint4 q = __ldcs(src + v);
                raw[it][4 * v + 0] = q.x;
                raw[it][4 * v + 1] = q.y;
                raw[it][4 * v + 2] = q.z;
                raw[it][4 * v + 3] = q.w;
            }
        } else {
#pragma unroll
            for (int v = 0; v < WORDS; ++v) raw[it][v] = 0u;
            if (e0[it] < n) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (e0[it] + i < n) {
                        if (BF16) {
                            uint32_t h = static_cast<const uint16_t*>(W)[e0[it] + i];
                            raw[it][i >> 1] |= h << ((i & 1) * 16);
                        } else {
                            raw[it][i] = __float_as_uint(static_cast<const float*>(W)[e0[it] + i]);
                        }
                    }
                }
            }
        }
    }

    double rowsum[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        // block absmax (exact: a max of magnitudes)
        float a;
        if (BF16) {
            // packed bf16 max of magnitudes (the sign of each half is the xor
            // of the signs, dropped at the end)
            uint32_t m = raw[it][0];
#pragma unroll
            for (int i = 1; i < 8; ++i)
                asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(raw[it][i]));
            m &= 0x7FFF7FFFu;
            m = max(m & 0xFFFFu, m >> 16);
            a = __uint_as_float(m << 16);
        } else {
            a = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(__uint_as_float(raw[it][i])));
        }
        for (int o = 1; o < blanes; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));

        const int64_t b = e0[it] >> bshift;
        const bool bvalid = b < nb;
        if (bvalid && (lane & (blanes - 1)) == 0 && absmax) absmax[b] = a;

        uint32_t c[16];
        if (a >= 1.17549435e-38f) {
            const float rcp = __frcp_rn(a);
            const uint64_t rcp2 = f2_pack(rcp, rcp);
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const uint32_t b0 = BF16 ? (raw[it][i >> 1] << 16) : raw[it][i];
                const uint32_t b1 = BF16 ? (raw[it][i >> 1] & 0xFFFF0000u) : raw[it][i + 1];
                nf4_search2<CT>(__uint_as_float(b0), __uint_as_float(b1), rcp2, st, c[i], c[i + 1]);
            }
        } else {
            // zero or subnormal block: exact power-of-two prescale 2^64
            const float p = 18446744073709551616.0f;
            const float rcp = (a == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(a, p));
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t bits = BF16 ? ((i & 1) ? (raw[it][i >> 1] & 0xFFFF0000u) : (raw[it][i >> 1] << 16))
                                           : raw[it][i];
                c[i] = nf4_search<CT>(__fmul_rn(__fmul_rn(__uint_as_float(bits), p), rcp), st);
            }
        }
        uint32_t lo[8], hi[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            lo[i] = c[i];
            hi[i] = c[8 + i];
        }
        const uint32_t w0 = pack8(lo), w1 = pack8(hi);
        if (e0[it] + 16 <= n) {
            __stcs(reinterpret_cast<uint2*>(codes + (e0[it] >> 1)), make_uint2(w0, w1));
        } else if (e0[it] < n) {
            const int valid = (int)(n - e0[it]);
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // static indices: c stays in registers
                if (2 * j < valid) {
                    uint32_t byte = c[2 * j] << 4;
                    if (2 * j + 1 < valid) byte |= c[2 * j + 1];
                    codes[(e0[it] >> 1) + j] = (uint8_t)byte;
                }
            }
        }

        // fp64 pairwise tree over the row's block maxima (8, 4 or 2 of them;
        // blocks beyond the tensor contribute zeros).
        double d = bvalid ? (double)a : 0.0;
        for (int o = blanes; o < 32; o <<= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        rowsum[it] = d;
    }
    if (group_sums) {
        if (lane == 0) s_wsum[warp] = (rowsum[0] + rowsum[1]) + (rowsum[2] + rowsum[3]);
        __syncthreads();
        if (threadIdx.x == 0) {
            double t0 = s_wsum[0] + s_wsum[1], t1 = s_wsum[2] + s_wsum[3];
            double t2 = s_wsum[4] + s_wsum[5], t3 = s_wsum[6] + s_wsum[7];
            group_sums[blockIdx.x] = (t0 + t1) + (t2 + t3);
        }
    }
}

// fp64 pairwise-tree sum of x[lo, lo + chunk) (chunk a power of two; entries
// at or past n count as 0; the values are non-negative) with a
// binary-counter stack over subtrees of 8 leaves: eight independent loads at
// a time are folded as a fixed subtree first (a chunk below 8 is one such
// subtree padded with zeros), the same tree with an eighth of the dependent
// memory round trips.
__device__ __forceinline__ double pairwise_chunk(const double* x, int64_t lo, int64_t chunk,
                                                 int64_t n) {
    double stack[40];
    int64_t cnt = 0;
    // leaves past the chunk (chunk < 8) or past n are +0.0: adding them
    // changes no sum of the non-negative values summed here
    for (int64_t i = 0; i < chunk; i += 8) {
        double e[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t idx = lo + i + j;
            e[j] = (i + j < chunk && idx < n) ? x[idx] : 0.0;
        }
        double v = ((e[0] + e[1]) + (e[2] + e[3])) + ((e[4] + e[5]) + (e[6] + e[7]));
        int lvl = 0;
        while ((cnt >> lvl) & 1) {
            v = stack[lvl] + v;
            ++lvl;
        }
        stack[lvl] = v;
        ++cnt;
    }
    int top = 0;
    while ((1ll << top) < cnt) ++top;
    return stack[top];
}

// ---------------------------------------------------------------------------
// K2: offset = fl32(S / nb), S = pairwise tree over the group sums padded
// with zeros to a power of two.  One CTA of 1024 threads; thread t sums a
// contiguous power-of-two chunk with a binary-counter pairwise sum.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_dq_offset(const double* sums, int64_t ng,
                                                    int64_t nb, float* offset) {
    __shared__ double s_w[32];
    pdl_trigger();
    pdl_wait();
    int64_t p2 = 1;
    while (p2 < ng) p2 <<= 1;
    const int64_t chunk = p2 > 1024 ? p2 / 1024 : 1;
    double t = pairwise_chunk(sums, (int64_t)threadIdx.x * chunk, chunk, ng);
    for (int o = 1; o < 32; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = t;
    __syncthreads();
    if (threadIdx.x < 32) {
        double u = s_w[threadIdx.x];
        for (int o = 1; o < 32; o <<= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
        if (threadIdx.x == 0) *offset = __double2float_rn(__ddiv_rn(u, (double)nb));
    }
}

// First level of the offset tree for many group sums: CTA c sums leaves
// [4096 c, 4096 c + 4096) of the zero-padded power-of-two leaf array, an
// aligned subtree of the same pairwise tree (16 leaves per thread, then the
// warp and CTA levels in the same pairing), so that a tree over the partials
// gives the same total as one over all sums.
constexpr int64_t kPartialLeaves = 4096;
__global__ void __launch_bounds__(256) k_dq_partials(const double* sums, int64_t ng,
                                                     double* partials) {
    __shared__ double s_w[8];
    pdl_trigger();
    pdl_wait();
    double t = pairwise_chunk(sums, (int64_t)blockIdx.x * kPartialLeaves + (int64_t)threadIdx.x * 16, 16, ng);
    for (int o = 1; o < 32; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = t;
    __syncthreads();
    if (threadIdx.x == 0)
        partials[blockIdx.x] = ((s_w[0] + s_w[1]) + (s_w[2] + s_w[3])) + ((s_w[4] + s_w[5]) + (s_w[6] + s_w[7]));
}

// Decision threshold k of the linear 8-bit code book, between t8[k] and
// t8[k+1] (k = 0..253): the smallest fp32 strictly above their exact
// midpoint (fp64 holds the midpoint of two fp32 values exactly), so that
// y >= T_k exactly when the nearest code of y, ties to the lower index, is
// above k.
__device__ __forceinline__ float t8_threshold(int k) {
    const double m = 0.5 * ((double)t8_value(k) + (double)t8_value(k + 1));
    float f = __double2float_rn(m);
    if ((double)f <= m) f = nextafterf(f, 3.0f);
    return f;
}

// Nearest 8-bit code of y in [-1, 1]: the candidate rint(127 y) + 127 is the
// nearest code or its neighbour (y is within half a step of t8[candidate]),
// so two fp32 compares with the thresholds on either side decide; ties go
// to the lower index.  thr = the 254 thresholds (shared memory).
__device__ __forceinline__ int nearest_t8(float y, const float* thr) {
    int k0 = __float2int_rn(__fmul_rn(y, 127.0f)) + 127;
    k0 = min(max(k0, 0), 254);
    const int down = (k0 > 0 && y < thr[k0 - 1]) ? 1 : 0;
    const int up = (k0 < 254 && y >= thr[k0]) ? 1 : 0;
    return k0 - down + up;
}

// Nearest FP8 (E4M3) code of y: the first table entry >= y by binary search
// over the 253 sorted values, then the exact fp64 distances of it and the
// entry below; ties to the lower index.
__device__ __forceinline__ int nearest_e4m3(float y, const float* t) {
    int lo = 0, hi = 253;  // first index with t[index] >= y, in [lo, hi]
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (t[mid] < y) lo = mid + 1; else hi = mid;
    }
    if (lo == 253) return 252;
    if (lo == 0) return 0;
    const double dl = fabs((double)y - (double)t[lo - 1]), dh = fabs((double)t[lo] - (double)y);
    return dl <= dh ? lo - 1 : lo;
}

// ---------------------------------------------------------------------------
// K3: second-level quantization; one warp per group of 256 block constants.
// ---------------------------------------------------------------------------
// With sums != nullptr every CTA first forms the offset itself from the
// nsums group sums (the same pairwise tree as K2, over 256 threads) and CTA 0
// also stores it; otherwise the offset is read from offset_ptr.
// dt: the 8-bit code book (0 linear, 1 FP8 E4M3).
__global__ void __launch_bounds__(256) k_dq_quantize(const float* absmax, int64_t nb,
                                                     float* offset_ptr,
                                                     uint8_t* q8,
                                                     float* c1,
                                                     const double* sums, int64_t nsums, int dt) {
    __shared__ float t8[256];  // E4M3: the 253 code values; linear: the 254 decision thresholds
    __shared__ double s_w[8];
    __shared__ float s_off;
    pdl_trigger();
    // blockDim.x == 256; shared memory only
    t8[threadIdx.x] = dt ? (threadIdx.x < 253 ? e4m3_value(threadIdx.x) : 2.0f)
                         : (threadIdx.x < 254 ? t8_threshold(threadIdx.x) : 3.0f);
    pdl_wait();
    // this warp's first group: 8 block maxima per lane, loaded before the
    // offset tree so that the two memory round trips overlap
    const int64_t g = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t ng = (nb + 255) >> 8;
    const int64_t bf = g * 256 + lane * 8;
    float am[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) am[i] = (g < ng && bf + i < nb) ? absmax[bf + i] : 0.0f;
    if (sums) {
        int64_t p2 = 1;
        while (p2 < nsums) p2 <<= 1;
        const int64_t chunk = p2 > 256 ? p2 / 256 : 1;
        double t = pairwise_chunk(sums, (int64_t)threadIdx.x * chunk, chunk, nsums);
        for (int o = 1; o < 32; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = t;
        __syncthreads();
        if (threadIdx.x == 0) {
            const double u = ((s_w[0] + s_w[1]) + (s_w[2] + s_w[3])) + ((s_w[4] + s_w[5]) + (s_w[6] + s_w[7]));
            s_off = __double2float_rn(__ddiv_rn(u, (double)nb));
            if (blockIdx.x == 0) *offset_ptr = s_off;
        }
    } else if (threadIdx.x == 0) {
        s_off = *offset_ptr;
    }
    __syncthreads();
    const float off = s_off;
    // one warp per group of 256 blocks; the grid is capped, so a warp takes
    // every (gridDim.x * 8)-th group
    for (int64_t gg = g; gg < ng; gg += (int64_t)gridDim.x * 8) {
        const int64_t b0 = gg * 256 + lane * 8;
        if (gg != g) {
#pragma unroll
            for (int i = 0; i < 8; ++i) am[i] = b0 + i < nb ? absmax[b0 + i] : 0.0f;
        }
        float d[8];
        float c = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            d[i] = (b0 + i < nb) ? __fsub_rn(am[i], off) : 0.0f;
            c = fmaxf(c, fabsf(d[i]));
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, o));
        float p = 1.0f;
        if (c < 1.17549435e-38f) p = 18446744073709551616.0f;
        const float rc = (c == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(c, p));
        uint32_t q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float y = __fmul_rn(__fmul_rn(d[i], p), rc);
            q[i] = (uint32_t)(dt ? nearest_e4m3(y, t8) : nearest_t8(y, t8));
        }
        if (b0 + 8 <= nb) {
            uint2 v;
            v.x = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
            v.y = q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24);
            *reinterpret_cast<uint2*>(q8 + b0) = v;
        } else {
            for (int i = 0; i < 8; ++i)
                if (b0 + i < nb) q8[b0 + i] = (uint8_t)q[i];
        }
        if (lane == 0) c1[gg] = c;
    }
}

// ---------------------------------------------------------------------------
// K4: standalone dequantization, one thread per 64-element block.  A warp
// covers 32 consecutive blocks; each thread expands its block into a
// 128-byte-swizzled shared-memory slot, then the warp writes its 4 KB of
// output with fully coalesced 16-byte stores.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_dequantize(const uint8_t* __restrict__ codes, int64_t n,
                                                    int dq, const float* __restrict__ absmax,
                                                    const uint8_t* __restrict__ q8,
                                                    const float* __restrict__ c1,
                                                    const float* __restrict__ offset_ptr,
                                                    uint16_t* __restrict__ out, QFormat fmt) {
    __shared__ __align__(16) uint8_t stage[8][4096];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = (int64_t)blockIdx.x * 256 + threadIdx.x;
    const int64_t nb = (n + 63) >> 6;
    const int64_t wb0 = (int64_t)blockIdx.x * 256 + warp * 32;  // first block of this warp
    const bool warp_full = (wb0 + 32) * 64 <= n;
    const int64_t bb = b >> fmt.bs_shift;  // the block (of the weight's size) holding this 64
    if (warp_full) {
        const float a = dq ? block_scale_dq(q8[bb], c1[bb >> 8], *offset_ptr, fmt.dq_type) : absmax[bb];
        const uint4* src = reinterpret_cast<const uint4*>(codes + b * 32);
        const uint4 c0 = __ldcs(src), c1v = __ldcs(src + 1);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1v.x, c1v.y, c1v.z, c1v.w};
        const Nf4BlockTable t = nf4_block_table(a, fmt.code_type);
        const uint32_t slot = smem_u32(&stage[warp][0]) + lane * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t o[4];
            nf4_expand_word(words[i], t, o);
            st_shared_v4(slot + ((i ^ (lane & 7)) << 4), o[0], o[1], o[2], o[3]);
        }
        __syncwarp();
        uint4* dst = reinterpret_cast<uint4*>(out + wb0 * 64);
        const uint32_t sbase = smem_u32(&stage[warp][0]);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int lin = i * 512 + lane * 16;  // linear byte offset in the warp's 4 KB
            const int blk = lin >> 7, q = (lin >> 4) & 7;
            const uint4 v = ld_shared_v4(sbase + blk * 128 + ((q ^ (blk & 7)) << 4));
            __stcs(dst + i * 32 + lane, v);
        }
        return;
    }
    if (b >= nb) return;
    const float a = dq ? block_scale_dq(q8[bb], c1[bb >> 8], *offset_ptr, fmt.dq_type) : absmax[bb];
    if ((b + 1) * 64 <= n) {
        const uint4* src = reinterpret_cast<const uint4*>(codes + b * 32);
        uint4 c0 = __ldg(src), c1v = __ldg(src + 1);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1v.x, c1v.y, c1v.z, c1v.w};
        const Nf4BlockTable t = nf4_block_table(a, fmt.code_type);
        uint4* dst = reinterpret_cast<uint4*>(out + b * 64);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t o[4];
            nf4_expand_word(words[i], t, o);
            dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    } else {
        for (int64_t e = b * 64; e < n; ++e) {
            uint8_t byte = codes[e >> 1];
            int c = (e & 1) ? (byte & 15) : (byte >> 4);
            __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(code_value(fmt.code_type, c), a));
            out[e] = *reinterpret_cast<uint16_t*>(&h);
        }
    }
}

// Block constants a' transposed for the GEMM producers: scales[kb*ld + n].
// Also zeroes `nflags` ints (the flags of the stream-K GEMM that follows).
__global__ void k_expand_scales(int64_t rows, int64_t kbs, int dq, const float* absmax,
                                const uint8_t* q8, const float* c1,
                                const float* offset_ptr, float* scales,
                                int64_t ld, int* flags, int nflags, QFormat fmt) {
    // the LoRA GEMM that follows reads none of this kernel's outputs; this
    // kernel's inputs (8-bit constants) and outputs (scales, flags of the
    // GEMM before) belong to the kernel before it
    pdl_trigger();
    pdl_wait();
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx < nflags) flags[idx] = 0;
    if (idx >= rows * kbs) return;
    const int64_t kb = idx / rows, n = idx - kb * rows;
    const int64_t b = (n * kbs + kb) >> fmt.bs_shift;  // flattened block of the weight's block size
    scales[kb * ld + n] = dq ? block_scale_dq(q8[b], c1[b >> 8], *offset_ptr, fmt.dq_type) : absmax[b];
}

__global__ void k_encode(const float* __restrict__ x, int64_t n, uint8_t* __restrict__ codes,
                         Nf4SearchTable tab) {
    __shared__ SearchSmem st;
    load_search_tables(st, tab);
    __syncthreads();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        float v = fminf(fmaxf(x[i], -1.0f), 1.0f);
        codes[i] = (uint8_t)nf4_search<0>(v, st);
    }
}

// Nearest 8-bit code of every y (test entry point: the search of the double
// quantization on arbitrary inputs).
__global__ void k_dq_encode(const float* __restrict__ y, int64_t n, uint8_t* __restrict__ codes, int dt) {
    __shared__ float t8[256];
    t8[threadIdx.x] = dt ? (threadIdx.x < 253 ? e4m3_value(threadIdx.x) : 2.0f)
                         : (threadIdx.x < 254 ? t8_threshold(threadIdx.x) : 3.0f);
    __syncthreads();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = fminf(fmaxf(y[i], -1.0f), 1.0f);
        codes[i] = (uint8_t)(dt ? nearest_e4m3(v, t8) : nearest_t8(v, t8));
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

inline void nf4_table_host(float out[16]) {
    for (int j = 0; j < 16; ++j) {
        uint32_t u = kNF4Bits[j];
        memcpy(&out[j], &u, 4);
    }
}

// Search table of a 16-value code book (ct 0 NF4, 1 FP4).  Threshold j is
// the smallest fp32 above which the nearest value (ties to the lower index)
// has an index above j: above the exact midpoint of values j and j+1, or,
// when the two values are equal (the two zeros of FP4, where index 8 is
// never the nearest), the next threshold.
inline Nf4SearchTable build_search_table(int ct) {
    float v[16];
    for (int j = 0; j < 16; ++j) {
        uint32_t u = kCodeBits[ct][j];
        memcpy(&v[j], &u, 4);
    }
    float thr[15];
    for (int j = 14; j >= 0; --j) {
        if ((double)v[j] == (double)v[j + 1]) {
            thr[j] = thr[j + 1];
            continue;
        }
        double mid = 0.5 * ((double)v[j] + (double)v[j + 1]);  // exact in fp64
        float f = (float)mid;
        if ((double)f <= mid) f = std::nextafter(f, INFINITY);
        thr[j] = f;
    }
    Nf4SearchTable t;
    for (int k = 0; k <= 32; ++k) {
        double lo = (k - 0.5) / 16.0 - 1.0, hi = (k + 0.5) / 16.0 - 1.0;
        int base = 0, inc = 0;
        float tk = 3.0f;  // no threshold inside the bucket
        for (int j = 0; j < 15; ++j) {
            if ((double)thr[j] <= lo) {
                ++base;
            } else if ((double)thr[j] <= hi) {
                tk = thr[j];
                ++inc;
            }
        }
        t.thr[k] = std::nextafter(tk, -INFINITY);  // P_key: x >= T_key  <=>  x > P_key
        t.base[k] = base;
        t.inc[k] = inc;
    }
    return t;
}

inline const Nf4SearchTable& search_table(int ct) {
    static const Nf4SearchTable t[2] = {build_search_table(0), build_search_table(1)};
    return t[ct];
}
inline const Nf4SearchTable& nf4_search_table() { return search_table(0); }

inline cudaError_t launch_quantize_blocks(const void* W, int is_bf16, int64_t n, uint8_t* codes,
                                          float* absmax, double* group_sums, cudaStream_t s,
                                          QFormat fmt = QFormat{0, 0, 0}) {
    const int64_t ng = (n + 16383) / 16384;
    if (ng == 0) return cudaSuccess;
    ProfileScope ps(QLORA_KERNEL_QUANTIZE, s);
    note_launch();
    const Nf4SearchTable& tab = search_table(fmt.code_type);
    auto kern = is_bf16 ? (fmt.code_type ? k_quantize_blocks<true, 1> : k_quantize_blocks<true, 0>)
                        : (fmt.code_type ? k_quantize_blocks<false, 1> : k_quantize_blocks<false, 0>);
    return launch_pdl(kern, dim3((unsigned)ng), dim3(256), 0, s, 0, W, n, codes, absmax, group_sums, tab,
                      fmt.bs_shift);
}

inline cudaError_t launch_dq_offset(const double* group_sums, int64_t ngroups, int64_t nb,
                                    float* offset, cudaStream_t s) {
    note_launch();
    return launch_pdl(k_dq_offset, dim3(1), dim3(1024), 0, s, 0, group_sums, ngroups, nb, offset);
}

inline cudaError_t launch_dq_quantize(const float* absmax, int64_t nb, float* offset, uint8_t* q8, float* c1,
                                      cudaStream_t s, const double* sums = nullptr, int64_t nsums = 0,
                                      int dt = 0) {
    const int64_t ng = (nb + 255) / 256;
    if (ng == 0) return cudaSuccess;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        nsm = 148;
    // at most 8 resident CTAs per SM; each forms the offset once
    const int64_t grid = std::min<int64_t>((ng + 7) / 8, (int64_t)8 * nsm);
    note_launch();
    return launch_pdl(k_dq_quantize, dim3((unsigned)grid), dim3(256), 0, s, 0, absmax, nb, offset, q8, c1, sums,
                      nsums, dt);
}

// Double quantization of the block maxima: offset, then 8-bit codes.  Up to
// kFusedSums group sums every CTA of the 8-bit kernel forms the offset
// itself (one launch); above, k_dq_partials first reduces aligned 4096-leaf
// subtrees into `partials` (dq_partial_count doubles) and the 8-bit kernel
// forms the offset from those.  Test mode 5, or no partials buffer: the
// one-CTA k_dq_offset kernel over all sums first.
constexpr int64_t kFusedSums = 8192;
inline int64_t dq_partial_count(int64_t nsums) {
    if (nsums <= kFusedSums) return 0;
    int64_t p2 = 1;
    while (p2 < nsums) p2 <<= 1;
    return p2 / kPartialLeaves;
}
inline cudaError_t launch_double_quant(const double* sums, int64_t nsums, const float* absmax, int64_t nb,
                                       float* offset, uint8_t* q8, float* c1, cudaStream_t s,
                                       double* partials = nullptr, int dt = 0) {
    if (nsums <= kFusedSums && inject_mode() != 5)
        return launch_dq_quantize(absmax, nb, offset, q8, c1, s, sums, nsums, dt);
    const int64_t G = dq_partial_count(nsums);
    if (G > 0 && partials && inject_mode() != 5) {
        note_launch();
        cudaError_t e = launch_pdl(k_dq_partials, dim3((unsigned)G), dim3(256), 0, s, 0, sums, nsums, partials);
        if (e != cudaSuccess) return e;
        return launch_dq_quantize(absmax, nb, offset, q8, c1, s, partials, G, dt);
    }
    cudaError_t e = launch_dq_offset(sums, nsums, nb, offset, s);
    if (e != cudaSuccess) return e;
    return launch_dq_quantize(absmax, nb, offset, q8, c1, s, nullptr, 0, dt);
}

inline QFormat weight_format(const qlora_nf4_weight& w) {
    return QFormat{w.code_type, w.dq_type, w.blocksize == 256 ? 2 : (w.blocksize == 128 ? 1 : 0)};
}

inline cudaError_t launch_dequantize(const qlora_nf4_weight& w, uint16_t* out, cudaStream_t s) {
    const int64_t n = w.rows * w.cols;
    const int64_t nb = (n + 63) / 64;
    if (nb == 0) return cudaSuccess;
    ProfileScope ps(QLORA_KERNEL_DEQUANTIZE, s);
    note_launch();
    k_dequantize<<<(unsigned)((nb + 255) / 256), 256, 0, s>>>(
        w.codes, n, w.double_quant, w.absmax, w.absmax_q8, w.absmax_scale, w.absmax_offset, out, weight_format(w));
    return cudaGetLastError();
}

inline cudaError_t launch_expand_scales(const qlora_nf4_weight& w, float* scales, int64_t ld,
                                        cudaStream_t s, int* flags = nullptr, int nflags = 0) {
    const int64_t kbs = w.cols / 64;
    const int64_t total = w.rows * kbs > nflags ? w.rows * kbs : nflags;
    if (total == 0) return cudaSuccess;
    note_launch();
    // dependent launch: the CTAs can be resident before the kernel ahead
    // ends and wait for it (pdl_wait) before any access
    return launch_pdl(k_expand_scales, dim3((unsigned)((total + 255) / 256)), dim3(256), 0, s, 0, w.rows, kbs,
                      (int)w.double_quant, (const float*)w.absmax, (const uint8_t*)w.absmax_q8,
                      (const float*)w.absmax_scale, (const float*)w.absmax_offset, scales, ld, flags, nflags,
                      weight_format(w));
}

inline cudaError_t launch_dq_encode(const float* y, int64_t n, uint8_t* codes, int dt, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    note_launch();
    k_dq_encode<<<(unsigned)blocks, 256, 0, s>>>(y, n, codes, dt);
    return cudaGetLastError();
}

inline cudaError_t launch_encode(const float* x, int64_t n, uint8_t* codes, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    note_launch();
    k_encode<<<(unsigned)blocks, 256, 0, s>>>(x, n, codes, nf4_search_table());
    return cudaGetLastError();
}

}  // namespace qlora
