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
// t = fl(128 x + 1.5 * 2^24 + 128) lies in [2^24, 2^25) for |x| <= 1.03,
// where the spacing of fp32 values is 2, so t = 1.5 * 2^24 + 2 v with
// v = RN(64 x + 64) and the low mantissa bits of t hold v; the bucket is
// key = floor(v / 4), and (t's bits & 0xFC) = 4 key is already the byte
// offset of the bucket's 4-byte table entries: one LOP forms the address
// of both tables, and 4-byte entries at a 4-byte stride put every bucket on
// its own shared-memory bank (keys 0 and 32 share one, and both are rare).
// Bucket key covers x in [(4 key - 64.5) / 64, (4 key - 60.5) / 64], an
// interval of width 1/16, narrower than the smallest gap between two
// decision thresholds (0.080), so each bucket holds at most one threshold
// T_key; base_key counts the thresholds at or below the bucket's lower edge.
// code(x) = base_key + (x >= T_key), where threshold j is the smallest fp32
// strictly above the exact midpoint of codes j and j+1 (so an exact tie
// stays with the lower code).  The table holds P_key, the largest fp32 below
// T_key (3.0 without a threshold): x >= T_key exactly when x > P_key.  The
// 8-bit mask keeps any input (NaN included) inside the 64-entry tables.
struct __align__(16) SearchSmem {
    float P[64];     // P_key
    uint32_t B[64];  // base_key | extra_key << 16
    float Q[64];     // -P_key * 2^100 (NF4 compare on the FMA pipe)
    float H[64];     // 16 base_key (the code in a byte's high nibble; NF4)
    float L[64];     // 2^23 + base_key (the low nibble, on the 2^23 integer grid)
};

__device__ __forceinline__ void load_search_tables(SearchSmem& st, const Nf4SearchTable& tab) {
    for (int i = threadIdx.x; i < 64; i += blockDim.x) {
        st.P[i] = i < kSearchBuckets ? tab.thr[i] : 3.0f;
        st.B[i] = i < kSearchBuckets ? (uint32_t)tab.base[i] | ((uint32_t)max(tab.inc[i] - 1, 0) << 16) : 15u;
        const float bk = i < kSearchBuckets ? (float)tab.base[i] : 15.0f;
        st.Q[i] = -st.P[i] * 1.26765060e30f;  // exact: a power-of-two scale
        st.H[i] = 16.0f * bk;
        st.L[i] = 8388608.0f + bk;
    }
}

constexpr float kKeyMagic = 25165952.0f;  // 1.5 * 2^24 + 128
constexpr float kKeyScale = 128.0f;

// CT = 1 (FP4): a bucket's threshold may count twice (inc = 2, stored as
// extra = inc - 1 in the entry's high half; NF4 entries have extra = 0).
template <int CT = 0>
__device__ __forceinline__ uint32_t nf4_lookup(float x, float t, const SearchSmem& st) {
    const uint32_t off = __float_as_uint(t) & 0xFCu;
    const float P = *reinterpret_cast<const float*>(reinterpret_cast<const char*>(st.P) + off);
    const uint32_t e = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(st.B) + off);
    const uint32_t above = P < x ? 1u : 0u;
    if (CT == 0) return e + above;
    return (e & 0xFFFFu) + above * ((e >> 16) + 1u);
}

template <int CT = 0>
__device__ __forceinline__ uint32_t nf4_search(float x, const SearchSmem& st) {
    return nf4_lookup<CT>(x, fmaf(x, kKeyScale, kKeyMagic), st);
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

// The two bf16 values of a packed word as an fp32 pair {low half, high
// half} in one 64-bit register (built in place, so no register moves).
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t r) {
    uint64_t d;
    asm("{\n\t.reg .b32 lo, hi;\n\tshl.b32 lo, %1, 16;\n\tand.b32 hi, %1, 0xFFFF0000;\n\tmov.b64 %0, {lo, hi};\n\t}"
        : "=l"(d)
        : "r"(r));
    return d;
}

// sat(x * 2^100 + q) with q = -P * 2^100: 1 exactly when x > P, else 0.
// The FMA rounds once, so the result has the sign of x - P.  With |P| at
// least 0.0398 (the NF4 thresholds; 3.0 where a bucket has none), two
// distinct fp32 values x and P differ by at least 2^-30, so a positive
// difference scales to at least 2^70 and saturates to 1; x == P gives 0,
// and a NaN x saturates to 0.
__device__ __forceinline__ float above_sat(float x, float q) {
    float a;
    asm("fma.rn.sat.f32 %0, %1, 0f71800000, %2;" : "=f"(a) : "f"(x), "f"(q));
    return a;
}

// The packed byte (code(x0) << 4) | code(x1) of two elements x = fl(w * rcp)
// (w2 = {w0, w1}), as the fp32 value 2^23 + byte (the byte in its low 8
// bits): one fp32x2 multiply and bucket-key FMA for both.  NF4: the byte is
// 16 (base0 + above0) + base1 + above1, from the high-nibble table of x0's
// bucket and the low-nibble table of x1's, all exact small integers in fp32.
// FP4 takes the general lookup.
template <int CT>
__device__ __forceinline__ uint32_t nf4_byte2(uint64_t w2, uint64_t rcp2, uint64_t k2, uint64_t m2,
                                              const SearchSmem& st) {
    const uint64_t x2 = f2_mul(w2, rcp2);
    const uint64_t t2 = f2_fma(x2, k2, m2);
    float x0, x1, t0, t1;
    f2_unpack(x2, x0, x1);
    f2_unpack(t2, t0, t1);
    if (CT != 0) return 0x4B000000u + (nf4_lookup<CT>(x0, t0, st) << 4) + nf4_lookup<CT>(x1, t1, st);
    const uint32_t o0 = __float_as_uint(t0) & 0xFCu, o1 = __float_as_uint(t1) & 0xFCu;
    auto at = [](const float* tab, uint32_t off) {
        return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(tab) + off);
    };
    const float a0 = above_sat(x0, at(st.Q, o0)), a1 = above_sat(x1, at(st.Q, o1));
    const float y0 = __fmaf_rn(a0, 16.0f, at(st.H, o0));
    const float y1 = __fadd_rn(a1, at(st.L, o1));
    return __float_as_uint(__fadd_rn(y0, y1));
}

// Four bytes b_k (the low byte of each word) as one word, b0 lowest.
__device__ __forceinline__ uint32_t pack4_low_bytes(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// Shape of the quantizer: one CTA per SM, 16 coding warps and a loader warp;
// a stage of the shared-memory ring holds one group of 16384 elements as
// 128-byte rows (64 bf16 or 32 fp32) in the TMA's 128-byte swizzle, and a
// lane codes 32 consecutive elements of a group.
template <bool BF16>
struct QuantRing {
    static constexpr int CW = 16;                          // coding warps
    static constexpr int THREADS = 32 * (CW + 1);          // + the loader warp
    static constexpr int STAGE = 16384 * (BF16 ? 2 : 4);   // bytes of one group
    static constexpr int NST = BF16 ? 6 : 3;               // stages
    static constexpr int ROWS = STAGE / 128;               // 128-byte rows of a stage
    static constexpr int BOX_ROWS = 256;                   // rows of one TMA box
    static constexpr int OFF_BAR = NST * STAGE;            // full[NST], empty[NST]
    static constexpr int OFF_PART = OFF_BAR + 16 * NST;    // double [NST + 1][CW]: warp subtree sums
    static constexpr int OFF_FLAG = OFF_PART + 8 * (NST + 1) * CW;  // abort flag
    static constexpr int SMEM = OFF_FLAG + 16 + 1024;      // + alignment slack
};

// One lane's share of a group: the block maxima of its 32 elements (raw, in
// order), their codes, and the warp's fp64 pairwise subtree sum of its
// blocks' maxima (the same value in every lane; 0 when not wanted).  e: the
// lane's first element.  WHOLE: all 32 lie inside the tensor.
template <bool BF16, int CT, int BS, bool WHOLE>
__device__ __forceinline__ double quant_lane(const uint32_t (&raw)[BF16 ? 16 : 32], int64_t e, int64_t n,
                                             int64_t nb, uint8_t* codes, float* absmax, bool sums,
                                             const SearchSmem& st, int lane) {
    constexpr int bshift = 6 + BS;   // log2 of the block size
    constexpr int blanes = 2 << BS;  // lanes per block
    // block absmax (exact: a max of magnitudes)
    float a;
    if (BF16) {
        // packed bf16 max of magnitudes (the sign of each half is the xor of
        // the signs, dropped at the end)
        uint32_t m = raw[0];
#pragma unroll
        for (int k = 1; k < 16; ++k) asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(raw[k]));
        m &= 0x7FFF7FFFu;
        m = max(m & 0xFFFFu, m >> 16);
        a = __uint_as_float(m << 16);
    } else {
        a = 0.0f;
#pragma unroll
        for (int k = 0; k < 32; ++k) a = fmaxf(a, fabsf(__uint_as_float(raw[k])));
    }
#pragma unroll
    for (int o = 1; o < blanes; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const int64_t b = e >> bshift;
    const bool bvalid = WHOLE || b < nb;
    if ((lane & (blanes - 1)) == 0 && bvalid && absmax && QLORA_CHECK(b >= 0 && b < nb)) absmax[b] = a;

    // codes: byte j of w[h] = (code[8h + 2j] << 4) | code[8h + 2j + 1]
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (a >= 1.17549435e-38f) {
        const float rcp = __frcp_rn(a);
        const uint64_t rcp2 = f2_pack(rcp, rcp);
        const uint64_t k2 = f2_pack(kKeyScale, kKeyScale), m2 = f2_pack(kKeyMagic, kKeyMagic);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            uint32_t by[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int k = 4 * h + j;
                const uint64_t w2 = BF16 ? bf16x2_to_f2(raw[k])
                                         : f2_pack(__uint_as_float(raw[2 * k]), __uint_as_float(raw[2 * k + 1]));
                by[j] = nf4_byte2<CT>(w2, rcp2, k2, m2, st);
            }
            w[h] = pack4_low_bytes(by[0], by[1], by[2], by[3]);
        }
    } else {
        // zero or subnormal block: exact power-of-two prescale 2^64
        const float p = 18446744073709551616.0f;
        const float rcp = (a == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(a, p));
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const uint32_t bits = BF16 ? ((k & 1) ? (raw[k >> 1] & 0xFFFF0000u) : (raw[k >> 1] << 16)) : raw[k];
            const uint32_t c = nf4_search<CT>(__fmul_rn(__fmul_rn(__uint_as_float(bits), p), rcp), st);
            w[k >> 3] += c << (4 * ((k & 7) ^ 1));
        }
    }
    if (WHOLE || e + 32 <= n) {
        if (QLORA_CHECK(e >= 0 && (e >> 1) + 16 <= (n + 1) / 2))
            __stcs(reinterpret_cast<uint4*>(codes + (e >> 1)), make_uint4(w[0], w[1], w[2], w[3]));
    } else if (e < n) {
        const int valid = (int)(n - e);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (2 * j < valid) {
                uint32_t byte = (w[j >> 2] >> (8 * (j & 3))) & 0xFFu;
                if (2 * j + 1 >= valid) byte &= 0xF0u;  // no element after the last one
                if (QLORA_CHECK((e >> 1) + j < (n + 1) / 2)) codes[(e >> 1) + j] = (uint8_t)byte;
            }
        }
    }
    double t = 0.0;
    if (sums) {
        // the warp's leaves in pairwise order: partners blanes, 2 blanes, ..
        // lanes apart (x + y and y + x are the same IEEE sum, so every lane
        // ends with the same value)
        t = bvalid ? (double)a : 0.0;
#pragma unroll
        for (int o = blanes; o < 32; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    }
    return t;
}

// fp64 pairwise sum of the 16 warp subtree sums of a group, in warp order.
__device__ __forceinline__ double quant_group_sum(const double* p) {
    double v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = p[k];
#pragma unroll
    for (int d = 1; d < 16; d <<= 1)
#pragma unroll
        for (int k = 0; k < 16; k += 2 * d) v[k] = v[k] + v[k + d];
    return v[0];
}

// ---------------------------------------------------------------------------
// K1: quantize.  A persistent grid of one CTA per SM; CTA c takes the
// groups of 16384 elements c, c + G, c + 2G, ...  The loader warp streams
// every whole group into the ring with one TMA box per 256 rows (refilled as
// the coding warps release a stage); a tensor's partial last group is read
// with plain, bounds-checked loads instead.  In a group, lane l of coding
// warp w takes elements [1024 w + 32 l, + 32) (bf16: half of row
// 16 w + l / 2; fp32: row 32 w + l), so 2 << BS lanes make one block (64,
// 128 or 256 elements); the swizzle puts the 16-byte chunks of the eight
// lanes of a quarter warp in distinct banks.  Also writes each group's fp64
// pairwise-tree sum of block maxima for the double-quantization offset: each
// warp adds its own leaves (a subtree) with shuffles and leaves the sum in
// shared memory before it releases the stage; the loader, which waits for
// that release anyway, adds the 16 subtree sums.  CT: code book (0 NF4, 1
// FP4).
// ---------------------------------------------------------------------------
template <bool BF16, int CT, int BS>
__global__ void __launch_bounds__(QuantRing<BF16>::THREADS, 1)
    k_quantize_blocks(const __grid_constant__ CUtensorMap tmW, const void* W, int64_t n, uint8_t* codes,
                      float* absmax, double* group_sums, Nf4SearchTable tab, uint64_t timeout_ns) {
    using R = QuantRing<BF16>;
    constexpr int CW = R::CW, NST = R::NST;
    constexpr int bshift = 6 + BS;  // log2 of the block size
    __shared__ SearchSmem st;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* gb = smem_raw + (base - raw_base);
    const uint32_t bar = base + R::OFF_BAR;
    auto full = [&](int s) { return bar + 8u * s; };
    auto empty = [&](int s) { return bar + 8u * (NST + s); };
    double* part = reinterpret_cast<double*>(gb + R::OFF_PART);  // [NST + 1][CW]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + R::OFF_FLAG);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WaitCfg wc{timeout_ns};
    const int64_t ng = (n + 16383) >> 14, nfull = n >> 14;
    const int64_t nb = (n + (1 << bshift) - 1) >> bshift;
    const int G = gridDim.x;
    // this CTA's groups, and how many of them are whole (the partial one, if
    // any, is the tensor's last group, so it comes last here too)
    const int64_t mine = blockIdx.x < ng ? (ng - blockIdx.x + G - 1) / G : 0;
    const int64_t mine_full = blockIdx.x < nfull ? (nfull - blockIdx.x + G - 1) / G : 0;
    const bool sums = group_sums != nullptr;

    // dependent launch: resident before the kernel ahead ends, no access to
    // global memory before it has.  The kernels that wait this way take no
    // __restrict__ pointers: with them the compiler may move loads of
    // "unchanging" data above griddepcontrol.wait.
    pdl_trigger();
    load_search_tables(st, tab);
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), CW);
        }
        *abort_flag = 0;
        fence_mbar_init();
        if (mine_full > 0) prefetch_tensormap(&tmW);
    }
    __syncthreads();
    pdl_wait();

    int issued[NST];  // loads issued into each stage (the loader lane)
#pragma unroll
    for (int s = 0; s < NST; ++s) issued[s] = 0;
    if (warp == CW) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            // group j of this CTA is released: its sum (stage j % NST)
            auto group_done = [&](int64_t j) {
                const int s = (int)(j % NST);
                if (*abort_flag || !mbar_wait_sleep(empty(s), (uint32_t)((j / NST) & 1), wc, 64)) {
                    *abort_flag = 1;
                    return false;
                }
                const int64_t g = blockIdx.x + j * G;
                if (sums && QLORA_CHECK(g < ng)) group_sums[g] = quant_group_sum(part + s * CW);
                return true;
            };
            bool ok = true;
            for (int64_t i = 0; i < mine_full && ok; ++i) {
                const int s = (int)(i % NST);
                // the coding warps have released the stage's previous group
                if (i >= NST && !(ok = group_done(i - NST))) break;
                const int64_t g = blockIdx.x + i * G;
                mbar_arrive_expect_tx(full(s), (uint32_t)R::STAGE);
#pragma unroll
                for (int b = 0; b < R::ROWS / R::BOX_ROWS; ++b)
                    tma_load_2d(base + (uint32_t)(s * R::STAGE + b * R::BOX_ROWS * 128), &tmW, full(s), 0,
                                (int)(g * R::ROWS + b * R::BOX_ROWS));
#pragma unroll
                for (int t = 0; t < NST; ++t) issued[t] += (t == s);
            }
            for (int64_t j = mine_full > NST ? mine_full - NST : 0; j < mine_full && ok; ++j) ok = group_done(j);
        }
    } else {
        // ------------------------------------------------------------ coding warps
        // 128-byte row of the stage and first 16-byte chunk of this lane
        const int row = BF16 ? 16 * warp + (lane >> 1) : 32 * warp + lane;
        const int chunk0 = BF16 ? 4 * (lane & 1) : 0;
        const uint32_t lane_off = (uint32_t)row * 128u;
        const uint32_t sw = (uint32_t)(row & 7);
        bool ok = true;
        for (int64_t i = 0; i < mine_full; ++i) {
            const int s = (int)(i % NST);
            const int64_t e = (blockIdx.x + i * G) * 16384 + (int64_t)warp * 1024 + lane * 32;  // first element
            // every lane waits (and so sees the TMA's writes); the warp leaves
            // together if any lane gave up
            ok = !*abort_flag && mbar_wait_hint(full(s), (uint32_t)((i / NST) & 1), wc, 1000);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                if (lane == 0) *abort_flag = 1;
                break;
            }
            uint32_t raw[BF16 ? 16 : 32];
            const uint32_t sb = base + (uint32_t)(s * R::STAGE) + lane_off;
#pragma unroll
            for (int v = 0; v < (BF16 ? 4 : 8); ++v) {
                const uint4 q = ld_shared_v4(sb + ((((uint32_t)(chunk0 + v)) ^ sw) << 4));
                raw[4 * v + 0] = q.x;
                raw[4 * v + 1] = q.y;
                raw[4 * v + 2] = q.z;
                raw[4 * v + 3] = q.w;
            }
            const double t = quant_lane<BF16, CT, BS, true>(raw, e, n, nb, codes, absmax, sums, st, lane);
            // the subtree sum, then the stage back to the loader (after every
            // lane's reads of it)
            if (lane == 0) part[s * CW + warp] = t;
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(s));
        }
        if (ok && mine > mine_full) {
            // the tensor's partial last group: plain loads, bounds-checked
            const int64_t e = (ng - 1) * 16384 + (int64_t)warp * 1024 + lane * 32;
            uint32_t raw[BF16 ? 16 : 32];
#pragma unroll
            for (int v = 0; v < (BF16 ? 16 : 32); ++v) raw[v] = 0u;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                if (e + k < n) {
                    if (BF16) {
                        const uint32_t h = static_cast<const uint16_t*>(W)[e + k];
                        raw[k >> 1] |= h << ((k & 1) * 16);
                    } else {
                        raw[k] = __float_as_uint(static_cast<const float*>(W)[e + k]);
                    }
                }
            }
            const double t = quant_lane<BF16, CT, BS, false>(raw, e, n, nb, codes, absmax, sums, st, lane);
            if (lane == 0) part[NST * CW + warp] = t;
        }
    }
    // every load issued into the ring has landed before the CTA exits, and
    // the kernel does not complete before the one it depends on
    __syncthreads();
    if (warp == CW && lane == 0) {
        if (sums && mine > mine_full && !*abort_flag && QLORA_CHECK(ng >= 1))
            group_sums[ng - 1] = quant_group_sum(part + NST * CW);
        for (int s = 0; s < NST; ++s)
            if (issued[s] > 0) mbar_wait(full(s), (uint32_t)((issued[s] - 1) & 1), wc);
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

// Nearest 8-bit code of y in [-1, 1]: the candidate k0 = RN(127 y + 127),
// formed by one FMA with 1.5 * 2^23 + 127 (the sum's low mantissa bits are
// k0), is the nearest code or its neighbour (y is within half a step of
// t8[k0]), so two fp32 compares with the thresholds on either side decide;
// ties go to the lower index.  thr = the padded thresholds (shared memory):
// thr[0] = -inf, thr[k + 1] = T_k (k = 0..253), thr[255..259] = +inf, so no
// candidate needs a range check (any input, NaN included, reads inside).
constexpr int kT8Pad = 260;
__device__ __forceinline__ float t8_threshold_padded(int i) {
    if (i == 0) return -INFINITY;
    return i <= 254 ? t8_threshold(i - 1) : INFINITY;
}
__device__ __forceinline__ int nearest_t8(float y, const float* thr) {
    const int k0 = (int)(__float_as_uint(__fmaf_rn(y, 127.0f, 12583039.0f)) & 0xFFu);
    const int down = y < thr[k0] ? 1 : 0;
    const int up = y >= thr[k0 + 1] ? 1 : 0;
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
    __shared__ float t8[kT8Pad];  // E4M3: the 253 code values; linear: the padded decision thresholds
    __shared__ double s_w[8];
    __shared__ float s_off;
    pdl_trigger();
    // shared memory only
    for (int i = threadIdx.x; i < kT8Pad; i += blockDim.x)
        t8[i] = dt ? (i < 253 ? e4m3_value(i) : 2.0f) : t8_threshold_padded(i);
    pdl_wait();
    // this warp's first group: 8 block maxima per lane, loaded before the
    // offset tree so that the two memory round trips overlap
    const int64_t g = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t ng = (nb + 255) >> 8;
    // 8 consecutive maxima of lane's share of group gg (two 16-byte loads
    // when all 8 exist)
    auto load8 = [&](int64_t gg, float (&a)[8]) {
        const int64_t b0 = gg * 256 + lane * 8;
        if (gg < ng && b0 + 8 <= nb) {
            const float4 v0 = *reinterpret_cast<const float4*>(absmax + b0);
            const float4 v1 = *reinterpret_cast<const float4*>(absmax + b0 + 4);
            a[0] = v0.x; a[1] = v0.y; a[2] = v0.z; a[3] = v0.w;
            a[4] = v1.x; a[5] = v1.y; a[6] = v1.z; a[7] = v1.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = (gg < ng && b0 + i < nb) ? absmax[b0 + i] : 0.0f;
        }
    };
    float am[8];
    load8(g, am);
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
    // every (gridDim.x * 8)-th group, loading the next group's maxima while
    // it quantizes the current one
    const int64_t gstride = (int64_t)gridDim.x * 8;
    for (int64_t gg = g; gg < ng; gg += gstride) {
        const int64_t b0 = gg * 256 + lane * 8;
        float nx[8];
        load8(gg + gstride, nx);
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
            if (QLORA_CHECK(b0 >= 0 && b0 + 8 <= nb)) *reinterpret_cast<uint2*>(q8 + b0) = v;
        } else {
            for (int i = 0; i < 8; ++i)
                if (b0 + i < nb) q8[b0 + i] = (uint8_t)q[i];
        }
        if (lane == 0 && QLORA_CHECK(gg < ng)) c1[gg] = c;
#pragma unroll
        for (int i = 0; i < 8; ++i) am[i] = nx[i];
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
            if (QLORA_CHECK((wb0 * 64 + (int64_t)(i * 32 + lane) * 8 + 8) <= n)) __stcs(dst + i * 32 + lane, v);
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
            if (QLORA_CHECK(e < n)) out[e] = *reinterpret_cast<uint16_t*>(&h);
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
    __shared__ float t8[kT8Pad];
    for (int i = threadIdx.x; i < kT8Pad; i += blockDim.x)
        t8[i] = dt ? (i < 253 ? e4m3_value(i) : 2.0f) : t8_threshold_padded(i);
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
    for (int k = 0; k < kSearchBuckets; ++k) {
        // key k: RN(64 x + 64) in [4k, 4k + 3]
        const double lo = (4.0 * k - 64.5) / 64.0, hi = (4.0 * k - 60.5) / 64.0;
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
    using Kern = void (*)(const CUtensorMap, const void*, int64_t, uint8_t*, float*, double*, Nf4SearchTable,
                          uint64_t);
    static constexpr Kern kTable[2][2][3] = {
        {{k_quantize_blocks<false, 0, 0>, k_quantize_blocks<false, 0, 1>, k_quantize_blocks<false, 0, 2>},
         {k_quantize_blocks<false, 1, 0>, k_quantize_blocks<false, 1, 1>, k_quantize_blocks<false, 1, 2>}},
        {{k_quantize_blocks<true, 0, 0>, k_quantize_blocks<true, 0, 1>, k_quantize_blocks<true, 0, 2>},
         {k_quantize_blocks<true, 1, 0>, k_quantize_blocks<true, 1, 1>, k_quantize_blocks<true, 1, 2>}}};
    const int ib = is_bf16 ? 1 : 0, ic = fmt.code_type ? 1 : 0, is = fmt.bs_shift;
    const Kern kern = kTable[ib][ic][is];
    const int smem = is_bf16 ? QuantRing<true>::SMEM : QuantRing<false>::SMEM;
    const int threads = is_bf16 ? QuantRing<true>::THREADS : QuantRing<false>::THREADS;
    static std::once_flag attr_once[2][2][3];
    static cudaError_t attr_err[2][2][3];
    std::call_once(attr_once[ib][ic][is], [&] {
        attr_err[ib][ic][is] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (attr_err[ib][ic][is] != cudaSuccess) return attr_err[ib][ic][is];
    // the whole groups as 128-byte rows (64 bf16 or 32 fp32), 256-row boxes
    CUtensorMap tm;
    memset(&tm, 0, sizeof(tm));
    const int64_t nfull = n >> 14;
    if (nfull > 0) {
        const bool ok = is_bf16 ? make_map(&tm, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, (uint64_t)nfull * 256,
                                           128, 64, QuantRing<true>::BOX_ROWS, CU_TENSOR_MAP_SWIZZLE_128B)
                                : make_map(&tm, W, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 32, (uint64_t)nfull * 512,
                                           128, 32, QuantRing<false>::BOX_ROWS, CU_TENSOR_MAP_SWIZZLE_128B);
        if (!ok) return cudaErrorInvalidValue;
    }
    // persistent: one CTA per SM, at most one per group
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        nsm = 148;
    const int64_t grid = std::min<int64_t>(ng, (int64_t)nsm);
    return launch_pdl(kern, dim3((unsigned)grid), dim3(threads), smem, s, 0, tm, W, n, codes, absmax, group_sums,
                      tab, wait_timeout_ns());
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
