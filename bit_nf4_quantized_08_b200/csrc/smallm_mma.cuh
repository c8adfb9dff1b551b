// smallm_mma.cuh -- the forward for few tokens (M <= 32), where the layer is
// bound by the bytes of the 4-bit weight.
//
//   Y^T [N x M] = W' [N x K] X^T + B [N x r] sU^T,   sU = bf16(s X A^T)
//
// The block constant is factored out of each 64-element block (QLoRA paper
// digest, sec. 4 doubleDequant: w' = nf4[code] * a'):
//   Y[m][n] = sum_b (a'_{n,b} / L) * sum_{k in b} (L nf4[c_{n,k}]) x[m][k]
// so the weight operand of the inner sum is one of 16 fixed values, taken
// from a table instead of being rebuilt per block; L = 1.18881 is a fixed
// prescale that halves the bf16 rounding error of those 16 values (largest
// relative error 1.6e-3 instead of 3.1e-3).  The inner sums are warp-level
// tensor-core MMAs (m16n8k16, bf16 in, fp32 out) fed from registers: 16
// weight rows by 8 tokens per instruction, so the expanded weight never
// touches shared memory and no MMA completion has to be signalled.
//
// Lookup: a 256-entry table of bf16 pairs, one entry per code byte (the two
// codes of two neighbouring elements), replicated for the 32 lanes at a
// 256-byte stride in shared memory, so entry e of lane l sits at
// base + e * 256 + l * 4: one PRMT forms the address from the code byte and
// the lane's base, one conflict-free LDS returns the two bf16 values of an
// MMA operand register.
//
// K permutation: within each 64-element block, MMA k-index j of thread
// group position t (the fragment's columns 2t, 2t+1, 2t+8, 2t+9 of chunk c)
// maps to the physical elements 16t + 4c + {0, 1, 2, 3}.  A sum over k does
// not depend on the order, as long as both operands use the same map; with
// it every thread reads 8 contiguous code bytes per weight row and 32
// contiguous bytes of X per token for a block.
//
// Work split: items are (group of 16R weight rows, four 64-element blocks),
// so that each row is read in whole 128-byte lines, with the LoRA
// up-projection as extra 64-wide items after the weight items; every warp of
// a persistent grid takes one contiguous share of the item list (stream-K),
// so each streams the same number of weight bytes, and loads the codes of
// its next item while it computes the current one.  A group cut
// between warps is finished by whichever of its warps arrives last (an
// integer counter): it adds every warp's fp32 partial in warp order
// (deterministic) and writes Y.  Nothing waits on another warp.
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

// Prescale L of the table per code book: for NF4 it halves the bf16 error of
// the 16 values; for FP4 (multiples of 1/12) 1.5 makes every value exact.
__device__ __forceinline__ float small_m_table_scale(int ct) { return ct ? 1.5f : 1.18881f; }

struct SmallMmaParams {
    const uint8_t* codes;   // [N][K/2]
    const uint8_t* q8;      // [N * K/64] (double quantization)
    const float* c1;
    const float* offset;
    const float* absmax;    // [N * K/64] without double quantization
    int dq;
    const uint16_t* X;      // [M][K] bf16
    const uint16_t* B;      // [N][r] bf16 (LoRA), unused when lora_ks == 0
    const uint16_t* sU;     // [M][rt] bf16
    int M, N, K, KB;        // KB = K / 64
    int r, rt, seg_rows, lora_ks;
    float inv_scale;        // 1 / L
    QFormat fmt;            // code book, 8-bit code book, block size
    int QW;                 // weight items per group: ceil(KB / QB)
    int GL;                 // items per group: QW + lora_ks
    int64_t items;          // groups * GL
    uint16_t* Y;            // [M][N]
    float* part;            // [warps][2][16R][8 NT8] fp32 partials
    uint32_t* counters;     // [groups]: (epoch << 8) | arrivals
    uint32_t epoch;         // 24 bits, nonzero
};

template <int NT8, int R>
struct SmallMmaShape {
    static constexpr int WARPS = 16;
    static constexpr int THREADS = 32 * WARPS;
    static constexpr int NPAD = 8 * NT8;
    static constexpr int GROWS = 16 * R;
    static constexpr int QB = 4;  // 64-element blocks per weight item: a 128-byte line of every row
    // 64 KB table at the first 64 KB-aligned shared address, the fp32 t8
    // table of the double quantization below it
    static constexpr int SMEM = 2 * 65536;
    static constexpr int PART_FLOATS = 2 * GROWS * NPAD;  // per warp
};

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ float lds_f32(uint32_t a) { return __uint_as_float(lds_u32(a)); }
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// Table entry of byte k (0..3) of word w for this lane: lane_base holds the
// table base (64 KB aligned) plus lane * 4, so the address is
// [lane_base.b3, lane_base.b2, w.byte_k, lane_base.b0].
template <int KBYTE>
__device__ __forceinline__ uint32_t lut(uint32_t w, uint32_t lane_base) {
    return lds_u32(prmt(w, lane_base, 0x7604u | (KBYTE << 4)));
}

// Index of the warp whose share [I w / G, I (w + 1) / G) holds item x.
__device__ __forceinline__ int owner_warp(int64_t x, int64_t I, int G) {
    int w = (int)((x * G) / I);
    while (w + 1 < G && (I * (w + 1)) / G <= x) ++w;
    while (w > 0 && (I * w) / G > x) --w;
    return w;
}

template <int NT8, int R>
__global__ void __launch_bounds__(SmallMmaShape<NT8, R>::THREADS, 1)
    k_smallm_mma(const __grid_constant__ SmallMmaParams p) {
    using S = SmallMmaShape<NT8, R>;
    constexpr int NPAD = S::NPAD, GROWS = S::GROWS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const uint32_t lut_base = (sbase + 0xFFFFu) & ~0xFFFFu;
    // the fp32 t8 table (1 KB): below the lookup table when there is room, else after it
    const uint32_t t8s = (lut_base - sbase >= 1024u) ? sbase : lut_base + 65536u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;

    // tables: entry e = {L nf4[e >> 4] (bits 0..15), L nf4[e & 15] (bits 16..31)}
    for (int idx = threadIdx.x; idx < 256 * 32; idx += blockDim.x) {
        const int e = idx >> 5, l = idx & 31;
        const float L = small_m_table_scale(p.fmt.code_type);
        const float vlo = __fmul_rn(code_value(p.fmt.code_type, e >> 4), L);
        const float vhi = __fmul_rn(code_value(p.fmt.code_type, e & 15), L);
        sts_u32(lut_base + (uint32_t)(e * 256 + l * 4), pack_bf16x2(vlo, vhi));
    }
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        sts_u32(t8s + 4u * i, __float_as_uint(dq_value(p.fmt.dq_type, (p.fmt.dq_type == 0 || i < 253) ? i : 0)));
    __syncthreads();
    // the weight, X and the adapter operands may come from the kernels just
    // before (the quantizer, the sU GEMM, an earlier layer): wait for them
    pdl_wait();
    const uint32_t lane_base = lut_base + (uint32_t)lane * 4u;
    const float off = p.dq ? __ldg(p.offset) : 0.0f;

    const int G = gridDim.x * S::WARPS;
    const int w = blockIdx.x * S::WARPS + warp;
    const int64_t I = p.items;
    const int64_t i0 = (I * w) / G, i1 = (I * (w + 1)) / G;
    const int64_t rowb = p.K / 2;  // code bytes per weight row
    constexpr int QB = S::QB;

    // code bytes (8 per row and block: this thread's quarter of each 32-byte
    // block chunk) and 8-bit block codes of one weight item, loaded one item
    // ahead of its use
    struct Pf {
        uint2 cw[R][2][QB];
        uint32_t q8[R][2];  // QB block codes, byte j = block j
    };
    auto prefetch = [&](int64_t item, Pf& f) {
        const int g = (int)(item / p.GL), kq = (int)(item - (int64_t)g * p.GL);
        if (kq >= p.QW) return;  // LoRA item: nothing to fetch ahead
        const int n0 = g * GROWS;
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int n = n0 + 16 * rt + gid + 8 * h;
                uint32_t q = 0;
#pragma unroll
                for (int j = 0; j < QB; ++j) {
                    const int kb = kq * QB + j;
                    if (n < p.N && kb < p.KB) {
                        f.cw[rt][h][j] = __ldcs(reinterpret_cast<const uint2*>(p.codes + (int64_t)n * rowb + kb * 32 + 8 * tig));
                        if (p.dq) q |= (uint32_t)__ldg(p.q8 + (((int64_t)n * p.KB + kb) >> p.fmt.bs_shift)) << (8 * j);
                    } else {
                        f.cw[rt][h][j] = make_uint2(0u, 0u);
                    }
                }
                f.q8[rt][h] = q;
            }
    };

    float acc[R][NT8][4];
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = 0; b < NT8; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.0f;
    Pf cur, nxt;
    if (i0 < i1) prefetch(i0, cur);
    for (int64_t it = i0; it < i1; ++it) {
        if (it + 1 < i1) prefetch(it + 1, nxt);
        const int g = (int)(it / p.GL);
        const int kq = (int)(it - (int64_t)g * p.GL);
        const int n0 = g * GROWS;
        if (kq < p.QW) {
            // ------------------------------------------------------ weight item: QB blocks
#pragma unroll
            for (int j = 0; j < QB; ++j) {
                const int kb = kq * QB + j;
                if (kb >= p.KB) break;
                uint32_t xf[NT8][8];
#pragma unroll
                for (int nt = 0; nt < NT8; ++nt) {
                    const int m = nt * 8 + gid;
                    if (m < p.M) {
                        const uint4* src = reinterpret_cast<const uint4*>(p.X + (int64_t)m * p.K + kb * 64 + 16 * tig);
                        const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
                        xf[nt][0] = u0.x; xf[nt][1] = u0.y; xf[nt][2] = u0.z; xf[nt][3] = u0.w;
                        xf[nt][4] = u1.x; xf[nt][5] = u1.y; xf[nt][6] = u1.z; xf[nt][7] = u1.w;
                    } else {
#pragma unroll
                        for (int q = 0; q < 8; ++q) xf[nt][q] = 0u;
                    }
                }
#pragma unroll
                for (int rt = 0; rt < R; ++rt) {
                    float sc[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int n = n0 + 16 * rt + gid + 8 * h;
                        float a = 0.0f;
                        if (n < p.N) {
                            const int64_t b = ((int64_t)n * p.KB + kb) >> p.fmt.bs_shift;
                            a = p.dq ? __fadd_rn(__fmul_rn(lds_f32(t8s + 4u * ((cur.q8[rt][h] >> (8 * j)) & 0xFFu)),
                                                           __ldg(p.c1 + (b >> 8))), off)
                                     : __ldg(p.absmax + b);
                        }
                        sc[h] = __fmul_rn(a, p.inv_scale);
                    }
                    float d[NT8][4];
#pragma unroll
                    for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                        for (int q = 0; q < 4; ++q) d[nt][q] = 0.0f;
                    const uint32_t g0x = cur.cw[rt][0][j].x, g0y = cur.cw[rt][0][j].y;
                    const uint32_t g8x = cur.cw[rt][1][j].x, g8y = cur.cw[rt][1][j].y;
                    {   // chunk 0: bytes 0, 1
                        const uint32_t a0 = lut<0>(g0x, lane_base), a2 = lut<1>(g0x, lane_base);
                        const uint32_t a1 = lut<0>(g8x, lane_base), a3 = lut<1>(g8x, lane_base);
#pragma unroll
                        for (int nt = 0; nt < NT8; ++nt) mma_16816(d[nt], a0, a1, a2, a3, xf[nt][0], xf[nt][1]);
                    }
                    {   // chunk 1: bytes 2, 3
                        const uint32_t a0 = lut<2>(g0x, lane_base), a2 = lut<3>(g0x, lane_base);
                        const uint32_t a1 = lut<2>(g8x, lane_base), a3 = lut<3>(g8x, lane_base);
#pragma unroll
                        for (int nt = 0; nt < NT8; ++nt) mma_16816(d[nt], a0, a1, a2, a3, xf[nt][2], xf[nt][3]);
                    }
                    {   // chunk 2: bytes 4, 5
                        const uint32_t a0 = lut<0>(g0y, lane_base), a2 = lut<1>(g0y, lane_base);
                        const uint32_t a1 = lut<0>(g8y, lane_base), a3 = lut<1>(g8y, lane_base);
#pragma unroll
                        for (int nt = 0; nt < NT8; ++nt) mma_16816(d[nt], a0, a1, a2, a3, xf[nt][4], xf[nt][5]);
                    }
                    {   // chunk 3: bytes 6, 7
                        const uint32_t a0 = lut<2>(g0y, lane_base), a2 = lut<3>(g0y, lane_base);
                        const uint32_t a1 = lut<2>(g8y, lane_base), a3 = lut<3>(g8y, lane_base);
#pragma unroll
                        for (int nt = 0; nt < NT8; ++nt) mma_16816(d[nt], a0, a1, a2, a3, xf[nt][6], xf[nt][7]);
                    }
#pragma unroll
                    for (int nt = 0; nt < NT8; ++nt) {
                        acc[rt][nt][0] = __fmaf_rn(sc[0], d[nt][0], acc[rt][nt][0]);
                        acc[rt][nt][1] = __fmaf_rn(sc[0], d[nt][1], acc[rt][nt][1]);
                        acc[rt][nt][2] = __fmaf_rn(sc[1], d[nt][2], acc[rt][nt][2]);
                        acc[rt][nt][3] = __fmaf_rn(sc[1], d[nt][3], acc[rt][nt][3]);
                    }
                }
            }
        } else {
            // ------------------------------------------------------ LoRA item: 64 adapter columns, B rows x sU
            const int j0 = (kq - p.QW) * 64 + 16 * tig;  // adapter column of this thread's 16
            const bool v0 = j0 + 8 <= p.r, v1 = j0 + 16 <= p.r;
            const int ucol = (p.seg_rows ? (n0 / p.seg_rows) * p.r : 0) + j0;
            uint32_t xf[NT8][8];
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt) {
                const int m = nt * 8 + gid;
                uint4 u0 = make_uint4(0, 0, 0, 0), u1 = make_uint4(0, 0, 0, 0);
                if (m < p.M) {
                    const uint4* src = reinterpret_cast<const uint4*>(p.sU + (int64_t)m * p.rt + ucol);
                    if (v0) u0 = __ldg(src);
                    if (v1) u1 = __ldg(src + 1);
                }
                xf[nt][0] = u0.x; xf[nt][1] = u0.y; xf[nt][2] = u0.z; xf[nt][3] = u0.w;
                xf[nt][4] = u1.x; xf[nt][5] = u1.y; xf[nt][6] = u1.z; xf[nt][7] = u1.w;
            }
#pragma unroll
            for (int rt = 0; rt < R; ++rt) {
                uint32_t bw[2][8];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int n = n0 + 16 * rt + gid + 8 * h;
                    uint4 u0 = make_uint4(0, 0, 0, 0), u1 = make_uint4(0, 0, 0, 0);
                    if (n < p.N) {
                        const uint4* src = reinterpret_cast<const uint4*>(p.B + (int64_t)n * p.r + j0);
                        if (v0) u0 = __ldg(src);
                        if (v1) u1 = __ldg(src + 1);
                    }
                    bw[h][0] = u0.x; bw[h][1] = u0.y; bw[h][2] = u0.z; bw[h][3] = u0.w;
                    bw[h][4] = u1.x; bw[h][5] = u1.y; bw[h][6] = u1.z; bw[h][7] = u1.w;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int nt = 0; nt < NT8; ++nt)
                        mma_16816(acc[rt][nt], bw[0][2 * c], bw[1][2 * c], bw[0][2 * c + 1], bw[1][2 * c + 1],
                                  xf[nt][2 * c], xf[nt][2 * c + 1]);
            }
        }
        cur = nxt;

        // ---------------------------------------------------------- end of a segment: output
        if (it + 1 < i1 && kq + 1 < p.GL) continue;
        const int64_t gstart = (int64_t)g * p.GL;
        const int64_t seg0 = i0 > gstart ? i0 : gstart;
        const bool whole = seg0 == gstart && kq + 1 == p.GL;
        bool write_y = whole;
        if (!whole) {
            const int slot = seg0 > gstart ? 0 : (i0 < gstart ? 1 : 0);
            float* mine = p.part + ((int64_t)w * 2 + slot) * (GROWS * NPAD);
#pragma unroll
            for (int rt = 0; rt < R; ++rt)
#pragma unroll
                for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        __stcg(reinterpret_cast<float2*>(mine + (16 * rt + gid + 8 * h) * NPAD + nt * 8 + 2 * tig),
                               make_float2(acc[rt][nt][2 * h], acc[rt][nt][2 * h + 1]));
            __threadfence();
            __syncwarp();
            // contributors: the warps from the one holding the group's first
            // item to the one holding its last, less any with an empty share
            const int wf = owner_warp(gstart, I, G), wl = owner_warp(gstart + p.GL - 1, I, G);
            uint32_t ncontrib = 0;
            for (int c = wf; c <= wl; ++c) ncontrib += ((I * c) / G < (I * (c + 1)) / G) ? 1u : 0u;
            // arrivals of this launch at the group's counter (epoch in the high bits)
            uint32_t before = 0;
            if (lane == 0) {
                uint32_t* ctr = p.counters + g;
                uint32_t cv = *reinterpret_cast<volatile uint32_t*>(ctr);
                while (true) {
                    const bool same = (cv >> 8) == p.epoch;
                    const uint32_t want = same ? cv + 1u : ((p.epoch << 8) | 1u);
                    const uint32_t prev = atomicCAS(ctr, cv, want);
                    if (prev == cv) {
                        before = same ? (cv & 0xFFu) : 0u;
                        break;
                    }
                    cv = prev;
                }
                if (before + 1 == ncontrib) *ctr = 0u;  // last arrival: reset for the next launch
            }
            before = __shfl_sync(0xffffffffu, before, 0);
            if (before + 1 == ncontrib) {
                __threadfence();
                // add every contributor's partial in warp order
#pragma unroll
                for (int rt = 0; rt < R; ++rt)
#pragma unroll
                    for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[rt][nt][q] = 0.0f;
                for (int c = wf; c <= wl; ++c) {
                    if ((I * c) / G == (I * (c + 1)) / G) continue;
                    const int cslot = ((I * c) / G < gstart) ? 1 : 0;
                    const float* src = p.part + ((int64_t)c * 2 + cslot) * (GROWS * NPAD);
#pragma unroll
                    for (int rt = 0; rt < R; ++rt)
#pragma unroll
                        for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const float2 v = __ldcg(reinterpret_cast<const float2*>(
                                    src + (16 * rt + gid + 8 * h) * NPAD + nt * 8 + 2 * tig));
                                acc[rt][nt][2 * h] = __fadd_rn(acc[rt][nt][2 * h], v.x);
                                acc[rt][nt][2 * h + 1] = __fadd_rn(acc[rt][nt][2 * h + 1], v.y);
                            }
                }
                write_y = true;
            }
        }
        if (write_y) {
#pragma unroll
            for (int rt = 0; rt < R; ++rt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int n = n0 + 16 * rt + gid + 8 * h;
                    if (n >= p.N) continue;
#pragma unroll
                    for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int m = nt * 8 + 2 * tig + e;
                            if (m < p.M)
                                p.Y[(int64_t)m * p.N + n] = (uint16_t)(pack_bf16x2(acc[rt][nt][2 * h + e], 0.0f) & 0xFFFFu);
                        }
                }
        }
#pragma unroll
        for (int a = 0; a < R; ++a)
#pragma unroll
            for (int b = 0; b < NT8; ++b)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.0f;
    }
}

}  // namespace qlora
