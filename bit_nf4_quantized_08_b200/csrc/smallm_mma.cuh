// smallm_mma.cuh -- the forward for few tokens (M <= 32), where the layer is
// bound by the bytes of the 4-bit weight.
//
//   Y [M x N] = X W'^T + sU B^T,   sU = bf16(s X A^T)
//
// The block constant is factored out of each 64-element block (QLoRA paper
// digest, sec. 4 doubleDequant: w' = nf4[code] * a'):
//   Y[m][n] = sum_b (a'_{n,b} / L) * sum_{k in b} (L nf4[c_{n,k}]) x[m][k]
// so the weight operand of the inner sum is one of 16 fixed values, taken
// from a table instead of being rebuilt per block; L = 1.18881 is a fixed
// prescale that halves the bf16 rounding error of those 16 values (largest
// relative error 1.6e-3 instead of 3.1e-3).  The inner sums are warp-level
// tensor-core MMAs (m16n8k16, bf16 in, fp32 out) fed from registers, with
// the tokens on the MMA's 16-row side (A) and 8 weight rows on its 8-column
// side (B), so the expanded weight never touches shared memory.
//
// Lookup: a 256-entry table of bf16 pairs, one entry per code byte (the two
// codes of two neighbouring elements), replicated for the 32 lanes at a
// 128-byte stride in shared memory (32 KB), so entry e of lane l sits at
// e * 128 + l * 4 and every lane reads its own bank: a shift and a LOP3 form
// the offset, one LDS returns the two bf16 values of a B operand register.
//
// K permutation: within each 64-element block, MMA k-index j of thread
// group position t (the fragment's k rows 2t, 2t+1, 2t+8, 2t+9 of chunk c)
// maps to the physical elements 16t + 4c + {0, 1, 2, 3}.  A sum over k does
// not depend on the order, as long as both operands use the same map; with
// it every thread reads 8 contiguous code bytes per weight row and 32
// contiguous bytes of X per token for a block.
//
// Work split: a unit is (224 weight rows, four consecutive 64-element
// blocks) for up to 16 tokens (128 rows where a fused projection's segment
// boundary would fall inside 224; 64 rows for up to 32 tokens), so that every
// row of the unit is one 128-byte line of codes; the LoRA up-projection adds
// units of four 64-wide adapter blocks after a row group's weight units.  A
// persistent grid of one CTA per SM takes contiguous shares of the unit list
// (stream-K), so every SM streams the same number of weight bytes.  The 14
// (or 8) MMA warps of a CTA split a unit into 7 (or 4) row slices x 2 block
// pairs, and a warp runs the MMA chains of its two blocks interleaved; the
// codes (one TMA box, 128-byte swizzle) and the four X blocks of each unit
// pass through a 4- (or 6-) stage ring filled by a loader warp (refilled as
// the MMA warps release a stage), and a second helper warp rewrites each
// landed X block into the MMA's operand order.  At the end of a row group the
// two warps of a slice add their accumulators in block order through shared
// memory; a group cut between CTAs is finished, per slice, by whichever
// contributing CTA arrives last (an integer counter with a launch epoch): it
// adds every contributor's fp32 partial in CTA order (deterministic) and
// writes Y.  Nothing waits on another CTA.
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

// Prescale L of the table per code book: for NF4 it halves the bf16 error of
// the 16 values; for FP4 (multiples of 1/12) 1.5 makes every value exact.
__device__ __forceinline__ float small_m_table_scale(int ct) { return ct ? 1.5f : 1.18881f; }

struct SmallMmaParams {
    CUtensorMap tmCodes;    // codes [N][K/2] bytes, box {128 B, UROWS rows}, 128-byte swizzle
    CUtensorMap tmX;        // X [M][K] bf16, box {64, 16 MT}, 128-byte swizzle
    CUtensorMap tmU;        // sU [M][rt] bf16, box {64, 16 MT}, 128-byte swizzle
    const uint8_t* q8;      // [N * K/64 >> bs_shift] (double quantization)
    const float* c1;
    const float* offset;
    const float* absmax;    // without double quantization
    int dq;
    const uint16_t* B;      // [N][r] bf16 (LoRA), unused when lora_ks == 0
    int M, N, KB;           // KB = K / 64
    int r, seg_rows, lora_ks;
    int KSU;                // units per row group: ceil(KB / 4) + ceil(lora_ks / 4)
    int64_t units;          // groups * KSU
    float inv_scale;        // 1 / L
    QFormat fmt;            // code book, 8-bit code book, block size
    uint16_t* Y;            // [M][N]
    float* part;            // [gridDim.x][2 slots][SLICES][SROWS rows][16 MT tokens] fp32 partials
    unsigned long long* counters;  // [groups * SLICES]: (epoch << 32) | arrivals
    int64_t part_cap, counter_cap;  // capacities: bounds checks of the debug build
    uint32_t epoch;         // nonzero
    uint64_t timeout_ns;
    int inject;             // test mode 1: issue no loads (the waits run out)
};

// Blocks of a unit per MMA warp (2; 1 doubles the MMA warps).
#ifndef QLORA_SMALLM_BPW
#define QLORA_SMALLM_BPW 2
#endif

// MT: token tiles of 16; SL: row slices of a unit (4, or QLORA_SMALLM_WIDE
// = 7 for MT = 1 where no fused projection's segment boundary falls inside a
// unit: 8 or 14 MMA warps, units of 128 or 224 rows).
#ifndef QLORA_SMALLM_WIDE
#define QLORA_SMALLM_WIDE 7
#endif
template <int MT, int SL = 4>
struct SmallMmaShape {
    static constexpr int BPW = QLORA_SMALLM_BPW;  // blocks of a unit per MMA warp
    static constexpr int SLICES = SL;             // row slices of a unit
    static constexpr int WARPS = SLICES * (4 / BPW);  // MMA warps: SLICES row slices x 4 / BPW block groups
    static constexpr int RT = MT == 1 ? 4 : 2;    // 8-row tiles per warp
    static constexpr int SROWS = 8 * RT;          // rows of a slice (32 or 16)
    static constexpr int UROWS = SLICES * SROWS;  // rows of a unit (128 or 224; 64 for MT = 2)
    static constexpr int THREADS = 32 * (WARPS + 2);  // + the warp that loads the ring, + the X reorderer
    static constexpr int XS = SL <= 4 ? 6 : SL <= 6 ? 5 : 4;  // ring stages
    static constexpr int X_TILE = 16 * MT * 128;  // 16 MT tokens x 64 bf16
    static constexpr int CODE_BYTES = UROWS * 128;  // codes of one unit (128-byte swizzle)
    static constexpr int STAGE = CODE_BYTES + 4 * X_TILE;
    // dynamic shared memory (1024-aligned): ring, t8 table, scale scratch,
    // accumulator exchange, barriers and stage counters
    static constexpr int OFF_T8 = XS * STAGE;
    static constexpr int OFF_SC = OFF_T8 + 1024;                     // [WARPS][2][BPW][SROWS] fp32
    static constexpr int XCH_FLOATS = RT * MT * 4 * 32;  // one warp's accumulators
    // [SLICES][warps per slice - 1][XCH_FLOATS] fp32: the slice's other warps
    // hand their accumulators to its first
    static constexpr int OFF_XCH = OFF_SC + WARPS * 2 * BPW * SROWS * 4;
    static constexpr int OFF_BAR = OFF_XCH + (WARPS - SLICES) * XCH_FLOATS * 4;  // full[XS], empty[XS], xready[XS]
    static constexpr int OFF_CNT = OFF_BAR + 24 * XS;               // issued[XS], abort flag
    static constexpr int SMEM = OFF_CNT + 4 * XS + 16 + 1024;       // + alignment slack
    static constexpr int PART_FLOATS = SROWS * 16 * MT;  // one slice's partial tile
    static constexpr int STATIC_SMEM = 256 * 32 * 4;     // the table (static shared memory)
};

// (not volatile: pure functions of their registers, so the compiler may
// interleave independent MMA chains)
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// d = A B (no accumulator input)
__device__ __forceinline__ void mma_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
    const float z = 0.0f;
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}


// The lookup table (static shared memory): entry e of lane l at e * 128 + l * 4.
__shared__ __align__(128) uint32_t g_small_m_lut[256 * 32];

// Table entry of byte k (0..3) of word w for this lane (lane4 = lane * 4).
// The table does not change after the kernel's first barrier, so the load is
// not volatile (its address depends on code words read after the stage's
// barrier wait).
__device__ __forceinline__ uint32_t lut_byte(uint32_t w, int k, uint32_t lane4) {
    const uint32_t off = (((w >> (8 * k)) << 7) & 0x7F80u) | lane4;
    return *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(g_small_m_lut) + off);
}
__device__ __forceinline__ uint2 ld_shared_v2(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

// Index of the CTA whose share [I c / G, I (c + 1) / G) holds unit x.
__device__ __forceinline__ int owner_cta(int64_t x, int64_t I, int G) {
    int c = (int)((x * G) / I);
    while (c + 1 < G && (I * (c + 1)) / G <= x) ++c;
    while (c > 0 && (I * c) / G > x) --c;
    return c;
}

__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int MT, int SL>
__global__ void __launch_bounds__(SmallMmaShape<MT, SL>::THREADS, 1)
    k_smallm_mma(const __grid_constant__ SmallMmaParams p) {
    using S = SmallMmaShape<MT, SL>;
    constexpr int RT = S::RT, XS = S::XS, SROWS = S::SROWS, UROWS = S::UROWS, WARPS = S::WARPS;
    constexpr int TOK = 16 * MT;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* gb = smem_raw + (base - raw_base);
    float* t8s = reinterpret_cast<float*>(gb + S::OFF_T8);
    float* xch = reinterpret_cast<float*>(gb + S::OFF_XCH);
    const uint32_t bar = base + S::OFF_BAR;
    auto full = [&](int s) { return bar + 8u * s; };
    auto empty = [&](int s) { return bar + 8u * (XS + s); };
    auto xready = [&](int s) { return bar + 8u * (2 * XS + s); };
    int* issued = reinterpret_cast<int*>(gb + S::OFF_CNT);  // loads issued into the stage
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + S::OFF_CNT + 4 * XS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    constexpr int BPW = S::BPW, WPS = 4 / BPW;   // blocks per warp, warps per slice
    const int slice = warp / WPS, bpair = warp % WPS;  // row slice; blocks BPW bpair .. + BPW - 1 of a unit
    const WaitCfg wc{p.timeout_ns};

    // table: entry e = {L v[e >> 4] (bits 0..15), L v[e & 15] (bits 16..31)}
    {
        const float L = small_m_table_scale(p.fmt.code_type);
        for (int idx = threadIdx.x; idx < 256 * 32; idx += blockDim.x) {
            const int e = idx >> 5;
            const float vlo = __fmul_rn(code_value(p.fmt.code_type, e >> 4), L);
            const float vhi = __fmul_rn(code_value(p.fmt.code_type, e & 15), L);
            g_small_m_lut[idx] = pack_bf16x2(vlo, vhi);
        }
    }
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        t8s[i] = dq_value(p.fmt.dq_type, (p.fmt.dq_type == 0 || i < 253) ? i : 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < XS; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), WARPS);
            mbar_init(xready(s), 1);
            issued[s] = 0;
        }
        *abort_flag = 0;
        fence_mbar_init();
        pdl_trigger();
        prefetch_tensormap(&p.tmCodes);
        prefetch_tensormap(&p.tmX);
        if (p.lora_ks) prefetch_tensormap(&p.tmU);
    }
    __syncthreads();
    // Dependent launch.  With an adapter the kernel before this one is the
    // sU GEMM, which waited for its own predecessors before it let this
    // kernel start: the codes, block constants and X are final, and only sU
    // (read by the adapter units' loads) needs the wait, taken by the thread
    // that issues those loads.  Without one the kernel before may still be
    // writing any input (the quantizer, say): every thread waits here.
    if (p.lora_ks == 0) pdl_wait();

    const int QW = (p.KB + 3) >> 2;        // weight units per row group
    const int64_t U = p.units;
    const int G = gridDim.x;
    const int64_t u0 = (U * blockIdx.x) / G, u1 = (U * (blockIdx.x + 1)) / G;
    const int n_units = (int)(u1 - u0);
    const int g_first = (int)(u0 / p.KSU), q_first = (int)(u0 - (int64_t)g_first * p.KSU);

    // loads of the CTA's unit i (row group g, unit q of the group) into stage i % XS
    auto issue = [&](int i, int g, int q) {
        const int s = i % XS;
        const uint32_t st = base + (uint32_t)(s * S::STAGE);
        if (p.inject) return;
        issued[s] += 1;
        if (q < QW) {
            const int nb = min(4, p.KB - 4 * q);
            mbar_arrive_expect_tx(full(s), (uint32_t)(S::CODE_BYTES + nb * S::X_TILE));
            tma_load_2d(st, &p.tmCodes, full(s), q * 128, g * UROWS);
            for (int c = 0; c < nb; ++c)
                tma_load_2d(st + (uint32_t)(S::CODE_BYTES + c * S::X_TILE), &p.tmX, full(s), (4 * q + c) * 64, 0);
        } else {
            pdl_wait();  // sU comes from the kernel before this one
            const int ql = q - QW;
            const int nb = min(4, p.lora_ks - 4 * ql);
            const int ucol = p.seg_rows ? ((g * UROWS) / p.seg_rows) * p.r : 0;
            mbar_arrive_expect_tx(full(s), (uint32_t)(nb * S::X_TILE));
            for (int c = 0; c < nb; ++c)
                tma_load_2d(st + (uint32_t)(S::CODE_BYTES + c * S::X_TILE), &p.tmU, full(s),
                            (4 * ql + c) * 64 + ucol, 0);
        }
    };
    if (warp == WARPS) {
        // ------------------------------------------------------------ ring loader
        if (lane == 0) {
            int g = g_first, q = q_first;
            for (int i = 0; i < n_units; ++i) {
                // the MMA warps have released the stage's previous unit
                if (i >= XS && (*abort_flag || !mbar_wait_hint(empty(i % XS), ((i / XS) - 1) & 1, wc, 2000))) {
                    *abort_flag = 1;
                    break;
                }
                // the reorderer's generic writes to the stage precede the TMA's
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                issue(i, g, q);
                if (++q == p.KSU) { q = 0; ++g; }
            }
        }
    } else if (warp == WARPS + 1) {
        // ------------------------------------------------------------ X reorderer
        // Rewrites each X (or sU) block of a landed unit in place, from the
        // TMA's 128-byte-swizzled rows into the MMA warps' operand order: the
        // 16-byte quad of lane (g, t) for chunk c and token tile mt holds
        // rows g and g + 8 (of tile mt) at the words 8 t + 2 c and 8 t + 2 c + 1,
        // i.e. the four A registers of that lane's m16n8k16 fragment, at
        // (((c * MT + mt) * 8 + g) * 4 + t) * 16.
        int g = g_first, q = q_first;
        for (int i = 0; i < n_units; ++i) {
            const int s = i % XS;
            if (*abort_flag || !mbar_wait_hint(full(s), (i / XS) & 1, wc, 1000)) {
                *abort_flag = 1;
                break;
            }
            const int nb = q < QW ? min(4, p.KB - 4 * q) : min(4, p.lora_ks - 4 * (q - QW));
            for (int b = 0; b < nb; ++b) {
                const uint32_t xs = base + (uint32_t)(s * S::STAGE + S::CODE_BYTES + b * S::X_TILE);
                uint2 w[MT][4][2];  // [mt][c][row g, row g + 8] = words 8 t + 2 c, + 1
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int r = 16 * mt + gid + 8 * h;
                            const uint32_t chunk = (uint32_t)((2 * tig + (c >> 1)) ^ (r & 7));
                            w[mt][c][h] = ld_shared_v2(xs + (uint32_t)r * 128u + (chunk << 4) + (uint32_t)(c & 1) * 8u);
                        }
                __syncwarp();
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        st_shared_v4(xs + (uint32_t)((((c * MT + mt) * 8 + gid) * 4 + tig) * 16), w[mt][c][0].x,
                                     w[mt][c][1].x, w[mt][c][0].y, w[mt][c][1].y);
                __syncwarp();
            }
            if (lane == 0) mbar_arrive(xready(s));
            if (++q == p.KSU) { q = 0; ++g; }
        }
    } else {

    const uint32_t lane4 = (uint32_t)lane * 4u;
    float* scr = reinterpret_cast<float*>(gb + S::OFF_SC) + warp * 2 * BPW * SROWS;  // [2][BPW][SROWS]
    const float off = p.dq ? __ldg(p.offset) : 0.0f;

    // raw block constants of row `lane` of the warp's slice (lanes < SROWS)
    // for its blocks of unit (g, q), loaded two units ahead of their use
    struct Pf {
        int q[BPW];    // 8-bit code (double quantization) or 0; -1: a' = 0
        float c[BPW];  // c1 or absmax
    };
    auto fetch = [&](int g, int q, bool valid) {
        Pf f;
#pragma unroll
        for (int bb = 0; bb < BPW; ++bb) {
            f.q[bb] = -1;
            f.c[bb] = 0.0f;
            const int kb = 4 * q + BPW * bpair + bb;
            if (!valid || q >= QW || kb >= p.KB || lane >= SROWS) continue;
            const int n = g * UROWS + slice * SROWS + lane;
            if (n < p.N) {
                const int64_t b = ((int64_t)n * p.KB + kb) >> p.fmt.bs_shift;
                if (p.dq) {
                    f.q[bb] = __ldg(p.q8 + b);
                    f.c[bb] = __ldg(p.c1 + (b >> 8));
                } else {
                    f.q[bb] = 0;
                    f.c[bb] = __ldg(p.absmax + b);
                }
            }
        }
        return f;
    };

    float acc[RT][MT][4];
#pragma unroll
    for (int j = 0; j < RT; ++j)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][mt][e] = 0.0f;
    bool dead = false;

    // end of this CTA's segment of row group g (its last unit u).  Every warp
    // comes here, also after a wait ran out, so that the slice's named
    // barriers are always met.  The block warps of the slice add their
    // accumulators in block order; the slice's first warp then writes Y, or
    // publishes the partial and lets the last contributor finish the rows.
    auto finish_group = [&](int g, int64_t u) {
        float* mx = xch + (int64_t)(slice * (WPS - 1) + bpair - 1) * S::XCH_FLOATS;
        if (bpair != 0) {
#pragma unroll
            for (int j = 0; j < RT; ++j)
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) mx[((j * MT + mt) * 4 + e) * 32 + lane] = acc[j][mt][e];
        }
        named_sync(1 + slice, 32 * WPS);
        if (bpair == 0) {
#pragma unroll
            for (int w = 1; w < WPS; ++w) {
                const float* ox = xch + (int64_t)(slice * (WPS - 1) + w - 1) * S::XCH_FLOATS;
#pragma unroll
                for (int j = 0; j < RT; ++j)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            acc[j][mt][e] = __fadd_rn(acc[j][mt][e], ox[((j * MT + mt) * 4 + e) * 32 + lane]);
            }
        }
        named_sync(1 + slice, 32 * WPS);  // the exchange buffers are free again
        if (bpair == 0 && !*abort_flag) {
            const int64_t gstart = (int64_t)g * p.KSU;
            const bool whole = u0 <= gstart && u == gstart + p.KSU - 1;
            const int nsl = g * UROWS + slice * SROWS;
            bool write_y = whole;
            if (!whole) {
                const int slot = u0 >= gstart ? 0 : 1;  // the CTA's first segment uses slot 0
                float* mine = p.part + (((int64_t)blockIdx.x * 2 + slot) * S::SLICES + slice) * S::PART_FLOATS;
#pragma unroll
                for (int j = 0; j < RT; ++j)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (QLORA_CHECK((mine - p.part) + (8 * j + 2 * tig + (e & 1)) * TOK + 16 * mt + gid +
                                                8 * (e >> 1) < p.part_cap))
                                __stcg(mine + (8 * j + 2 * tig + (e & 1)) * TOK + 16 * mt + gid + 8 * (e >> 1),
                                       acc[j][mt][e]);
                __threadfence();
                __syncwarp();
                // contributors: the CTAs from the one holding the group's first
                // unit to the one holding its last, less any with an empty share
                const int cf = owner_cta(gstart, U, G), cl = owner_cta(gstart + p.KSU - 1, U, G);
                uint32_t ncontrib = 0;
                for (int c = cf; c <= cl; ++c) ncontrib += ((U * c) / G < (U * (c + 1)) / G) ? 1u : 0u;
                uint32_t before = 0;
                if (lane == 0 && QLORA_CHECK((int64_t)g * S::SLICES + slice < p.counter_cap)) {
                    // arrivals of this launch (epoch in the high word; a value of
                    // another epoch counts as none)
                    unsigned long long* ctr = p.counters + (int64_t)g * S::SLICES + slice;
                    unsigned long long cv = *reinterpret_cast<volatile unsigned long long*>(ctr);
                    const unsigned long long ep = (unsigned long long)p.epoch << 32;
                    while (true) {
                        const bool same = (cv & 0xFFFFFFFF00000000ull) == ep;
                        const unsigned long long want = same ? cv + 1ull : (ep | 1ull);
                        const unsigned long long prev = atomicCAS(ctr, cv, want);
                        if (prev == cv) {
                            before = same ? (uint32_t)(cv & 0xFFFFFFFFull) : 0u;
                            break;
                        }
                        cv = prev;
                    }
                    if (before + 1 == ncontrib) *ctr = 0ull;  // last arrival: reset for the next launch
                }
                before = __shfl_sync(0xffffffffu, before, 0);
                if (before + 1 == ncontrib) {
                    __threadfence();
#pragma unroll
                    for (int j = 0; j < RT; ++j)
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) acc[j][mt][e] = 0.0f;
                    for (int c = cf; c <= cl; ++c) {
                        if ((U * c) / G == (U * (c + 1)) / G) continue;
                        const int cslot = (U * c) / G >= gstart ? 0 : 1;
                        const float* src = p.part + (((int64_t)c * 2 + cslot) * S::SLICES + slice) * S::PART_FLOATS;
#pragma unroll
                        for (int j = 0; j < RT; ++j)
#pragma unroll
                            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    acc[j][mt][e] = __fadd_rn(
                                        acc[j][mt][e],
                                        __ldcg(src + (8 * j + 2 * tig + (e & 1)) * TOK + 16 * mt + gid + 8 * (e >> 1)));
                    }
                    write_y = true;
                }
            }
            if (write_y) {
#pragma unroll
                for (int j = 0; j < RT; ++j) {
                    const int n = nsl + 8 * j + 2 * tig;
                    if (n >= p.N) continue;
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int m = 16 * mt + gid + 8 * h;
                            if (m >= p.M) continue;
                            const uint32_t v = pack_bf16x2(acc[j][mt][2 * h], acc[j][mt][2 * h + 1]);
                            uint16_t* dst = p.Y + (int64_t)m * p.N + n;
                            if (!QLORA_CHECK(m < p.M && n < p.N)) continue;
                            if (n + 1 < p.N && ((reinterpret_cast<uintptr_t>(dst) & 3u) == 0)) {
                                *reinterpret_cast<uint32_t*>(dst) = v;
                            } else {
                                dst[0] = (uint16_t)(v & 0xFFFFu);
                                if (n + 1 < p.N) dst[1] = (uint16_t)(v >> 16);
                            }
                        }
                }
            }
        }
#pragma unroll
        for (int j = 0; j < RT; ++j)
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[j][mt][e] = 0.0f;
    };

    // block constants two units ahead: (g, q) is unit i, (g1, q1) unit i + 1
    int g = g_first, q = q_first;
    int g1 = g, q1 = q + 1;
    if (q1 == p.KSU) { q1 = 0; ++g1; }
    Pf cur = fetch(g, q, n_units > 0), nxt = fetch(g1, q1, n_units > 1);
    for (int i = 0; i < n_units; ++i) {
        const int s = i % XS;
        const int64_t u = u0 + i;
        const int nsl = g * UROWS + slice * SROWS;  // first row of this warp's slice
        if (!dead && !mbar_wait_hint(xready(s), (i / XS) & 1, wc, 1000)) {
            *abort_flag = 1;
            dead = true;
        }
        const bool wunit = q < QW;
        const uint32_t st = base + (uint32_t)(s * S::STAGE);
        // a warp whose rows all lie past the weight skips the unit
        if (!dead && nsl < p.N && wunit) {
            // ------------------------------------------------------ weight blocks
            // Both blocks of the warp in one pass, so that their MMA chains
            // (RT x BPW independent ones) interleave.  X (reordered by the X
            // warp: the quad of chunk c and token tile mt is the A operand
            // as it is) of a block past K reads as zeros; its codes are the
            // TMA's zero fill and its block constant is 0.
            uint4 xq[BPW][MT][4];
#pragma unroll
            for (int bb = 0; bb < BPW; ++bb) {
                const int bq = BPW * bpair + bb;
                const uint32_t xs = st + (uint32_t)(S::CODE_BYTES + bq * S::X_TILE);
                const bool bv = 4 * q + bq < p.KB;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        xq[bb][mt][c] = bv ? ld_shared_v4(xs + (uint32_t)((((c * MT + mt) * 8 + gid) * 4 + tig) * 16))
                                           : make_uint4(0u, 0u, 0u, 0u);
            }
            float* sc = scr + (i & 1) * BPW * SROWS;  // [BPW][SROWS]
            if (lane < SROWS) {
#pragma unroll
                for (int bb = 0; bb < BPW; ++bb) {
                    float a = 0.0f;
                    if (cur.q[bb] >= 0) a = p.dq ? __fadd_rn(__fmul_rn(t8s[cur.q[bb]], cur.c[bb]), off) : cur.c[bb];
                    sc[bb * SROWS + lane] = __fmul_rn(a, p.inv_scale);
                }
            }
            __syncwarp();
            // codes of unit row r = slice * SROWS + 8 j + gid: bytes
            // 32 bq + 8 tig .. + 7 of its 128-byte line (128-byte swizzle)
            uint32_t cw[BPW][RT][2];
#pragma unroll
            for (int bb = 0; bb < BPW; ++bb)
#pragma unroll
                for (int j = 0; j < RT; ++j) {
                    const int bq = BPW * bpair + bb;
                    const int r = slice * SROWS + 8 * j + gid;
                    const uint32_t chunk = (uint32_t)((2 * bq + (tig >> 1)) ^ (r & 7));
                    const uint2 v = ld_shared_v2(st + (uint32_t)r * 128u + (chunk << 4) + (uint32_t)(tig & 1) * 8u);
                    cw[bb][j][0] = v.x;
                    cw[bb][j][1] = v.y;
                }
            // chunk by chunk over both blocks and all row tiles
            float d[BPW][RT][MT][4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int bb = 0; bb < BPW; ++bb) {
                    uint32_t b0[RT], b1[RT];
#pragma unroll
                    for (int j = 0; j < RT; ++j) {
                        b0[j] = lut_byte(cw[bb][j][c >> 1], 2 * (c & 1), lane4);
                        b1[j] = lut_byte(cw[bb][j][c >> 1], 2 * (c & 1) + 1, lane4);
                    }
#pragma unroll
                    for (int j = 0; j < RT; ++j)
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const uint4 x = xq[bb][mt][c];
                            if (c == 0)
                                mma_16816_z(d[bb][j][mt], x.x, x.y, x.z, x.w, b0[j], b1[j]);
                            else
                                mma_16816(d[bb][j][mt], x.x, x.y, x.z, x.w, b0[j], b1[j]);
                        }
                }
            }
#pragma unroll
            for (int bb = 0; bb < BPW; ++bb)
#pragma unroll
                for (int j = 0; j < RT; ++j) {
                    const float2 sj = *reinterpret_cast<const float2*>(sc + bb * SROWS + 8 * j + 2 * tig);
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        acc[j][mt][0] = __fmaf_rn(sj.x, d[bb][j][mt][0], acc[j][mt][0]);
                        acc[j][mt][1] = __fmaf_rn(sj.y, d[bb][j][mt][1], acc[j][mt][1]);
                        acc[j][mt][2] = __fmaf_rn(sj.x, d[bb][j][mt][2], acc[j][mt][2]);
                        acc[j][mt][3] = __fmaf_rn(sj.y, d[bb][j][mt][3], acc[j][mt][3]);
                    }
                }
            // the adapter rows of the group into L2 a few units before their use
            if (p.lora_ks && q == max(QW - 2, 0) && bpair == 0 && lane < SROWS) {
                const int n = nsl + lane;
                if (n < p.N)
                    for (int c = 0; c < p.r * 2; c += 128)
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(
                            reinterpret_cast<const uint8_t*>(p.B + (int64_t)n * p.r) + c));
            }
        }
#pragma unroll
        for (int bb = 0; bb < BPW; ++bb) {
        const int bq = BPW * bpair + bb;
        const int jb = 4 * (q - QW) + bq;  // this warp's adapter block
        // a warp whose rows all lie past the weight, or whose block lies past
        // r, skips the block
        if (!dead && nsl < p.N && !wunit && jb < p.lora_ks) {
            const uint32_t xs = st + (uint32_t)(S::CODE_BYTES + bq * S::X_TILE);
            // sU fragments, reordered by the X warp
            uint4 xq[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    xq[mt][c] = ld_shared_v4(xs + (uint32_t)((((c * MT + mt) * 8 + gid) * 4 + tig) * 16));
            {
                // -------------------------------------------------- adapter block: B rows x sU
                const int j0 = jb * 64 + 16 * tig;  // adapter column of this lane's 16
                const bool v0 = j0 + 8 <= p.r, v1 = j0 + 16 <= p.r;
                uint4 bw[RT][2];
#pragma unroll
                for (int j = 0; j < RT; ++j) {
                    const int n = nsl + 8 * j + gid;
                    bw[j][0] = make_uint4(0, 0, 0, 0);
                    bw[j][1] = make_uint4(0, 0, 0, 0);
                    if (n < p.N) {
                        const uint4* src = reinterpret_cast<const uint4*>(p.B + (int64_t)n * p.r + j0);
                        if (v0) bw[j][0] = __ldg(src);
                        if (v1) bw[j][1] = __ldg(src + 1);
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < RT; ++j) {
                        const uint4 h = bw[j][c >> 1];
                        const uint32_t w0 = (c & 1) ? h.z : h.x, w1 = (c & 1) ? h.w : h.y;
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
                            mma_16816(acc[j][mt], xq[mt][c].x, xq[mt][c].y, xq[mt][c].z, xq[mt][c].w, w0, w1);
                    }
            }
        }
        }
        if (!dead) {
            // release the stage to the loader (an arrival with release semantics,
            // after every lane's reads of it)
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(s));
        }
        // unit i + 2's block constants, issued after the release so that the
        // arrival does not wait for them
        int g2 = g1, q2 = q1 + 1;
        if (q2 == p.KSU) { q2 = 0; ++g2; }
        const Pf nxt2 = fetch(g2, q2, i + 2 < n_units);
        if (q == p.KSU - 1 || i == n_units - 1) finish_group(g, u);
        cur = nxt;
        nxt = nxt2;
        g = g1;
        q = q1;
        g1 = g2;
        q1 = q2;
    }
    }
    // every load issued into the ring has landed before the CTA exits, and
    // the kernel does not complete before the one it depends on
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int s = 0; s < XS; ++s)
            if (issued[s] > 0) mbar_wait(full(s), (issued[s] - 1) & 1, wc);
        pdl_wait();
    }
}

}  // namespace qlora
