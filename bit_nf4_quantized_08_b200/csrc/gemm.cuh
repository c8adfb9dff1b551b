// gemm.cuh -- warp-specialized tcgen05 GEMM for sm_100a with an optional
// NF4 dequantizing producer.
//
// Computes D[i][j] = sum_k Aop[i][k] * Bop[j][k] for one 128 x BN tile per
// CTA, accumulating in TMEM (fp32), k in steps of 64 (one NF4 block column).
//   warp 0           TMA / bulk-copy producer (one elected lane)
//   warp 1           TMEM allocation + tcgen05.mma issue (one elected lane)
//   warps 2..        dequant producers (expand NF4 codes into the swizzled
//                    bf16 operand tile in shared memory), then the epilogue
//                    (tcgen05.ld -> bf16/fp32 -> global)
// Operand tiles use the 128-byte swizzle.  A K-major tile of R rows keeps
// row r at byte r*128 (8-row groups 1024 B apart).  An MN-major tile keeps
// 64-element MN chunks 8192 B apart and k-row j at byte j*128 inside a chunk.
//
// Dequant modes (the frozen weight W [N, K] is never written to HBM):
//   DQ_B_K   B operand = W' rows (forward: Y = X W'^T), R = BN rows
//   DQ_B_MN  B operand = W' viewed [k_out][n] (backward: dX = dY W'), the
//            reduction runs over W rows, 64 per step, 256 output columns
//   DQ_A_K   A operand = W' rows (swap-AB small-M forward: Y^T = W' X^T)
// LoRA steps (digest sec. 4 / reproduction blog forward): extra k-steps whose
// operands both come from TMA (e.g. [X | sU] . [W' | B]^T).
#pragma once

#include "common.cuh"
#include "internal.h"
#include "nf4.cuh"

namespace qlora {

enum { DQ_NONE = 0, DQ_B_K = 1, DQ_B_MN = 2, DQ_A_K = 3 };
enum { EPI_BF16 = 0, EPI_BF16_T = 1, EPI_F32 = 2, EPI_F32_T = 3 };

struct GemmParams {
    CUtensorMap tmA, tmB;    // main k-steps (unused for the dequantized operand)
    CUtensorMap tmA2, tmB2;  // LoRA k-steps
    CUtensorMap tmCodes;     // packed NF4 codes viewed [W rows][K/2 bytes]
    CUtensorMap tmOut;       // bf16 output [rows][cols], 64 x 128 boxes, 128B swizzle (EPI_BF16)
    const float* scales;     // block constants a' laid out [kb][scales_ld]
    int64_t scales_ld;
    int dq_rows;             // valid W rows (the rest of a dequant tile is 0)
    int dq_kbs;              // valid block columns K/64
    int ks_main, ks_lora;    // number of k-steps of each kind
    int ks_per_split;        // main k-steps per blockIdx.z
    int rows, cols;          // valid extent of D
    void* out;
    int64_t out_ld;          // elements
    int64_t out_split_stride;  // elements between split-K partial planes
    uint64_t timeout_ns;
    int inject;
    // stream-K schedule (persistent grid of gridDim.x CTAs)
    int streamk;
    int tiles_n, tiles_total;
    int n_in_x;              // pair grid schedule: weight column tiles in blockIdx.x / 2 (only when
                             // there are more than 65535 of them; else token tiles in x, columns in y)
    float* sk_part;   // [gridDim.x][BM*BN] fp32 partial tiles
    int* sk_flags;    // [gridDim.x], zero before the launch
    // CTA-pair kernel: wait for the previous kernel of the stream only before
    // the first LoRA k-step (that kernel has itself waited for the block
    // constants before it let this one launch); 0: before any load
    int late_wait;
    // adapters of a fused projection (one weight, nseg row segments of
    // lora_seg_rows rows, each with its own rank-lora_seg_r adapter): the
    // LoRA k-steps of an output tile read the sU columns of the tile's
    // segment, starting at (n0 / lora_seg_rows) * lora_seg_r; 0 = one adapter
    int lora_seg_rows, lora_seg_r;
    int code_type;  // 4-bit code book of the weight (0 NF4, 1 FP4)
};

// First sU column of the adapter of the output rows starting at n0.
__device__ __forceinline__ int lora_col0(const GemmParams& p, int n0) {
    return p.lora_seg_rows ? (n0 / p.lora_seg_rows) * p.lora_seg_r : 0;
}

// MT = number of 128-row MMA sub-tiles on the A side (1 or 2).  With MT = 2
// one dequantized B tile feeds two accumulators (256 A rows per CTA), which
// halves the dequant work per MMA flop.
template <int BN, int A_MN, int B_MN, int DQ, int MT>
struct GemmShape {
    static constexpr int BM = 128 * MT;
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int DQ_ROWS = DQ == DQ_B_K ? BN : (DQ == DQ_A_K ? 128 : (DQ == DQ_B_MN ? 256 : 0));
    static constexpr int NDQ_WARPS = DQ_ROWS / 32;
    static constexpr int CODE_BYTES = DQ == DQ_B_MN ? 64 * 128 : DQ_ROWS * 32;
    static constexpr int SCALE_BYTES = DQ == DQ_NONE ? 0 : (DQ == DQ_B_MN ? 4 * 64 * 4 : DQ_ROWS * 4);
    static constexpr int STAGE_RAW = A_BYTES + B_BYTES + CODE_BYTES + SCALE_BYTES;
    static constexpr int STAGE_BYTES = (STAGE_RAW + 1023) / 1024 * 1024;
    static constexpr int NE_WARPS = NDQ_WARPS > 4 ? NDQ_WARPS : 4;
    static constexpr int THREADS = 32 * (2 + NE_WARPS);
    static constexpr int ACC_COLS = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
    static constexpr int TMEM_COLS = ACC_COLS * MT;
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
    static_assert(MT == 1 || MT == 2, "MT");
    static_assert(DQ != DQ_A_K || MT == 1, "a dequantized A operand is one 128-row tile");
};

template <int BN, int A_MN, int B_MN, int DQ, int STAGES, int MT>
constexpr int gemm_smem_bytes() {
    return GemmShape<BN, A_MN, B_MN, DQ, MT>::STAGE_BYTES * STAGES + 1024 /*align*/ + 256 /*barriers*/;
    // barriers: 3*STAGES + 2 mbarriers, the TMEM address and the abort flag
}

// Physical offset of a logical byte offset inside a TMA tile written with the
// 32-byte swizzle (16-byte chunk index bit 0 XOR address bit 7).
__device__ __forceinline__ uint32_t sw32(uint32_t off) { return off ^ ((off >> 3) & 0x10u); }

__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// One unit of work: output tile (tm, tn) over the k-step range [k0, k1) of
// that tile.  Steps [0, ks_main) are main steps, [ks_main, ks_main+ks_lora)
// are LoRA steps.
struct Seg {
    int tm, tn, k0, k1;
    int split;   // grid split index (grid schedule)
};

// Work schedule of one CTA.  Grid schedule: one segment, the tile and split
// of blockIdx.  Stream-K schedule (p.streamk): the CTA owns the contiguous
// share [c*I/G, (c+1)*I/G) of all I = tiles * KS (tile, k-step) iterations,
// G = gridDim.x, tiles ordered with tn fastest.
struct Schedule {
    int64_t pos, end;
    int KS, tiles_n;
    bool grid_done;
    __device__ Schedule(const GemmParams& p) {
        KS = p.ks_main + p.ks_lora;
        tiles_n = p.tiles_n;
        grid_done = false;
        if (p.streamk) {
            const int64_t I = (int64_t)p.tiles_total * KS;
            pos = I * blockIdx.x / gridDim.x;
            end = I * (blockIdx.x + 1) / gridDim.x;
        } else {
            pos = end = 0;
        }
    }
    __device__ bool next(const GemmParams& p, Seg& sg) {
        if (!p.streamk) {
            if (grid_done) return false;
            grid_done = true;
            sg.tn = blockIdx.x;
            sg.tm = blockIdx.y;
            sg.split = blockIdx.z;
            sg.k0 = blockIdx.z * p.ks_per_split;
            const bool last = blockIdx.z == gridDim.z - 1;
            sg.k1 = last ? KS : min(p.ks_main, sg.k0 + p.ks_per_split);
            return sg.k1 > sg.k0 || last;
        }
        if (pos >= end) return false;
        const int t = (int)(pos / KS);
        sg.tm = t / tiles_n;
        sg.tn = t % tiles_n;
        sg.k0 = (int)(pos - (int64_t)t * KS);
        const int64_t room = end - pos;
        sg.k1 = (int)min((int64_t)KS, (int64_t)sg.k0 + room);
        sg.split = 0;
        pos += sg.k1 - sg.k0;
        return true;
    }
};

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int BN, int A_MN, int B_MN, int DQ, int EPI, int STAGES, int MT>
__global__ void __launch_bounds__(GemmShape<BN, A_MN, B_MN, DQ, MT>::THREADS, 1)
    k_gemm(const __grid_constant__ GemmParams p) {
    using S = GemmShape<BN, A_MN, B_MN, DQ, MT>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw_base);
    const uint32_t bar_base = base + S::STAGE_BYTES * STAGES;
    // barriers at bar_base + 8*i: full_tma[STAGES], full_dq[STAGES], empty[STAGES], acc_full, acc_empty
    auto full_tma = [&](int s) { return bar_base + 8u * s; };
    auto full_dq = [&](int s) { return bar_base + 8u * (STAGES + s); };
    auto empty = [&](int s) { return bar_base + 8u * (2 * STAGES + s); };
    const uint32_t acc_full = bar_base + 8u * (3 * STAGES);
    const uint32_t acc_empty = bar_base + 8u * (3 * STAGES + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + S::STAGE_BYTES * STAGES + 8 * (3 * STAGES + 2));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WaitCfg wc{p.timeout_ns};
    const int KS = p.ks_main + p.ks_lora;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_tma(s), 1);
            mbar_init(full_dq(s), S::NDQ_WARPS > 0 ? S::NDQ_WARPS : 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, S::NE_WARPS);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&p.tmA);
        prefetch_tensormap(&p.tmB);
        if (p.ks_lora) {
            prefetch_tensormap(&p.tmA2);
            prefetch_tensormap(&p.tmB2);
        }
        if (DQ != DQ_NONE) prefetch_tensormap(&p.tmCodes);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), S::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && !p.inject) {
            int last_use[STAGES];
            for (int s = 0; s < STAGES; ++s) last_use[s] = -1;
            bool ok = true;
            int it = 0;
            Schedule sch(p);
            Seg sg;
            while (ok && sch.next(p, sg)) {
                const int m0 = sg.tm * S::BM, n0 = sg.tn * BN;
                for (int k = sg.k0; k < sg.k1; ++k, ++it) {
                    const int s = it % STAGES, u = it / STAGES;
                    if (!mbar_wait(empty(s), (u & 1) ^ 1, wc)) { ok = false; *abort_flag = 1; break; }
                    const uint32_t sA = base + s * S::STAGE_BYTES;
                    const uint32_t sB = sA + S::A_BYTES;
                    const uint32_t sC = sB + S::B_BYTES;
                    const uint32_t sS = sC + S::CODE_BYTES;
                    const bool lora = k >= p.ks_main;
                    const int kc = lora ? (k - p.ks_main) : k;
                    uint32_t bytes = 0;
                    if (!lora) {
                        if (DQ != DQ_A_K) bytes += S::A_BYTES;
                        if (DQ != DQ_B_K && DQ != DQ_B_MN) bytes += S::B_BYTES;
                        if (DQ != DQ_NONE) bytes += S::CODE_BYTES;
                        if (DQ == DQ_B_K || DQ == DQ_A_K) bytes += S::DQ_ROWS * 4;
                        if (DQ == DQ_B_MN) {
                            for (int c = 0; c < 4; ++c)
                                if (n0 / 64 + c < p.dq_kbs) bytes += 256;
                        }
                    } else {
                        bytes = (DQ == DQ_A_K ? 16384 : S::A_BYTES) + S::B_BYTES;
                    }
                    mbar_arrive_expect_tx(full_tma(s), bytes);
                    const CUtensorMap* mA = lora ? &p.tmA2 : &p.tmA;
                    const CUtensorMap* mB = lora ? &p.tmB2 : &p.tmB;
                    if (lora || DQ != DQ_A_K) {
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            if (A_MN) {
                                tma_load_2d(sA + mt * 16384, mA, full_tma(s), m0 + 128 * mt, kc * 64);
                                tma_load_2d(sA + mt * 16384 + 8192, mA, full_tma(s), m0 + 128 * mt + 64, kc * 64);
                            } else {
                                tma_load_2d(sA + mt * 16384, mA, full_tma(s), kc * 64 + (lora ? lora_col0(p, n0) : 0),
                                            m0 + 128 * mt);
                            }
                        }
                    }
                    if (lora || (DQ != DQ_B_K && DQ != DQ_B_MN)) {
                        if (B_MN) {
                            for (int c = 0; c < BN / 64; ++c)
                                tma_load_2d(sB + 8192 * c, mB, full_tma(s), n0 + 64 * c, kc * 64);
                        } else {
                            tma_load_2d(sB, mB, full_tma(s), kc * 64, n0);
                        }
                    }
                    if (!lora && DQ != DQ_NONE) {
                        if (DQ == DQ_B_MN) {
                            tma_load_2d(sC, &p.tmCodes, full_tma(s), n0 / 2, kc * 64);
                            for (int c = 0; c < 4; ++c)
                                if (n0 / 64 + c < p.dq_kbs)
                                    bulk_load(sS + 256 * c,
                                              p.scales + (int64_t)(n0 / 64 + c) * p.scales_ld + kc * 64,
                                              256, full_tma(s));
                        } else {
                            const int w0 = DQ == DQ_B_K ? n0 : m0;
                            tma_load_2d(sC, &p.tmCodes, full_tma(s), kc * 32, w0);
                            bulk_load(sS, p.scales + (int64_t)kc * p.scales_ld + w0, S::DQ_ROWS * 4,
                                      full_tma(s));
                        }
                    }
                    last_use[s] = u;
                }
            }
            // drain: every issued copy has landed before the CTA may exit
            for (int s = 0; s < STAGES; ++s)
                if (last_use[s] >= 0) mbar_wait(full_tma(s), last_use[s] & 1, wc);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, BN, A_MN, B_MN);
            bool ok = true;
            int it = 0, seg_i = 0;
            Schedule sch(p);
            Seg sg;
            while (ok && sch.next(p, sg)) {
                if (seg_i > 0 && !mbar_wait(acc_empty, (seg_i - 1) & 1, wc)) { ok = false; *abort_flag = 1; break; }
                tc_fence_after();
                for (int k = sg.k0; k < sg.k1; ++k, ++it) {
                    const int s = it % STAGES, u = it / STAGES;
                    if (!mbar_wait(full_tma(s), u & 1, wc)) { ok = false; *abort_flag = 1; break; }
                    if (DQ != DQ_NONE) {
                        if (!mbar_wait(full_dq(s), u & 1, wc)) { ok = false; *abort_flag = 1; break; }
                    }
                    tc_fence_after();
                    const uint32_t sA = base + s * S::STAGE_BYTES;
                    const uint32_t sB = sA + S::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bd = B_MN ? smem_desc_sw128(sB + kk * 2048, 8192, 1024)
                                                 : smem_desc_sw128(sB + kk * 32, 16, 1024);
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const uint32_t a_t = sA + mt * 16384;
                            const uint64_t ad = A_MN ? smem_desc_sw128(a_t + kk * 2048, 8192, 1024)
                                                     : smem_desc_sw128(a_t + kk * 32, 16, 1024);
                            umma_bf16(tmem + mt * S::ACC_COLS, ad, bd, idesc,
                                      (k > sg.k0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    umma_commit(empty(s));
                }
                if (!ok) break;
                umma_commit(acc_full);
                ++seg_i;
            }
            if (!ok) {
                umma_commit(acc_full);
                mbar_wait(acc_full, seg_i & 1, wc);  // issued MMAs finish before TMEM is freed
            }
        }
    } else {
        const int ew = warp - 2;  // epilogue / dequant warp index
        // ------------------------------------------------------------ dequant setup
        uint32_t code_off = 0, code_off2 = 0, out_off = 0;
        int scale_idx = 0, wrow = 0, kb_off = 0;
        const bool dq_warp = DQ != DQ_NONE && ew < S::NDQ_WARPS;
        if (dq_warp) {
            const int t = ew * 32 + lane;  // block-row index inside the tile
            if (DQ == DQ_B_MN) {
                // codes tile [64 rows][128 B], TMA 128-byte swizzle
                const int j = t >> 2, c = t & 3;
                code_off = sw128(j * 128 + c * 32);
                code_off2 = sw128(j * 128 + c * 32 + 16);
                scale_idx = c * 64 + j;
                out_off = c * 8192 + j * 128;
                wrow = j;
                kb_off = c;
            } else {
                // codes tile [rows][32 B], TMA 32-byte swizzle
                code_off = sw32(t * 32);
                code_off2 = sw32(t * 32 + 16);
                scale_idx = t;
                out_off = t * 128;
                wrow = t;
            }
        }
        const uint32_t tile_off = (DQ == DQ_A_K) ? 0u : (uint32_t)S::A_BYTES;
        constexpr int GROUPS = S::NE_WARPS / 4;
        constexpr int COLS_PER_GROUP = BN / GROUPS;
        const int quarter = warp & 3;
        const int group = ew / 4;
        const int row = quarter * 32 + lane;  // accumulator row inside a 128-row sub-tile (TMEM lane)
        bool ok = true;
        int it = 0, seg_i = 0;
        Schedule sch(p);
        Seg sg;
        while (ok && sch.next(p, sg)) {
            const int m0 = sg.tm * S::BM, n0 = sg.tn * BN;
            // ---------------------------------------------------------- dequant
            if (DQ != DQ_NONE) {
                for (int k = sg.k0; k < sg.k1; ++k, ++it) {
                    if (!dq_warp) continue;
                    const int s = it % STAGES, u = it / STAGES;
                    if (!mbar_wait(full_tma(s), u & 1, wc)) { ok = false; *abort_flag = 1; break; }
                    if (k < p.ks_main) {
                        const uint32_t st = base + s * S::STAGE_BYTES;
                        const uint32_t sC = st + S::A_BYTES + S::B_BYTES;
                        const uint32_t sOut = st + tile_off;
                        bool valid;
                        if (DQ == DQ_B_MN)
                            valid = (64 * k + wrow < p.dq_rows) && (n0 / 64 + kb_off < p.dq_kbs);
                        else
                            valid = true;  // rows beyond the weight only feed masked outputs
                        if (valid) {
                            const float a = ld_shared_f32(sC + S::CODE_BYTES + 4u * scale_idx);
                            const uint4 c0 = ld_shared_v4(sC + code_off);
                            const uint4 c1 = ld_shared_v4(sC + code_off2);
                            const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                            const Nf4BlockTable tb = nf4_block_table(a, p.code_type);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                uint32_t o[4];
                                nf4_expand_word(words[q], tb, o);
                                st_shared_v4(sOut + sw128(out_off + q * 16), o[0], o[1], o[2], o[3]);
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                st_shared_v4(sOut + sw128(out_off + q * 16), 0u, 0u, 0u, 0u);
                        }
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(full_dq(s));
                }
                if (!ok) break;
            }
            // ---------------------------------------------------------- epilogue
            if (!mbar_wait(acc_full, seg_i & 1, wc)) { ok = false; *abort_flag = 1; break; }
            tc_fence_after();
            const bool full_tile = sg.k0 == 0 && sg.k1 == KS;
            // stream-K roles: a CTA whose segment starts inside a tile hands its
            // partial sum to the CTA that holds the tile's first k-steps
            const bool sk_writer = p.streamk && sg.k0 != 0;
            const bool sk_owner = p.streamk && sg.k0 == 0 && sg.k1 < KS;
            int first_c = 0, last_c = -1;
            if (sk_owner && !*abort_flag) {
                const int64_t I = (int64_t)p.tiles_total * KS;
                const int64_t t0 = (int64_t)(sg.tm * p.tiles_n + sg.tn) * KS;
                first_c = blockIdx.x + 1;
                last_c = blockIdx.x;
                for (int c = first_c; c < (int)gridDim.x; ++c) {
                    const int64_t sc = I * c / gridDim.x;
                    if (sc >= t0 + KS) break;
                    last_c = c;
                }
                // wait until every contributor has published its partial
                // (CTAs with an empty share publish nothing and add nothing)
                for (int c = first_c; c <= last_c; ++c) {
                    if (I * (c + 1) / gridDim.x == I * c / gridDim.x) continue;
                    const int* f = p.sk_flags + c;
                    if (ld_acquire_gpu(f) == 0) {
                        const uint64_t t_start = globaltimer_ns();
                        while (ld_acquire_gpu(f) == 0) {
                            if (globaltimer_ns() - t_start > p.timeout_ns) {
                                set_status(4);
                                *abort_flag = 1;
                                break;
                            }
                        }
                    }
                }
            }
            // warp-uniform decision (tcgen05.ld below is a warp-wide instruction)
            const bool skip = __any_sync(0xffffffffu, *abort_flag != 0);
            // Grid schedule with bf16 output: the pipeline is idle once the
            // accumulator is complete, so the tile is staged in the stage
            // buffers (128B-swizzled 64-column panels) and written with TMA.
            constexpr bool kStage = EPI == EPI_BF16;
            const bool staged = kStage && !p.streamk;
            constexpr int ITC = MT * (COLS_PER_GROUP / 32);
            const int tid_e = ew * 32 + lane;
            for (int itc = 0; itc < ITC && !skip; ++itc) {
                const int mt = itc / (COLS_PER_GROUP / 32);
                const int cc = (itc % (COLS_PER_GROUP / 32)) * 32;
                const int trow = 128 * mt + row;  // row inside the CTA tile
                const int grow = m0 + trow;
                const bool row_ok = grow < p.rows;
                const int col0 = group * COLS_PER_GROUP + cc;
                uint32_t v[32];
                __syncwarp();
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(mt * S::ACC_COLS + col0), v);
                tmem_ld_wait();
                const int gcol0 = n0 + col0;
                if (sg.k1 <= sg.k0) {
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] = 0u;
                }
                // stream-K partial tiles use a thread-major layout so that every
                // warp access is 512 contiguous bytes
                if (sk_writer) {
                    float* o = p.sk_part + ((int64_t)blockIdx.x * ITC + itc) * 8 * (S::NE_WARPS * 32 * 4);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4*>(o + ((int64_t)q * S::NE_WARPS * 32 + tid_e) * 4) =
                            make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    continue;
                }
                if (sk_owner) {
                    const int64_t I = (int64_t)p.tiles_total * KS;
                    for (int c = first_c; c <= last_c; ++c) {
                        if (I * (c + 1) / gridDim.x == I * c / gridDim.x) continue;
                        const float* o = p.sk_part + ((int64_t)c * ITC + itc) * 8 * (S::NE_WARPS * 32 * 4);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 w4 = __ldcg(reinterpret_cast<const float4*>(
                                o + ((int64_t)q * S::NE_WARPS * 32 + tid_e) * 4));
                            v[4 * q + 0] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * q + 0]), w4.x));
                            v[4 * q + 1] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * q + 1]), w4.y));
                            v[4 * q + 2] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * q + 2]), w4.z));
                            v[4 * q + 3] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * q + 3]), w4.w));
                        }
                    }
                }
                if (kStage && staged) {
                    // panel (mt, col0/64): rows 0..127 of 128 B, 16-byte chunk j of row r
                    // at ((j ^ r%8) * 16); this thread's 32 columns are chunks h..h+3
                    const uint32_t panel = base + (uint32_t)(mt * (BN / 64) + (col0 >> 6)) * 16384u;
                    const int h = (col0 & 63) >> 3;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t w0 = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                        const uint32_t w1 = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                        const uint32_t w2 = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                        const uint32_t w3 = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                        st_shared_v4(panel + sw128((uint32_t)row * 128u + (uint32_t)(h + q) * 16u), w0, w1, w2, w3);
                    }
                    continue;
                }
                if (!row_ok) continue;
                if (EPI == EPI_BF16) {
                    uint16_t* o = static_cast<uint16_t*>(p.out) + (int64_t)grow * p.out_ld + gcol0;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (gcol0 + 8 * q + 8 <= p.cols) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                            w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                            w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                            w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                            *reinterpret_cast<uint4*>(o + 8 * q) = w;
                        }
                    }
                } else if (EPI == EPI_BF16_T) {
                    uint16_t* o = static_cast<uint16_t*>(p.out) + grow;
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        if (gcol0 + q < p.cols) {
                            uint32_t h = pack_bf16x2(__uint_as_float(v[q]), 0.0f) & 0xFFFFu;
                            o[(int64_t)(gcol0 + q) * p.out_ld] = (uint16_t)h;
                        }
                    }
                } else if (EPI == EPI_F32) {
                    float* o = static_cast<float*>(p.out) + (int64_t)sg.split * p.out_split_stride +
                               (int64_t)grow * p.out_ld + gcol0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (gcol0 + 4 * q + 4 <= p.cols)
                            *reinterpret_cast<uint4*>(o + 4 * q) =
                                make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                } else {  // EPI_F32_T
                    float* o = static_cast<float*>(p.out) + (int64_t)sg.split * p.out_split_stride + grow;
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        if (gcol0 + q < p.cols) o[(int64_t)(gcol0 + q) * p.out_ld] = __uint_as_float(v[q]);
                }
            }
            if (staged) {
                // all panels written -> visible to the TMA engine -> one thread stores
                fence_proxy_async_smem();
                named_bar(1, S::NE_WARPS * 32);
                if (ew == 0 && lane == 0 && !skip) {
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int c = 0; c < BN / 64; ++c)
                            tma_store_2d(&p.tmOut, base + (uint32_t)(mt * (BN / 64) + c) * 16384u, n0 + 64 * c,
                                         m0 + 128 * mt);
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
                named_bar(1, S::NE_WARPS * 32);
            }
            if (sk_writer) {
                // publish the partial: every epilogue thread's stores, then one flag
                __threadfence();
                named_bar(1, S::NE_WARPS * 32);
                if (ew == 0 && lane == 0 && !*abort_flag) st_release_gpu(p.sk_flags + blockIdx.x, 1);
            }
            (void)full_tile;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
            ++seg_i;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, S::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// split-K reduction: out = cast(scale * sum_z part[z][i][j]) in fixed z order
// ---------------------------------------------------------------------------
enum { RED_BF16 = 0, RED_F32 = 1, RED_F32_T = 2 };

__global__ void k_splitk_reduce(const float* __restrict__ part, int splits, int64_t split_stride,
                                int rows, int cols, int64_t part_ld, float scale, int mode,
                                void* __restrict__ out, int64_t out_ld) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)rows * cols) return;
    const int64_t i = idx / cols, j = idx - i * cols;
    float acc = 0.0f;
    for (int z = 0; z < splits; ++z) acc = __fadd_rn(acc, part[z * split_stride + i * part_ld + j]);
    acc = __fmul_rn(acc, scale);
    if (mode == RED_BF16) {
        uint32_t h = pack_bf16x2(acc, 0.0f) & 0xFFFFu;
        static_cast<uint16_t*>(out)[i * out_ld + j] = (uint16_t)h;
    } else if (mode == RED_F32) {
        static_cast<float*>(out)[i * out_ld + j] = acc;
    } else {
        static_cast<float*>(out)[j * out_ld + i] = acc;
    }
}

__global__ void k_fill_zero_f32(float* __restrict__ p, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = 0.0f;
}

}  // namespace qlora
