// gemm_pair.cuh -- the large-M dequant GEMMs on CTA pairs (tcgen05 cta_group::2).
//
// A cluster of two CTAs computes one 512 x 256 output tile: D = Aop * Bop^T
// with Aop the activations (token rows, K-major, TMA) and Bop the frozen NF4
// weight, expanded to bf16 in shared memory by dequant warps.  Each CTA holds
// token rows {256*mt + 128*rank + [0, 128)} (mt = 0, 1) and dequantizes its
// 128-column half of Bop; the leader issues M=256, N=256 pair MMAs into two
// TMEM accumulators (512 columns in each CTA).  Per SM, a k-step dequantizes
// 128 x 64 weights while the pair computes 512 x 256 x 64: a quarter of the
// dequant work per MMA flop of a single-CTA 128 x 256 tile.
//
// Synchronization: every CTA's TMA loads complete on its own full_tma
// barrier; its dequant warps wait on it, write their half of Bop, fence the
// generic->async proxy and arrive on the LEADER's full_dq barrier (remote
// arrive).  The leader's MMA warp waits on full_dq, issues the MMAs and
// commits to empty / acc_full in both CTAs (commit multicast).  No TMA load
// uses cluster multicast.
#pragma once

#include "common.cuh"
#include "gemm.cuh"
#include "nf4.cuh"

namespace qlora {

template <int DQ>
struct PairShape {
    static_assert(DQ == DQ_B_K || DQ == DQ_B_MN, "pair kernel dequantizes the B operand");
    static constexpr int A_BYTES = 2 * 16384;       // two 128-row K-major token tiles
    static constexpr int B_BYTES = 128 * 128;       // this CTA's 128 Bop columns x 64 k
    static constexpr int CODE_BYTES = 4096;         // forward: 128 rows x 32 B; dX: 64 rows x 64 B
    static constexpr int SCALE_BYTES = 512;         // 128 block constants
    static constexpr int STAGE_RAW = A_BYTES + B_BYTES + CODE_BYTES + SCALE_BYTES;
    static constexpr int STAGE_BYTES = (STAGE_RAW + 1023) / 1024 * 1024;
    static constexpr int NDQ_WARPS = 4;
    static constexpr int THREADS = 32 * (2 + NDQ_WARPS);
    static constexpr int TMEM_COLS = 512;
};

template <int DQ, int STAGES>
constexpr int pair_smem_bytes() {
    return PairShape<DQ>::STAGE_BYTES * STAGES + 1024 + 256;
}

// Physical offset inside a TMA tile written with the 64-byte swizzle.
__device__ __forceinline__ uint32_t sw64(uint32_t off) { return off ^ (((off >> 7) & 3u) << 4); }

template <int DQ, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairShape<DQ>::THREADS, 1)
    k_gemm_pair(const __grid_constant__ GemmParams p) {
    using S = PairShape<DQ>;
    constexpr int B_MN = DQ == DQ_B_MN ? 1 : 0;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw_base);
    const uint32_t bar_base = base + S::STAGE_BYTES * STAGES;
    auto full_tma = [&](int s) { return bar_base + 8u * s; };
    auto full_dq = [&](int s) { return bar_base + 8u * (STAGES + s); };
    auto empty = [&](int s) { return bar_base + 8u * (2 * STAGES + s); };
    const uint32_t acc_full = bar_base + 8u * (3 * STAGES);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + S::STAGE_BYTES * STAGES + 8 * (3 * STAGES + 2));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const WaitCfg wc{p.timeout_ns};
    const int KS = p.ks_main + p.ks_lora;
    const int tn = blockIdx.x >> 1, tm = blockIdx.y;
    const int m0 = tm * 512, n0 = tn * 256;
    const int nb0 = n0 + 128 * (int)rank;  // first Bop column of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_tma(s), 1);
            mbar_init(full_dq(s), 2 * S::NDQ_WARPS);  // dequant warps of both CTAs (leader's copy is used)
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&p.tmA);
        prefetch_tensormap(&p.tmCodes);
        prefetch_tensormap(&p.tmOut);
        if (p.ks_lora) {
            prefetch_tensormap(&p.tmA2);
            prefetch_tensormap(&p.tmB2);
        }
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(tmem_holder), S::TMEM_COLS);
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialized, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0 && !p.inject) {
            int last_use[STAGES];
            for (int s = 0; s < STAGES; ++s) last_use[s] = -1;
            for (int k = 0; k < KS; ++k) {
                const int s = k % STAGES, u = k / STAGES;
                if (!mbar_wait(empty(s), (u & 1) ^ 1, wc)) { *abort_flag = 1; break; }
                const uint32_t sA = base + s * S::STAGE_BYTES;
                const uint32_t sB = sA + S::A_BYTES;
                const uint32_t sC = sB + S::B_BYTES;
                const uint32_t sS = sC + S::CODE_BYTES;
                const bool lora = k >= p.ks_main;
                const int kc = lora ? k - p.ks_main : k;
                uint32_t bytes = S::A_BYTES;
                if (lora) {
                    bytes += S::B_BYTES;
                } else {
                    bytes += S::CODE_BYTES;
                    if (DQ == DQ_B_K) {
                        bytes += 512;
                    } else {
                        for (int c = 0; c < 2; ++c)
                            if (nb0 / 64 + c < p.dq_kbs) bytes += 256;
                    }
                }
                mbar_arrive_expect_tx(full_tma(s), bytes);
                const CUtensorMap* mA = lora ? &p.tmA2 : &p.tmA;
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
                    tma_load_2d(sA + mt * 16384, mA, full_tma(s), kc * 64, m0 + 256 * mt + 128 * (int)rank);
                if (lora) {
                    if (B_MN) {
                        for (int c = 0; c < 2; ++c)
                            tma_load_2d(sB + 8192 * c, &p.tmB2, full_tma(s), nb0 + 64 * c, kc * 64);
                    } else {
                        tma_load_2d(sB, &p.tmB2, full_tma(s), kc * 64, nb0);
                    }
                } else if (DQ == DQ_B_K) {
                    tma_load_2d(sC, &p.tmCodes, full_tma(s), kc * 32, nb0);
                    bulk_load(sS, p.scales + (int64_t)kc * p.scales_ld + nb0, 512, full_tma(s));
                } else {
                    tma_load_2d(sC, &p.tmCodes, full_tma(s), nb0 / 2, kc * 64);
                    for (int c = 0; c < 2; ++c)
                        if (nb0 / 64 + c < p.dq_kbs)
                            bulk_load(sS + 256 * c, p.scales + (int64_t)(nb0 / 64 + c) * p.scales_ld + kc * 64,
                                      256, full_tma(s));
                }
                last_use[s] = u;
            }
            for (int s = 0; s < STAGES; ++s)
                if (last_use[s] >= 0) mbar_wait(full_tma(s), last_use[s] & 1, wc);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(256, 256, 0, B_MN);
            bool ok = true;
            for (int k = 0; k < KS; ++k) {
                const int s = k % STAGES, u = k / STAGES;
                if (!mbar_wait(full_dq(s), u & 1, wc)) { ok = false; *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t sA = base + s * S::STAGE_BYTES;
                const uint32_t sB = sA + S::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bd = B_MN ? smem_desc_sw128(sB + kk * 2048, 8192, 1024)
                                             : smem_desc_sw128(sB + kk * 32, 16, 1024);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        const uint64_t ad = smem_desc_sw128(sA + mt * 16384 + kk * 32, 16, 1024);
                        umma_bf16_pair(tmem + mt * 256, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                umma_commit_pair_mc(empty(s), 0x3);
            }
            umma_commit_pair_mc(acc_full, 0x3);
            if (!ok) mbar_wait(acc_full, 0, wc);
        }
    } else {
        // ------------------------------------------------------------ dequant (both CTAs)
        const int ew = warp - 2;
        const int t = ew * 32 + lane;  // block-row of this CTA's Bop half
        uint32_t code_off, code_off2, out_off;
        int scale_idx, wrow = 0, kb_off = 0;
        if (DQ == DQ_B_MN) {
            // codes tile [64 rows][64 B], TMA 64-byte swizzle; Bop = 2 MN chunks of 64
            const int j = t >> 1, c = t & 1;
            code_off = sw64(j * 64 + c * 32);
            code_off2 = sw64(j * 64 + c * 32 + 16);
            scale_idx = c * 64 + j;
            out_off = c * 8192 + j * 128;
            wrow = j;
            kb_off = c;
        } else {
            code_off = sw32(t * 32);
            code_off2 = sw32(t * 32 + 16);
            scale_idx = t;
            out_off = t * 128;
        }
        for (int k = 0; k < KS; ++k) {
            const int s = k % STAGES, u = k / STAGES;
            if (!mbar_wait(full_tma(s), u & 1, wc)) { *abort_flag = 1; break; }
            if (k < p.ks_main) {
                const uint32_t st = base + s * S::STAGE_BYTES;
                const uint32_t sOut = st + S::A_BYTES;
                const uint32_t sC = sOut + S::B_BYTES;
                const bool valid = DQ == DQ_B_MN ? (64 * k + wrow < p.dq_rows) && (nb0 / 64 + kb_off < p.dq_kbs)
                                                 : true;
                if (valid) {
                    const float a = ld_shared_f32(sC + S::CODE_BYTES + 4u * scale_idx);
                    const uint4 c0 = ld_shared_v4(sC + code_off);
                    const uint4 c1 = ld_shared_v4(sC + code_off2);
                    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                    const Nf4BlockTable tb = nf4_block_table(a);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint32_t o[4];
                        nf4_expand_word(words[q], tb, o);
                        st_shared_v4(sOut + sw128(out_off + q * 16), o[0], o[1], o[2], o[3]);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) st_shared_v4(sOut + sw128(out_off + q * 16), 0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(full_dq(s), 0));
        }
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        bool ok = mbar_wait(acc_full, 0, wc);
        if (ok) tc_fence_after();
        const bool skip = __any_sync(0xffffffffu, !ok || *abort_flag != 0);
        if (!skip) {
#pragma unroll 1
            for (int itc = 0; itc < 16; ++itc) {
                const int mt = itc >> 3, col0 = (itc & 7) * 32;
                uint32_t v[32];
                __syncwarp();
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(mt * 256 + col0), v);
                tmem_ld_wait();
                const uint32_t panel = base + (uint32_t)(mt * 4 + (col0 >> 6)) * 16384u;
                const int h = (col0 & 63) >> 3;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t w0 = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                    const uint32_t w1 = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                    const uint32_t w2 = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                    const uint32_t w3 = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                    st_shared_v4(panel + sw128((uint32_t)row * 128u + (uint32_t)(h + q) * 16u), w0, w1, w2, w3);
                }
            }
        }
        fence_proxy_async_smem();
        named_bar(1, S::NDQ_WARPS * 32);
        if (ew == 0 && lane == 0 && !skip) {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tma_store_2d(&p.tmOut, base + (uint32_t)(mt * 4 + c) * 16384u, n0 + 64 * c,
                                 m0 + 256 * mt + 128 * (int)rank);
            bulk_commit_group();
            bulk_wait_group_read0();
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the leader's MMAs and remote arrivals are done in both CTAs
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, S::TMEM_COLS);
    }
}

}  // namespace qlora
