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

// Work of one CTA pair: a list of segments (tile, k-step range).  Grid
// schedule: one segment, the whole k-range of tile (tm = blockIdx.x/2,
// tn = blockIdx.y).  Stream-K schedule (p.streamk): the pair c of
// G = gridDim.x/2 owns the contiguous share [c*I/G, (c+1)*I/G) of all
// I = tiles * KS (tile, k-step) iterations; a tile cut between pairs is
// finished by the pair that holds its first k-steps (the owner), which adds
// the fp32 partial sums the other pairs publish, in pair order.  Both orders
// run the token tiles fastest: the pairs resident at once share a few weight
// column tiles, so each tile of codes is read from DRAM once and then hits
// in L2 for the other token tiles (with the token tiles slowest, a weight
// larger than L2 -- the 65B gate/up codes are 180 MB -- was read once per
// token tile).
struct PairSeg {
    int tm, tn, k0, k1;
};

template <bool SK>
struct PairSchedule {
    int64_t pos, end;
    int KS;
    bool grid_done;
    __device__ PairSchedule(const GemmParams& p) {
        KS = p.ks_main + p.ks_lora;
        grid_done = false;
        pos = end = 0;
        if (SK) {
            const int64_t I = (int64_t)p.tiles_total * KS;
            const int c = blockIdx.x >> 1, G = gridDim.x >> 1;
            pos = I * c / G;
            end = I * (c + 1) / G;
        }
    }
    __device__ bool next(const GemmParams& p, PairSeg& sg) {
        if (!SK) {
            if (grid_done) return false;
            grid_done = true;
            sg.tm = p.n_in_x ? blockIdx.y : blockIdx.x >> 1;
            sg.tn = p.n_in_x ? blockIdx.x >> 1 : blockIdx.y;
            sg.k0 = 0;
            sg.k1 = KS;
            return true;
        }
        if (pos >= end) return false;
        const int t = (int)(pos / KS);
        const int tiles_m = p.tiles_total / p.tiles_n;
        sg.tn = t / tiles_m;
        sg.tm = t % tiles_m;
        sg.k0 = (int)(pos - (int64_t)t * KS);
        sg.k1 = (int)min((int64_t)KS, (int64_t)sg.k0 + (end - pos));
        pos += sg.k1 - sg.k0;
        return true;
    }
    __device__ bool more() const { return SK && pos < end; }
};

template <int DQ, int STAGES, bool SK>
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
    const uint32_t acc_empty = bar_base + 8u * (3 * STAGES + 1);
    // stream-K owner: ring of PF_SLOTS 16 KB slots (after the 128 KB of output
    // panels) that the contributors' partial chunks are bulk-loaded into
    constexpr int PF_SLOTS = 5;
    static_assert(8 * 16384 + PF_SLOTS * 16384 <= S::STAGE_BYTES * STAGES, "prefetch ring fits the stage buffers");
    auto pf_full = [&](int j) { return bar_base + 8u * (3 * STAGES + 2 + j); };
    uint32_t* tmem_holder =
        reinterpret_cast<uint32_t*>(gbase + S::STAGE_BYTES * STAGES + 8 * (3 * STAGES + 2 + PF_SLOTS));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* epi_skip = reinterpret_cast<volatile int*>(tmem_holder + 2);  // [2]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const WaitCfg wc{p.timeout_ns};

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_tma(s), 1);
            mbar_init(full_dq(s), 2 * S::NDQ_WARPS);  // dequant warps of both CTAs (leader's copy is used)
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * S::NDQ_WARPS);  // epilogue warps of both CTAs (leader's copy is used)
        for (int j = 0; j < PF_SLOTS; ++j) mbar_init(pf_full(j), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        pdl_trigger();
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
        // the block constants and the LoRA operand come from earlier kernels;
        // with late_wait only the LoRA operand is still being written
        if (lane == 0 && !p.late_wait) pdl_wait();
        bool waited = !p.late_wait;
        if (lane == 0 && !p.inject) {
            int last_use[STAGES];
            for (int s = 0; s < STAGES; ++s) last_use[s] = -1;
            PairSchedule<SK> sch(p);
            PairSeg sg;
            int it = 0;
            bool ok = true;
            while (ok && sch.next(p, sg)) {
                const int m0 = sg.tm * 512;
                const int nb0 = sg.tn * 256 + 128 * (int)rank;  // first Bop column of this CTA
                for (int k = sg.k0; k < sg.k1; ++k, ++it) {
                    const int s = it % STAGES, u = it / STAGES;
                    if (k >= p.ks_main && !waited) {
                        pdl_wait();
                        waited = true;
                    }
                    if (!mbar_wait(empty(s), (u & 1) ^ 1, wc)) { *abort_flag = 1; ok = false; break; }
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
                        tma_load_2d(sA + mt * 16384, mA, full_tma(s), kc * 64 + (lora ? lora_col0(p, sg.tn * 256) : 0),
                                    m0 + 256 * mt + 128 * (int)rank);
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
            }
            // every load has landed before the CTA can exit
            for (int s = 0; s < STAGES; ++s)
                if (last_use[s] >= 0) mbar_wait(full_tma(s), last_use[s] & 1, wc);
        }
        // the kernel does not complete before the previous one
        if (lane == 0 && !waited) pdl_wait();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(256, 256, 0, B_MN);
            bool ok = true;
            PairSchedule<SK> sch(p);
            PairSeg sg;
            int it = 0, seg_i = 0;
            while (ok && sch.next(p, sg)) {
                // the epilogue of the previous segment has read both CTAs' accumulators
                if (seg_i > 0 && !mbar_wait(acc_empty, (seg_i - 1) & 1, wc)) {
                    ok = false;
                    *abort_flag = 1;
                } else {
                    tc_fence_after();
                }
                for (int k = sg.k0; ok && k < sg.k1; ++k, ++it) {
                    const int s = it % STAGES, u = it / STAGES;
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
                            umma_bf16_pair(tmem + mt * 256, ad, bd, idesc, (k > sg.k0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    umma_commit_pair_mc(empty(s), 0x3);
                }
                // one acc_full phase per segment, also when it was cut short
                umma_commit_pair_mc(acc_full, 0x3);
                ++seg_i;
            }
            // on an abort, nothing may still be in flight when the CTA exits
            if (!ok) mbar_wait(acc_full, (seg_i - 1) & 1, wc);
        }
    } else {
        // ------------------------------------------------------------ dequant + epilogue (both CTAs)
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
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // TMEM lane = accumulator row of this thread
        const int KS = p.ks_main + p.ks_lora;
        PairSchedule<SK> sch(p);
        PairSeg sg;
        int it = 0, seg_i = 0;
        // After a wait runs out the warp stops waiting and working ("dead")
        // but still walks every segment, so that the four epilogue warps
        // reach the same named barriers in the same order.
        bool dead = false;
        while (sch.next(p, sg)) {
            const int m0 = sg.tm * 512, n0 = sg.tn * 256;
            const int nb0 = n0 + 128 * (int)rank;
            for (int k = sg.k0; k < sg.k1; ++k, ++it) {
                const int s = it % STAGES, u = it / STAGES;
                if (dead) continue;
                if (!mbar_wait(full_tma(s), u & 1, wc)) {
                    *abort_flag = 1;
                    dead = true;
                    continue;
                }
                if (k < p.ks_main) {
                    const uint32_t st = base + s * S::STAGE_BYTES;
                    const uint32_t sOut = st + S::A_BYTES;
                    const uint32_t sC = sOut + S::B_BYTES;
                    const bool valid = DQ == DQ_B_MN
                                           ? (64 * k + wrow < p.dq_rows) && (nb0 / 64 + kb_off < p.dq_kbs)
                                           : true;
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
                        for (int q = 0; q < 8; ++q) st_shared_v4(sOut + sw128(out_off + q * 16), 0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(full_dq(s), 0));
            }

            // -------------------------------------------------------- epilogue of the segment
            if (!dead) {
                if (mbar_wait(acc_full, seg_i & 1, wc)) {
                    tc_fence_after();
                } else {
                    *abort_flag = 1;
                    dead = true;
                }
            }
            const bool sk_writer = SK && sg.k0 != 0;
            const bool sk_owner = SK && sg.k0 == 0 && sg.k1 < KS;
            // the pipeline is idle after the last segment: stage the tile in
            // its buffers and store it with TMA
            const bool staged = !sk_writer && !sch.more();
            int first_c = 0, last_c = -1;
            const int cid = blockIdx.x >> 1, G = gridDim.x >> 1;
            const int64_t I = (int64_t)p.tiles_total * KS;
            if (sk_owner && !*abort_flag) {
                const int64_t t0 = (int64_t)(sg.tn * (p.tiles_total / p.tiles_n) + sg.tm) * KS;
                first_c = cid + 1;
                last_c = cid;
                for (int c = first_c; c < G; ++c) {
                    if (I * c / G >= t0 + KS) break;
                    last_c = c;
                }
                // every contributor (same rank in a later pair) publishes its partial
                for (int c = first_c; c <= last_c; ++c) {
                    if (I * (c + 1) / G == I * c / G) continue;
                    const int* f = p.sk_flags + 2 * c + (int)rank;
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
            // one decision for all four epilogue warps (they meet at named barriers below)
            if (ew == 0 && lane == 0) epi_skip[seg_i & 1] = 0;
            named_bar(1, S::NDQ_WARPS * 32);
            if (lane == 0 && (dead || *abort_flag != 0)) epi_skip[seg_i & 1] = 1;
            named_bar(1, S::NDQ_WARPS * 32);
            const bool skip = epi_skip[seg_i & 1] != 0;
            const int tid_e = ew * 32 + lane;
            // owner: contributors with a non-empty share, and the prefetch of
            // their chunks (chunk j = itc * nc + ci) into the slot ring
            int nc = 0;
            if (sk_owner && !skip) {
                for (int c = first_c; c <= last_c; ++c)
                    if (I * (c + 1) / G != I * c / G) ++nc;
            }
            auto chunk_src = [&](int j) {
                const int itc = j / nc, ci = j - (j / nc) * nc;
                int c = first_c, seen = -1;
                for (; c <= last_c; ++c) {
                    if (I * (c + 1) / G == I * c / G) continue;
                    if (++seen == ci) break;
                }
                return p.sk_part + ((int64_t)(2 * c + (int)rank) * 16 + itc) * 8 * 128 * 4;
            };
            const uint32_t pf_base = base + 8u * 16384u;
            if (nc > 0 && ew == 0 && lane == 0) {
                // the partials were acquired through the flags; order the bulk
                // copies' (async proxy) reads after that
                asm volatile("fence.proxy.async.global;" ::: "memory");
                for (int j = 0; j < PF_SLOTS && j < 16 * nc; ++j) {
                    mbar_arrive_expect_tx(pf_full(j), 16384);
                    bulk_load(pf_base + 16384u * j, chunk_src(j), 16384, pf_full(j));
                }
            }
            if (!skip) {
#pragma unroll 1
                for (int itc = 0; itc < 16; ++itc) {
                    const int mt = itc >> 3, col0 = (itc & 7) * 32;
                    uint32_t v[32];
                    __syncwarp();
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(mt * 256 + col0), v);
                    tmem_ld_wait();
                    if (sk_writer) {
                        // thread-major partial layout: each warp access is 512 contiguous bytes
                        float* o = p.sk_part + ((int64_t)blockIdx.x * 16 + itc) * 8 * 128 * 4;
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<uint4*>(o + ((int64_t)q * 128 + tid_e) * 4) =
                                make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                        continue;
                    }
                    if (nc > 0) {
                        // add the contributors' partials in pair order
                        for (int ci = 0; ci < nc; ++ci) {
                            const int j = itc * nc + ci;
                            const int slot = j % PF_SLOTS;
                            const bool got = mbar_wait(pf_full(slot), (j / PF_SLOTS) & 1, wc);
                            if (!got) *abort_flag = 1;
                            const uint32_t src = pf_base + 16384u * slot;
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const uint4 w4 = ld_shared_v4(src + (uint32_t)((q * 128 + tid_e) * 16));
                                v[4 * q + 0] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * q + 0]), __uint_as_float(w4.x)));
                                v[4 * q + 1] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * q + 1]), __uint_as_float(w4.y)));
                                v[4 * q + 2] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * q + 2]), __uint_as_float(w4.z)));
                                v[4 * q + 3] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * q + 3]), __uint_as_float(w4.w)));
                            }
                            // every thread has read the slot: refill it with chunk j + PF_SLOTS
                            named_bar(1, S::NDQ_WARPS * 32);
                            if (ew == 0 && lane == 0 && j + PF_SLOTS < 16 * nc) {
                                mbar_arrive_expect_tx(pf_full(slot), 16384);
                                bulk_load(pf_base + 16384u * slot, chunk_src(j + PF_SLOTS), 16384, pf_full(slot));
                            }
                        }
                    }
                    if (staged) {
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
                    } else {
                        // a later segment follows: direct stores (the stage buffers are in use)
                        const int grow = m0 + 256 * mt + 128 * (int)rank + row;
                        const int gcol0 = n0 + col0;
                        if (grow < p.rows) {
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
                        }
                    }
                }
            }
            if (staged) {
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
            if (sk_writer) {
                // publish the partial: every epilogue thread's stores, then one flag
                __threadfence();
                named_bar(1, S::NDQ_WARPS * 32);
                if (ew == 0 && lane == 0 && !*abort_flag) st_release_gpu(p.sk_flags + blockIdx.x, 1);
            }
            // this CTA's accumulators are free for the next segment
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && !dead) mbar_arrive_cluster(mapa_shared(acc_empty, 0));
            ++seg_i;
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
