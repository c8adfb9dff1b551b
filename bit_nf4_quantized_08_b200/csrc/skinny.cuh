// skinny.cuh -- the rank-r LoRA GEMMs (U = X A^T, G = dY B, dA = G^T X,
// dB = dY^T U): a tall operand times an r-column operand, r <= 256.
//
// out[i][j] = scale * sum_k Aop[i][k] * Bop[j][k]   (i < rows, j < r)
// They are HBM-bound (each streams X or dY once), so the reduction dimension
// is split across the CS CTAs of a thread-block cluster: each CTA runs a TMA
// -> tcgen05 pipeline over its k-range into TMEM, then sends every row of
// its fp32 partial tile to the CTA that owns the row with asynchronous
// distributed-shared-memory stores that complete on the owner's mbarrier.
// Each owner waits for its CS partials, sums them in rank order
// (deterministic) and writes the final output.  One launch carries one or
// two independent problems of the same r (U and G, or dA and dB); the
// cluster index selects the problem and its 128-row tile.
//
// The reduction buffer has its own shared memory, except for r > 128
// (RED_OVERLAY), where it reuses the pipeline buffers once every CTA of the
// cluster has drained its pipeline.
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace qlora {

enum { SK_OUT_BF16 = 0, SK_OUT_F32 = 1, SK_OUT_F32_T = 2 };

struct SkinnyProblem {
    CUtensorMap tmA, tmB;
    int rows, r;     // output extent
    int ksteps;      // 64-wide k-steps of the whole reduction
    int per;         // k-steps per cluster rank
    int a_mn, b_mn;  // operand majorness (1: MN-major)
    int tiles;       // 128-row tiles
    float scale;
    int out_mode;
    void* out;
    int64_t out_ld;  // elements
    // adapters of a fused projection (row segments of seg_rows, rank seg_r
    // each).  SK_SEG_REDUCE: the MN-major B operand's columns are shifted by
    // -(segment of the k-step's reduction index) * seg_r, so each output
    // column block only gathers its own segment (G = dY B per segment);
    // SK_SEG_ROWS: shifted by +(segment of the tile's output rows) * seg_r
    // (dB of a segment reads its own sU columns).  Shifted-out columns read
    // the load's zero fill.
    int seg_mode, seg_rows, seg_r;
};

enum { SK_SEG_NONE = 0, SK_SEG_REDUCE = 1, SK_SEG_ROWS = 2 };

// Column offset of the B operand of problem P at k-step k of the tile at row m0.
__device__ __forceinline__ int skinny_b_col0(const SkinnyProblem& P, int k, int m0) {
    if (P.seg_mode == SK_SEG_REDUCE) return -((k * 64) / P.seg_rows) * P.seg_r;
    if (P.seg_mode == SK_SEG_ROWS) return (m0 / P.seg_rows) * P.seg_r;
    return 0;
}

struct SkinnyParams {
    SkinnyProblem pr[3];
    int nprob;
    uint64_t timeout_ns;
    int inject;
    int wait_first;  // the operands may come from the previous kernel: wait before loading
    // pack: the launch's clusters of 2 only place two CTAs on one TPC; each
    // CTA reduces its own tile alone (reduction cluster of 1).  CTAs past the
    // last tile (odd tile counts) load nothing and write nothing.
    int pack;
    int total_tiles;
    // k_lora_stream only: tiles taken from *tile_ctr (zero before the
    // launch) in problem order instead of round-robin; problem dep_prob (if
    // >= 0) reads the output of problem 0, whose finished tiles are counted
    // (per epilogue warp) in *done_ctr (zero before the launch)
    int* tile_ctr;
    int* done_ctr;
    int dep_prob;
    // k_lora_stream with wait_first == 0: problems (bit i = problem i) whose
    // operands come from the previous kernel; the producer waits for it
    // before the first such tile only
    int wait_mask;
};

template <int BN>
struct SkinnyShape {
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int PART_LD = BN + 4;  // fp32 row pitch of the reduction buffer (floats)
    // reduction buffer [cs][128 / cs][PART_LD] (cs a power of two <= 8)
    static constexpr int RED_BYTES = 128 * PART_LD * 4;
    static constexpr bool RED_OVERLAY = BN > 128;
    static constexpr int STAGES = BN <= 64 ? 7 : (BN <= 128 ? 4 : 3);
    static constexpr int PIPE_BYTES = STAGE_BYTES * STAGES;
    static constexpr int RED_OFF = RED_OVERLAY ? 0 : PIPE_BYTES;
    static constexpr int REGION = RED_OVERLAY ? (PIPE_BYTES > RED_BYTES ? PIPE_BYTES : RED_BYTES)
                                              : PIPE_BYTES + RED_BYTES;
    static constexpr int SMEM = REGION + 1024 + 256;
    static constexpr int THREADS = 32 * 6;  // producer, MMA, 4 epilogue warps
};

__device__ __forceinline__ void cluster_arrive() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    __syncwarp();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 16 bytes into another CTA's shared memory; completes 16 transaction bytes
// on the destination CTA's mbarrier (both addresses in the cluster window).
__device__ __forceinline__ void st_async_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                            uint32_t bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
        "r"(a), "r"(b), "r"(c), "r"(d), "r"(bar)
        : "memory");
}

template <int BN>
__global__ void __launch_bounds__(SkinnyShape<BN>::THREADS, 1) k_skinny(const __grid_constant__ SkinnyParams p) {
    using S = SkinnyShape<BN>;
    constexpr int STAGES = S::STAGES;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw_base);
    const uint32_t red_base = base + S::RED_OFF;
    const uint32_t bar_base = base + S::REGION;
    auto full = [&](int s) { return bar_base + 8u * s; };
    auto empty = [&](int s) { return bar_base + 8u * (STAGES + s); };
    const uint32_t acc_full = bar_base + 8u * (2 * STAGES);
    const uint32_t red_full = bar_base + 8u * (2 * STAGES + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + S::REGION + 8 * (2 * STAGES + 2));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WaitCfg wc{p.timeout_ns};
    const int cs = p.pack ? 1 : (int)cluster_nctarank();
    const int z = p.pack ? 0 : (int)cluster_ctarank();
    const uint32_t self_rank = p.pack ? cluster_ctarank() : 0u;  // owner rank offset in the launch cluster
    const bool spare = p.pack && (int)blockIdx.x >= p.total_tiles;
    int tile = spare ? 0 : (int)blockIdx.x / cs;
    const int pi = (p.nprob > 1 && tile >= p.pr[0].tiles) ? 1 : 0;
    if (pi) tile -= p.pr[0].tiles;
    const SkinnyProblem& P = p.pr[pi];
    const int a_mn = P.a_mn, b_mn = P.b_mn;
    const int m0 = spare ? P.rows : tile * 128;
    const int k0 = z * P.per;
    const int k1 = spare ? k0 : min(P.ksteps, k0 + P.per);
    const int nk = k1 > k0 ? k1 - k0 : 0;
    const int rows_per = 128 / cs;  // tile rows owned by each rank
    const int rc = (P.r + 3) & ~3;  // columns sent per row

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(red_full, 1);
        // every rank (this one included) sends rows_per rows of rc floats here
        mbar_arrive_expect_tx(red_full, (uint32_t)(cs * rows_per * rc * 4));
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&P.tmA);
        prefetch_tensormap(&P.tmB);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), BN < 32 ? 32 : BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // First cluster barrier: every CTA's red_full is initialized (waited on
    // before the first remote store).  With RED_OVERLAY it also marks the
    // end of every CTA's pipeline, so it is arrived at after the main loop.
    if (!S::RED_OVERLAY) cluster_arrive();

    // ---------------------------------------------------------------- k-range pipeline
    if (warp == 0) {
        // Operands from the previous kernel: wait for it first.  The next
        // kernel may start once this one has passed that point (it may read
        // inputs that this kernel's predecessors wrote).
        if (lane == 0) {
            if (p.wait_first) pdl_wait();
            pdl_trigger();
        }
        if (lane == 0 && !p.inject) {
            int last_use[STAGES];
            for (int s = 0; s < STAGES; ++s) last_use[s] = -1;
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES, u = i / STAGES;
                if (!mbar_wait(empty(s), (u & 1) ^ 1, wc)) { *abort_flag = 1; break; }
                const int k = k0 + i;
                const uint32_t sA = base + s * S::STAGE_BYTES;
                const uint32_t sB = sA + S::A_BYTES;
                mbar_arrive_expect_tx(full(s), S::A_BYTES + S::B_BYTES);
                if (a_mn) {
                    tma_load_2d(sA, &P.tmA, full(s), m0, k * 64);
                    tma_load_2d(sA + 8192, &P.tmA, full(s), m0 + 64, k * 64);
                } else {
                    tma_load_2d(sA, &P.tmA, full(s), k * 64, m0);
                }
                if (b_mn) {
                    for (int c = 0; c < BN / 64; ++c)
                        tma_load_2d(sB + 8192 * c, &P.tmB, full(s), 64 * c + skinny_b_col0(P, k, m0), k * 64);
                } else {
                    tma_load_2d(sB, &P.tmB, full(s), k * 64, 0);
                }
                last_use[s] = u;
            }
            // every load has landed before the buffers are reused or the CTA exits
            for (int s = 0; s < STAGES; ++s)
                if (last_use[s] >= 0) mbar_wait(full(s), last_use[s] & 1, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, BN, a_mn, b_mn);
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES, u = i / STAGES;
                if (!mbar_wait(full(s), u & 1, wc)) { *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t sA = base + s * S::STAGE_BYTES;
                const uint32_t sB = sA + S::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = a_mn ? smem_desc_sw128(sA + kk * 2048, 8192, 1024)
                                             : smem_desc_sw128(sA + kk * 32, 16, 1024);
                    const uint64_t bd = b_mn ? smem_desc_sw128(sB + kk * 2048, 8192, 1024)
                                             : smem_desc_sw128(sB + kk * 32, 16, 1024);
                    umma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(empty(s));
            }
            umma_commit(acc_full);
            // the MMAs (and their reads of shared memory) are complete before
            // the buffers are reused or the CTA exits
            mbar_wait(acc_full, 0, wc);
        }
    }

    if (warp < 2) {
        // producer and MMA warps: nothing left but the two cluster barriers
        if (S::RED_OVERLAY) cluster_arrive();
        cluster_wait();
        cluster_arrive();
        cluster_wait();
    } else {
        // ------------------------------------------------------------ send partial rows to their owners
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // tile row = TMEM lane of this thread
        const bool ok = mbar_wait(acc_full, 0, wc);
        if (ok) tc_fence_after();
        const bool skip = __any_sync(0xffffffffu, !ok || *abort_flag != 0 || nk == 0);
        if (S::RED_OVERLAY) cluster_arrive();
        cluster_wait();
        const int owner = row / rows_per;
        const int orow = row - owner * rows_per;
        const uint32_t dst =
            mapa_shared(red_base + (uint32_t)((z * rows_per + orow) * S::PART_LD) * 4u, (uint32_t)owner + self_rank);
        const uint32_t dst_bar = mapa_shared(red_full, (uint32_t)owner + self_rank);
#pragma unroll 1
        for (int c0 = 0; c0 < BN && c0 < rc; c0 += 64) {
            uint32_t v0[32], v1[32];
            if (!skip) {
                __syncwarp();
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, v0);
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(c0 + 32), v1);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) v0[q] = v1[q] = 0u;
            }
#pragma unroll
            for (int q = 0; q < 32; q += 4)
                if (c0 + q < rc) st_async_v4(dst + (uint32_t)(c0 + q) * 4u, v0[q], v0[q + 1], v0[q + 2], v0[q + 3], dst_bar);
#pragma unroll
            for (int q = 0; q < 32; q += 4)
                if (c0 + 32 + q < rc)
                    st_async_v4(dst + (uint32_t)(c0 + 32 + q) * 4u, v1[q], v1[q + 1], v1[q + 2], v1[q + 3], dst_bar);
        }
        // second cluster barrier (waited on before exit): no CTA leaves
        // while another may still send to it
        cluster_arrive();

        // ------------------------------------------------------------ fixed-order reduction of the owned rows
        const bool got = mbar_wait(red_full, 0, wc);
        const int t = threadIdx.x - 64;  // 0..127
        const int r0 = z * rows_per;
        const int nrows = got ? max(0, min(rows_per, min(128, P.rows - m0) - r0)) : 0;
        const float* red = reinterpret_cast<const float*>(gbase + S::RED_OFF);
        constexpr int LD = S::PART_LD;
        if (P.out_mode == SK_OUT_F32_T) {
            // out[j][m0 + r0 + rr]: consecutive threads take consecutive rows
            float* out = static_cast<float*>(P.out);
            for (int e = t; e < nrows * P.r; e += 128) {
                const int j = e / nrows, rr = e - j * nrows;
                float acc = red[rr * LD + j];
                for (int zz = 1; zz < cs; ++zz) acc = __fadd_rn(acc, red[(zz * rows_per + rr) * LD + j]);
                out[(int64_t)j * P.out_ld + m0 + r0 + rr] = __fmul_rn(acc, P.scale);
            }
        } else {
            // four consecutive columns per thread (r % 8 == 0)
            const int r4 = P.r >> 2;
            for (int e = t; e < nrows * r4; e += 128) {
                const int rr = e / r4, j = (e - rr * r4) * 4;
                float4 acc = *reinterpret_cast<const float4*>(&red[rr * LD + j]);
                for (int zz = 1; zz < cs; ++zz) {
                    const float4 b = *reinterpret_cast<const float4*>(&red[(zz * rows_per + rr) * LD + j]);
                    acc.x = __fadd_rn(acc.x, b.x);
                    acc.y = __fadd_rn(acc.y, b.y);
                    acc.z = __fadd_rn(acc.z, b.z);
                    acc.w = __fadd_rn(acc.w, b.w);
                }
                acc.x = __fmul_rn(acc.x, P.scale);
                acc.y = __fmul_rn(acc.y, P.scale);
                acc.z = __fmul_rn(acc.z, P.scale);
                acc.w = __fmul_rn(acc.w, P.scale);
                const int64_t o = (int64_t)(m0 + r0 + rr) * P.out_ld + j;
                if (P.out_mode == SK_OUT_F32) {
                    *reinterpret_cast<float4*>(static_cast<float*>(P.out) + o) = acc;
                } else {
                    uint2 h;
                    h.x = pack_bf16x2(acc.x, acc.y);
                    h.y = pack_bf16x2(acc.z, acc.w);
                    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(P.out) + o) = h;
                }
            }
        }
        cluster_wait();
    }
    // the kernel does not complete before the previous one (its dependents
    // may rely on both)
    if (threadIdx.x == 0) pdl_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, BN < 32 ? 32 : BN);
    }
}


// ---------------------------------------------------------------------------
// Persistent LoRA GEMMs for work that runs beside another kernel (the dA, dB
// and sU GEMMs of the backward, next to the dX GEMM): each CTA takes tiles
// blockIdx.x, blockIdx.x + gridDim.x, ... of the one or two problems and
// reduces each 128-row tile alone over the whole k range.  One TMA ring runs
// through all of a CTA's tiles; the accumulator is double-buffered in TMEM,
// so a tile's epilogue (TMEM -> registers -> global) overlaps the next
// tile's loads and MMAs.  Same operands, layouts and output modes as
// k_skinny; per tile the result equals k_skinny's with a cluster of 1.
// ---------------------------------------------------------------------------
template <int BN>
struct StreamShape {
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = BN <= 64 ? 8 : (BN <= 128 ? 6 : 4);
    // stages are released in groups of CG k-steps: one tcgen05.commit per
    // group (a commit costs about as much as the small MMAs it follows)
    static constexpr int CG = 2;
    static_assert(STAGES % CG == 0, "the ring holds whole commit groups");
    static constexpr int PIPE_BYTES = STAGE_BYTES * STAGES;
    static constexpr int SMEM = PIPE_BYTES + 1024 + 512;
    static constexpr int THREADS = 32 * 6;  // producer, MMA, 4 epilogue warps
    static constexpr int TMEM_COLS = 2 * BN;
};

template <int BN>
__global__ void __launch_bounds__(StreamShape<BN>::THREADS, 1) k_lora_stream(const __grid_constant__ SkinnyParams p) {
    using S = StreamShape<BN>;
    constexpr int STAGES = S::STAGES;
    constexpr int RING = 4;  // tile indices handed from the producer to the MMA and epilogue warps
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw_base);
    const uint32_t bar_base = base + S::PIPE_BYTES;
    auto full = [&](int s) { return bar_base + 8u * s; };
    auto empty = [&](int s) { return bar_base + 8u * (STAGES + s); };
    auto acc_full = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
    auto acc_empty = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };
    auto tile_full = [&](int j) { return bar_base + 8u * (2 * STAGES + 4 + j); };
    auto tile_empty = [&](int j) { return bar_base + 8u * (2 * STAGES + 4 + RING + j); };
    int* ring = reinterpret_cast<int*>(gbase + S::PIPE_BYTES + 8 * (2 * STAGES + 4 + 2 * RING));
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ring + RING);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WaitCfg wc{p.timeout_ns};
    const int total = p.total_tiles;
    // tile t of the launch -> problem and 128-row tile within it
    auto locate = [&](int t, int& pi, int& tile) {
        pi = 0;
        tile = t;
        while (pi + 1 < p.nprob && tile >= p.pr[pi].tiles) {
            tile -= p.pr[pi].tiles;
            ++pi;
        }
    };
    // tile index of local tile li (all roles), -1 past the end
    auto take_tile = [&](int li, bool& ok) -> int {
        const int j = li % RING, u = li / RING;
        if (!mbar_wait(tile_full(j), u & 1, wc)) {
            ok = false;
            return -1;
        }
        return *reinterpret_cast<volatile int*>(ring + j);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), 4);  // one arrive per epilogue warp
        }
        for (int j = 0; j < RING; ++j) {
            mbar_init(tile_full(j), 1);
            mbar_init(tile_empty(j), 5);  // MMA thread + 4 epilogue warps
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < p.nprob; ++i) {
            prefetch_tensormap(&p.pr[i].tmA);
            prefetch_tensormap(&p.pr[i].tmB);
        }
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), S::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            if (p.wait_first) pdl_wait();
            pdl_trigger();
        }
        if (lane == 0) {
            int last_use[STAGES];
            for (int s = 0; s < STAGES; ++s) last_use[s] = -1;
            int it = 0;
            bool ok = true, dep_ready = p.dep_prob < 0, prev_done = p.wait_first != 0;
            for (int li = 0;; ++li) {
                const int j = li % RING, u = li / RING;
                // the slot's previous tile index has been read by every role
                if (!mbar_wait(tile_empty(j), (u & 1) ^ 1, wc)) { *abort_flag = 1; ok = false; }
                int t = -1;
                if (ok) t = p.tile_ctr ? atomicAdd(p.tile_ctr, 1) : (int)blockIdx.x + li * (int)gridDim.x;
                if (t >= total) t = -1;
                ring[j] = t;
                mbar_arrive(tile_full(j));
                if (t < 0) break;
                int pi, tile;
                locate(t, pi, tile);
                const SkinnyProblem& P = p.pr[pi];
                if (!prev_done && ((p.wait_mask >> pi) & 1)) {
                    pdl_wait();
                    prev_done = true;
                }
                if (pi == p.dep_prob && !dep_ready) {
                    // problem 0's output (read through TMA) is complete
                    const int target = 4 * p.pr[0].tiles;
                    const uint64_t t_start = globaltimer_ns();
                    while (ld_acquire_gpu(p.done_ctr) < target) {
                        __nanosleep(256);
                        if (globaltimer_ns() - t_start > p.timeout_ns) {
                            set_status(4);
                            *abort_flag = 1;
                            break;
                        }
                    }
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    dep_ready = true;
                }
                if (p.inject || *abort_flag) continue;  // loads skipped: the waits below run out
                const int m0 = tile * 128;
                for (int k = 0; k < P.ksteps; ++k, ++it) {
                    const int s = it % STAGES, us = it / STAGES;
                    // the stage's previous k-step (it - STAGES) is in commit group
                    // it / CG - STAGES / CG, released on the same group barrier
                    const int gi = it / S::CG;
                    if (!mbar_wait(empty(gi % (STAGES / S::CG)), ((gi / (STAGES / S::CG)) & 1) ^ 1, wc)) {
                        *abort_flag = 1;
                        break;
                    }
                    const uint32_t sA = base + s * S::STAGE_BYTES;
                    const uint32_t sB = sA + S::A_BYTES;
                    mbar_arrive_expect_tx(full(s), S::A_BYTES + S::B_BYTES);
                    if (P.a_mn) {
                        tma_load_2d(sA, &P.tmA, full(s), m0, k * 64);
                        tma_load_2d(sA + 8192, &P.tmA, full(s), m0 + 64, k * 64);
                    } else {
                        tma_load_2d(sA, &P.tmA, full(s), k * 64, m0);
                    }
                    if (P.b_mn) {
                        for (int c = 0; c < BN / 64; ++c)
                            tma_load_2d(sB + 8192 * c, &P.tmB, full(s), 64 * c + skinny_b_col0(P, k, m0), k * 64);
                    } else {
                        tma_load_2d(sB, &P.tmB, full(s), k * 64, 0);
                    }
                    last_use[s] = us;
                }
            }
            // every load has landed before the CTA exits
            for (int s = 0; s < STAGES; ++s)
                if (last_use[s] >= 0) mbar_wait(full(s), last_use[s] & 1, wc);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0, last_buf = -1, last_use = 0;
            bool ok = true;
            for (int li = 0;; ++li) {
                const int t = take_tile(li, ok);
                mbar_arrive(tile_empty(li % RING));
                if (t < 0 || !ok) break;
                int pi, tile;
                locate(t, pi, tile);
                const SkinnyProblem& P = p.pr[pi];
                const int buf = li & 1, use = li >> 1;
                if (!mbar_wait(acc_empty(buf), (use & 1) ^ 1, wc)) { *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(buf * BN);
                const uint32_t idesc = idesc_bf16_f32(128, BN, P.a_mn, P.b_mn);
                for (int k = 0; ok && k < P.ksteps; ++k, ++it) {
                    const int s = it % STAGES, us = it / STAGES;
                    if (!mbar_wait(full(s), us & 1, wc)) { *abort_flag = 1; ok = false; break; }
                    tc_fence_after();
                    const uint32_t sA = base + s * S::STAGE_BYTES;
                    const uint32_t sB = sA + S::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = P.a_mn ? smem_desc_sw128(sA + kk * 2048, 8192, 1024)
                                                   : smem_desc_sw128(sA + kk * 32, 16, 1024);
                        const uint64_t bd = P.b_mn ? smem_desc_sw128(sB + kk * 2048, 8192, 1024)
                                                   : smem_desc_sw128(sB + kk * 32, 16, 1024);
                        umma_bf16(acc, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
                    }
                    if (it % S::CG == S::CG - 1) umma_commit(empty((it / S::CG) % (STAGES / S::CG)));
                }
                // committed also after an abort, so that the wait below covers
                // every MMA issued
                umma_commit(acc_full(buf));
                last_buf = buf;
                last_use = use;
                if (!ok) break;
            }
            // the MMAs (and their reads of shared memory) are complete before the CTA exits
            if (last_buf >= 0) mbar_wait(acc_full(last_buf), last_use & 1, wc);
        }
    } else {
        // ------------------------------------------------------------ epilogue: one row per thread
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        bool ok = true;
        for (int li = 0;; ++li) {
            const int t = take_tile(li, ok);
            __syncwarp();
            if (lane == 0) mbar_arrive(tile_empty(li % RING));
            if (__any_sync(0xffffffffu, t < 0 || !ok)) break;
            int pi, tile;
            locate(t, pi, tile);
            const SkinnyProblem& P = p.pr[pi];
            const int buf = li & 1, use = li >> 1;
            const bool got = mbar_wait(acc_full(buf), use & 1, wc);
            if (__any_sync(0xffffffffu, !got || *abort_flag != 0)) break;
            tc_fence_after();
            const int m = tile * 128 + row;
            const bool live = m < P.rows;
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
#pragma unroll 1
            for (int c0 = 0; c0 < BN && c0 < P.r; c0 += 32) {
                uint32_t v[32];
                __syncwarp();
                tmem_ld_32x32b_x32(taddr + (uint32_t)c0, v);
                tmem_ld_wait();
                if (!live) continue;
                if (P.out_mode == SK_OUT_F32_T) {
                    float* out = static_cast<float*>(P.out);
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        if (c0 + q < P.r)
                            out[(int64_t)(c0 + q) * P.out_ld + m] = __fmul_rn(__uint_as_float(v[q]), P.scale);
                } else if (P.out_mode == SK_OUT_F32) {
                    float* out = static_cast<float*>(P.out) + (int64_t)m * P.out_ld;
#pragma unroll
                    for (int q = 0; q < 32; q += 4)
                        if (c0 + q < P.r)
                            *reinterpret_cast<float4*>(out + c0 + q) =
                                make_float4(__fmul_rn(__uint_as_float(v[q]), P.scale),
                                            __fmul_rn(__uint_as_float(v[q + 1]), P.scale),
                                            __fmul_rn(__uint_as_float(v[q + 2]), P.scale),
                                            __fmul_rn(__uint_as_float(v[q + 3]), P.scale));
                } else {
                    uint16_t* out = static_cast<uint16_t*>(P.out) + (int64_t)m * P.out_ld;
#pragma unroll
                    for (int q = 0; q < 32; q += 8)
                        if (c0 + q < P.r) {
                            uint4 h;
                            h.x = pack_bf16x2(__fmul_rn(__uint_as_float(v[q]), P.scale),
                                              __fmul_rn(__uint_as_float(v[q + 1]), P.scale));
                            h.y = pack_bf16x2(__fmul_rn(__uint_as_float(v[q + 2]), P.scale),
                                              __fmul_rn(__uint_as_float(v[q + 3]), P.scale));
                            h.z = pack_bf16x2(__fmul_rn(__uint_as_float(v[q + 4]), P.scale),
                                              __fmul_rn(__uint_as_float(v[q + 5]), P.scale));
                            h.w = pack_bf16x2(__fmul_rn(__uint_as_float(v[q + 6]), P.scale),
                                              __fmul_rn(__uint_as_float(v[q + 7]), P.scale));
                            *reinterpret_cast<uint4*>(out + c0 + q) = h;
                        }
                }
            }
            // this warp has read its rows of the buffer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(acc_empty(buf));
                if (pi == 0 && p.done_ctr) {
                    // the warp's rows of a problem-0 tile are in global memory
                    __threadfence();
                    atomicAdd(p.done_ctr, 1);
                }
            }
        }
    }
    // the kernel does not complete before the previous one
    if (threadIdx.x == 0) pdl_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, S::TMEM_COLS);
    }
}

}  // namespace qlora
