// skinny.cuh -- the rank-r LoRA GEMMs (U = X A^T, G = dY B, dA = G^T X,
// dB = dY^T U): a tall operand times an r-column operand, r <= 256.
//
// out[i][j] = scale * sum_k Aop[i][k] * Bop[j][k]   (i < rows, j < r)
// They are HBM-bound (each streams X or dY once), so the reduction dimension
// is split across the CS CTAs of a thread-block cluster: each CTA runs a TMA
// -> tcgen05 pipeline over its k-range into TMEM, parks its fp32 partial tile
// in its own shared memory, and after a cluster barrier CTA z sums rows
// [z*128/CS, (z+1)*128/CS) of all CS partials over distributed shared memory
// in a fixed order (deterministic) and writes the final output directly.
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace qlora {

enum { SK_OUT_BF16 = 0, SK_OUT_F32 = 1, SK_OUT_F32_T = 2 };

struct SkinnyParams {
    CUtensorMap tmA, tmB;
    int rows, r;          // output extent
    int ksteps;           // 64-wide k-steps of the whole reduction
    int per;              // k-steps per cluster rank
    float scale;
    int out_mode;
    void* out;
    int64_t out_ld;       // elements
    uint64_t timeout_ns;
    int inject;
};

template <int BN>
struct SkinnyShape {
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int PART_LD = BN + 4;  // fp32 partial row pitch (floats), breaks bank aliasing
    static constexpr int PART_BYTES = 128 * PART_LD * 4;
    static constexpr int THREADS = 32 * 6;  // producer, MMA, 4 epilogue warps
};

template <int BN, int STAGES>
constexpr int skinny_smem_bytes() {
    constexpr int pipe = SkinnyShape<BN>::STAGE_BYTES * STAGES;
    constexpr int part = SkinnyShape<BN>::PART_BYTES;
    return (pipe > part ? pipe : part) + 1024 + 256;
}

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

// Sum of the fp32 at local offset `off` over CTAs 0..cs-1 of the cluster, in
// rank order (all loads issued before the ordered additions).
__device__ __forceinline__ float cluster_sum(uint32_t off, uint32_t cs) {
    float v[8];
#pragma unroll
    for (int zz = 0; zz < 8; ++zz) v[zz] = zz < (int)cs ? ld_shared_cluster_f32(mapa_shared(off, zz)) : 0.0f;
    float acc = v[0];
#pragma unroll
    for (int zz = 1; zz < 8; ++zz)
        if (zz < (int)cs) acc = __fadd_rn(acc, v[zz]);
    return acc;
}

template <int BN, int A_MN, int B_MN, int STAGES>
__global__ void __launch_bounds__(SkinnyShape<BN>::THREADS, 1) k_skinny(const __grid_constant__ SkinnyParams p) {
    using S = SkinnyShape<BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw_base);
    constexpr int REGION = S::STAGE_BYTES * STAGES > S::PART_BYTES ? S::STAGE_BYTES * STAGES : S::PART_BYTES;
    const uint32_t bar_base = base + REGION;
    auto full = [&](int s) { return bar_base + 8u * s; };
    auto empty = [&](int s) { return bar_base + 8u * (STAGES + s); };
    const uint32_t acc_full = bar_base + 8u * (2 * STAGES);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + REGION + 8 * (2 * STAGES + 1));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WaitCfg wc{p.timeout_ns};
    const uint32_t cs = cluster_nctarank();
    const uint32_t z = cluster_ctarank();
    const int tile = blockIdx.x / (int)cs;
    const int m0 = tile * 128;
    const int k0 = (int)z * p.per;
    const int k1 = min(p.ksteps, k0 + p.per);
    const int nk = k1 > k0 ? k1 - k0 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&p.tmA);
        prefetch_tensormap(&p.tmB);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), BN < 32 ? 32 : BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
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
                if (A_MN) {
                    tma_load_2d(sA, &p.tmA, full(s), m0, k * 64);
                    tma_load_2d(sA + 8192, &p.tmA, full(s), m0 + 64, k * 64);
                } else {
                    tma_load_2d(sA, &p.tmA, full(s), k * 64, m0);
                }
                if (B_MN) {
                    for (int c = 0; c < BN / 64; ++c) tma_load_2d(sB + 8192 * c, &p.tmB, full(s), 64 * c, k * 64);
                } else {
                    tma_load_2d(sB, &p.tmB, full(s), k * 64, 0);
                }
                last_use[s] = u;
            }
            for (int s = 0; s < STAGES; ++s)
                if (last_use[s] >= 0) mbar_wait(full(s), last_use[s] & 1, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, BN, A_MN, B_MN);
            bool ok = true;
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES, u = i / STAGES;
                if (!mbar_wait(full(s), u & 1, wc)) { ok = false; *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t sA = base + s * S::STAGE_BYTES;
                const uint32_t sB = sA + S::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = A_MN ? smem_desc_sw128(sA + kk * 2048, 8192, 1024)
                                             : smem_desc_sw128(sA + kk * 32, 16, 1024);
                    const uint64_t bd = B_MN ? smem_desc_sw128(sB + kk * 2048, 8192, 1024)
                                             : smem_desc_sw128(sB + kk * 32, 16, 1024);
                    umma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(empty(s));
            }
            umma_commit(acc_full);
            if (!ok) mbar_wait(acc_full, 0, wc);
        }
    } else {
        // ---------------------------------------------------------------- partial tile -> own smem
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const bool ok = mbar_wait(acc_full, 0, wc);
        if (ok) tc_fence_after();
        const bool skip = __any_sync(0xffffffffu, !ok || *abort_flag != 0 || nk == 0);
        float* part = reinterpret_cast<float*>(gbase);
        for (int c0 = 0; c0 < BN; c0 += 32) {
            uint32_t v[32];
            if (!skip) {
                __syncwarp();
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, v);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] = 0u;
            }
#pragma unroll
            for (int q = 0; q < 32; q += 4)
                *reinterpret_cast<uint4*>(part + row * S::PART_LD + c0 + q) =
                    make_uint4(v[q], v[q + 1], v[q + 2], v[q + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // every CTA's partial tile is in its shared memory

    // ---------------------------------------------------------------- fixed-order cluster reduction
    if (warp >= 2) {
        const int t = threadIdx.x - 64;  // 0..127
        const int rows_per = 128 / (int)cs;
        const int r0 = (int)z * rows_per;
        const uint32_t part_base = base;
        if (p.out_mode == SK_OUT_F32_T) {
            // out[j][m0 + row]: consecutive threads take consecutive rows
            for (int e = t; e < rows_per * p.r; e += 128) {
                const int j = e / rows_per, rr = r0 + e % rows_per;
                if (m0 + rr >= p.rows) continue;
                const float acc = cluster_sum(part_base + (uint32_t)(rr * S::PART_LD + j) * 4u, cs);
                static_cast<float*>(p.out)[(int64_t)j * p.out_ld + m0 + rr] = __fmul_rn(acc, p.scale);
            }
        } else {
            for (int e = t; e < rows_per * p.r; e += 128) {
                const int rr = r0 + e / p.r, j = e % p.r;
                if (m0 + rr >= p.rows) continue;
                const float acc = __fmul_rn(cluster_sum(part_base + (uint32_t)(rr * S::PART_LD + j) * 4u, cs), p.scale);
                if (p.out_mode == SK_OUT_F32) {
                    static_cast<float*>(p.out)[(int64_t)(m0 + rr) * p.out_ld + j] = acc;
                } else {
                    const uint32_t h = pack_bf16x2(acc, 0.0f) & 0xFFFFu;
                    static_cast<uint16_t*>(p.out)[(int64_t)(m0 + rr) * p.out_ld + j] = (uint16_t)h;
                }
            }
        }
    }
    cluster_sync();  // no CTA leaves while a peer may still read its partial
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, BN < 32 ? 32 : BN);
    }
}

}  // namespace qlora
