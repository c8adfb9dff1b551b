// merge.cuh -- LoRA merge and unmerge on the dequantized frozen weight.
//
// Merge (QLoRA tutorial "11.3 QLoRA", pitfalls: merging into the 4-bit base
// adds error, so the base is dequantized first; LoRA reproduction blog,
// "LoRA formula and tensor shapes": the adapter's update of W0 is
// (alpha/r) B A):
//     W_merged[n][k] = bf16_rne( w'[n][k] + s * sum_j B[n][j] A[j][k] )
// with w' the doubleDequant weight (the bf16 values the fused linear feeds
// its tensor cores).  Unmerge subtracts the same update from a dense bf16
// weight:  W[n][k] = bf16_rne( W_merged[n][k] - s * sum_j B[n][j] A[j][k] ).
//
// One CTA per 128 x 128 output tile.  The rank-r product is one tcgen05 MMA
// chain (M = 128 rows of B, N = 128 columns of A, K = r in steps of 16) into
// TMEM: B [N][r] is the K-major A operand, A [r][K] the MN-major B operand,
// both brought by TMA with the 128-byte swizzle.  The four warps then read
// their 32 rows of the fp32 product, rebuild the exact bf16 base values of
// the same elements (NF4 codes expanded with the per-block byte tables, or
// the dense bf16 input), form fma(s, product, base) in fp32, round once to
// bf16 and store.  The base is read and the output written once: the kernel
// is bound by those HBM bytes (0.52 B read + 2 B written per element for an
// NF4 base with double quantization).
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

struct MergeParams {
    CUtensorMap tmB;          // B [N][r] bf16, box {64, 128}, 128-byte swizzle
    CUtensorMap tmA;          // A [r][K] bf16, box {64, 64}, 128-byte swizzle
    const uint8_t* codes;     // NF4 base (merge)
    const float* absmax;      // without double quantization
    const uint8_t* q8;
    const float* c1;
    const float* offset;
    int dq;
    const uint16_t* dense;    // dense bf16 base [N][K] (unmerge); null for an NF4 base
    uint16_t* out;            // bf16 [N][K]
    int N, K, r_chunks;       // r_chunks = ceil(r / 64)
    QFormat fmt;              // code book, 8-bit code book, block size of the NF4 base
    float scale;              // +s (merge) or -s (unmerge)
    uint64_t timeout_ns;
};

struct MergeShape {
    static constexpr int CHUNK_BYTES = 32768;  // per 64 of r: B tile 16 KB + A tile 16 KB
    static constexpr int THREADS = 128;
    static constexpr int TMEM_COLS = 128;
    static constexpr int smem(int r_chunks) { return 1024 + r_chunks * CHUNK_BYTES + 64; }
    static constexpr int MAX_SMEM = 1024 + 4 * CHUNK_BYTES + 64;  // r <= 256
};

__global__ void __launch_bounds__(MergeShape::THREADS) k_lora_merge(const __grid_constant__ MergeParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw_base);
    const int rc = p.r_chunks;
    const uint32_t bar_full = base + (uint32_t)(rc * MergeShape::CHUNK_BYTES);
    const uint32_t bar_acc = bar_full + 8;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + rc * MergeShape::CHUNK_BYTES + 16);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.y * 128, k0 = blockIdx.x * 128;
    const WaitCfg wc{p.timeout_ns};

    if (threadIdx.x == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_acc, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&p.tmA);
        prefetch_tensormap(&p.tmB);
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_holder), MergeShape::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar_full, (uint32_t)(rc * MergeShape::CHUNK_BYTES));
        for (int c = 0; c < rc; ++c) {
            const uint32_t sB = base + (uint32_t)(c * MergeShape::CHUNK_BYTES);
            const uint32_t sA = sB + 16384;
            tma_load_2d(sB, &p.tmB, bar_full, c * 64, n0);
            tma_load_2d(sA, &p.tmA, bar_full, k0, c * 64);
            tma_load_2d(sA + 8192, &p.tmA, bar_full, k0 + 64, c * 64);
        }
        if (mbar_wait(bar_full, 0, wc)) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 1);
            for (int c = 0; c < rc; ++c) {
                const uint32_t sB = base + (uint32_t)(c * MergeShape::CHUNK_BYTES);
                const uint32_t sA = sB + 16384;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem, smem_desc_sw128(sB + kk * 32, 16, 1024),
                              smem_desc_sw128(sA + kk * 2048, 8192, 1024), idesc, (c | kk) ? 1u : 0u);
            }
            umma_commit(bar_acc);
        } else {
            // the loads never landed: let the epilogue warps go (they write
            // nothing), after every copy in flight has ended (bounded)
            *abort_flag = 1;
            mbar_wait(bar_full, 0, wc);
            mbar_arrive(bar_acc);
        }
    }

    const int row = warp * 32 + lane;  // TMEM lane = output row of this thread
    const int n = n0 + row;
    const bool row_ok = n < p.N;
    // base values of this row's 128 columns, fetched while the MMAs run
    uint4 cw[4];      // NF4 codes: 64 bytes = 128 elements
    float a_blk[2];   // block constants of the row's two 64-element blocks
    const int kbs = p.K / 64;
    if (row_ok && !p.dense) {
        const uint8_t* crow = p.codes + ((int64_t)n * p.K + k0) / 2;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            cw[i] = (k0 + 32 * i < p.K) ? __ldg(reinterpret_cast<const uint4*>(crow) + i) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int kb = k0 / 64 + h;
            float a = 0.0f;
            if (kb < kbs) {
                const int64_t b = ((int64_t)n * kbs + kb) >> p.fmt.bs_shift;
                a = p.dq ? block_scale_dq(__ldg(p.q8 + b), __ldg(p.c1 + (b >> 8)), __ldg(p.offset), p.fmt.dq_type)
                         : __ldg(p.absmax + b);
            }
            a_blk[h] = a;
        }
    }
    const bool got = mbar_wait_sleep(bar_acc, 0, wc, 256) && !*abort_flag;
    tc_fence_after();
    if (got) {
        Nf4BlockTable tb[2];
        if (!p.dense) {
            tb[0] = nf4_block_table(a_blk[0], p.fmt.code_type);
            tb[1] = nf4_block_table(a_blk[1], p.fmt.code_type);
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            uint32_t v[32];
            __syncwarp();
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(cc * 32), v);
            tmem_ld_wait();
            const int kc = k0 + cc * 32;
            if (!row_ok || kc >= p.K) continue;
            uint32_t wb[16];  // 32 bf16 base values, element 2j in the low half of wb[j]
            if (p.dense) {
                const uint4* src = reinterpret_cast<const uint4*>(p.dense + (int64_t)n * p.K + kc);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 u = __ldg(src + i);
                    wb[4 * i] = u.x;
                    wb[4 * i + 1] = u.y;
                    wb[4 * i + 2] = u.z;
                    wb[4 * i + 3] = u.w;
                }
            } else {
                const uint4 c = cw[cc];
                const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t o[4];
                    nf4_expand_word(words[i], tb[cc >> 1], o);
                    wb[4 * i] = o[0];
                    wb[4 * i + 1] = o[1];
                    wb[4 * i + 2] = o[2];
                    wb[4 * i + 3] = o[3];
                }
            }
            uint32_t res[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float lo = __uint_as_float(wb[j] << 16), hi = __uint_as_float(wb[j] & 0xFFFF0000u);
                res[j] = pack_bf16x2(__fmaf_rn(p.scale, __uint_as_float(v[2 * j]), lo),
                                     __fmaf_rn(p.scale, __uint_as_float(v[2 * j + 1]), hi));
            }
            uint4* dst = reinterpret_cast<uint4*>(p.out + (int64_t)n * p.K + kc);
            if (QLORA_CHECK(n < p.N && kc + 32 <= p.K))
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    __stcs(dst + i, make_uint4(res[4 * i], res[4 * i + 1], res[4 * i + 2], res[4 * i + 3]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, MergeShape::TMEM_COLS);
    }
}

}  // namespace qlora
