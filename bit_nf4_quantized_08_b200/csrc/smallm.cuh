// smallm.cuh -- the forward dequant GEMM for few tokens (M <= 64: decoding
// and small batches), where the frozen weight is streamed once and the NF4
// expansion, not the tensor core, sets the pace.
//
//   Y^T [N x M] = W' [N x K] X^T  +  B [N x r] sU^T,   sU = bf16(s X A^T)
//
// Swap-AB: 128 weight rows on the MMA's M side, the tokens on N = NT (16, 32
// or 64).  The work is the list of (row tile, k-step) units, tiles x KS with
// KS = K/64 + ceil(r/64); a persistent grid of one CTA per SM takes
// contiguous shares of it (stream-K), so every SM streams the same number of
// weight bytes whatever the tile count.  A tile cut between CTAs is finished
// by the CTA that holds its first k-steps (the owner): the other CTAs publish
// fp32 partial tiles (NT x 128) with a per-launch epoch in a flag, and the
// owner adds them in CTA order (deterministic) and clears the flag.
//
// Roles (one CTA): warp 0 issues the TMA loads (NF4 codes, X or the LoRA
// operands), warp 1 the MMAs, warps 2-5 drain the accumulators (double
// buffered in TMEM, so a tile's epilogue overlaps the next tile's MMAs), and
// NG groups of four dequant warps expand the NF4 codes of alternate k-steps
// into bf16 (one thread per weight row).  The block constant a' of every
// (row, k-step) comes straight from the 8-bit codes (t8[q8] * c1 + offset,
// the doubleDequant of the QLoRA digest, sec. 4), prefetched two visits
// ahead, so no expanded scale array is read.
#pragma once

#include "common.cuh"
#include "gemm.cuh"
#include "nf4.cuh"

namespace qlora {

struct SmallMParams {
    CUtensorMap tmCodes;  // codes [N][K/2] bytes, box {32 B, 128 rows}, 32-byte swizzle
    CUtensorMap tmX;      // X [M][K] bf16, box {64, NT}, 128-byte swizzle
    CUtensorMap tmB;      // B [N][r] bf16, box {64, 128}, 128-byte swizzle
    CUtensorMap tmU;      // sU [M][r] bf16, box {64, NT}, 128-byte swizzle
    const uint8_t* q8;
    const float* c1;
    const float* offset;
    const float* absmax;  // without double quantization
    int dq;
    int N, M, kbs;        // kbs = K / 64
    int ks_main, ks_lora, tiles;
    int seg_rows, seg_r;  // fused projection: sU columns of tile t start at (128 t / seg_rows) seg_r
    QFormat fmt;          // code book, 8-bit code book, block size
    uint16_t* Y;          // [M][N] bf16
    float* part;          // [gridDim.x][NT][128] fp32 partial tiles
    uint32_t* flags;      // [gridDim.x][4] epoch of the published partial, per TMEM quarter
    int64_t part_cap, flag_cap;  // capacities (floats, words): bounds checks of the debug build
    uint32_t epoch;
    uint64_t timeout_ns;
    int inject;
};

template <int NT, int NG>
struct SmallMShape {
    // Two rings: TMA stages (X or sU tile + NF4 codes of one k-step, deep, to
    // keep enough weight bytes in flight per SM) and A slots (the 128 x 64
    // bf16 operand the dequant warps write, or the LoRA B tile).
    static constexpr int A_BYTES = 128 * 128;   // 128 rows x 64 k bf16
    static constexpr int A_SLOTS = 4;
    static constexpr int X_BYTES = NT * 128;    // NT rows x 64 k bf16 (multiple of 1024)
    static constexpr int CODE_BYTES = 128 * 32;
    static constexpr int T_BYTES = X_BYTES + CODE_BYTES;
    static constexpr int T_STAGES = NT >= 64 ? 10 : 16;
    static constexpr int T_OFF = A_BYTES * A_SLOTS;
    static constexpr int T8_OFF = T_OFF + T_BYTES * T_STAGES;  // fp32 t8 table [256]
    static constexpr int BAR_OFF = T8_OFF + 1024;
    static constexpr int SMEM = BAR_OFF + 512 + 1024;
    static constexpr int ACC_COLS = NT < 32 ? 32 : NT;  // one TMEM accumulator
    static constexpr int TMEM_COLS = 2 * ACC_COLS;
    static constexpr int FIRST_DQ_WARP = 6;
    static constexpr int THREADS = 32 * (FIRST_DQ_WARP + 4 * NG);
};

template <int NT, int NG>
__global__ void __launch_bounds__(SmallMShape<NT, NG>::THREADS, 1)
    k_smallm(const __grid_constant__ SmallMParams p) {
    using S = SmallMShape<NT, NG>;
    constexpr int TS = S::T_STAGES, AS = S::A_SLOTS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw_base);
    float* t8s = reinterpret_cast<float*>(gbase + S::T8_OFF);
    auto slotA = [&](int a) { return base + (uint32_t)(a * S::A_BYTES); };
    auto stX = [&](int s) { return base + (uint32_t)(S::T_OFF + s * S::T_BYTES); };
    auto stC = [&](int s) { return base + (uint32_t)(S::T_OFF + s * S::T_BYTES + S::X_BYTES); };
    const uint32_t bar_base = base + S::BAR_OFF;
    auto full_tma = [&](int s) { return bar_base + 8u * s; };
    auto empty_tma = [&](int s) { return bar_base + 8u * (TS + s); };
    auto a_full = [&](int a) { return bar_base + 8u * (2 * TS + a); };
    auto a_empty = [&](int a) { return bar_base + 8u * (2 * TS + AS + a); };
    auto acc_full = [&](int b) { return bar_base + 8u * (2 * TS + 2 * AS + b); };
    auto acc_empty = [&](int b) { return bar_base + 8u * (2 * TS + 2 * AS + 2 + b); };
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + S::BAR_OFF + 8 * (2 * TS + 2 * AS + 4));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WaitCfg wc{p.timeout_ns};
    const int KS = p.ks_main + p.ks_lora;
    const int64_t I = (int64_t)p.tiles * KS;
    const int64_t r_begin = I * blockIdx.x / gridDim.x;
    const int64_t r_end = I * (blockIdx.x + 1) / gridDim.x;
    const int nunits = (int)(r_end - r_begin);

    if (threadIdx.x == 0) {
        for (int s = 0; s < TS; ++s) {
            mbar_init(full_tma(s), 1);
            mbar_init(empty_tma(s), 1);
        }
        for (int a = 0; a < AS; ++a) {
            mbar_init(a_full(a), 4);  // the four warps of the unit's dequant group
            mbar_init(a_empty(a), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), 4);  // the four epilogue warps
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < 256; i += blockDim.x) t8s[i] = dq_value(p.fmt.dq_type, (p.fmt.dq_type == 0 || i < 253) ? i : 0);
    if (warp == 0 && lane == 0) {
        pdl_trigger();
        prefetch_tensormap(&p.tmCodes);
        prefetch_tensormap(&p.tmX);
        if (p.ks_lora) {
            prefetch_tensormap(&p.tmB);
            prefetch_tensormap(&p.tmU);
        }
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), S::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // Dependent launch: with an adapter the kernel before is the sU GEMM,
    // which waited for its own predecessors before it let this one start, so
    // only sU needs the wait (the producer takes it before the first adapter
    // step).  Without one the kernel before may still be writing any input
    // (the quantizer, say): every thread waits here.
    if (p.ks_lora == 0) pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && !p.inject) {
            bool waited = false;
            int last_use[TS];
            for (int s = 0; s < TS; ++s) last_use[s] = -1;
            for (int it = 0; it < nunits; ++it) {
                const int s = it % TS, u = it / TS;
                if (!mbar_wait(empty_tma(s), (u & 1) ^ 1, wc)) { *abort_flag = 1; break; }
                const int64_t unit = r_begin + it;
                const int tile = (int)(unit / KS), k = (int)(unit - (int64_t)tile * KS);
                const int n0 = tile * 128;
                if (k < p.ks_main) {
                    mbar_arrive_expect_tx(full_tma(s), S::CODE_BYTES + S::X_BYTES);
                    tma_load_2d(stC(s), &p.tmCodes, full_tma(s), k * 32, n0);
                    tma_load_2d(stX(s), &p.tmX, full_tma(s), k * 64, 0);
                } else {
                    // LoRA step: the sU tile here; the B tile is loaded into the
                    // unit's A slot by its dequant group (which is never more
                    // than one use of the slot ahead of the MMA).  sU comes
                    // from the kernel before this one.
                    if (!waited) {
                        pdl_wait();
                        waited = true;
                    }
                    mbar_arrive_expect_tx(full_tma(s), S::X_BYTES);
                    const int ucol0 = p.seg_rows ? (n0 / p.seg_rows) * p.seg_r : 0;
                    tma_load_2d(stX(s), &p.tmU, full_tma(s), (k - p.ks_main) * 64 + ucol0, 0);
                }
                last_use[s] = u;
            }
            for (int s = 0; s < TS; ++s)
                if (last_use[s] >= 0) mbar_wait(full_tma(s), last_use[s] & 1, wc);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, NT, 0, 0);
            bool ok = true;
            int seg = 0;
            int it = 0;
            while (ok && it < nunits) {
                const int64_t unit0 = r_begin + it;
                const int tile = (int)(unit0 / KS), k0 = (int)(unit0 - (int64_t)tile * KS);
                const int len = (int)min((int64_t)(KS - k0), (int64_t)(nunits - it));
                const int ab = seg & 1;
                if (seg >= 2 && !mbar_wait(acc_empty(ab), ((seg >> 1) - 1) & 1, wc)) {
                    ok = false;
                    *abort_flag = 1;
                }
                tc_fence_after();
                for (int j = 0; ok && j < len; ++j, ++it) {
                    const int s = it % TS, a = it % AS;
                    if (!mbar_wait(a_full(a), (it / AS) & 1, wc)) { ok = false; *abort_flag = 1; break; }
                    tc_fence_after();
                    const uint32_t sA = slotA(a), sX = stX(s);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem + (uint32_t)(ab * S::ACC_COLS), smem_desc_sw128(sA + kk * 32, 16, 1024),
                                  smem_desc_sw128(sX + kk * 32, 16, 1024), idesc, (j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(a_empty(a));
                    umma_commit(empty_tma(s));
                }
                umma_commit(acc_full(ab));  // one phase per segment, also when cut short
                ++seg;
            }
            if (!ok && seg > 0) mbar_wait(acc_full((seg - 1) & 1), ((seg - 1) >> 1) & 1, wc);
        }
    } else if (warp < S::FIRST_DQ_WARP) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // TMEM lane = weight row inside the tile
        bool dead = false;
        int seg = 0;
        for (int it = 0; it < nunits; ++seg) {
            const int64_t unit0 = r_begin + it;
            const int tile = (int)(unit0 / KS), k0 = (int)(unit0 - (int64_t)tile * KS);
            const int len = (int)min((int64_t)(KS - k0), (int64_t)(nunits - it));
            it += len;
            const int k1 = k0 + len;
            const int ab = seg & 1;
            const int n = tile * 128 + row;
            float v[NT];
            if (!dead && !mbar_wait(acc_full(ab), (seg >> 1) & 1, wc)) {
                *abort_flag = 1;
                dead = true;
            }
            if (!dead) {
                tc_fence_after();
                uint32_t w[32];
#pragma unroll
                for (int c = 0; c < NT; c += 32) {
                    __syncwarp();
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * S::ACC_COLS + c), w);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 32 && c + q < NT; ++q) v[c + q] = __uint_as_float(w[q]);
                }
            }
            // the accumulator buffer is free for the segment after next
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && !dead) mbar_arrive(acc_empty(ab));
            if (dead) continue;
            if (k0 != 0) {
                // part of a tile begun by an earlier CTA: publish the partial,
                // one flag per warp (the owner's thread for a row waits for the
                // warp of the same TMEM quarter)
                float* o = p.part + (int64_t)blockIdx.x * NT * 128;
#pragma unroll
                for (int j = 0; j < NT; ++j)
                    if (QLORA_CHECK((int64_t)blockIdx.x * NT * 128 + j * 128 + row < p.part_cap)) o[j * 128 + row] = v[j];
                __threadfence();
                __syncwarp();
                if (lane == 0 && QLORA_CHECK((int64_t)blockIdx.x * 4 + quarter < p.flag_cap)) {
                    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p.flags + blockIdx.x * 4 + quarter),
                                 "r"(p.epoch)
                                 : "memory");
                }
                continue;
            }
            if (k1 < KS) {
                // owner of a tile that later CTAs finish: add their partials in CTA order
                const int64_t t_end = (int64_t)tile * KS + KS;
                for (int c = blockIdx.x + 1; c < (int)gridDim.x; ++c) {
                    const int64_t cb = I * c / gridDim.x, ce = I * (c + 1) / gridDim.x;
                    if (cb >= t_end) break;
                    if (ce == cb) continue;
                    const uint32_t* f = p.flags + c * 4 + quarter;
                    uint32_t fv;
                    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(fv) : "l"(f) : "memory");
                    if (fv != p.epoch) {
                        const uint64_t t_start = globaltimer_ns();
                        while (true) {
                            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(fv) : "l"(f) : "memory");
                            if (fv == p.epoch) break;
                            if (globaltimer_ns() - t_start > p.timeout_ns) {
                                set_status(4);
                                *abort_flag = 1;
                                dead = true;
                                break;
                            }
                        }
                    }
                    if (dead) break;
                    const float* o = p.part + (int64_t)c * NT * 128;
                    float w[NT];
#pragma unroll
                    for (int j = 0; j < NT; ++j) w[j] = __ldcg(o + j * 128 + row);
#pragma unroll
                    for (int j = 0; j < NT; ++j) v[j] = __fadd_rn(v[j], w[j]);
                    // consumed: clear the flag, so that a replay of the same
                    // launch (same epoch, e.g. in a CUDA graph) cannot take it
                    // for a fresh one
                    __syncwarp();
                    if (lane == 0) *const_cast<uint32_t*>(f) = 0u;
                }
                if (dead) continue;
            }
            if (n < p.N) {
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j < p.M) {
                        const uint32_t h = pack_bf16x2(v[j], 0.0f) & 0xFFFFu;
                        if (QLORA_CHECK(n < p.N)) p.Y[(int64_t)j * p.N + n] = (uint16_t)h;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ dequant groups
        const int dw = warp - S::FIRST_DQ_WARP;
        const int g = dw >> 2;               // this warp's group: units it with it % NG == g
        const int t = (dw & 3) * 32 + lane;  // weight row inside the tile
        const uint32_t code_off = sw32(t * 32), code_off2 = sw32(t * 32 + 16);
        const uint32_t out_off = t * 128;
        const float off = p.dq ? *p.offset : 0.0f;
        // raw block constant of unit `it` of this CTA: the 8-bit code and c1
        // (or the fp32 absmax), loaded two visits ahead of its use; a' itself
        // is formed at the use, so that no instruction waits on the loads
        // early.  Rows past the weight and LoRA steps get a' = 0.
        struct Raw {
            int q;     // q8 code, or -1 for "a' = 0"
            float c;   // c1 (double quantization) or absmax
        };
        auto fetch = [&](int it) -> Raw {
            Raw r{-1, 0.0f};
            if (it >= nunits) return r;
            const int64_t unit = r_begin + it;
            const int tile = (int)(unit / KS), k = (int)(unit - (int64_t)tile * KS);
            const int n = tile * 128 + t;
            if (k >= p.ks_main || n >= p.N) return r;
            const int64_t b = ((int64_t)n * p.kbs + k) >> p.fmt.bs_shift;
            if (!p.dq) {
                r.q = 0;
                r.c = __ldg(p.absmax + b);
            } else {
                r.q = __ldg(p.q8 + b);
                r.c = __ldg(p.c1 + (b >> 8));
            }
            return r;
        };
        auto block_const = [&](const Raw& r) -> float {
            if (r.q < 0) return 0.0f;
            return p.dq ? __fadd_rn(__fmul_rn(t8s[r.q], r.c), off) : r.c;
        };
        Raw r_next0 = fetch(g), r_next1 = fetch(g + NG);
        bool dead = false;
        for (int it = g; it < nunits; it += NG) {
            const Raw rw = r_next0;
            r_next0 = r_next1;
            r_next1 = fetch(it + 2 * NG);
            if (dead) continue;
            const int s = it % TS, a = it % AS;
            if (!mbar_wait(full_tma(s), (it / TS) & 1, wc)) {
                *abort_flag = 1;
                dead = true;
                continue;
            }
            const int64_t unit = r_begin + it;
            const int tile = (int)(unit / KS), k = (int)(unit - (int64_t)tile * KS);
            // the A slot is free once the MMAs of its previous unit are done
            if (!mbar_wait(a_empty(a), ((it / AS) & 1) ^ 1, wc)) {
                *abort_flag = 1;
                dead = true;
                continue;
            }
            if (k >= p.ks_main) {
                // LoRA step: one thread loads the B tile into the slot; its
                // arrival carries the transaction bytes, the other three warps
                // arrive below
                if (dw % 4 == 0) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(a_full(a), S::A_BYTES);
                        tma_load_2d(slotA(a), &p.tmB, a_full(a), (k - p.ks_main) * 64, tile * 128);
                    }
                    continue;
                }
            } else {
                const uint32_t sA = slotA(a);
                const uint32_t sC = stC(s);
                const uint4 c0 = ld_shared_v4(sC + code_off);
                const uint4 c1 = ld_shared_v4(sC + code_off2);
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                const Nf4BlockTable tb = nf4_block_table(block_const(rw), p.fmt.code_type);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t o[4];
                    nf4_expand_word(words[q], tb, o);
                    st_shared_v4(sA + sw128(out_off + q * 16), o[0], o[1], o[2], o[3]);
                }
                fence_proxy_async_smem();
            }
            (void)tile;
            __syncwarp();
            if (lane == 0) mbar_arrive(a_full(a));
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
