// linear.cuh -- host side of the QLoRA linear forward and backward: tensor
// maps, workspace carving, split-K choices and the launch sequence.
//
// Forward (reproduction blog "LoRA formula and tensor shapes"; digest sec. 4):
//   M > 64 :  sU = bf16(s * X A^T)   (skinny tcgen05 GEMM, split-K + reduce)
//             Y  = [X | sU] [W' | B]^T   (dequant GEMM, LoRA as extra k-steps)
//   M <= 64:  sU as above, then Y^T = [W' | B] [X | sU]^T with the weight as
//             the 128-row MMA operand (tokens as the narrow N side).
// Backward (digest sec. 4 steps 4: gradients pass through W^BF16; W frozen):
//   sU = bf16(s X A^T), sG = bf16(s dY B)          (skinny GEMMs)
//   dX = [dY | sG] [W' ; A]                       (dequant GEMM, MN-major W')
//   dA = sG^T X,  dB = dY^T sU                     (skinny GEMMs over M)
#pragma once

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "skinny.cuh"
#include "smallm.cuh"
#include "smallm_mma.cuh"
#include "internal.h"
#include "quantize.cuh"

namespace qlora {

// bf16 row-major [outer][inner], 64 x box_outer boxes, 128-byte swizzle.
inline bool map_bf16(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                     uint32_t box_outer) {
    return make_map(m, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, inner, outer, inner * 2, 64,
                    box_outer, CU_TENSOR_MAP_SWIZZLE_128B);
}

// ---------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------
template <int BN, int A_MN, int B_MN, int DQ, int EPI, int STAGES, int MT = 1>
inline cudaError_t launch_gemm(const GemmParams& p, dim3 grid, cudaStream_t s, int prof_kind = -1) {
    using Sh = GemmShape<BN, A_MN, B_MN, DQ, MT>;
    constexpr int smem = gemm_smem_bytes<BN, A_MN, B_MN, DQ, STAGES, MT>();
    static_assert(smem <= 232448, "shared memory per CTA");
    auto kern = k_gemm<BN, A_MN, B_MN, DQ, EPI, STAGES, MT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ProfileScope ps(prof_kind, s);
    note_launch();
    kern<<<grid, Sh::THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

inline int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Split-K choice: about two CTAs per SM, every split at least one k-step.
inline void choose_splits(int tiles, int ksteps, int* splits, int* per) {
    int S = std::max(1, (2 * 148 + tiles - 1) / std::max(1, tiles));
    S = std::min(S, std::max(1, ksteps));
    int p = std::max(1, (ksteps + S - 1) / S);
    *per = p;
    *splits = std::max(1, (ksteps + p - 1) / p);
}

inline int lora_bn(int r) { return r <= 64 ? 64 : (r <= 128 ? 128 : 256); }

constexpr int kSmallM = 64;

struct WsCarve {
    char* p;
    size_t used;
    void* take(size_t bytes) {
        void* r = p ? p + used : nullptr;
        used += align256(bytes);
        return r;
    }
};

// Skinny GEMMs out[rows][r] = scale * sum_k Aop[row][k] Bop[j][k]: 128-row
// tiles, the reduction split across a cluster of up to 8 CTAs and summed over
// distributed shared memory (deterministic); one launch for one or two
// independent problems of the same r.
// How many clusters of cs CTAs of k_skinny<BN> can be resident at
// once on the current device (queried once per device, BN and cs).
template <int BN>
inline int skinny_active_clusters(int cs) {
    static std::mutex mu;
    static int cache[64][4];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
    const int lg = cs == 1 ? 0 : (cs == 2 ? 1 : (cs == 4 ? 2 : 3));
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev][lg] > 0) return cache[dev][lg];
    constexpr int smem = SkinnyShape<BN>::SMEM;
    auto kern = k_skinny<BN>;
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3((unsigned)(cs * 64), 1, 1);
        cfg.blockDim = dim3(SkinnyShape<BN>::THREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = (unsigned)cs;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
    }
    if (n < 1) n = 1;
    cache[dev][lg] = n;
    return n;
}

template <int BN>
inline cudaError_t launch_skinny(SkinnyParams& p, int tiles, int kmin, int kmax, cudaStream_t s) {
    constexpr int smem = SkinnyShape<BN>::SMEM;
    static_assert(smem <= 232448, "shared memory per CTA");
    // Cluster size: fewest rounds of resident clusters times k-steps per CTA
    // (plus a fixed per-CTA cost of about three k-steps), at least one
    // k-step per CTA of the shorter problem.  Packed launches reduce each
    // tile on one CTA.
    int cs = 1;
    if (p.pack) {
        cs = 1;
    } else {
        int64_t best = -1;
        for (int c = 8; c >= 1; c >>= 1) {
            if (c > 1 && kmin < c) continue;
            const int64_t rounds = ceil_div(tiles, skinny_active_clusters<BN>(c));
            const int64_t cost = rounds * (ceil_div(kmax, c) + 3);
            if (best < 0 || cost < best) {
                best = cost;
                cs = c;
            }
        }
    }
    for (int i = 0; i < p.nprob; ++i) p.pr[i].per = ceil_div(p.pr[i].ksteps, cs);
    p.total_tiles = tiles;
    auto kern = k_skinny<BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ProfileScope ps(QLORA_KERNEL_LORA_GEMM, s);
    note_launch();
    if (p.pack)  // two independent tiles per cluster of 2: one TPC each
        return launch_pdl(kern, dim3((unsigned)((tiles + 1) & ~1), 1, 1), dim3(SkinnyShape<BN>::THREADS, 1, 1), smem,
                          s, 2, p);
    return launch_pdl(kern, dim3((unsigned)(tiles * cs), 1, 1), dim3(SkinnyShape<BN>::THREADS, 1, 1), smem, s, cs,
                      p);
}

template <int BN>
inline cudaError_t launch_lora_stream(SkinnyParams& p, int tiles, int nctas, cudaStream_t s) {
    constexpr int smem = StreamShape<BN>::SMEM;
    static_assert(smem <= 232448, "shared memory per CTA");
    for (int i = 0; i < p.nprob; ++i) p.pr[i].per = p.pr[i].ksteps;
    p.total_tiles = tiles;
    p.pack = 0;
    auto kern = k_lora_stream<BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ProfileScope ps(QLORA_KERNEL_LORA_GEMM, s);
    note_launch();
    // clusters of 2 only for placement (the CTAs are independent): whole
    // TPCs, never one SM of a TPC that a CTA-pair kernel beside it could use
    const int grid = (std::max(1, std::min(tiles, nctas)) + 1) & ~1;
    return launch_pdl(kern, dim3((unsigned)grid, 1, 1), dim3(StreamShape<BN>::THREADS, 1, 1), smem, s, 2, p);
}

// One skinny problem: operands (tensor maps and majorness), extent and output.
struct SkinnyDesc {
    CUtensorMap tA, tB;
    int a_mn, b_mn;
    int rows, ksteps;
    float scale;
    int out_mode;  // SK_OUT_*
    void* out;
    int64_t out_ld;
    int r;         // output columns (0: the launch's r)
    int seg_mode, seg_rows, seg_r;  // SK_SEG_* (fused projections)
};

// wait_first: the operands may have been written by the kernel just before on
// the stream (or by an unknown earlier one), so the loads wait for it.
// place: SKP_SPLIT (cluster size from the cost model, the reduction split
// across it), SKP_PACKED (one CTA per 128-row tile, two tiles per TPC: work
// that leaves whole TPCs to a CTA-pair GEMM beside it), SKP_STREAM (the
// persistent kernel on up to nctas CTAs: work beside a kernel that holds
// most SMs; with ctrs the CTAs take tiles from a shared counter).
enum { SKP_SPLIT = 0, SKP_PACKED = 1, SKP_STREAM = 2 };
// SKP_STREAM with ctrs (two ints, zero before the launch): tiles taken in
// problem order from ctrs[0]; problem dep_prob reads problem 0's output.
// wait_mask (SKP_STREAM with wait_first == 0): problems that read the
// previous kernel's output, waited for before their first tile.
inline qlora_status skinny(const SkinnyDesc* d, int nprob, int r, cudaStream_t s, int wait_first,
                           int place = SKP_SPLIT, int nctas = 0, int* ctrs = nullptr, int dep_prob = -1,
                           int wait_mask = 0) {
    SkinnyParams p;
    memset(&p, 0, sizeof(p));
    p.wait_first = wait_first;
    p.pack = place == SKP_PACKED ? 1 : 0;
    p.tile_ctr = ctrs;
    p.done_ctr = ctrs ? ctrs + 1 : nullptr;
    p.dep_prob = ctrs ? dep_prob : -1;
    p.wait_mask = wait_mask;
    int tiles = 0, kmin = 1 << 30, kmax = 0;
    for (int i = 0; i < nprob; ++i) {
        tiles += ceil_div(d[i].rows, 128);
        kmin = std::min(kmin, d[i].ksteps);
        kmax = std::max(kmax, d[i].ksteps);
    }
    for (int i = 0; i < nprob; ++i) {
        SkinnyProblem& q = p.pr[i];
        q.tmA = d[i].tA;
        q.tmB = d[i].tB;
        q.a_mn = d[i].a_mn;
        q.b_mn = d[i].b_mn;
        q.rows = d[i].rows;
        q.r = d[i].r > 0 ? d[i].r : r;
        q.seg_mode = d[i].seg_mode;
        q.seg_rows = d[i].seg_rows;
        q.seg_r = d[i].seg_r;
        q.ksteps = d[i].ksteps;
        q.tiles = ceil_div(d[i].rows, 128);
        q.scale = d[i].scale;
        q.out_mode = d[i].out_mode;
        q.out = d[i].out;
        q.out_ld = d[i].out_ld;
    }
    p.nprob = nprob;
    p.timeout_ns = wait_timeout_ns();
    p.inject = inject_mode() == 1 ? 1 : 0;
    const int bn = lora_bn(r);
    cudaError_t e;
    if (place == SKP_STREAM) {
        if (bn == 64)
            e = launch_lora_stream<64>(p, tiles, nctas, s);
        else if (bn == 128)
            e = launch_lora_stream<128>(p, tiles, nctas, s);
        else
            e = launch_lora_stream<256>(p, tiles, nctas, s);
        return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
    }
    if (bn == 64)
        e = launch_skinny<64>(p, tiles, kmin, kmax, s);
    else if (bn == 128)
        e = launch_skinny<128>(p, tiles, kmin, kmax, s);
    else
        e = launch_skinny<256>(p, tiles, kmin, kmax, s);
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// Most CTAs of the small-M kernel's persistent grid (partial tiles and flags).
constexpr int kMaxSmallMCtas = 256;

inline int small_m_nt(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

// M <= kSmallMmaDefault (or M <= kSmallMma in test mode 7): the register-fed warp-MMA kernel
// (smallm_mma.cuh) on a persistent grid of at most kSmallMmaMaxCtas CTAs of
// 16 warps; its workspace holds two fp32 partial slots per CTA and row slice
// (32 rows x 16 tokens or 16 rows x 32 tokens) and one 64-bit counter per
// row slice of a 128- or 64-row group.
constexpr int kSmallMma = 32;
constexpr int kSmallMmaDefault = 16;
constexpr int kSmallMmaMaxCtas = 160;
constexpr int kSmallMmaPartFloatsPerCta = 32768;  // at least 2 slots x 4 slices x 32 rows x 32 tokens

inline int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// Largest stream-K grid; also sizes the partial-tile workspace.
constexpr int kMaxStreamK = 256;

// Workspace layout shared by the query and the launches.
struct LinearWs {
    float* scales;
    int64_t scales_ld;
    uint16_t* sU;
    uint16_t* sG;
    float* part;          // small-M partial tiles
    uint32_t* sm_flags;   // small-M partial flags
    size_t part_floats;   // capacity of part (floats)
    size_t nflags;        // capacity of sm_flags (32-bit words)
    float* sk_part;  // stream-K partial tiles [kMaxStreamK][256*256]
    int* sk_flags;   // [kMaxStreamK] stream-K flags, then the 2 tile counters of the backward's side launch
    size_t bytes;
};

inline LinearWs carve_linear_ws(void* ws, int64_t M, int64_t N, int64_t K, int r, int bwd) {
    WsCarve c{static_cast<char*>(ws), 0};
    LinearWs L;
    const bool big = bwd || M > kSmallM;
    L.scales_ld = ((N + 255) / 256) * 256;
    L.scales = big ? static_cast<float*>(c.take((size_t)(K / 64) * L.scales_ld * 4)) : nullptr;
    L.sU = r > 0 ? static_cast<uint16_t*>(c.take((size_t)M * r * 2)) : nullptr;
    L.sG = (r > 0 && bwd) ? static_cast<uint16_t*>(c.take((size_t)M * r * 2)) : nullptr;
    // small-M forward: partial tiles [kMaxSmallMCtas][NT][128] and flags
    // [kMaxSmallMCtas][4] of the tcgen05 kernel; for M <= 32 also room for
    // the warp-MMA kernel's partial slots and its counters, one per row slice
    // of each unit of 64 to 224 rows, at most N / 16 + 8 (test mode 7 picks
    // that kernel at run time, so both layouts must fit)
    size_t part_floats = (size_t)kMaxSmallMCtas * small_m_nt(M) * 128;
    size_t nflags = (size_t)kMaxSmallMCtas * 4;
    if (M <= kSmallMma) {
        part_floats = std::max(part_floats, (size_t)kSmallMmaMaxCtas * kSmallMmaPartFloatsPerCta);
        nflags = std::max(nflags, (size_t)((N + 15) / 16 + 8) * 2);  // 64-bit counters: groups x slices
    }
    L.part = big ? nullptr : static_cast<float*>(c.take(part_floats * 4));
    L.sm_flags = big ? nullptr : static_cast<uint32_t*>(c.take(nflags * 4));
    L.part_floats = big ? 0 : part_floats;
    L.nflags = big ? 0 : nflags;
    L.sk_part = big ? static_cast<float*>(c.take((size_t)kMaxStreamK * 256 * 256 * 4)) : nullptr;
    L.sk_flags = big ? static_cast<int*>(c.take((size_t)(kMaxStreamK + 2) * 4)) : nullptr;
    L.bytes = c.used;
    return L;
}

inline size_t linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int r, int bwd) {
    return carve_linear_ws(nullptr, M, N, K, r, bwd).bytes;
}

// Packed codes viewed [rows][K/2 bytes].  32-byte boxes use the 32-byte
// swizzle and 128-byte boxes the 128-byte swizzle, so that the dequant
// threads' 16-byte reads of a tile are free of bank conflicts.
// Tile schedule of the dequant GEMMs: stream-K over a persistent grid of
// one CTA per SM when there are at least two k-steps per CTA, else one CTA
// per tile.  Debug mode 2 forces stream-K on 7 CTAs (tests of the merge).
template <int DQ, int STAGES>
inline cudaError_t launch_gemm_pair(const GemmParams& p, dim3 grid, cudaStream_t s, int prof_kind) {
    constexpr int smem = pair_smem_bytes<DQ, STAGES>();
    static_assert(smem <= 232448, "shared memory per CTA");
    auto kern = p.streamk ? k_gemm_pair<DQ, STAGES, true> : k_gemm_pair<DQ, STAGES, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ProfileScope ps(prof_kind, s);
    note_launch();
    // cluster shape from the kernel's __cluster_dims__
    return launch_pdl(kern, grid, dim3(PairShape<DQ>::THREADS, 1, 1), smem, s, 0, p);
}

// Which large-M GEMM runs: CTA pairs with one pair per tile (default), CTA
// pairs with the stream-K schedule, or the single-CTA kernel on the grid or
// stream-K schedule.  QLORA_SCHEDULE=pair|pairsk|grid|streamk selects one;
// test mode 2 forces single-CTA stream-K, mode 3 the single-CTA grid, mode 4
// pair stream-K on 4 pairs.
enum { SCHED_PAIR = 0, SCHED_GRID = 1, SCHED_STREAMK = 2, SCHED_PAIR_SK = 3 };
inline int large_m_schedule() {
    if (inject_mode() == 2) return SCHED_STREAMK;
    if (inject_mode() == 3) return SCHED_GRID;
    if (inject_mode() == 4) return SCHED_PAIR_SK;
    static int v = [] {
        const char* e = getenv("QLORA_SCHEDULE");
        if (!e) return (int)SCHED_PAIR;
        if (!strcmp(e, "grid")) return (int)SCHED_GRID;
        if (!strcmp(e, "streamk")) return (int)SCHED_STREAMK;
        if (!strcmp(e, "pairsk")) return (int)SCHED_PAIR_SK;
        return (int)SCHED_PAIR;
    }();
    return v;
}

// CTA pairs of k_gemm_pair<DQ, STAGES> that can be resident at once on the
// current device (queried once per device).
template <int DQ, int STAGES>
inline int pair_active_clusters() {
    static std::mutex mu;
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] > 0) return cache[dev];
    constexpr int smem = pair_smem_bytes<DQ, STAGES>();
    auto kern = k_gemm_pair<DQ, STAGES, true>;
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3(2 * 64, 1, 1);
        cfg.blockDim = dim3(PairShape<DQ>::THREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
    }
    if (n < 1) n = 1;
    cache[dev] = n;
    return n;
}

// Tile schedule of the pair GEMM over tiles_m x tiles_n tiles of 512 x 256:
// one pair per tile, or (SCHED_PAIR_SK) stream-K over all resident pairs;
// test mode 4 runs stream-K on 4 pairs, so that tiles are cut between pairs
// and merged even at small sizes.
template <int DQ, int STAGES>
inline dim3 schedule_pair(GemmParams& p, int tiles_n, int tiles_m, const LinearWs& L) {
    const int64_t tiles = (int64_t)tiles_n * tiles_m;
    p.tiles_n = tiles_n;
    p.tiles_total = (int)tiles;
    p.sk_part = L.sk_part;
    p.sk_flags = L.sk_flags;
    p.streamk = 0;
    int G = 0;
    if (inject_mode() == 4)
        G = 4;
    else if (large_m_schedule() == SCHED_PAIR_SK)
        G = std::min(pair_active_clusters<DQ, STAGES>(), kMaxStreamK / 2);
    if (G > 0 && L.sk_part && L.sk_flags) {
        p.streamk = 1;
        return dim3((unsigned)(2 * G), 1, 1);
    }
    // token tiles fastest (blockIdx.x / 2), weight column tiles in y (the
    // grid's y extent is at most 65535: beyond it, columns in x)
    p.n_in_x = tiles_n > 65535 ? 1 : 0;
    if (p.n_in_x) return dim3((unsigned)(2 * tiles_n), (unsigned)tiles_m, 1);
    return dim3((unsigned)(2 * tiles_m), (unsigned)tiles_n, 1);
}

inline dim3 schedule_gemm(GemmParams& p, int tiles_n, int tiles_m, const LinearWs& L) {
    const int KS = p.ks_main + p.ks_lora;
    const int64_t tiles = (int64_t)tiles_n * tiles_m;
    int G = std::min(sm_count(), kMaxStreamK);
    if (inject_mode() == 2) G = 7;
    p.tiles_n = tiles_n;
    p.tiles_total = (int)tiles;
    p.sk_part = L.sk_part;
    p.sk_flags = L.sk_flags;
    const bool sk = large_m_schedule() == SCHED_STREAMK;
    p.streamk = sk ? 1 : 0;
    if (!sk) return dim3(tiles_n, tiles_m, 1);
    return dim3((unsigned)std::min<int64_t>(G, tiles * KS), 1, 1);
}

inline bool map_codes(CUtensorMap* m, const qlora_nf4_weight& w, uint32_t box_bytes,
                      uint32_t box_rows) {
    return make_map(m, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)w.cols / 2,
                    (uint64_t)w.rows, (uint64_t)w.cols / 2, box_bytes, box_rows,
                    box_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                    : (box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B));
}

// sU = bf16(scale * X A^T): Aop = X [m][k] (K-major), Bop = A [j][k] (K-major)
// (A = [A_0; A_1; ...] of a fused projection: every adapter's sU in one pass over X)
inline bool desc_sU(SkinnyDesc* d, const void* X, const LinearArgs& a, const void* A, void* sU) {
    memset(d, 0, sizeof(*d));
    if (!map_bf16(&d->tA, X, a.K, a.M, 128)) return false;
    if (!map_bf16(&d->tB, A, a.K, a.rt(), lora_bn(a.rt()))) return false;
    d->rows = (int)a.M;
    d->ksteps = (int)(a.K / 64);
    d->scale = a.scale;
    d->out_mode = SK_OUT_BF16;
    d->out = sU;
    d->out_ld = a.rt();
    d->r = a.rt();
    return true;
}

// Launch identifier of the small-M kernel's partial-tile flags: a flag holds
// the epoch of the launch that published it, so stale flags of earlier
// launches (or an uninitialized workspace) never match.  Starts at a
// clock-derived value and never returns 0.
inline uint32_t next_epoch() {
    static std::atomic<uint32_t> e{(uint32_t)(std::chrono::steady_clock::now().time_since_epoch().count() * 2654435761ull) | 1u};
    uint32_t v = e.fetch_add(1) + 1;
    if (v == 0) v = e.fetch_add(1) + 1;
    return v;
}

template <int NT, int NG>
inline cudaError_t launch_small_m_kernel(const SmallMParams& p, int grid, cudaStream_t s) {
    constexpr int smem = SmallMShape<NT, NG>::SMEM;
    static_assert(smem <= 232448, "shared memory per CTA");
    auto kern = k_smallm<NT, NG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ProfileScope ps(QLORA_KERNEL_SMALLM_GEMM, s);
    note_launch();
    return launch_pdl(kern, dim3((unsigned)grid, 1, 1), dim3(SmallMShape<NT, NG>::THREADS, 1, 1), smem, s, 0, p);
}

template <int MT, int SL>
inline cudaError_t launch_small_m_mma_kernel(SmallMmaParams& p, cudaStream_t s) {
    using S = SmallMmaShape<MT, SL>;
    static_assert(S::SMEM + S::STATIC_SMEM <= 232448, "shared memory per CTA");
    static_assert(2 * S::SLICES * S::PART_FLOATS <= kSmallMmaPartFloatsPerCta, "partial workspace");
    const int64_t groups = (p.N + S::UROWS - 1) / S::UROWS;
    p.KSU = (p.KB + 3) / 4 + (p.lora_ks + 3) / 4;
    p.units = groups * p.KSU;
    // at least 4 units per CTA; at most one CTA per SM
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(std::min(sm_count(), kSmallMmaMaxCtas),
                                                                p.units / 4));
    auto kern = k_smallm_mma<MT, SL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
    if (e != cudaSuccess) return e;
    ProfileScope ps(QLORA_KERNEL_SMALLM_GEMM, s);
    note_launch();
    return launch_pdl(kern, dim3((unsigned)ctas, 1, 1), dim3(S::THREADS, 1, 1), S::SMEM, s, 0, p);
}

// Y = X W'^T + sU B^T for M <= 32: table-lookup expansion into warp MMAs.
inline qlora_status launch_small_m_mma(const void* X, const LinearArgs& a, const void* B, void* Y,
                                       const LinearWs& L, cudaStream_t s) {
    const qlora_nf4_weight& w = *a.w;
    const int MT = a.M <= 16 ? 1 : 2;
    // the wide unit (seven row slices, 224 rows) unless a fused projection's
    // segment boundary would fall inside one (each unit takes one adapter)
    using Wide = SmallMmaShape<1, QLORA_SMALLM_WIDE>;
    const bool six = MT == 1 && (a.nseg <= 1 || a.seg_rows % Wide::UROWS == 0);
    const int urows = six ? Wide::UROWS : MT == 1 ? SmallMmaShape<1>::UROWS : SmallMmaShape<2>::UROWS;
    SmallMmaParams p;
    memset(&p, 0, sizeof(p));
    // codes [N][K/2] bytes: 128-byte boxes (four blocks of a row) of UROWS
    // rows, 128-byte swizzle (a warp's 8-byte reads of 8 rows hit 8 banks)
    if (!make_map(&p.tmCodes, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(a.K / 2), (uint64_t)a.N,
                  (uint64_t)(a.K / 2), 128, (uint32_t)urows, CU_TENSOR_MAP_SWIZZLE_128B))
        return QLORA_ERR_CUDA;
    if (!map_bf16(&p.tmX, X, a.K, a.M, 16 * MT)) return QLORA_ERR_CUDA;
    if (a.r > 0 && !map_bf16(&p.tmU, L.sU, a.rt(), a.M, 16 * MT)) return QLORA_ERR_CUDA;
    p.q8 = w.absmax_q8;
    p.c1 = w.absmax_scale;
    p.offset = w.absmax_offset;
    p.absmax = w.absmax;
    p.dq = w.double_quant;
    p.B = static_cast<const uint16_t*>(B);
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.KB = (int)(a.K / 64);
    p.r = a.r;
    p.seg_rows = a.nseg > 1 ? (int)a.seg_rows : 0;
    p.lora_ks = a.r > 0 ? ceil_div(a.r, 64) : 0;
    p.fmt = weight_format(w);
    p.inv_scale = w.code_type ? 1.0f / 1.5f : 1.0f / 1.18881f;
    p.Y = static_cast<uint16_t*>(Y);
    p.part = L.part;
    p.counters = reinterpret_cast<unsigned long long*>(L.sm_flags);
    p.part_cap = (int64_t)L.part_floats;
    p.counter_cap = (int64_t)(L.nflags / 2);
    p.epoch = next_epoch();
    if (p.epoch == 0) p.epoch = 1;
    p.timeout_ns = wait_timeout_ns();
    p.inject = inject_mode() == 1 ? 1 : 0;
    const cudaError_t e = six       ? launch_small_m_mma_kernel<1, QLORA_SMALLM_WIDE>(p, s)
                          : MT == 1 ? launch_small_m_mma_kernel<1, 4>(p, s)
                                    : launch_small_m_mma_kernel<2, 4>(p, s);
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// Y = X W'^T + sU B^T for M <= 64 on a persistent stream-K grid (one CTA per
// SM, at least four (tile, k-step) units per CTA).
inline qlora_status launch_small_m(const void* X, const LinearArgs& a, const void* B, void* Y,
                                   const LinearWs& L, cudaStream_t s) {
    // M <= 16: the warp-MMA kernel (test mode 8: the tcgen05 kernel instead);
    // 17 <= M <= 32: the tcgen05 kernel (test mode 7: the warp-MMA kernel)
    const int mode = inject_mode();
    if ((a.M <= kSmallMmaDefault && mode != 8) || (a.M <= kSmallMma && mode == 7))
        return launch_small_m_mma(X, a, B, Y, L, s);
    const qlora_nf4_weight& w = *a.w;
    const int NT = small_m_nt(a.M);
    SmallMParams p;
    memset(&p, 0, sizeof(p));
    if (!map_codes(&p.tmCodes, w, 32, 128)) return QLORA_ERR_CUDA;
    if (!map_bf16(&p.tmX, X, a.K, a.M, NT)) return QLORA_ERR_CUDA;
    if (a.r > 0) {
        if (!map_bf16(&p.tmB, B, a.r, a.N, 128)) return QLORA_ERR_CUDA;
        if (!map_bf16(&p.tmU, L.sU, a.rt(), a.M, NT)) return QLORA_ERR_CUDA;
        if (a.nseg > 1) {
            p.seg_rows = (int)a.seg_rows;
            p.seg_r = a.r;
        }
    } else {
        p.tmB = p.tmX;
        p.tmU = p.tmX;
    }
    p.q8 = w.absmax_q8;
    p.c1 = w.absmax_scale;
    p.offset = w.absmax_offset;
    p.absmax = w.absmax;
    p.dq = w.double_quant;
    p.fmt = weight_format(w);
    p.N = (int)a.N;
    p.M = (int)a.M;
    p.kbs = (int)(a.K / 64);
    p.ks_main = (int)(a.K / 64);
    p.ks_lora = a.r > 0 ? ceil_div(a.r, 64) : 0;
    p.tiles = ceil_div(a.N, 128);
    p.Y = static_cast<uint16_t*>(Y);
    p.part = L.part;
    p.flags = L.sm_flags;
    p.part_cap = (int64_t)L.part_floats;
    p.flag_cap = (int64_t)L.nflags;
    p.epoch = next_epoch();
    p.timeout_ns = wait_timeout_ns();
    p.inject = inject_mode() == 1 ? 1 : 0;
    const int64_t units = (int64_t)p.tiles * (p.ks_main + p.ks_lora);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(std::min(sm_count(), kMaxSmallMCtas), units / 4));
    cudaError_t e;
    if (NT == 16)
        e = launch_small_m_kernel<16, 3>(p, grid, s);
    else if (NT == 32)
        e = launch_small_m_kernel<32, 3>(p, grid, s);
    else
        e = launch_small_m_kernel<64, 3>(p, grid, s);
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

inline qlora_status linear_fwd_impl(const void* X, const LinearArgs& a, const void* A,
                                    const void* B, void* Y, void* ws, size_t ws_bytes,
                                    cudaStream_t s) {
    (void)ws_bytes;
    const qlora_nf4_weight& w = *a.w;
    LinearWs L = carve_linear_ws(ws, a.M, a.N, a.K, a.rt(), 0);
    if (a.M > kSmallM &&
        launch_expand_scales(w, L.scales, L.scales_ld, s, L.sk_flags, L.sk_flags ? kMaxStreamK + 2 : 0) != cudaSuccess)
        return QLORA_ERR_CUDA;
    if (a.r > 0) {
        SkinnyDesc d;
        if (!desc_sU(&d, X, a, A, L.sU)) return QLORA_ERR_CUDA;
        // M > 64: one CTA per 128-row tile (16 for 2048 tokens), launched
        // after the block-constant expansion has completed; the pair GEMM
        // starts beside it on the other SMs and waits for sU only before its
        // LoRA k-step.  Small M: the cost-model cluster size.
        qlora_status st = skinny(&d, 1, a.rt(), s, 1, a.M > kSmallM ? SKP_PACKED : SKP_SPLIT);
        if (st != QLORA_OK) return st;
    }
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.scales = L.scales;
    p.scales_ld = L.scales_ld;
    p.dq_rows = (int)a.N;
    p.dq_kbs = (int)(a.K / 64);
    p.ks_main = (int)(a.K / 64);
    p.ks_lora = a.r > 0 ? ceil_div(a.r, 64) : 0;
    p.timeout_ns = wait_timeout_ns();
    p.inject = inject_mode() == 1 ? 1 : 0;
    p.out = Y;
    p.code_type = w.code_type;
    if (a.r > 0 && a.nseg > 1) {
        p.lora_seg_rows = (int)a.seg_rows;
        p.lora_seg_r = a.r;
    }
    if (a.M > kSmallM) {
        // Y = [X | sU] [W' | B]^T : 128 x 256 tiles, W' dequantized into the B slot.
        if (!map_bf16(&p.tmA, X, a.K, a.M, 128)) return QLORA_ERR_CUDA;
        p.tmB = p.tmA;
        if (!map_codes(&p.tmCodes, w, 32, 256)) return QLORA_ERR_CUDA;
        if (a.r > 0) {
            if (!map_bf16(&p.tmA2, L.sU, a.rt(), a.M, 128)) return QLORA_ERR_CUDA;
            if (!map_bf16(&p.tmB2, B, a.r, a.N, 256)) return QLORA_ERR_CUDA;
        } else {
            p.tmA2 = p.tmA;
            p.tmB2 = p.tmA;
        }
        p.ks_per_split = p.ks_main;
        p.rows = (int)a.M;
        p.cols = (int)a.N;
        p.out_ld = a.N;
        if (!map_bf16(&p.tmOut, Y, a.N, a.M, 128)) return QLORA_ERR_CUDA;
        if (large_m_schedule() == SCHED_PAIR || large_m_schedule() == SCHED_PAIR_SK) {
            if (!map_codes(&p.tmCodes, w, 32, 128)) return QLORA_ERR_CUDA;
            if (a.r > 0 && !map_bf16(&p.tmB2, B, a.r, a.N, 128)) return QLORA_ERR_CUDA;
            p.late_wait = a.r > 0 ? 1 : 0;
            dim3 grid = schedule_pair<DQ_B_K, 4>(p, ceil_div(a.N, 256), ceil_div(a.M, 512), L);
            if (launch_gemm_pair<DQ_B_K, 4>(p, grid, s, QLORA_KERNEL_FWD_GEMM) != cudaSuccess)
                return QLORA_ERR_CUDA;
            return QLORA_OK;
        }
        dim3 grid = schedule_gemm(p, ceil_div(a.N, 256), ceil_div(a.M, 256), L);
        if (launch_gemm<256, 0, 0, DQ_B_K, EPI_BF16, 3, 2>(p, grid, s, QLORA_KERNEL_FWD_GEMM) != cudaSuccess)
            return QLORA_ERR_CUDA;
        return QLORA_OK;
    }
    // small M: Y^T = [W' | B] [X | sU]^T, weight rows on the 128-lane side
    return launch_small_m(X, a, B, Y, L, s);
}

// sG = bf16(scale dY B): Aop = dY [m][n] (K-major), Bop = B viewed [j][n] (MN-major).
// (fused projection: sG = [dY_0 B_0 | dY_1 B_1 | ...], each k-step of dY rows
// shifted onto its own segment's output columns)
inline bool desc_sG(SkinnyDesc* d, const CUtensorMap& tdY, const LinearArgs& a, const void* B, void* sG) {
    memset(d, 0, sizeof(*d));
    d->tA = tdY;
    if (!map_bf16(&d->tB, B, a.r, a.N, 64)) return false;
    d->b_mn = 1;
    d->rows = (int)a.M;
    d->ksteps = ceil_div(a.N, 64);
    d->scale = a.scale;
    d->out_mode = SK_OUT_BF16;
    d->out = sG;
    d->out_ld = a.rt();
    d->r = a.rt();
    if (a.nseg > 1) {
        d->seg_mode = SK_SEG_REDUCE;
        d->seg_rows = (int)a.seg_rows;
        d->seg_r = a.r;
    }
    return true;
}

// dA^T [K][r] = X^T sG : Aop = X viewed [k][m] (MN-major), Bop = sG viewed [j][m] (MN-major)
// dB [N][r] = dY^T sU : Aop = dY viewed [n][m] (MN-major), Bop = sU viewed [j][m]
inline bool desc_dA_dB(SkinnyDesc* d, const void* dY, const void* X, const LinearArgs& a, const LinearWs& L,
                       float* dA, float* dB) {
    memset(d, 0, 2 * sizeof(*d));
    if (!map_bf16(&d[0].tA, X, a.K, a.M, 64)) return false;
    if (!map_bf16(&d[0].tB, L.sG, a.rt(), a.M, 64)) return false;
    d[0].rows = (int)a.K;
    d[0].out_mode = SK_OUT_F32_T;
    d[0].out = dA;
    d[0].out_ld = a.K;
    d[0].r = a.rt();
    if (!map_bf16(&d[1].tA, dY, a.N, a.M, 64)) return false;
    if (!map_bf16(&d[1].tB, L.sU, a.rt(), a.M, 64)) return false;
    d[1].rows = (int)a.N;
    d[1].out_mode = SK_OUT_F32;
    d[1].out = dB;
    d[1].out_ld = a.r;
    d[1].r = a.r;
    if (a.nseg > 1) {  // the dB rows of a segment read that segment's sU columns
        d[1].seg_mode = SK_SEG_ROWS;
        d[1].seg_rows = (int)a.seg_rows;
        d[1].seg_r = a.r;
    }
    for (int i = 0; i < 2; ++i) {
        d[i].a_mn = 1;
        d[i].b_mn = 1;
        d[i].ksteps = ceil_div(a.M, 64);
        d[i].scale = 1.0f;
    }
    return true;
}

// dX = [dY | sG] [w' ; A] on stream s.  late_wait: the kernel before it on s
// has waited for the block-constant expansion, only sG is still being written.
inline qlora_status launch_dx_gemm(const void* A, void* dX, const LinearArgs& a, const LinearWs& L,
                                   const CUtensorMap& tdY, int late_wait, cudaStream_t s) {
    const qlora_nf4_weight& w = *a.w;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.tmA = tdY;
    p.tmB = tdY;
    if (!map_codes(&p.tmCodes, w, 128, 64)) return QLORA_ERR_CUDA;
    if (a.r > 0) {
        if (!map_bf16(&p.tmA2, L.sG, a.rt(), a.M, 128)) return QLORA_ERR_CUDA;
        if (!map_bf16(&p.tmB2, A, a.K, a.rt(), 64)) return QLORA_ERR_CUDA;
    } else {
        p.tmA2 = tdY;
        p.tmB2 = tdY;
    }
    p.scales = L.scales;
    p.scales_ld = L.scales_ld;
    p.code_type = w.code_type;
    p.dq_rows = (int)a.N;
    p.dq_kbs = (int)(a.K / 64);
    p.ks_main = ceil_div(a.N, 64);
    p.ks_lora = a.r > 0 ? ceil_div(a.rt(), 64) : 0;
    p.ks_per_split = p.ks_main;
    p.rows = (int)a.M;
    p.cols = (int)a.K;
    p.out = dX;
    p.out_ld = a.K;
    if (!map_bf16(&p.tmOut, dX, a.K, a.M, 128)) return QLORA_ERR_CUDA;
    p.timeout_ns = wait_timeout_ns();
    p.inject = inject_mode() == 1 ? 1 : 0;
    if (large_m_schedule() == SCHED_PAIR || large_m_schedule() == SCHED_PAIR_SK) {
        if (!map_codes(&p.tmCodes, w, 64, 64)) return QLORA_ERR_CUDA;
        p.late_wait = late_wait;
        dim3 grid = schedule_pair<DQ_B_MN, 4>(p, ceil_div(a.K, 256), ceil_div(a.M, 512), L);
        if (launch_gemm_pair<DQ_B_MN, 4>(p, grid, s, QLORA_KERNEL_DX_GEMM) != cudaSuccess) return QLORA_ERR_CUDA;
    } else {
        dim3 grid = schedule_gemm(p, ceil_div(a.K, 256), ceil_div(a.M, 256), L);
        if (launch_gemm<256, 0, 1, DQ_B_MN, EPI_BF16, 3, 2>(p, grid, s, QLORA_KERNEL_DX_GEMM) != cudaSuccess)
            return QLORA_ERR_CUDA;
    }
    return QLORA_OK;
}

// The backward forks its adapter GEMMs onto the side stream when the dX GEMM
// runs on the CTA-pair kernel, one pair per tile.
inline bool side_fork_ok() { return large_m_schedule() == SCHED_PAIR; }

// Backward with dX and an adapter, on the caller's stream s and the side
// stream:
//   s:    expansion -> sG (one CTA per 128-token tile, after the expansion)
//         -> dX GEMM (starts beside the sG kernel, waits for sG only before
//         its LoRA k-step) -> wait for the side stream
//   side: wait for sG -> sU -> dA, dB (one CTA per tile each), on the SMs the
//         GEMM leaves free
inline qlora_status linear_bwd_forked(const void* dY, const void* X, const LinearArgs& a, const void* A,
                                      const void* B, void* dX, float* dA, float* dB, const LinearWs& L,
                                      const CUtensorMap& tdY, const SideStream& side, cudaStream_t s) {
    SkinnyDesc dg;
    if (!desc_sG(&dg, tdY, a, B, L.sG)) return QLORA_ERR_CUDA;
    qlora_status st = skinny(&dg, 1, a.rt(), s, 1, SKP_PACKED);
    if (st != QLORA_OK) return st;
    if (cudaEventRecord(side.fork, s) != cudaSuccess) return QLORA_ERR_CUDA;
    if (cudaStreamWaitEvent(side.st, side.fork, 0) != cudaSuccess) return QLORA_ERR_CUDA;
    // from here on the side stream is joined back whatever happens
    st = launch_dx_gemm(A, dX, a, L, tdY, 1, s);
    // sU, dA and dB in one persistent launch over every SM: the CTAs that
    // find an SM beside the GEMM take tiles from the shared counter while it
    // runs, the rest start as it ends.  sU tiles (inputs only) start at once,
    // dA tiles wait for sG (the kernel before), dB tiles for the sU tiles.
    SkinnyDesc d3[3];
    if (st == QLORA_OK && !desc_sU(&d3[0], X, a, A, L.sU)) st = QLORA_ERR_CUDA;
    if (st == QLORA_OK && !desc_dA_dB(d3 + 1, dY, X, a, L, dA, dB)) st = QLORA_ERR_CUDA;
    if (st == QLORA_OK)
        st = skinny(d3, 3, a.rt(), side.st, 0, SKP_STREAM, sm_count(), L.sk_flags + kMaxStreamK, 2, 1 << 1);
    if (cudaEventRecord(side.join, side.st) != cudaSuccess || cudaStreamWaitEvent(s, side.join, 0) != cudaSuccess)
        st = QLORA_ERR_CUDA;
    return st;
}

inline qlora_status linear_bwd_impl(const void* dY, const void* X, const LinearArgs& a,
                                    const void* A, const void* B, void* dX, float* dA, float* dB,
                                    void* ws, size_t ws_bytes, cudaStream_t s) {
    (void)ws_bytes;
    const qlora_nf4_weight& w = *a.w;
    LinearWs L = carve_linear_ws(ws, a.M, a.N, a.K, a.rt(), 1);
    if (a.M == 0) {
        if (a.r > 0) {
            note_launch();
            k_fill_zero_f32<<<64, 256, 0, s>>>(dA, (int64_t)a.rt() * a.K);
            note_launch();
            k_fill_zero_f32<<<64, 256, 0, s>>>(dB, a.N * a.r);
            if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
        }
        return QLORA_OK;
    }
    if (dX && launch_expand_scales(w, L.scales, L.scales_ld, s, L.sk_flags, kMaxStreamK + 2) != cudaSuccess)
        return QLORA_ERR_CUDA;
    CUtensorMap tdY;
    if (!map_bf16(&tdY, dY, a.N, a.M, 128)) return QLORA_ERR_CUDA;
    SideStream side{nullptr, nullptr, nullptr};
    if (dX && a.r > 0 && side_fork_ok() && side_stream_acquire(s, &side)) {
        const qlora_status st = linear_bwd_forked(dY, X, a, A, B, dX, dA, dB, L, tdY, side, s);
        side_stream_release();
        return st;
    }
    // serial path: sU and sG in one launch, dX GEMM, dA and dB
    if (a.r > 0) {
        SkinnyDesc d[2];
        if (!desc_sU(&d[0], X, a, A, L.sU)) return QLORA_ERR_CUDA;
        if (!desc_sG(&d[1], tdY, a, B, L.sG)) return QLORA_ERR_CUDA;
        // waits for the kernel before (the expansion, a dependent launch that
        // lets this one start early) before it loads: the workspace it writes
        // may still be read by the call before
        qlora_status st = skinny(d, 2, a.rt(), s, 1);
        if (st != QLORA_OK) return st;
    }
    if (dX) {
        qlora_status st = launch_dx_gemm(A, dX, a, L, tdY, 0, s);
        if (st != QLORA_OK) return st;
    }
    if (a.r > 0) {
        SkinnyDesc d[2];
        if (!desc_dA_dB(d, dY, X, a, L, dA, dB)) return QLORA_ERR_CUDA;
        // sG and sU come from the LoRA GEMMs above
        qlora_status st = skinny(d, 2, a.rt(), s, 1);
        if (st != QLORA_OK) return st;
    }
    return QLORA_OK;
}

}  // namespace qlora
