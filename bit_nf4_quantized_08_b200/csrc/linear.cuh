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
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "skinny.cuh"
#include "internal.h"
#include "quantize.cuh"

namespace qlora {

// ---------------------------------------------------------------------------
// tensor maps
// ---------------------------------------------------------------------------
typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);

inline PFN_encodeTiled_t encode_fn() {
    static PFN_encodeTiled_t fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled_t>(p);
    });
    return fn;
}

// 2-D tiled map over a row-major [outer][inner] tensor.
inline bool make_map(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int esize,
                     uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                     uint32_t box_outer, CUtensorMapSwizzle swz) {
    PFN_encodeTiled_t fn = encode_fn();
    if (!fn) return false;
    (void)esize;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

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
template <int BN, int STAGES>
inline cudaError_t launch_skinny(const SkinnyParams& p, int tiles, int cs, cudaStream_t s) {
    constexpr int smem = skinny_smem_bytes<BN, STAGES>();
    static_assert(smem <= 232448, "shared memory per CTA");
    auto kern = k_skinny<BN, STAGES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(tiles * cs), 1, 1);
    cfg.blockDim = dim3(SkinnyShape<BN>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    note_launch();
    return cudaLaunchKernelEx(&cfg, kern, p);
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
};

inline qlora_status skinny(const SkinnyDesc* d, int nprob, int r, cudaStream_t s) {
    SkinnyParams p;
    memset(&p, 0, sizeof(p));
    int tiles = 0, kmin = 1 << 30;
    for (int i = 0; i < nprob; ++i) {
        tiles += ceil_div(d[i].rows, 128);
        kmin = std::min(kmin, d[i].ksteps);
    }
    // clusters of up to 8 CTAs, two resident CTAs per SM, >= 2 k-steps per CTA
    int cs = 8;
    while (cs > 1 && ((int64_t)tiles * cs > 2 * 148 || kmin < 2 * cs)) cs >>= 1;
    for (int i = 0; i < nprob; ++i) {
        SkinnyProblem& q = p.pr[i];
        q.tmA = d[i].tA;
        q.tmB = d[i].tB;
        q.a_mn = d[i].a_mn;
        q.b_mn = d[i].b_mn;
        q.rows = d[i].rows;
        q.r = r;
        q.ksteps = d[i].ksteps;
        q.per = ceil_div(d[i].ksteps, cs);
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
    if (bn == 64)
        e = launch_skinny<64, 4>(p, tiles, cs, s);
    else if (bn == 128)
        e = launch_skinny<128, 4>(p, tiles, cs, s);
    else
        e = launch_skinny<256, 3>(p, tiles, cs, s);
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

inline size_t small_m_part_bytes(int64_t M, int64_t N, int64_t K) {
    int splits, per;
    choose_splits(ceil_div(N, 128), (int)(K / 64), &splits, &per);
    return splits > 1 ? (size_t)splits * M * N * 4 : 0;
}

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
    float* part;
    float* sk_part;  // stream-K partial tiles [kMaxStreamK][256*256]
    int* sk_flags;   // [kMaxStreamK]
    size_t bytes;
};

inline LinearWs carve_linear_ws(void* ws, int64_t M, int64_t N, int64_t K, int r, int bwd) {
    WsCarve c{static_cast<char*>(ws), 0};
    LinearWs L;
    L.scales_ld = ((N + 255) / 256) * 256;
    L.scales = static_cast<float*>(c.take((size_t)(K / 64) * L.scales_ld * 4));
    L.sU = r > 0 ? static_cast<uint16_t*>(c.take((size_t)M * r * 2)) : nullptr;
    L.sG = (r > 0 && bwd) ? static_cast<uint16_t*>(c.take((size_t)M * r * 2)) : nullptr;
    size_t part = 0;
    if (!bwd && M <= kSmallM) part = small_m_part_bytes(M, N, K);
    L.part = part ? static_cast<float*>(c.take(part)) : nullptr;
    const bool big = bwd || M > kSmallM;
    L.sk_part = big ? static_cast<float*>(c.take((size_t)kMaxStreamK * 256 * 256 * 4)) : nullptr;
    L.sk_flags = big ? static_cast<int*>(c.take((size_t)kMaxStreamK * 4)) : nullptr;
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
    auto kern = k_gemm_pair<DQ, STAGES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ProfileScope ps(prof_kind, s);
    note_launch();
    kern<<<grid, PairShape<DQ>::THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

// Which large-M GEMM runs: CTA pairs (default), or the single-CTA kernel on
// the grid or stream-K schedule.  QLORA_SCHEDULE=pair|grid|streamk selects
// one; test mode 2 forces stream-K, test mode 3 the single-CTA grid.
enum { SCHED_PAIR = 0, SCHED_GRID = 1, SCHED_STREAMK = 2 };
inline int large_m_schedule() {
    if (inject_mode() == 2) return SCHED_STREAMK;
    if (inject_mode() == 3) return SCHED_GRID;
    static int v = [] {
        const char* e = getenv("QLORA_SCHEDULE");
        if (!e) return (int)SCHED_PAIR;
        if (!strcmp(e, "grid")) return (int)SCHED_GRID;
        if (!strcmp(e, "streamk")) return (int)SCHED_STREAMK;
        return (int)SCHED_PAIR;
    }();
    return v;
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
inline bool desc_sU(SkinnyDesc* d, const void* X, const LinearArgs& a, const void* A, void* sU) {
    memset(d, 0, sizeof(*d));
    if (!map_bf16(&d->tA, X, a.K, a.M, 128)) return false;
    if (!map_bf16(&d->tB, A, a.K, a.r, lora_bn(a.r))) return false;
    d->rows = (int)a.M;
    d->ksteps = (int)(a.K / 64);
    d->scale = a.scale;
    d->out_mode = SK_OUT_BF16;
    d->out = sU;
    d->out_ld = a.r;
    return true;
}

inline qlora_status linear_fwd_impl(const void* X, const LinearArgs& a, const void* A,
                                    const void* B, void* Y, void* ws, size_t ws_bytes,
                                    cudaStream_t s) {
    (void)ws_bytes;
    const qlora_nf4_weight& w = *a.w;
    LinearWs L = carve_linear_ws(ws, a.M, a.N, a.K, a.r, 0);
    if (launch_expand_scales(w, L.scales, L.scales_ld, s, L.sk_flags, L.sk_flags ? kMaxStreamK : 0) !=
        cudaSuccess)
        return QLORA_ERR_CUDA;
    if (a.r > 0) {
        SkinnyDesc d;
        if (!desc_sU(&d, X, a, A, L.sU)) return QLORA_ERR_CUDA;
        qlora_status st = skinny(&d, 1, a.r, s);
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
    if (a.M > kSmallM) {
        // Y = [X | sU] [W' | B]^T : 128 x 256 tiles, W' dequantized into the B slot.
        if (!map_bf16(&p.tmA, X, a.K, a.M, 128)) return QLORA_ERR_CUDA;
        p.tmB = p.tmA;
        if (!map_codes(&p.tmCodes, w, 32, 256)) return QLORA_ERR_CUDA;
        if (a.r > 0) {
            if (!map_bf16(&p.tmA2, L.sU, a.r, a.M, 128)) return QLORA_ERR_CUDA;
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
        if (large_m_schedule() == SCHED_PAIR) {
            if (!map_codes(&p.tmCodes, w, 32, 128)) return QLORA_ERR_CUDA;
            if (a.r > 0 && !map_bf16(&p.tmB2, B, a.r, a.N, 128)) return QLORA_ERR_CUDA;
            dim3 grid(2 * ceil_div(a.N, 256), ceil_div(a.M, 512), 1);
            if (launch_gemm_pair<DQ_B_K, 4>(p, grid, s, QLORA_KERNEL_FWD_GEMM) != cudaSuccess)
                return QLORA_ERR_CUDA;
            return QLORA_OK;
        }
        dim3 grid = schedule_gemm(p, ceil_div(a.N, 256), ceil_div(a.M, 256), L);
        if (launch_gemm<256, 0, 0, DQ_B_K, EPI_BF16, 3, 2>(p, grid, s, QLORA_KERNEL_FWD_GEMM) != cudaSuccess)
            return QLORA_ERR_CUDA;
        return QLORA_OK;
    }
    // small M: Y^T = [W' | B] [X | sU]^T, weight rows on the 128-lane side.
    const int bn = a.M <= 32 ? 32 : 64;
    if (!map_bf16(&p.tmB, X, a.K, a.M, bn)) return QLORA_ERR_CUDA;
    p.tmA = p.tmB;
    if (!map_codes(&p.tmCodes, w, 32, 128)) return QLORA_ERR_CUDA;
    if (a.r > 0) {
        if (!map_bf16(&p.tmA2, B, a.r, a.N, 128)) return QLORA_ERR_CUDA;
        if (!map_bf16(&p.tmB2, L.sU, a.r, a.M, bn)) return QLORA_ERR_CUDA;
    } else {
        p.tmA2 = p.tmB;
        p.tmB2 = p.tmB;
    }
    const int tiles = ceil_div(a.N, 128);
    int splits, per;
    choose_splits(tiles, p.ks_main, &splits, &per);
    p.ks_per_split = per;
    p.rows = (int)a.N;
    p.cols = (int)a.M;
    dim3 grid(1, tiles, splits);
    cudaError_t e;
    if (splits == 1) {
        p.out_ld = a.N;
        if (bn == 32)
            e = launch_gemm<32, 0, 0, DQ_A_K, EPI_BF16_T, 6>(p, grid, s, QLORA_KERNEL_SMALLM_GEMM);
        else
            e = launch_gemm<64, 0, 0, DQ_A_K, EPI_BF16_T, 6>(p, grid, s, QLORA_KERNEL_SMALLM_GEMM);
        return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
    }
    p.out = L.part;
    p.out_ld = a.N;
    p.out_split_stride = a.M * a.N;
    if (bn == 32)
        e = launch_gemm<32, 0, 0, DQ_A_K, EPI_F32_T, 6>(p, grid, s, QLORA_KERNEL_SMALLM_GEMM);
    else
        e = launch_gemm<64, 0, 0, DQ_A_K, EPI_F32_T, 6>(p, grid, s, QLORA_KERNEL_SMALLM_GEMM);
    if (e != cudaSuccess) return QLORA_ERR_CUDA;
    const int64_t total = a.M * a.N;
    note_launch();
    k_splitk_reduce<<<ceil_div(total, 256), 256, 0, s>>>(L.part, splits, a.M * a.N, (int)a.M,
                                                         (int)a.N, a.N, 1.0f, RED_BF16, Y, a.N);
    return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

inline qlora_status linear_bwd_impl(const void* dY, const void* X, const LinearArgs& a,
                                    const void* A, const void* B, void* dX, float* dA, float* dB,
                                    void* ws, size_t ws_bytes, cudaStream_t s) {
    (void)ws_bytes;
    const qlora_nf4_weight& w = *a.w;
    LinearWs L = carve_linear_ws(ws, a.M, a.N, a.K, a.r, 1);
    if (a.M == 0) {
        if (a.r > 0) {
            note_launch();
            k_fill_zero_f32<<<64, 256, 0, s>>>(dA, (int64_t)a.r * a.K);
            note_launch();
            k_fill_zero_f32<<<64, 256, 0, s>>>(dB, a.N * a.r);
            if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
        }
        return QLORA_OK;
    }
    if (dX && launch_expand_scales(w, L.scales, L.scales_ld, s, L.sk_flags, kMaxStreamK) != cudaSuccess)
        return QLORA_ERR_CUDA;
    CUtensorMap tdY;
    if (!map_bf16(&tdY, dY, a.N, a.M, 128)) return QLORA_ERR_CUDA;
    if (a.r > 0) {
        // sU = bf16(scale X A^T) and sG = bf16(scale dY B) in one launch;
        // sG: Aop = dY [m][n] (K-major), Bop = B viewed [j][n] (MN-major)
        SkinnyDesc d[2];
        if (!desc_sU(&d[0], X, a, A, L.sU)) return QLORA_ERR_CUDA;
        memset(&d[1], 0, sizeof(d[1]));
        d[1].tA = tdY;
        if (!map_bf16(&d[1].tB, B, a.r, a.N, 64)) return QLORA_ERR_CUDA;
        d[1].b_mn = 1;
        d[1].rows = (int)a.M;
        d[1].ksteps = ceil_div(a.N, 64);
        d[1].scale = a.scale;
        d[1].out_mode = SK_OUT_BF16;
        d[1].out = L.sG;
        d[1].out_ld = a.r;
        qlora_status st = skinny(d, 2, a.r, s);
        if (st != QLORA_OK) return st;
    }
    if (dX) {
        GemmParams p;
        memset(&p, 0, sizeof(p));
        p.tmA = tdY;
        p.tmB = tdY;
        if (!map_codes(&p.tmCodes, w, 128, 64)) return QLORA_ERR_CUDA;
        if (a.r > 0) {
            if (!map_bf16(&p.tmA2, L.sG, a.r, a.M, 128)) return QLORA_ERR_CUDA;
            if (!map_bf16(&p.tmB2, A, a.K, a.r, 64)) return QLORA_ERR_CUDA;
        } else {
            p.tmA2 = tdY;
            p.tmB2 = tdY;
        }
        p.scales = L.scales;
        p.scales_ld = L.scales_ld;
        p.dq_rows = (int)a.N;
        p.dq_kbs = (int)(a.K / 64);
        p.ks_main = ceil_div(a.N, 64);
        p.ks_lora = a.r > 0 ? ceil_div(a.r, 64) : 0;
        p.ks_per_split = p.ks_main;
        p.rows = (int)a.M;
        p.cols = (int)a.K;
        p.out = dX;
        p.out_ld = a.K;
        if (!map_bf16(&p.tmOut, dX, a.K, a.M, 128)) return QLORA_ERR_CUDA;
        p.timeout_ns = wait_timeout_ns();
        p.inject = inject_mode() == 1 ? 1 : 0;
        if (large_m_schedule() == SCHED_PAIR) {
            if (!map_codes(&p.tmCodes, w, 64, 64)) return QLORA_ERR_CUDA;
            dim3 grid(2 * ceil_div(a.K, 256), ceil_div(a.M, 512), 1);
            if (launch_gemm_pair<DQ_B_MN, 4>(p, grid, s, QLORA_KERNEL_DX_GEMM) != cudaSuccess)
                return QLORA_ERR_CUDA;
        } else {
            dim3 grid = schedule_gemm(p, ceil_div(a.K, 256), ceil_div(a.M, 256), L);
            if (launch_gemm<256, 0, 1, DQ_B_MN, EPI_BF16, 3, 2>(p, grid, s, QLORA_KERNEL_DX_GEMM) != cudaSuccess)
                return QLORA_ERR_CUDA;
        }
    }
    if (a.r > 0) {
        // dA^T [K][r] = X^T sG : Aop = X viewed [k][m] (MN-major), Bop = sG viewed [j][m] (MN-major)
        // dB [N][r] = dY^T sU : Aop = dY viewed [n][m] (MN-major), Bop = sU viewed [j][m]
        // (both in one launch)
        SkinnyDesc d[2];
        memset(d, 0, sizeof(d));
        if (!map_bf16(&d[0].tA, X, a.K, a.M, 64)) return QLORA_ERR_CUDA;
        if (!map_bf16(&d[0].tB, L.sG, a.r, a.M, 64)) return QLORA_ERR_CUDA;
        d[0].rows = (int)a.K;
        d[0].out_mode = SK_OUT_F32_T;
        d[0].out = dA;
        d[0].out_ld = a.K;
        if (!map_bf16(&d[1].tA, dY, a.N, a.M, 64)) return QLORA_ERR_CUDA;
        if (!map_bf16(&d[1].tB, L.sU, a.r, a.M, 64)) return QLORA_ERR_CUDA;
        d[1].rows = (int)a.N;
        d[1].out_mode = SK_OUT_F32;
        d[1].out = dB;
        d[1].out_ld = a.r;
        for (int i = 0; i < 2; ++i) {
            d[i].a_mn = 1;
            d[i].b_mn = 1;
            d[i].ksteps = ceil_div(a.M, 64);
            d[i].scale = 1.0f;
        }
        qlora_status st = skinny(d, 2, a.r, s);
        if (st != QLORA_OK) return st;
    }
    return QLORA_OK;
}

}  // namespace qlora
