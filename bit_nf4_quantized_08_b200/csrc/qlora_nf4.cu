// qlora_nf4.cu -- the C ABI of include/qlora_nf4.h: argument validation,
// workspace queries, the device status word, and dispatch to the kernels.
// Single translation unit: the kernel headers below are compiled here.
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include <math.h>

#include <nvtx3/nvToolsExt.h>

#include "../../include/qlora_nf4.h"
#include "adamw.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "internal.h"
#include "linear.cuh"
#include "merge.cuh"
#include "nf4.cuh"
#include "quantize.cuh"

namespace qlora {


static std::atomic<uint64_t> g_timeout_ns{10ull * 1000 * 1000 * 1000};
static std::atomic<int> g_inject{0};

static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// Event timing of tracked kernels (enabled by qlora_profile_enable).
struct ProfRecord {
    int kind;
    cudaEvent_t start, stop;
};
static std::mutex g_prof_mu;
static std::atomic<int> g_prof_on{0};
static std::vector<ProfRecord> g_prof;  // recorded pairs, in launch order
static std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_prof_pool;
static size_t g_prof_used = 0;

ProfileScope::ProfileScope(int k, cudaStream_t st) : kind(k), s(st), slot(-1) {
    if (k < 0 || !g_prof_on.load()) return;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (g_prof_used == g_prof_pool.size()) {
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess) return;
        if (cudaEventCreate(&b) != cudaSuccess) return;
        g_prof_pool.push_back({a, b});
    }
    auto pr = g_prof_pool[g_prof_used++];
    slot = (int)g_prof.size();
    g_prof.push_back({kind, pr.first, pr.second});
    cudaEventRecord(pr.first, s);
}

ProfileScope::~ProfileScope() {
    if (slot < 0) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEventRecord(g_prof[slot].stop, s);
}

uint64_t wait_timeout_ns() { return g_timeout_ns.load(); }
int inject_mode() { return g_inject.load(); }

static std::mutex g_side_mu;
struct SideSlot {
    bool tried;
    SideStream ss;
};
static SideSlot g_side[64];

bool side_stream_acquire(cudaStream_t s, SideStream* out) {
    if (inject_mode() == 6) return false;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return false;
    }
    g_side_mu.lock();
    SideSlot& slot = g_side[dev];
    if (!slot.tried) {
        // streams and events are not created inside a stream capture
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(s, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
            cudaGetLastError();
            g_side_mu.unlock();
            return false;
        }
        slot.tried = true;
        SideStream ss{nullptr, nullptr, nullptr};
        if (cudaStreamCreateWithFlags(&ss.st, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) == cudaSuccess) {
            slot.ss = ss;
        } else {
            cudaGetLastError();
            slot.ss = SideStream{nullptr, nullptr, nullptr};
        }
    }
    if (!slot.ss.st) {
        g_side_mu.unlock();
        return false;
    }
    *out = slot.ss;
    return true;
}

void side_stream_release() { g_side_mu.unlock(); }

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// An NVTX range named after the entry point around the host side of every
// call that launches work (header-only NVTX: a no-op unless a profiler or
// tracer is attached), so that timelines group each call's kernels.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

static const int64_t kMaxElems = (int64_t)1 << 40;

// Checks shared by every call that reads a quantized weight.
static qlora_status check_weight(const qlora_nf4_weight* w, bool need_codes) {
    if (!w) return QLORA_ERR_INVALID_ARG;
    if (w->rows < 0 || w->cols < 0) return QLORA_ERR_INVALID_ARG;
    if (w->rows > 0 && w->cols > kMaxElems / w->rows) return QLORA_ERR_INVALID_ARG;
    if (w->double_quant != 0 && w->double_quant != 1) return QLORA_ERR_INVALID_ARG;
    if (w->code_type != QLORA_CODE_NF4 && w->code_type != QLORA_CODE_FP4) return QLORA_ERR_INVALID_ARG;
    if (w->dq_type != QLORA_DQ_INT8 && w->dq_type != QLORA_DQ_FP8) return QLORA_ERR_INVALID_ARG;
    if (w->blocksize != 64 && w->blocksize != 128 && w->blocksize != 256) return QLORA_ERR_UNSUPPORTED;
    const int64_t n = w->rows * w->cols;
    if (n == 0) return QLORA_OK;
    if (need_codes && (!w->codes || !aligned(w->codes, 16))) return QLORA_ERR_INVALID_ARG;
    if (w->double_quant) {
        if (!w->absmax_q8 || !aligned(w->absmax_q8, 8)) return QLORA_ERR_INVALID_ARG;
        if (!w->absmax_scale || !aligned(w->absmax_scale, 4)) return QLORA_ERR_INVALID_ARG;
        if (!w->absmax_offset || !aligned(w->absmax_offset, 4)) return QLORA_ERR_INVALID_ARG;
    } else {
        if (!w->absmax || !aligned(w->absmax, 4)) return QLORA_ERR_INVALID_ARG;
    }
    return QLORA_OK;
}

// Workspace of qlora_nf4_quantize with double quantization: block maxima
// [nb] f32, group sums [ng] f64, first-level offset partials (many groups).
static size_t quantize_ws(int64_t n, int dq, int64_t bs) {
    if (!dq || n == 0) return 0;
    const int64_t nb = (n + bs - 1) / bs;
    const int64_t ng = (n + 16383) / 16384;
    return align256((size_t)nb * 4) + align256((size_t)ng * 8) + align256((size_t)dq_partial_count(ng) * 8);
}

// Scratch of qlora_nf4_quantize_static: the fp32 maximum of every 64-element
// block, then the fp64 sum of every 16384-element group, for tensors of up to
// QLORA_STATIC_QUANTIZE_MAX_ELEMS elements.  A fixed device array so that the
// call needs no allocation; each call writes every slot it reads.
static constexpr int64_t kStaticAbsmaxBytes = (QLORA_STATIC_QUANTIZE_MAX_ELEMS / 64) * 4;
static constexpr int64_t kStaticSumsBytes = (QLORA_STATIC_QUANTIZE_MAX_ELEMS / 16384) * 8;
static __device__ __align__(256) unsigned char g_quant_scratch[kStaticAbsmaxBytes + kStaticSumsBytes];

// Device address of g_quant_scratch on the current device, looked up once
// per device ordinal and kept.
static constexpr int kMaxDevices = 64;
static std::atomic<void*> g_scratch_addr[kMaxDevices];
static std::mutex g_scratch_mu;

static qlora_status static_quant_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_UNSUPPORTED;
    void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lk(g_scratch_mu);
        p = g_scratch_addr[dev].load(std::memory_order_relaxed);
        if (!p) {
            if (cudaGetSymbolAddress(&p, g_quant_scratch) != cudaSuccess || !p) return QLORA_ERR_CUDA;
            g_scratch_addr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return QLORA_OK;
}

static qlora_status check_linear(int64_t M, const qlora_nf4_weight* w, int32_t r) {
    qlora_status st = check_weight(w, true);
    if (st != QLORA_OK) return st;
    if (M < 0 || M > ((int64_t)1 << 31)) return QLORA_ERR_INVALID_ARG;
    if (r < 0) return QLORA_ERR_INVALID_ARG;
    if (w->cols < 64 || w->rows < 1) return QLORA_ERR_UNSUPPORTED;
    if (w->cols % 64 != 0 || w->rows % 8 != 0) return QLORA_ERR_UNSUPPORTED;
    if (w->rows >= ((int64_t)1 << 31) || w->cols >= ((int64_t)1 << 31)) return QLORA_ERR_UNSUPPORTED;
    if (r % 8 != 0 || r > 256) return QLORA_ERR_UNSUPPORTED;
    return QLORA_OK;
}

// LoRA merge (base = NF4 weight) or unmerge (base = dense bf16 weight):
// out = bf16(base + scale * B A), one CTA per 128 x 128 tile.
static qlora_status lora_merge_impl(const qlora_nf4_weight* w, const void* dense, int64_t N, int64_t K,
                                    const void* A, const void* B, int32_t r, float scale, void* out,
                                    cudaStream_t s) {
    MergeParams p;
    memset(&p, 0, sizeof(p));
    if (!map_bf16(&p.tmB, B, (uint64_t)r, (uint64_t)N, 128)) return QLORA_ERR_CUDA;
    if (!map_bf16(&p.tmA, A, (uint64_t)K, (uint64_t)r, 64)) return QLORA_ERR_CUDA;
    if (w) {
        p.fmt = weight_format(*w);
        p.codes = w->codes;
        p.dq = w->double_quant;
        p.absmax = w->absmax;
        p.q8 = w->absmax_q8;
        p.c1 = w->absmax_scale;
        p.offset = w->absmax_offset;
    } else {
        p.dense = static_cast<const uint16_t*>(dense);
    }
    p.out = static_cast<uint16_t*>(out);
    p.N = (int)N;
    p.K = (int)K;
    p.r_chunks = (r + 63) / 64;
    p.scale = scale;
    p.timeout_ns = wait_timeout_ns();
    const int smem = MergeShape::smem(p.r_chunks);
    if (cudaFuncSetAttribute(k_lora_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, MergeShape::MAX_SMEM) !=
        cudaSuccess)
        return QLORA_ERR_CUDA;
    dim3 grid((unsigned)((K + 127) / 128), (unsigned)((N + 127) / 128));
    ProfileScope ps(QLORA_KERNEL_MERGE, s);
    note_launch();
    k_lora_merge<<<grid, MergeShape::THREADS, smem, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

static qlora_status check_merge(int64_t N, int64_t K, const void* A, const void* B, int32_t r,
                                const void* out) {
    if (N < 0 || K < 0 || r < 1) return QLORA_ERR_INVALID_ARG;
    if (N == 0 || K == 0) return QLORA_OK;
    if (K % 64 != 0 || N % 8 != 0 || r % 8 != 0 || r > 256) return QLORA_ERR_UNSUPPORTED;
    if (N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31) || N > kMaxElems / K) return QLORA_ERR_UNSUPPORTED;
    if (!A || !aligned(A, 16) || !B || !aligned(B, 16) || !out || !aligned(out, 16))
        return QLORA_ERR_INVALID_ARG;
    return QLORA_OK;
}

// A fused projection: nseg equal row segments, each segment a whole number
// of 256-row output tiles (so that no tile of any kernel straddles two
// adapters), nseg * r <= 256 adapter columns in all.
static qlora_status check_fused(int64_t M, const qlora_nf4_weight* w, int32_t nseg, int32_t r) {
    qlora_status st = check_linear(M, w, r);
    if (st != QLORA_OK) return st;
    if (nseg < 1) return QLORA_ERR_INVALID_ARG;
    if (nseg == 1) return QLORA_OK;
    if (nseg > 8 || w->rows % nseg != 0 || (w->rows / nseg) % 256 != 0 || (int64_t)nseg * r > 256)
        return QLORA_ERR_UNSUPPORTED;
    return QLORA_OK;
}

}  // namespace qlora

using namespace qlora;

extern "C" {

size_t qlora_nf4_quantize_workspace(int64_t rows, int64_t cols, int32_t blocksize,
                                    int32_t double_quant) {
    if (rows < 0 || cols < 0 || (blocksize != 64 && blocksize != 128 && blocksize != 256)) return 0;
    if (rows > 0 && cols > kMaxElems / rows) return 0;
    return quantize_ws(rows * cols, double_quant, blocksize);
}

qlora_status qlora_nf4_quantize(const void* W, qlora_dtype wdtype, const qlora_nf4_weight* out,
                                void* ws, size_t ws_bytes, qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_nf4_quantize");
    qlora_status st = check_weight(out, true);
    if (st != QLORA_OK) return st;
    if (wdtype != QLORA_F32 && wdtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
    const int64_t n = out->rows * out->cols;
    if (n == 0) return QLORA_OK;
    if (!W || !aligned(W, 16)) return QLORA_ERR_INVALID_ARG;
    if (!out->double_quant && (!out->absmax || !aligned(out->absmax, 4))) return QLORA_ERR_INVALID_ARG;
    const size_t need = quantize_ws(n, out->double_quant, out->blocksize);
    if (need > 0 && (!ws || !aligned(ws, 16) || ws_bytes < need)) return QLORA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int is_bf16 = wdtype == QLORA_BF16;
    const int64_t nb = (n + out->blocksize - 1) / out->blocksize;
    const QFormat fmt = weight_format(*out);
    if (!out->double_quant) {
        if (launch_quantize_blocks(W, is_bf16, n, out->codes, out->absmax, nullptr, s, fmt) != cudaSuccess)
            return QLORA_ERR_CUDA;
        return QLORA_OK;
    }
    float* absmax = static_cast<float*>(ws);
    double* sums = reinterpret_cast<double*>(static_cast<char*>(ws) + align256((size_t)nb * 4));
    const int64_t ng = (n + 16383) / 16384;
    double* partials = reinterpret_cast<double*>(reinterpret_cast<char*>(sums) + align256((size_t)ng * 8));
    if (launch_quantize_blocks(W, is_bf16, n, out->codes, absmax, sums, s, fmt) != cudaSuccess)
        return QLORA_ERR_CUDA;
    if (launch_double_quant(sums, ng, absmax, nb, out->absmax_offset, out->absmax_q8, out->absmax_scale, s,
                            partials, fmt.dq_type) != cudaSuccess)
        return QLORA_ERR_CUDA;
    return QLORA_OK;
}

qlora_status qlora_nf4_quantize_static(const void* W, qlora_dtype wdtype, const qlora_nf4_weight* out,
                                       qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_nf4_quantize_static");
    qlora_status st = check_weight(out, true);
    if (st != QLORA_OK) return st;
    if (wdtype != QLORA_F32 && wdtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
    const int64_t n = out->rows * out->cols;
    if (n == 0) return QLORA_OK;
    if (!W || !aligned(W, 16)) return QLORA_ERR_INVALID_ARG;
    if (n > QLORA_STATIC_QUANTIZE_MAX_ELEMS) return QLORA_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int is_bf16 = wdtype == QLORA_BF16;
    const QFormat fmt = weight_format(*out);
    if (!out->double_quant) {
        if (launch_quantize_blocks(W, is_bf16, n, out->codes, out->absmax, nullptr, s, fmt) != cudaSuccess)
            return QLORA_ERR_CUDA;
        return QLORA_OK;
    }
    void* scratch = nullptr;
    st = static_quant_scratch(&scratch);
    if (st != QLORA_OK) return st;
    const int64_t nb = (n + out->blocksize - 1) / out->blocksize;
    const int64_t ng = (n + 16383) / 16384;
    float* absmax = static_cast<float*>(scratch);
    double* sums = reinterpret_cast<double*>(static_cast<char*>(scratch) + kStaticAbsmaxBytes);
    if (launch_quantize_blocks(W, is_bf16, n, out->codes, absmax, sums, s, fmt) != cudaSuccess)
        return QLORA_ERR_CUDA;
    if (launch_double_quant(sums, ng, absmax, nb, out->absmax_offset, out->absmax_q8, out->absmax_scale, s,
                            nullptr, fmt.dq_type) != cudaSuccess)
        return QLORA_ERR_CUDA;
    return QLORA_OK;
}

qlora_status qlora_nf4_dequantize(const qlora_nf4_weight* w, void* out, qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_nf4_dequantize");
    qlora_status st = check_weight(w, true);
    if (st != QLORA_OK) return st;
    if (w->rows * w->cols == 0) return QLORA_OK;
    if (!out || !aligned(out, 16)) return QLORA_ERR_INVALID_ARG;
    if (launch_dequantize(*w, static_cast<uint16_t*>(out), reinterpret_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return QLORA_ERR_CUDA;
    return QLORA_OK;
}

size_t qlora_fused_linear_workspace(int64_t M, const qlora_nf4_weight* w, int32_t nseg, int32_t r,
                                    int32_t bwd) {
    if (check_fused(M, w, nseg, r) != QLORA_OK) return 0;
    return linear_workspace_bytes(M, w->rows, w->cols, r * nseg, bwd ? 1 : 0);
}

size_t qlora_linear_workspace(int64_t M, const qlora_nf4_weight* w, int32_t r, int32_t bwd) {
    return qlora_fused_linear_workspace(M, w, 1, r, bwd);
}

qlora_status qlora_fused_linear_fwd(const void* X, int64_t M, const qlora_nf4_weight* w, int32_t nseg,
                                    const void* A, const void* B, int32_t r, float scale, void* Y,
                                    void* ws, size_t ws_bytes, qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_fused_linear_fwd");
    qlora_status st = check_fused(M, w, nseg, r);
    if (st != QLORA_OK) return st;
    if (M == 0) return QLORA_OK;
    if (!X || !aligned(X, 16) || !Y || !aligned(Y, 16)) return QLORA_ERR_INVALID_ARG;
    if (r > 0 && (!A || !aligned(A, 16) || !B || !aligned(B, 16))) return QLORA_ERR_INVALID_ARG;
    const size_t need = linear_workspace_bytes(M, w->rows, w->cols, r * nseg, 0);
    if (!ws || !aligned(ws, 16) || ws_bytes < need) return QLORA_ERR_INVALID_ARG;
    LinearArgs a{M, w->rows, w->cols, r, scale, w, nseg, w->rows / nseg};
    return linear_fwd_impl(X, a, A, B, Y, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

qlora_status qlora_linear_fwd(const void* X, int64_t M, const qlora_nf4_weight* w, const void* A,
                              const void* B, int32_t r, float scale, void* Y, void* ws,
                              size_t ws_bytes, qlora_stream_t stream) {
    return qlora_fused_linear_fwd(X, M, w, 1, A, B, r, scale, Y, ws, ws_bytes, stream);
}

qlora_status qlora_fused_linear_bwd(const void* dY, const void* X, int64_t M, const qlora_nf4_weight* w,
                                    int32_t nseg, const void* A, const void* B, int32_t r, float scale,
                                    void* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                                    qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_fused_linear_bwd");
    qlora_status st = check_fused(M, w, nseg, r);
    if (st != QLORA_OK) return st;
    if (r > 0 && (!A || !aligned(A, 16) || !B || !aligned(B, 16) || !dA || !aligned(dA, 16) ||
                  !dB || !aligned(dB, 16)))
        return QLORA_ERR_INVALID_ARG;
    if (M > 0) {
        if (!dY || !aligned(dY, 16) || !X || !aligned(X, 16)) return QLORA_ERR_INVALID_ARG;
        if (dX && !aligned(dX, 16)) return QLORA_ERR_INVALID_ARG;
    }
    const size_t need = linear_workspace_bytes(M, w->rows, w->cols, r * nseg, 1);
    if (!ws || !aligned(ws, 16) || ws_bytes < need) return QLORA_ERR_INVALID_ARG;
    LinearArgs a{M, w->rows, w->cols, r, scale, w, nseg, w->rows / nseg};
    return linear_bwd_impl(dY, X, a, A, B, dX, dA, dB, ws, ws_bytes,
                           reinterpret_cast<cudaStream_t>(stream));
}

qlora_status qlora_linear_bwd(const void* dY, const void* X, int64_t M, const qlora_nf4_weight* w,
                              const void* A, const void* B, int32_t r, float scale, void* dX,
                              float* dA, float* dB, void* ws, size_t ws_bytes,
                              qlora_stream_t stream) {
    return qlora_fused_linear_bwd(dY, X, M, w, 1, A, B, r, scale, dX, dA, dB, ws, ws_bytes, stream);
}

qlora_status qlora_lora_merge(const qlora_nf4_weight* w, const void* A, const void* B, int32_t r,
                              float scale, void* W_merged, qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_lora_merge");
    qlora_status st = check_weight(w, true);
    if (st != QLORA_OK) return st;
    st = check_merge(w->rows, w->cols, A, B, r, W_merged);
    if (st != QLORA_OK || w->rows * w->cols == 0) return st;
    return lora_merge_impl(w, nullptr, w->rows, w->cols, A, B, r, scale, W_merged,
                           reinterpret_cast<cudaStream_t>(stream));
}

qlora_status qlora_lora_unmerge(const void* W_merged, int64_t rows, int64_t cols, const void* A,
                                const void* B, int32_t r, float scale, void* W_out,
                                qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_lora_unmerge");
    qlora_status st = check_merge(rows, cols, A, B, r, W_out);
    if (st != QLORA_OK || rows * cols == 0) return st;
    if (!W_merged || !aligned(W_merged, 16)) return QLORA_ERR_INVALID_ARG;
    return lora_merge_impl(nullptr, W_merged, rows, cols, A, B, r, -scale, W_out,
                           reinterpret_cast<cudaStream_t>(stream));
}

qlora_status qlora_adamw_step(float* param, float* exp_avg, float* exp_avg_sq, const float* grad,
                              void* param_bf16, int64_t n, const qlora_adamw_config* cfg,
                              qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_adamw_step");
    if (!cfg || n < 0) return QLORA_ERR_INVALID_ARG;
    if (cfg->step < 1 || !(cfg->lr >= 0.0f) || !(cfg->beta1 >= 0.0f && cfg->beta1 < 1.0f) ||
        !(cfg->beta2 >= 0.0f && cfg->beta2 < 1.0f) || !(cfg->eps > 0.0f) || !(cfg->weight_decay >= 0.0f))
        return QLORA_ERR_INVALID_ARG;
    if (n == 0) return QLORA_OK;
    if (!param || !exp_avg || !exp_avg_sq || !grad || !aligned(param, 16) || !aligned(exp_avg, 16) ||
        !aligned(exp_avg_sq, 16) || !aligned(grad, 16))
        return QLORA_ERR_INVALID_ARG;
    if (param_bf16 && !aligned(param_bf16, 8)) return QLORA_ERR_INVALID_ARG;
    AdamWParams a;
    a.p = param;
    a.m = exp_avg;
    a.v = exp_avg_sq;
    a.g = grad;
    a.p_bf16 = static_cast<uint16_t*>(param_bf16);
    a.n = n;
    a.lr = cfg->lr;
    a.b1 = cfg->beta1;
    a.b2 = cfg->beta2;
    a.eps = cfg->eps;
    a.decay = (float)(1.0 - (double)cfg->lr * (double)cfg->weight_decay);
    const double bc1 = 1.0 - pow((double)cfg->beta1, (double)cfg->step);
    const double bc2 = 1.0 - pow((double)cfg->beta2, (double)cfg->step);
    a.step_size = (float)((double)cfg->lr / bc1);
    a.rsqrt_bc2 = (float)(1.0 / sqrt(bc2));
    a.grad_scale = cfg->grad_scale;
    const int64_t nv = (n + 3) / 4;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((nv + 255) / 256, (int64_t)sm_count() * 8));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    note_launch();
    k_adamw<<<grid, 256, 0, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_paged_alloc(size_t bytes, void** ptr) {
    if (!ptr) return QLORA_ERR_INVALID_ARG;
    *ptr = nullptr;
    if (bytes == 0) return QLORA_OK;
    if (cudaMallocManaged(ptr, bytes, cudaMemAttachGlobal) != cudaSuccess) {
        cudaGetLastError();
        *ptr = nullptr;
        return QLORA_ERR_CUDA;
    }
    return QLORA_OK;
}

qlora_status qlora_paged_free(void* ptr) {
    if (!ptr) return QLORA_OK;
    return cudaFree(ptr) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_paged_prefetch(const void* ptr, size_t bytes, int32_t to_host, qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_paged_prefetch");
    if (!ptr && bytes) return QLORA_ERR_INVALID_ARG;
    if (bytes == 0) return QLORA_OK;
    int dev = 0;
    if (!to_host && cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
    if (cudaMemPrefetchAsync(ptr, bytes, to_host ? cudaCpuDeviceId : dev,
                             reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return QLORA_ERR_CUDA;
    }
    return QLORA_OK;
}

qlora_status qlora_get_last_error(qlora_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return QLORA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    if (v != 0) {
        int zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    return static_cast<qlora_status>(v);
}

void qlora_nf4_table(float out[16]) { nf4_table_host(out); }

qlora_status qlora_nf4_encode(const float* x, int64_t n, uint8_t* codes, qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_nf4_encode");
    if (n < 0) return QLORA_ERR_INVALID_ARG;
    if (n == 0) return QLORA_OK;
    if (!x || !codes || !aligned(x, 4)) return QLORA_ERR_INVALID_ARG;
    if (launch_encode(x, n, codes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return QLORA_ERR_CUDA;
    return QLORA_OK;
}

qlora_status qlora_dq_encode(const float* y, int64_t n, uint8_t* codes, int32_t dq_type, qlora_stream_t stream) {
    NvtxRange nvtx_range("qlora_dq_encode");
    if (n < 0 || (dq_type != QLORA_DQ_INT8 && dq_type != QLORA_DQ_FP8)) return QLORA_ERR_INVALID_ARG;
    if (n == 0) return QLORA_OK;
    if (!y || !codes || !aligned(y, 4)) return QLORA_ERR_INVALID_ARG;
    if (launch_dq_encode(y, n, codes, dq_type, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return QLORA_ERR_CUDA;
    return QLORA_OK;
}

void qlora_set_wait_timeout_ns(uint64_t ns) {
    g_timeout_ns.store(ns ? ns : 10ull * 1000 * 1000 * 1000);
}

void qlora_debug_inject(int32_t mode) { g_inject.store(mode); }

uint64_t qlora_kernel_launches(void) { return g_launches.load(); }

void qlora_profile_enable(int32_t on) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.clear();
    g_prof_used = 0;
    // create the event pairs up front, so that recording adds no event
    // creation to the measured launches
    while (on && g_prof_pool.size() < 2048) {
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess) break;
        if (cudaEventCreate(&b) != cudaSuccess) {
            cudaEventDestroy(a);
            break;
        }
        g_prof_pool.push_back({a, b});
    }
    g_prof_on.store(on ? 1 : 0);
}

qlora_status qlora_profile_read(int32_t kind, double* total_ms, int64_t* launches) {
    if (kind < 0 || kind >= QLORA_KERNEL_KINDS || !total_ms || !launches) return QLORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    double t = 0.0;
    int64_t n = 0;
    for (const auto& r : g_prof) {
        if (r.kind != kind) continue;
        if (cudaEventSynchronize(r.stop) != cudaSuccess) return QLORA_ERR_CUDA;
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) return QLORA_ERR_CUDA;
        t += ms;
        ++n;
    }
    *total_ms = t;
    *launches = n;
    return QLORA_OK;
}

}  // extern "C"
