// internal.h -- launchers shared between the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qlora_nf4.h"

namespace qlora {

// Launch accounting and optional event timing of tracked kernels.
void note_launch();
struct ProfileScope {
    int kind;
    cudaStream_t s;
    int slot;
    ProfileScope(int kind, cudaStream_t s);
    ~ProfileScope();
};

// Bound of every in-kernel wait of the next launches (ns).
uint64_t wait_timeout_ns();
int inject_mode();

// Per-device side stream of the backward: work that does not feed the next
// kernel of the caller's stream (dA, dB) runs there, beside the dX GEMM, on
// the SMs that the GEMM's grid leaves idle.  side_stream_acquire returns
// false (serial path) when the side stream cannot be used: test mode 6, a
// first use while the caller's stream is capturing, or a failed creation.
// On true the side-stream lock is held until side_stream_release().
struct SideStream {
    cudaStream_t st;
    cudaEvent_t fork, join;
};
bool side_stream_acquire(cudaStream_t s, SideStream* out);
void side_stream_release();

// ---- quantizer (quantize.cuh) ----
// Host-built search table of the fast nearest-code search (33 buckets of
// width 1/16 over [-1, 1]; bucket k holds the x with RN(64 x + 64) in
// [4k, 4k + 3], see quantize.cuh): per bucket the largest fp32 below its
// decision threshold (3.0 without one) and the count of thresholds below the
// bucket.
// inc: how many thresholds sit at the bucket's one threshold value (1; 2 for
// the FP4 code book, whose +0 code is never chosen, so that its threshold
// coincides with the next one).
constexpr int kSearchBuckets = 33;
struct Nf4SearchTable {
    float thr[kSearchBuckets];
    int base[kSearchBuckets];
    int inc[kSearchBuckets];
};
const Nf4SearchTable& nf4_search_table();
void nf4_table_host(float out[16]);
cudaError_t launch_dequantize(const qlora_nf4_weight& w, uint16_t* out, cudaStream_t s);
cudaError_t launch_encode(const float* x, int64_t n, uint8_t* codes, cudaStream_t s);

// Block constants a' of a weight, written transposed as scales[kb * ld + n]
// (kb = block column, n = row) for the GEMM producers.
cudaError_t launch_expand_scales(const qlora_nf4_weight& w, float* scales, int64_t ld,
                                 cudaStream_t s, int* flags, int nflags);

// ---- GEMMs (gemm.cu) ----
// r is the rank of each adapter.  A fused projection (nseg > 1) is one
// weight whose N rows are nseg segments of seg_rows rows that share the
// input X, segment i with its own adapter: rows i*r .. i*r + r - 1 of
// A [nseg*r][K] and rows i*seg_rows .. of B [N][r].
struct LinearArgs {
    int64_t M, N, K;
    int r;
    float scale;
    const qlora_nf4_weight* w;
    int nseg;
    int64_t seg_rows;
    int rt() const { return r * nseg; }  // columns of sU and sG
};
qlora_status linear_fwd_impl(const void* X, const LinearArgs& a, const void* A, const void* B,
                             void* Y, void* ws, size_t ws_bytes, cudaStream_t s);
qlora_status linear_bwd_impl(const void* dY, const void* X, const LinearArgs& a, const void* A,
                             const void* B, void* dX, float* dA, float* dB, void* ws,
                             size_t ws_bytes, cudaStream_t s);
size_t linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int r, int bwd);

}  // namespace qlora
