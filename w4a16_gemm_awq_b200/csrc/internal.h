// internal.h -- launchers behind the C ABI (not part of the public interface).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "w4a16.h"

namespace w4a16 {

// Bits of the per-device status word that kernels set when they find a problem.
enum : unsigned { kErrValue = 1u, kErrShape = 2u, kErrTimeout = 4u };

// Group sizes the quantizer supports: 128, 256, 512, 1024, or a multiple of 1024 that
// divides K, up to kQuantMaxLargeGroup (its scales sit in shared memory).
constexpr int kQuantMaxLargeGroup = 32768;
bool quantize_group_size_ok(int K, int gs);

// bits: 4 (qweight [N][K/8]) or 3 (qweight [N][3K/32], group sizes up to 1024; see quantize.cu).
cudaError_t launch_awq_quantize(const float* W, const float* act, float alpha, int N, int K, int gs,
                                uint32_t* qweight, uint16_t* scales, uint32_t* zeros, float* s_out, int num_sms,
                                unsigned* err, cudaStream_t stream, int bits = 4);

// s_k = max(float(pow(a_k, alpha)), 1e-4) into s_out (quantize.cu).
cudaError_t launch_awq_scale(const float* act, float alpha, int K, float* s_out, unsigned* err, cudaStream_t stream);

// NVFP4 weights (see nvfp4.cu): qweight [N][K/8] E2M1 codes, scales8 [K/16][N] E4M3, *gscale
// the fp32 tensor scale, s_out [K] the channel scales.  N % 8 == 0, K % 16 == 0.
cudaError_t launch_awq_quantize_nvfp4(const float* W, const float* act, float alpha, int N, int K, uint32_t* qweight,
                                      uint8_t* scales8, float* gscale, float* s_out, int num_sms, unsigned* err,
                                      cudaStream_t stream);

// Decode GEMV on NVFP4 weights (see nvfp4.cu): 1 <= M <= 16, N % 16 == 0, K % 16 == 0.
cudaError_t launch_gemv_nvfp4(const uint16_t* x, const uint32_t* qweight, const uint8_t* scales8, const float* gscale,
                              uint16_t* y, int M, int N, int K, cudaStream_t stream);

// Tensor map the GEMV needs: qweight uint32 [N][K/8] seen as 3-D (16 words of a group,
// N rows, K/128 groups; strides K/2 and 64 bytes), box 16 x 128 x 4, no swizzle.  One copy
// brings 4 groups of 128 rows and lays them out group by group: [4][128 rows][64 bytes].
// For 3-bit codes: qweight [N][3K/32] as (12 words, N, K/128; strides 3K/8 and 48 bytes),
// box 12 x 128 x 4: [4][128 rows][48 bytes].
struct GemvMaps {
    CUtensorMap w;
};

// Largest K the GEMV supports.
int gemv_max_k();

// Whether the GEMV's 32-bit work-unit arithmetic covers this shape (units x CTAs < 2^32).
bool gemv_fits(int N, int K, int num_sms);

// One fp32 partial tile of the GEMV's workspace: 128 rows x 16 token columns.
constexpr int kGemvSlotFloats = 128 * 16;

// Device scratch of the GEMV: fp32 partial tiles (gemv_partial_bytes: two per SM, any
// contents) and one counter per row block (gemv_counter_bytes, 256-byte padded), which must be
// zero when a call starts; every call that completes leaves them zero.
size_t gemv_partial_bytes(int num_sms);
size_t gemv_counter_bytes(int N);

// A GEMV launch: schedule (W4A16_GEMV_STREAM_K or _CLUSTER), CTAs per cluster (0 for
// stream-K), clusters and CTAs of the grid.  ctas == 0: the requested schedule cannot run.
struct GemvPlan {
    int schedule;
    int cluster;
    int clusters;
    int ctas;
};

// The launch for a schedule (W4A16_GEMV_AUTO, _STREAM_K or _CLUSTER) on the current device.
GemvPlan gemv_plan(int M, int N, int K, int num_sms, int schedule);

// group_ratio: the quantization group size / 128 (1 for g128; K / 128 for one group per row).
// ysp: nullptr, or the CSR term [N][M] fp32 written by launch_csr_rows just before (the GEMV
// adds it to each output before rounding, after the previous kernel has finished).
// bits: 4, or 3 for 3-bit codes (qweight [N][3K/32], the map's inner extent 12 words a group).
cudaError_t launch_gemv(const GemvMaps& maps, const GemvPlan& plan, int group_ratio, const uint16_t* x,
                        const uint16_t* scales, const uint32_t* zeros, const float* ysp, uint16_t* y,
                        float* partials, unsigned* counters, int M, int N, int K, unsigned* err,
                        cudaStream_t stream, int bits = 4);

// The CSR term of the decode path: ysp[n][m] = sum_j float(val_j) * float(x[m][col_j]) over
// row n's entries, in fp32 (see csr.cu).  1 <= M <= 16.  The next kernel on the stream may
// start while it runs (programmatic dependent launch) and must wait for it before reading ysp.
// xT: nullptr, or room for x transposed ([K][csr_token_stride(M)] bf16, written first by a
// transpose kernel) so that each entry's tokens are one load.
cudaError_t launch_csr_rows(const uint16_t* x, uint16_t* xT, const int32_t* row_ptr, const int32_t* col_idx,
                            const uint16_t* vals, long long nnz, int M, int N, int K, float* ysp, unsigned* err,
                            cudaStream_t stream);

// The CSR term of the prefill path (see csr.cu): x is transposed into xT [K][ld] bf16, then
// ysp[n][m] (row stride ld) is computed from it.  ld = csr_token_stride(M).  The GEMM launched
// next may start while these run and waits for them before it reads ysp.
inline int csr_token_stride(int64_t M) { return (int)((M + 7) / 8 * 8); }
cudaError_t launch_csr_prefill(const uint16_t* x, const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* vals,
                               long long nnz, int M, int N, int K, uint16_t* xT, float* ysp, unsigned* err,
                               cudaStream_t stream);

// Dense-and-sparse split of W on the GPU (see outliers.cu).  N * K < 2^32, 1 <= nnz <= N * K.
size_t split_workspace_bytes(int64_t N);
cudaError_t launch_split_outliers(const float* W, const float* act, float alpha, uint32_t N, uint32_t K, uint32_t nnz,
                                  float* W_dense, int32_t* row_ptr, int32_t* col_idx, uint16_t* values,
                                  void* workspace, int num_sms, unsigned* err, cudaStream_t stream);

// Kernels of the AWQ alpha search (see search.cu).
cudaError_t launch_search_ref(const uint16_t* x, const float* W, float* yref, int M, int N, int K, cudaStream_t stream);
cudaError_t launch_search_fold(const uint16_t* x, const float* s, uint16_t* xs, int M, int K, cudaStream_t stream);
cudaError_t launch_search_err(const uint16_t* yq, const float* yref, long long count, double* acc, double* ref2,
                              int num_sms, cudaStream_t stream);

// A kernel whose only wait never completes: it gives up after limit_ns and records
// kErrTimeout (tests the bounded-wait path without any fault).
cudaError_t launch_selftest_timeout(unsigned long long limit_ns, unsigned* err, cudaStream_t stream);

// The quantizer's division against the IEEE one on its whole domain (see selftest.cu):
// mismatches and first[4] (b, a, got, want bits of the first mismatch) must start at zero.
cudaError_t launch_selftest_quotient(unsigned long long* mismatches, unsigned* first, cudaStream_t stream);

// Tensor maps the GEMM needs, encoded by the caller (api.cu) with the driver's encoder.
struct GemmMaps {
    CUtensorMap x;   // bf16 [M][K], box 64 (k) x BN (tokens), 128-byte swizzle
    CUtensorMap qw;  // uint32 [N][K/8], box 16 words (one group) x 128 rows, 64-byte swizzle
};

// A GEMM launch: token tile BN (32, 64, 128 or 256), CTAs per output tile along K (splits,
// each over `slices` 128-k slices) and the bytes of fp32 partial tiles that split-K needs.
// Splitting is limited to kMaxGemmTiles tiles (their counters live in the workspace's counter
// region), kMaxGemmSplits CTAs per tile and kMaxGemmPartialBytes of partial tiles.
constexpr int kMaxGemmTiles = 4096;
constexpr int kMaxGemmSplits = 8;
constexpr size_t kMaxGemmPartialBytes = size_t(64) << 20;
struct GemmPlan {
    int bn;
    int splits;
    int slices;
    size_t partial_bytes;
};
GemmPlan gemm_plan(int64_t M, int64_t N, int64_t K, int num_sms);

// partials and counters: the workspace's split-K parts (unused when plan.splits == 1; the
// counters must be zero and are left zero).  ysp: nullptr or the CSR term from
// launch_csr_prefill, row stride ysp_ld.
cudaError_t launch_gemm(const GemmMaps& maps, const GemmPlan& plan, int group_ratio, const uint16_t* scales,
                        const uint32_t* zeros, const float* ysp, int ysp_ld, uint16_t* y, float* partials,
                        unsigned* counters, int M, int N, int K, unsigned* err, cudaStream_t stream);

}  // namespace w4a16
