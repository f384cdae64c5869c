// csr.cu -- the sparse term of the decode path, y_sparse = x . W_sparse^T, in fp32.
//
// [SqueezeLLM article, section 2.3: the sensitive weights stay in an fp16 sparse matrix whose
//  product with the input is added to the dense product; section 2.2: W = W_dense + W_sparse.]
//
// The decode GEMV adds this term to each output before its one rounding to bf16.  It is
// computed just before the GEMV by this kernel, which writes ysp[n][m] (row-major over n, so
// that the GEMV's epilogue reads a row's M values contiguously).  Both are launched with
// programmatic dependent launch: this kernel fetches its CSR entries while the previous kernel
// finishes and reads x after it; the GEMV streams its weights meanwhile and reads ysp only
// after this kernel has finished.
//
// Work split: 4 lanes per (row n, token m); lane q takes the row's entries j0 + q, j0 + q + 4,
// ... and accumulates val * x[m][col] in fp32 from -0 (the additive identity, so an empty row
// adds nothing to the dense sum's bits); the 4 partial sums are then combined as
// (p0 + p1) + (p2 + p3) by two shuffle steps.  The order is fixed, so every call gives the
// same bits.  Entries are independent within a lane, so their loads overlap; with many rows in
// flight across the GPU the gathers of x (small, L2-resident) are latency-, not bandwidth-bound.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kCsrLanes = 4;  // lanes per (row, token)
constexpr int kCsrAhead = 8;  // entries per lane fetched before waiting for the previous kernel

__global__ void __launch_bounds__(256)
csr_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                const uint16_t* __restrict__ vals, long long nnz, int M, int N, int K, float* __restrict__ ysp,
                unsigned* err) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int q = (int)(t % kCsrLanes);
    const long long rm = t / kCsrLanes;  // (row, token) index, token fastest
    const bool live = rm < (long long)N * M;
    const int n = live ? (int)(rm / M) : 0, m = live ? (int)(rm % M) : 0;
    // The CSR arrays do not come from the previous kernel (as for the weights): this lane's
    // first kCsrAhead entries are fetched before waiting for it; x after.
    int j0 = 0, j1 = 0;
    if (live) {
        j0 = row_ptr[n];
        j1 = row_ptr[n + 1];
        if (j0 < 0 || j1 < j0 || (long long)j1 > nnz) {
            if (q == 0) record_error(err, kErrShape);
            j1 = j0;
        }
    }
    int c[kCsrAhead];
    float v[kCsrAhead];
#pragma unroll
    for (int e = 0; e < kCsrAhead; ++e) {
        const int j = j0 + q + kCsrLanes * e;
        c[e] = j < j1 ? __ldg(col_idx + j) : -1;
        v[e] = j < j1 ? fp16_bits_to_float(__ldg(vals + j)) : 0.0f;
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // x belongs to the stream order
    float acc = -0.0f;
    const uint16_t* xr = x + (size_t)m * K;
#pragma unroll
    for (int e = 0; e < kCsrAhead; ++e) {
        const int j = j0 + q + kCsrLanes * e;
        if (j < j1) {
            if ((unsigned)c[e] >= (unsigned)K) record_error(err, kErrShape);  // the entry is skipped
            else acc = fmaf(v[e], bf16_bits_to_float(__ldcg(xr + c[e])), acc);
        }
    }
#pragma unroll 4
    for (int j = j0 + q + kCsrLanes * kCsrAhead; j < j1; j += kCsrLanes) {
        const int cj = __ldg(col_idx + j);
        if ((unsigned)cj >= (unsigned)K) {
            record_error(err, kErrShape);
            continue;
        }
        acc = fmaf(fp16_bits_to_float(__ldg(vals + j)), bf16_bits_to_float(__ldcg(xr + cj)), acc);
    }
    // (p0 + p1) + (p2 + p3); the 4 lanes of a (row, token) are adjacent and in one warp
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (live && q == 0) ysp[(size_t)n * M + m] = acc;
}

cudaError_t launch_csr_rows(const uint16_t* x, const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* vals,
                            long long nnz, int M, int N, int K, float* ysp, unsigned* err, cudaStream_t stream) {
    const long long threads = (long long)N * M * kCsrLanes;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((threads + 255) / 256), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, csr_rows_kernel, x, row_ptr, col_idx, vals, nnz, M, N, K, ysp, err);
}

}  // namespace w4a16
