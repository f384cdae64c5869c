// csr.cu -- the sparse term y_sparse = x . W_sparse^T in fp32, for the decode GEMV and for the
// prefill GEMM.
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
// Work split: one warp per row n.  Lane l takes the row's entries j0 + l, j0 + l + 32, ...
// (its column and value are read once for all tokens) and keeps one fp32 partial sum per token,
// accumulated from -0 (the additive identity, so an empty row adds nothing to the dense sum's
// bits).  The 32 partial sums of each token are then added by a butterfly (xor 16, 8, 4, 2, 1),
// whose order is fixed, so every call gives the same bits.  Lane m writes token m.  CTAs are
// 4 warps, small enough in registers that many fit beside each other and the whole grid
// starts at once.  With a workspace, x is first transposed (xT[k][m], token stride 8 or 16,
// the transpose kernel below), so an entry's tokens are one 16- or 32-byte load instead of M
// loads from M rows of x; without one (w4a16_gemv_noalloc) the kernel gathers from x.  Both
// read the same values in the same order and give the same bits.
//
// Prefill (M > 16): the same term for many tokens.  Gathering x[m][col] for a fixed column
// over many tokens would touch one 32-byte sector per token, so x is first transposed into
// xT[k][m] (token stride padded to a multiple of 8).  A warp then takes one row n and up to 256
// tokens: lane l owns tokens m0 + 8l .. m0 + 8l + 7, reads them with one 16-byte load per
// entry (a warp reads 512 contiguous bytes of xT per entry) and accumulates in fp32 from -0,
// entry after entry in CSR order.  ysp[n][m] has the same padded token stride, so the GEMM's
// epilogue reads a row's tokens contiguously.  (A persistent grid of two CTAs per SM, so that
// the GEMM could start beside it, was measured slower: the two slowed each other.  Batching
// four entries' loads per step did not help either.)
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kCsrWarps = 4;  // warps (rows) per CTA of the decode kernel

__global__ void __launch_bounds__(32 * kCsrWarps)
csr_rows_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ xT, int ld,
                const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                const uint16_t* __restrict__ vals, long long nnz, int M, int N, int K, float* __restrict__ ysp,
                unsigned* err) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * kCsrWarps + (threadIdx.x >> 5);
    if (n >= N) return;
    // The CSR arrays do not come from the previous kernel (as for the weights): this lane's
    // first entry is fetched before waiting for it; x after.
    int j0 = row_ptr[n], j1 = row_ptr[n + 1];
    if (j0 < 0 || j1 < j0 || (long long)j1 > nnz) {
        if (lane == 0) record_error(err, kErrShape);
        j1 = j0;
    }
    int c = -1;
    float v = 0.0f;
    if (j0 + lane < j1) {
        c = __ldg(col_idx + j0 + lane);
        v = fp16_bits_to_float(__ldg(vals + j0 + lane));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // x belongs to the stream order
    float acc[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) acc[m] = -0.0f;
    for (int j = j0 + lane; j < j1; j += 32) {
        if (j != j0 + lane) {
            c = __ldg(col_idx + j);
            v = fp16_bits_to_float(__ldg(vals + j));
        }
        if ((unsigned)c >= (unsigned)K) {  // the entry is skipped
            record_error(err, kErrShape);
            continue;
        }
        if (xT != nullptr) {  // the entry's tokens, contiguous (ld = 8 or 16)
            uint4 q[2];
            q[0] = __ldg(reinterpret_cast<const uint4*>(xT + (size_t)c * ld));
            q[1] = ld > 8 ? __ldg(reinterpret_cast<const uint4*>(xT + (size_t)c * ld + 8)) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const uint32_t pr = u4_get(q[m >> 3], (m & 7) >> 1);
                const float xv = __uint_as_float((m & 1) ? (pr & 0xFFFF0000u) : (pr << 16));
                if (m < M) acc[m] = fmaf(v, xv, acc[m]);
            }
        } else {
#pragma unroll
            for (int m = 0; m < 16; ++m)
                if (m < M) acc[m] = fmaf(v, bf16_bits_to_float(__ldg(x + (size_t)m * K + c)), acc[m]);
        }
    }
    float mine = 0.0f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (m < M) {
            float t = acc[m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
            if (lane == m) mine = t;
        }
    }
    if (lane < M) ysp[(size_t)n * M + lane] = mine;
}

cudaError_t launch_transpose_x(const uint16_t* x, uint16_t* xT, int M, int K, int ld, bool pdl, cudaStream_t stream);

cudaError_t launch_csr_rows(const uint16_t* x, uint16_t* xT, const int32_t* row_ptr, const int32_t* col_idx,
                            const uint16_t* vals, long long nnz, int M, int N, int K, float* ysp, unsigned* err,
                            cudaStream_t stream) {
    const int ld = csr_token_stride(M);
    if (xT != nullptr) {
        cudaError_t e = launch_transpose_x(x, xT, M, K, ld, true, stream);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + kCsrWarps - 1) / kCsrWarps), 1, 1);
    cfg.blockDim = dim3(32 * kCsrWarps, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, csr_rows_kernel, x, (const uint16_t*)xT, ld, row_ptr, col_idx, vals, nnz, M, N, K,
                              ysp, err);
}

// xT[k][m] = x[m][k] for m < M; xT has ld (>= M, a multiple of 8) elements per row.  32 x 32
// tiles through shared memory, so both the reads and the writes are coalesced.  It reads x
// only after the previous kernel on the stream has finished (a no-op when launched without
// programmatic dependent launch).
__global__ void __launch_bounds__(256)
transpose_x_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ xT, int M, int K, int ld) {
    __shared__ uint16_t tile[32][33];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int k0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of 32 per pass
#pragma unroll
    for (int r = ty; r < 32; r += 8) {
        const int m = m0 + r;
        tile[r][tx] = m < M ? x[(size_t)m * K + k0 + tx] : (uint16_t)0;
    }
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#pragma unroll
    for (int r = ty; r < 32; r += 8) {
        const int m = m0 + tx;
        if (m < ld) xT[(size_t)(k0 + r) * ld + m] = tile[tx][r];
    }
}

constexpr int kSpmmTokens = 256;  // tokens per warp: 8 per lane

__global__ void __launch_bounds__(256)
csr_spmm_kernel(const uint16_t* __restrict__ xT, const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                const uint16_t* __restrict__ vals, long long nnz, int M, int N, int K, int ld, float* __restrict__ ysp,
                unsigned* err) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int chunks = (M + kSpmmTokens - 1) / kSpmmTokens;
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // (row, token chunk)
    if (w >= (long long)N * chunks) return;
    const int n = (int)(w / chunks);
    const int m = (int)(w % chunks) * kSpmmTokens + 8 * lane;  // this lane's first token
    int j0 = row_ptr[n], j1 = row_ptr[n + 1];
    if (j0 < 0 || j1 < j0 || (long long)j1 > nnz) {
        if (lane == 0) record_error(err, kErrShape);
        j1 = j0;
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // xT comes from the previous kernel
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = -0.0f;
    const bool mine = m < M;
    for (int jb = j0; jb < j1; jb += 32) {
        const int jl = jb + lane;
        const int cl = jl < j1 ? __ldg(col_idx + jl) : 0;
        const float vl = jl < j1 ? fp16_bits_to_float(__ldg(vals + jl)) : 0.0f;
        const int cnt = min(32, j1 - jb);
        for (int t = 0; t < cnt; ++t) {
            const int c = __shfl_sync(0xffffffffu, cl, t);
            const float v = __shfl_sync(0xffffffffu, vl, t);
            if ((unsigned)c >= (unsigned)K) {  // the entry is skipped
                if (lane == 0) record_error(err, kErrShape);
                continue;
            }
            if (mine) {
                const uint4 q = __ldcg(reinterpret_cast<const uint4*>(xT + (size_t)c * ld + m));
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t pr = u4_get(q, i);
                    acc[2 * i] = fmaf(v, __uint_as_float(pr << 16), acc[2 * i]);
                    acc[2 * i + 1] = fmaf(v, __uint_as_float(pr & 0xFFFF0000u), acc[2 * i + 1]);
                }
            }
        }
    }
    if (mine) {
        float4* out = reinterpret_cast<float4*>(ysp + (size_t)n * ld + m);
        out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

cudaError_t launch_csr_prefill(const uint16_t* x, const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* vals,
                               long long nnz, int M, int N, int K, uint16_t* xT, float* ysp, unsigned* err,
                               cudaStream_t stream) {
    const int ld = csr_token_stride(M);
    cudaError_t e = launch_transpose_x(x, xT, M, K, ld, false, stream);
    if (e != cudaSuccess) return e;
    const long long warps = (long long)N * ((M + kSpmmTokens - 1) / kSpmmTokens);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((warps * 32 + 255) / 256), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, csr_spmm_kernel, (const uint16_t*)xT, row_ptr, col_idx, vals, nnz, M, N, K, ld, ysp,
                              err);
}

cudaError_t launch_transpose_x(const uint16_t* x, uint16_t* xT, int M, int K, int ld, bool pdl, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(K / 32, (ld + 31) / 32, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, transpose_x_kernel, x, xT, M, K, ld);
}

}  // namespace w4a16
