// search.cu -- kernels of the AWQ scale search (the host loop is awq_search_alpha in api.cu).
//
// [AWQ (MLSys 2024) translation, section 3.2: the per-channel scaling factor is searched so
//  that the quantized layer's output on calibration activations stays closest to the
//  full-precision output; with s = a^alpha the search runs over the exponent alpha.]
//
// For every alpha of a grid the host launches the quantize kernel (W * s -> packed), the fold
// below (x' = bf16(x / s)), the W4A16 product on x' (the GEMV or GEMM of this library) and
// the error reduction against the full-precision output, which is computed once:
//   err(alpha) = sum (y_q - y_ref)^2 / sum y_ref^2,   y_ref = x . W^T.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kRefTM = 16, kRefTN = 64, kRefTK = 32;

// y_ref[m][n] = sum_k float(x[m][k]) * W[n][k] in fp32: a 16 x 64 output tile per CTA of
// 256 threads, 32-k slices of x (bf16 -> fp32) and W staged in shared memory.
__global__ void __launch_bounds__(256)
search_ref_kernel(const uint16_t* __restrict__ x, const float* __restrict__ W, float* __restrict__ yref, int M, int N,
                  int K) {
    __shared__ float xs[kRefTM][kRefTK + 1];
    __shared__ float ws[kRefTN][kRefTK + 1];
    const int n0 = blockIdx.x * kRefTN, m0 = blockIdx.y * kRefTM;
    const int tid = threadIdx.x;
    const int tn = tid & 63, tm = tid >> 6;  // thread: row n0 + tn, tokens m0 + tm + 4 i
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int k0 = 0; k0 < K; k0 += kRefTK) {
        for (int i = tid; i < kRefTM * kRefTK; i += 256) {
            const int r = i / kRefTK, c = i % kRefTK;
            xs[r][c] = m0 + r < M ? bf16_bits_to_float(x[(size_t)(m0 + r) * K + k0 + c]) : 0.0f;
        }
        for (int i = tid; i < kRefTN * kRefTK; i += 256) {
            const int r = i / kRefTK, c = i % kRefTK;
            ws[r][c] = W[(size_t)(n0 + r) * K + k0 + c];
        }
        __syncthreads();
#pragma unroll 8
        for (int c = 0; c < kRefTK; ++c) {
            const float w = ws[tn][c];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = fmaf(xs[tm + 4 * i][c], w, acc[i]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + tm + 4 * i;
        if (m < M) yref[(size_t)m * N + n0 + tn] = acc[i];
    }
}

// x'[m][k] = bf16(float(x[m][k]) / s[k]), IEEE division then round-to-nearest-even.
__global__ void search_fold_kernel(const uint16_t* __restrict__ x, const float* __restrict__ s,
                                   uint16_t* __restrict__ xs, int M, int K) {
    const int m = blockIdx.y;  // the grid has exactly M rows of blocks
    if (m >= M) return;
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x)
        xs[(size_t)m * K + k] = float_to_bf16_bits(__fdiv_rn(bf16_bits_to_float(x[(size_t)m * K + k]), s[k]));
}

// acc[0] += sum (y_q - y_ref)^2, and when ref2 is given, *ref2 += sum y_ref^2 (double).
__global__ void __launch_bounds__(256)
search_err_kernel(const uint16_t* __restrict__ yq, const float* __restrict__ yref, long long count,
                  double* __restrict__ acc, double* __restrict__ ref2) {
    __shared__ double s_e[8], s_r[8];
    double e = 0.0, r = 0.0;
    for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < count; i += (long long)gridDim.x * 256) {
        const double ref = (double)yref[i];
        const double d = (double)bf16_bits_to_float(yq[i]) - ref;
        e += d * d;
        r += ref * ref;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        e += __shfl_xor_sync(0xffffffffu, e, o);
        r += __shfl_xor_sync(0xffffffffu, r, o);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_e[warp] = e;
        s_r[warp] = r;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double te = 0.0, tr = 0.0;
        for (int w = 0; w < 8; ++w) {
            te += s_e[w];
            tr += s_r[w];
        }
        atomicAdd(acc, te);
        if (ref2 != nullptr) atomicAdd(ref2, tr);
    }
}

cudaError_t launch_search_ref(const uint16_t* x, const float* W, float* yref, int M, int N, int K,
                              cudaStream_t stream) {
    dim3 grid(N / kRefTN, (M + kRefTM - 1) / kRefTM);
    search_ref_kernel<<<grid, 256, 0, stream>>>(x, W, yref, M, N, K);
    return cudaGetLastError();
}

cudaError_t launch_search_fold(const uint16_t* x, const float* s, uint16_t* xs, int M, int K, cudaStream_t stream) {
    dim3 grid((K + 255) / 256, M);
    search_fold_kernel<<<grid, 256, 0, stream>>>(x, s, xs, M, K);
    return cudaGetLastError();
}

cudaError_t launch_search_err(const uint16_t* yq, const float* yref, long long count, double* acc, double* ref2,
                              int num_sms, cudaStream_t stream) {
    long long blocks = (count + 255) / 256;
    if (blocks > 4LL * num_sms) blocks = 4LL * num_sms;
    search_err_kernel<<<(int)blocks, 256, 0, stream>>>(yq, yref, count, acc, ref2);
    return cudaGetLastError();
}

}  // namespace w4a16
