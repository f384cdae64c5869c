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

// x'[m][k] = bf16(float(x[m][k]) / s[k]), IEEE division then round-to-nearest-even.  A thread
// converts 8 consecutive channels with 16-byte loads and stores when K % 8 == 0, else one.
// The kernel lets the next kernel on the stream start at once (programmatic dependent launch):
// a GEMV that follows it fetches its weights meanwhile and reads x' only after this grid ends.
__global__ void search_fold_kernel(const uint16_t* __restrict__ x, const float* __restrict__ s,
                                   uint16_t* __restrict__ xs, int M, int K) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int m = blockIdx.y;  // the grid has exactly M rows of blocks
    if (m >= M) return;
    const uint16_t* xr = x + (size_t)m * K;
    uint16_t* yr = xs + (size_t)m * K;
    if ((K & 7) == 0) {
        for (int k = 8 * (blockIdx.x * blockDim.x + threadIdx.x); k < K; k += 8 * gridDim.x * blockDim.x) {
            const uint4 v = *reinterpret_cast<const uint4*>(xr + k);
            const float4 s0 = *reinterpret_cast<const float4*>(s + k);
            const float4 s1 = *reinterpret_cast<const float4*>(s + k + 4);
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t w = u4_get(v, e);
                const uint32_t lo = float_to_bf16_bits(__fdiv_rn(bf16_bits_to_float((uint16_t)(w & 0xFFFFu)), sv[2 * e]));
                const uint32_t hi = float_to_bf16_bits(__fdiv_rn(bf16_bits_to_float((uint16_t)(w >> 16)), sv[2 * e + 1]));
                o[e] = lo | (hi << 16);
            }
            *reinterpret_cast<uint4*>(yr + k) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    } else {
        for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x)
            yr[k] = float_to_bf16_bits(__fdiv_rn(bf16_bits_to_float(xr[k]), s[k]));
    }
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
    const int per = (K & 7) == 0 ? 8 : 1;  // channels per thread
    dim3 grid((K + 256 * per - 1) / (256 * per), M);
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
