// nvfp4.cu -- AWQ-scaled weights quantized to NVFP4: FP4 E2M1 codes, one FP8 E4M3 scale per
// 16 consecutive weights along K, one fp32 scale per tensor.
//
// [DeepCompressor README: the toolbox quantizes to FP4_E2M1 and its tables report NVFP4
//  models; the pages do not define the layout, which is read as the published one.  AWQ
//  translation, section 3.2: the weights are multiplied by the activation-aware scale s.]
//
// On w' = w * s_k (one fp32 multiply), with one IEEE operation per step:
//   g  = amax|W'| / 2688 (= 6 * 448), or 1 for an all-zero W'
//   sb = amax|block| / fp32(6 g);   s8 = E4M3(sb), nearest even, saturating at 448
//   S  = fp32(float(s8) g);         q  = E2M1(fp32(w' / S)), nearest even, saturating at 6,
//                                        sign bit from the quotient; q = 0 where S = 0
// Codes are packed 8 per word with the 4-bit path's interleave (element ORDER[j] in nibble
// j, ORDER = {0,2,4,6,1,3,5,7}), qweight [N][K/8]; scales8 [K/16][N] bytes, group-major.
//
// Quantizer.  Three passes: the s kernel (launch_awq_scale, quantize.cu), a grid-wide amax of |W'|
// (atomicMax on the bits of a non-negative float, into the tensor-scale slot), then one
// thread per 16-weight block; a last one-thread kernel turns the amax into g.  The E4M3
// conversions are CUDA's (cuda_fp8.h, round to nearest even with saturation); the E2M1
// rounding compares with the midpoints of the grid.
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace w4a16 {

namespace {

constexpr int kNvThreads = 256;
constexpr float kNvMax = 2688.0f;  // largest E2M1 magnitude (6) times largest E4M3 (448)

// Nibble of element e (0..7) of an 8-code word: ORDER[nibble] = e.
__device__ __forceinline__ int nv_nibble_of(int e) { return (e & 1) ? 4 + (e >> 1) : (e >> 1); }

// E2M1 code of r: the magnitude index counts the grid midpoints below |r|; a midpoint goes
// to the neighbour whose code is even (0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2,
// 3.5 -> 4, 5 -> 4); beyond 6 the code saturates.  Bit 3 is the sign of r.
__device__ __forceinline__ uint32_t e2m1_code(float r) {
    const float a = fabsf(r);
    const uint32_t idx = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) +
                         (uint32_t)(a >= 1.75f) + (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) +
                         (uint32_t)(a > 5.0f);
    return idx | (signbit(r) ? 8u : 0u);
}

__device__ __forceinline__ float e4m3_to_float(__nv_fp8_storage_t b) {
    return __half2float(__half(__nv_cvt_fp8_to_halfraw(b, __NV_E4M3)));
}

// max |W[n][k] s[k]| over the grid's elements into *amax_bits (as float bits; the caller
// zeroes it).  A non-finite product is a value error.
__global__ void __launch_bounds__(kNvThreads) nvfp4_amax_kernel(const float* __restrict__ W, const float* __restrict__ s,
                                                               int N, int K, unsigned* amax_bits, unsigned* err) {
    const long long total4 = (long long)N * K / 4;
    const long long stride = (long long)gridDim.x * blockDim.x;
    float m = 0.0f;
    bool bad = false;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total4; i += stride) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(W) + i);
        const int k = (int)((i * 4) % K);
        const float4 sv = __ldg(reinterpret_cast<const float4*>(s + k));
        const float p[4] = {__fmul_rn(w.x, sv.x), __fmul_rn(w.y, sv.y), __fmul_rn(w.z, sv.z), __fmul_rn(w.w, sv.w)};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            bad |= !isfinite(p[j]);
            m = fmaxf(m, fabsf(p[j]));
        }
    }
    if (bad) record_error(err, kErrValue);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float wm[kNvThreads / 32];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = wm[0];
        for (int i = 1; i < kNvThreads / 32; ++i) b = fmaxf(b, wm[i]);
        atomicMax(amax_bits, __float_as_uint(b));  // non-negative floats order like their bits
    }
}

__device__ __forceinline__ float tensor_scale(unsigned amax_bits) {
    const float amax = __uint_as_float(amax_bits);
    return amax > 0.0f ? __fdiv_rn(amax, kNvMax) : 1.0f;
}

// One thread per block of 16 weights (row n, block b).
__global__ void __launch_bounds__(kNvThreads) nvfp4_quantize_kernel(const float* __restrict__ W,
                                                                   const float* __restrict__ s, int N, int K,
                                                                   const unsigned* amax_bits,
                                                                   uint32_t* __restrict__ qweight,
                                                                   uint8_t* __restrict__ scales8) {
    const int KB = K / 16;
    const long long total = (long long)N * KB;
    const float g = tensor_scale(*amax_bits);
    const float six_g = __fmul_rn(6.0f, g);
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int n = (int)(i / KB), b = (int)(i % KB);
        const float4* wr = reinterpret_cast<const float4*>(W + (size_t)n * K + 16 * b);
        const float4* sr = reinterpret_cast<const float4*>(s + 16 * b);
        float w[16];
        float bmax = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float4 a = __ldg(wr + c), sv = __ldg(sr + c);
            w[4 * c] = __fmul_rn(a.x, sv.x);
            w[4 * c + 1] = __fmul_rn(a.y, sv.y);
            w[4 * c + 2] = __fmul_rn(a.z, sv.z);
            w[4 * c + 3] = __fmul_rn(a.w, sv.w);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(w[j]));
        const float sb = __fdiv_rn(bmax, six_g);
        const __nv_fp8_storage_t s8 = __nv_cvt_float_to_fp8(sb, __NV_SATFINITE, __NV_E4M3);
        const float S = __fmul_rn(e4m3_to_float(s8), g);
        uint32_t word[2] = {0u, 0u};
        if (S != 0.0f) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                word[j >> 3] |= e2m1_code(__fdiv_rn(w[j], S)) << (4 * nv_nibble_of(j & 7));
        }
        *reinterpret_cast<uint2*>(qweight + (size_t)n * (K / 8) + 2 * b) = make_uint2(word[0], word[1]);
        scales8[(size_t)b * N + n] = (uint8_t)s8;
    }
}

__global__ void nvfp4_gscale_kernel(float* gscale) { *gscale = tensor_scale(*reinterpret_cast<unsigned*>(gscale)); }

// ---------------------------------------------------------------------------------------
// Decode GEMV on NVFP4 weights (1 <= M <= 16):
//   y[m][n] = bf16( g * sum_b (s8[b][n] / 2) * sum_{k in block b} (2 e2m1(q[n][k])) x[m][k] )
// Twice an E2M1 value is one of the integers 0, 1, 2, 3, 4, 6, 8, 12, exact in bf16, so the
// codes enter mma.sync m16n8k16 (rows: 16 channels, columns: 8 tokens, depth: 16 k = one
// scale block) as exact bf16 values; each MMA's fp32 result is scaled by its block's E4M3
// scale / 2 and accumulated, and the tensor scale multiplies the sum once.  A CTA of 8 warps
// (three per SM) takes 16 rows; warp w takes an eighth of the blocks along K, issuing the
// loads of four blocks at a time, and the warps' sums are added in warp order through shared memory.
// Weights and x are read straight from global memory (a 32-byte sector of codes serves four
// consecutive blocks through L1).

// bf16 pair (2 e2m1(c_lo), 2 e2m1(c_hi)) of the nibble pair (c, c + 4) of a word: byte
// lookups of the low and high bytes of the bf16 values, then the sign bits.
__device__ __forceinline__ uint32_t e2m1x2_to_bf16x2(uint32_t word, int c) {
    const uint32_t t = word >> (4 * c);
    const uint32_t sel = (t & 0x7u) | ((t >> 12) & 0x70u);   // code of the low half, of the high half
    const uint32_t lo = __byte_perm(0x40008000u, 0x4000C080u, sel);  // low bytes of bf16(0,1,2,3,4,6,8,12)
    const uint32_t hi = __byte_perm(0x40403F00u, 0x41414040u, sel);  // high bytes
    return __byte_perm(lo, hi, 0x5140u) | ((t & 0x00080008u) << 12);
}

constexpr int kNvGemvWarps = 8;   // warps per CTA, each a share of the blocks along K
constexpr int kNvGemvBatch = 4;   // blocks whose loads are issued together

template <int NT>
__global__ void __launch_bounds__(32 * kNvGemvWarps, 3) nvfp4_gemv_kernel(const uint16_t* __restrict__ x,
                                                                      const uint32_t* __restrict__ qweight,
                                                                      const uint8_t* __restrict__ scales8,
                                                                      const float* __restrict__ gscale,
                                                                      uint16_t* __restrict__ y, int M, int N, int K) {
    __shared__ float red[kNvGemvWarps][32][NT * 4];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int n0 = blockIdx.x * 16;
    const int KB = K / 16, per = (KB + kNvGemvWarps - 1) / kNvGemvWarps;
    const int b0 = min(KB, warp * per), b1 = min(KB, b0 + per);
    const uint2* w0 = reinterpret_cast<const uint2*>(qweight + (size_t)(n0 + g) * (K / 8));
    const uint2* w1 = reinterpret_cast<const uint2*>(qweight + (size_t)(n0 + g + 8) * (K / 8));
    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.0f;
    for (int bb = b0; bb < b1; bb += kNvGemvBatch) {
        // the batch's loads first (blocks past b1 load nothing and add nothing)
        uint2 q0[kNvGemvBatch], q1[kNvGemvBatch];
        uint8_t s0[kNvGemvBatch], s1[kNvGemvBatch];
        uint32_t xb[kNvGemvBatch][NT][2];
#pragma unroll
        for (int u = 0; u < kNvGemvBatch; ++u) {
            const int b = bb + u;
            const bool live = b < b1;
            q0[u] = live ? __ldg(w0 + b) : make_uint2(0u, 0u);
            q1[u] = live ? __ldg(w1 + b) : make_uint2(0u, 0u);
            s0[u] = live ? __ldg(scales8 + (size_t)b * N + n0 + g) : (uint8_t)0;
            s1[u] = live ? __ldg(scales8 + (size_t)b * N + n0 + g + 8) : (uint8_t)0;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const int tok = 8 * j + g;
                xb[u][j][0] = 0u;
                xb[u][j][1] = 0u;
                if (live && tok < M) {
                    const uint32_t* xr = reinterpret_cast<const uint32_t*>(x + (size_t)tok * K + 16 * b + 2 * c);
                    xb[u][j][0] = __ldg(xr);
                    xb[u][j][1] = __ldg(xr + 4);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kNvGemvBatch; ++u) {
            if (bb + u >= b1) break;
            const uint32_t A[4] = {e2m1x2_to_bf16x2(q0[u].x, c), e2m1x2_to_bf16x2(q1[u].x, c),
                                   e2m1x2_to_bf16x2(q0[u].y, c), e2m1x2_to_bf16x2(q1[u].y, c)};
            const float sa = 0.5f * e4m3_to_float(s0[u]);
            const float sb = 0.5f * e4m3_to_float(s1[u]);
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                float d[4];
                mma_16816_bf16_zero(d, A, xb[u][j]);
                acc[j][0] = fmaf(sa, d[0], acc[j][0]);
                acc[j][1] = fmaf(sa, d[1], acc[j][1]);
                acc[j][2] = fmaf(sb, d[2], acc[j][2]);
                acc[j][3] = fmaf(sb, d[3], acc[j][3]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) red[warp][lane][4 * j + e] = acc[j][e];
    __syncthreads();
    if (warp != 0) return;
    const float gs = *gscale;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float v = red[0][lane][4 * j + e];
#pragma unroll
            for (int w = 1; w < kNvGemvWarps; ++w) v += red[w][lane][4 * j + e];
            const int tok = 8 * j + 2 * c + (e & 1), n = n0 + g + 8 * (e >> 1);
            if (tok < M) y[(size_t)tok * N + n] = float_to_bf16_bits(__fmul_rn(gs, v));
        }
}

}  // namespace

cudaError_t launch_gemv_nvfp4(const uint16_t* x, const uint32_t* qweight, const uint8_t* scales8, const float* gscale,
                              uint16_t* y, int M, int N, int K, cudaStream_t stream) {
    if (M < 1 || M > 16 || N % 16 != 0 || K % 16 != 0) return cudaErrorInvalidValue;
    if (M <= 8)
        nvfp4_gemv_kernel<1><<<N / 16, 32 * kNvGemvWarps, 0, stream>>>(x, qweight, scales8, gscale, y, M, N, K);
    else
        nvfp4_gemv_kernel<2><<<N / 16, 32 * kNvGemvWarps, 0, stream>>>(x, qweight, scales8, gscale, y, M, N, K);
    return cudaGetLastError();
}

cudaError_t launch_awq_quantize_nvfp4(const float* W, const float* act, float alpha, int N, int K, uint32_t* qweight,
                                      uint8_t* scales8, float* gscale, float* s_out, int num_sms, unsigned* err,
                                      cudaStream_t stream) {
    cudaError_t e = launch_awq_scale(act, alpha, K, s_out, err, stream);
    if (e != cudaSuccess) return e;
    unsigned* amax = reinterpret_cast<unsigned*>(gscale);  // the slot holds the amax until the last kernel
    e = cudaMemsetAsync(amax, 0, sizeof(unsigned), stream);
    if (e != cudaSuccess) return e;
    const long long total4 = (long long)N * K / 4;
    const int grid_a = (int)std::min<long long>((total4 + kNvThreads - 1) / kNvThreads, 8LL * num_sms);
    nvfp4_amax_kernel<<<grid_a, kNvThreads, 0, stream>>>(W, s_out, N, K, amax, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)N * (K / 16);
    const int grid_q = (int)std::min<long long>((blocks + kNvThreads - 1) / kNvThreads, 16LL * num_sms);
    nvfp4_quantize_kernel<<<grid_q, kNvThreads, 0, stream>>>(W, s_out, N, K, amax, qweight, scales8);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    nvfp4_gscale_kernel<<<1, 1, 0, stream>>>(gscale);
    return cudaGetLastError();
}

}  // namespace w4a16
