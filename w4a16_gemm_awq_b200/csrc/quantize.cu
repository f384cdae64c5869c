// quantize.cu -- AWQ activation-aware scaling + group-wise asymmetric uint4 RTN + packing.
//
// [AWQ (MLSys 2024) translation, section 3.2: per-input-channel scaling of the weights by a
//  factor derived from the activation magnitude; section 2: round-to-nearest; DeepCompressor
//  README, perplexity table row "W4A16 g128": groups of 128 along K; AWQ translation
//  section 1: TinyChat's 4-bit packing, 8 codes per 32-bit word.]
//
// Work decomposition.  A CTA of 8 warps owns a tile of kRowsPerCta rows x 1024 columns
// (8 groups).  It first computes the 1024 per-channel scales s_k into
// shared memory (double pow, as the definition states).  Then each warp quantizes one row
// of the tile at a time: 32 lanes x 16 bytes is exactly one group of 128 fp32 weights,
// so the row's 8 groups arrive as 8 coalesced 128-bit loads per lane, all issued before
// the first group is processed.  The group's min/max is a 5-step warp-shuffle reduction.
// Each lane quantizes its 4 weights.  Lane pairs (2i, 2i+1) merge their nibbles into
// packed word i with one shuffle.  The fp16 scales and zero points of the tile are collected
// in shared memory and written group-major at the end (scales[g][n], zeros[g][n/8] with the
// nibbles of 8 consecutive rows), so those stores are coalesced too.
//
// Bit-exactness: every float step is a single IEEE operation with round-to-nearest-even
// (__fmul_rn, __fsub_rn, __fdiv_rn, __fadd_rn, __float2half_rn) or an exact equivalent of
// one.  The build does not use fast-math or flush-to-zero, so any correct implementation of
// the same steps gives the same bits.
//
// Throughput: the quarter-rate XU pipe (reciprocal, rounding, float-to-integer conversion)
// is the limiting unit, so only the division stays there.  rint(v) is computed as
// (v + 1.5 * 2^23) - 1.5 * 2^23 on the FMA pipe: for |v| < 2^22 this is exactly
// round-to-nearest-even, and larger magnitudes end up clamped to 0 or 15 either way.  The
// integer code of an integral float c in [0, 15] is the low mantissa bits of c + 2^23.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kQuantThreads = 256;
constexpr int kRowsPerCta = 64;

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kIntMagic = 8388608.0f;      // 2^23

// round-to-nearest-even to an integral float; exact for |v| < 2^22 (see above)
__device__ __forceinline__ float round_rne(float v) { return __fsub_rn(__fadd_rn(v, kRoundMagic), kRoundMagic); }

// the integer value of an integral float in [0, 2^22)
__device__ __forceinline__ uint32_t int_bits(float c) { return __float_as_uint(__fadd_rn(c, kIntMagic)) & 0x3FFFFFu; }

// Nibble position of each of a lane's 4 elements inside the packed word.  Element e of an
// 8-wide block sits in nibble j with ORDER[j] = e, ORDER = {0,2,4,6,1,3,5,7}.  The even
// lane holds elements 0..3, which go to nibbles 0,4,1,5.  The odd lane holds elements
// 4..7, which go to nibbles 2,6,3,7.
__device__ __forceinline__ uint32_t place_nibbles(const float q[4], bool odd) {
    const uint32_t q0 = int_bits(q[0]), q1 = int_bits(q[1]), q2 = int_bits(q[2]), q3 = int_bits(q[3]);
    if (!odd) return q0 | (q1 << 16) | (q2 << 4) | (q3 << 20);
    return (q0 << 8) | (q1 << 24) | (q2 << 12) | (q3 << 28);
}

// Groups of 128 R weights, R in {1, 2, 4, 8}: a 1024-column chunk holds 8 / R whole groups.
template <int R>
__global__ void __launch_bounds__(kQuantThreads)
awq_quantize_kernel(const float* __restrict__ W, const float* __restrict__ act, float alpha, int N, int K,
                    uint32_t* __restrict__ qweight, uint16_t* __restrict__ scales,
                    uint32_t* __restrict__ zeros, float* __restrict__ s_out, unsigned* err) {
    constexpr int GC = 8 / R;  // groups per chunk
    __shared__ __align__(16) float s_sm[1024];
    __shared__ __align__(16) uint16_t sc_sm[GC][kRowsPerCta];  // fp16 scale bits per (group, row)
    __shared__ uint8_t zc_sm[GC][kRowsPerCta];                 // zero point per (group, row)
    const int kc = blockIdx.x;                 // 1024-column chunk (groups GC kc .. GC kc + GC - 1)
    const int row0 = blockIdx.y * kRowsPerCta;

    for (int i = threadIdx.x; i < 1024; i += kQuantThreads) {
        const float a = act[(size_t)kc * 1024 + i];
        const float p = (float)pow((double)a, (double)alpha);
        if (!(a >= 0.0f) || isinf(a) || !isfinite(p)) record_error(err, kErrValue);
        const float s = p > 1e-4f ? p : 1e-4f;
        s_sm[i] = s;
        if (s_out != nullptr && blockIdx.y == 0) s_out[(size_t)kc * 1024 + i] = s;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool odd = lane & 1;
    for (int r = warp; r < kRowsPerCta; r += kQuantThreads / 32) {
        const int n = row0 + r;
        if (n >= N) break;  // warp-uniform
        const float* wrow = W + (size_t)n * K + (size_t)kc * 1024 + 4 * lane;
        float4 v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 u = ldg_stream(wrow + c * 128);
            v[c] = make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z),
                               __uint_as_float(u.w));
        }
        bool bad = false;
#pragma unroll
        for (int gi = 0; gi < GC; ++gi) {
            // the group's R slices of 128: this lane's 4 scaled weights of each
            float w[R][4];
            float mx = 0.0f, mn = 0.0f;
#pragma unroll
            for (int c = 0; c < R; ++c) {
                const int sl = gi * R + c;
                const float4 sv = *reinterpret_cast<const float4*>(&s_sm[sl * 128 + 4 * lane]);
                w[c][0] = __fmul_rn(v[sl].x, sv.x);
                w[c][1] = __fmul_rn(v[sl].y, sv.y);
                w[c][2] = __fmul_rn(v[sl].z, sv.z);
                w[c][3] = __fmul_rn(v[sl].w, sv.w);
                if (c == 0) mx = mn = w[0][0];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    bad |= !isfinite(w[c][i]);
                    mx = fmaxf(mx, w[c][i]);
                    mn = fminf(mn, w[c][i]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            }
            float scale32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
            if (scale32 < 1e-5f) scale32 = 1e-5f;
            const __half h = __float2half_rn(scale32);
            const float sf = __half2float(h);
            bad |= isinf(scale32) || isinf(sf);
            float zf = rintf(__fdiv_rn(-mn, sf));
            zf = fminf(fmaxf(zf, 0.0f), 15.0f);
#pragma unroll
            for (int c = 0; c < R; ++c) {
                float q[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float t = __fadd_rn(round_rne(__fdiv_rn(w[c][i], sf)), zf);
                    q[i] = fminf(fmaxf(t, 0.0f), 15.0f);
                }
                uint32_t part = place_nibbles(q, odd);
                part |= __shfl_xor_sync(0xffffffffu, part, 1);
                if (!odd) qweight[(size_t)n * (K >> 3) + (size_t)kc * 128 + (gi * R + c) * 16 + (lane >> 1)] = part;
            }
            if (lane == 0) {
                sc_sm[gi][r] = __half_as_ushort(h);
                zc_sm[gi][r] = (uint8_t)int_bits(zf);
            }
        }
        if (bad) record_error(err, kErrValue);
    }
    __syncthreads();

    // group-major parameters: scales[g][n] (row pairs as one 32-bit store) and zeros[g][n/8]
    // (the nibbles of 8 consecutive rows), both coalesced along n
    {
        const int g = threadIdx.x >> 5, j = threadIdx.x & 31;  // up to 8 groups x 32 row pairs
        const int r = 2 * j;
        if (g < GC && row0 + r < N) {
            const uint32_t pair = (uint32_t)sc_sm[g][r] | ((uint32_t)sc_sm[g][r + 1] << 16);
            *reinterpret_cast<uint32_t*>(scales + ((size_t)kc * GC + g) * N + row0 + r) = pair;
        }
        if (threadIdx.x < 64) {
            const int gz = threadIdx.x >> 3, w = threadIdx.x & 7;
            if (gz < GC && row0 + 8 * w < N) {
                uint32_t word = 0;
#pragma unroll
                for (int b = 0; b < 8; ++b) word |= (uint32_t)(zc_sm[gz][8 * w + b] & 15u) << (4 * b);
                zeros[((size_t)kc * GC + gz) * (N >> 3) + (row0 >> 3) + w] = word;
            }
        }
    }
}

// Groups of gs = 1024 j weights (up to one group per row): a CTA takes kLargeRows rows of
// one group.  Each warp reads a row's group twice: once for its minimum and maximum, once to
// quantize (the second read mostly hits L2).  s for the group's columns is in shared memory.
constexpr int kLargeRows = 8;

__global__ void __launch_bounds__(kQuantThreads)
awq_quantize_large_kernel(const float* __restrict__ W, const float* __restrict__ act, float alpha, int N, int K,
                          int gs, uint32_t* __restrict__ qweight, uint16_t* __restrict__ scales,
                          uint32_t* __restrict__ zeros, float* __restrict__ s_out, unsigned* err) {
    extern __shared__ __align__(16) float s_g[];  // gs scales of this group's columns
    __shared__ __align__(16) uint16_t sc_sm[kLargeRows];
    __shared__ uint8_t zc_sm[kLargeRows];
    const int g = blockIdx.x;
    const int row0 = blockIdx.y * kLargeRows;
    const size_t c0 = (size_t)g * gs;

    for (int i = threadIdx.x; i < gs; i += kQuantThreads) {
        const float a = act[c0 + i];
        const float p = (float)pow((double)a, (double)alpha);
        if (!(a >= 0.0f) || isinf(a) || !isfinite(p)) record_error(err, kErrValue);
        const float s = p > 1e-4f ? p : 1e-4f;
        s_g[i] = s;
        if (s_out != nullptr && blockIdx.y == 0) s_out[c0 + i] = s;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool odd = lane & 1;
    for (int r = warp; r < kLargeRows; r += kQuantThreads / 32) {
        const int n = row0 + r;
        if (n >= N) break;  // warp-uniform
        const float* wrow = W + (size_t)n * K + c0 + 4 * lane;
        bool bad = false;
        float mx = 0.0f, mn = 0.0f;
        for (int c = 0; c < gs; c += 128) {
            const float4 u = *reinterpret_cast<const float4*>(wrow + c);
            const float4 sv = *reinterpret_cast<const float4*>(&s_g[c + 4 * lane]);
            const float w[4] = {__fmul_rn(u.x, sv.x), __fmul_rn(u.y, sv.y), __fmul_rn(u.z, sv.z),
                                __fmul_rn(u.w, sv.w)};
            if (c == 0) mx = mn = w[0];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                bad |= !isfinite(w[i]);
                mx = fmaxf(mx, w[i]);
                mn = fminf(mn, w[i]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        }
        float scale32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        if (scale32 < 1e-5f) scale32 = 1e-5f;
        const __half h = __float2half_rn(scale32);
        const float sf = __half2float(h);
        bad |= isinf(scale32) || isinf(sf);
        float zf = rintf(__fdiv_rn(-mn, sf));
        zf = fminf(fmaxf(zf, 0.0f), 15.0f);
        for (int c = 0; c < gs; c += 128) {
            const float4 u = *reinterpret_cast<const float4*>(wrow + c);
            const float4 sv = *reinterpret_cast<const float4*>(&s_g[c + 4 * lane]);
            const float w[4] = {__fmul_rn(u.x, sv.x), __fmul_rn(u.y, sv.y), __fmul_rn(u.z, sv.z),
                                __fmul_rn(u.w, sv.w)};
            float q[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float t = __fadd_rn(round_rne(__fdiv_rn(w[i], sf)), zf);
                q[i] = fminf(fmaxf(t, 0.0f), 15.0f);
            }
            uint32_t part = place_nibbles(q, odd);
            part |= __shfl_xor_sync(0xffffffffu, part, 1);
            if (!odd) qweight[(size_t)n * (K >> 3) + ((c0 + c) >> 3) + (lane >> 1)] = part;
        }
        if (lane == 0) {
            sc_sm[r] = __half_as_ushort(h);
            zc_sm[r] = (uint8_t)int_bits(zf);
        }
        if (bad) record_error(err, kErrValue);
    }
    __syncthreads();
    if (threadIdx.x < kLargeRows / 2) {
        const int r = 2 * threadIdx.x;
        if (row0 + r < N) {
            const uint32_t pair = (uint32_t)sc_sm[r] | ((uint32_t)sc_sm[r + 1] << 16);
            *reinterpret_cast<uint32_t*>(scales + (size_t)g * N + row0 + r) = pair;
        }
    }
    if (threadIdx.x < kLargeRows / 8) {
        const int w = threadIdx.x;
        if (row0 + 8 * w < N) {
            uint32_t word = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) word |= (uint32_t)(zc_sm[8 * w + b] & 15u) << (4 * b);
            zeros[(size_t)g * (N >> 3) + (row0 >> 3) + w] = word;
        }
    }
}

bool quantize_group_size_ok(int K, int gs) {
    if (gs == 128 || gs == 256 || gs == 512 || gs == 1024) return K % 1024 == 0;
    return gs > 1024 && gs % 1024 == 0 && gs <= kQuantMaxLargeGroup && K % gs == 0;
}

cudaError_t launch_awq_quantize(const float* W, const float* act, float alpha, int N, int K, int gs,
                                uint32_t* qweight, uint16_t* scales, uint32_t* zeros, float* s_out, unsigned* err,
                                cudaStream_t stream) {
    if (!quantize_group_size_ok(K, gs)) return cudaErrorInvalidValue;
    if (gs > 1024) {
        const int smem = gs * 4;
        cudaError_t e = cudaFuncSetAttribute(awq_quantize_large_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             smem);
        if (e != cudaSuccess) return e;
        dim3 grid(K / gs, (N + kLargeRows - 1) / kLargeRows);
        awq_quantize_large_kernel<<<grid, kQuantThreads, smem, stream>>>(W, act, alpha, N, K, gs, qweight, scales,
                                                                         zeros, s_out, err);
        return cudaGetLastError();
    }
    dim3 grid(K / 1024, (N + kRowsPerCta - 1) / kRowsPerCta);
    auto* kernel = gs == 128 ? awq_quantize_kernel<1>
                 : gs == 256 ? awq_quantize_kernel<2>
                 : gs == 512 ? awq_quantize_kernel<4>
                             : awq_quantize_kernel<8>;
    kernel<<<grid, kQuantThreads, 0, stream>>>(W, act, alpha, N, K, qweight, scales, zeros, s_out, err);
    return cudaGetLastError();
}

}  // namespace w4a16
