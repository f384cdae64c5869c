// quantize.cu -- AWQ activation-aware scaling + group-wise asymmetric uint4 RTN + packing.
//
// [AWQ (MLSys 2024) translation, section 3.2: per-input-channel scaling of the weights by a
//  factor derived from the activation magnitude; section 2: round-to-nearest; DeepCompressor
//  README, perplexity table row "W4A16 g128": groups of 128 along K; AWQ translation
//  section 1: TinyChat's 4-bit packing, 8 codes per 32-bit word.]
//
// Work decomposition (groups of up to 1024).  A CTA of 8 warps owns a tile of 64 rows x 1024
// columns (8 slices of 128); a warp quantizes one row at a time.  Lane l owns the 32
// consecutive weights l*32 .. l*32+31 of the row's chunk: a quarter of slice l/4.  So a group
// of 128 R weights belongs to 4 R neighbouring lanes: its min/max takes log2(4 R) shuffle
// rounds, the group's scale, zero point and reciprocal are computed once per lane for 32
// weights, and the lane's 32 codes are exactly 4 packed words, stored as one 16-byte store
// (the warp writes the row's 512 bytes of codes contiguously).  The lane's weights arrive as
// 8 16-byte loads through L1, where the first brings the warp's lines.  The fp16 scales and
// zero points of the tile are collected in shared memory and written group-major at the end
// (scales[g][n], zeros[g][n/8] with the nibbles of 8 consecutive rows), so those stores are
// coalesced too.
//
// Bit-exactness: every float step is a single IEEE operation with round-to-nearest-even
// (__fmul_rn, __fsub_rn, __fdiv_rn, __fadd_rn, __float2half_rn) or an exact equivalent of
// one.  The build does not use fast-math or flush-to-zero, so any correct implementation of
// the same steps gives the same bits.
//
// Throughput.  The weights stream once from HBM; the arithmetic per weight is kept to a few
// FMA-pipe and ALU operations, so that HBM rather than instruction issue is the limit:
//   - s is computed once per call by a small kernel (double pow, as the definition states)
//     into s_out, and the quantize kernel, launched so that it may start while that kernel
//     runs, fetches its first rows of W meanwhile.  Without s_out, every CTA computes the s
//     of its own 1024 columns.
//   - The per-weight division w' / sf is Markstein's method (P. Markstein, "Computation of
//     elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
//     1990): with y = RN(1/sf), the correctly rounded reciprocal, computed once per group,
//     q0 = RN(w' y), e = RN(w' - sf q0) (exact with an FMA), q1 = RN(q0 + e y).  It gives
//     q1 = RN(w' / sf), the IEEE quotient, for the divisors that occur here (sf has the 11
//     significant bits of an fp16); a GPU self-test (w4a16_selftest_quotient) compares it
//     with the IEEE division on every 11-bit divisor significand and every dividend
//     significand over the quotient range where rounding decides the code.  Groups whose
//     quotients could exceed 2^20 in magnitude clamp w' first; their codes saturate either
//     way.
//   - rint(q) + z and the integer code come from one add of 1.5 * 2^23 (round to nearest
//     even, exact for |q| < 2^22) and the float's low bits, clamped as integers.
//   - The group's minimum and maximum use NaN-propagating min/max, so one finiteness test
//     per group replaces one per weight.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kQuantThreads = 256;

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kIntMagic = 8388608.0f;      // 2^23

// round-to-nearest-even to an integral float; exact for |v| < 2^22 (see above)
__device__ __forceinline__ float round_rne(float v) { return __fsub_rn(__fadd_rn(v, kRoundMagic), kRoundMagic); }

// rint(v) as an integer, for |v| < 2^22: v + 1.5 * 2^23 lies in [2^23, 2^24), where the float's
// unit is 1, so the addition rounds v to the nearest integer (ties to even) and the low bits
// hold 2^22 + rint(v).
__device__ __forceinline__ int rint_int(float v) {
    return (int)(__float_as_uint(__fadd_rn(v, kRoundMagic)) - 0x4B400000u);
}

__device__ __forceinline__ float max_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ float min_nan(float a, float b) {
    float r;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// The code of w' in a group with scale sf (y = RN(1/sf)) and integer zero point z:
// clamp(rint(w' / sf) + z, 0, qmax), for |w' / sf| < 2^21 (qmax = 15 for 4-bit codes, 7 for 3-bit).
template <int QMAX>
__device__ __forceinline__ uint32_t code_of(float w, float sf, float y, int z) {
    const int t = rint_int(quotient_markstein(w, sf, y)) + z;
    return (uint32_t)min(max(t, 0), QMAX);
}

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

// s_k = max(float(pow(double(a_k), double(alpha))), 1e-4), once per call.  The next kernel on
// the stream (the quantizer) may start at once and fetch its first weights meanwhile.
__global__ void __launch_bounds__(256) awq_scale_kernel(const float* __restrict__ act, float alpha, int K,
                                                        float* __restrict__ s, unsigned* err) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int k = blockIdx.x * 256 + threadIdx.x;
    if (k >= K) return;
    const float a = act[k];
    const float p = (float)pow((double)a, (double)alpha);
    if (!(a >= 0.0f) || isinf(a) || !isfinite(p)) record_error(err, kErrValue);
    s[k] = p > 1e-4f ? p : 1e-4f;
}

// CTAs of the g128 kernel resident per SM (the register budget per thread follows from it).
#ifndef W4A16_QUANT_CTAS_PER_SM
#define W4A16_QUANT_CTAS_PER_SM 4
#endif

// Nibble position of element e (0..7) of an 8-wide block: ORDER[pos] = e with
// ORDER = {0,2,4,6,1,3,5,7}.
__device__ __forceinline__ constexpr int nibble_of(int e) { return (e & 1) ? 4 + (e >> 1) : (e >> 1); }

// Groups of 128 R weights, R in {1, 2, 4, 8}: a 1024-column chunk holds 8 / R whole groups.
// A CTA takes ROWS (32 or 64) rows.  s_pre: the channel scales computed by awq_scale_kernel
// just before (read after it has finished), or nullptr: the CTA computes the s of its columns.
// BITS = 4: codes 0..15, 8 per word, qweight [N][K/8].  BITS = 3 (SqueezeLLM article,
// sections 2.1-2.2: eight levels): codes 0..7, the 32 codes of k = 32b .. 32b + 31 in the
// three words qweight[n][3b + w]: bits 4j .. 4j+2 of word w hold element 8w + ORDER[j], bit
// 4j + 3 holds bit w of element 24 + ORDER[j]; qweight [N][3K/32].
template <int R, int ROWS, int BITS>
__global__ void __launch_bounds__(kQuantThreads, W4A16_QUANT_CTAS_PER_SM)
awq_quantize_kernel(const float* __restrict__ W, const float* __restrict__ act, const float* s_pre, float alpha,
                    int N, int K, uint32_t* __restrict__ qweight, uint16_t* __restrict__ scales,
                    uint32_t* __restrict__ zeros, unsigned* err) {
    constexpr int GC = 8 / R;  // groups per chunk
    constexpr int LG = 4 * R;  // lanes per group
    constexpr int QMAX = BITS == 4 ? 15 : 7;
    static_assert(BITS == 4 || BITS == 3, "4- or 3-bit codes");
    // s of the chunk, lane l's 32 values in 8 16-byte pieces, piece c at l*128 + 16 (c ^ (l & 7)),
    // so that a quarter warp's 16-byte reads hit 8 different bank groups
    __shared__ __align__(16) float s_sm[1024];
    __shared__ __align__(16) uint16_t sc_sm[GC][ROWS];  // fp16 scale bits per (group, row)
    __shared__ uint8_t zc_sm[GC][ROWS];                 // zero point per (group, row)
    const int kc = blockIdx.x;                 // 1024-column chunk (groups GC kc .. GC kc + GC - 1)
    const int row0 = blockIdx.y * ROWS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sw = lane & 7;                   // this lane's swizzle

    // the warp's first row, fetched before s is available; w holds the row's weights, then
    // the scaled weights in place
    float w[32];
    auto load_row = [&](int n) {
        const float4* wrow = reinterpret_cast<const float4*>(W + (size_t)n * K + (size_t)kc * 1024 + 32 * lane);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 u = ldg_cached(wrow + c);
            w[4 * c] = __uint_as_float(u.x);
            w[4 * c + 1] = __uint_as_float(u.y);
            w[4 * c + 2] = __uint_as_float(u.z);
            w[4 * c + 3] = __uint_as_float(u.w);
        }
    };
    if (row0 + warp < N) load_row(row0 + warp);

    // thread i places s[4 i .. 4 i + 3]: owner lane i / 8, piece i % 8
    if (s_pre != nullptr) {
        asm volatile("griddepcontrol.wait;" ::: "memory");  // s was written by the previous kernel
        const float4 sv = reinterpret_cast<const float4*>(s_pre + (size_t)kc * 1024)[threadIdx.x];
        const int ol = threadIdx.x >> 3, c = threadIdx.x & 7;
        reinterpret_cast<float4*>(s_sm)[ol * 8 + (c ^ (ol & 7))] = sv;
    } else {
        float sv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float a = act[(size_t)kc * 1024 + 4 * threadIdx.x + e];
            const float p = (float)pow((double)a, (double)alpha);
            if (!(a >= 0.0f) || isinf(a) || !isfinite(p)) record_error(err, kErrValue);
            sv[e] = p > 1e-4f ? p : 1e-4f;
        }
        const int ol = threadIdx.x >> 3, c = threadIdx.x & 7;
        reinterpret_cast<float4*>(s_sm)[ol * 8 + (c ^ (ol & 7))] = make_float4(sv[0], sv[1], sv[2], sv[3]);
    }
    __syncthreads();

    for (int r = warp; r < ROWS; r += kQuantThreads / 32) {
        const int n = row0 + r;
        if (n >= N) break;  // warp-uniform
        if (r != warp) load_row(n);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 s4 = reinterpret_cast<const float4*>(s_sm)[lane * 8 + (c ^ sw)];  // s of these 4 columns
            w[4 * c] = __fmul_rn(w[4 * c], s4.x);
            w[4 * c + 1] = __fmul_rn(w[4 * c + 1], s4.y);
            w[4 * c + 2] = __fmul_rn(w[4 * c + 2], s4.z);
            w[4 * c + 3] = __fmul_rn(w[4 * c + 3], s4.w);
        }
        float mx = w[0], mn = w[0];
#pragma unroll
        for (int i = 1; i < 32; ++i) {
            mx = max_nan(mx, w[i]);
            mn = min_nan(mn, w[i]);
        }
#pragma unroll
        for (int o = 1; o < LG; o <<= 1) {
            mx = max_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mn = min_nan(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        }
        const bool bad_range = !isfinite(mx) || !isfinite(mn);  // NaN or Inf anywhere in the group
        float scale32 = __fdiv_rn(__fsub_rn(mx, mn), (float)QMAX);
        if (scale32 < 1e-5f) scale32 = 1e-5f;
        const __half h = __float2half_rn(scale32);
        const float sf = __half2float(h);
        const bool bad = bad_range || isinf(scale32) || isinf(sf);
        float zf = rintf(__fdiv_rn(-mn, sf));
        zf = fminf(fmaxf(zf, 0.0f), (float)QMAX);
        const int zi = (int)int_bits(zf);
        const float y = __frcp_rn(sf);
        // |w' / sf| < 2^20 for the whole group: no clamp before dividing
        const bool small = __fmul_rn(fmaxf(fabsf(mx), fabsf(mn)), y) < 1048576.0f;
        if (!small) {
            const float lim = __fmul_rn(sf, 1048576.0f);  // exact: sf times a power of two
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = fminf(fmaxf(w[i], -lim), lim);
        }
        if constexpr (BITS == 4) {
            uint32_t word[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                uint32_t acc = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) acc |= code_of<QMAX>(w[8 * b + e], sf, y, zi) << (4 * nibble_of(e));
                word[b] = acc;
            }
            *reinterpret_cast<uint4*>(qweight + (size_t)n * (K >> 3) + (size_t)kc * 128 + 4 * lane) =
                make_uint4(word[0], word[1], word[2], word[3]);
        } else {
            uint32_t word[3] = {0u, 0u, 0u};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int j = nibble_of(e);
                const uint32_t hi = code_of<QMAX>(w[24 + e], sf, y, zi);  // its 3 bits go to the 3 words
#pragma unroll
                for (int b = 0; b < 3; ++b)
                    word[b] |= (code_of<QMAX>(w[8 * b + e], sf, y, zi) | (((hi >> b) & 1u) << 3)) << (4 * j);
            }
            uint32_t* dst = qweight + (size_t)n * (3 * (K >> 5)) + (size_t)kc * 96 + 3 * lane;
            dst[0] = word[0];
            dst[1] = word[1];
            dst[2] = word[2];
        }
        if ((lane & (LG - 1)) == 0) {
            sc_sm[lane / LG][r] = __half_as_ushort(h);
            zc_sm[lane / LG][r] = (uint8_t)zi;
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(err, kErrValue);
    }
    __syncthreads();

    // group-major parameters: scales[g][n] (row pairs as one 32-bit store) and zeros[g][n/8]
    // (the nibbles of 8 consecutive rows), both coalesced along n
    {
        const int g = threadIdx.x >> 5, j = threadIdx.x & 31;  // up to 8 groups x 32 row pairs
        const int r = 2 * j;
        if (g < GC && r < ROWS && row0 + r < N) {
            const uint32_t pair = (uint32_t)sc_sm[g][r] | ((uint32_t)sc_sm[g][r + 1] << 16);
            *reinterpret_cast<uint32_t*>(scales + ((size_t)kc * GC + g) * N + row0 + r) = pair;
        }
        if (threadIdx.x < 8 * (ROWS / 8)) {
            const int gz = threadIdx.x / (ROWS / 8), w8 = threadIdx.x % (ROWS / 8);
            if (gz < GC && row0 + 8 * w8 < N) {
                uint32_t word = 0;
#pragma unroll
                for (int b = 0; b < 8; ++b) word |= (uint32_t)(zc_sm[gz][8 * w8 + b] & 15u) << (4 * b);
                zeros[((size_t)kc * GC + gz) * (N >> 3) + (row0 >> 3) + w8] = word;
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

cudaError_t launch_awq_scale(const float* act, float alpha, int K, float* s_out, unsigned* err, cudaStream_t stream) {
    awq_scale_kernel<<<(K + 255) / 256, 256, 0, stream>>>(act, alpha, K, s_out, err);
    return cudaGetLastError();
}

bool quantize_group_size_ok(int K, int gs) {
    if (gs == 128 || gs == 256 || gs == 512 || gs == 1024) return K % 1024 == 0;
    return gs > 1024 && gs % 1024 == 0 && gs <= kQuantMaxLargeGroup && K % gs == 0;
}

cudaError_t launch_awq_quantize(const float* W, const float* act, float alpha, int N, int K, int gs,
                                uint32_t* qweight, uint16_t* scales, uint32_t* zeros, float* s_out, int num_sms,
                                unsigned* err, cudaStream_t stream, int bits) {
    if (!quantize_group_size_ok(K, gs) || (bits != 4 && bits != 3) || (bits == 3 && gs > 1024))
        return cudaErrorInvalidValue;
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
    // 64-row tiles, or 32-row ones when 64-row tiles would not fill the resident CTA slots twice
    const bool small = (long long)(K / 1024) * ((N + 63) / 64) < 2LL * W4A16_QUANT_CTAS_PER_SM * num_sms;
    const int rows = small ? 32 : 64;
    using Kernel = void (*)(const float*, const float*, const float*, float, int, int, uint32_t*, uint16_t*,
                            uint32_t*, unsigned*);
    static const Kernel k4[2][4] = {
        {awq_quantize_kernel<1, 64, 4>, awq_quantize_kernel<2, 64, 4>, awq_quantize_kernel<4, 64, 4>,
         awq_quantize_kernel<8, 64, 4>},
        {awq_quantize_kernel<1, 32, 4>, awq_quantize_kernel<2, 32, 4>, awq_quantize_kernel<4, 32, 4>,
         awq_quantize_kernel<8, 32, 4>}};
    static const Kernel k3[2][4] = {
        {awq_quantize_kernel<1, 64, 3>, awq_quantize_kernel<2, 64, 3>, awq_quantize_kernel<4, 64, 3>,
         awq_quantize_kernel<8, 64, 3>},
        {awq_quantize_kernel<1, 32, 3>, awq_quantize_kernel<2, 32, 3>, awq_quantize_kernel<4, 32, 3>,
         awq_quantize_kernel<8, 32, 3>}};
    const int ri = gs == 128 ? 0 : gs == 256 ? 1 : gs == 512 ? 2 : 3;
    const Kernel kernel = (bits == 4 ? k4 : k3)[small ? 1 : 0][ri];
    const dim3 grid(K / 1024, (N + rows - 1) / rows);
    if (s_out == nullptr) {
        kernel<<<grid, kQuantThreads, 0, stream>>>(W, act, nullptr, alpha, N, K, qweight, scales, zeros, err);
        return cudaGetLastError();
    }
    // s once into s_out, then the quantizer, which streams its weights while s is computed
    awq_scale_kernel<<<(K + 255) / 256, 256, 0, stream>>>(act, alpha, K, s_out, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kQuantThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, W, act, (const float*)s_out, alpha, N, K, qweight, scales, zeros, err);
}

}  // namespace w4a16
