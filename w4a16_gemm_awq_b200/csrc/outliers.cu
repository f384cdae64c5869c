// outliers.cu -- dense-and-sparse split of a weight matrix on the GPU.
//
// [SqueezeLLM article, section 2.2: a small set of sensitive weights is kept in fp16 as a
//  sparse matrix and removed from the dense part, W = W_dense + W_sparse; section 5.3: the
//  sparsity ratio 0.45%.  The sensitivity is read as |w| * a_k with a_k the mean |x| of input
//  channel k: the article's Hessian-based score needs gradients of a trained model.]
//
// What it computes (the same rule as the CPU oracle):
//   score(n, k) = fp32(|w(n, k)| * a_k)            (one IEEE multiply)
//   key = (bits(score) << 32) | (0xFFFFFFFF - (n K + k))
//   the nnz entries with the largest keys are the outliers: larger score first, and among
//   equal scores the lower linear index first;
//   W_dense = W with those entries set to 0;
//   CSR: row_ptr [N+1], col_idx ascending within each row, values fp16(w * s_k) with
//   s_k = max(float(pow(a_k, alpha)), 1e-4) (the AWQ scale, so the values live in the same
//   scaled space as the packed dense part).
//
// Design: a radix select on the 32-bit score (non-negative floats order like their bit
// patterns), then the ties at the threshold score are resolved in index order.
//   1. Three histogram passes over digits of 12, 10 and 10 bits of the score.  Each pass
//      counts only the entries whose higher digits equal the prefix found so far (shared-
//      memory histogram per CTA, then global atomics).  After each pass one CTA scans the
//      histogram from the top and finds the digit where the running count reaches the number
//      still needed.  The result is the threshold score T and the number r of entries with
//      score == T to take (1 <= r <= their count).
//   2. A row pass counts, per row, the entries with score > T and those with score == T.
//   3. One CTA scans the rows: the ties are taken in index order, so row n takes
//      clamp(r - ties_before_row_n, 0, ties_in_row_n); row_ptr is the running sum of
//      (greater + taken).
//   4. A fill pass (one warp per row, columns in order) writes col_idx and values through a
//      ballot/popc compaction, and W_dense.
// Every pass streams W (and a) once; all control stays on the device, so the host issues the
// whole sequence without waiting.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kSplitThreads = 256;
constexpr int kSplitBins = 4096;  // the widest digit (12 bits)

// Device-side state of the selection: the prefix found so far and the count still needed.
struct SplitState {
    uint32_t prefix;  // the score bits fixed so far (high digits), left-aligned
    uint32_t need;    // entries still to take at or below the current prefix
    uint32_t err;     // unused, keeps the struct 16 bytes
    uint32_t pad;
};

// digit boundaries: bits [31:20], [19:10], [9:0]
__device__ __forceinline__ int digit_shift(int level) { return level == 0 ? 20 : (level == 1 ? 10 : 0); }
__device__ __forceinline__ int digit_bins(int level) { return level == 0 ? 4096 : 1024; }

__device__ __forceinline__ uint32_t score_bits(float w, float a) { return __float_as_uint(__fmul_rn(fabsf(w), a)); }

// Calls f(k, w, a) for every element of row `row` (K entries), lanes of a warp along the row.
// VEC: K % 4 == 0 and 16-byte aligned rows and act, so that each lane reads 4 consecutive
// entries with one 128-bit load.
template <bool VEC, typename F>
__device__ __forceinline__ void for_row(const float* __restrict__ row, const float* __restrict__ act, uint32_t K,
                                        int lane, F&& f) {
    if (VEC) {
        const float4* r4 = reinterpret_cast<const float4*>(row);
        const float4* a4 = reinterpret_cast<const float4*>(act);
        for (uint32_t q = lane; q < (K >> 2); q += 32) {
            const float4 w = r4[q], a = __ldg(a4 + q);
            f(4 * q, w.x, a.x);
            f(4 * q + 1, w.y, a.y);
            f(4 * q + 2, w.z, a.z);
            f(4 * q + 3, w.w, a.w);
        }
    } else {
        for (uint32_t k = lane; k < K; k += 32) f(k, row[k], __ldg(act + k));
    }
}

// Histogram of digit `level` over the entries whose higher digits equal state->prefix.
template <bool VEC>
__global__ void __launch_bounds__(kSplitThreads)
split_hist_kernel(const float* __restrict__ W, const float* __restrict__ act, uint32_t N, uint32_t K, int level,
                  const SplitState* __restrict__ state, unsigned* __restrict__ hist, unsigned* err) {
    __shared__ unsigned h[kSplitBins];
    const int bins = digit_bins(level), shift = digit_shift(level);
    for (int i = threadIdx.x; i < bins; i += kSplitThreads) h[i] = 0;
    __syncthreads();
    const uint32_t prefix = level == 0 ? 0u : state->prefix;
    const uint32_t hi_mask = level == 0 ? 0u : (0xFFFFFFFFu << (shift + 10));  // the digits above this one
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    bool bad = false;
    // one warp per row, lanes along the row (coalesced, and a_k indexed directly)
    for (uint32_t n = blockIdx.x * (kSplitThreads / 32) + warp; n < N; n += gridDim.x * (kSplitThreads / 32)) {
        for_row<VEC>(W + (size_t)n * K, act, K, lane, [&](uint32_t, float w, float a) {
            if (level == 0 && (!isfinite(w) || !(a >= 0.0f) || isinf(a))) bad = true;
            const uint32_t b = score_bits(w, a);
            if ((b & hi_mask) == prefix) atomicAdd(&h[(b >> shift) & (uint32_t)(bins - 1)], 1u);
        });
    }
    if (bad) record_error(err, kErrValue);
    __syncthreads();
    for (int i = threadIdx.x; i < bins; i += kSplitThreads)
        if (h[i]) atomicAdd(&hist[i], h[i]);
}

// One CTA: the digit d where the running count from the top reaches state->need; the prefix
// gains d and need becomes need - (entries in higher digits).  Clears the histogram for the
// next pass.
__global__ void __launch_bounds__(1024)
split_select_kernel(unsigned* __restrict__ hist, int level, SplitState* __restrict__ state) {
    __shared__ unsigned part[1024];
    __shared__ unsigned found_digit, found_above;
    const int bins = digit_bins(level), shift = digit_shift(level);
    const int per = bins / 1024;  // 4 or 1 bins per thread, taken from the top down
    const int t = threadIdx.x;
    // thread t owns bins [bins - (t+1) per, bins - t per): descending order across threads
    unsigned c[4] = {0, 0, 0, 0};
    unsigned sum = 0;
    for (int j = 0; j < per; ++j) {
        c[j] = hist[bins - 1 - (t * per + j)];
        sum += c[j];
    }
    part[t] = sum;
    if (t == 0) {
        found_digit = 0xFFFFFFFFu;
        found_above = 0;
    }
    __syncthreads();
    // inclusive scan of part[] (counts from the top)
    for (int off = 1; off < 1024; off <<= 1) {
        const unsigned v = t >= off ? part[t - off] : 0u;
        __syncthreads();
        part[t] += v;
        __syncthreads();
    }
    const unsigned need = state->need;
    const unsigned before = t > 0 ? part[t - 1] : 0u;  // entries in bins above this thread's
    if (before < need && part[t] >= need) {
        unsigned run = before;
        for (int j = 0; j < per; ++j) {
            if (run + c[j] >= need) {
                found_digit = (unsigned)(bins - 1 - (t * per + j));
                found_above = run;
                break;
            }
            run += c[j];
        }
    }
    __syncthreads();
    if (t == 0 && found_digit != 0xFFFFFFFFu) {
        state->prefix = (level == 0 ? 0u : state->prefix) | (found_digit << shift);
        state->need = need - found_above;
    }
    __syncthreads();
    for (int i = t; i < bins; i += 1024) hist[i] = 0;
}

// Per row: entries with score > T and with score == T (T = state->prefix after 3 levels).
template <bool VEC>
__global__ void __launch_bounds__(kSplitThreads)
split_rowcount_kernel(const float* __restrict__ W, const float* __restrict__ act, uint32_t N, uint32_t K,
                      const SplitState* __restrict__ state, unsigned* __restrict__ gt, unsigned* __restrict__ ties) {
    const uint32_t T = state->prefix;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (uint32_t n = blockIdx.x * (kSplitThreads / 32) + warp; n < N; n += gridDim.x * (kSplitThreads / 32)) {
        unsigned g = 0, e = 0;
        for_row<VEC>(W + (size_t)n * K, act, K, lane, [&](uint32_t, float w, float a) {
            const uint32_t b = score_bits(w, a);
            g += b > T;
            e += b == T;
        });
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            e += __shfl_xor_sync(0xffffffffu, e, o);
        }
        if (lane == 0) {
            gt[n] = g;
            ties[n] = e;
        }
    }
}

// One CTA: ties are taken in index order (row by row), row_ptr is the running sum.
__global__ void __launch_bounds__(1024)
split_scan_kernel(uint32_t N, const SplitState* __restrict__ state, const unsigned* __restrict__ gt,
                  unsigned* __restrict__ ties_take, int32_t* __restrict__ row_ptr, unsigned* err) {
    __shared__ unsigned s_tie[1024], s_cnt[1024];
    __shared__ unsigned carry_tie, carry_cnt;
    const unsigned r = state->need;
    const int t = threadIdx.x;
    if (t == 0) {
        carry_tie = 0;
        carry_cnt = 0;
        row_ptr[0] = 0;
    }
    __syncthreads();
    for (uint32_t base = 0; base < N; base += 1024) {
        const uint32_t n = base + t;
        const unsigned e = n < N ? ties_take[n] : 0u;  // ties in the row (rowcount wrote them here)
        s_tie[t] = e;
        __syncthreads();
        for (int off = 1; off < 1024; off <<= 1) {
            const unsigned v = t >= off ? s_tie[t - off] : 0u;
            __syncthreads();
            s_tie[t] += v;
            __syncthreads();
        }
        const unsigned tie_before = carry_tie + s_tie[t] - e;
        const unsigned take = tie_before >= r ? 0u : (r - tie_before < e ? r - tie_before : e);
        const unsigned cnt = n < N ? gt[n] + take : 0u;
        s_cnt[t] = cnt;
        __syncthreads();
        for (int off = 1; off < 1024; off <<= 1) {
            const unsigned v = t >= off ? s_cnt[t - off] : 0u;
            __syncthreads();
            s_cnt[t] += v;
            __syncthreads();
        }
        if (n < N) {
            ties_take[n] = take;
            row_ptr[n + 1] = (int32_t)(carry_cnt + s_cnt[t]);
        }
        __syncthreads();
        if (t == 1023) {
            carry_tie += s_tie[1023];
            carry_cnt += s_cnt[1023];
        }
        __syncthreads();
    }
    (void)err;
}

// Exclusive prefix sum over the warp's lanes, and the warp total.
__device__ __forceinline__ unsigned warp_excl_scan(unsigned v, int lane, unsigned* total) {
    unsigned x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    *total = __shfl_sync(0xffffffffu, x, 31);
    return x - v;
}

// The CSR entry of a chosen weight: column k, value fp16(w * s_k).
__device__ __forceinline__ bool write_entry(uint32_t at, uint32_t nnz, uint32_t k, float w, float a, float alpha,
                                            int32_t* col_idx, uint16_t* values, unsigned* err) {
    if (at >= nnz) {  // never true (the counts are exact); never write past the arrays
        record_error(err, kErrShape);
        return false;
    }
    const float p = (float)pow((double)a, (double)alpha);
    const float s = p > 1e-4f ? p : 1e-4f;
    const __half hv = __float2half_rn(__fmul_rn(w, s));
    col_idx[at] = (int32_t)k;
    values[at] = __half_as_ushort(hv);
    return isinf(__half2float(hv));
}

// One warp per row: columns in order, chosen = score > T or (score == T and among the
// row's first ties_take[n] ties).  Writes the CSR entries and W_dense.  VEC: each lane takes
// 4 consecutive columns of every 128-column chunk (ranks within the chunk by a warp scan of
// the lanes' counts); otherwise one column per lane and 32-column chunks (ranks by ballot).
template <bool VEC>
__global__ void __launch_bounds__(kSplitThreads)
split_fill_kernel(const float* __restrict__ W, const float* __restrict__ act, float alpha, uint32_t N, uint32_t K,
                  uint32_t nnz, const SplitState* __restrict__ state, const unsigned* __restrict__ ties_take,
                  const int32_t* __restrict__ row_ptr, float* __restrict__ W_dense, int32_t* __restrict__ col_idx,
                  uint16_t* __restrict__ values, unsigned* err) {
    const uint32_t T = state->prefix;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    bool bad = false;
    for (uint32_t n = blockIdx.x * (kSplitThreads / 32) + warp; n < N; n += gridDim.x * (kSplitThreads / 32)) {
        const float* row = W + (size_t)n * K;
        float* drow = W_dense + (size_t)n * K;
        uint32_t pos = (uint32_t)row_ptr[n];
        const unsigned take = ties_take[n];
        unsigned ties_seen = 0;
        if (VEC) {
            for (uint32_t q0 = 0; q0 < (K >> 2); q0 += 32) {
                const uint32_t q = q0 + lane;
                const bool in = q < (K >> 2);
                const float4 w4 = in ? reinterpret_cast<const float4*>(row)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
                const float4 a4 = in ? __ldg(reinterpret_cast<const float4*>(act) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
                const float w[4] = {w4.x, w4.y, w4.z, w4.w}, a[4] = {a4.x, a4.y, a4.z, a4.w};
                bool gt[4], tie[4];
                unsigned nt = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t b = score_bits(w[j], a[j]);
                    gt[j] = in && b > T;
                    tie[j] = in && b == T;
                    nt += tie[j];
                }
                unsigned tie_total, ch_total;
                unsigned tie_rank = ties_seen + warp_excl_scan(nt, lane, &tie_total);
                bool chosen[4];
                unsigned nc = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    chosen[j] = gt[j] || (tie[j] && tie_rank < take);
                    tie_rank += tie[j];
                    nc += chosen[j];
                }
                uint32_t at = pos + warp_excl_scan(nc, lane, &ch_total);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (chosen[j]) bad |= write_entry(at++, nnz, 4 * q + j, w[j], a[j], alpha, col_idx, values, err);
                if (in)
                    reinterpret_cast<float4*>(drow)[q] = make_float4(chosen[0] ? 0.f : w[0], chosen[1] ? 0.f : w[1],
                                                                     chosen[2] ? 0.f : w[2], chosen[3] ? 0.f : w[3]);
                pos += ch_total;
                ties_seen += tie_total;
            }
        } else {
            for (uint32_t k0 = 0; k0 < K; k0 += 32) {
                const uint32_t k = k0 + lane;
                const bool in = k < K;
                const float w = in ? row[k] : 0.0f;
                const float a = in ? act[k] : 0.0f;
                const uint32_t b = score_bits(w, a);
                const bool tie = in && b == T;
                const unsigned tie_mask = __ballot_sync(0xffffffffu, tie);
                const unsigned tie_rank = ties_seen + __popc(tie_mask & ((1u << lane) - 1u));
                const bool chosen = in && (b > T || (tie && tie_rank < take));
                const unsigned ch_mask = __ballot_sync(0xffffffffu, chosen);
                if (chosen)
                    bad |= write_entry(pos + __popc(ch_mask & ((1u << lane) - 1u)), nnz, k, w, a, alpha, col_idx,
                                       values, err);
                if (in) drow[k] = chosen ? 0.0f : w;
                pos += __popc(ch_mask);
                ties_seen += __popc(tie_mask);
            }
        }
    }
    if (bad) record_error(err, kErrValue);
}

// The selection state starts at (prefix 0, need nnz) and the histogram at zero.  A kernel
// (not a host-to-device copy) sets them, so the whole split can be captured in a CUDA graph.
__global__ void split_init_kernel(SplitState* state, unsigned* hist, uint32_t nnz) {
    if (threadIdx.x == 0) {
        state->prefix = 0u;
        state->need = nnz;
        state->err = 0u;
        state->pad = 0u;
    }
    for (int i = threadIdx.x; i < kSplitBins; i += blockDim.x) hist[i] = 0;
}

size_t split_workspace_bytes(int64_t N) {
    return 256 + (size_t)kSplitBins * 4 + 3 * (((size_t)N * 4 + 255) / 256) * 256;
}

cudaError_t launch_split_outliers(const float* W, const float* act, float alpha, uint32_t N, uint32_t K, uint32_t nnz,
                                  float* W_dense, int32_t* row_ptr, int32_t* col_idx, uint16_t* values,
                                  void* workspace, int num_sms, unsigned* err, cudaStream_t stream) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    SplitState* state = reinterpret_cast<SplitState*>(ws);
    unsigned* hist = reinterpret_cast<unsigned*>(ws + 256);
    const size_t row_bytes = (((size_t)N * 4 + 255) / 256) * 256;
    unsigned* gt = reinterpret_cast<unsigned*>(ws + 256 + kSplitBins * 4);
    unsigned* ties = reinterpret_cast<unsigned*>(ws + 256 + kSplitBins * 4 + row_bytes);
    split_init_kernel<<<1, 1024, 0, stream>>>(state, hist, nnz);
    const int grid = 4 * num_sms;
    auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    const bool vec = (K & 3u) == 0 && a16(W) && a16(act) && a16(W_dense);
    for (int level = 0; level < 3; ++level) {
        if (vec)
            split_hist_kernel<true><<<grid, kSplitThreads, 0, stream>>>(W, act, N, K, level, state, hist, err);
        else
            split_hist_kernel<false><<<grid, kSplitThreads, 0, stream>>>(W, act, N, K, level, state, hist, err);
        split_select_kernel<<<1, 1024, 0, stream>>>(hist, level, state);
    }
    if (vec)
        split_rowcount_kernel<true><<<grid, kSplitThreads, 0, stream>>>(W, act, N, K, state, gt, ties);
    else
        split_rowcount_kernel<false><<<grid, kSplitThreads, 0, stream>>>(W, act, N, K, state, gt, ties);
    split_scan_kernel<<<1, 1024, 0, stream>>>(N, state, gt, ties, row_ptr, err);
    if (vec)
        split_fill_kernel<true><<<grid, kSplitThreads, 0, stream>>>(W, act, alpha, N, K, nnz, state, ties, row_ptr,
                                                                    W_dense, col_idx, values, err);
    else
        split_fill_kernel<false><<<grid, kSplitThreads, 0, stream>>>(W, act, alpha, N, K, nnz, state, ties, row_ptr,
                                                                     W_dense, col_idx, values, err);
    return cudaGetLastError();
}

}  // namespace w4a16
