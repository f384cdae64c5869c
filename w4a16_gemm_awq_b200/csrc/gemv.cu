// gemv.cu -- decode W4A16 GEMV (1 <= M <= 16): y = bf16(x . dequant(Q)^T [+ x . W_sparse^T]).
//
// [AWQ (MLSys 2024) translation, section 1: TinyChat computes the linear layer from packed
//  4-bit weights dequantized on the fly; at decode batch sizes the layer is bound by memory
//  bandwidth (section 2: weight-only quantization relieves the memory bottleneck).
//  SqueezeLLM article, section 2.3: the fp16 sparse term is added to the dense product.]
//
// Design (B200).  Each packed weight byte is streamed once from HBM by a persistent grid of
// one CTA per SM.
//   - Work units are (128-channel row block, block of 4 quantization groups = 512 k): 32 KB
//     of packed weights, brought in by ONE TMA copy.  A CTA's TMA copies are served nearly
//     one after another, so the bytes per copy set the streaming rate of a CTA: 8 KB copies
//     stream at ~16 GB/s per CTA, 32 KB copies at ~40 GB/s, enough for one CTA per SM to
//     saturate HBM.  The copy uses a 3-D view of qweight (16 words of a group, rows, groups;
//     strides K/2 and 64 bytes), so it lands as [4 groups][128 rows][64 bytes] and the
//     consumers' 128-bit loads of one group are free of bank conflicts.
//   - Stream-K: CTA p takes the contiguous unit range [p*T/P, (p+1)*T/P), ordered row block
//     by row block, so every CTA streams the same number of bytes in one balanced wave.  A
//     row block processed whole by one CTA is written straight to y.  A row block split
//     between CTAs leaves fp32 partial tiles in the caller's workspace.  Each contributing
//     CTA then increments the row block's counter.  The CTA that completes the count sums
//     the partials once its own stream has ended, writes y and resets the counter to zero.
//     No CTA waits for another, and the workspace is all-zero again after every call.
//   - Warps: 8 consumers, 1 TMA producer (weights), 2 helpers, 1 epilogue.  Everything
//     except the weights comes in through the helpers with ordinary loads, so the weights
//     are the only TMA traffic.  For their 2 groups of each unit the helpers
//       * copy the activations from global memory (L2-resident) into shared memory, already
//         in the order of the MMA B fragments;
//       * compute the group sums X_g of every token with tensor-core MMAs against an
//         all-ones A operand;
//       * decode the scales and zero points of the unit's 128 rows into fp32 pairs
//         (s, -(128 + z)).
//   - Consumer warp c owns rows 32 (c % 4) .. +31 and groups 2 (c / 4), +1 of every unit
//     (two m16 tiles x two groups).  The MMA is the legacy mma.sync m16n8k16 with swapped
//     operands: rows are 16 channels, columns 8 tokens (two tiles when M > 8), depth 16 input
//     channels.  The A operand (weights) goes from shared memory to registers.  One LOP3 per
//     nibble pair makes the bf16 pair (128 + q_lo, 128 + q_hi) (exponent bits 0x43), and
//     those exact values feed the MMA unchanged.  The zero point and the scale are applied
//     once per group in fp32:
//         acc += s * ( sum_k (128 + q_k) x_k  -  (128 + z) * X_g ).
//   - Which physical k feeds which MMA slot.  Thread t (= lane % 4) takes words 4t..4t+3 of
//     a row's group, i.e. k in [32t, 32t+32).  MMA pair w (0..3) uses word w: nibble pairs
//     (0,1) in the first MMA and (2,3) in the second.  Pair p of word w holds
//     k = 32t + 8w + 2p + {0,1}.  The B fragment of thread (token g, t) is then the 16 bytes
//     x[g][32t + 8w .. +8], whose four 32-bit parts are the same pairs.
//   - At the end of a row-block segment the consumers drop their accumulators into a
//     shared-memory partial tile (one half per group pair) and go on streaming; the
//     epilogue warp adds the halves and does the workspace exchange, the CSR term and the
//     stores of y.
//   - Programmatic dependent launch.  The weights may be fetched before the previous kernel
//     on the stream has finished.  The helpers wait for it before they load x; the
//     epilogue and the completion phase wait before they touch the workspace or y.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kGemvRows = 128;                                  // output channels per row block
constexpr int kGemvUnitGroups = 4;                              // groups of 128 k per work unit
constexpr int kGemvGroupBytes = kGemvRows * 64;                 // one group of packed weights, 128 rows
constexpr int kGemvWBytes = kGemvUnitGroups * kGemvGroupBytes;  // 32 KB per unit
constexpr int kGemvConsumers = 8;                               // warps 0..7
constexpr int kGemvProducer = 8;                                // warp 8
constexpr int kGemvHelper0 = 9;                                 // warps 9, 10
constexpr int kGemvHelpers = 2;
constexpr int kGemvEpilogue = 11;                               // warp 11
constexpr int kGemvThreads = 32 * 12;
constexpr int kGemvStages = 4;
constexpr int kGemvSlotFloats = kGemvRows * 16;                 // one partial tile in the workspace

struct GemvArgs {
    const uint16_t* x;
    const uint16_t* scales;
    const uint32_t* zeros;
    const int32_t* row_ptr;
    const int32_t* col_idx;
    const uint16_t* vals;
    long long nnz;
    uint16_t* y;
    float* partials;     // workspace: [2P][128][16] fp32
    unsigned* counters;  // workspace: [N/128], zero between calls
    int M, N, K;
    uint32_t T;          // work units = (N/128) * (K/512); T * P < 2^32 (checked by the caller)
    int P;               // CTAs
    unsigned* err;
};

template <int NT>
struct GemvSmem {
    static constexpr int kCols = 8 * NT;                                    // token columns
    static constexpr int kXBytes = kGemvUnitGroups * NT * 4 * 32 * 16;      // B fragments of a unit
    static constexpr int kParBytes = kGemvUnitGroups * kGemvRows * 8;       // (s, -(128+z)) per group, row
    static constexpr int kSumBytes = kGemvUnitGroups * 16 * 4;              // X_g per group, token
    static constexpr int kXOff = kGemvStages * kGemvWBytes;
    static constexpr int kParOff = kXOff + kGemvStages * kXBytes;
    static constexpr int kSumOff = kParOff + kGemvStages * kParBytes;
    static constexpr int kPartOff = kSumOff + kGemvStages * kSumBytes;      // [2 halves][128 rows][kCols]
    static constexpr int kBarOff = kPartOff + 2 * kGemvRows * kCols * 4;
    static constexpr int kListOff = kBarOff + (4 * kGemvStages + 2) * 8;    // row blocks this CTA completes
    static constexpr int kBytes = kListOff + 16 * 4;
    static_assert(kBytes <= 227 * 1024, "shared memory of one CTA");
};

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// bf16 pairs (128 + q_lo, 128 + q_hi) of the 4 nibble pairs of a packed word.
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t out[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(out[i]) : "r"(w >> (4 * i)), "r"(0x000F000Fu), "r"(0x43004300u));
}

// Stream-K index arithmetic in 32 bits (T * P < 2^32), which is far cheaper than 64-bit
// division on the GPU.
__device__ __forceinline__ uint32_t unit_begin(uint32_t p, uint32_t T, uint32_t P) { return T * p / P; }

// The CTA whose unit range contains unit u: the largest p with floor(p*T/P) <= u.
__device__ __forceinline__ int cta_of_unit(uint32_t u, uint32_t T, uint32_t P) { return (int)(((u + 1) * P - 1) / T); }

// y[m][n] for every token m of channel row n: v[m] + the CSR term of row n, rounded once.
__device__ __forceinline__ void write_row(const GemvArgs& p, int n, float v[16]) {
    if (p.row_ptr != nullptr) {
        const int j0 = p.row_ptr[n], j1 = p.row_ptr[n + 1];
        if (j0 < 0 || j1 < j0 || (long long)j1 > p.nnz) {
            record_error(p.err, kErrShape);
        } else {
            for (int j = j0; j < j1; ++j) {
                const int c = p.col_idx[j];
                if ((unsigned)c >= (unsigned)p.K) {
                    record_error(p.err, kErrShape);
                    continue;
                }
                const float val = fp16_bits_to_float(p.vals[j]);
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    if (m < p.M) v[m] = fmaf(val, bf16_bits_to_float(p.x[(size_t)m * p.K + c]), v[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < 16; ++m)
        if (m < p.M) p.y[(size_t)m * p.N + n] = float_to_bf16_bits(v[m]);
}

template <int NT>
__global__ void __launch_bounds__(kGemvThreads, 1)
gemv_w4a16_kernel(const __grid_constant__ CUtensorMap map_w, const GemvArgs p) {
    using L = GemvSmem<NT>;
    constexpr int S = kGemvStages;
    constexpr int C = L::kCols;
    // Pointers into shared memory derive from the array itself (no integer round trip), so the
    // compiler keeps the shared address space and issues shared-memory loads and stores.
    extern __shared__ __align__(128) uint8_t smem[];
    if (smem_u32(smem) & 127u) {  // the TMA destinations need 128-byte alignment
        if (threadIdx.x == 0) record_error(p.err, kErrShape);
        return;
    }
    uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* wempty = wfull + S;   // the consumers have read the weights of a stage
    uint64_t* xfull = wempty + S;   // the helpers have filled a stage's activations and parameters
    uint64_t* xempty = xfull + S;   // the consumers are done with them
    uint64_t* pfull = xempty + S;   // the partial tile holds a finished segment
    uint64_t* pempty = pfull + 1;   // the epilogue is done with it
    float* part = reinterpret_cast<float*>(smem + L::kPartOff);
    int* reduce_list = reinterpret_cast<int*>(smem + L::kListOff);  // [0] = count, then row blocks

    const int GB = p.K >> 9;  // units per row block
    const uint32_t u0 = unit_begin(blockIdx.x, p.T, (uint32_t)p.P);
    const int n = (int)(unit_begin(blockIdx.x + 1, p.T, (uint32_t)p.P) - u0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // one barrier per thread, so that the prologue is short
    if (threadIdx.x < 4 * S + 2) {
        const int i = threadIdx.x;
        const uint32_t count = i < S ? 1u : i < 2 * S ? (uint32_t)kGemvConsumers : i < 3 * S ? (uint32_t)kGemvHelpers
                             : i < 4 * S ? (uint32_t)kGemvConsumers : i == 4 * S ? (uint32_t)kGemvConsumers : 1u;
        mbar_init(&wfull[i], count);  // wfull, wempty, xfull, xempty, pfull, pempty are contiguous
        if (i == 0) reduce_list[0] = 0;
        fence_mbarrier_init();
    }
    __syncthreads();

    if (warp == kGemvProducer) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&map_w);
            int issued = 0;
            for (int s = 0; s < n; ++s) {
                const int slot = s % S;
                if (s >= S && !mbar_wait_bounded(&wempty[slot], ((s / S) - 1) & 1)) {
                    record_error(p.err, kErrTimeout);
                    break;
                }
                const uint32_t u = u0 + (uint32_t)s;
                const int rb = (int)(u / (uint32_t)GB), gb = (int)(u - (uint32_t)rb * GB);
                mbar_arrive_expect_tx(&wfull[slot], (uint32_t)kGemvWBytes);
                tma_load_3d(smem + slot * kGemvWBytes, &map_w, &wfull[slot], 0, rb * kGemvRows, gb * kGemvUnitGroups);
                ++issued;
            }
            // the copies this CTA started must land before it may exit
            for (int s = issued > S ? issued - S : 0; s < issued; ++s)
                (void)mbar_wait_bounded(&wfull[s % S], (s / S) & 1);
        }
    } else if (warp >= kGemvHelper0 && warp < kGemvHelper0 + kGemvHelpers) {
        // ------------------------------------------------------------------ helpers
        // Helper h serves groups 2h, 2h+1 of every unit.  Lane (gq, t) loads the B fragments
        // of token tile j: x[8j + gq][k0 + 32t + 8w .. +8] for w = 0..3, and the parameters of
        // rows 4 lane .. 4 lane + 3.
        const int h = warp - kGemvHelper0;
        const int gq = lane >> 2, t = lane & 3;
        const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};  // bf16 1.0 pairs
        for (int s = 0; s < n; ++s) {
            const int slot = s % S;
            const uint32_t u = u0 + (uint32_t)s;
            const int rb = (int)(u / (uint32_t)GB), gb = (int)(u - (uint32_t)rb * GB);
            // global loads first: they do not touch the ring and overlap the wait below.  The
            // scales and zero points do not depend on the previous kernel, so the first unit's
            // are in flight while the helper waits for it; x is loaded after the wait.
            uint4 xv[2][NT][4];
            uint2 scv[2];
            uint32_t zw[2];
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int g = gb * kGemvUnitGroups + 2 * h + gg;
                scv[gg] = __ldg(reinterpret_cast<const uint2*>(p.scales + (size_t)g * p.N + (size_t)rb * kGemvRows) + lane);
                zw[gg] = __ldg(p.zeros + (size_t)g * (p.N >> 3) + (size_t)rb * (kGemvRows / 8) + (lane >> 1));
            }
            if (s == 0) griddep_wait();  // x belongs to the stream order
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int g = gb * kGemvUnitGroups + 2 * h + gg;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    const int m = 8 * j + gq;
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        xv[gg][j][w] = m < p.M ? ldg_cached(p.x + (size_t)m * p.K + ((size_t)g << 7) + 32 * t + 8 * w)
                                               : make_uint4(0u, 0u, 0u, 0u);
                }
            }
            if (s >= S && !__all_sync(0xffffffffu, mbar_wait_bounded(&xempty[slot], ((s / S) - 1) & 1))) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            uint8_t* xs = smem + L::kXOff + slot * L::kXBytes;
            float4* par = reinterpret_cast<float4*>(smem + L::kParOff + slot * L::kParBytes);
            float* sum = reinterpret_cast<float*>(smem + L::kSumOff + slot * L::kSumBytes);
#pragma unroll
            for (int gg = 0; gg < 2; ++gg)
#pragma unroll
                for (int j = 0; j < NT; ++j)
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        *reinterpret_cast<uint4*>(xs + (((((2 * h + gg) * NT + j) * 4 + w) * 32) + lane) * 16) =
                            xv[gg][j][w];
            // X_g of tokens 8j + 2t, 8j + 2t + 1: column sums of B against all-ones rows, in
            // 4 NT independent chains of 4 MMAs
            float dx[2][NT][2][4];
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int gg = 0; gg < 2; ++gg)
#pragma unroll
                    for (int j = 0; j < NT; ++j)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t B[2] = {u4_get(xv[gg][j][w], 2 * hh), u4_get(xv[gg][j][w], 2 * hh + 1)};
                            if (w == 0)
                                mma_16816_bf16_zero_nv(dx[gg][j][hh], ones, B);
                            else
                                mma_16816_bf16_nv(dx[gg][j][hh], ones, B);
                        }
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int gp = 2 * h + gg;  // group within the unit
#pragma unroll
                for (int j = 0; j < NT; ++j)
                    if (gq == 0)
                        *reinterpret_cast<float2*>(&sum[gp * 16 + 8 * j + 2 * t]) =
                            make_float2(dx[gg][j][0][0] + dx[gg][j][1][0], dx[gg][j][0][1] + dx[gg][j][1][1]);
                // rows 4 lane + i: scale bits in scv, zero point in nibble (4 lane + i) % 8 of zw
                const uint32_t zsh = 16u * (lane & 1);
                float sv[4], bv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t bits = (i < 2 ? scv[gg].x : scv[gg].y) >> (16 * (i & 1));
                    sv[i] = fp16_bits_to_float((uint16_t)(bits & 0xFFFFu));
                    bv[i] = -(float)(128u + ((zw[gg] >> (zsh + 4 * i)) & 15u));
                }
                par[gp * (kGemvRows / 2) + 2 * lane] = make_float4(sv[0], bv[0], sv[1], bv[1]);
                par[gp * (kGemvRows / 2) + 2 * lane + 1] = make_float4(sv[2], bv[2], sv[3], bv[3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&xfull[slot]);
        }
    } else if (warp < kGemvConsumers) {
        // ------------------------------------------------------------------ consumers
        const int gq = lane >> 2, t = lane & 3;
        const int half = warp >> 2;                  // groups 2 half, 2 half + 1 of each unit
        const int rbase = 32 * (warp & 3) + gq;      // rows rbase + 16 i + 8 hh
        int seg = 0;
        float acc[2][NT][4];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.0f;

        int rb = (int)(u0 / (uint32_t)GB), gb = (int)(u0 - (uint32_t)rb * GB);  // coordinates of unit u0 + s
        for (int s = 0; s < n; ++s, (gb + 1 == GB ? (gb = 0, ++rb) : ++gb)) {
            const int slot = s % S;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&wfull[slot], (s / S) & 1))) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            const uint8_t* ws = smem + slot * kGemvWBytes;
            uint4 wv[2][2][2];  // [group][tile i][row half hh]
#pragma unroll
            for (int gg = 0; gg < 2; ++gg)
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        wv[gg][i][hh] = *reinterpret_cast<const uint4*>(
                            ws + (2 * half + gg) * kGemvGroupBytes + (rbase + 16 * i + 8 * hh) * 64 + 16 * t);
            __syncwarp();
            if (lane == 0) mbar_arrive(&wempty[slot]);
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&xfull[slot], (s / S) & 1))) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            const uint8_t* xs = smem + L::kXOff + slot * L::kXBytes;
            const float2* par = reinterpret_cast<const float2*>(smem + L::kParOff + slot * L::kParBytes);
            const float* sum = reinterpret_cast<const float*>(smem + L::kSumOff + slot * L::kSumBytes);
            // GI groups at a time: both for M <= 8 (4 independent MMA chains per warp), one for
            // M > 8 (already 4 chains: 2 tiles x 2 token tiles), which keeps the registers in bounds
            constexpr int GI = NT == 1 ? 2 : 1;
#pragma unroll
            for (int pass = 0; pass < 2 / GI; ++pass) {
                uint4 xv[GI][NT][4];
#pragma unroll
                for (int g2 = 0; g2 < GI; ++g2)
#pragma unroll
                    for (int j = 0; j < NT; ++j)
#pragma unroll
                        for (int w = 0; w < 4; ++w)
                            xv[g2][j][w] = *reinterpret_cast<const uint4*>(
                                xs + (((((2 * half + pass * GI + g2) * NT + j) * 4 + w) * 32) + lane) * 16);
                float d[GI][2][NT][4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
#pragma unroll
                    for (int g2 = 0; g2 < GI; ++g2) {
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            uint32_t pa0[4], pa1[4];
                            unpack_word(u4_get(wv[pass * GI + g2][i][0], w), pa0);
                            unpack_word(u4_get(wv[pass * GI + g2][i][1], w), pa1);
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                const uint32_t A[4] = {pa0[2 * hh], pa1[2 * hh], pa0[2 * hh + 1], pa1[2 * hh + 1]};
#pragma unroll
                                for (int j = 0; j < NT; ++j) {
                                    const uint32_t B[2] = {u4_get(xv[g2][j][w], 2 * hh), u4_get(xv[g2][j][w], 2 * hh + 1)};
                                    if (w == 0 && hh == 0)
                                        mma_16816_bf16_zero_nv(d[g2][i][j], A, B);
                                    else
                                        mma_16816_bf16_nv(d[g2][i][j], A, B);
                                }
                            }
                        }
                    }
                }
                // the group's zero point and scale, applied in fp32: acc += s (d - (128 + z) X_g)
#pragma unroll
                for (int g2 = 0; g2 < GI; ++g2) {
                    const int gp = 2 * half + pass * GI + g2;
                    float2 sp[4];  // rows rbase + 8k, k = 2i + hh
#pragma unroll
                    for (int k = 0; k < 4; ++k) sp[k] = par[gp * kGemvRows + rbase + 8 * k];
                    float2 X[NT];
#pragma unroll
                    for (int j = 0; j < NT; ++j) X[j] = *reinterpret_cast<const float2*>(&sum[gp * 16 + 8 * j + 2 * t]);
#pragma unroll
                    for (int i = 0; i < 2; ++i)
#pragma unroll
                        for (int j = 0; j < NT; ++j) {
                            const float2 a = sp[2 * i], b = sp[2 * i + 1];
                            acc[i][j][0] = fmaf(a.x, fmaf(a.y, X[j].x, d[g2][i][j][0]), acc[i][j][0]);
                            acc[i][j][1] = fmaf(a.x, fmaf(a.y, X[j].y, d[g2][i][j][1]), acc[i][j][1]);
                            acc[i][j][2] = fmaf(b.x, fmaf(b.y, X[j].x, d[g2][i][j][2]), acc[i][j][2]);
                            acc[i][j][3] = fmaf(b.x, fmaf(b.y, X[j].y, d[g2][i][j][3]), acc[i][j][3]);
                        }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&xempty[slot]);

            if (gb == GB - 1 || s == n - 1) {
                // ---------------------------------------------------------- segment end
                if (seg > 0 && !__all_sync(0xffffffffu, mbar_wait_bounded(pempty, (seg - 1) & 1))) {
                    if (lane == 0) record_error(p.err, kErrTimeout);
                    break;
                }
                float* pt = part + half * (kGemvRows * C);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int c0 = rbase + 16 * i, c1 = c0 + 8;
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        const int tk = 8 * j + 2 * t;
                        *reinterpret_cast<float2*>(&pt[c0 * C + tk]) = make_float2(acc[i][j][0], acc[i][j][1]);
                        *reinterpret_cast<float2*>(&pt[c1 * C + tk]) = make_float2(acc[i][j][2], acc[i][j][3]);
                        acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.0f;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(pfull);
                ++seg;
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue warp
        // Walks the same segments as the consumers.  Lane l owns rows l, l+32, l+64, l+96.
        bool waited = false;
        int seg = 0;
        uint32_t seg_first = u0;  // first unit of the current segment
        for (int s = 0; s < n; ++s) {
            const uint32_t u = u0 + (uint32_t)s;
            const int rb = (int)(u / (uint32_t)GB), gb = (int)(u - (uint32_t)rb * GB);
            if (!(gb == GB - 1 || s == n - 1)) continue;
            const bool whole = seg_first == (uint32_t)rb * GB && gb == GB - 1;
            seg_first = u + 1;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(pfull, seg & 1))) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            if (!waited) {
                griddep_wait();  // the workspace, x and y belong to the stream order
                waited = true;
            }
            const float* p0 = part;
            const float* p1 = part + kGemvRows * C;
            if (whole) {
                for (int r = lane; r < kGemvRows; r += 32) {
                    float v[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[c] = 0.0f;
#pragma unroll
                    for (int c = 0; c < C; c += 4) {
                        const float4 a = *reinterpret_cast<const float4*>(&p0[r * C + c]);
                        const float4 b = *reinterpret_cast<const float4*>(&p1[r * C + c]);
                        v[c] = a.x + b.x;
                        v[c + 1] = a.y + b.y;
                        v[c + 2] = a.z + b.z;
                        v[c + 3] = a.w + b.w;
                    }
                    write_row(p, rb * kGemvRows + r, v);
                }
            } else {
                const int pf = cta_of_unit((uint32_t)rb * GB, p.T, (uint32_t)p.P);
                const int pl = cta_of_unit((uint32_t)rb * GB + GB - 1, p.T, (uint32_t)p.P);
                const int mine = 2 * (int)blockIdx.x + (u0 >= (uint32_t)rb * GB ? 0 : 1);
                float4* dst = reinterpret_cast<float4*>(p.partials + (size_t)mine * kGemvSlotFloats);
                const float4* a4 = reinterpret_cast<const float4*>(p0);
                const float4* b4 = reinterpret_cast<const float4*>(p1);
                for (int q = lane; q < kGemvRows * C / 4; q += 32) {
                    const float4 a = a4[q], b = b4[q];
                    __stcg(dst + q, make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w));
                }
                // release the partial tile to the completing CTA: the warp's stores, then the
                // counter increment by lane 0 with acquire-release semantics at GPU scope.  It
                // orders the warp's stores (which __syncwarp orders before it) ahead of the
                // increment, and in the CTA that completes the count it acquires every earlier
                // contributor's partial; the barrier of the completion phase passes that on.
                __syncwarp();
                unsigned old = 0;
                if (lane == 0) old = atomic_add_acq_rel_gpu(p.counters + rb, 1u);
                old = __shfl_sync(0xffffffffu, old, 0);
                // the CTA that completes the row block sums its partials after the stream ends
                if (lane == 0 && old == (unsigned)(pl - pf) && reduce_list[0] < 15)
                    reduce_list[1 + reduce_list[0]++] = rb;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(pempty);
            ++seg;
        }
    }
    griddep_launch_dependents();

    // ---------------------------------------------------------------------- completions
    // The consumer warps and the epilogue warp sum the partial tiles of the row blocks this
    // CTA completed: thread r (< 128) owns row r, loads of several slots are in flight at once.
    if (warp < kGemvConsumers || warp == kGemvEpilogue) {
        asm volatile("bar.sync 2, %0;" ::"r"(32 * (kGemvConsumers + 1)) : "memory");
        const int count = reduce_list[0];
        const int r = threadIdx.x < kGemvRows ? (int)threadIdx.x : -1;
        if (count > 0) {
            griddep_wait();
            fence_acq_rel_gpu();  // acquire: every other contributor's partial is visible
        }
        for (int e = 0; e < count && r >= 0; ++e) {
            const int rb = reduce_list[1 + e];
            const int pf = cta_of_unit((uint32_t)rb * GB, p.T, (uint32_t)p.P);
            const int pl = cta_of_unit((uint32_t)rb * GB + GB - 1, p.T, (uint32_t)p.P);
            const bool first_starts_here = unit_begin((uint32_t)pf, p.T, (uint32_t)p.P) == (uint32_t)rb * GB;
            float v[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) v[m] = 0.0f;
            constexpr int QB = NT == 1 ? 8 : 4;  // contributors whose loads are in flight together
            for (int q0 = pf; q0 <= pl; q0 += QB) {
                float4 a[QB][C / 4];
#pragma unroll
                for (int qq = 0; qq < QB; ++qq) {
                    const int q = q0 + qq;
                    if (q <= pl) {
                        // a contributor after the first starts inside the row block, so the row
                        // block is its first segment; the first one may have started before it
                        const int slotq = 2 * q + (q == pf && !first_starts_here ? 1 : 0);
                        const float4* sp =
                            reinterpret_cast<const float4*>(p.partials + (size_t)slotq * kGemvSlotFloats + r * C);
#pragma unroll
                        for (int c = 0; c < C / 4; ++c) a[qq][c] = __ldcg(sp + c);
                    }
                }
#pragma unroll
                for (int qq = 0; qq < QB; ++qq) {
                    if (q0 + qq <= pl) {
#pragma unroll
                        for (int c = 0; c < C / 4; ++c) {
                            v[4 * c] += a[qq][c].x;
                            v[4 * c + 1] += a[qq][c].y;
                            v[4 * c + 2] += a[qq][c].z;
                            v[4 * c + 3] += a[qq][c].w;
                        }
                    }
                }
            }
            write_row(p, rb * kGemvRows + r, v);
        }
        asm volatile("bar.sync 2, %0;" ::"r"(32 * (kGemvConsumers + 1)) : "memory");
        if (threadIdx.x == 0)
            for (int e = 0; e < count; ++e) atomicExch(p.counters + reduce_list[1 + e], 0u);
    }
}

int gemv_max_k() { return 1 << 20; }

int gemv_ctas(int N, int K, int num_sms) {
    const long long T = (long long)(N / kGemvRows) * (K / (128 * kGemvUnitGroups));
    return (int)(T < num_sms ? T : num_sms);
}

bool gemv_fits(int N, int K, int num_sms) {
    const unsigned long long T = (unsigned long long)(N / kGemvRows) * (K / (128 * kGemvUnitGroups));
    return T * (unsigned long long)gemv_ctas(N, K, num_sms) < (1ull << 32);
}

size_t gemv_workspace_bytes(int N, int num_sms) {
    const size_t partials = (size_t)2 * num_sms * kGemvSlotFloats * sizeof(float);
    const size_t counters = (size_t)(N / kGemvRows) * sizeof(unsigned);
    return partials + ((counters + 255) / 256) * 256;
}

cudaError_t launch_gemv(const GemvMaps& maps, const uint16_t* x, const uint16_t* scales, const uint32_t* zeros,
                        const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* vals, long long nnz,
                        uint16_t* y, void* workspace, int M, int N, int K, int num_sms, unsigned* err,
                        cudaStream_t stream) {
    GemvArgs a{};
    a.x = x;
    a.scales = scales;
    a.zeros = zeros;
    a.row_ptr = row_ptr;
    a.col_idx = col_idx;
    a.vals = vals;
    a.nnz = nnz;
    a.y = y;
    a.M = M;
    a.N = N;
    a.K = K;
    a.T = (uint32_t)((N / kGemvRows) * (K / (128 * kGemvUnitGroups)));
    a.P = gemv_ctas(N, K, num_sms);
    a.err = err;
    const size_t partial_bytes = (size_t)2 * num_sms * kGemvSlotFloats * sizeof(float);
    a.partials = static_cast<float*>(workspace);
    a.counters = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(workspace) + partial_bytes);

    const bool two = M > 8;
    const int smem = two ? GemvSmem<2>::kBytes : GemvSmem<1>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(two ? gemv_w4a16_kernel<2> : gemv_w4a16_kernel<1>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.P, 1, 1);
    cfg.blockDim = dim3(kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (two) return cudaLaunchKernelEx(&cfg, gemv_w4a16_kernel<2>, maps.w, a);
    return cudaLaunchKernelEx(&cfg, gemv_w4a16_kernel<1>, maps.w, a);
}

}  // namespace w4a16
