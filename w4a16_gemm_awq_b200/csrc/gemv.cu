// gemv.cu -- decode W4A16 GEMV (1 <= M <= 16): y = bf16(x . dequant(Q)^T [+ x . W_sparse^T]).
//
// [AWQ (MLSys 2024) translation, section 1: TinyChat computes the linear layer from packed
//  4-bit weights dequantized on the fly; at decode batch sizes the layer is bound by memory
//  bandwidth (section 2: weight-only quantization relieves the memory bottleneck).
//  SqueezeLLM article, section 2.3: the fp16 sparse term is added to the dense product.]
//
// Design (B200).  Each packed weight byte is streamed once from HBM by a grid of at most one
// CTA per SM.
//   - Work units are (128-channel row block, 4 slices of 128 k = 512 k): 32 KB of packed
//     weights, brought in by ONE TMA copy.  A slice is a quantization group for g128; with
//     larger groups, consecutive slices share their group's scale and zero point.  A CTA's
//     TMA copies are served nearly one after another, so the bytes per copy set the
//     streaming rate of a CTA: 8 KB copies stream at ~16 GB/s per CTA, 32 KB copies at
//     ~40 GB/s, enough for one CTA per SM to saturate HBM.  The copy uses a 3-D view of
//     qweight (16 words of a group, rows, groups; strides K/2 and 64 bytes), so it lands as
//     [4 groups][128 rows][64 bytes] and the consumers' 128-bit loads of one group are free
//     of bank conflicts.
//   - Stream-K: CTA p takes the contiguous unit range [p*T/P, (p+1)*T/P), ordered row block
//     by row block, so every CTA streams the same number of bytes in one balanced wave.  A
//     row block processed whole by one CTA is written straight to y.  A row block split
//     between CTAs leaves fp32 partial tiles in the caller's workspace.  Each contributing
//     CTA then increments the row block's counter.  The CTA that completes the count sums
//     the partials once its own stream has ended, writes y and resets the counter to zero.
//     No CTA waits for another, and the workspace is all-zero again after every call.
//   - Warps: 8 consumers, 4 helpers, 1 TMA producer (weights), 1 epilogue.  Everything
//     except the weights comes in through the helpers with ordinary loads, so the weights
//     are the only TMA traffic.  Warp w runs on SM sub-partition w % 4: the consumers take
//     two warps of each, the helpers (warps 8..11) one each, so the staging work is spread
//     evenly (with two helpers it sat on two sub-partitions, measured 4-13% slower).  For
//     its group of each unit a helper
//       * copies the activations from global memory (L2-resident) into shared memory,
//         already in the order of the MMA B fragments;
//       * computes the group sums X_g of every token with tensor-core MMAs against an
//         all-ones A operand;
//       * decodes the scales and zero points of the unit's 128 rows into fp32 pairs
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
//     shared-memory partial tile (warps 0-3 write it, warps 4-7 add theirs) and go on
//     streaming; the epilogue warp does the exchange between CTAs, the CSR term and the
//     stores of y.
//   - Two schedules share everything above and differ in how units map to CTAs:
//       * stream-K (above): completes split row blocks through the workspace.  A CTA's
//         last row block is usually shared with the next CTA, which took it first; its
//         partial tile is then fetched while this CTA still computes, and the row block is
//         completed without a counter increment.
//       * cluster split-K: for shapes with few row blocks, thread-block clusters of 2..8
//         CTAs take whole row blocks, each CTA an equal share of its 512-k units; the
//         cluster sums its tiles through distributed shared memory, with no workspace
//         traffic and no CTA waiting on a global counter.
//   - Programmatic dependent launch.  The weights may be fetched before the previous kernel
//     on the stream has finished.  The helpers wait for it before they load x; the
//     epilogue and the completion phase wait before they touch the workspace or y.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kGemvRows = 128;                                  // output channels per row block
constexpr int kGemvUnitGroups = 4;                              // groups of 128 k per work unit
// Packed weights of a unit in shared memory, [4 groups][128 rows][row bytes]: 64 bytes a row
// and group for 4-bit codes (32 KB a unit), 48 for 3-bit codes (24 KB).
template <int BITS>
struct GemvW {
    static_assert(BITS == 4 || BITS == 3, "4- or 3-bit codes");
    static constexpr int kRowBytes = 16 * BITS;
    static constexpr int kGroupBytes = kGemvRows * kRowBytes;
    static constexpr int kWBytes = kGemvUnitGroups * kGroupBytes;
};
constexpr int kGemvConsumers = 8;                               // warps 0..7
constexpr int kGemvProducer = 12;                               // warp 12
constexpr int kGemvHelper0 = 8;                                 // warps 8..11, one per SMSP
constexpr int kGemvHelpers = 4;
constexpr int kGemvEpilogue = 13;                               // warp 13
constexpr int kGemvThreads = 32 * 14;
constexpr int kGemvHG = kGemvUnitGroups / kGemvHelpers;         // groups per helper and unit
constexpr int kGemvStages = 4;

struct GemvArgs {
    const uint16_t* x;
    const uint16_t* scales;
    const uint32_t* zeros;
    const float* ysp;    // nullptr, or the CSR term [N][M] fp32 (csr_rows_kernel, the previous kernel)
    uint16_t* y;
    float* partials;     // workspace: [2P][128][16] fp32 (stream-K)
    unsigned* counters;  // workspace: [N/128], zero between calls (stream-K)
    int M, N, K;
    uint32_t T;          // work units = (N/128) * (K/512); T * P < 2^32 (checked by the caller)
    int P;               // CTAs
    int gr;              // quantization group size / 128: scales and zeros of 128-slice g are those of group g / gr
    int cl;              // 0: stream-K; else the cluster size of the cluster split-K (2..8, <= K/512)
    int ncl;             // cluster split-K: clusters (<= N/128); cluster j takes row blocks j, j + ncl, ...
    unsigned* err;
};

template <int NT, int BITS = 4>
struct GemvSmem {
    static constexpr int kCols = 8 * NT;                                    // token columns
    static constexpr int kXBytes = kGemvUnitGroups * NT * 4 * 32 * 16;      // B fragments of a unit
    static constexpr int kParBytes = kGemvUnitGroups * kGemvRows * 8;       // (s, -(128+z)) per group, row
    static constexpr int kSumBytes = kGemvUnitGroups * 16 * 4;              // X_g per group, token
    static constexpr int kXOff = kGemvStages * GemvW<BITS>::kWBytes;
    static constexpr int kParOff = kXOff + kGemvStages * kXBytes;
    static constexpr int kSumOff = kParOff + kGemvStages * kParBytes;
    static constexpr int kPartOff = kSumOff + kGemvStages * kSumBytes;      // [128 rows][kCols]
    static constexpr int kRecvOff = kPartOff + kGemvRows * kCols * 4;       // cluster split-K: rows received
    static constexpr int kBarOff = kRecvOff + kGemvRows * kCols * 4;
    static constexpr int kListOff = kBarOff + (4 * kGemvStages + 5) * 8;    // row blocks this CTA completes
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

// The bf16 pairs of "word" w (0..3) of a thread's 32 codes: for 4-bit codes v holds the 4
// packed words.  For 3-bit codes v holds the 3 words of the 32 codes: pairs of words 0..2 are
// their nibbles' low 3 bits, and "word" 3 gathers the bit-3 planes: bit 4i + 3 of word b is
// bit b of the codes of nibbles i and i + 4 of the fourth 8-code block.
template <int BITS>
__device__ __forceinline__ void unpack_codes(const uint4& v, int w, uint32_t out[4]) {
    if constexpr (BITS == 4) {
        unpack_word(u4_get(v, w), out);
    } else if (w < 3) {
        const uint32_t word = u4_get(v, w);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(out[i]) : "r"(word >> (4 * i)), "r"(0x00070007u),
                "r"(0x43004300u));
    } else {
        // gather the three bit-3 planes into one word whose nibble j is the code of element
        // 24 + ORDER[j], then unpack it like a 4-bit word: 6 operations for the planes and 2
        // per pair, instead of 7 per pair
        uint32_t p;
        asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(p) : "r"(v.x >> 3), "r"(0x11111111u),
            "r"((v.y >> 2) & 0x22222222u));
        asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(p) : "r"(v.z >> 1), "r"(0x44444444u), "r"(p));
        unpack_word(p, out);
    }
}

// Next unit of a CTA's walk: gb runs over [kb, ke) within a row block, then the walk moves
// `step` row blocks on.
__device__ __forceinline__ void walk_next(int& rb, int& gb, int kb, int ke, int step) {
    if (++gb == ke) {
        gb = kb;
        rb += step;
    }
}

// Stream-K index arithmetic in 32 bits (T * P < 2^32), which is far cheaper than 64-bit
// division on the GPU.
__device__ __forceinline__ uint32_t unit_begin(uint32_t p, uint32_t T, uint32_t P) { return T * p / P; }

// The CTA whose unit range contains unit u: the largest p with floor(p*T/P) <= u.
__device__ __forceinline__ int cta_of_unit(uint32_t u, uint32_t T, uint32_t P) { return (int)(((u + 1) * P - 1) / T); }

// y[m][n] for every token m of channel row n: v[m] + the CSR term of row n (computed by
// csr_rows_kernel into ysp[n][m] before this kernel reads it), rounded once.
__device__ __forceinline__ void write_row(const GemvArgs& p, int n, const float v[16]) {
    if (p.ysp != nullptr) {
        const float* sp = p.ysp + (size_t)n * p.M;
#pragma unroll
        for (int m = 0; m < 16; ++m)
            if (m < p.M) p.y[(size_t)m * p.N + n] = float_to_bf16_bits(v[m] + __ldcg(sp + m));
        return;
    }
#pragma unroll
    for (int m = 0; m < 16; ++m)
        if (m < p.M) p.y[(size_t)m * p.N + n] = float_to_bf16_bits(v[m]);
}

// Row block rb split between exactly two CTAs: when the other one has published its partial
// tile (the counter, read with acquire semantics, is 1), loads that tile's rows lane + 32 i
// into t[i] and returns true.  The calling CTA is then the row block's last contributor and
// completes it itself.  It adds (0 + own) + other; the completion phase adds the two tiles
// the same way in contributor order, and since fp32 addition is commutative the two give
// the same bits, so y does not depend on which CTA finishes last.
// Returns false otherwise (t undefined).  All lanes of the warp take part.
template <int C>
__device__ __forceinline__ bool gather_other(const GemvArgs& p, int rb, int GB, int lane, float t[4][C]) {
    const uint32_t rb0 = (uint32_t)rb * GB;
    const int pf = cta_of_unit(rb0, p.T, (uint32_t)p.P);
    const int pl = cta_of_unit(rb0 + GB - 1, p.T, (uint32_t)p.P);
    if (pl - pf != 1) return false;
    if (!__all_sync(0xffffffffu, ld_acquire_gpu(p.counters + rb) == 1u)) return false;
    const int q = pf == (int)blockIdx.x ? pl : pf;
    // the second contributor starts inside the row block, so the row block is its first
    // segment; the first one may have started before it
    const bool first_starts_here = unit_begin((uint32_t)pf, p.T, (uint32_t)p.P) == rb0;
    const int slot = 2 * q + (q == pf && !first_starts_here ? 1 : 0);
    const float4* sp = reinterpret_cast<const float4*>(p.partials + (size_t)slot * kGemvSlotFloats);
    float4 a[4][C / 4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < C / 4; ++c) a[i][c] = __ldcg(sp + (lane + 32 * i) * (C / 4) + c);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < C / 4; ++c) {
            t[i][4 * c] = a[i][c].x;
            t[i][4 * c + 1] = a[i][c].y;
            t[i][4 * c + 2] = a[i][c].z;
            t[i][4 * c + 3] = a[i][c].w;
        }
    return true;
}

template <int NT, int BITS>
__global__ void __launch_bounds__(kGemvThreads, 1)
gemv_w4a16_kernel(const __grid_constant__ CUtensorMap map_w, const GemvArgs p) {
    using L = GemvSmem<NT, BITS>;
    constexpr int kWBytes = GemvW<BITS>::kWBytes;
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
    uint64_t* cready = pempty + 1;  // cluster split-K: the rows the other CTAs send have landed
    uint64_t* cdone = cready + 1;   // cluster split-K: the other CTAs have summed what this one sent
    uint64_t* phalf = cdone + 1;    // consumer warps 0-3 have written their part of the tile
    float* part = reinterpret_cast<float*>(smem + L::kPartOff);
    int* reduce_list = reinterpret_cast<int*>(smem + L::kListOff);  // [0] = count, then row blocks

    // The CTA's work: n units, walked row block by row block.  Within a row block the unit
    // index gb runs over [kb, ke); then the walk moves `step` row blocks on.
    const int GB = p.K >> 9;  // units per row block
    uint32_t u0 = 0;          // stream-K: first unit
    int n, rb_first, gb_first, kb, ke, step;
    uint32_t crank = 0;       // cluster split-K: rank in the cluster
    if (p.cl == 0) {
        u0 = unit_begin(blockIdx.x, p.T, (uint32_t)p.P);
        n = (int)(unit_begin(blockIdx.x + 1, p.T, (uint32_t)p.P) - u0);
        rb_first = (int)(u0 / (uint32_t)GB);
        gb_first = (int)(u0 - (uint32_t)rb_first * GB);
        kb = 0;
        ke = GB;
        step = 1;
    } else {
        // rank r of cluster j takes units [r GB / cl, (r+1) GB / cl) of row blocks j, j + ncl, ...
        crank = cluster_ctarank();
        const int j = (int)cluster_id_x();
        kb = (int)crank * GB / p.cl;
        ke = ((int)crank + 1) * GB / p.cl;
        rb_first = j;
        gb_first = kb;
        step = p.ncl;
        n = ((p.N / kGemvRows - 1 - j) / p.ncl + 1) * (ke - kb);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // The producer thread initialises the weight ring's full barriers itself and starts its
    // first copies before the CTA-wide barrier: the first weights are what a call waits for
    // first.  The copies touch nothing of the previous kernel on the stream.
    int pre = 0;                       // copies issued here (producer thread only)
    int prb = rb_first, pgb = gb_first;  // coordinates of the producer's next copy
    if (threadIdx.x == kGemvProducer * 32) {
        prefetch_tensormap(&map_w);
        for (int i = 0; i < S; ++i) mbar_init(&wfull[i], 1u);
        fence_mbarrier_init();
        fence_proxy_async_smem();
        for (; pre < S && pre < n; ++pre, walk_next(prb, pgb, kb, ke, step)) {
            mbar_arrive_expect_tx(&wfull[pre], (uint32_t)kWBytes);
            tma_load_3d(smem + pre * kWBytes, &map_w, &wfull[pre], 0, prb * kGemvRows, pgb * kGemvUnitGroups);
        }
    }
    // the other barriers, one per thread, so that the prologue is short
    if (threadIdx.x >= S && threadIdx.x < 4 * S + 5) {
        const int i = threadIdx.x;
        const uint32_t peers = p.cl > 1 ? 32u * (uint32_t)(p.cl - 1) : 1u;  // every epilogue lane of every other CTA
        const uint32_t count = i < S ? 1u : i < 2 * S ? (uint32_t)kGemvConsumers : i < 3 * S ? (uint32_t)kGemvHelpers
                             : i < 4 * S ? (uint32_t)kGemvConsumers : i == 4 * S ? (uint32_t)kGemvConsumers
                             : i == 4 * S + 3 ? peers : i == 4 * S + 4 ? (uint32_t)(kGemvConsumers / 2) : 1u;
        mbar_init(&wfull[i], count);  // the ring, pfull, pempty, cready, cdone and phalf are contiguous
        if (i == S) reduce_list[0] = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    // The other CTAs of the cluster arrive on cready and cdone, so those must be initialised
    // first: every thread arrives on the cluster barrier here, and the epilogue warp waits on
    // it before its first remote arrival.  The other roles start at once.
    if (p.cl != 0) cluster_arrive_relaxed();
    // The next kernel on the stream may be scheduled once every CTA of this grid is running:
    // its CTAs then take SMs as this grid's CTAs leave them and fetch their weights, while
    // everything it reads or writes of ours waits for this grid to complete.
    griddep_launch_dependents();

    if (warp == kGemvProducer) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = pre;
            for (int s = pre; s < n; ++s, walk_next(prb, pgb, kb, ke, step)) {
                const int slot = s % S;
                if (s >= S && !mbar_wait_bounded(&wempty[slot], ((s / S) - 1) & 1)) {
                    record_error(p.err, kErrTimeout);
                    break;
                }
                mbar_arrive_expect_tx(&wfull[slot], (uint32_t)kWBytes);
                tma_load_3d(smem + slot * kWBytes, &map_w, &wfull[slot], 0, prb * kGemvRows, pgb * kGemvUnitGroups);
                ++issued;
            }
            // the copies this CTA started must land before it may exit
            for (int s = issued > S ? issued - S : 0; s < issued; ++s)
                (void)mbar_wait_bounded(&wfull[s % S], (s / S) & 1);
        }
    } else if (warp >= kGemvHelper0 && warp < kGemvHelper0 + kGemvHelpers) {
        // ------------------------------------------------------------------ helpers
        // Helper h serves group h of every unit.  Lane (gq, t) loads the B fragments
        // of token tile j: x[8j + gq][k0 + 32t + 8w .. +8] for w = 0..3, and the parameters of
        // rows 4 lane .. 4 lane + 3.
        const int h = warp - kGemvHelper0;
        const int gq = lane >> 2, t = lane & 3;
        const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};  // bf16 1.0 pairs
        int rb = rb_first, gb = gb_first;
        for (int s = 0; s < n; ++s, walk_next(rb, gb, kb, ke, step)) {
            const int slot = s % S;
            // global loads first: they do not touch the ring and overlap the wait below.  The
            // scales and zero points do not depend on the previous kernel, so the first unit's
            // are in flight while the helper waits for it; x is loaded after the wait.
            uint4 xv[kGemvHG][NT][4];
            uint2 scv[kGemvHG];
            uint32_t zw[kGemvHG];
#pragma unroll
            for (int gg = 0; gg < kGemvHG; ++gg) {
                const int g = (gb * kGemvUnitGroups + kGemvHG * h + gg) / p.gr;  // the quantization group
                scv[gg] = __ldg(reinterpret_cast<const uint2*>(p.scales + (size_t)g * p.N + (size_t)rb * kGemvRows) + lane);
                zw[gg] = __ldg(p.zeros + (size_t)g * (p.N >> 3) + (size_t)rb * (kGemvRows / 8) + (lane >> 1));
            }
            if (s == 0) griddep_wait();  // x belongs to the stream order
#pragma unroll
            for (int gg = 0; gg < kGemvHG; ++gg) {
                const int g = gb * kGemvUnitGroups + kGemvHG * h + gg;
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
            for (int gg = 0; gg < kGemvHG; ++gg)
#pragma unroll
                for (int j = 0; j < NT; ++j)
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        *reinterpret_cast<uint4*>(xs + (((((kGemvHG * h + gg) * NT + j) * 4 + w) * 32) + lane) * 16) =
                            xv[gg][j][w];
            // X_g of tokens 8j + 2t, 8j + 2t + 1: column sums of B against all-ones rows, in
            // 4 NT independent chains of 4 MMAs
            float dx[kGemvHG][NT][2][4];
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int gg = 0; gg < kGemvHG; ++gg)
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
            for (int gg = 0; gg < kGemvHG; ++gg) {
                const int gp = kGemvHG * h + gg;  // group within the unit
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

        int rb = rb_first, gb = gb_first;
        for (int s = 0; s < n; ++s, walk_next(rb, gb, kb, ke, step)) {
            const int slot = s % S;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&wfull[slot], (s / S) & 1))) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            const uint8_t* ws = smem + slot * kWBytes;
            uint4 wv[2][2][2];  // [group][tile i][row half hh]
#pragma unroll
            for (int gg = 0; gg < 2; ++gg)
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint8_t* src = ws + (2 * half + gg) * GemvW<BITS>::kGroupBytes +
                                             (rbase + 16 * i + 8 * hh) * GemvW<BITS>::kRowBytes;
                        if constexpr (BITS == 4) {
                            wv[gg][i][hh] = *reinterpret_cast<const uint4*>(src + 16 * t);
                        } else {  // the thread's 3 words of 32 codes
                            const uint32_t* s3 = reinterpret_cast<const uint32_t*>(src + 12 * t);
                            wv[gg][i][hh] = make_uint4(s3[0], s3[1], s3[2], 0u);
                        }
                    }
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
                            unpack_codes<BITS>(wv[pass * GI + g2][i][0], w, pa0);
                            unpack_codes<BITS>(wv[pass * GI + g2][i][1], w, pa1);
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

            if (gb == ke - 1 || s == n - 1) {
                // ---------------------------------------------------------- segment end
                if (seg > 0 && !__all_sync(0xffffffffu, mbar_wait_bounded(pempty, (seg - 1) & 1))) {
                    if (lane == 0) record_error(p.err, kErrTimeout);
                    break;
                }
                // Warps 0-3 (groups 0, 1 of every unit) write the tile; warps 4-7 (groups 2, 3)
                // then add theirs to the same rows and tokens.
                if (half == 1 && !__all_sync(0xffffffffu, mbar_wait_bounded(phalf, seg & 1))) {
                    if (lane == 0) record_error(p.err, kErrTimeout);
                    break;
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int c0 = rbase + 16 * i, c1 = c0 + 8;
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        const int tk = 8 * j + 2 * t;
                        float2* q0 = reinterpret_cast<float2*>(&part[c0 * C + tk]);
                        float2* q1 = reinterpret_cast<float2*>(&part[c1 * C + tk]);
                        if (half == 0) {
                            *q0 = make_float2(acc[i][j][0], acc[i][j][1]);
                            *q1 = make_float2(acc[i][j][2], acc[i][j][3]);
                        } else {
                            const float2 a = *q0, b = *q1;
                            *q0 = make_float2(a.x + acc[i][j][0], a.y + acc[i][j][1]);
                            *q1 = make_float2(b.x + acc[i][j][2], b.y + acc[i][j][3]);
                        }
                        acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.0f;
                    }
                }
                if (p.cl != 0) fence_proxy_async_smem();  // the tile leaves by bulk copy
                __syncwarp();
                if (lane == 0) {
                    if (half == 0) mbar_arrive(phalf);
                    mbar_arrive(pfull);
                }
                ++seg;
            }
        }
    } else if (p.cl != 0) {
        // ------------------------------------------------------------------ epilogue warp,
        // cluster split-K.  Every CTA of the cluster holds a partial tile of the same row
        // block.  Rank r owns rows [128 r / cl, 128 (r+1) / cl): each other CTA sends it
        // those rows of its tile with one bulk copy into r's shared memory, whose bytes
        // complete r's cready barrier; r then sums the cluster's tiles for its rows in rank
        // order and writes them.  With several row blocks per cluster, a CTA sends the next
        // row block's rows only once every receiver has summed the previous ones (cdone).  A
        // failed wait is recorded and the exchange goes on, so that no CTA leaves while data
        // may still arrive for it.
        const int cl = p.cl;
        const int row0 = (int)crank * kGemvRows / cl, row1 = ((int)crank + 1) * kGemvRows / cl;
        const int nrow = row1 - row0;  // at most 64
        const int nseg = n / (ke - kb);
        const float* recv = reinterpret_cast<const float*>(smem + L::kRecvOff);  // [cl - 1][nrow][C]
        float* recv_w = reinterpret_cast<float*>(smem + L::kRecvOff);
        const uint32_t recv_bytes = (uint32_t)((cl - 1) * nrow * C * 4);
        if (lane == 0) mbar_arrive_expect_tx(cready, recv_bytes);
        cluster_wait_acquire();  // every CTA of the cluster has initialised its barriers
        griddep_wait();          // y belongs to the stream order
        int rb = rb_first;
        for (int seg = 0; seg < nseg; ++seg, rb += step) {
            bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(pfull, seg & 1));
            if (seg > 0) ok = __all_sync(0xffffffffu, mbar_wait_cluster_bounded(cdone, (seg - 1) & 1)) && ok;
            if (lane == 0) {
                for (int r = 0; r < cl; ++r) {
                    if (r == (int)crank) continue;
                    const int r0 = r * kGemvRows / cl, nr = (r + 1) * kGemvRows / cl - r0;
                    const int slot = (int)crank < r ? (int)crank : (int)crank - 1;  // this CTA's slot at rank r
                    bulk_copy_to_cluster(cluster_map(recv_w + slot * nr * C, (uint32_t)r), part + r0 * C,
                                         (uint32_t)(nr * C * 4), cluster_map(cready, (uint32_t)r));
                }
                bulk_commit_group();
            }
            float own[2][C];  // rows row0 + lane + 32 i of this CTA's tile
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int r = row0 + lane + 32 * i;
#pragma unroll
                for (int c = 0; c < C; ++c) own[i][c] = r < row1 ? part[r * C + c] : 0.0f;
            }
            if (lane == 0) bulk_wait_read_all();  // the copies have read the tile
            __syncwarp();
            if (lane == 0) mbar_arrive(pempty);  // the consumers may overwrite the tile
            ok = __all_sync(0xffffffffu, mbar_wait_cluster_bounded(cready, seg & 1)) && ok;
            float v[2][16];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int c = 0; c < 16; ++c) v[i][c] = 0.0f;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int r = row0 + lane + 32 * i;
                if (r < row1) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (q >= cl) continue;
                        if (q == (int)crank) {
#pragma unroll
                            for (int c = 0; c < C; ++c) v[i][c] += own[i][c];
                        } else {
                            const float4* t = reinterpret_cast<const float4*>(
                                recv + ((q < (int)crank ? q : q - 1) * nrow + (r - row0)) * C);
#pragma unroll
                            for (int c = 0; c < C / 4; ++c) {
                                const float4 a = t[c];
                                v[i][4 * c] += a.x;
                                v[i][4 * c + 1] += a.y;
                                v[i][4 * c + 2] += a.z;
                                v[i][4 * c + 3] += a.w;
                            }
                        }
                    }
                }
            }
            if (seg + 1 < nseg) {
                // ready for the next row block's rows; tell every sender its rows were summed
                if (lane == 0) mbar_arrive_expect_tx(cready, recv_bytes);
                for (int q = 0; q < cl; ++q)
                    if (q != (int)crank) mbar_arrive_cluster(cluster_map(cdone, (uint32_t)q));
            }
            if (ok) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int r = row0 + lane + 32 * i;
                    if (r < row1) write_row(p, rb * kGemvRows + r, v[i]);
                }
            } else if (lane == 0) {
                record_error(p.err, kErrTimeout);
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue warp,
        // stream-K.  Walks the same segments as the consumers.  Lane l owns rows l, l+32,
        // l+64, l+96.
        bool waited = false;
        int seg = 0;
        const uint32_t u_end = u0 + (uint32_t)n;
        for (uint32_t first = u0; first < u_end; ++seg) {
            const int rb = (int)(first / (uint32_t)GB);
            const uint32_t rb0 = (uint32_t)rb * GB;
            const uint32_t end = rb0 + GB < u_end ? rb0 + GB : u_end;
            const bool whole = first == rb0 && end == rb0 + GB;
            const bool last = end == u_end;
            first = end;
            // The other contributor of the stream's last row block takes it at the start of
            // its own stream, so it has usually published its partial by the time this CTA
            // begins the row block: fetch it now, while the consumers are still computing.
            float other[4][C];
            bool gathered = false;
            if (!whole && last) {
                if (!waited) {
                    griddep_wait();  // the workspace belongs to the stream order
                    waited = true;
                }
                gathered = gather_other<C>(p, rb, GB, lane, other);
            }
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(pfull, seg & 1))) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            if (!waited) {
                griddep_wait();  // the workspace, x and y belong to the stream order
                waited = true;
            }
            const float* p0 = part;
            if (!whole && !gathered) {
                // publish this CTA's partial tile
                const int pf = cta_of_unit(rb0, p.T, (uint32_t)p.P);
                const int pl = cta_of_unit(rb0 + GB - 1, p.T, (uint32_t)p.P);
                const int mine = 2 * (int)blockIdx.x + (u0 >= rb0 ? 0 : 1);
                float4* dst = reinterpret_cast<float4*>(p.partials + (size_t)mine * kGemvSlotFloats);
                const float4* a4 = reinterpret_cast<const float4*>(p0);
                for (int q = lane; q < kGemvRows * C / 4; q += 32) __stcg(dst + q, a4[q]);
                {
                    // release the partial tile to the completing CTA: the warp's stores, then
                    // the counter increment by lane 0 with acquire-release semantics at GPU
                    // scope.  It orders the warp's stores (which __syncwarp orders before it)
                    // ahead of the increment, and in the CTA that completes the count it
                    // acquires every earlier contributor's partial; the barrier of the
                    // completion phase passes that on.
                    __syncwarp();
                    unsigned old = 0;
                    if (lane == 0) old = atomic_add_acq_rel_gpu(p.counters + rb, 1u);
                    old = __shfl_sync(0xffffffffu, old, 0);
                    // the CTA that completes the row block sums its partials after the stream ends
                    // (a stream-K CTA shares at most its first and its last row block)
                    if (lane == 0 && old == (unsigned)(pl - pf)) {
                        if (reduce_list[0] < 15)
                            reduce_list[1 + reduce_list[0]++] = rb;
                        else
                            record_error(p.err, kErrShape);
                    }
                }
            }
            if (whole || gathered) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = lane + 32 * i;
                    float v[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[c] = 0.0f;
#pragma unroll
                    for (int c = 0; c < C; c += 4) {
                        const float4 a = *reinterpret_cast<const float4*>(&p0[r * C + c]);
                        v[c] = a.x;
                        v[c + 1] = a.y;
                        v[c + 2] = a.z;
                        v[c + 3] = a.w;
                        if (gathered) {  // (0 + own) + other, as the completion phase adds
#pragma unroll
                            for (int e = 0; e < 4; ++e) v[c + e] = (0.0f + v[c + e]) + other[i][c + e];
                        }
                    }
                    write_row(p, rb * kGemvRows + r, v);
                }
                // the other contributor has arrived, so nothing else touches the counter
                if (gathered && lane == 0) atomicExch(p.counters + rb, 0u);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(pempty);
        }
    }
    // every thread that arrived on the cluster barrier also waits on it (the epilogue warp
    // did so before its exchange)
    if (p.cl != 0 && warp != kGemvEpilogue) cluster_wait_acquire();

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

size_t gemv_partial_bytes(int num_sms) { return (size_t)2 * num_sms * kGemvSlotFloats * sizeof(float); }

size_t gemv_counter_bytes(int N) { return ((size_t)(N / kGemvRows) * sizeof(unsigned) + 255) / 256 * 256; }

namespace {

// Cost of a schedule, in work units of the slowest CTA, plus an estimate of the end of the
// call: stream-K completes split row blocks through the workspace (a release, an acquire and
// loads of the other partials from L2, about two units' time), the cluster split-K through
// distributed shared memory (about half a unit).
constexpr double kStreamKExchange = 2.0;
constexpr double kClusterExchange = 0.5;

// Most clusters of `cl` CTAs of the kernel instance that can be resident at once (0 when
// none), per device; asked once and kept.
int max_active_clusters(bool two, int cl) {
    constexpr int kDevices = 64;
    static std::atomic<int> cache[kDevices][2][9];
    static std::atomic<bool> init{false};
    static std::mutex mu;
    if (!init.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> g(mu);
        if (!init.load(std::memory_order_relaxed)) {
            for (auto& d : cache)
                for (auto& t : d)
                    for (auto& c : t) c.store(-1, std::memory_order_relaxed);
            init.store(true, std::memory_order_release);
        }
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices || cl < 2 || cl > 8) return 0;
    std::atomic<int>& slot = cache[dev][two ? 1 : 0][cl];
    int v = slot.load(std::memory_order_relaxed);
    if (v >= 0) return v;
    // the 4-bit kernel's figures; the 3-bit one needs less shared memory, so they hold for it too
    const int smem = two ? GemvSmem<2, 4>::kBytes : GemvSmem<1, 4>::kBytes;
    const void* fn = two ? (const void*)gemv_w4a16_kernel<2, 4> : (const void*)gemv_w4a16_kernel<1, 4>;
    v = 0;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cl, 1, 1);
        cfg.blockDim = dim3(kGemvThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cl;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) == cudaSuccess && n > 0) v = n;
    }
    (void)cudaGetLastError();  // a refused query only rules the cluster schedule out
    slot.store(v, std::memory_order_relaxed);
    return v;
}

}  // namespace

GemvPlan gemv_plan(int M, int N, int K, int num_sms, int schedule) {
    const bool two = M > 8;
    const int NRB = N / kGemvRows, GB = K / (128 * kGemvUnitGroups);
    const long long T = (long long)NRB * GB;
    GemvPlan sk{W4A16_GEMV_STREAM_K, 0, 0, gemv_ctas(N, K, num_sms)};
    const long long per = (T + sk.ctas - 1) / sk.ctas;
    const bool split = T % sk.ctas != 0 || (T / sk.ctas) % GB != 0;
    const double cost_sk = (double)per + (split ? kStreamKExchange : 0.0);
    GemvPlan best{W4A16_GEMV_CLUSTER, 0, 0, 0};
    double cost_best = 0.0;
    if (schedule != W4A16_GEMV_STREAM_K) {
        for (int cl = 2; cl <= 8 && cl <= GB; ++cl) {
            const int mac = max_active_clusters(two, cl);
            if (mac < 1) continue;
            const int ncl = NRB < mac ? NRB : mac;
            // The automatic choice keeps to one row block per cluster: with several, each
            // exchange must hide behind the next row block's units, which few CTAs per
            // cluster can only do for long row blocks.
            if (schedule == W4A16_GEMV_AUTO && ncl < NRB) continue;
            const double cost = (double)((NRB + ncl - 1) / ncl) * ((GB + cl - 1) / cl) + kClusterExchange;
            if (best.cluster == 0 || cost < cost_best) {
                best = GemvPlan{W4A16_GEMV_CLUSTER, cl, ncl, ncl * cl};
                cost_best = cost;
            }
        }
    }
    if (schedule == W4A16_GEMV_CLUSTER) return best;  // cluster == 0: not possible here
    if (schedule == W4A16_GEMV_STREAM_K || best.cluster == 0 || cost_best >= cost_sk) return sk;
    return best;
}

template <int NT, int BITS>
static cudaError_t launch_gemv_kernel(const GemvMaps& maps, const GemvPlan& plan, const GemvArgs& a,
                                      cudaStream_t stream) {
    const int smem = GemvSmem<NT, BITS>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(gemv_w4a16_kernel<NT, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.P, 1, 1);
    cfg.blockDim = dim3(kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = plan.cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = plan.cluster != 0 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, gemv_w4a16_kernel<NT, BITS>, maps.w, a);
}

cudaError_t launch_gemv(const GemvMaps& maps, const GemvPlan& plan, int group_ratio, const uint16_t* x,
                        const uint16_t* scales, const uint32_t* zeros, const float* ysp, uint16_t* y,
                        float* partials, unsigned* counters, int M, int N, int K, unsigned* err,
                        cudaStream_t stream, int bits) {
    GemvArgs a{};
    a.x = x;
    a.scales = scales;
    a.zeros = zeros;
    a.ysp = ysp;
    a.y = y;
    a.M = M;
    a.N = N;
    a.K = K;
    a.T = (uint32_t)((N / kGemvRows) * (K / (128 * kGemvUnitGroups)));
    a.P = plan.ctas;
    a.gr = group_ratio;
    a.cl = plan.cluster;
    a.ncl = plan.clusters;
    a.err = err;
    if (plan.ctas < 1 || (plan.cluster != 0 && plan.ctas != plan.cluster * plan.clusters)) return cudaErrorInvalidValue;
    a.partials = partials;
    a.counters = counters;

    const bool two = M > 8;
    if (bits == 3) return two ? launch_gemv_kernel<2, 3>(maps, plan, a, stream) : launch_gemv_kernel<1, 3>(maps, plan, a, stream);
    if (bits != 4) return cudaErrorInvalidValue;
    return two ? launch_gemv_kernel<2, 4>(maps, plan, a, stream) : launch_gemv_kernel<1, 4>(maps, plan, a, stream);
}

}  // namespace w4a16
