// gemv.cu -- decode W4A16 GEMV (1 <= M <= 16): y = bf16(x . dequant(Q)^T [+ x . W_sparse^T]).
//
// [AWQ (MLSys 2024) translation, section 1: TinyChat computes the linear layer from packed
//  4-bit weights dequantized on the fly; at decode batch sizes the layer is bound by memory
//  bandwidth (section 2: weight-only quantization relieves the memory bottleneck).
//  SqueezeLLM article, section 2.3: the fp16 sparse term is added to the dense product.]
//
// Design (B200).  Each packed weight byte is streamed once from HBM through a TMA pipeline
// by a persistent, evenly balanced grid.
//   - Work units are (128-channel row block, quantization group of 128 k), ordered row block
//     by row block.  The grid has P = min(2 x SMs, units) CTAs; CTA p takes the contiguous
//     unit range [p*T/P, (p+1)*T/P), so every CTA streams the same number of bytes and the
//     GPU runs one balanced wave (stream-K).  Two resident CTAs per SM keep enough TMA
//     traffic in flight to saturate HBM.
//   - A row block processed whole by one CTA is written straight to y.  A row block split
//     between CTAs leaves fp32 partial tiles in the caller's workspace.  Each contributing
//     CTA then increments the row block's counter.  The CTA that completes the count sums
//     the partials once its own stream has ended, writes y and resets the counter to zero.
//     No CTA waits for another, and the workspace is all-zero again after every call.
//   - CTA = 4 consumer warps (32 channels each, two m16 tiles), 1 TMA producer warp, 1 sum
//     warp and 1 epilogue warp.  At the end of each row-block segment the consumers drop
//     their accumulators into one of two shared-memory partial tiles and go on streaming;
//     the epilogue warp does the workspace exchange, the CSR term and the stores of y.  One pipeline stage holds one unit: the packed weights of the 128 channels
//     (TMA box 16 words x 128 rows, 8 KB) and the group's activations (two TMA boxes of
//     64 k x (Mpad + 2) tokens, 128-byte swizzle).  The second box is loaded from token -2.
//     Its rows therefore sit two swizzle phases after the first box's rows, which makes
//     every B-fragment load below free of shared-memory bank conflicts.
//   - On B200 the CUDA cores cannot do one FMA per weight per token at HBM rate, so the
//     multiply-adds go to the tensor cores (mma.sync m16n8k16) with the operands swapped.
//     The MMA rows are 16 channels, the columns are 8 tokens (two tiles when M > 8), and
//     the depth is 16 input channels.  The A operand (the weights) goes from shared memory
//     to registers.  One LOP3 per nibble pair makes the bf16 pair (128 + q_lo, 128 + q_hi)
//     (exponent bits 0x43), and those exact values feed the MMA unchanged.  The zero point
//     and the scale are applied once per group in fp32:
//         y += s * ( sum_k (128 + q_k) x_k  -  (128 + z) * X_g ),   X_g = sum_{k in g} x_k.
//     The sum warp computes X_g for every staged group from the x tile, so the per-weight
//     work is one shift and one LOP3 per two weights plus the MMA.
//   - Which physical k feeds which MMA slot.  Thread t (= lane % 4) takes words 4t..4t+3 of
//     a row's group, i.e. k in [32t, 32t+32).  MMA pair w (0..3) uses word w: nibble pairs
//     (0,1) in the first MMA and (2,3) in the second.  Pair p of word w holds
//     k = 32t + 8w + 2p + {0,1}.  The B fragment of thread (token g, t) is then one
//     128-bit load of x[g][32t + 8w .. +8], whose four 32-bit parts are the same pairs.
//   - Scales and zero points are stored group-major, so a unit's parameters (128 fp16 scales
//     and 16 words of zero points) are two contiguous runs that 1D bulk copies bring into the
//     same stage.
//   - Programmatic dependent launch.  The weights of the first stages may be fetched before
//     the previous kernel on the stream has finished.  The producer waits for that kernel
//     before it loads x.  The epilogue warp waits before it touches the workspace, gathers x
//     for the CSR term, or writes y.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kGemvRows = 128;
constexpr int kGemvConsumers = 4;                         // warps 0..3
constexpr int kGemvProducer = kGemvConsumers;             // warp 4: TMA
constexpr int kGemvSummer = kGemvConsumers + 1;           // warp 5: per-group token sums X_g
constexpr int kGemvEpilogue = kGemvConsumers + 2;         // warp 6: partial exchange, CSR, y
constexpr int kGemvThreads = 32 * (kGemvConsumers + 3);
constexpr int kGemvStages = 6;
constexpr int kGemvWBytes = kGemvRows * 64;  // one group of packed weights for 128 rows
constexpr int kGemvCtasPerSm = 2;
constexpr int kGemvSlotFloats = kGemvRows * 16;  // one partial tile [128][16] fp32

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
    long long T;         // work units = (N/128) * (K/128)
    int P;               // CTAs
    unsigned* err;
};

template <int NT>
struct GemvSmem {
    static constexpr int kMpad = 8 * NT;
    static constexpr int kXRows = kMpad + 2;                       // tokens -2 .. Mpad-1 (box 1)
    static constexpr int kXTx = kXRows * 128;                        // bytes one x box brings
    static constexpr int kXBox = ((kXTx + 1023) / 1024) * 1024;      // 1024-aligned slot
    static constexpr int kStage = kGemvWBytes + 2 * kXBox;   // 1024-aligned: the x boxes are swizzled
    static constexpr int kParOff = kGemvStages * kStage;       // [stage]: scales 256 B + zeros 64 B
    static constexpr int kPartOff = kParOff + kGemvStages * 512;
    static constexpr int kXsumOff = kPartOff + 2 * kGemvSlotFloats * 4;  // [stage][16] fp32
    static constexpr int kBarOff = kXsumOff + kGemvStages * 16 * 4;
    static constexpr int kListOff = kBarOff + (4 * kGemvStages + 4) * 8;  // row blocks this CTA completes
    static constexpr int kBytes = kListOff + 16 * 4;
    static_assert(kStage % 1024 == 0, "128-byte-swizzled TMA boxes need 1024-byte aligned stages");
};

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

// bf16 pairs (128 + q_lo, 128 + q_hi) of the 4 nibble pairs of a packed word.
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t out[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(out[i]) : "r"(w >> (4 * i)), "r"(0x000F000Fu), "r"(0x43004300u));
}

// fp32 sum of the 64 bf16 values of one 128-byte row of an x box (the order within the row
// does not matter, so the swizzle does not either).
__device__ __forceinline__ float row_sum_128b(const uint8_t* row) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = lds128(row + 16 * c);
        a0 += __uint_as_float(v.x << 16) + __uint_as_float(v.x & 0xFFFF0000u);
        a1 += __uint_as_float(v.y << 16) + __uint_as_float(v.y & 0xFFFF0000u);
        a2 += __uint_as_float(v.z << 16) + __uint_as_float(v.z & 0xFFFF0000u);
        a3 += __uint_as_float(v.w << 16) + __uint_as_float(v.w & 0xFFFF0000u);
    }
    return (a0 + a1) + (a2 + a3);
}

__device__ __forceinline__ long long unit_begin(int p, long long T, int P) { return T * p / P; }

// The CTA whose unit range contains unit u: the largest p with floor(p*T/P) <= u.
__device__ __forceinline__ int cta_of_unit(long long u, long long T, int P) {
    return (int)(((u + 1) * (long long)P - 1) / T);
}

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
__global__ void __launch_bounds__(kGemvThreads, kGemvCtasPerSm)
gemv_w4a16_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                  const GemvArgs p) {
    using L = GemvSmem<NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + kGemvStages;
    uint64_t* xfull = empty + kGemvStages;
    uint64_t* xempty = xfull + kGemvStages;
    uint64_t* pfull = xempty + kGemvStages;   // [2] a partial tile is ready for the epilogue
    uint64_t* pempty = pfull + 2;             // [2] the epilogue is done with a partial tile
    float* part = reinterpret_cast<float*>(smem + L::kPartOff);     // [2][row][token]
    float* xsum = reinterpret_cast<float*>(smem + L::kXsumOff);     // [stage][token]
    int* reduce_list = reinterpret_cast<int*>(smem + L::kListOff);  // [0] = count, then row blocks

    const int G = p.K >> 7;
    const long long u0 = unit_begin(blockIdx.x, p.T, p.P);
    const int n = (int)(unit_begin(blockIdx.x + 1, p.T, p.P) - u0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kGemvStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kGemvConsumers + 1);  // consumers + the sum warp read the stage
            mbar_init(&xfull[i], 1);
            mbar_init(&xempty[i], kGemvConsumers);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&pfull[i], kGemvConsumers);
            mbar_init(&pempty[i], 1);
        }
        reduce_list[0] = 0;
        fence_mbarrier_init();
    }
    __syncthreads();

    if (warp == kGemvSummer) {
        // ------------------------------------------------------------------ sum warp
        // lane l sums token l/2, half l%2 (k 0..63 from box 0, k 64..127 from box 1 at row +2)
        const int tok = lane >> 1, half = lane & 1;
        for (int s = 0; s < n; ++s) {
            const int slot = s % kGemvStages;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full[slot], (s / kGemvStages) & 1) &&
                                                        (s < kGemvStages ||
                                                         mbar_wait_bounded(&xempty[slot], ((s / kGemvStages) - 1) & 1)));
            if (!ok) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            float v = 0.0f;
            if (tok < L::kMpad) {
                const uint8_t* xs = smem + slot * L::kStage + kGemvWBytes + half * L::kXBox;
                v = row_sum_128b(xs + (tok + 2 * half) * 128);
            }
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            if (half == 0 && tok < L::kMpad) xsum[slot * 16 + tok] = v;
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&empty[slot]);
                mbar_arrive(&xfull[slot]);
            }
        }
    } else if (warp == kGemvProducer) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&map_w);
            prefetch_tensormap(&map_x);
            const uint32_t tx = (uint32_t)(kGemvWBytes + 2 * L::kXTx + 256 + 64);
            // the unit's scales (128 fp16 of row block rb, group g) and zero points (16 words)
            auto load_params = [&](int slot, int rb, int g, uint64_t* bar) {
                uint8_t* par = smem + L::kParOff + slot * 512;
                bulk_load(par, p.scales + (size_t)g * p.N + (size_t)rb * kGemvRows, 256, bar);
                bulk_load(par + 256, p.zeros + (size_t)g * (p.N >> 3) + (size_t)rb * (kGemvRows / 8), 64, bar);
            };
            auto coords = [&](int s, int& rb, int& g) {
                const long long u = u0 + s;
                rb = (int)(u / G);
                g = (int)(u - (long long)rb * G);
            };
            const int pre = n < kGemvStages ? n : kGemvStages;
            for (int s = 0; s < pre; ++s) {   // weights do not depend on the previous kernel
                int rb, g;
                coords(s, rb, g);
                mbar_arrive_expect_tx(&full[s], tx);
                tma_load_2d(smem + s * L::kStage, &map_w, &full[s], g * 16, rb * kGemvRows);
                load_params(s, rb, g, &full[s]);
            }
            griddep_wait();
            for (int s = 0; s < pre; ++s) {
                int rb, g;
                coords(s, rb, g);
                uint8_t* xs = smem + s * L::kStage + kGemvWBytes;
                tma_load_2d(xs, &map_x, &full[s], g * 128, 0);
                tma_load_2d(xs + L::kXBox, &map_x, &full[s], g * 128 + 64, -2);
            }
            int issued = pre;
            for (int s = pre; s < n; ++s) {
                const int slot = s % kGemvStages;
                if (!mbar_wait_bounded(&empty[slot], ((s / kGemvStages) - 1) & 1)) {
                    record_error(p.err, kErrTimeout);
                    break;
                }
                int rb, g;
                coords(s, rb, g);
                uint8_t* st = smem + slot * L::kStage;
                mbar_arrive_expect_tx(&full[slot], tx);
                tma_load_2d(st, &map_w, &full[slot], g * 16, rb * kGemvRows);
                load_params(slot, rb, g, &full[slot]);
                tma_load_2d(st + kGemvWBytes, &map_x, &full[slot], g * 128, 0);
                tma_load_2d(st + kGemvWBytes + L::kXBox, &map_x, &full[slot], g * 128 + 64, -2);
                ++issued;
            }
            // the copies this CTA started must land before it may exit
            for (int s = issued > kGemvStages ? issued - kGemvStages : 0; s < issued; ++s)
                (void)mbar_wait_bounded(&full[s % kGemvStages], (s / kGemvStages) & 1);
        }
    } else if (warp < kGemvConsumers) {
        // ------------------------------------------------------------------ consumers
        const int gq = lane >> 2, t = lane & 3;
        const int rbase = 32 * warp + gq;  // this thread's rows: rbase + 16 i + 8 h
        int seg = 0;                       // segments handed to the epilogue so far
        float acc[2][NT][4];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.0f;

        int rb = (int)(u0 / G), g = (int)(u0 - (long long)rb * G);  // coordinates of unit u0 + s
        for (int s = 0; s < n; ++s, (g + 1 == G ? (g = 0, ++rb) : ++g)) {
            const int slot = s % kGemvStages;

            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full[slot], (s / kGemvStages) & 1));
            if (!ok) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            const uint8_t* ws = smem + slot * L::kStage;
            const uint8_t* xs = ws + kGemvWBytes;
            uint4 wv[2][2];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) wv[i][h] = lds128(ws + (rbase + 16 * i + 8 * h) * 64 + t * 16);
            uint4 xv[NT][4];
#pragma unroll
            for (int j = 0; j < NT; ++j) {
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int b = t >> 1, c = 4 * (t & 1) + w;
                    const int row = 8 * j + gq + 2 * b;
                    xv[j][w] = lds128(xs + b * L::kXBox + row * 128 + ((c ^ (row & 7)) << 4));
                }
            }
            uint32_t sz4[4];  // rows rbase + 0, 8, 16, 24: scale bits | zero << 16
            {
                const uint8_t* par = smem + L::kParOff + slot * 512;
                const uint16_t* sc = reinterpret_cast<const uint16_t*>(par);
                const uint32_t* zw = reinterpret_cast<const uint32_t*>(par + 256);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int row = rbase + 8 * k;
                    sz4[k] = (uint32_t)sc[row] | (((zw[row >> 3] >> (4 * (row & 7))) & 15u) << 16);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);

            // MMA chains: kParts independent partial accumulators per (tile, token tile), one per
            // packed word (M <= 8) or per pair of words (M <= 16), so that the dependent
            // mma.sync chains are short and the tensor pipe sees several in flight.
            constexpr int kParts = NT == 1 ? 4 : 2;
            float d[2][NT][4];
            {
                float dp[kParts][2][NT][4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int part_i = w % kParts;
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        uint32_t pa0[4], pa1[4];
                        unpack_word(u4_get(wv[i][0], w), pa0);
                        unpack_word(u4_get(wv[i][1], w), pa1);
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t A[4] = {pa0[2 * hh], pa1[2 * hh], pa0[2 * hh + 1], pa1[2 * hh + 1]};
#pragma unroll
                            for (int j = 0; j < NT; ++j) {
                                const uint32_t B[2] = {u4_get(xv[j][w], 2 * hh), u4_get(xv[j][w], 2 * hh + 1)};
                                if (w < kParts && hh == 0)
                                    mma_16816_bf16_zero(dp[part_i][i][j], A, B);
                                else
                                    mma_16816_bf16(dp[part_i][i][j], A, B);
                            }
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int j = 0; j < NT; ++j)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float v = dp[0][i][j][e];
#pragma unroll
                            for (int q = 1; q < kParts; ++q) v += dp[q][i][j][e];
                            d[i][j][e] = v;
                        }
            }
            // the group's zero point and scale, applied in fp32:
            //   acc += s * d - s * (128 + z) * X_g
            const bool xok = __all_sync(0xffffffffu, mbar_wait_bounded(&xfull[slot], (s / kGemvStages) & 1));
            if (!xok) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            float2 X[NT];
#pragma unroll
            for (int j = 0; j < NT; ++j) X[j] = *reinterpret_cast<const float2*>(&xsum[slot * 16 + 8 * j + 2 * t]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&xempty[slot]);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                // rows rbase + 16 i (index 2i) and rbase + 16 i + 8 (index 2i + 1)
                const float sc0 = fp16_bits_to_float((uint16_t)(sz4[2 * i] & 0xFFFFu));
                const float sc1 = fp16_bits_to_float((uint16_t)(sz4[2 * i + 1] & 0xFFFFu));
                const float b0 = -(float)(128u + (sz4[2 * i] >> 16)), b1 = -(float)(128u + (sz4[2 * i + 1] >> 16));
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    acc[i][j][0] = fmaf(sc0, fmaf(b0, X[j].x, d[i][j][0]), acc[i][j][0]);
                    acc[i][j][1] = fmaf(sc0, fmaf(b0, X[j].y, d[i][j][1]), acc[i][j][1]);
                    acc[i][j][2] = fmaf(sc1, fmaf(b1, X[j].x, d[i][j][2]), acc[i][j][2]);
                    acc[i][j][3] = fmaf(sc1, fmaf(b1, X[j].y, d[i][j][3]), acc[i][j][3]);
                }
            }

            if (g == G - 1 || s == n - 1) {
                // ---------------------------------------------------------- segment end
                // hand the accumulators to the epilogue warp through partial tile `buf`
                const int buf = seg & 1;
                const bool ok2 = seg < 2 || __all_sync(0xffffffffu, mbar_wait_bounded(&pempty[buf], ((seg >> 1) - 1) & 1));
                if (!ok2) {
                    if (lane == 0) record_error(p.err, kErrTimeout);
                    break;
                }
                float* pt = part + buf * kGemvSlotFloats;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int c0 = rbase + 16 * i, c1 = c0 + 8;
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        const int tk = 8 * j + 2 * t;
                        *reinterpret_cast<float2*>(&pt[c0 * 16 + tk]) = make_float2(acc[i][j][0], acc[i][j][1]);
                        *reinterpret_cast<float2*>(&pt[c1 * 16 + tk]) = make_float2(acc[i][j][2], acc[i][j][3]);
                        acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.0f;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&pfull[buf]);
                ++seg;
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue warp
        // Walks the same segments as the consumers.  Lane l owns rows l, l+32, l+64, l+96.
        bool waited = false;
        int seg = 0;
        int seg_g0 = (int)(u0 % G);
        for (int s = 0; s < n; ++s) {
            const long long u = u0 + s;
            const int rb = (int)(u / G), g = (int)(u - (long long)rb * G);
            if (!(g == G - 1 || s == n - 1)) continue;
            const bool whole = seg_g0 == 0 && g == G - 1;
            seg_g0 = 0;
            const int buf = seg & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&pfull[buf], (seg >> 1) & 1));
            if (!ok) {
                if (lane == 0) record_error(p.err, kErrTimeout);
                break;
            }
            if (!waited) {
                griddep_wait();  // the workspace, x and y belong to the stream order
                waited = true;
            }
            const float* pt = part + buf * kGemvSlotFloats;
            if (whole) {
                for (int r = lane; r < kGemvRows; r += 32) {
                    float v[16];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float4 a = *reinterpret_cast<const float4*>(&pt[r * 16 + 4 * c]);
                        v[4 * c] = a.x;
                        v[4 * c + 1] = a.y;
                        v[4 * c + 2] = a.z;
                        v[4 * c + 3] = a.w;
                    }
                    write_row(p, rb * kGemvRows + r, v);
                }
            } else {
                const int pf = cta_of_unit((long long)rb * G, p.T, p.P);
                const int pl = cta_of_unit((long long)rb * G + G - 1, p.T, p.P);
                const int mine = 2 * (int)blockIdx.x + (u0 >= (long long)rb * G ? 0 : 1);
                float4* dst = reinterpret_cast<float4*>(p.partials + (size_t)mine * kGemvSlotFloats);
                const float4* srcp = reinterpret_cast<const float4*>(pt);
                for (int q = lane; q < kGemvSlotFloats / 4; q += 32) __stcg(dst + q, srcp[q]);
                // release the partial tile to the completing CTA: the warp's stores, then a fence
                // and the counter increment by lane 0; the completing CTA fences after it
                __syncwarp();
                unsigned old = 0;
                if (lane == 0) {
                    __threadfence();
                    old = atomicAdd(p.counters + rb, 1u);
                    __threadfence();
                }
                old = __shfl_sync(0xffffffffu, old, 0);
                // the CTA that completes the row block sums its partials after the stream ends
                if (lane == 0 && old == (unsigned)(pl - pf) && reduce_list[0] < 15)
                    reduce_list[1 + reduce_list[0]++] = rb;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[buf]);
            ++seg;
        }
    }
    griddep_launch_dependents();

    // ---------------------------------------------------------------------- completions
    // The consumer warps and the epilogue warp sum the partial tiles of the row blocks this
    // CTA completed: thread r (< 128) owns row r, loads of several slots are in flight at once.
    if (warp < kGemvConsumers || warp == kGemvEpilogue) {
        asm volatile("bar.sync 2, %0;" ::"r"(32 * (kGemvConsumers + 1)) : "memory");
        const int r = warp < kGemvConsumers ? (int)threadIdx.x : -1;
        const int count = reduce_list[0];
        if (count > 0) __threadfence();  // acquire: every other contributor's partial is visible
        for (int e = 0; e < count && r >= 0; ++e) {
            const int rb = reduce_list[1 + e];
            const int pf = cta_of_unit((long long)rb * G, p.T, p.P);
            const int pl = cta_of_unit((long long)rb * G + G - 1, p.T, p.P);
            float v[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) v[m] = 0.0f;
            for (int q0 = pf; q0 <= pl; q0 += 2) {
                float4 a[2][4];
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const int q = q0 + qq;
                    if (q <= pl) {
                        const int slotq = 2 * q + (unit_begin(q, p.T, p.P) >= (long long)rb * G ? 0 : 1);
                        const float4* sp = reinterpret_cast<const float4*>(p.partials +
                                                                           (size_t)slotq * kGemvSlotFloats + r * 16);
#pragma unroll
                        for (int c = 0; c < 4; ++c) a[qq][c] = __ldcg(sp + c);
                    }
                }
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    if (q0 + qq <= pl) {
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
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
    const long long T = (long long)(N / kGemvRows) * (K / 128);
    const long long P = (long long)kGemvCtasPerSm * num_sms;
    return (int)(T < P ? T : P);
}

size_t gemv_workspace_bytes(int N, int num_sms) {
    const size_t partials = (size_t)2 * kGemvCtasPerSm * num_sms * kGemvSlotFloats * sizeof(float);
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
    a.T = (long long)(N / kGemvRows) * (K / 128);
    a.P = gemv_ctas(N, K, num_sms);
    a.err = err;
    const size_t partial_bytes = (size_t)2 * kGemvCtasPerSm * num_sms * kGemvSlotFloats * sizeof(float);
    a.partials = static_cast<float*>(workspace);
    a.counters = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(workspace) + partial_bytes);

    const bool two = M > 8;
    const int smem = (two ? GemvSmem<2>::kBytes : GemvSmem<1>::kBytes) + 1024;
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
    if (two) return cudaLaunchKernelEx(&cfg, gemv_w4a16_kernel<2>, maps.w, maps.x, a);
    return cudaLaunchKernelEx(&cfg, gemv_w4a16_kernel<1>, maps.w, maps.x, a);
}

}  // namespace w4a16
