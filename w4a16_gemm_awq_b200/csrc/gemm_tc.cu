// gemm_tc.cu -- prefill W4A16 GEMM on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// y[m][n] = bf16( sum_k x[m][k] * w~[n][k]  (+ ysp[n][m]) ),  w~ = bf16((q - z) * scale)
//
// [AWQ (MLSys 2024) translation, section 1: TinyChat dequantizes the packed 4-bit weights on
//  the fly inside the linear-layer kernel; SqueezeLLM article, section 2.3: W x = W_dense x +
//  W_sparse x.  At prefill sizes the layer is a dense contraction and runs on tensor cores.]
//
// Design (B200, one CTA per SM, one 128-channel x BN-token output tile per CTA):
//   - Swap-AB.  MMA M = 128 output channels, MMA N = BN tokens, both operands K-major.
//     D[channel][token] accumulates in TMEM (fp32, BN columns).
//   - The A operand (the weights) lives in TMEM.  Four dequant warps each own 32 TMEM lanes,
//     one channel row per thread.  Each thread reads its row's 8 packed words per 64-k
//     stage from shared memory and dequantizes them in registers: LOP3 magic-number unpack
//     to bf16 (128 + q), exact subtraction of (128 + z), multiplication by the bf16 group
//     scale.  The thread then writes the 32 bf16x2 columns into a TMEM A-stage with
//     tcgen05.st.  The dequantized weights never pass through shared memory, so shared
//     memory bandwidth serves only the TMA fills and the MMA's reads of x.
//   - The B operand (x) is TMA-staged: a 64-k x BN-token box, 128-byte swizzle, matching the
//     canonical K-major SW128 UMMA layout.  The packed weights of the stage (128 rows x 32
//     bytes) arrive on the same mbarrier.
//   - Warp roles: warp 0 issues the TMA, warp 1 issues tcgen05.mma from one thread, and
//     warps 2..5 dequantize and then run the epilogue.  There are four smem stages and
//     four TMEM A-stages, linked by mbarriers; tcgen05.commit releases the stages.
//   - Split-K for small grids: when the output tiles alone would leave SMs idle, the grid's
//     z dimension splits K into equal runs of whole 128-k slices.  Every CTA of a tile writes
//     its fp32 partial tile to the workspace and counts itself in the tile's counter; the CTA
//     that arrives last adds the partials in split order (its own from TMEM), so the sum's
//     order, and every bit of y, is the same whichever CTA finishes last.  It then resets the
//     counter to zero.  No CTA waits for another.
//   - CSR outlier term: the kernels of csr.cu compute ysp[n][m] = x . W_sparse^T in fp32
//     just before this kernel, which may start meanwhile (programmatic dependent launch).
//     The epilogue waits for them and adds ysp to the fp32 sum before the one rounding.
//   - Every mbarrier wait is bounded.  On timeout the CTA records kErrTimeout, stops its
//     loops, drains its own TMA and MMA work with bounded waits, and frees its TMEM.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kGemmThreads = 192;
constexpr int kStages = 4;
constexpr int kAStages = 4;
constexpr int kBK = 64;                          // k per pipeline stage
constexpr int kWStageBytes = 128 * kBK / 2;      // 128 rows x 32 bytes of packed weights
constexpr uint32_t kACols = kBK / 2;             // TMEM columns per A-stage (bf16 pairs)

struct GemmArgs {
    const uint16_t* scales;
    const uint32_t* zeros;
    const float* ysp;  // the CSR term [N][ysp_ld] fp32, or nullptr
    int ysp_ld;
    uint16_t* y;
    float* partials;    // split-K: fp32 tiles [tile][split][BN tokens][128 rows]
    unsigned* counters; // split-K: one per tile, zero between calls
    int M, N, K;
    int gr;      // quantization group size / 128: scales and zeros of 128-slice g are those of group g / gr
    int splits;  // CTAs per output tile along K (gridDim.z)
    int slices;  // 128-k slices per split
    unsigned* err;
};

template <int BN>
struct GemmSmem {
    static constexpr int kXStageBytes = BN * kBK * 2;
    static constexpr int kXOff = 0;
    static constexpr int kWOff = kStages * kXStageBytes;
    static constexpr int kParOff = kWOff + kStages * kWStageBytes;  // per stage: 256 B scales + 64 B zeros
    static constexpr int kBarOff = kParOff + kStages * 512;
    static constexpr int kBytes = kBarOff + 256;
    static constexpr uint32_t kTmemCols = (BN + kAStages * kACols) <= 256 ? 256u : 512u;
    static_assert(kXStageBytes % 1024 == 0 && kWOff % 1024 == 0,
                  "128-byte-swizzled TMA boxes need 1024-byte aligned stages");
};

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, rows of 128 bytes, 8-row
// groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;            // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset
    d |= (uint64_t)1 << 46;            // descriptor version for sm_100
    d |= (uint64_t)2 << 61;            // SWIZZLE_128B
    return d;
}

// kind::f16 instruction descriptor: D fp32, A bf16, B bf16, both K-major, M = 128, N = BN.
template <int BN>
__device__ __forceinline__ constexpr uint32_t idesc_bf16_m128() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Barrier 1 among the four epilogue warps (warps 2..5).
__device__ __forceinline__ void epilogue_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_w4a16_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                     const GemmArgs p) {
    using L = GemmSmem<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + kStages;
    uint64_t* afull = empty + kStages;
    uint64_t* aempty = afull + kAStages;
    uint64_t* accfull = aempty + kAStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * 128, m0 = blockIdx.y * BN;
    // this CTA's stages: [s0, s0 + nK), whole 128-k slices (a slice's first stage brings its
    // scales and zero points)
    const int s0 = (int)blockIdx.z * p.slices * 2;
    const int nK = min(p.slices * 2, p.K / kBK - s0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1 + 4);  // the MMA commit + one arrive per dequant warp
        }
        for (int i = 0; i < kAStages; ++i) {
            mbar_init(&afull[i], 4);
            mbar_init(&aempty[i], 1);
        }
        mbar_init(accfull, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&map_x);
        prefetch_tensormap(&map_w);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t a_col0 = (uint32_t)BN;  // A-stages follow the accumulator columns

    auto fail = [&]() {
        record_error(p.err, kErrTimeout);
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int s = 0; s < nK; ++s) {
                const int slot = s % kStages;
                if (*abort_flag) break;
                if (s >= kStages && !mbar_wait_bounded(&empty[slot], ((s / kStages) - 1) & 1)) {
                    fail();
                    break;
                }
                // a stage that starts a slice also brings the slice's 128 scales and 16 zero words
                const int sg = s0 + s;  // stage index along K
                const bool first_half = (sg & 1) == 0;
                mbar_arrive_expect_tx(&full[slot],
                                      (uint32_t)(L::kXStageBytes + kWStageBytes + (first_half ? 256 + 64 : 0)));
                tma_load_2d(smem + L::kXOff + slot * L::kXStageBytes, &map_x, &full[slot], sg * kBK, m0);
                tma_load_2d(smem + L::kWOff + slot * kWStageBytes, &map_w, &full[slot], sg * (kBK / 8), n0);
                if (first_half) {
                    const int g = (sg >> 1) / p.gr;  // the quantization group of this 128-slice
                    uint8_t* par = smem + L::kParOff + slot * 512;
                    bulk_load(par, p.scales + (size_t)g * p.N + n0, 256, &full[slot]);
                    bulk_load(par + 256, p.zeros + (size_t)g * (p.N >> 3) + (n0 >> 3), 64, &full[slot]);
                }
                ++issued;
            }
            // the copies this CTA started must land before it may exit
            for (int s = issued > kStages ? issued - kStages : 0; s < issued; ++s)
                (void)mbar_wait_bounded(&full[s % kStages], (s / kStages) & 1);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_m128<BN>();
            for (int s = 0; s < nK; ++s) {
                const int slot = s % kStages, as = s % kAStages;
                if (*abort_flag) break;
                if (!mbar_wait_bounded(&full[slot], (s / kStages) & 1) ||
                    !mbar_wait_bounded(&afull[as], (s / kAStages) & 1)) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t xs = smem_u32(smem + L::kXOff + slot * L::kXStageBytes);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    tc_mma_ts(tmem, tmem + a_col0 + (uint32_t)as * kACols + (uint32_t)kk * 8u,
                              desc_k_sw128(xs + kk * 32), idesc, (s | kk) != 0 ? 1u : 0u);
                }
                tc_commit(&empty[slot]);
                tc_commit(&aempty[as]);
            }
            tc_commit(accfull);
            if (*abort_flag) (void)mbar_wait_bounded(accfull, 0);  // MMAs in flight finish first
        }
    } else {
        // ---------------------------------------------------------------- dequant + epilogue
        const int quarter = warp & 3;             // TMEM lanes 32*quarter .. +31
        const int row = 32 * quarter + lane;      // channel within the tile == TMEM lane
        const int n = n0 + row;
        const uint32_t t_lane = (uint32_t)(32 * quarter) << 16;
        uint32_t sb = 0, zb = 0;

        // waits and abort checks are made warp-uniform: tcgen05.st/ld are .sync.aligned
        auto warp_wait = [&](uint64_t* bar, uint32_t parity) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity));
            if (!ok && lane == 0) fail();
            return ok;
        };
        auto warp_abort = [&]() { return __any_sync(0xffffffffu, *abort_flag != 0); };

        for (int s = 0; s < nK; ++s) {
            const int slot = s % kStages, as = s % kAStages;
            if (warp_abort()) break;
            if (!warp_wait(&full[slot], (s / kStages) & 1)) break;
            // the row's 32 bytes in the 32-byte-swizzled W stage: chunk c at c ^ ((row >> 2) & 1)
            const uint8_t* wrow = smem + L::kWOff + slot * kWStageBytes + row * 32;
            const int sw = (row >> 2) & 1;
            const uint4 wa = *reinterpret_cast<const uint4*>(wrow + ((0 ^ sw) << 4));
            const uint4 wb = *reinterpret_cast<const uint4*>(wrow + ((1 ^ sw) << 4));
            if (((s0 + s) & 1) == 0) {  // a new slice of 128 k: its scale and zero point from the stage
                const uint8_t* par = smem + L::kParOff + slot * 512;
                const uint16_t sbits = reinterpret_cast<const uint16_t*>(par)[row];
                const uint32_t z = (reinterpret_cast<const uint32_t*>(par + 256)[row >> 3] >> (4 * (row & 7))) & 15u;
                const uint32_t sbf = float_to_bf16_bits(fp16_bits_to_float(sbits));
                sb = sbf | (sbf << 16);
                zb = 0x43004300u | z | (z << 16);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);

            uint32_t v[32];
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const uint32_t word = w < 4 ? u4_get(wa, w) : u4_get(wb, w - 4);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t t;
                    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(t) : "r"(word >> (4 * i)), "r"(0x000F000Fu),
                        "r"(0x43004300u));
                    v[4 * w + i] = bf16x2_mul(bf16x2_sub(t, zb), sb);
                }
            }

            if (s >= kAStages && !warp_wait(&aempty[as], ((s / kAStages) - 1) & 1)) break;
            tc_fence_after();
            tmem_st_32x32b_x32(tmem + t_lane + a_col0 + (uint32_t)as * kACols, v);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[as]);
        }
        const bool aborted = warp_abort();

        // epilogue: TMEM -> registers (-> split-K reduction) (+ CSR term) -> bf16 -> y[m][n]
        if (!aborted && warp_wait(accfull, 0)) {
            tc_fence_after();
            const size_t tile = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
            const int z = (int)blockIdx.z;
            bool last = true;
            if (p.splits > 1) {
                // this CTA's partial tile, token-major ([BN][128]): for each token the 32 lanes of a
                // warp write 32 consecutive floats, so every store is one coalesced 128-byte line
                float* mine = p.partials + (tile * p.splits + z) * 128 * BN + row;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem + t_lane + (uint32_t)c0, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) __stcg(mine + (c0 + j) * 128, __uint_as_float(r[j]));
                }
                __threadfence();
                epilogue_sync();
                if (warp == 2 && lane == 0) {
                    const unsigned before = atomicAdd(p.counters + tile, 1u);
                    const bool is_last = before == (unsigned)(p.splits - 1);
                    if (is_last) p.counters[tile] = 0u;  // every split has counted itself
                    *last_flag = is_last ? 1 : 0;
                }
                epilogue_sync();
                last = *last_flag != 0;
                if (last) __threadfence();
            }
            if (p.splits == 1 && p.ysp == nullptr) {
                // the common case, kept minimal: one TMEM chunk at a time straight to y
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem + t_lane + (uint32_t)c0, r);
                    tmem_ld_wait();
                    if (m0 + c0 >= p.M) break;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + c0 + j;
                        if (m < p.M) p.y[(size_t)m * p.N + n] = float_to_bf16_bits(__uint_as_float(r[j]));
                    }
                }
            } else if (last) {
                const float* ysr = nullptr;
                if (p.ysp != nullptr) {
                    asm volatile("griddepcontrol.wait;" ::: "memory");  // ysp is complete
                    ysr = p.ysp + (size_t)n * p.ysp_ld;
                }
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem + t_lane + (uint32_t)c0, r);
                    tmem_ld_wait();
                    if (m0 + c0 >= p.M) break;
                    float acc[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc[j] = __uint_as_float(r[j]);
                    if (p.splits > 1) {
                        // sum of the partial tiles in split order; this CTA's own is in acc
                        float own[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) own[j] = acc[j];
#pragma unroll 1
                        for (int zz = 0; zz < p.splits; ++zz) {
                            float v[32];
                            if (zz == z) {
#pragma unroll
                                for (int j = 0; j < 32; ++j) v[j] = own[j];
                            } else {
                                const float* src = p.partials + (tile * p.splits + zz) * 128 * BN + c0 * 128 + row;
#pragma unroll
                                for (int j = 0; j < 32; ++j) v[j] = __ldcg(src + j * 128);
                            }
#pragma unroll
                            for (int j = 0; j < 32; ++j) acc[j] = zz == 0 ? v[j] : acc[j] + v[j];
                        }
                    }
                    if (ysr != nullptr) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (m0 + c0 + j < p.M) acc[j] += __ldcg(ysr + m0 + c0 + j);
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + c0 + j;
                        if (m < p.M) p.y[(size_t)m * p.N + n] = float_to_bf16_bits(acc[j]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int BN>
static cudaError_t launch_bn(const GemmMaps& maps, const GemmArgs& a, bool after_csr, cudaStream_t stream) {
    using L = GemmSmem<BN>;
    // At most 512 / kTmemCols CTAs may share an SM, or a tcgen05.alloc would have to wait for
    // another CTA's TMEM: the shared-memory request enforces that bound.
    constexpr int kMinSmem = L::kTmemCols == 512u ? 120 * 1024 : 80 * 1024;
    const int smem = (L::kBytes + 1024) > kMinSmem ? (L::kBytes + 1024) : kMinSmem;
    cudaError_t e = cudaFuncSetAttribute(gemm_w4a16_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.N / 128, (a.M + BN - 1) / BN, a.splits);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_csr ? 1 : 0;  // overlap the CSR kernels; otherwise plain stream order
    return cudaLaunchKernelEx(&cfg, gemm_w4a16_tc_kernel<BN>, maps.x, maps.qw, a);
}

GemmPlan gemm_plan(int64_t M, int64_t N, int64_t K, int num_sms) {
    GemmPlan g{};
    g.bn = M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    const int64_t tiles = (N / 128) * ((M + g.bn - 1) / g.bn);
    const int64_t nslices = K / 128;
    g.splits = 1;
    g.slices = (int)nslices;
    // Time model in slices: the longer of one CTA's run and the grid's total work spread over
    // the SMs, plus the split's own cost (partial tiles written and read back), about half a
    // slice per extra split and 64 tokens.  Only grids of under two waves are split, and only
    // while the partial tiles stay within kMaxGemmPartialBytes.  Measured on B200, 256-token
    // tiles lose when the split grid needs a second wave (their CTAs' partial tiles, 128 KB
    // each, cost several microseconds to write and read back), so those split only within
    // one wave.
    if (tiles < 2 * (int64_t)num_sms && tiles <= kMaxGemmTiles) {
        const double sms = (double)num_sms;
        double best = std::max((double)nslices, (double)(tiles * nslices) / sms);
        for (int S = 2; S <= kMaxGemmSplits; ++S) {
            const int64_t per = (nslices + S - 1) / S;
            const int64_t used = (nslices + per - 1) / per;  // no empty split
            if (used != S || per < 4 || (size_t)tiles * S * 128 * g.bn * 4 > kMaxGemmPartialBytes) continue;
            if (g.bn == 256 && tiles * S > num_sms) continue;
            const double cost = std::max((double)per, (double)(tiles * S * per) / sms) + 0.5 * (S - 1) * g.bn / 64.0;
            if (cost < best - 0.5) {
                best = cost;
                g.splits = S;
                g.slices = (int)per;
            }
        }
    }
    g.partial_bytes = g.splits > 1 ? (size_t)tiles * g.splits * 128 * g.bn * 4 : 0;
    return g;
}

cudaError_t launch_gemm(const GemmMaps& maps, const GemmPlan& plan, int group_ratio, const uint16_t* scales,
                        const uint32_t* zeros, const float* ysp, int ysp_ld, uint16_t* y, float* partials,
                        unsigned* counters, int M, int N, int K, unsigned* err, cudaStream_t stream) {
    GemmArgs a{scales, zeros, ysp, ysp_ld, y, partials, counters, M, N, K, group_ratio, plan.splits, plan.slices, err};
    const bool after_csr = ysp != nullptr;
    switch (plan.bn) {
        case 32: return launch_bn<32>(maps, a, after_csr, stream);
        case 64: return launch_bn<64>(maps, a, after_csr, stream);
        case 128: return launch_bn<128>(maps, a, after_csr, stream);
        case 256: return launch_bn<256>(maps, a, after_csr, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace w4a16
