// gemv.cu -- decode W4A16 GEMV (1 <= M <= 16): y = bf16(x . dequant(Q)^T [+ x . W_sparse^T]).
//
// [AWQ (MLSys 2024) translation, section 1: TinyChat computes the linear layer from packed
//  4-bit weights dequantized on the fly; at decode batch sizes the layer is bound by
//  memory bandwidth (section 2, weight-only quantization eases the memory bottleneck).
//  SqueezeLLM article, section 2.3: the fp16 sparse term is added to the dense product.]
//
// Design (B200).  The kernel streams the packed weights once at HBM rate.  On B200 the CUDA
// cores cannot do one FMA per weight per token at that rate, so the multiply-adds go to
// the tensor cores with the operands swapped:
//   MMA rows (M of m16n8k16)  = 16 output channels,
//   MMA cols (N)              = 8 tokens (M <= 8) or two tiles of 8 (M <= 16),
//   MMA depth (K)             = 16 input channels.
// The A operand (the weights) never touches shared memory.  Each thread loads its 128-bit
// slice of two channel rows, unpacks nibble pairs with one LOP3 into bf16 "128 + q"
// (exponent bits 0x43), and subtracts the bf16 "128 + z" to get the exact integer q - z.
// Those registers are the A fragment.  The per-group scale is applied in fp32 after the
// group's 8 MMAs, so the weight values inside the MMA are exact.
//
// The K dimension is split across the S CTAs of a thread-block cluster.  Each CTA leaves its
// fp32 partial tile in shared memory.  After a cluster barrier, each CTA reduces a slice of
// the outputs by reading all S partials over DSMEM, adds the CSR outlier term for those
// outputs, rounds to bf16 once and stores.  There is no global scratch and no atomics.
//
// Which physical k feeds which MMA slot: thread t (= lane % 4) loads words 4t..4t+3 of a
// group, i.e. k in [32t, 32t+32).  MMA j (0..7) of the group takes word w = j/2: nibble
// pairs (0,1) when j is even and (2,3) when j is odd.  Pair p of word w holds
// k = 32t + 8w + 2p + {0,1}.  The B fragment of thread (token g, t) is then one 128-bit
// load of x[g][32t + 8w .. +8], whose four 32-bit parts are the same four pairs.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

constexpr int kGemvWarps = 4;
constexpr int kGemvRows = 16 * kGemvWarps;  // output channels per CTA
constexpr int kGemvPF = 4;                  // groups of weights in flight per thread

struct GemvArgs {
    const uint16_t* x;
    const uint32_t* qw;
    const uint16_t* scales;
    const uint32_t* zeros;
    const int32_t* row_ptr;
    const int32_t* col_idx;
    const uint16_t* vals;
    long long nnz;
    uint16_t* y;
    int M, N, K, S;
    unsigned* err;
};

// (128+q_lo, 128+q_hi) - (128+z, 128+z) for the 4 nibble pairs of a packed word.
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t zb, uint32_t out[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t v;
        asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(v) : "r"(w >> (4 * i)), "r"(0x000F000Fu), "r"(0x43004300u));
        out[i] = bf16x2_sub(v, zb);
    }
}

// Sum of the CSR row n against token m of x, in row order.
__device__ __forceinline__ float csr_row_dot(const GemvArgs& p, int n, int m) {
    const int j0 = p.row_ptr[n], j1 = p.row_ptr[n + 1];
    if (j0 < 0 || j1 < j0 || (long long)j1 > p.nnz) {
        record_error(p.err, kErrShape);
        return 0.0f;
    }
    const uint16_t* xr = p.x + (size_t)m * p.K;
    float acc = 0.0f;
#pragma unroll 4
    for (int j = j0; j < j1; ++j) {
        const int c = p.col_idx[j];
        if ((unsigned)c >= (unsigned)p.K) {
            record_error(p.err, kErrShape);
            continue;
        }
        acc = fmaf(fp16_bits_to_float(p.vals[j]), bf16_bits_to_float(xr[c]), acc);
    }
    return acc;
}

template <int NT>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_w4a16_kernel(const GemvArgs p) {
    __shared__ float part[kGemvRows * 16];  // [channel][token] fp32 partial sums of this K-slice

    const int G = p.K >> 7;
    const int rank = blockIdx.y;  // K-slice == rank in the (1, S, 1) cluster
    const int g0 = (int)((long long)G * rank / p.S);
    const int g1 = (int)((long long)G * (rank + 1) / p.S);
    const int nG = g1 - g0;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, t = lane & 3;
    const int r0 = blockIdx.x * kGemvRows + warp * 16 + gq;
    const int r1 = r0 + 8;
    const size_t Kw = (size_t)(p.K >> 3);

    const uint32_t* q0 = p.qw + (size_t)r0 * Kw + 4 * t + (size_t)g0 * 16;
    const uint32_t* q1 = p.qw + (size_t)r1 * Kw + 4 * t + (size_t)g0 * 16;
    const uint16_t* s0 = p.scales + (size_t)r0 * G + g0;
    const uint16_t* s1 = p.scales + (size_t)r1 * G + g0;
    const uint32_t* z0 = p.zeros + (size_t)r0 * (G >> 3);
    const uint32_t* z1 = p.zeros + (size_t)r1 * (G >> 3);

    bool tok_ok[NT];
    const uint16_t* xr[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        const int tok = gq + 8 * j;
        tok_ok[j] = tok < p.M;
        xr[j] = p.x + (size_t)(tok_ok[j] ? tok : 0) * p.K + 32 * t + (size_t)g0 * 128;
    }

    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[j][i] = 0.0f;

    // ring of weights in flight: 2 rows x 128 bits, plus scale bits and zero word per row
    uint4 wq[kGemvPF][2];
    uint32_t sz[kGemvPF][2];
    auto load_group = [&](int slot, int gi) {
        wq[slot][0] = ldg_stream(q0 + (size_t)gi * 16);
        wq[slot][1] = ldg_stream(q1 + (size_t)gi * 16);
        const int g = g0 + gi;
        const uint32_t zs = (uint32_t)(4 * (g & 7));
        sz[slot][0] = (uint32_t)s0[gi] | (((__ldg(z0 + (g >> 3)) >> zs) & 15u) << 16);
        sz[slot][1] = (uint32_t)s1[gi] | (((__ldg(z1 + (g >> 3)) >> zs) & 15u) << 16);
    };
    auto load_x = [&](uint4 (&xb)[NT][4], int gi) {
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int w = 0; w < 4; ++w)
                xb[j][w] = tok_ok[j] ? ldg_cached(xr[j] + (size_t)gi * 128 + 8 * w) : make_uint4(0, 0, 0, 0);
    };

#pragma unroll
    for (int s = 0; s < kGemvPF; ++s)
        if (s < nG) load_group(s, s);
    uint4 xc[NT][4];
    if (nG > 0) load_x(xc, 0);

    for (int i = 0; i < nG; i += kGemvPF) {
#pragma unroll
        for (int s = 0; s < kGemvPF; ++s) {
            const int gi = i + s;
            if (gi < nG) {
                uint4 xn[NT][4];
                if (gi + 1 < nG) load_x(xn, gi + 1);
                const uint4 a0 = wq[s][0], a1 = wq[s][1];
                const uint32_t sz0 = sz[s][0], sz1 = sz[s][1];
                if (gi + kGemvPF < nG) load_group(s, gi + kGemvPF);

                const uint32_t zv0 = sz0 >> 16, zv1 = sz1 >> 16;
                const uint32_t zb0 = 0x43004300u | zv0 | (zv0 << 16);
                const uint32_t zb1 = 0x43004300u | zv1 | (zv1 << 16);
                float d[NT][4];
#pragma unroll
                for (int j = 0; j < NT; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) d[j][e] = 0.0f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t pa0[4], pa1[4];
                    unpack_word(u4_get(a0, w), zb0, pa0);
                    unpack_word(u4_get(a1, w), zb1, pa1);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t A[4] = {pa0[2 * h], pa1[2 * h], pa0[2 * h + 1], pa1[2 * h + 1]};
#pragma unroll
                        for (int j = 0; j < NT; ++j) {
                            const uint32_t B[2] = {u4_get(xc[j][w], 2 * h), u4_get(xc[j][w], 2 * h + 1)};
                            mma_16816_bf16(d[j], A, B);
                        }
                    }
                }
                const float sc0 = fp16_bits_to_float((uint16_t)(sz0 & 0xFFFFu));
                const float sc1 = fp16_bits_to_float((uint16_t)(sz1 & 0xFFFFu));
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    acc[j][0] = fmaf(sc0, d[j][0], acc[j][0]);
                    acc[j][1] = fmaf(sc0, d[j][1], acc[j][1]);
                    acc[j][2] = fmaf(sc1, d[j][2], acc[j][2]);
                    acc[j][3] = fmaf(sc1, d[j][3], acc[j][3]);
                }
                if (gi + 1 < nG) {
#pragma unroll
                    for (int j = 0; j < NT; ++j)
#pragma unroll
                        for (int w = 0; w < 4; ++w) xc[j][w] = xn[j][w];
                }
            }
        }
    }

    // partial tile -> shared memory: part[channel][token]
    const int c0 = warp * 16 + gq, c1 = c0 + 8;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        const int tk = 8 * j + 2 * t;
        part[c0 * 16 + tk] = acc[j][0];
        part[c0 * 16 + tk + 1] = acc[j][1];
        part[c1 * 16 + tk] = acc[j][2];
        part[c1 * 16 + tk + 1] = acc[j][3];
    }
    cluster_sync_all();

    // this CTA's slice of the (token, channel) outputs, channel fastest for coalesced stores
    const int T = kGemvRows * p.M;
    const int o0 = (int)((long long)T * rank / p.S), o1 = (int)((long long)T * (rank + 1) / p.S);
    for (int o = o0 + (int)threadIdx.x; o < o1; o += kGemvWarps * 32) {
        const int m = o / kGemvRows, cl = o % kGemvRows;
        float v = 0.0f;
        for (int q = 0; q < p.S; ++q) v += ld_dsmem_f32(&part[cl * 16 + m], (uint32_t)q);
        const int n = blockIdx.x * kGemvRows + cl;
        if (p.row_ptr != nullptr) v += csr_row_dot(p, n, m);
        p.y[(size_t)m * p.N + n] = float_to_bf16_bits(v);
    }
    cluster_sync_all();
}

static int gemv_splits(int N, int K, int num_sms) {
    const int row_blocks = N / kGemvRows;
    const int G = K / 128;
    int S = 1;
    while (S < 8 && row_blocks * S < 4 * num_sms && G / (2 * S) >= 2) S *= 2;
    return S;
}

cudaError_t launch_gemv(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales, const uint32_t* zeros,
                        const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* vals, long long nnz,
                        uint16_t* y, int M, int N, int K, int num_sms, unsigned* err, cudaStream_t stream) {
    GemvArgs a{x, qweight, scales, zeros, row_ptr, col_idx, vals, nnz, y, M, N, K, 1, err};
    a.S = gemv_splits(N, K, num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(N / kGemvRows, a.S, 1);
    cfg.blockDim = dim3(kGemvWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = a.S;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (M <= 8) return cudaLaunchKernelEx(&cfg, gemv_w4a16_kernel<1>, a);
    return cudaLaunchKernelEx(&cfg, gemv_w4a16_kernel<2>, a);
}

}  // namespace w4a16
