// api.cu -- the extern "C" entry points of libw4a16.so: argument validation, dispatch on M,
// TMA tensor-map encoding and the per-device status word.  The operations and formats are
// documented in include/w4a16.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "w4a16.h"

namespace w4a16 {

// Problems found by kernels while they run (bit set of kErrValue / kErrShape / kErrTimeout).
__device__ unsigned g_device_status;

// Result of w4a16_selftest_quotient: mismatch count, then the first mismatch (b, a, got, want).
__device__ unsigned long long g_quotient_mismatches;
__device__ unsigned g_quotient_first[4];

// Scratch of w4a16_gemv_noalloc: the decode GEMV's row-block counters for N up to
// kNoallocMaxN, then its fp32 partial tiles for devices with up to kNoallocMaxSms SMs.  It is
// part of the loaded module: every GPU that loads the library holds it until the process
// exits, and every call of w4a16_gemv_noalloc on that GPU uses it.
constexpr int kNoallocMaxSms = 160;
constexpr int kNoallocMaxN = 131072;
constexpr size_t kNoallocCounterBytes = (size_t)(kNoallocMaxN / 128) * sizeof(unsigned);
constexpr size_t kNoallocCsrMax = 262144;  // N x M of a call with a CSR term
constexpr size_t kNoallocPartialBytes = (size_t)2 * kNoallocMaxSms * kGemvSlotFloats * sizeof(float);
constexpr size_t kNoallocScratchBytes = kNoallocCounterBytes + kNoallocPartialBytes + kNoallocCsrMax * sizeof(float);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxN = int64_t(1) << 22;
// The decode workspace of the public entry points starts with the row-block counters of the
// largest N, so that their place never depends on the call's sizes.
constexpr size_t kCounterRegionBytes = (size_t)(kMaxN / 128) * sizeof(unsigned);
constexpr int64_t kMaxK = int64_t(1) << 20;
constexpr int64_t kMaxM = int64_t(1) << 24;

struct DeviceInfo {
    bool ready = false;
    bool sm100 = false;
    int num_sms = 0;
    unsigned* status = nullptr;  // device address of g_device_status
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

w4a16_status device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W4A16_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return W4A16_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return W4A16_ERR_CUDA;
        d.sm100 = prop.major == 10 && prop.minor == 0;
        d.num_sms = prop.multiProcessorCount;
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_device_status) != cudaSuccess) return W4A16_ERR_CUDA;
        d.status = static_cast<unsigned*>(addr);
        d.ready = true;
    }
    *out = &d;
    return d.sm100 ? W4A16_OK : W4A16_ERR_UNSUPPORTED;
}

// Device address of g_noalloc_scratch for the current device.  In host code the array's
// name only stands in for the symbol; the address comes from cudaGetSymbolAddress, taken
// once per device with that device current.
w4a16_status noalloc_scratch(void** out) {
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W4A16_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return W4A16_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return W4A16_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return W4A16_OK;
}

w4a16_status encoder(EncodeTiledFn* out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return W4A16_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    *out = g_encode;
    return W4A16_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline w4a16_status from_cuda(cudaError_t e) { return e == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA; }

struct LinearArgs {
    const uint16_t* x;
    const uint32_t* qweight;
    const uint16_t* scales;
    const uint32_t* zeros;
    const int32_t* row_ptr = nullptr;
    const int32_t* col_idx = nullptr;
    const uint16_t* vals = nullptr;
    long long nnz = 0;
    uint16_t* y;
    int64_t M, N, K;
    int group_ratio = 1;  // group size / 128
    int bits = 4;         // code width: 4, or 3 (qweight [N][3K/32], decode GEMV only)
    float* partials = nullptr;   // the GEMV's scratch (gemv_partial_bytes)
    unsigned* counters = nullptr;  // zero when the call starts (gemv_counter_bytes)
    float* ysp = nullptr;          // the CSR term: decode [N][M], prefill [N][ld] fp32 (only with a CSR)
    uint16_t* xT = nullptr;        // with a CSR: x transposed, [K][ld] bf16 (decode: nullptr gathers from x)
};

w4a16_status validate_linear(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                             const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N,
                             int64_t K, LinearArgs* a) {
    if (!x || !qweight || !scales || !zeros || !y) return W4A16_ERR_NULL;
    if (M < 1 || M > kMaxM || N < 128 || N % 128 != 0 || N > kMaxN || K < 1024 || K % 1024 != 0 || K > kMaxK)
        return W4A16_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(qweight, 16) || !aligned(scales, 16) || !aligned(zeros, 16) || !aligned(y, 16))
        return W4A16_ERR_ALIGN;
    *a = LinearArgs{x, qweight, scales, zeros};
    a->y = y;
    a->M = M;
    a->N = N;
    a->K = K;
    if (outliers != nullptr) {
        if (outliers->nnz < 0 || outliers->nnz > INT_MAX) return W4A16_ERR_SHAPE;
        if (outliers->nnz > 0 || outliers->row_ptr != nullptr) {
            if (!outliers->row_ptr) return W4A16_ERR_NULL;
            if (outliers->nnz > 0 && (!outliers->col_idx || !outliers->values)) return W4A16_ERR_NULL;
            if (!aligned(outliers->row_ptr, 4) || (outliers->col_idx && !aligned(outliers->col_idx, 4)) ||
                (outliers->values && !aligned(outliers->values, 2)))
                return W4A16_ERR_ALIGN;
            a->row_ptr = outliers->row_ptr;
            a->col_idx = outliers->col_idx;
            a->vals = outliers->values;
            a->nnz = outliers->nnz;
        }
    }
    return W4A16_OK;
}


bool valid_schedule(int schedule) {
    return schedule == W4A16_GEMV_AUTO || schedule == W4A16_GEMV_STREAM_K || schedule == W4A16_GEMV_CLUSTER;
}

w4a16_status run_gemv(const LinearArgs& a, cudaStream_t stream, int schedule = W4A16_GEMV_AUTO) {
    if (!valid_schedule(schedule)) return W4A16_ERR_VALUE;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    if (a.K > gemv_max_k() || !gemv_fits((int)a.N, (int)a.K, d->num_sms)) return W4A16_ERR_UNSUPPORTED;
    const GemvPlan plan = gemv_plan((int)a.M, (int)a.N, (int)a.K, d->num_sms, schedule);
    if (plan.ctas < 1) return W4A16_ERR_UNSUPPORTED;
    if (a.partials == nullptr || a.counters == nullptr) return W4A16_ERR_NULL;
    GemvMaps maps;
    {
        EncodeTiledFn enc = nullptr;
        st = encoder(&enc);
        if (st != W4A16_OK) return st;
        // qweight: the words of a group (16 for 4-bit codes, 12 for 3-bit) x 128 rows x 4 groups
        const cuuint64_t gw = a.bits == 3 ? 12 : 16;  // words per row and group
        cuuint64_t dims[3] = {gw, (cuuint64_t)a.N, (cuuint64_t)(a.K / 128)};
        cuuint64_t strides[2] = {(cuuint64_t)(a.K / 128) * gw * 4, gw * 4};
        cuuint32_t box[3] = {(cuuint32_t)gw, 128, 4};
        cuuint32_t estr[3] = {1, 1, 1};
        if (enc(&maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(a.qweight), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4A16_ERR_CUDA;
    }
    const float* ysp = nullptr;
    if (a.row_ptr != nullptr) {
        // the sparse term first, into the workspace; the GEMV streams its weights meanwhile
        if (a.ysp == nullptr) return W4A16_ERR_NULL;
        // x transposed first when an entry's tokens would otherwise be several scattered loads
        uint16_t* xT = a.M > 2 ? a.xT : nullptr;
        st = from_cuda(launch_csr_rows(a.x, xT, a.row_ptr, a.col_idx, a.vals, a.nnz, (int)a.M, (int)a.N, (int)a.K,
                                       a.ysp, d->status, stream));
        if (st != W4A16_OK) return st;
        ysp = a.ysp;
    }
    return from_cuda(launch_gemv(maps, plan, a.group_ratio, a.x, a.scales, a.zeros, ysp, a.y, a.partials,
                                 a.counters, (int)a.M, (int)a.N, (int)a.K, d->status, stream, a.bits));
}

// The decode workspace of the public entry points:
//   [0, kCounterRegionBytes)   the GEMV's row-block counters (zero between calls);
//   then gemv_partial_bytes    its fp32 partial tiles;
//   then M x K bf16            x / s of w4a16_gemv_folded, rounded up to 256 bytes;
//   then N x M fp32            the CSR term, rounded up to 256 bytes;
//   then K x 16 bf16           x transposed for the CSR term, rounded up to 256 bytes.
// Only the last two parts depend on the call's sizes, and they lie after everything that must
// stay zero, so one zeroed workspace serves calls of any sizes in stream order.
size_t fold_region_bytes(int64_t M, int64_t K) { return ((size_t)M * (size_t)K * 2 + 255) / 256 * 256; }
size_t csr_region_bytes(int64_t M, int64_t N) { return ((size_t)M * (size_t)N * 4 + 255) / 256 * 256; }
size_t xt_region_bytes(int64_t K) { return ((size_t)K * 16 * 2 + 255) / 256 * 256; }

size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
    return kCounterRegionBytes + gemv_partial_bytes(num_sms) + fold_region_bytes(M, K) + csr_region_bytes(M, N) +
           xt_region_bytes(K);
}

// Checks the caller's decode workspace and points a at its parts; *fold = the x / s region.
w4a16_status take_decode_workspace(LinearArgs* a, void* workspace, size_t workspace_bytes, uint16_t** fold) {
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    if (workspace == nullptr) return W4A16_ERR_NULL;
    if (!aligned(workspace, 16)) return W4A16_ERR_ALIGN;
    if (workspace_bytes < decode_workspace_bytes(a->M, a->N, a->K, d->num_sms)) return W4A16_ERR_SHAPE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const size_t fold_off = kCounterRegionBytes + gemv_partial_bytes(d->num_sms);
    a->counters = reinterpret_cast<unsigned*>(ws);
    a->partials = reinterpret_cast<float*>(ws + kCounterRegionBytes);
    if (fold) *fold = reinterpret_cast<uint16_t*>(ws + fold_off);
    a->ysp = reinterpret_cast<float*>(ws + fold_off + fold_region_bytes(a->M, a->K));
    a->xT = reinterpret_cast<uint16_t*>(ws + fold_off + fold_region_bytes(a->M, a->K) + csr_region_bytes(a->M, a->N));
    return W4A16_OK;
}

// The prefill workspace (M > 16):
//   [0, kCounterRegionBytes)   the split-K tile counters (zero between calls; shared with the
//                              decode layout, which keeps its counters there too);
//   then plan.partial_bytes    fp32 partial tiles of split-K, rounded up to 256 bytes;
//   then K x ld bf16           x transposed (only with a CSR), rounded up to 256 bytes;
//   then N x ld fp32           the CSR term (only with a CSR); ld = csr_token_stride(M).
size_t up256(size_t b) { return (b + 255) / 256 * 256; }

size_t prefill_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms, bool csr) {
    const GemmPlan g = gemm_plan(M, N, K, num_sms);
    size_t b = kCounterRegionBytes + up256(g.partial_bytes);
    if (csr) {
        const size_t ld = (size_t)csr_token_stride(M);
        b += up256((size_t)K * ld * 2) + up256((size_t)N * ld * 4);
    }
    return b;
}

// The prefill GEMM.  workspace may be nullptr when there is no CSR term: the GEMM then runs
// without split-K.
w4a16_status run_gemm(const LinearArgs& a, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    EncodeTiledFn enc = nullptr;
    st = encoder(&enc);
    if (st != W4A16_OK) return st;
    const bool csr = a.row_ptr != nullptr;
    GemmPlan plan = gemm_plan(a.M, a.N, a.K, d->num_sms);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (ws == nullptr) {
        if (csr) return W4A16_ERR_NULL;
        plan = GemmPlan{plan.bn, 1, (int)(a.K / 128), 0};
    } else {
        if (!aligned(ws, 16)) return W4A16_ERR_ALIGN;
        if (workspace_bytes < prefill_workspace_bytes(a.M, a.N, a.K, d->num_sms, csr)) return W4A16_ERR_SHAPE;
    }
    const int bn = plan.bn;
    if ((a.M + bn - 1) / bn > 65535) return W4A16_ERR_UNSUPPORTED;  // grid y limit
    if (csr && ((int64_t)csr_token_stride(a.M) / 32 + 1 > 65535 ||
                a.N * ((a.M + 255) / 256) * 32 >= ((int64_t)1 << 31)))
        return W4A16_ERR_UNSUPPORTED;  // launch limits of the CSR kernels
    GemmMaps maps;
    {   // x: bf16 [M][K]; box 64 k (128 bytes) x bn tokens; 128-byte swizzle
        cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
        cuuint64_t strides[1] = {(cuuint64_t)a.K * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)bn};
        cuuint32_t estr[2] = {1, 1};
        if (enc(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.x), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4A16_ERR_CUDA;
    }
    {   // qweight: uint32 [N][K/8]; box 8 words (64 k) x 128 rows; 32-byte swizzle
        cuuint64_t dims[2] = {(cuuint64_t)(a.K / 8), (cuuint64_t)a.N};
        cuuint64_t strides[1] = {(cuuint64_t)(a.K / 8) * 4};
        cuuint32_t box[2] = {8, 128};
        cuuint32_t estr[2] = {1, 1};
        if (enc(&maps.qw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(a.qweight), dims, strides, box,
                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4A16_ERR_CUDA;
    }
    unsigned* counters = ws != nullptr ? reinterpret_cast<unsigned*>(ws) : nullptr;
    float* partials = ws != nullptr ? reinterpret_cast<float*>(ws + kCounterRegionBytes) : nullptr;
    const float* ysp = nullptr;
    const int ld = csr_token_stride(a.M);
    if (csr) {
        uint8_t* base = ws + kCounterRegionBytes + up256(plan.partial_bytes);
        uint16_t* xT = reinterpret_cast<uint16_t*>(base);
        float* yspw = reinterpret_cast<float*>(base + up256((size_t)a.K * ld * 2));
        st = from_cuda(launch_csr_prefill(a.x, a.row_ptr, a.col_idx, a.vals, a.nnz, (int)a.M, (int)a.N, (int)a.K, xT,
                                          yspw, d->status, stream));
        if (st != W4A16_OK) return st;
        ysp = yspw;
    }
    return from_cuda(launch_gemm(maps, plan, a.group_ratio, a.scales, a.zeros, ysp, ld, a.y, partials, counters,
                                 (int)a.M, (int)a.N, (int)a.K, d->status, stream));
}

// ---------------------------------------------------------------------------------------
// AWQ alpha search: layout of the workspace (every part 256-byte aligned).
struct SearchLayout {
    size_t qw, sc, z, s, xs, yq, yref, acc, gemv, total;
};

SearchLayout search_layout(int64_t M, int64_t N, int64_t K, int n_alpha, int num_sms) {
    auto up = [](size_t b) { return (b + 255) / 256 * 256; };
    SearchLayout L{};
    size_t off = 0;
    L.qw = off; off += up((size_t)N * K / 2);
    L.sc = off; off += up((size_t)N * (K / 128) * 2);
    L.z = off; off += up((size_t)N * (K / 1024) * 4);
    L.s = off; off += up((size_t)K * 4);
    L.xs = off; off += up((size_t)M * K * 2);
    L.yq = off; off += up((size_t)M * N * 2);
    L.yref = off; off += up((size_t)M * N * 4);
    L.acc = off; off += up((size_t)(n_alpha + 1) * 8);
    L.gemv = off; off += M <= 16 ? gemv_counter_bytes((int)N) + up(gemv_partial_bytes(num_sms)) : 0;
    L.total = off;
    return L;
}

constexpr int kMaxAlphas = 64;

}  // namespace
}  // namespace w4a16

using namespace w4a16;

extern "C" {

w4a16_status awq_quantize(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                          int64_t group_size, uint32_t* qweight, uint16_t* scales, uint32_t* zeros, float* s_out,
                          void* stream) {
    if (!W || !act_absmean || !qweight || !scales || !zeros) return W4A16_ERR_NULL;
    if (N < 8 || N % 8 != 0 || N > kMaxN || K < 1024 || K % 1024 != 0 || K > kMaxK) return W4A16_ERR_SHAPE;
    if (group_size < 128 || group_size > K || !quantize_group_size_ok((int)K, (int)group_size)) return W4A16_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(act_absmean, 16) || !aligned(qweight, 16) || !aligned(scales, 16) ||
        !aligned(zeros, 16) || (s_out && !aligned(s_out, 16)))
        return W4A16_ERR_ALIGN;
    if (!std::isfinite(alpha)) return W4A16_ERR_VALUE;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    return from_cuda(launch_awq_quantize(W, act_absmean, alpha, (int)N, (int)K, (int)group_size, qweight, scales,
                                         zeros, s_out, d->num_sms, d->status, static_cast<cudaStream_t>(stream)));
}

w4a16_status awq_quantize_g128(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                               uint32_t* qweight, uint16_t* scales, uint32_t* zeros, float* s_out, void* stream) {
    return awq_quantize(W, act_absmean, alpha, N, K, 128, qweight, scales, zeros, s_out, stream);
}

size_t w4a16_workspace_bytes_ex(int64_t M, int64_t N, int64_t K, int with_csr) {
    if (M < 1 || M > kMaxM || N < 128 || N % 128 != 0 || N > kMaxN || K < 1024 || K % 1024 != 0 || K > kMaxK)
        return 0;
    DeviceInfo* d = nullptr;
    if (device_info(&d) != W4A16_OK) return 0;
    if (M <= 16 && K <= gemv_max_k()) return decode_workspace_bytes(M, N, K, d->num_sms);
    return prefill_workspace_bytes(M, N, K, d->num_sms, with_csr != 0);
}

size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K) { return w4a16_workspace_bytes_ex(M, N, K, 1); }

w4a16_status w4a16_gemv(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales, const uint32_t* zeros,
                        const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N, int64_t K, void* workspace,
                        size_t workspace_bytes, void* stream) {
    LinearArgs a;
    w4a16_status st = validate_linear(x, qweight, scales, zeros, outliers, y, M, N, K, &a);
    if (st != W4A16_OK) return st;
    if (M > 16) return W4A16_ERR_SHAPE;
    st = take_decode_workspace(&a, workspace, workspace_bytes, nullptr);
    if (st != W4A16_OK) return st;
    return run_gemv(a, static_cast<cudaStream_t>(stream));
}

w4a16_status w4a16_gemv_ex(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                           const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N,
                           int64_t K, void* workspace, size_t workspace_bytes, int schedule, void* stream) {
    LinearArgs a;
    w4a16_status st = validate_linear(x, qweight, scales, zeros, outliers, y, M, N, K, &a);
    if (st != W4A16_OK) return st;
    if (M > 16) return W4A16_ERR_SHAPE;
    if (!valid_schedule(schedule)) return W4A16_ERR_VALUE;
    st = take_decode_workspace(&a, workspace, workspace_bytes, nullptr);
    if (st != W4A16_OK) return st;
    return run_gemv(a, static_cast<cudaStream_t>(stream), schedule);
}

w4a16_status awq_quantize3(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                           int64_t group_size, uint32_t* qweight3, uint16_t* scales, uint32_t* zeros, float* s_out,
                           void* stream) {
    if (!W || !act_absmean || !qweight3 || !scales || !zeros) return W4A16_ERR_NULL;
    if (N < 8 || N % 8 != 0 || N > kMaxN || K < 1024 || K % 1024 != 0 || K > kMaxK) return W4A16_ERR_SHAPE;
    if (group_size != 128 && group_size != 256 && group_size != 512 && group_size != 1024) return W4A16_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(act_absmean, 16) || !aligned(qweight3, 16) || !aligned(scales, 16) ||
        !aligned(zeros, 16) || (s_out && !aligned(s_out, 16)))
        return W4A16_ERR_ALIGN;
    if (!std::isfinite(alpha)) return W4A16_ERR_VALUE;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    return from_cuda(launch_awq_quantize(W, act_absmean, alpha, (int)N, (int)K, (int)group_size, qweight3, scales,
                                         zeros, s_out, d->num_sms, d->status, static_cast<cudaStream_t>(stream), 3));
}

w4a16_status awq_quantize_nvfp4(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                                uint32_t* qweight, uint8_t* scales8, float* gscale, float* s_out, void* stream) {
    if (!W || !act_absmean || !qweight || !scales8 || !gscale || !s_out) return W4A16_ERR_NULL;
    if (N < 8 || N % 8 != 0 || N > kMaxN || K < 16 || K % 16 != 0 || K > kMaxK) return W4A16_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(act_absmean, 16) || !aligned(qweight, 16) || !aligned(gscale, 4) ||
        !aligned(s_out, 16))
        return W4A16_ERR_ALIGN;
    if (!std::isfinite(alpha)) return W4A16_ERR_VALUE;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    return from_cuda(launch_awq_quantize_nvfp4(W, act_absmean, alpha, (int)N, (int)K, qweight, scales8, gscale, s_out,
                                               d->num_sms, d->status, static_cast<cudaStream_t>(stream)));
}

w4a16_status w4a16_gemv_nvfp4(const uint16_t* x, const uint32_t* qweight, const uint8_t* scales8,
                              const float* gscale, uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream) {
    if (!x || !qweight || !scales8 || !gscale || !y) return W4A16_ERR_NULL;
    if (M < 1 || M > 16 || N < 16 || N % 16 != 0 || N > kMaxN || K < 16 || K % 16 != 0 || K > kMaxK)
        return W4A16_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(qweight, 16) || !aligned(gscale, 4) || !aligned(y, 2)) return W4A16_ERR_ALIGN;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    return from_cuda(launch_gemv_nvfp4(x, qweight, scales8, gscale, y, (int)M, (int)N, (int)K,
                                       static_cast<cudaStream_t>(stream)));
}

w4a16_status w3a16_gemv(const uint16_t* x, const uint32_t* qweight3, const uint16_t* scales, const uint32_t* zeros,
                        const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N, int64_t K, int64_t group_size,
                        void* workspace, size_t workspace_bytes, int schedule, void* stream) {
    LinearArgs a;
    w4a16_status st = validate_linear(x, qweight3, scales, zeros, outliers, y, M, N, K, &a);
    if (st != W4A16_OK) return st;
    if (M > 16 || K > gemv_max_k()) return W4A16_ERR_SHAPE;
    if (group_size < 128 || group_size % 128 != 0 || group_size > K || K % group_size != 0) return W4A16_ERR_SHAPE;
    if (!valid_schedule(schedule)) return W4A16_ERR_VALUE;
    a.group_ratio = (int)(group_size / 128);
    a.bits = 3;
    st = take_decode_workspace(&a, workspace, workspace_bytes, nullptr);
    if (st != W4A16_OK) return st;
    return run_gemv(a, static_cast<cudaStream_t>(stream), schedule);
}

w4a16_status w4a16_gemv_folded(const uint16_t* x, const float* s, const uint32_t* qweight, const uint16_t* scales,
                               const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N,
                               int64_t K, int64_t group_size, void* workspace, size_t workspace_bytes, int schedule,
                               void* stream) {
    LinearArgs a;
    w4a16_status st = validate_linear(x, qweight, scales, zeros, outliers, y, M, N, K, &a);
    if (st != W4A16_OK) return st;
    if (M > 16) return W4A16_ERR_SHAPE;
    if (group_size < 128 || group_size % 128 != 0 || group_size > K || K % group_size != 0) return W4A16_ERR_SHAPE;
    if (!valid_schedule(schedule)) return W4A16_ERR_VALUE;
    if (s != nullptr && !aligned(s, 16)) return W4A16_ERR_ALIGN;
    a.group_ratio = (int)(group_size / 128);
    uint16_t* xf = nullptr;
    st = take_decode_workspace(&a, workspace, workspace_bytes, &xf);
    if (st != W4A16_OK) return st;
    if (s != nullptr) {
        // x' = x / s goes to the workspace's fold region, once per call; the GEMV then streams
        // its weights while the fold runs and reads x' when the fold has finished
        st = from_cuda(launch_search_fold(x, s, xf, (int)M, (int)K, static_cast<cudaStream_t>(stream)));
        if (st != W4A16_OK) return st;
        a.x = xf;
    }
    return run_gemv(a, static_cast<cudaStream_t>(stream), schedule);
}

w4a16_status w4a16_gemm_plan(int64_t M, int64_t N, int64_t K, int num_sms, int* token_tile, int* splits,
                             int* slices_per_split, size_t* partial_bytes) {
    if (M < 1 || M > kMaxM || N < 128 || N % 128 != 0 || N > kMaxN || K < 1024 || K % 1024 != 0 || K > kMaxK)
        return W4A16_ERR_SHAPE;
    if (num_sms < 1 || num_sms > 4096) return W4A16_ERR_VALUE;
    const GemmPlan g = gemm_plan(M, N, K, num_sms);
    if (token_tile) *token_tile = g.bn;
    if (splits) *splits = g.splits;
    if (slices_per_split) *slices_per_split = g.slices;
    if (partial_bytes) *partial_bytes = g.partial_bytes;
    return W4A16_OK;
}

w4a16_status w4a16_gemv_plan(int64_t M, int64_t N, int64_t K, int schedule, int* resolved, int* cluster_size,
                             int* ctas) {
    if (M < 1 || M > 16 || N < 128 || N % 128 != 0 || N > kMaxN || K < 1024 || K % 1024 != 0 || K > kMaxK)
        return W4A16_ERR_SHAPE;
    if (!valid_schedule(schedule)) return W4A16_ERR_VALUE;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    if (K > gemv_max_k() || !gemv_fits((int)N, (int)K, d->num_sms)) return W4A16_ERR_UNSUPPORTED;
    const GemvPlan plan = gemv_plan((int)M, (int)N, (int)K, d->num_sms, schedule);
    if (plan.ctas < 1) return W4A16_ERR_UNSUPPORTED;
    if (resolved) *resolved = plan.schedule;
    if (cluster_size) *cluster_size = plan.cluster;
    if (ctas) *ctas = plan.ctas;
    return W4A16_OK;
}

w4a16_status w4a16_gemm(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales, const uint32_t* zeros,
                        const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N, int64_t K, void* workspace,
                        size_t workspace_bytes, void* stream) {
    LinearArgs a;
    w4a16_status st = validate_linear(x, qweight, scales, zeros, outliers, y, M, N, K, &a);
    if (st != W4A16_OK) return st;
    return run_gemm(a, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

w4a16_status w4a16_linear(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                          const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N,
                          int64_t K, void* workspace, size_t workspace_bytes, void* stream) {
    LinearArgs a;
    w4a16_status st = validate_linear(x, qweight, scales, zeros, outliers, y, M, N, K, &a);
    if (st != W4A16_OK) return st;
    const bool decode = M <= 16 && K <= gemv_max_k();
    if (!decode) return run_gemm(a, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
    st = take_decode_workspace(&a, workspace, workspace_bytes, nullptr);
    if (st != W4A16_OK) return st;
    return run_gemv(a, static_cast<cudaStream_t>(stream));
}

w4a16_status w4a16_linear_ex(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                             const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N,
                             int64_t K, int64_t group_size, void* workspace, size_t workspace_bytes, int schedule,
                             void* stream) {
    LinearArgs a;
    w4a16_status st = validate_linear(x, qweight, scales, zeros, outliers, y, M, N, K, &a);
    if (st != W4A16_OK) return st;
    if (group_size < 128 || group_size % 128 != 0 || group_size > K || K % group_size != 0) return W4A16_ERR_SHAPE;
    if (!valid_schedule(schedule)) return W4A16_ERR_VALUE;
    a.group_ratio = (int)(group_size / 128);
    const bool decode = M <= 16 && K <= gemv_max_k();
    if (!decode) return run_gemm(a, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
    st = take_decode_workspace(&a, workspace, workspace_bytes, nullptr);
    if (st != W4A16_OK) return st;
    return run_gemv(a, static_cast<cudaStream_t>(stream), schedule);
}

w4a16_status w4a16_gemv_noalloc(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                                const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y, int64_t M,
                                int64_t N, int64_t K, void* stream) {
    LinearArgs a;
    w4a16_status st = validate_linear(x, qweight, scales, zeros, outliers, y, M, N, K, &a);
    if (st != W4A16_OK) return st;
    if (M > 16) return W4A16_ERR_SHAPE;
    if (N > kNoallocMaxN) return W4A16_ERR_UNSUPPORTED;
    if (a.row_ptr != nullptr && (size_t)(N * M) > kNoallocCsrMax) return W4A16_ERR_UNSUPPORTED;
    DeviceInfo* d = nullptr;
    st = device_info(&d);
    if (st != W4A16_OK) return st;
    if (d->num_sms > kNoallocMaxSms) return W4A16_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != W4A16_OK) return st;
    // The row-block counters must start at zero.  A completed call leaves them zero, but one
    // that failed may not have, so clear them.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(scratch, 0, (size_t)(N / 128) * sizeof(unsigned), s) != cudaSuccess) return W4A16_ERR_CUDA;
    a.counters = static_cast<unsigned*>(scratch);
    a.partials = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + kNoallocCounterBytes);
    a.ysp = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + kNoallocCounterBytes + kNoallocPartialBytes);
    return run_gemv(a, s);
}

size_t awq_split_outliers_workspace_bytes(int64_t N, int64_t K) {
    if (N < 1 || K < 1) return 0;
    return split_workspace_bytes(N);
}

w4a16_status awq_split_outliers(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                                int64_t nnz, float* W_dense, int32_t* row_ptr, int32_t* col_idx, uint16_t* values,
                                void* workspace, size_t workspace_bytes, void* stream) {
    if (!W || !act_absmean || !W_dense || !row_ptr) return W4A16_ERR_NULL;
    if (N < 1 || K < 1 || nnz < 0 || nnz > N * K || (uint64_t)N * (uint64_t)K >= (1ull << 32) || nnz > 0x7FFFFFFFll)
        return W4A16_ERR_SHAPE;
    if (!std::isfinite(alpha) || alpha < 0.0f) return W4A16_ERR_VALUE;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (nnz == 0) {  // nothing moves: W_dense = W, an empty CSR
        if (cudaMemcpyAsync(W_dense, W, sizeof(float) * (size_t)(N * K), cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemsetAsync(row_ptr, 0, sizeof(int32_t) * (size_t)(N + 1), s) != cudaSuccess)
            return W4A16_ERR_CUDA;
        return W4A16_OK;
    }
    if (!col_idx || !values || !workspace) return W4A16_ERR_NULL;
    if (!aligned(workspace, 256)) return W4A16_ERR_ALIGN;
    if (workspace_bytes < split_workspace_bytes(N)) return W4A16_ERR_SHAPE;
    return from_cuda(launch_split_outliers(W, act_absmean, alpha, (uint32_t)N, (uint32_t)K, (uint32_t)nnz, W_dense,
                                           row_ptr, col_idx, values, workspace, d->num_sms, d->status, s));
}

size_t awq_search_alpha_workspace_bytes(int64_t M, int64_t N, int64_t K, int n_alpha) {
    if (M < 1 || M > 65535 || N < 128 || N % 128 != 0 || N > kMaxN || K < 1024 || K % 1024 != 0 || K > kMaxK ||
        n_alpha < 1 || n_alpha > kMaxAlphas)
        return 0;
    DeviceInfo* d = nullptr;
    if (device_info(&d) != W4A16_OK) return 0;
    return search_layout(M, N, K, n_alpha, d->num_sms).total;
}

w4a16_status awq_search_alpha(const float* W, const float* act_absmean, const uint16_t* x_calib, int64_t M,
                              int64_t N, int64_t K, const float* alphas, int n_alpha, float* errors, int* best,
                              void* workspace, size_t workspace_bytes, void* stream) {
    if (!W || !act_absmean || !x_calib || !alphas || !errors || !best || !workspace) return W4A16_ERR_NULL;
    if (M < 1 || M > 65535 || N < 128 || N % 128 != 0 || N > kMaxN || K < 1024 || K % 1024 != 0 || K > kMaxK ||
        n_alpha < 1 || n_alpha > kMaxAlphas)
        return W4A16_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(act_absmean, 16) || !aligned(x_calib, 16) || !aligned(workspace, 256))
        return W4A16_ERR_ALIGN;
    for (int i = 0; i < n_alpha; ++i)
        if (!std::isfinite(alphas[i]) || alphas[i] < 0.0f) return W4A16_ERR_VALUE;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    const SearchLayout L = search_layout(M, N, K, n_alpha, d->num_sms);
    if (workspace_bytes < L.total) return W4A16_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint32_t* qw = reinterpret_cast<uint32_t*>(ws + L.qw);
    uint16_t* sc = reinterpret_cast<uint16_t*>(ws + L.sc);
    uint32_t* z = reinterpret_cast<uint32_t*>(ws + L.z);
    float* sv = reinterpret_cast<float*>(ws + L.s);
    uint16_t* xs = reinterpret_cast<uint16_t*>(ws + L.xs);
    uint16_t* yq = reinterpret_cast<uint16_t*>(ws + L.yq);
    float* yref = reinterpret_cast<float*>(ws + L.yref);
    double* acc = reinterpret_cast<double*>(ws + L.acc);  // [0] = sum yref^2, [1 + a] = error sums
    // the error sums start at zero; so does the GEMV's workspace
    if (cudaMemsetAsync(acc, 0, (size_t)(n_alpha + 1) * 8, s) != cudaSuccess) return W4A16_ERR_CUDA;
    if (M <= 16 && cudaMemsetAsync(ws + L.gemv, 0, L.total - L.gemv, s) != cudaSuccess) return W4A16_ERR_CUDA;
    st = from_cuda(launch_search_ref(x_calib, W, yref, (int)M, (int)N, (int)K, s));
    for (int i = 0; i < n_alpha && st == W4A16_OK; ++i) {
        st = from_cuda(launch_awq_quantize(W, act_absmean, alphas[i], (int)N, (int)K, 128, qw, sc, z, sv, d->num_sms,
                                           d->status, s));
        if (st != W4A16_OK) break;
        st = from_cuda(launch_search_fold(x_calib, sv, xs, (int)M, (int)K, s));
        if (st != W4A16_OK) break;
        LinearArgs a;
        st = validate_linear(xs, qw, sc, z, nullptr, yq, M, N, K, &a);
        if (st != W4A16_OK) break;
        if (M <= 16) {
            a.counters = reinterpret_cast<unsigned*>(ws + L.gemv);
            a.partials = reinterpret_cast<float*>(ws + L.gemv + gemv_counter_bytes((int)N));
            st = run_gemv(a, s);
        } else {
            st = run_gemm(a, nullptr, 0, s);
        }
        if (st != W4A16_OK) break;
        st = from_cuda(launch_search_err(yq, yref, (long long)(M * N), acc + 1 + i, i == 0 ? acc : nullptr,
                                         d->num_sms, s));
    }
    if (st != W4A16_OK) return st;
    double host[kMaxAlphas + 1];
    if (cudaMemcpyAsync(host, acc, (size_t)(n_alpha + 1) * 8, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return W4A16_ERR_CUDA;
    // any problem a kernel recorded (bad values, a timeout) makes the result invalid
    st = w4a16_check_device_status(stream);
    if (st != W4A16_OK) return st;
    int bi = 0;
    for (int i = 0; i < n_alpha; ++i) {
        errors[i] = (float)(host[0] > 0.0 ? host[1 + i] / host[0] : host[1 + i]);
        if (errors[i] < errors[bi]) bi = i;
    }
    *best = bi;
    return W4A16_OK;
}

w4a16_status awq_fold_activations(const uint16_t* x, const float* s, uint16_t* x_out, int64_t M, int64_t K,
                                  void* stream) {
    if (!x || !s || !x_out) return W4A16_ERR_NULL;
    if (M < 1 || M > 65535 || K < 1 || K > kMaxK) return W4A16_ERR_SHAPE;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    return from_cuda(launch_search_fold(x, s, x_out, (int)M, (int)K, static_cast<cudaStream_t>(stream)));
}

w4a16_status w4a16_selftest_quotient(uint64_t* mismatches, uint32_t first[4], void* stream) {
    if (!mismatches) return W4A16_ERR_NULL;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    void* cnt = nullptr;
    void* fst = nullptr;
    if (cudaGetSymbolAddress(&cnt, g_quotient_mismatches) != cudaSuccess ||
        cudaGetSymbolAddress(&fst, g_quotient_first) != cudaSuccess)
        return W4A16_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned long long host_count = 0;
    unsigned host_first[4] = {0, 0, 0, 0};
    if (cudaMemsetAsync(cnt, 0, sizeof(unsigned long long), s) != cudaSuccess ||
        cudaMemsetAsync(fst, 0, sizeof(host_first), s) != cudaSuccess)
        return W4A16_ERR_CUDA;
    st = from_cuda(launch_selftest_quotient(static_cast<unsigned long long*>(cnt), static_cast<unsigned*>(fst), s));
    if (st != W4A16_OK) return st;
    if (cudaMemcpyAsync(&host_count, cnt, sizeof(host_count), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyAsync(host_first, fst, sizeof(host_first), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return W4A16_ERR_CUDA;
    *mismatches = host_count;
    if (first)
        for (int i = 0; i < 4; ++i) first[i] = host_first[i];
    return W4A16_OK;
}

w4a16_status w4a16_selftest_timeout(int64_t limit_ns, void* stream) {
    if (limit_ns < 0 || limit_ns > 10000000000ll) return W4A16_ERR_VALUE;
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    return from_cuda(launch_selftest_timeout((unsigned long long)limit_ns, d->status, static_cast<cudaStream_t>(stream)));
}

w4a16_status w4a16_check_device_status(void* stream) {
    DeviceInfo* d = nullptr;
    w4a16_status st = device_info(&d);
    if (st != W4A16_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return W4A16_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, d->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return W4A16_ERR_CUDA;
    if (v != 0 && cudaMemset(d->status, 0, sizeof(v)) != cudaSuccess) return W4A16_ERR_CUDA;
    if (v & kErrTimeout) return W4A16_ERR_TIMEOUT;
    if (v & kErrShape) return W4A16_ERR_SHAPE;
    if (v & kErrValue) return W4A16_ERR_VALUE;
    return W4A16_OK;
}

const char* w4a16_status_string(w4a16_status status) {
    switch (status) {
        case W4A16_OK: return "ok";
        case W4A16_ERR_NULL: return "null pointer";
        case W4A16_ERR_SHAPE: return "bad shape or CSR structure";
        case W4A16_ERR_ALIGN: return "misaligned pointer";
        case W4A16_ERR_VALUE: return "non-finite or out-of-range value";
        case W4A16_ERR_CUDA: return "CUDA runtime error";
        case W4A16_ERR_TIMEOUT: return "kernel pipeline wait timed out";
        case W4A16_ERR_UNSUPPORTED: return "unsupported device or size";
    }
    return "unknown status";
}

int w4a16_version(void) { return 100; }

}  // extern "C"
