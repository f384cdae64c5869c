/*
 * w4a16.h -- C ABI of the B200 (sm_100a) W4A16 quantized-linear library, libw4a16.so.
 *
 * The operations are those of activation-aware weight quantization (AWQ) and of the
 * dense-and-sparse decomposition of SqueezeLLM:
 *   - awq_quantize_g128: per-input-channel activation-aware scaling, then asymmetric
 *     uint4 round-to-nearest in groups of 128 along K, packed 8 codes per 32-bit word
 *     [AWQ (MLSys 2024) translation, sections 2, 3.1 and 3.2; DeepCompressor README,
 *     perplexity table row "W4A16 g128"; AWQ translation section 1 for TinyChat's
 *     4-bit packing];
 *   - w4a16_linear / w4a16_gemv / w4a16_gemm: y = x . dequant(Wq)^T (+ x . W_sparse^T)
 *     with the weights dequantized on the fly [AWQ translation, section 1: TinyChat's
 *     on-the-fly dequantization; SqueezeLLM article, sections 2.2 and 2.3: W x =
 *     W_dense x + W_sparse x, the sparse part an fp16 matrix].
 *
 * Conventions for every entry point
 *   - Tensor arguments are DEVICE pointers, allocated and owned by the caller.  So is
 *     the decode path's workspace (see w4a16_workspace_bytes).  The library keeps no
 *     pointer after a call returns.  It allocates no device memory at run time: its only
 *     device memory is static, part of the loaded module on every GPU that loads it (a
 *     status word, the scratch of w4a16_gemv_noalloc, the self-test's counters).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream).  The return value covers argument validation and the kernel launch.
 *     Problems found while a kernel runs are reported later: the kernel records them in
 *     the device status word, and w4a16_check_device_status() returns them.  These
 *     problems are non-finite inputs, fp16 overflow, CSR indices out of range, and a
 *     pipeline wait that ran out.  When a call fails, its outputs are unspecified.
 *   - Element types are passed as raw bits: bf16 and fp16 as uint16_t, fp32 as float.
 *   - Shapes: W is [N][K] (out x in), x is [M][K], y is [M][N], all row-major and dense.
 *     K must be a positive multiple of 1024 and N a positive multiple of 128 (the quantizer
 *     accepts any positive multiple of 8, so zero points fill whole words).  Every pointer
 *     must be 16-byte aligned, except the CSR arrays, which need only natural alignment.
 *
 * Packed weight format (shared with any reader of the quantized weights):
 *   qweight[n][k/8]  uint32.  Nibble j (bits 4j..4j+3) holds the code of element
 *                    k = 8*(k/8) + ORDER[j], ORDER = {0,2,4,6,1,3,5,7}.  Hence
 *                    (word >> 4i) & 0x000F000F holds elements 2i and 2i+1 in its low
 *                    and high 16-bit halves.
 *   scales[g][n]     fp16 bits, g = k/128 (group-major).
 *   zeros[g][n/8]    uint32.  Nibble j holds the zero point of row 8*(n/8) + j in group g.
 *   Dequantized weight: w = (q - z) * scale.  This is exact in fp32.
 *   Group-major parameters put the scales and zero points of consecutive output channels
 *   of one group next to each other, so a kernel fetches a tile's parameters as one
 *   contiguous run.
 *
 * CSR outlier matrix (w4a16_csr), in the same scaled space as the packed weights:
 *   row_ptr[N+1] int32, row_ptr[0] = 0, row_ptr[N] = nnz, non-decreasing;
 *   col_idx[nnz] int32, strictly ascending within a row, each in [0, K);
 *   values[nnz]  fp16 bits.
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4A16_OK = 0,
    W4A16_ERR_NULL = 1,        /* a required pointer is NULL */
    W4A16_ERR_SHAPE = 2,       /* bad size (M, N, K, nnz) or CSR structure */
    W4A16_ERR_ALIGN = 3,       /* a pointer is not aligned as required */
    W4A16_ERR_VALUE = 4,       /* non-finite input, negative act_absmean, fp16 overflow */
    W4A16_ERR_CUDA = 5,        /* a CUDA runtime call failed */
    W4A16_ERR_TIMEOUT = 6,     /* a kernel's bounded pipeline wait ran out */
    W4A16_ERR_UNSUPPORTED = 7  /* no sm_100 device, or a size beyond a documented limit */
} w4a16_status;

typedef struct {
    const int32_t* row_ptr;  /* [N+1] device */
    const int32_t* col_idx;  /* [nnz] device, ascending within each row */
    const uint16_t* values;  /* [nnz] device, fp16 bits */
    int64_t nnz;
} w4a16_csr;

/*
 * awq_quantize_g128 -- activation-aware scaling + group-wise uint4 RTN + packing.
 *   [AWQ translation, 3.2 (per-channel scaling); 2 (RTN); DeepCompressor "W4A16 g128"]
 *
 *   s_k      = max( float(pow(double(act_absmean[k]), double(alpha))), 1e-4 )
 *   w'       = float(W[n][k] * s_k)
 *   per group of 128 along K:
 *     scale  = fp16_rne( max((max w' - min w') / 15, 1e-5) )
 *     z      = clamp(rint(-min w' / scale), 0, 15)
 *     q      = clamp(rint(w' / scale) + z, 0, 15)       (rint: ties to even)
 *   Every float step is a single IEEE-754 operation with round-to-nearest-even.  The
 *   outputs are therefore bit-reproducible by any correct implementation of these steps.
 *
 *   W            [N][K] fp32, device.
 *   act_absmean  [K] fp32, device: mean |x| per input channel over calibration data.
 *                Each value must be finite and >= 0.
 *   alpha        finite exponent (AWQ searches it in [0, 1]).
 *   qweight      [N][K/8] uint32, device, output.
 *   scales       [K/128][N] fp16 bits, device, output.
 *   zeros        [K/128][N/8] uint32, device, output.
 *   s_out        [K] fp32, device, output, may be NULL.  The caller divides the layer's
 *                input by s (x' = x / s) before calling w4a16_linear.
 *   Errors: NULL, SHAPE, ALIGN and VALUE (non-finite alpha) when called.  Later, through
 *   w4a16_check_device_status: VALUE for a non-finite W, s or w', a negative
 *   act_absmean, or a scale that overflows fp16.
 */
w4a16_status awq_quantize_g128(const float* W, const float* act_absmean, float alpha, int64_t N,
                               int64_t K, uint32_t* qweight, uint16_t* scales, uint32_t* zeros,
                               float* s_out, void* stream);

/*
 * awq_quantize -- awq_quantize_g128 with groups of group_size weights along K instead of 128
 * [SqueezeLLM article, 4.1: the group size option, one group per row by default].
 *   group_size   128, 256, 512, 1024, or a multiple of 1024 that divides K and is at most
 *                32768.  group_size = K gives one scale and zero point per output channel.
 *   scales       [K/group_size][N] fp16 bits; zeros [K/group_size][N/8] uint32.
 *   Everything else, including the arithmetic per group, is as for awq_quantize_g128.
 *   Groups above 1024 are read twice from device memory: once for their range, once to
 *   quantize.  Errors: as awq_quantize_g128, plus SHAPE for an unsupported group_size.
 */
w4a16_status awq_quantize(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                          int64_t group_size, uint32_t* qweight, uint16_t* scales, uint32_t* zeros,
                          float* s_out, void* stream);

/*
 * Workspace.  A caller-provided device buffer holds the library's scratch:
 *   - Decode path (M <= 16).  The GEMV splits the output row blocks evenly over a
 *     persistent grid.  Row blocks shared by two or more CTAs are combined through fp32
 *     partial tiles and per-row-block counters; w4a16_gemv_folded also writes its x / s
 *     there, and a CSR term goes there as N x M fp32 (with x transposed beside it).
 *   - Prefill path (the GEMM).  When the output tiles alone would leave SMs idle, the GEMM
 *     splits K over several CTAs per tile; their fp32 partial tiles and per-tile counters
 *     live in the workspace.  With a CSR term, x transposed (K x M' bf16) and the term
 *     itself (N x M' fp32) go there too, M' = M rounded up to a multiple of 8.
 *   - It must hold at least w4a16_workspace_bytes_ex(M, N, K, with_csr) bytes (with_csr: 1
 *     when a CSR term is passed) and be 16-byte aligned.  w4a16_workspace_bytes(M, N, K) is
 *     the size with a CSR term, enough either way.
 *   - It must be zero-filled before its first use.  Every call that completes leaves the
 *     parts that must start at zero zero-filled again, whatever its sizes, so one workspace
 *     of the largest size needed serves any number of calls of any sizes in stream order.
 *   - Calls that may run at the same time (on different streams without ordering between
 *     them) need different workspaces.
 *   - After a call reports W4A16_ERR_TIMEOUT, zero the workspace again before reusing it.
 * Both functions return the size for the CURRENT device (it depends on the number of SMs),
 * or 0 for invalid sizes.  Decode: 128 KiB of counters, 16 KiB of partial tiles per SM,
 * M x K bf16 for the folded activations, N x M fp32 for the CSR term and K x 16 bf16 for
 * the activations transposed for it.  Prefill: 128 KiB
 * of counters, the split-K partial tiles (none for grids that fill the GPU, else about
 * splits x M x N x 4 bytes, at most 64 MiB), then the CSR parts above.  Each part is
 * rounded up to 256 bytes.
 */
size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K);
size_t w4a16_workspace_bytes_ex(int64_t M, int64_t N, int64_t K, int with_csr);

/*
 * w4a16_linear -- y = bf16_rne( x . dequant(Q)^T + x . W_sparse^T ), fp32 accumulation.
 *   [AWQ translation, 1 (TinyChat on-the-fly dequantization); SqueezeLLM article 2.3]
 *
 *   x        [M][K] bf16 bits, device.  This is the layer input already divided by s.
 *   qweight, scales, zeros: the packed weights, laid out as above.
 *   outliers host pointer to a w4a16_csr whose arrays are on the device, or NULL when
 *            there is no sparse term.  nnz may be 0.
 *   y        [M][N] bf16 bits, device, output.  It must not overlap any input.
 *   workspace, workspace_bytes: see above.  Required when M <= 16 or when a CSR is given.
 *            Otherwise it may be NULL, and the GEMM then does not split K.
 *   M >= 1.  M <= 16 runs the decode GEMV; larger M runs the tensor-core GEMM.
 *   With a CSR, small kernels first write the sparse term x . W_sparse^T in fp32 to the
 *   workspace (fp16 values times bf16 activations, fp32 sums, entries in CSR order), while
 *   the GEMV or GEMM already runs its main loop; its epilogue adds the term to each fp32
 *   output before the one rounding to bf16.
 *   Errors: NULL, SHAPE, ALIGN and UNSUPPORTED when called (SHAPE also for a workspace that
 *   is too small).  Later: SHAPE if a CSR index is out of range (that entry is skipped),
 *   TIMEOUT if a pipeline wait runs out.
 */
w4a16_status w4a16_linear(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                          const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y,
                          int64_t M, int64_t N, int64_t K, void* workspace,
                          size_t workspace_bytes, void* stream);

/* w4a16_gemv -- the decode path of w4a16_linear, restricted to 1 <= M <= 16
 * (W4A16_ERR_SHAPE otherwise).  Arguments and result are as for w4a16_linear; the
 * workspace is required.
 * Launch overlap: the kernel may start fetching its packed weights, scales and zeros
 * before the previous kernel on the stream has finished.  It reads x, touches the
 * workspace and writes y only after that kernel has finished.  The output y of an earlier
 * library call on the same stream must therefore not alias this call's qweight, scales,
 * zeros or CSR. */
w4a16_status w4a16_gemv(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                        const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y,
                        int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * Schedules of the decode GEMV.  Both stream every packed weight byte once; they differ in
 * how the work is spread over the SMs and how row blocks split along K are summed.
 *   STREAM_K  one persistent CTA per SM takes an equal contiguous range of (row block,
 *             512-k) units.  A row block split between CTAs is completed through fp32
 *             partial tiles and a counter in the workspace; the last CTA to finish sums.
 *   CLUSTER   thread-block clusters of 2 to 8 CTAs.  Each cluster takes whole row blocks;
 *             its CTAs split every row block along K and sum their tiles through
 *             distributed shared memory.  Suits shapes with few row blocks (N / 128 well
 *             under the SM count), where the workspace exchange would dominate.
 *   AUTO      the library's choice for the shape and the current device.
 * Results of different schedules may differ in the last bit (summation order); a given
 * schedule gives the same bits on every call.
 */
typedef enum {
    W4A16_GEMV_AUTO = 0,
    W4A16_GEMV_STREAM_K = 1,
    W4A16_GEMV_CLUSTER = 2
} w4a16_gemv_schedule;

/* w4a16_gemv_ex -- w4a16_gemv with an explicit schedule (w4a16_gemv uses AUTO).  The
 * workspace is required for every schedule.  UNSUPPORTED when the schedule cannot run this
 * shape on the current device (CLUSTER needs K >= 1024 and a cluster launch the device
 * can hold). */
w4a16_status w4a16_gemv_ex(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                           const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y,
                           int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                           int schedule, void* stream);

/* w4a16_gemm_plan -- the launch that the prefill GEMM would make on a device with num_sms
 * SMs (host arithmetic only, no device needed): the token tile (32, 64, 128 or 256), the CTAs
 * per output tile along K (splits, 1 = no split-K), the 128-k slices each of them takes, and
 * the bytes of fp32 partial tiles split-K needs in the workspace.  Errors: SHAPE for sizes
 * the GEMM does not take, VALUE for num_sms outside 1..4096. */
w4a16_status w4a16_gemm_plan(int64_t M, int64_t N, int64_t K, int num_sms, int* token_tile, int* splits,
                             int* slices_per_split, size_t* partial_bytes);

/* w4a16_gemv_plan -- the launch that w4a16_gemv_ex(schedule) would make on the current
 * device, without launching: *resolved = STREAM_K or CLUSTER, *cluster_size = CTAs per
 * cluster (0 for STREAM_K), *ctas = CTAs of the grid.  Any output pointer may be NULL.
 * SHAPE for invalid sizes (as w4a16_gemv), UNSUPPORTED as w4a16_gemv_ex. */
w4a16_status w4a16_gemv_plan(int64_t M, int64_t N, int64_t K, int schedule, int* resolved,
                             int* cluster_size, int* ctas);

/* w4a16_linear_ex -- w4a16_linear for weights quantized in groups of group_size along K
 * (awq_quantize), with the decode GEMV's schedule (w4a16_gemv_schedule; ignored when
 * M > 16).  group_size: a multiple of 128 that divides K; scales and zeros have
 * K/group_size groups.  SHAPE for another group_size, VALUE for an unknown schedule.
 * Everything else is as for w4a16_linear. */
w4a16_status w4a16_linear_ex(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                             const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y,
                             int64_t M, int64_t N, int64_t K, int64_t group_size, void* workspace,
                             size_t workspace_bytes, int schedule, void* stream);

/*
 * 3-bit codes [SqueezeLLM article, 2.1-2.2: once its few sensitive weights are split off, the
 * dense part takes uniform quantization with as few as eight levels; 4.1 / 5.3: 3-bit runs].
 *
 * awq_quantize3 -- awq_quantize with codes 0..7: the same activation-aware scaling, groups,
 *   scale and zero-point rules with 2^3 - 1 steps (scale = fp16(max((max - min) / 7, 1e-5)),
 *   z = clamp(rint(-min / scale), 0, 7), q = clamp(rint(w' / scale) + z, 0, 7)).
 *   qweight3 [N][3K/32] uint32: the 32 codes of k = 32b .. 32b + 31 of row n sit in the three
 *            words qweight3[n][3b + w], w = 0..2: bits 4j .. 4j+2 of word w hold the code of
 *            element 8w + ORDER[j]; bit 4j + 3 of word w holds bit w of the code of element
 *            24 + ORDER[j] (ORDER as for 4-bit codes).
 *   scales   [K/group_size][N] fp16 bits; zeros [K/group_size][N/8] (nibbles, values 0..7).
 *   group_size  128, 256, 512 or 1024.  Everything else as awq_quantize.
 */
w4a16_status awq_quantize3(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                           int64_t group_size, uint32_t* qweight3, uint16_t* scales, uint32_t* zeros,
                           float* s_out, void* stream);

/*
 * w3a16_gemv -- the decode GEMV (1 <= M <= 16) on 3-bit codes laid out as awq_quantize3
 *   writes them, with the optional CSR term: y = bf16_rne(x . dequant3(Q)^T + x . W_sparse^T).
 *   The kernel is the 4-bit GEMV's with 24 KB units (12 words a row and group); codes 0..7
 *   enter the MMA as the exact bf16 values 128 + q, so the arithmetic and the error bound are
 *   those of w4a16_gemv_ex.  group_size: a multiple of 128 dividing K.  workspace: as for
 *   w4a16_gemv (w4a16_workspace_bytes).  schedule: as w4a16_gemv_ex.  Errors as w4a16_gemv_ex.
 *   The prefill GEMM has no 3-bit form (M > 16: W4A16_ERR_SHAPE).
 */
w4a16_status w3a16_gemv(const uint16_t* x, const uint32_t* qweight3, const uint16_t* scales,
                        const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N,
                        int64_t K, int64_t group_size, void* workspace, size_t workspace_bytes, int schedule,
                        void* stream);

/*
 * awq_quantize_nvfp4 -- the AWQ-scaled weights quantized to NVFP4 [DeepCompressor README:
 *   FP4_E2M1 among the toolbox's data types, NVFP4 in its result tables; the pages do not
 *   define the layout, which is read as the published one].  On w' = float(w * s_k):
 *     g   = amax|W'| / 2688 (2688 = 6 * 448; 1 for an all-zero W'), written to *gscale;
 *     per block of 16 consecutive k of a row: s8 = E4M3(amax|block| / fp32(6 g)), round to
 *     nearest even, saturating at 448; S = fp32(float(s8) * g);
 *     q = E2M1(fp32(w' / S)): nearest of +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}, ties to the even
 *     code, saturating at 6, bit 3 the sign of the quotient; q = 0 where S = 0.
 *   The dequantized weight is E2M1(q) * float(s8) * g.
 *   qweight  [N][K/8] uint32, device: 8 codes a word, element ORDER[j] of 8 in nibble j.
 *   scales8  [K/16][N] bytes (E4M3), device, group-major.
 *   gscale   one fp32, device, 4-byte aligned.  s_out [K] fp32, device, required.
 *   N a positive multiple of 8, K of 16.  Errors: NULL, SHAPE, ALIGN, VALUE (non-finite
 *   alpha) when called; later, VALUE for a non-finite W' or s.  w4a16_gemv_nvfp4 is the
 *   decode product on these weights.
 */
w4a16_status awq_quantize_nvfp4(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                                uint32_t* qweight, uint8_t* scales8, float* gscale, float* s_out, void* stream);

/*
 * w4a16_gemv_nvfp4 -- the decode product on NVFP4 weights as awq_quantize_nvfp4 writes them:
 *   y = bf16_rne( g * sum_b (s8_b / 2) * sum_{k in block b} (2 e2m1(q_k)) x'_k ), fp32 sums.
 *   The doubled codes are exact bf16 integers fed to mma.sync m16n8k16 (16 k = one scale
 *   block); each MMA's result is scaled by its block's E4M3 scale in fp32.  No CSR term, no
 *   workspace.  1 <= M <= 16; N a positive multiple of 16; K of 16.  x [M][K] bf16 bits and
 *   qweight 16-byte aligned; gscale the device fp32 tensor scale.
 *   Errors: NULL, SHAPE, ALIGN when called.
 */
w4a16_status w4a16_gemv_nvfp4(const uint16_t* x, const uint32_t* qweight, const uint8_t* scales8,
                              const float* gscale, uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream);

/* w4a16_gemv_folded -- the decode GEMV on the layer input BEFORE the AWQ scaling, as one call.
 * [AWQ translation, 3.2: the weights are multiplied by s and the activations divided by it.]
 *   x   [M][K] bf16 bits, device: the raw layer input.
 *   s   [K] fp32, device, 16-byte aligned: the scales awq_quantize wrote to s_out; or NULL,
 *       for an x that is already divided (the call is then w4a16_linear_ex's decode path).
 *   With s, the call first writes x'[m][k] = bf16_rne(float(x[m][k]) / s[k]) (IEEE division)
 *   into the workspace, once, and the GEMV (launched so that it streams its weights while
 *   that pass runs) then reads x' for the quantized product and the sparse term: the values
 *   awq_fold_activations writes, so y is bit-identical to awq_fold_activations followed by
 *   w4a16_gemv_ex with the same schedule.  (Dividing inside the GEMV's own activation load
 *   was built and measured slower: every CTA divides the activations of every unit it
 *   streams, so each element is divided once per row block instead of once.)
 *   group_size, schedule: as w4a16_linear_ex.  1 <= M <= 16 (SHAPE otherwise).
 *   Everything else is as for w4a16_gemv_ex; ALIGN also for a misaligned s.
 * For M > 16 run awq_fold_activations first, then w4a16_gemm. */
w4a16_status w4a16_gemv_folded(const uint16_t* x, const float* s, const uint32_t* qweight,
                               const uint16_t* scales, const uint32_t* zeros,
                               const w4a16_csr* outliers, uint16_t* y, int64_t M, int64_t N,
                               int64_t K, int64_t group_size, void* workspace,
                               size_t workspace_bytes, int schedule, void* stream);

/* w4a16_gemm -- the tcgen05 tensor-core path of w4a16_linear, for any M >= 1.  Arguments
 * and result are as for w4a16_linear, with the prefill workspace (see above): required with
 * a CSR, optional without (NULL: one CTA per output tile).  Weights are dequantized to bf16
 * inside the kernel; the sum over K is fp32 and, with split-K, its partial sums are added
 * in a fixed order, so the result does not depend on which CTA finishes first.
 * Launch overlap with a CSR: the GEMM may start its main loop while the CSR kernels run and
 * waits for them only before it adds the sparse term. */
w4a16_status w4a16_gemm(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                        const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y,
                        int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * w4a16_gemv_noalloc -- the decode GEMV of w4a16_gemv without a caller workspace.  The
 * paper has no counterpart; this entry point exists for callers that cannot allocate
 * device memory around the call.  Examples are a plugin of an inference engine that is
 * handed only its input and output buffers (the engine plans all memory ahead and forbids
 * allocations while it executes), and code that runs inside an allocator or memory-pool
 * callback, where calling cudaMalloc would re-enter the allocator.
 *   - Arguments, result and limits are those of w4a16_gemv, minus the workspace.
 *     N <= 131072 and at most 160 SMs on the device; otherwise W4A16_ERR_UNSUPPORTED.
 *   - With a CSR term, N x M <= 262144 as well (UNSUPPORTED otherwise).
 *   - Its scratch is a static device array of about 3.5 MiB inside the library.  Every GPU
 *     that loads the library holds one until the process exits.  The call allocates
 *     nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); the first call with M <= 8 and the first with M > 8 also
 *     cache the device's properties, the driver's tensor-map encoder and the occupancy of
 *     that kernel instance.  Make one call of each kind before any stream capture.
 *   - Each call clears the scratch's counters with cudaMemsetAsync on `stream`, and then
 *     runs the GEMV.
 *   - All calls on a device share the one array, which keeps the last call's contents.
 *     Calls that overlap on the GPU (different streams without ordering) race on it and
 *     give wrong results.
 */
w4a16_status w4a16_gemv_noalloc(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                                const uint32_t* zeros, const w4a16_csr* outliers, uint16_t* y,
                                int64_t M, int64_t N, int64_t K, void* stream);

/*
 * awq_split_outliers -- the dense-and-sparse split of a weight matrix, on the GPU.
 * [SqueezeLLM article, section 2.2: sensitive weights stay in fp16 in a sparse matrix and
 *  leave the dense part, W = W_dense + W_sparse; section 5.3: sparsity ratio 0.45%.  The
 *  sensitivity is read as |w| * a_k, a_k the mean |x| of input channel k.]
 *   W            fp32 [N][K] device, input (row-major, rows are output channels).
 *   act_absmean  fp32 [K] device, a_k >= 0 and finite.
 *   alpha        >= 0: the AWQ exponent; CSR values are fp16(w * s_k) with
 *                s_k = max(float(pow(a_k, alpha)), 1e-4), the scaled space of the packed
 *                dense part (see awq_quantize_g128).
 *   nnz          number of outliers, 0 <= nnz <= N * K (for the 0.45% ratio:
 *                floor(0.0045 * N * K)).  N * K < 2^32 and nnz < 2^31.
 *   W_dense      fp32 [N][K] device, output: W with the outliers set to 0 (may not alias W).
 *   row_ptr      int32 [N + 1], col_idx int32 [nnz], values fp16 bits [nnz], device,
 *                outputs: CSR with ascending columns in every row.
 *   workspace    device scratch of awq_split_outliers_workspace_bytes(N, K) bytes, 256-byte
 *                aligned; its contents need not be initialised.
 * Selection: the nnz entries with the largest score fp32(|w| * a_k); among equal scores the
 * lower linear index n * K + k wins.  The result is unique, so it is bit-exact against any
 * correct implementation of the same rule.
 * Errors: NULL, SHAPE (sizes, workspace too small), ALIGN, VALUE (alpha < 0 or not finite)
 * at launch; a non-finite W or a_k, or an fp16 overflow of a value, sets VALUE in the
 * device status word.  nnz = 0 copies W to W_dense and zeroes row_ptr (no workspace used).
 */
size_t awq_split_outliers_workspace_bytes(int64_t N, int64_t K);
w4a16_status awq_split_outliers(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                                int64_t nnz, float* W_dense, int32_t* row_ptr, int32_t* col_idx,
                                uint16_t* values, void* workspace, size_t workspace_bytes, void* stream);

/*
 * awq_search_alpha -- the AWQ scale search over a grid of exponents, on the GPU.
 * [AWQ (MLSys 2024) translation, section 3.2: the per-channel scaling factor is searched so
 *  that the quantized layer's output on calibration activations stays closest to the
 *  full-precision output; with s = a^alpha the search runs over alpha.]
 * For every alpha[i] it quantizes W with awq_quantize_g128, folds the scales into the
 * calibration activations (x' = bf16(x / s_k), IEEE division), runs the W4A16 product of this
 * library (the GEMV for M <= 16, else the GEMM) and scores it against the fp32 product:
 *     errors[i] = sum (y_q - y_ref)^2 / sum y_ref^2,   y_ref = x . W^T,
 * and *best is the index of the smallest error (the first one on ties).
 *   W fp32 [N][K], act_absmean fp32 [K], x_calib bf16 [M][K]: device inputs (x_calib are the
 *   activations before the fold).  alphas [n_alpha] (1..64 values, each >= 0 and finite),
 *   errors [n_alpha] and best: HOST memory.  workspace: device scratch of
 *   awq_search_alpha_workspace_bytes(M, N, K, n_alpha) bytes, 256-byte aligned.
 * N % 128 == 0, K % 1024 == 0, 1 <= M <= 65535.
 * The call is synchronous on `stream` (it reads the errors back) and it also reports any
 * problem the kernels recorded (as w4a16_check_device_status does).
 */
size_t awq_search_alpha_workspace_bytes(int64_t M, int64_t N, int64_t K, int n_alpha);
w4a16_status awq_search_alpha(const float* W, const float* act_absmean, const uint16_t* x_calib, int64_t M,
                              int64_t N, int64_t K, const float* alphas, int n_alpha, float* errors, int* best,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * awq_fold_activations -- x_out[m][k] = bf16(float(x[m][k]) / s[k]) (IEEE division, then
 * round-to-nearest-even): the runtime activation x' = x / s that the linear entry points
 * take, for callers that cannot fold 1/s into the preceding operator.
 * [AWQ (MLSys 2024) translation, section 3.2: the weights are multiplied by s and the
 *  activations divided by it.]
 *   x bf16 [M][K], s fp32 [K] (e.g. s_out of awq_quantize_g128), x_out bf16 [M][K]: device.
 *   1 <= M <= 65535, 1 <= K <= 2^20.  x_out may alias x.
 */
w4a16_status awq_fold_activations(const uint16_t* x, const float* s, uint16_t* x_out, int64_t M, int64_t K,
                                  void* stream);

/*
 * w4a16_selftest_timeout -- launch a one-thread kernel whose pipeline wait can never
 * complete and whose limit is limit_ns nanoseconds (0 .. 1e10; else W4A16_ERR_VALUE).  The
 * wait runs out through the same bounded-wait loop the kernels use, the kernel records a
 * timeout in the device status word and returns, and the next
 * w4a16_check_device_status(stream) reports W4A16_ERR_TIMEOUT.  It exists so that the
 * timeout path can be tested on a GPU without hanging or faulting it.  The pages have no
 * counterpart.
 */
w4a16_status w4a16_selftest_timeout(int64_t limit_ns, void* stream);

/*
 * w4a16_selftest_quotient -- check, on the current GPU, the division the quantizer uses per
 * weight (Markstein's correction of the product with the correctly rounded reciprocal of the
 * group's fp16 scale) against the IEEE division, for every 11-bit divisor significand and
 * every dividend significand, both signs, over the quotient range that decides a 4-bit code.
 * Synchronous on `stream`.  *mismatches (host) receives the number of differing quotients,
 * which must be 0; first (host, may be NULL) the bits of the first difference found: divisor,
 * dividend, result, IEEE result.  The pages have no counterpart: it is the evidence that the
 * faster division leaves awq_quantize_g128 bit-exact.
 */
w4a16_status w4a16_selftest_quotient(uint64_t* mismatches, uint32_t first[4], void* stream);

/*
 * w4a16_check_device_status -- synchronize `stream` and return the first problem that a
 * kernel recorded since the last call, or W4A16_OK.  This clears the record.  The record
 * is per device and shared by all streams of that device.
 */
w4a16_status w4a16_check_device_status(void* stream);

/* Static, human-readable name of a status value. */
const char* w4a16_status_string(w4a16_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int w4a16_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
