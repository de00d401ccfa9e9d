/*
 * fp8bs.h - C ABI of the fine-grained (block-scaled, group-128) FP8 linear
 * layer for NVIDIA B200 (sm_100a).
 *
 * The layer computes Y = X . W^T for bf16 X [M, K] and W [N, K] through 8-bit
 * floating point:
 *
 *   - activations are quantised per token in groups of 128 input channels,
 *     one fp32 scale per group, computed at run time ("FP8 à granularité
 *     fine", Hugging Face transformers docs, opening bullets and section
 *     "Chemin rapide de DeepGEMM": activation_scheme="dynamic");
 *   - weights are quantised per 128x128 block, one fp32 scale per block (same
 *     page, opening bullets: weight_block_size=(128, 128); section "Format
 *     d'échelle UE8M0": scales kept as plain float32, scale_fmt="float");
 *   - Y[m,n] = sum_kb sA[m,kb] * sW[n/128,kb] * sum_{k in kb} qA[m,k] qW[n,k],
 *     accumulated in fp32 and rounded to bf16;
 *   - a 2:4 variant keeps the two largest |w| of every 4 contiguous weights
 *     along K ("Déployer la parcimonie 2:4 avec FP8 sur Hopper", steps 2, 4,
 *     6 and "Exemples pratiques 1"; "Combiner élagage et quantification ...",
 *     section "La clé : la sparsité structurée 2:4") and multiplies the
 *     compressed weights.
 *
 * Number format: OCP FP8 E4M3 ("fn": bias 7, no infinities, max 448).
 * Scale of a group or block: s = amax / 448 (fp32 IEEE division). Element
 * code: e4m3(x / s) with one fp32 IEEE division, round-to-nearest-even,
 * saturating to +-448. A group or block whose amax is 0 has s = 0 and every
 * element encodes as a zero carrying the element's sign (0x00 or 0x80).
 *
 * Conventions shared by every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller. The library
 *     never allocates, frees or synchronises; every call is asynchronous on
 *     `stream` (a cudaStream_t; NULL means the legacy default stream).
 *   - All matrices are dense row-major, with no leading-dimension argument.
 *   - K must be a positive multiple of 128. M == 0 or N == 0 is a no-op that
 *     returns FP8BS_OK.
 *   - Every matrix pointer (activations, weights, codes, metadata, outputs)
 *     must be 16-byte aligned; fp32 scale arrays and expert indices need
 *     4-byte alignment; UE8M0 scale-code arrays (bytes) need none.
 *   - Arguments are validated before anything is launched; on an error
 *     nothing is written and a nonzero FP8BS_ERR_* code is returned.
 *   - A launch failure returns FP8BS_ERR_CUDA. A kernel that gave up a bounded
 *     internal wait records FP8BS_ERR_DEVICE_TIMEOUT in a device error word,
 *     read by fp8bs_get_device_error().
 *   - Input and output buffers must not overlap.
 */
#ifndef FP8BS_H_
#define FP8BS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP8BS_OK = 0,
  FP8BS_ERR_NULL = 1,           /* a required pointer is NULL */
  FP8BS_ERR_SHAPE = 2,          /* K % 128 != 0, K <= 0, M/N < 0, or a size too large */
  FP8BS_ERR_ALIGN = 3,          /* a pointer is not aligned (16 bytes; 4 for scales / indices) */
  FP8BS_ERR_WORKSPACE = 4,      /* workspace smaller than fp8bs_gemm_workspace_bytes() */
  FP8BS_ERR_CUDA = 5,           /* a CUDA runtime/driver call failed */
  FP8BS_ERR_DEVICE_TIMEOUT = 6, /* a kernel gave up a bounded wait */
  FP8BS_ERR_ARCH = 7,           /* the current device is not sm_100 */
  FP8BS_ERR_SCRATCH_LIMIT = 8   /* the problem needs more than the fixed no-allocation scratch */
} fp8bs_status;

/*
 * Dynamic per-token activation quantization in 1x128 groups along K
 * ("FP8 à granularité fine", opening bullets; "Chemin rapide de DeepGEMM").
 *
 *   x_bf16   [M][K] bf16, input.
 *   qa_e4m3  [M][K] E4M3 bytes, output: qa[m][k] = e4m3(x[m][k] / sa[m][k/128]).
 *   sa       [M][K/128] fp32, output: sa[m][g] = amax_{k in group g} |x[m][k]| / 448.
 */
int fp8_quant_act_group128(const void* x_bf16, int64_t M, int64_t K, void* qa_e4m3, float* sa,
                           void* stream);

/*
 * Weight quantization in 128x128 blocks ("FP8 à granularité fine", opening
 * bullets, weight_block_size=(128, 128)).
 *
 *   w_bf16   [N][K] bf16, input.
 *   qw_e4m3  [N][K] E4M3 bytes, output.
 *   sw       [ceil(N/128)][K/128] fp32, output: block amax / 448. The last row
 *            block covers only the valid rows when N % 128 != 0.
 */
int fp8_quant_weight_block128(const void* w_bf16, int64_t N, int64_t K, void* qw_e4m3, float* sw,
                              void* stream);

/*
 * 2:4 magnitude pruning along K, then block quantization and compression
 * ("Déployer la parcimonie 2:4 avec FP8 sur Hopper", steps 2, 4 and 6;
 * "Combiner élagage et quantification ...", section on 2:4 sparsity).
 *
 * In every group of 4 contiguous weights along K the two largest |w| are kept
 * (equal magnitudes: the lower index wins) and the other two become +0. The
 * pruned matrix is then quantized exactly like fp8_quant_weight_block128
 * (scales recomputed after pruning).
 *
 *   w_bf16         [N][K] bf16, input.
 *   vals_e4m3      [N][K/2] E4M3 bytes, output: the two kept codes of group g
 *                  at [n][2g] and [n][2g+1], in order of position.
 *   meta           [N][K/8] bytes, output: byte j holds group 2j in bits 0-3
 *                  and group 2j+1 in bits 4-7; each nibble is i0 | (i1 << 2)
 *                  with i0 < i1 the kept positions (0..3) within the group.
 *   sw             [ceil(N/128)][K/128] fp32, output.
 *   w_pruned_bf16  [N][K] bf16, optional output (may be NULL): the pruned
 *                  weights in bf16.
 */
int prune24_compress(const void* w_bf16, int64_t N, int64_t K, void* vals_e4m3, uint8_t* meta,
                     float* sw, void* w_pruned_bf16, void* stream);

/*
 * Block-scaled FP8 GEMM ("FP8 à granularité fine": 1x128 activation groups
 * against 128x128 weight blocks):
 *   y[m][n] = bf16_rn( sum_kb sa[m][kb] * sw[n/128][kb] * sum_{k in kb} qa[m][k] * qw[n][k] )
 * with fp32 accumulation.
 *
 *   qa  [M][K] E4M3, sa [M][K/128] fp32  (from fp8_quant_act_group128)
 *   qw  [N][K] E4M3, sw [ceil(N/128)][K/128] fp32  (from fp8_quant_weight_block128)
 *   y_bf16 [M][N] bf16, output. N must be a multiple of 8.
 *   workspace / workspace_bytes: scratch of at least
 *       fp8bs_gemm_workspace_bytes(M, N, K, 0) bytes (may be NULL when that is 0).
 * Results are deterministic: the same inputs give the same bytes every call.
 */
int fp8_block_gemm(const void* qa, const float* sa, const void* qw, const float* sw, void* y_bf16,
                   int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * fp8_block_gemm with the next layer's input quantization fused in: the same
 * y, and qy / sy = fp8_quant_act_group128(y) of that bf16 y, i.e. y's rows
 * cut into 1x128 groups along N ("FP8 à granularité fine": the output of one
 * linear is the activation of the next, quantized per token per 128
 * channels). For M > 256 the GEMM's epilogue quantizes its own tile (each
 * promotion thread holds one group); for M <= 16 with unsplit decode tiles
 * (N of at least 75 row blocks on 148 SMs) the decode-order epilogue
 * quantizes each token's staged group; otherwise y is written and then
 * quantized by the activation quantizer.
 *
 *   y_bf16  [M][N] bf16, output; may be NULL when M > 256 (then only the codes
 *           are written), required when M <= 256.
 *   qy_e4m3 [M][N] E4M3 codes, output; sy [M][N/128] fp32 scales, output.
 *   N must be a multiple of 128; the other arguments as fp8_block_gemm.
 * Returns FP8BS_ERR_SHAPE for N % 128 != 0 and FP8BS_ERR_NULL for a missing
 * qy / sy (or y with M <= 256).
 */
int fp8_block_gemm_quant(const void* qa, const float* sa, const void* qw, const float* sw,
                         void* y_bf16, void* qy_e4m3, float* sy, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * The block-scaled GEMM with 2:4-compressed weights (vals, meta, sw as written
 * by prune24_compress). Same result definition as fp8_block_gemm with qw the
 * decompressed codes (pruned positions are code 0).
 */
int fp8_sparse24_gemm(const void* qa, const float* sa, const void* vals, const uint8_t* meta,
                      const float* sw, void* y_bf16, int64_t M, int64_t N, int64_t K,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * UE8M0 scale variant ("FP8 à granularité fine", section "Format d'échelle
 * UE8M0": scales stored as float8_e8m0fnu, a bare power of two). A scale is
 * kept as one code byte c standing for 2^(c - 127); it is the smallest power
 * of two s with 448 * s >= amax (so no element saturates), codes clamped to
 * 0..254, amax == 0 -> code 0. Elements are e4m3(x / s) as above (the quotient
 * by a power of two is exact unless it underflows).
 *
 *   fp8_quant_act_group128_ue8m0:    x_bf16 [M][K] -> qa_e4m3 [M][K], sa_ue8m0 [M][K/128]
 *   fp8_quant_weight_block128_ue8m0: w_bf16 [N][K] -> qw_e4m3 [N][K],
 *                                    sw_ue8m0 [ceil(N/128)][K/128]
 *   fp8_block_gemm_ue8m0: y = sum_kb 2^(sa - 127) 2^(sw - 127) (qa_kb . qw_kb^T),
 *       fp32 accumulation, bf16 out (N a multiple of 8); the tensor cores apply
 *       the scales themselves (block-scaled MMA), so there is no per-K-block
 *       promotion. Workspace as fp8_block_gemm (none needed).
 * Argument rules and errors as the fp32-scale entry points.
 */
int fp8_quant_act_group128_ue8m0(const void* x_bf16, int64_t M, int64_t K, void* qa_e4m3,
                                 uint8_t* sa_ue8m0, void* stream);
int fp8_quant_weight_block128_ue8m0(const void* w_bf16, int64_t N, int64_t K, void* qw_e4m3,
                                    uint8_t* sw_ue8m0, void* stream);
int fp8_block_gemm_ue8m0(const void* qa, const uint8_t* sa_ue8m0, const void* qw,
                         const uint8_t* sw_ue8m0, void* y_bf16, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Grouped (mixture-of-experts) block-scaled GEMMs ("FP8 à granularité fine",
 * section "Chemin rapide de DeepGEMM": the experts' products run through
 * grouped kernels; with UE8M0 scales on SM100 per section "Format d'échelle
 * UE8M0", with fp32 scales as a grouped matmul). The token rows are grouped
 * by expert in one matrix (the contiguous layout):
 *
 *   y[m][n] = sum_kb sa[m][kb] * sw[e][n/128][kb] * sum_{k in kb} qa[m][k] qw[e][n][k],
 *             e = m_indices[m]
 *
 *   qa [M][K] E4M3, sa [M][K/128] (fp32, or UE8M0 codes for the _ue8m0 form).
 *   qw [E][N][K] E4M3, sw [E][ceil(N/128)][K/128] (fp32, or UE8M0 codes).
 *   m_indices [M] int32, device memory: the expert of each row, or -1 for a
 *       padding row. Every aligned group of 128 rows (rows 128t .. 128t+127)
 *       must hold rows of a single expert plus padding rows: each expert's
 *       rows start at a multiple of 128. The expert of a tile is read from its
 *       first row; an index outside [0, E) there counts as expert 0.
 *   y_bf16 [M][N]: rows of real tokens are written; padding rows receive
 *       values with no defined meaning.
 * N a multiple of 8, K of 128, E >= 1. Same errors as fp8_block_gemm.
 */
int fp8_grouped_gemm(const void* qa, const float* sa, const void* qw, const float* sw,
                     const int32_t* m_indices, void* y_bf16, int64_t M, int64_t N, int64_t K,
                     int64_t E, void* workspace, size_t workspace_bytes, void* stream);
int fp8_grouped_gemm_ue8m0(const void* qa, const uint8_t* sa_ue8m0, const void* qw,
                           const uint8_t* sw_ue8m0, const int32_t* m_indices, void* y_bf16,
                           int64_t M, int64_t N, int64_t K, int64_t E, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * The gated MLP's gate+up GEMM with SwiGLU fused into its epilogue, keeping
 * both block scales (TensorRT-LLM docs, performance/fp8-quantization, section
 * "GEMM + SwiGLU Fusion in Gated-MLP": two matmuls and the SwiGLU in one
 * kernel), and the down projection's input quantization after it:
 *
 *   g, u = the block-scaled GEMM of qa with the gate rows [0, I) and the up
 *          rows [I, 2I) of qw_gate_up, in fp32;
 *   h    = bf16_rn( silu(g) * u ),  silu(g) = g / (1 + e^-g);
 *   qh, sh = fp8_quant_act_group128(h)   (1x128 groups along I).
 *
 *   qa [M][K], sa [M][K/128]           (the activations, as fp8_block_gemm)
 *   qw_gate_up [2I][K], sw_gate_up [2I/128][K/128]  ([W_gate; W_up] quantized
 *       with fp8_quant_weight_block128)
 *   h_bf16 [M][I] bf16, output, may be NULL; qh_e4m3 [M][I], sh [M][I/128].
 *   workspace: at least fp8bs_swiglu_workspace_bytes(M, I) bytes, 16-byte
 *       aligned (required for M <= 256 only, else may be NULL): there the
 *       call may run the decode-order GEMM of the 2I weight rows into this
 *       scratch (g and u rounded to bf16) and a second kernel that forms h and
 *       its codes; otherwise (M > 256, or M > 64 with 2I wide enough that
 *       tiles of 128 tokens x 256 weight rows fill at least three quarters of
 *       the GPU) one kernel does all of it from the fp32 accumulators. Both
 *       forms meet the same tolerance on h.
 *   I must be a positive multiple of 128. Same errors as fp8_block_gemm;
 *   FP8BS_ERR_WORKSPACE for a missing or short workspace.
 */
int fp8_gemm_swiglu_quant(const void* qa, const float* sa, const void* qw_gate_up,
                          const float* sw_gate_up, void* h_bf16, void* qh_e4m3, float* sh,
                          int64_t M, int64_t I, int64_t K, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Scratch bytes fp8_gemm_swiglu_quant needs for M tokens and intermediate size I. */
size_t fp8bs_swiglu_workspace_bytes(int64_t M, int64_t I);

/*
 * fp8_gemm_swiglu_quant without a workspace and without any device allocation
 * (no cudaMalloc / cudaFree, no allocating library call). The paper (the
 * pages this library follows) has no counterpart: it exists for callers that
 * cannot hand over or obtain device memory per call, such as a C host that
 * owns every buffer and passes only operands in and out (a plugin or
 * custom-op interface with no workspace slot), or a decode loop that must not
 * enter an allocator because
 * cudaMalloc / cudaFree may synchronise the device and fail once a memory
 * pool has reserved the free memory.
 *
 * Same operands, results and tolerance as fp8_gemm_swiglu_quant. For
 * M <= 256 the [M][2I] bf16 intermediate lives in one fixed device array of
 * FP8BS_NOALLOC_SCRATCH_BYTES (16 MiB) per device, reserved when the library's
 * module is loaded; calls needing more (M <= 256 and M * 2I * 2 bytes above
 * it: every M for I <= 16384; for I = 28672, M in 147 .. 256) return
 * FP8BS_ERR_SCRATCH_LIMIT before anything is launched. Nothing in the array
 * must start at zero: each call writes all of it that it reads. For M > 256
 * no scratch is used.
 *
 * Setup: the first call on a device (any M, including 0, with that device
 * current) looks up the array's address (cudaGetSymbolAddress) and caches it;
 * make it before any stream capture. Calls on one device share the array:
 * calls that overlap in time (other streams or host threads without ordering
 * between them) race on it and give wrong results.
 */
#define FP8BS_NOALLOC_SCRATCH_BYTES (16u << 20)
int fp8_gemm_swiglu_quant_noalloc(const void* qa, const float* sa, const void* qw_gate_up,
                                  const float* sw_gate_up, void* h_bf16, void* qh_e4m3,
                                  float* sh, int64_t M, int64_t I, int64_t K, void* stream);

/*
 * Output-column (N) split over P ranks (tensor parallelism; TensorRT-LLM docs,
 * performance/fp8-quantization: the Llama-3.3-70B case study runs tensor
 * parallel over 4 GPUs). Rank p holds weight rows [p Np, (p + 1) Np) (Np a
 * multiple of 128, so whole 128x128 blocks) and computes those columns of Y;
 * an all-gather over the ranks leaves them rank-major, [P][M][Np]. This call
 * turns that into the full rows: dst[m][p Np + j] = src[p][m][j].
 *   src_bf16 [P][M][Np], dst_bf16 [M][P Np], both bf16, no overlap;
 *   Np a multiple of 8.
 */
int fp8_gather_columns(const void* src_bf16, int64_t P, int64_t M, int64_t Np, void* dst_bf16,
                       void* stream);

/* Scratch bytes needed by the GEMMs for this shape (sparse != 0: the 2:4 GEMM). */
size_t fp8bs_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int sparse);

/*
 * Synchronises `stream`, then returns and clears the device error word of the
 * current device (FP8BS_OK if no kernel recorded an error).
 */
int fp8bs_get_device_error(void* stream);

/*
 * Upper bound, in SM clock cycles, of each internal wait of the GEMM kernels
 * (default about two seconds). cycles <= 0 restores the default. A wait that
 * runs out makes the kernel stop early and record FP8BS_ERR_DEVICE_TIMEOUT.
 * Intended for tests of the timeout path.
 */
void fp8bs_set_wait_limit(long long cycles);

/* Static description of a status code. */
const char* fp8bs_status_string(int status);

/* Library version, as MAJOR * 10000 + MINOR * 100 + PATCH. */
int fp8bs_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8BS_H_ */
