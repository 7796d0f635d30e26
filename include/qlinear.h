/*
 * qlinear.h -- C ABI of libqlinear: a W4A4 quantized linear layer y = X W^T for NVIDIA B200
 * (sm_100a), with block-scaled FP4 weights (E8M0-B32 or E4M3-B16 scales), PRQuant tail-block
 * residuals, MXCode VQ codebook weights, CodeQuant-style cluster-codebook MoE experts and
 * MosaicQuant-style INT4 dense + block-sparse weights.
 *
 * Sources of the operations (page title, section / table):
 *   - MXCode (MX-Native Codebook Quantization), Table 1: the block-scaled FP4 formats
 *     (E2M1 elements; E8M0 scales per 32, or E4M3 scales per 16 plus an FP32 tensor scale).
 *   - PRQuant: Permutation Residual Quantization, §4 Method, "Kernel design for efficient
 *     inference": one MXFP4 GEMM whose reduction is extended from C to C + k by an offline
 *     weight residual on the permuted tail channels; the activation is quantized once and its
 *     quantized tail reused.
 *   - MXCode abstract: reconstruct MX-native W4A4 operands from VQ indices and FP4 codebooks
 *     without materialising high-precision weights.
 *   - CodeQuant, Figure 4: per-tile lookup table kept in SM shared memory.
 *   - MosaicQuant, "ZipperEngine": dense INT4 base and sparse INT4 residual fused into one GEMM.
 *
 * Conventions
 *   - All matrices are row-major.  Activations are bf16 [M, K] (token-major); outputs are bf16
 *     [M, N] (optionally also fp32).  "Device" pointers must be CUDA device memory of the
 *     current device; "host" pointers are ordinary CPU memory.
 *   - FP4 codes are packed two per byte, element 2j in the low nibble of byte j; bit 3 of a
 *     code is its sign.  E8M0 scale bytes hold exponent + 127.  E4M3 scales are OCP FP8 E4M3.
 *   - Calls that take a cudaStream_t are asynchronous and never synchronise the stream; the
 *     caller keeps every device buffer alive until the stream has run the work.
 *   - Every call returns a ql_status.  Argument and shape checks happen before any launch and
 *     leave device memory untouched.  ql_last_error() gives a thread-local message for the
 *     last non-OK status.  Kernels whose bounded waits expire set a device error word that
 *     ql_check() reports (QL_ERR_TIMEOUT); they never trap.  No call falls back to the CPU.
 */
#ifndef QLINEAR_H_
#define QLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ql_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent descriptor */
  QL_ERR_UNSUPPORTED = 2, /* shape outside what the kernels implement (see each call) */
  QL_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  QL_ERR_OOM = 4,         /* device allocation failed (create calls only) */
  QL_ERR_TIMEOUT = 5,     /* a kernel's bounded wait expired (reported by ql_check) */
  QL_ERR_WORKSPACE = 6    /* workspace pointer null/misaligned or smaller than required */
} ql_status;

typedef enum {
  QL_W_MXFP4_E8M0_B32 = 1,       /* codes [N,K/2] + E8M0 bytes [N,K/32]; optional PRQuant tail */
  QL_W_NVFP4_E4M3_B16 = 2,       /* codes [N,K/2] + E4M3 bytes [N,K/16] + fp32 tensor scale */
  QL_W_VQ_PRESCALE_E4M3_B16 = 3, /* MXCode PreScale: uint8 indices [N,K/4] into per-QBlock
                                    codebooks of 256 x 4 E2M1 codes, E4M3 bytes [N,K/16],
                                    fp32 tensor scale */
  QL_W_CLUSTER4_ROW16_BF16 = 4,  /* CodeQuant-style: 4-bit indices [N,K/2] into 16 bf16
                                    centroids per output row */
  QL_W_INT4_G128_BSR = 5,        /* INT4 codes [N,K/2] + fp16 scale per (row,128-group), plus a
                                    block-sparse INT4 residual on 16x128 blocks (BSR) */
  QL_W_VQ_POSTSCALE_E4M3_B16 = 6,    /* MXCode PostScale: uint8 indices [N,K/4] into per-QBlock
                                        codebooks of 256 x 4 E2M1 codes, ONE E4M3 scale byte per
                                        QBlock [N/64,K/64] (scales), fp32 tensor scale */
  QL_W_VQ_PRESCALE_PLUS_E4M3_B16 = 7 /* MXCode PreScale+: indices and codebooks as PreScale; the
                                        E4M3 block scales by VQ: uint8 scale indices [N,K/128]
                                        (scales) into scale_codebook [256][8] E4M3 bytes; fp32
                                        tensor scale */
} ql_wformat;

typedef enum {
  QL_A_MXFP4_E8M0_B32 = 1,  /* codes [M,K/2] + E8M0 bytes [M,K/32] */
  QL_A_FP4_E4M3_B16_TS = 2, /* codes [M,K/2] + E4M3 bytes [M,K/16] + fp32 tensor scale */
  QL_A_INT4_TOK_G128 = 3    /* int4 codes [M,K/2] + fp32 scale per (token,128-group) */
} ql_aformat;

/* Weight description.  Every array pointer is HOST memory; *_create copies and repacks it. */
typedef struct ql_weight_desc {
  ql_wformat wfmt;
  int64_t N;          /* output features */
  int64_t K;          /* reduction width of the weight (includes k_tail) */
  int32_t k_tail;     /* PRQuant: width of the residual K-extension (0 = none); the activation
                         has K - k_tail channels and its last k_tail channels are reused */
  const void* codes;  /* packed 4-bit codes (FP4 or INT4) [N, K/2]; cluster indices for fmt 4 */
  const void* scales; /* E8M0 [N,K/32] | E4M3 [N,K/16] | fp16 [N,K/128] (INT4) */
  float w_tensor_scale;       /* E4M3-B16 formats: FP32 tensor scale of W (else ignored) */
  const uint8_t* indices;     /* VQ: [N, K/4] */
  const void* codebooks;      /* VQ: uint8 [N/qn][K/qk][256][2] (4 packed E2M1 per entry);
                                 cluster: bf16 [N][16] */
  int32_t qblock_n, qblock_k; /* VQ QBlock shape (64 x 64) */
  const int32_t* bsr_rowptr;  /* INT4 residual: [N/bsr_block_n + 1] */
  const int16_t* bsr_col;     /* [nnzb] 128-group index of each block */
  const void* bsr_codes;      /* [nnzb][bsr_block_n][bsr_block_k/2] int4 */
  const void* bsr_scales;     /* [nnzb][bsr_block_n] fp16 */
  int32_t bsr_block_n, bsr_block_k, bsr_nnzb;
  const uint8_t* scale_codebook;       /* VQ PreScale+: [scale_codebook_entries][scale_group] */
  int32_t scale_codebook_entries;      /* 256 */
  int32_t scale_group;                 /* 8 consecutive E4M3 block scales along K per index */
  int32_t had_block;   /* 0, or 32: the layer's activation (MXFP4 layers; MoE: x for gate/up,
                          h for down) passes an online block-32 Hadamard before quantization
                          (CodeQuant's "had" variants), and the weight is given rotated,
                          W . blockdiag(H_32) / 32; see quantize_act_hadamard */
  int32_t tail_copy;   /* MXFP4 layers with k_tail > 0: 0 = the GEMM reads the activation's last
                          k_tail channels a second time for the tail stages (PRQuant "online"
                          tail); 1 = the activation quantizer writes the augmented activation
                          [Z~, Z~_tail] (C + k_tail channels, the tail copied behind, PRQuant §4
                          "Activation tail construction", offline copy) and the GEMM reads it
                          straight through.  Same results. */
} ql_weight_desc;

typedef struct ql_linear ql_linear;
typedef struct ql_moe ql_moe;

/* Version and device queries. */
const char* ql_version(void);
const char* ql_last_error(void);

/* Create a linear layer (MXCode Table 1 formats; PRQuant §4 "Offline residual augmentation" for
 * the tail; MXCode abstract for VQ codebooks; MosaicQuant "Dense Base and Sparse Residuals"):
 * validates the descriptor, copies the weights to device memory owned by the returned handle
 * and repacks them, with their scales, into the tiled layout the MMA consumes.
 * Supported:
 *   QL_W_MXFP4_E8M0_B32        N % 16 == 0, K % 128 == 0, k_tail % 128 == 0, 0 <= k_tail < K;
 *                              activations quantized to MXFP4 (E8M0-B32).
 *   QL_W_NVFP4_E4M3_B16        N % 16 == 0, K % 64 == 0, no tail; activations E4M3-B16 + FP32
 *                              tensor scale; y = (sum) * ts_x * ts_w.
 *   QL_W_VQ_PRESCALE_E4M3_B16  N % 128 == 0, K % 256 == 0, 64 x 64 QBlocks, no tail; indices,
 *                              codebooks, E4M3 scales [N,K/16] and w_tensor_scale; the weight
 *                              operand is rebuilt from the codebooks inside the GEMM.
 *   QL_W_VQ_POSTSCALE_E4M3_B16 as PreScale, with scales = one E4M3 byte per QBlock [N/64,K/64]
 *                              (the decoder gives every 16-block of the QBlock that scale).
 *   QL_W_VQ_PRESCALE_PLUS_E4M3_B16 as PreScale, with scales = scale indices [N,K/128] into
 *                              scale_codebook [256][8] (block scale 8g+i of a row is
 *                              scale_codebook[index g][i]); scale_codebook_entries = 256,
 *                              scale_group = 8.
 *   QL_W_INT4_G128_BSR         N % 128 == 0, K % 128 == 0, no tail; codes [N,K/2] (INT4, two's
 *                              complement nibbles), fp16 scales [N,K/128], and a 16 x 128
 *                              block-sparse INT4 residual (bsr_*: rowptr [N/16+1], col = group,
 *                              codes [nnzb][16][64], fp16 scales [nnzb][16]); activations INT4
 *                              per (token, 128-group); y = sum_g sx*sw*I_g + residual terms,
 *                              both branches in one fused tcgen05 kind::i8 GEMM.
 * Synchronous with respect to `stream` (uses it for the uploads). */
ql_status qlinear_create(const ql_weight_desc* desc, ql_stream_t stream, ql_linear** out);
ql_status qlinear_destroy(ql_linear* layer);

/* Bytes of device workspace that qlinear_forward needs for M tokens: the quantized activation
 * (codes and tiled scales; PRQuant §4 quantizes it once), the grid-wide agreement words and the
 * split-K partial tiles.  Host-only; *bytes is host memory. */
ql_status qlinear_workspace_bytes(const ql_linear* layer, int64_t M, size_t* bytes);

/* y[M,N] = X[M, K-k_tail] (quantized online) times the layer's weight: the quantized linear
 * layer the pages share -- PRQuant §4 "Kernel design for efficient inference" (the activation
 * quantized to MXFP4 once, its tail reused, one GEMM over C + k), MXCode abstract and Table 1
 * (E4M3-B16 activations, MX-native operands rebuilt from the codebooks), MosaicQuant
 * "ZipperEngine" (INT4 base and residual in one GEMM).  x_bf16, y_bf16 and the workspace are
 * device pointers; y_f32 (device, [M,N]) may be NULL.  ws must be 256-byte aligned and at least
 * qlinear_workspace_bytes(M) long; its contents on entry do not matter: the grid-wide agreements
 * (the E4M3-B16 tensor amax, the split-K hand-off) go through workspace words that carry a
 * per-launch tag derived from a launch counter kept there, so nothing needs clearing, and after
 * a device timeout the counter has moved past every tag the failed launch left.  Calls that
 * share a workspace must be stream-ordered.  Rows of x are contiguous (row stride K - k_tail
 * elements, with or without tail_copy).  M may be 0 (no-op).  Where the decode kernel runs
 * (ql_decode_fuse_mode; by default M = 1, and MXFP4 layers from 33 to 64 tokens) the forward is
 * ONE launch whose own warps quantize x before its MMAs need it, while the weights already
 * stream; otherwise it is the activation quantizer followed by the split-K or prefill GEMM.
 * Kernels are launched with programmatic stream serialization and release the next such grid at
 * once: a following qlinear call on the stream may start streaming its weights while this one
 * finishes, and reads this call's results only after it has completed. */
ql_status qlinear_forward(const ql_linear* layer, const void* x_bf16, int64_t M, void* y_bf16,
                          float* y_f32, void* ws, size_t ws_bytes, ql_stream_t stream);

/* The two halves of qlinear_forward.  qlinear_quantize_input quantizes x into the workspace
 * (MXFP4 codes and tiled scales); qlinear_gemm runs
 * the tcgen05 GEMM from that workspace.  Called in this order on one stream with the same M and
 * workspace they equal qlinear_forward.  A caller whose several layers share one input (gate and
 * up projections, say) can quantize once; the split also lets a profiler time the GEMM alone.
 * qlinear_gemm may be repeated on one quantized workspace: the split-K arrival counters it keeps
 * there are cleared by qlinear_quantize_input and left cleared by every qlinear_gemm.  The GEMM
 * is launched with programmatic stream serialization: it may start while the kernel before it on
 * the stream is still running, streams (and decodes) weights meanwhile, and waits for that kernel
 * to complete before it reads the workspace, writes y or reads the activation tensor scale. */
ql_status qlinear_quantize_input(const ql_linear* layer, const void* x_bf16, int64_t M, void* ws,
                                 size_t ws_bytes, ql_stream_t stream);
ql_status qlinear_gemm(const ql_linear* layer, int64_t M, void* y_bf16, float* y_f32, void* ws,
                       size_t ws_bytes, ql_stream_t stream);

/* qlinear_forward without a caller-supplied workspace, for callers that cannot allocate device
 * memory (an engine that plans all device memory ahead and forbids allocation during a forward,
 * a plugin whose host exposes no allocator, a latency-critical loop that must not enter the
 * allocator).  No step of the method corresponds to this call; it is a packaging convenience.
 * The workspace is a fixed 8 MiB array inside the library (each GPU that loads the library keeps
 * it until the process exits); M whose qlinear_workspace_bytes exceeds 8 MiB is rejected with
 * QL_ERR_WORKSPACE.  Nothing is allocated: no cudaMalloc/cudaFree, no library allocator.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress with that
 * device current) and caches it with the current context; a call that finds another context
 * current (after cudaDeviceReset, say) looks it up again.  Make the first call on a device, and
 * the first after a context change, before any stream capture.  All calls share the one
 * array, which keeps whatever the last call left in it (the parts that must start at zero are
 * cleared by each call): calls that may overlap on the GPU (different streams, or different host
 * threads) race on it and must be serialised by the caller.  x, y and y_f32 are device pointers
 * as for qlinear_forward. */
ql_status qlinear_forward_fixed_scratch(const ql_linear* layer, const void* x_bf16, int64_t M,
                                        void* y_bf16, float* y_f32, ql_stream_t stream);

/* Online activation quantization (device pointers).
 * QL_A_MXFP4_E8M0_B32: K % 32 == 0; codes [M,K/2], scales E8M0 [M,K/32]; tensor_scale unused.
 * Rule (OCP MX, as the PRQuant page applies it): per 32 elements e = floor(log2 amax) - 2
 * clamped to [-127,127], byte e+127 (0 for an all-zero block), code = E2M1 RNE of x/2^e with
 * saturation at +-6 and the sign of x.
 * QL_A_FP4_E4M3_B16_TS: K % 16 == 0; codes [M,K/2], E4M3 scales [M,K/16], *tensor_scale (device
 * float) receives ts = amax(x)/2688 (1 for an all-zero x); per 16 elements
 * s = E4M3_RNE_satfinite((amax/6)/ts), code = E2M1 RNE of x/(dec(s)*ts) (MXCode Table 1 row
 * E4M3-B16-FP4), each step an IEEE fp32 operation.
 * QL_A_INT4_TOK_G128: K % 128 == 0; codes [M,K/2] (two's-complement nibbles), scales float
 * [M,K/128]: per (token, 128-group) s = amax/7 (fp32), q = clamp(rint(x/s), -7, 7) (MosaicQuant's
 * W4A4 INT4 path; the granularity is a reading). */
ql_status quantize_act(ql_aformat fmt, const void* x_bf16, int64_t M, int64_t K, void* codes,
                       void* scales, float* tensor_scale, ql_stream_t stream);

/* Tensor-pipe throughput probe (measurement only; no step of the method).  Launches `ctas` CTAs
 * (one per SM at most is useful) that each issue iters x 4 back-to-back tcgen05.mma instructions
 * of one kind (kind 0: kind::mxf4.block_scale.block32; 1: kind::mxf4nvf4.block_scale.block16;
 * 2: kind::i8; 3: kind::f16 with bf16 operands) with M = 128 and N = n (128 or 256) on operands
 * resident in shared memory, into one TMEM accumulator; *flops_per_launch (host, may be NULL)
 * receives 2 * 128 * n * K_mma * 4 * iters * ctas.  The caller times the launch on `stream`
 * (CUDA events); the quotient is the peak a GEMM of that kind can approach on this GPU, the
 * denominator of its roofline.  Asynchronous; nothing is read back. */
ql_status ql_tensor_peak(int32_t kind, int32_t n, int32_t iters, int32_t ctas,
                         double* flops_per_launch, ql_stream_t stream);

/* Test hook for the timeout path (no step of the method).  Sets the limit of every bounded wait
 * in the library's kernels (wait_limit_ns; 0 restores the default 2 s) and names one CTA index
 * (withhold_cta >= 0; -1: none) whose grid-wide publications are withheld: its slot in the
 * E4M3-B16 amax agreement and its flags in the decode GEMM are never written, so the waits on
 * them run out after the limit, the kernels record QL_ERR_TIMEOUT in the device error word and
 * return, and ql_check reports it.  Nothing faults or hangs.  Synchronises the device; affects
 * every later launch on it until called again with (-1, 0).  The workspaces stay usable
 * afterwards: the launch counters of the grid-wide protocols move past every tag a failed
 * launch left behind. */
ql_status ql_debug_inject(int32_t withhold_cta, uint64_t wait_limit_ns);

/* How qlinear_forward's decode kernel (M <= 64, FP4 and VQ layers) is organised:
 * 0 = no decode kernel: the separate quantizer, then the general split-K GEMM;
 * 1 = the CTAs share the activation units out, exchange the E4M3 tensor amax and the finished
 * stage tiles through the workspace; 2 = every CTA quantizes the activations of its own K stages
 * straight into shared memory (the E4M3 amax read from all of x while x is small, else gathered
 * over the grid through the workspace); 3 = the K-splits of each weight tile are launched as one
 * thread-block cluster: the split-K partials (and the E4M3 amax shares) meet in distributed
 * shared memory and no CTA waits on another outside its cluster; each CTA quantizes x for its
 * own stages as in 2 while that is little work (M * stages small), else the separate quantizer
 * runs first.  -1 (the default) = the decode kernel for M = 1, and for MXFP4 layers above 32
 * tokens, else 0 (what measured faster on the B200); where it runs, 3 if the device holds every
 * cluster at once, else 2 or 1, chosen from M, the split and the width.  A forced mode that a launch cannot take
 * falls back to the separate quantizer launch.  Quantized codes are identical in every mode;
 * outputs are identical between modes with the same K split (1 and 2), while mode 3 may split K
 * into fewer parts (its clusters must fit the device at once), which reorders the fp32 split-K
 * sum.  Process-wide; for tests and tuning.  QL_ERR_INVALID_ARG for other values. */
ql_status ql_decode_fuse_mode(int32_t mode);

/* MXFP4 activation quantization with an online block Hadamard in front (CodeQuant, accuracy
 * tables: the "had" variants enable online Hadamard transforms during quantization; the size and
 * algorithm are readings): each 32-element block of x (bf16, device) becomes x . H_32 (Sylvester,
 * unnormalised) computed in fp32 by the Walsh-Hadamard butterfly h = 1, 2, 4, 8, 16, each step
 * (a, b) -> (a + b, a - b) one IEEE fp32 operation; the result is quantized by the
 * QL_A_MXFP4_E8M0_B32 rule of quantize_act.  fmt must be QL_A_MXFP4_E8M0_B32 and had_block 32;
 * K % 32 == 0; codes [M,K/2], E8M0 scales [M,K/32] (device).  The matching weight is
 * W . blockdiag(H_32) / 32, so the layer's product is unchanged. */
ql_status quantize_act_hadamard(ql_aformat fmt, int32_t had_block, const void* x_bf16, int64_t M,
                                int64_t K, void* codes, void* scales, ql_stream_t stream);

/* MXFP4 activation quantization of a PRQuant-reordered activation with its tail appended
 * (PRQuant §4 "Activation tail construction" and "Kernel design for efficient inference": the
 * activation is quantized once and the quantized tail block is appended): x bf16 [M, C] (device);
 * codes [M, (C + k_tail)/2] and E8M0 scales [M, (C + k_tail)/32] (device) hold Q(x) followed by a
 * copy of the codes and scales of its last k_tail channels.  fmt must be QL_A_MXFP4_E8M0_B32;
 * C % 32 == 0, k_tail % 32 == 0, 0 <= k_tail <= C (k_tail = 0 is quantize_act). */
ql_status quantize_act_augmented(ql_aformat fmt, const void* x_bf16, int64_t M, int64_t C,
                                 int32_t k_tail, void* codes, void* scales, ql_stream_t stream);

/* Synchronise `stream` and report (then clear) the device error word. */
ql_status ql_check(ql_stream_t stream);

/* ---- Offline weight preparation (host memory, CPU; not on the forward path) ----------------
 * PRQuant, §4 "Offline scaling and channel reordering" / "Offline residual augmentation", with
 * the AWQ scaling taken as identity: MXFP4-quantize W (bf16 [N,C]) along C; per input channel
 * sum over rows of the squared quantization error; the k largest (ties to the lower index)
 * become the tail; perm lists the kept channels then the tail channels, each ascending;
 * W~ = W[:, perm] is re-quantized; R = W~[:, C-k:] - deq(Q(W~))[:, C-k:] is quantized; the
 * outputs are perm [C] (int32), codes [N,(C+k)/2] and E8M0 bytes [N,(C+k)/32] of Q([W~, R]).
 * Requires C % 128 == 0, k % 128 == 0, 0 < k <= C. */
ql_status qlinear_prepare_prquant(const uint16_t* w_bf16, int64_t N, int64_t C, int32_t k,
                                  int32_t* perm_out, uint8_t* codes_out, uint8_t* scales_out);
/* The same with scale_search = 1: every weight block (the per-column error pass, W~ and R) takes
 * the E8M0-W local block-scale search of PRQuant §5.3 ("PRQuant (E8M0-W)"): per 32-block the
 * OCP exponent e0 and its neighbours e0 + 1 and e0 - 1 (clamped to [-127,127]) are tried in that
 * order with the same element rule, and the block keeps the first with the smallest sum of
 * squared errors (double, element order; a later candidate only if strictly better).
 * scale_search = 0 is qlinear_prepare_prquant. */
ql_status qlinear_prepare_prquant_ex(const uint16_t* w_bf16, int64_t N, int64_t C, int32_t k,
                                     int32_t scale_search, int32_t* perm_out, uint8_t* codes_out,
                                     uint8_t* scales_out);

/* ---- MoE grouped FFN (CodeQuant-style cluster-codebook experts) ----------------------------
 * CodeQuant abstract and Figure 4 (table in SM shared memory); gated FFN of PRQuant's Eq. (1).
 * gate_up: wfmt QL_W_CLUSTER4_ROW16_BF16, N = E*2I rows (per expert: gate rows 0..I-1, then up
 *          rows I..2I-1), K = H; codes = 4-bit indices [N, H/2] (element 2j in the low nibble),
 *          codebooks = bf16 [N][16] centroids.
 * down:    same format, N = E*H rows, K = I.
 * Requirements: E <= 256, top_k <= 16, I % 64 == 0, H % 128 == 0.  Weights are copied (and the
 * gate/up rows reordered for the fused SwiGLU) into library-owned device memory. */
ql_status moe_create(const ql_weight_desc* gate_up, const ql_weight_desc* down, int32_t E,
                     int32_t top_k, ql_stream_t stream, ql_moe** out);
ql_status moe_destroy(ql_moe* moe);
/* When enabled, moe_grouped_forward also writes the fp32 intermediate h (before its MXFP4
 * requantization) into the workspace (for inspection and stage-wise testing). */
ql_status moe_capture_intermediate(ql_moe* moe, int32_t enable);
ql_status moe_workspace_bytes(const ql_moe* moe, int64_t T, size_t* bytes);

/* Byte offsets, inside the workspace, of the forward's stage buffers (SIZE_MAX if absent):
 * counts int[E], offsets int[E+1], entries int[T*k] (routed entries f = t*k+s, expert by expert,
 * ascending f inside an expert), ids int[T,k], gates float[T,k], x_codes [T,H/2], x_scales
 * [T,H/32] (MXFP4 of x), x_dq bf16 [T,H] (its exact values), h_codes [T*k,I/2], h_scales
 * [T*k,I/32] (MXFP4 of h, rows in entry order), h_dq bf16 [T*k,I], h32 float [T*k,I] (only when
 * captured), yslot float [T*k,H] (gate-weighted expert outputs by entry f).  The workspace also
 * holds buffers that are not listed (the bf16 x row of every routed entry, expert-sorted, that
 * the gate/up GEMM reads as contiguous tiles). */
typedef struct ql_moe_ws_layout {
  size_t counts, offsets, entries, ids, gates, x_codes, x_scales, x_dq, h_codes, h_scales, h_dq,
      h32, yslot, total;
} ql_moe_ws_layout;
ql_status moe_workspace_layout(const ql_moe* moe, int64_t T, ql_moe_ws_layout* out);

/* out[T,H] = sum_s gate[t,s] * down_e(MXFP4(silu(gate_e(x_q)) * up_e(x_q))), e = ids[t,s]:
 * router logits fp32 [T,E] (device) -> top-k (descending logit, ties to the lower id), gate
 * weights = softmax of the k logits (fp32); x bf16 [T,H] (device) quantized to MXFP4 E8M0-B32;
 * per expert a grouped bf16 tcgen05 GEMM over its routed tokens with weights decoded from the
 * row codebooks in shared memory; SwiGLU and the MXFP4 requantization of h fused into the
 * gate/up epilogue; the down epilogue writes gate-weighted slot outputs; the slots are summed in
 * slot order.  y bf16 [T,H]; y_f32, ids_out int32 [T,k] and gates_out float [T,k] may be NULL. */
ql_status moe_grouped_forward(const ql_moe* moe, const void* x_bf16, int64_t T,
                              const float* router_logits, void* y_bf16, float* y_f32,
                              int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes,
                              ql_stream_t stream);

/* MXCode PreScale VQ preparation (MXCode abstract: PreScale extracts the MX scales before the
 * codebook is learned; Table 1 row E4M3-B16-FP4).  w_bf16 [N,K]; codebooks = packed E2M1 entries
 * [N/64][K/64][256][2] (entry element 2i in the low nibble of byte i); outputs: the FP32 tensor
 * scale ts = amax(W)/2688 (1 for an all-zero W), E4M3 block scales [N,K/16]
 * (s = E4M3_RNE_satfinite((amax16/6)/ts), fp32 steps), and uint8 indices [N,K/4]: the entry of
 * the row's QBlock nearest (squared distance, exact in double; ties to the lowest index) to
 * W[n,4j:4j+4] / (dec(s)*ts) (0 in a block whose scale is 0).  qn == qk == 64. Host, CPU. */
ql_status qlinear_prepare_vq_prescale(const uint16_t* w_bf16, int64_t N, int64_t K,
                                      const uint8_t* codebooks, int32_t qn, int32_t qk,
                                      float* ts_out, uint8_t* scales_out, uint8_t* idx_out);

/* MXCode PostScale preparation (MXCode abstract: PostScale "quantizes learned codebooks to
 * MXFP4"; reading: one E4M3 scale per QBlock codebook, relative to an FP32 tensor scale over all
 * codebooks, so the decoded weight is an MX-native E4M3-B16 operand with no per-weight scales).
 * w_bf16 [N,K]; centroids = learned codebooks, float [N/64][K/64][256][4] (bf16 values).
 * Outputs: ts = amax(all centroids)/2688 (1 if 0); per QBlock the E4M3 byte
 * s = E4M3_RNE_satfinite((amax(codebook)/6)/ts) (qscales [N/64][K/64]) and the packed E2M1
 * entries code = E2M1_RNE(c / (dec(s)*ts)) (codebooks [N/64][K/64][256][2], element 2i low);
 * indices [N,K/4]: the entry whose decoded value e2m1 * dec(s) * ts is nearest (squared distance
 * in double, ties to the lowest index) to W[n,4j:4j+4].  fp32 steps in that order; qn == qk == 64.
 * Host, CPU. */
ql_status qlinear_prepare_vq_postscale(const uint16_t* w_bf16, int64_t N, int64_t K,
                                       const float* centroids, int32_t qn, int32_t qk,
                                       float* ts_out, uint8_t* codebooks_out,
                                       uint8_t* qscales_out, uint8_t* idx_out);

/* MXCode PreScale+ preparation (MXCode abstract: PreScale's scales "further compressed using VQ";
 * appendix Table 4 caption: Ks = 256, ds = 8).  The PreScale E4M3 block scales of W, 8
 * consecutive along K, become the nearest of the 256 vectors of scale_codebook [256][8] (E4M3
 * bytes; squared distance of decoded values in double, ties to the lowest index); W is then
 * normalised by the compressed scales and assigned to its QBlock codebook as in PreScale.
 * Outputs: ts, the compressed scale bytes [N,K/16], the scale indices [N,K/128] and the weight
 * indices [N,K/4].  K % 128 == 0, qn == qk == 64.  Host, CPU. */
ql_status qlinear_prepare_vq_prescale_plus(const uint16_t* w_bf16, int64_t N, int64_t K,
                                           const uint8_t* codebooks, const uint8_t* scale_codebook,
                                           int32_t qn, int32_t qk, float* ts_out,
                                           uint8_t* scales_out, uint8_t* sidx_out,
                                           uint8_t* idx_out);

/* MosaicQuant-style INT4 dense + block-sparse residual preparation (MosaicQuant, "Dense Base and
 * Sparse Residuals" and "Activation-aware Delta-Hessian Block Selection"; formulas are readings).
 * w_bf16 [N,K] (N % 16 == 0, K % 128 == 0), calibration activations x_calib_bf16 [T,K].
 * Base per (row, 128-group): s = fp16_RNE(amax/7) (fp32 divide), q = clamp(rint(w/s), -7, 7).
 * dW = W - base; block (nb, g) of 16 rows x 128 columns scores sum_rows sum_cols abar_k |dW|
 * (abar_k = mean_t |x[t,k]|; sums in that order, double); the round(density * N/16 * K/128)
 * best blocks (ties to the lower id nb*(K/128)+g) keep a residual quantized per row like the
 * base on fp32(dW).  Outputs: codes [N,K/2] (two's-complement nibbles, element 2j low), fp16
 * scale bits [N,K/128], rowptr int32 [N/16+1], col int16 [nnzb] (group index), residual codes
 * [nnzb][16][64], residual fp16 scale bits [nnzb][16]; nnzb <= capacity. Host, CPU. */
ql_status qlinear_prepare_int4_bsr(const uint16_t* w_bf16, int64_t N, int64_t K,
                                   const uint16_t* x_calib_bf16, int64_t T, float density,
                                   uint8_t* codes_out, uint16_t* scales_out, int32_t* rowptr_out,
                                   int16_t* col_out, uint8_t* rcodes_out, uint16_t* rscales_out,
                                   int32_t capacity, int32_t* nnzb_out);

#ifdef __cplusplus
}
#endif
#endif /* QLINEAR_H_ */
