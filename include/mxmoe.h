/*
 * mxmoe.h -- C ABI of the MXFP8 routed-experts MLP library (libmxmoe.so).
 *
 * What the library computes (the routed-experts MLP of the torchtitan page
 * "Wire the fully-fused grouped-GEMM MXFP8 plan behind fusion_plan", section
 * "What it adds", and the page "fused gated-activation (SwiGLU) + MXFP8
 * quantization kernel override", section "Summary"):
 *
 *   forward   h13 = x_e . W13[e]^T        (FC1 grouped GEMM, per expert e)
 *             h   = silu(gate) * up       (fused SwiGLU + dual MXFP8 quant)
 *             y   = h_e . W2[e]^T         (FC2 grouped GEMM)
 *   backward  dh  = dy_e . W2[e]; dh13 = dSwiGLU(dh, h13)  (fused)
 *             dW2[e] = dy_e^T . h_e, dx = dh13_e . W13[e], dW13[e] = dh13_e^T . x_e
 *
 * around it the token dispatcher (routing to the padded expert-major layout,
 * gather fused with the cast, weighted combine and its gradients; the
 * moe_layer_* composites run the whole token-major layer), the standalone
 * casts and dequantization (E4M3, and E5M2 for the transport payload).
 *
 * MXFP8 format (A2E MXFP8 pages, "quant_mode=4 ... E4M3 ... E8M0 MX scale"):
 * each block of 32 consecutive elements is stored as 32 E4M3 codes (uint8)
 * plus one E8M0 scale byte.  Scale rule (OCP MX v1.0): shared exponent
 * floor(log2(amax)) - 8, byte = clamp(exp + 127, 0, 254); all-zero blocks get
 * byte 0; a block holding NaN/Inf gets byte 0xFF and codes 0x7F|sign.
 * Elements: x / 2^exp rounded to nearest-even E4M3, saturated to +-448.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates device memory (composites take a caller workspace).
 *  - bf16 tensors are passed as void* (IEEE bfloat16, row-major, dense).
 *  - Every call is asynchronous on `stream` and returns an mxmoe_status; on
 *    an error nothing is launched and mxmoe_last_error_message() names the argument.
 *  - ROW quantization: blocks along the last (contiguous) dimension;
 *    COL quantization: blocks over 32 consecutive rows of one column, stored
 *    TRANSPOSED (codes [cols, rows]) so the contraction dimension is contiguous.
 *  - Scale layouts:
 *      MXFP8_SCALE_PLAIN: uint8 [R, ceil(C/32)] row-major for a matrix [R, C].
 *      MXFP8_SCALE_MMA  : the tensor-core layout of a matrix [R, C] with
 *        R % 128 == 0 and C % 128 == 0: 512-byte atoms, atom (R/128, C/128)
 *        at byte ((r/128)*(C/128) + c/128)*512; inside it, the scale of row r
 *        and 32-column block kb = c/32 sits at (r%32)*16 + ((r%128)/32)*4 + kb%4.
 *      Grouped GEMM operands always use MXFP8_SCALE_MMA.
 *  - expert_offsets: DEVICE int32 [E+1], offsets[0] == 0, non-decreasing,
 *    every offset a multiple of pad_multiple (itself a multiple of 128), and
 *    offsets[E] <= M.  Rows at or past offsets[E] are never read or written.
 *    The GEMM kernels re-check this on the device; a bad table makes them do
 *    nothing and raises MXMOE_ERR_OFFSETS in mxmoe_check_device_error().
 */
#ifndef MXMOE_H
#define MXMOE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MXMOE_OK = 0,
  MXMOE_ERR_NULL = 1,           /* a required pointer is NULL                       */
  MXMOE_ERR_SHAPE = 2,          /* a dimension is zero/negative or not a multiple   */
  MXMOE_ERR_ALIGN = 3,          /* a pointer is not 16-byte aligned                  */
  MXMOE_ERR_OFFSETS = 4,        /* expert_offsets table invalid (device-detected)    */
  MXMOE_ERR_ARCH = 5,           /* current device is not sm_100                      */
  MXMOE_ERR_CUDA = 6,           /* a CUDA runtime/driver call failed                 */
  MXMOE_ERR_DEVICE_TIMEOUT = 7, /* a bounded device-side wait expired                */
  MXMOE_ERR_WORKSPACE = 8,      /* workspace missing or too small                    */
  MXMOE_ERR_ARG = 9             /* an enum/flag argument is out of range             */
} mxmoe_status;

#define MXFP8_ROW 1
#define MXFP8_COL 2
#define MXFP8_SCALE_PLAIN 0
#define MXFP8_SCALE_MMA 1

/* Text of the last host-side error of the calling thread ("" if none). */
const char* mxmoe_last_error_message(void);

/* Device-side error word of the current device.  Kernels set it when they
 * find a bad table (GEMMs: an offsets table -> MXMOE_ERR_OFFSETS; route: an
 * expert id outside [0, E) -> MXMOE_ERR_ARG, a layout past m_cap ->
 * MXMOE_ERR_SHAPE; gather/combine: a slot or row out of range ->
 * MXMOE_ERR_OFFSETS) or when a bounded mbarrier wait expires
 * (MXMOE_ERR_DEVICE_TIMEOUT).
 * Synchronizes `stream`, returns the first error code recorded (MXMOE_OK if
 * none) in *code and, if reset != 0, clears it.  Returns MXMOE_ERR_CUDA if
 * the read itself failed. */
int mxmoe_check_device_error(cudaStream_t stream, int reset, int* code);

/* Library version string. */
const char* mxmoe_version(void);

/* Self-test of the failure path: launches one thread that waits, with the
 * same bounded mbarrier wait the GEMM and cast kernels use, on a barrier that
 * nothing ever arrives on.  After the wait limit (about 2^32 SM cycles, ~2 s)
 * the kernel records MXMOE_ERR_DEVICE_TIMEOUT in the device error word and
 * returns normally, leaving the context usable; read it with
 * mxmoe_check_device_error(). */
int mxmoe_selftest_wait_timeout(cudaStream_t stream);

/* -------------------------------------------------------------------------
 * mxfp8_quantize -- bf16 -> MXFP8 cast, row-wise and/or column-wise.
 * (Standalone cast kernels of the SwiGLU-boundary page, "Summary": the
 * unfused path launches 6 + 6 of them per MLP; A2E MXFP8 page: the
 * attention side quantizes the activation so "the payload halves".)
 *
 *  x        bf16 [batch, rows, cols]
 *  modes    MXFP8_ROW | MXFP8_COL (at least one)
 *  ROW out  row_codes  uint8 [batch, rows, cols];
 *           row_scales PLAIN [batch*rows, ceil(cols/32)] (short last block
 *           allowed when cols % 32 != 0) or MMA layout of [batch*rows, cols].
 *  COL out  col_codes  uint8 [batch, cols, rows] (each batch transposed);
 *           col_scales PLAIN [batch*cols, rows/32] or MMA layout of the
 *           [batch*cols, rows] matrix.  Needs rows % 32 == 0.
 *  MMA layout needs rows % 128 == 0 and cols % 128 == 0.
 * Unused output pointers may be NULL.
 * ------------------------------------------------------------------------- */
int mxfp8_quantize(const void* x, int64_t batch, int64_t rows, int64_t cols,
                   int modes, int scale_layout,
                   uint8_t* row_codes, uint8_t* row_scales,
                   uint8_t* col_codes, uint8_t* col_scales,
                   cudaStream_t stream);

/* mxfp8_quantize with E5M2 elements (A2E transport page, "quant_mode=4": the
 * activation is quantized to E4M3 or E5M2 with its E8M0 block scale).  Same
 * arguments, layouts and rules; the block exponent is floor(log2(amax)) - 15
 * (15 = largest E5M2 exponent), elements round to nearest-even E5M2 and
 * saturate at +-57344; NaN/Inf blocks get byte 0xFF and codes 0x7F | sign. */
int mxfp8_quantize_e5m2(const void* x, int64_t batch, int64_t rows, int64_t cols,
                        int modes, int scale_layout,
                        uint8_t* row_codes, uint8_t* row_scales,
                        uint8_t* col_codes, uint8_t* col_scales,
                        cudaStream_t stream);

/* -------------------------------------------------------------------------
 * mxfp8_swiglu_quant -- fused SwiGLU + dual MXFP8 quantization.
 * (SwiGLU-boundary page, "Summary": fused SwiGLU + dual MXFP8 quantization;
 * the bf16 post-activation is never materialized.)
 *
 *  h13   bf16 [rows, 2F]; columns 0..F-1 gate (a), F..2F-1 up (b)
 *  h     = bf16(silu(a) * b) computed in fp32, never written to memory
 *  outputs as mxfp8_quantize of h [rows, F] with batch = 1.
 *  Needs F % 32 == 0; COL needs rows % 32 == 0; MMA layout needs rows and F
 *  multiples of 128.
 * ------------------------------------------------------------------------- */
int mxfp8_swiglu_quant(const void* h13, int64_t rows, int64_t F,
                       int modes, int scale_layout,
                       uint8_t* row_codes, uint8_t* row_scales,
                       uint8_t* col_codes, uint8_t* col_scales,
                       cudaStream_t stream);

/* -------------------------------------------------------------------------
 * mxfp8_dequantize -- MXFP8 (ROW, PLAIN scales) -> bf16.
 * (A2E transport page, review "[P2] Handle the two E8M0 endpoint encodings":
 * byte 0x00 is 2^-127, byte 0xFF is NaN.)  out = bf16(code * 2^(byte-127)).
 *  codes [rows, cols], scales [rows, ceil(cols/32)], out bf16 [rows, cols].
 * ------------------------------------------------------------------------- */
int mxfp8_dequantize(const uint8_t* codes, const uint8_t* scales,
                     int64_t rows, int64_t cols, void* out, cudaStream_t stream);

/* mxfp8_dequantize for E5M2 codes (+-infinity codes stay infinite, NaN codes
 * give NaN). */
int mxfp8_dequantize_e5m2(const uint8_t* codes, const uint8_t* scales,
                          int64_t rows, int64_t cols, void* out, cudaStream_t stream);

/* -------------------------------------------------------------------------
 * mxfp8_grouped_gemm -- ragged-M grouped GEMM (FC2 / dgrad form).
 * (Fully-fused plan page, "What it adds": FC2 GEMM.)
 *
 *  out[m, n] = sum_k A[m, k] * W[e, n, k] for offsets[e] <= m < offsets[e+1],
 *  with both operands dequantized from MXFP8 and accumulated in fp32 on the
 *  tensor cores; out is bf16 [M, N] (rows >= offsets[E] untouched).
 *  a, a_scales : codes [M, K], MMA scales of [M, K]
 *  w, w_scales : codes [E, N, K], MMA scales of [E*N, K]
 *  Needs M, N, K multiples of 128.
 * ------------------------------------------------------------------------- */
int mxfp8_grouped_gemm(const uint8_t* a, const uint8_t* a_scales, int64_t M, int64_t K,
                       const uint8_t* w, const uint8_t* w_scales, int E, int64_t N,
                       const int32_t* expert_offsets, int pad_multiple,
                       void* out, cudaStream_t stream);

/* -------------------------------------------------------------------------
 * mxfp8_grouped_gemm_wgrad -- ragged-K grouped GEMM (weight gradients).
 * (Fully-fused plan page, "What it adds": wgrad; "Evidence": zero-token
 * experts give exact-zero grads.)
 *
 *  dw[e, n, j] = sum over m in expert e's rows of G[m, n] * X[m, j]
 *  gt, gt_scales : COL codes of G, [N, M], MMA scales of [N, M]
 *  xt, xt_scales : COL codes of X, [Kx, M], MMA scales of [Kx, M]
 *  dw            : bf16 [E, N, Kx]; an expert with no rows gets exact zeros.
 *  expert_rows   : DEVICE int32 [E] or NULL.  The number of token rows at the
 *                  head of each expert's segment, the rest being padding
 *                  (0 <= expert_rows[e] <= offsets[e+1] - offsets[e], else
 *                  nothing is written and MXMOE_ERR_OFFSETS is raised on the
 *                  device).  The padding's 128-row K blocks are then skipped:
 *                  the sum runs over the token rows only (with zero pad rows,
 *                  as the route and gather produce, the result is the same).
 *  Needs N, Kx, M multiples of 128.
 * ------------------------------------------------------------------------- */
int mxfp8_grouped_gemm_wgrad(const uint8_t* gt, const uint8_t* gt_scales, int64_t N,
                             const uint8_t* xt, const uint8_t* xt_scales, int64_t Kx,
                             int64_t M, const int32_t* expert_offsets, const int32_t* expert_rows,
                             int E, int pad_multiple, void* dw, cudaStream_t stream);

/* -------------------------------------------------------------------------
 * mxfp8_grouped_gemm_swiglu_quant -- FC1 grouped GEMM with the SwiGLU + dual
 * quantization epilogue in one launch (fully-fused plan page, "What it adds":
 * "FC1 grouped GEMM + SwiGLU + dual MXFP8 quantization in one launch").
 *
 *  h13 = x_e . W13[e]^T (fp32 accumulate, rounded to bf16), h = bf16(silu(a)*b)
 *  a, a_scales     : x codes [M, K], MMA scales
 *  w13, w13_scales : codes [E, 2F, K] (rows 0..F-1 gate, F..2F-1 up), MMA scales of [E*2F, K]
 *  h13_out         : bf16 [M, 2F] (saved for the backward), may be NULL
 *  h_row_codes/scales : [M, F], MMA scales of [M, F]    (FC2 operand)
 *  h_col_codes/scales : [F, M], MMA scales of [F, M]    (dW2 operand)
 *  Needs M, K, F multiples of 128.
 * ------------------------------------------------------------------------- */
int mxfp8_grouped_gemm_swiglu_quant(const uint8_t* a, const uint8_t* a_scales,
                                    int64_t M, int64_t K,
                                    const uint8_t* w13, const uint8_t* w13_scales,
                                    int E, int64_t F,
                                    const int32_t* expert_offsets, int pad_multiple,
                                    void* h13_out,
                                    uint8_t* h_row_codes, uint8_t* h_row_scales,
                                    uint8_t* h_col_codes, uint8_t* h_col_scales,
                                    cudaStream_t stream);

/* -------------------------------------------------------------------------
 * mxfp8_grouped_gemm_dswiglu_quant -- FC2 dgrad with the fused dSwiGLU +
 * dual quantization epilogue (fully-fused plan page: "fused dSwiGLU backward").
 *
 *  dh = bf16(dy_e . W2[e]) (contraction over D), then with a, b from h13:
 *  s = sigmoid(a); dgate = dh*b*s*(1 + a*(1-s)); dup = dh*a*s (fp32, -> bf16)
 *  dy, dy_scales   : codes [M, D], MMA scales
 *  w2t, w2t_scales : COL codes of W2 per expert, [E, F, D], MMA scales of [E*F, D]
 *  h13             : bf16 [M, 2F] saved by the forward
 *  g_row_codes/scales : dh13 codes [M, 2F], MMA scales of [M, 2F]   (dx operand)
 *  g_col_codes/scales : dh13 codes [2F, M], MMA scales of [2F, M]   (dW13 operand)
 *  Needs M, D, F multiples of 128.
 * ------------------------------------------------------------------------- */
int mxfp8_grouped_gemm_dswiglu_quant(const uint8_t* dy, const uint8_t* dy_scales,
                                     int64_t M, int64_t D,
                                     const uint8_t* w2t, const uint8_t* w2t_scales,
                                     int E, int64_t F,
                                     const int32_t* expert_offsets, int pad_multiple,
                                     const void* h13,
                                     uint8_t* g_row_codes, uint8_t* g_row_scales,
                                     uint8_t* g_col_codes, uint8_t* g_col_scales,
                                     cudaStream_t stream);

/* -------------------------------------------------------------------------
 * Composites.  All buffers caller-owned.  x, dy: bf16 [M, D] (pad rows zero);
 * w13: bf16 [E, 2F, D]; w2: bf16 [E, D, F].  The saved tensors are what the
 * backward needs: h13 (bf16 [M, 2F]), the COL-quantized h ([F, M] codes + MMA
 * scales) and the COL-quantized x ([D, M] codes + MMA scales).  The bf16
 * post-activation h is never written.
 * Workspace: mxmoe_workspace_size(which = 1 fwd, 2 bwd) bytes, 256-aligned.
 * ------------------------------------------------------------------------- */
typedef struct {
  void* h13;               /* bf16 [M, 2F]                     */
  uint8_t* h_col_codes;    /* [F, M]                            */
  uint8_t* h_col_scales;   /* MMA scales of [F, M]              */
  uint8_t* x_col_codes;    /* [D, M]                            */
  uint8_t* x_col_scales;   /* MMA scales of [D, M]              */
} mxmoe_saved;

/* Workspace bytes: which = 1 moe_mlp_fwd, 2 moe_mlp_bwd, 3 moe_mlp_fwd_q,
 * 4 moe_mlp_bwd_q (0 for bad arguments). */
size_t mxmoe_workspace_size(int64_t M, int64_t D, int E, int64_t F, int which);

int moe_mlp_fwd(const void* x, int64_t M, int64_t D,
                const void* w13, const void* w2, int E, int64_t F,
                const int32_t* expert_offsets, int pad_multiple,
                void* y, const mxmoe_saved* saved,
                void* workspace, size_t workspace_bytes, cudaStream_t stream);

int moe_mlp_bwd(const void* dy, int64_t M, int64_t D,
                const void* w13, const void* w2, int E, int64_t F,
                const int32_t* expert_offsets, int pad_multiple,
                const mxmoe_saved* saved,
                void* dx, void* dw13, void* dw2,
                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* -------------------------------------------------------------------------
 * Pre-quantized weights.  A training step uses every weight in both passes
 * (ROW-quantized along D resp. F in the forward, COL-quantized along 2F resp.
 * D in the backward); mxmoe_quantize_weights produces all four with one dual
 * (ROW + COL) cast per weight, i.e. one read of each bf16 weight per step, and
 * the _q composites consume them instead of re-casting the bf16 weights.
 * All buffers caller-owned device memory; scales in the MMA layout.
 * ------------------------------------------------------------------------- */
typedef struct {
  uint8_t* w13_codes;     /* ROW of W13: [E, 2F, D]            (FC1 operand)  */
  uint8_t* w13_scales;    /* MMA scales of [E*2F, D]                          */
  uint8_t* w13t_codes;    /* COL of each W13[e]: [E, D, 2F]    (dx operand)   */
  uint8_t* w13t_scales;   /* MMA scales of [E*D, 2F]                          */
  uint8_t* w2_codes;      /* ROW of W2: [E, D, F]              (FC2 operand)  */
  uint8_t* w2_scales;     /* MMA scales of [E*D, F]                           */
  uint8_t* w2t_codes;     /* COL of each W2[e]: [E, F, D]      (dh operand)   */
  uint8_t* w2t_scales;    /* MMA scales of [E*F, D]                           */
} mxmoe_qweights;

int mxmoe_quantize_weights(const void* w13, const void* w2, int E, int64_t D, int64_t F,
                           const mxmoe_qweights* qw, cudaStream_t stream);

/* moe_mlp_fwd / moe_mlp_bwd with the weights given pre-quantized (the
 * forward reads the ROW fields of qw, the backward the COL fields). */
int moe_mlp_fwd_q(const void* x, int64_t M, int64_t D, const mxmoe_qweights* qw, int E, int64_t F,
                  const int32_t* expert_offsets, int pad_multiple,
                  void* y, const mxmoe_saved* saved,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* moe_mlp_fwd_unfused_q -- the unfused ("swiglu" plan) forward, the baseline
 * of the fully-fused plan page ("Performance": +2.3 % / +5.0 % tokens/s over
 * the pad-matched unfused MXFP8 baseline): FC1 grouped GEMM to a bf16 h13 in
 * HBM, the standalone SwiGLU + dual quantization kernel, FC2.  Same arguments,
 * outputs and workspace (which = 3) as moe_mlp_fwd_q; bitwise equal results. */
int moe_mlp_fwd_unfused_q(const void* x, int64_t M, int64_t D, const mxmoe_qweights* qw, int E, int64_t F,
                          const int32_t* expert_offsets, int pad_multiple,
                          void* y, const mxmoe_saved* saved,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream);

int moe_mlp_bwd_q(const void* dy, int64_t M, int64_t D, const mxmoe_qweights* qw, int E, int64_t F,
                  const int32_t* expert_offsets, int pad_multiple,
                  const mxmoe_saved* saved,
                  void* dx, void* dw13, void* dw2,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* -------------------------------------------------------------------------
 * moe_mlp_fwd_noalloc -- moe_mlp_fwd for callers that cannot allocate.
 * (No counterpart in the source pages: this is a library-integration entry.)
 *
 * Some callers have no way to obtain device memory at call time: code that
 * runs inside a host framework whose memory is fully owned by its own pool
 * (an inference-server plugin, a runtime that forbids cudaMalloc after
 * start-up because it would synchronize the device or fragment the pool), or
 * a caller with a fixed memory budget that cannot reserve a workspace of
 * data-dependent size.  This entry point takes the same arguments as
 * moe_mlp_fwd minus the workspace and uses instead a scratch area compiled
 * into the library: a file-scope device array of MXMOE_NOALLOC_SCRATCH_BYTES
 * (32 MiB) that every GPU loading the library holds until the process exits.
 * It never calls cudaMalloc/cudaFree or any allocating routine.
 *
 *  - Layers whose forward workspace (mxmoe_workspace_size(..., 1)) exceeds the
 *    scratch size are rejected with MXMOE_ERR_WORKSPACE and a message giving
 *    both sizes; nothing is launched.
 *  - The first call on a device looks up the device address of the scratch
 *    array (cudaGetSymbolAddress, with that device current); make that first
 *    call before any CUDA stream capture begins.  The address is kept per
 *    device and CUDA context: after cudaDeviceReset, or under another
 *    context, the next call looks it up again (again outside any capture).
 *  - All calls on a device share the one scratch area, which keeps whatever
 *    the previous call left there (every byte a call reads is written by that
 *    call first).  Calls whose executions overlap on the GPU (different
 *    streams without ordering, or concurrent host threads) race on it:
 *    serialize them.
 *  - Inputs, outputs and `saved` are caller-owned exactly as for moe_mlp_fwd.
 * ------------------------------------------------------------------------- */
#define MXMOE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

int moe_mlp_fwd_noalloc(const void* x, int64_t M, int64_t D,
                        const void* w13, const void* w2, int E, int64_t F,
                        const int32_t* expert_offsets, int pad_multiple,
                        void* y, const mxmoe_saved* saved, cudaStream_t stream);

/* -------------------------------------------------------------------------
 * Token dispatcher around the MLP.
 *
 * The fully-fused plan page ("What it adds") installs a dispatcher that pads
 * each expert's token rows to a multiple of pad_multiple, and the
 * SwiGLU-boundary page ("Usage") has it produce the padded expert-major
 * layout the kernels consume.  Slot s = t*top_k + j is token t's j-th routed
 * copy, sent to expert topk_ids[s].  Expert e's segment
 * [offsets[e], offsets[e+1]) lists its slots in ascending slot order
 * (ascending token order), then pad rows up to the next multiple of
 * pad_multiple; an expert with no slot has an empty segment.
 *
 *   forward   rows   = permute(x)               row m <- x[row_slot[m] / top_k]
 *             out[t] = sum_j w[t,j] * y[slot_row[t*top_k + j]]    (combine)
 *   backward  dy[row(t,j)] = bf16(w[t,j] * dout[t])               (permute, weighted)
 *             dw[t,j]      = <dout[t], y[row(t,j)]>              (combine_weight_grad)
 *             dx_tok[t]    = sum_j dx[row(t,j)]                  (combine, no weights)
 * ------------------------------------------------------------------------- */

/* Rows a layout can need: T*top_k real rows plus at most pad_multiple-1 pad
 * rows for each expert that receives a slot, rounded up to a multiple of 128
 * (the grouped GEMMs' row tile).  Host-only arithmetic; returns -1 for
 * non-positive or overflowing arguments. */
int64_t mxmoe_route_capacity(int64_t T, int top_k, int E, int pad_multiple);

/* Bytes of device workspace mxmoe_route needs: 4 * E * ceil(T*top_k / 4096). */
size_t mxmoe_route_workspace_size(int64_t T, int top_k, int E);

/* Build the padded expert-major layout from a top-k routing (three kernels:
 * per-chunk histogram, padded scan, stable ranking).
 *   topk_ids  DEVICE int32 [T, top_k], ids in [0, E) (ids outside raise
 *             MXMOE_ERR_ARG in mxmoe_check_device_error and their slot gets row -1)
 *   E <= 1024, pad_multiple >= 1, T*top_k < 2^31
 *   m_cap     rows of row_slot (use mxmoe_route_capacity); a routing that
 *             needs more raises MXMOE_ERR_SHAPE on the device and rows past
 *             m_cap are not written
 *   offsets   DEVICE int32 [E+1] out: offsets[0] = 0, offsets[E] = M
 *   row_slot  DEVICE int32 [m_cap] out: slot of each row, -1 for pad rows and
 *             for rows [M, m_cap)
 *   slot_row  DEVICE int32 [T*top_k] out: row of each slot
 * The result is deterministic (a stable counting sort). */
int mxmoe_route(const int32_t* topk_ids, int64_t T, int top_k, int E, int pad_multiple, int64_t m_cap,
                int32_t* offsets, int32_t* row_slot, int32_t* slot_row,
                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Gather token rows into the layout and MXFP8-quantize them in the same pass
 * (the x cast of the forward, and with slot_weights the dY cast of the
 * backward): row m is x_tokens[row_slot[m] / top_k] ([T, D] bf16), zero when
 * row_slot[m] < 0; with slot_weights (DEVICE fp32 [T*top_k], may be NULL)
 * it is bf16(slot_weights[s] * x) with one fp32 product per element.
 *   m_cap % 128 == 0 and D % 128 == 0 with MXFP8_SCALE_MMA, D % 32 == 0 and
 *   m_cap % 32 == 0 otherwise; x_tokens 16-byte aligned.
 *   rows_dev  DEVICE int32* (may be NULL), e.g. offsets + E: rows at or past
 *             *rows_dev are neither read nor written
 *   outputs   as mxfp8_quantize for a [m_cap, D] matrix (COL codes [D, m_cap]).
 * A slot >= T*top_k in row_slot raises MXMOE_ERR_OFFSETS and that row reads as
 * zero. */
int mxmoe_permute_quant(const void* x_tokens, int64_t T, int64_t D, const int32_t* row_slot, int top_k,
                        const float* slot_weights, int64_t m_cap, const int32_t* rows_dev,
                        int modes, int scale_layout,
                        uint8_t* row_codes, uint8_t* row_scales,
                        uint8_t* col_codes, uint8_t* col_scales, cudaStream_t stream);

/* out[t] = bf16( sum_j w[t*top_k+j] * y[slot_row[t*top_k+j]] ), fp32
 * accumulation in j order; w = 1 when slot_weights is NULL.  y [m_rows, D]
 * bf16, out [T, D] bf16, D % 8 == 0, top_k <= 64, 16-byte aligned y/out.
 * slot_row entries of -1 contribute nothing; entries >= m_rows raise
 * MXMOE_ERR_OFFSETS and contribute nothing. */
int mxmoe_unpermute_combine(const void* y, int64_t m_rows, int64_t D, const int32_t* slot_row,
                            const float* slot_weights, int64_t T, int top_k, void* out, cudaStream_t stream);

/* dweights[t*top_k+j] = <dout[t], y[slot_row[t*top_k+j]]> in fp32 (0 for a
 * slot whose row is -1).  dout [T, D] bf16, y [m_rows, D] bf16, D % 8 == 0,
 * 16-byte aligned. */
int mxmoe_combine_weight_grad(const void* dout, const void* y, int64_t m_rows, int64_t D,
                              const int32_t* slot_row, int64_t T, int top_k, float* dweights,
                              cudaStream_t stream);

/* -------------------------------------------------------------------------
 * Token-major layer composites: the dispatcher around the MLP.
 * (Fully-fused plan page, "What it adds": the padded dispatcher feeding the
 * four fused ops; SwiGLU-boundary page, "Usage".)
 *
 * Forward:  route topk_ids -> padded layout (saved tables); gather x_tokens
 *           into it fused with the x cast (ROW + COL); FC1 + SwiGLU + dual
 *           quant; FC2 -> saved y rows; weighted combine -> out_tokens.
 * Backward: gather dout_tokens scaled by the router weights fused with the
 *           dY cast; FC2 dgrad + dSwiGLU + dual quant; dW2; dx rows; dW13;
 *           dx_tokens = sum of a token's dx rows; dweights = <dout, y rows>.
 *           The weight gradients take each expert's token-row count from the
 *           saved route tables and skip the all-padding K blocks.
 *
 * The layout capacity is m_cap = mxmoe_route_capacity(T, top_k, E,
 * pad_multiple); every row buffer below has m_cap rows and only the rows
 * below offsets[E] (known on the device) are touched.  Needs D, F multiples
 * of 128, pad_multiple a multiple of 128, 1 <= top_k <= min(64, E),
 * E <= 1024.  Weights come from mxmoe_quantize_weights (ROW copies for the
 * forward, COL copies for the backward).  topk_weights: fp32 [T, top_k].
 * ------------------------------------------------------------------------- */
typedef struct {
  int32_t* offsets;    /* [E+1] */
  int32_t* row_slot;   /* [m_cap] */
  int32_t* slot_row;   /* [T*top_k] */
  void* y;             /* bf16 [m_cap, D]: FC2 output rows (the combine's input) */
  mxmoe_saved mlp;     /* h13 [m_cap, 2F], h COL, x COL, each with m_cap rows */
} mxmoe_layer_saved;

/* which = 1: forward workspace, 2: backward workspace (bytes; 0 on bad sizes). */
size_t moe_layer_workspace_size(int64_t T, int top_k, int64_t D, int E, int64_t F, int pad_multiple, int which);

int moe_layer_fwd_q(const void* x_tokens, int64_t T, int64_t D, const int32_t* topk_ids,
                    const float* topk_weights, int top_k, const mxmoe_qweights* qw, int E, int64_t F,
                    int pad_multiple, void* out_tokens, const mxmoe_layer_saved* saved,
                    void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* dweights (fp32 [T, top_k]) may be NULL. */
int moe_layer_bwd_q(const void* dout_tokens, int64_t T, int64_t D, const float* topk_weights, int top_k,
                    const mxmoe_qweights* qw, int E, int64_t F, int pad_multiple,
                    const mxmoe_layer_saved* saved, void* dx_tokens, void* dw13, void* dw2, float* dweights,
                    void* workspace, size_t workspace_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MXMOE_H */
