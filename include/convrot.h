/*
 * convrot.h - C ABI of libconvrot.so: ConvRot W8A8 / W4A8 INT8 linear layers
 * for NVIDIA B200 (sm_100a).
 *
 * The method, as the model cards describe it:
 *  - "MOSS-Image Qwen3.5-9B text encoder, INT8 (W8A8, ConvRot)", file table:
 *    the "Quantized" row (each weight rotated per 256-column group by a
 *    Hadamard matrix, int8 with one fp32 weight_scale per output row), the
 *    "Matmul" row (the input is rotated by the same Hadamard and rounded to
 *    int8 per token; W8A8 matmul) and the "Changed" row plus "How it was made"
 *    (fp32 RMSNorm weights carrying SmoothQuant scales folded as (1+w)/s - 1).
 *  - "Qwen3.5 INT8 ConvRot Text Encoders for ComfyUI", "Why ConvRot" and
 *    "Quantization Recipe": group-wise Hadamard, group 256, row scaling.
 *  - "Qwen3-VL-8B-Heretic-1.3.0 - INT8 ConvRot (ComfyUI)", "Quantization
 *    metadata": convrot true, convrot_groupsize 256, per_row true.
 *  - "Qwen3-VL 8B - INT8 ConvRot", "Layer and group selection": widths the
 *    group does not divide fall back to plain row-wise INT8 (group = 0 here);
 *    the vision tower's widths 1152 and 4304 use 16-point groups instead
 *    ("Original version conversion": vision ConvRot group size 16).
 *  - "MossInt4", "Format": the convrot_w4a4 layout (signed 4-bit codes, two
 *    per byte, one F32 scale per row from a per-row clip search, 8-bit
 *    activations).
 *
 * Notation: x [M, K] activations (one row per token), W [N, K] the linear's
 * weight (out, in), G = 256 the group size, H = H_256 / 16 the Sylvester
 * Hadamard matrix (entry (i, j) = (-1)^popcount(i & j) / 16), R the
 * block-diagonal matrix of K / G copies of H.
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers unless stated; the caller allocates and owns
 *    every buffer.  The library allocates no device memory.
 *  - Every tensor is contiguous and row-major with the shapes given; bf16
 *    tensors are passed as void* holding IEEE bfloat16 bit patterns.
 *  - Matrices (x, W, Xq, Wq, Wq4, Y, acc) and the per-column vectors
 *    (norm_w, col_scale) must be 16-byte aligned; per-row scale vectors
 *    (s_tok, s_row) 4-byte aligned; workspaces 256-byte aligned.
 *  - Work is enqueued on `stream` (NULL = legacy default stream) and runs
 *    asynchronously; no call synchronises the stream.  The per-token kernels
 *    (convrot_rotate_quant_act, the linears and GEMMs) are launched with
 *    programmatic dependent launch: their set-up may overlap the end of the
 *    previous kernel on the stream, and each waits for that kernel to
 *    complete before it reads or writes any memory, so stream order holds.
 *  - Arguments are validated on the host before anything is enqueued; on a
 *    validation error nothing is launched.  M = 0 (or N = 0) returns
 *    CONVROT_OK without launching.  A failed launch returns CONVROT_ERR_CUDA.
 *  - Kernels bound every wait they perform; a wait that runs out sets a
 *    device-side error word (read with convrot_device_status) and the kernel
 *    returns early instead of hanging.
 *  - No exceptions cross this interface.
 */
#ifndef CONVROT_H
#define CONVROT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* convrot_stream_t;

typedef enum {
  CONVROT_OK = 0,
  CONVROT_ERR_NULL = 1,            /* a required pointer is NULL */
  CONVROT_ERR_SHAPE = 2,           /* a size is negative, too large or not a required multiple */
  CONVROT_ERR_ALIGN = 3,           /* a pointer is not aligned as required */
  CONVROT_ERR_UNSUPPORTED = 4,     /* e.g. a group size other than 0, 16 or 256 */
  CONVROT_ERR_CUDA = 5,            /* a CUDA runtime or driver call failed */
  CONVROT_ERR_DEVICE_TIMEOUT = 6,  /* a kernel gave up on a bounded wait */
  CONVROT_ERR_WORKSPACE = 7        /* workspace missing or smaller than required */
} convrot_status;

/* Largest supported input width: |acc| <= 127 * 127 * K must fit in int32. */
#define CONVROT_MAX_K 131072

/* Version of this interface, (major << 16) | minor. */
int convrot_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* convrot_status_string(convrot_status st);

/*
 * Reads and clears the device error word after synchronising `stream`.
 * Returns CONVROT_OK if no kernel has reported a problem since the last call,
 * CONVROT_ERR_DEVICE_TIMEOUT if one gave up on a bounded wait, or
 * CONVROT_ERR_CUDA if the synchronisation itself failed.  If detail is not
 * NULL it receives the raw error word (0 when clean).
 */
convrot_status convrot_device_status(convrot_stream_t stream, uint32_t* detail);

/*
 * Diagnostic (no counterpart on the pages): the failure path of the bounded
 * waits, exercised without a fault.  Enqueues one small kernel whose mbarrier
 * wait is made to run out (nothing arrives on the barrier); after about
 * `limit_cycles` SM cycles the wait records a timeout in the device error word
 * (bit 0, wait site 15 in bits 8..15) and the kernel returns.  A following
 * convrot_device_status reports CONVROT_ERR_DEVICE_TIMEOUT with that detail.
 * limit_cycles must lie in [1000, 100000000] (else CONVROT_ERR_SHAPE, nothing
 * launched); the kernel may run up to ~1.5 ms longer than the limit.
 */
convrot_status convrot_selftest_wait_timeout(uint32_t limit_cycles, convrot_stream_t stream);

/* --------------------------------------------------------------------------
 * Offline weight preparation (not on the per-token path).
 * ------------------------------------------------------------------------ */

/*
 * ConvRot int8 weight ("Quantized" row of the MOSS-Image card's file table;
 * "Quantization Recipe": --int8 --scaling_mode row --simple --convrot
 * --convrot-group-size 256).
 *   W' = (W * diag(col_scale)) * R           (col_scale NULL = all ones;
 *                                             group 0 = no rotation)
 *   s_row[n] = max_k |W'[n,k]| / 127          (fp32; 0 for an all-zero row)
 *   Wq[n,k]  = clamp(rint(W'[n,k] / s_row[n]), -127, 127), round-half-even
 * W      bf16 [N, K]            in
 * col_scale fp32 [K] or NULL    in   SmoothQuant scale s folded into the weight
 * Wq     int8 [N, K]            out
 * s_row  fp32 [N]               out
 * group  256 (K % 256 == 0), 16 (K % 16 == 0; H = H_16 / 4 per 16 columns)
 *        or 0 (no rotation, K % 16 == 0)
 */
convrot_status convrot_quantize_weight(const void* W, int N, int K, int group,
                                       const float* col_scale, int8_t* Wq, float* s_row,
                                       convrot_stream_t stream);

/*
 * convrot_w4a4 weight layout ("MossInt4", "Format").
 *   W' as above; for each row and each clip c_i = clip_lo + (clip_hi - clip_lo)
 *   * i / (clip_steps - 1), i = 0 .. clip_steps-1:
 *     s = c_i * max|W'| / 7, q = clamp(rint(W'/s), -7, 7),
 *     err = sum_k (W' - s q)^2;
 *   the smallest err wins (the smaller c on ties); s_row = that s.
 * Wq4    uint8 [N, K/2]  out   byte j of a row holds code 2j in bits 0-3 and
 *                              code 2j+1 in bits 4-7, two's complement
 * s_row  fp32 [N]        out
 * group 256, 16 or 0 as convrot_quantize_weight; K % 32 == 0 (and K % 256 == 0
 * when group == 256); 1 <= clip_steps <= 64.
 */
convrot_status convrot_quantize_weight_w4(const void* W, int N, int K, int group,
                                          const float* col_scale, float clip_lo,
                                          float clip_hi, int clip_steps, uint8_t* Wq4,
                                          float* s_row, convrot_stream_t stream);

/*
 * SmoothQuant scales for a norm-carrying linear (MOSS-Image card, "How it was
 * made": alpha 0.5, folded into the preceding RMSNorm as (1 + w) / s - 1).
 *   a = x * (mean_k x^2 + eps)^(-1/2) * (1 + norm_w)     (the linear's input)
 *   smooth[c] = clamp(max_m |a[m,c]|^alpha / max_n |W[n,c]|^(1-alpha), 1e-5, 1e5)
 *              (1 where the activation or weight column is all zero)
 *   norm_w_folded[c] = (1 + norm_w[c]) / smooth[c] - 1
 * The weight is then prepared with col_scale = smooth.
 * x bf16 [M, K], norm_w fp32 [K], W bf16 [N, K] in; smooth, norm_w_folded
 * fp32 [K] out; norm_w_folded must not alias norm_w (both outputs are
 * used as scratch for the column maxima before the final values are written).
 * norm_w may be NULL for a linear without a preceding norm (down_proj, whose
 * input is the MLP's SiLU(gate) * up): then a = x, the scales are folded into
 * the rows that produce x instead (convrot_fold_row_scales), and
 * norm_w_folded is scratch only (its contents on return are unspecified).
 * K % 16 == 0.
 */
convrot_status convrot_smoothquant_calibrate(const void* x, int M, int K, const float* norm_w,
                                             float eps, const void* W, int N, float alpha,
                                             float* smooth, float* norm_w_folded,
                                             convrot_stream_t stream);

/* --------------------------------------------------------------------------
 * Per-token path.
 * ------------------------------------------------------------------------ */

/*
 * Activation rotate-and-quantise ("Matmul" row of the MOSS-Image card's file
 * table), with an optional fused RMSNorm ("Changed" row; "How it was made").
 *   u = x * (1 + norm_w)                      (norm_w NULL: u = x, no norm)
 *   r = (mean_k x^2 + eps)^(-1/2)             (1 without norm)
 *   v = r * u * R                             (group 0: no rotation)
 *   s_tok[m] = max_k |v[m,k]| / 127           (0 for an all-zero row)
 *   Xq[m,k]  = clamp(rint(v[m,k] / s_tok[m]), -127, 127), round-half-even
 * x bf16 [M, K] in, norm_w fp32 [K] or NULL in, Xq int8 [M, K] out,
 * s_tok fp32 [M] out.  group 256 (K % 256 == 0), 16 or 0 (K % 16 == 0).
 * The rotation is computed in fp32 registers; codes can differ from an exact
 * evaluation only where v / s_tok lies within fp32 rounding of a tie.
 */
convrot_status convrot_rotate_quant_act(const void* x, int M, int K, int group,
                                        const float* norm_w, float eps, int8_t* Xq,
                                        float* s_tok, convrot_stream_t stream);

/*
 * Bytes of workspace convrot_int8_linear / convrot_w4a8_linear need for this
 * shape on the current device (0 means workspace may be NULL).
 * weight_bits is 8 or 4.  Returns 0 for invalid shapes.
 */
size_t convrot_linear_workspace_bytes(int M, int N, int K, int weight_bits);

/*
 * W8A8 linear ("Matmul" row of the MOSS-Image card's file table).
 *   acc[m,n] = sum_k Xq[m,k] * Wq[n,k]         (exact int32)
 *   Y[m,n]   = bf16_rn(float(acc) * s_tok[m] * s_row[n])
 * Xq int8 [M, K], s_tok fp32 [M], Wq int8 [N, K], s_row fp32 [N] in;
 * Y bf16 [M, N] out.  K % 16 == 0, K <= CONVROT_MAX_K, N % 8 == 0.
 * workspace: device buffer of at least convrot_linear_workspace_bytes(M, N,
 * K, 8) bytes, zero-filled before its first use.  Output tiles whose K range
 * is split across CTAs are summed there: one int32 accumulator and one
 * arrival counter per such tile.  Every call whose kernels complete leaves
 * the whole buffer zero-filled again, so it can be passed to later calls of
 * any shape without clearing.  A call whose kernel gave up on a bounded wait
 * (reported later by convrot_device_status as CONVROT_ERR_DEVICE_TIMEOUT)
 * may leave partial sums behind: zero-fill the workspace again after such a
 * report.  Calls that share one workspace must not run concurrently.
 */
convrot_status convrot_int8_linear(const int8_t* Xq, const float* s_tok, const int8_t* Wq,
                                   const float* s_row, int M, int N, int K, void* Y,
                                   void* workspace, size_t workspace_bytes,
                                   convrot_stream_t stream);

/*
 * W4A8 linear on the convrot_w4a4 weight layout ("MossInt4", "Format": int4
 * weights, 8-bit activations).  Same as convrot_int8_linear with
 * Wq[n, 2j] = low nibble and Wq[n, 2j+1] = high nibble of Wq4[n, j].
 * Wq4 uint8 [N, K/2].  K % 32 == 0, K <= CONVROT_MAX_K, N % 8 == 0.
 */
convrot_status convrot_w4a8_linear(const int8_t* Xq, const float* s_tok, const uint8_t* Wq4,
                                   const float* s_row, int M, int N, int K, void* Y,
                                   void* workspace, size_t workspace_bytes,
                                   convrot_stream_t stream);

/*
 * MLP boundary: the gate/up projections of an MLP block as one W8A8 GEMM
 * whose epilogue forms the down_proj input (the Heretic card's "Precision
 * layout" quantises mlp.gate_proj, mlp.up_proj and mlp.down_proj; the block
 * computes down(SiLU(gate(x)) * up(x))).
 *   Wq_gu int8 [2I, K]: gate and up rows interleaved in blocks of 16 (see
 *         convrot_interleave_gate_up), s_row_gu fp32 [2I] likewise;
 *   g[m,i], u[m,i] = float(acc) * s_tok[m] * s_row   of the matching rows;
 *   H[m,i] = bf16_rn(SiLU(g) * u),  SiLU(g) = g / (1 + exp(-g))   (fp32).
 * Xq int8 [M, K], s_tok fp32 [M] in; H bf16 [M, I] out (16-byte aligned).
 * I % 16 == 0; K as convrot_int8_linear.  H then goes through
 * convrot_rotate_quant_act (no norm) into the down_proj linear.
 * workspace: at least convrot_swiglu_workspace_bytes(M, I, K, bits) bytes,
 * with the rules of convrot_int8_linear.
 */
size_t convrot_swiglu_workspace_bytes(int M, int I, int K, int weight_bits);
convrot_status convrot_int8_linear_swiglu(const int8_t* Xq, const float* s_tok,
                                          const int8_t* Wq_gu, const float* s_row_gu, int M,
                                          int I, int K, void* H, void* workspace,
                                          size_t workspace_bytes, convrot_stream_t stream);
/* The same on int4 weights (Wq4_gu uint8 [2I, K/2], layout of convrot_w4a8_linear). */
convrot_status convrot_w4a8_linear_swiglu(const int8_t* Xq, const float* s_tok,
                                          const uint8_t* Wq4_gu, const float* s_row_gu, int M,
                                          int I, int K, void* H, void* workspace,
                                          size_t workspace_bytes, convrot_stream_t stream);

/*
 * Offline layout for convrot_*_linear_swiglu: out row r is gate row
 * 16 (r / 32) + r % 32 when r % 32 < 16, else up row 16 (r / 32) + r % 32 - 16.
 * Wg, Wu [I rows of row_bytes] in, out [2I rows] out; works on bf16 weights,
 * quantised rows (int8 or packed int4) and the fp32 row scales alike.
 * I % 16 == 0, row_bytes % 4 == 0, pointers 4-byte aligned; out must not
 * overlap the inputs.
 */
convrot_status convrot_interleave_gate_up(const void* Wg, const void* Wu, int I,
                                          size_t row_bytes, void* out, convrot_stream_t stream);

/*
 * Folds a per-channel SmoothQuant scale into the rows of a row-quantised
 * weight: s_row[i] /= smooth[i], in place, fp32.  Used for down_proj, whose
 * scales go "into up_proj's rows" (MOSS-Image card, "How it was made"): each
 * ConvRot row is rotated and quantised on its own with an absmax scale, so
 * dividing row i by smooth[i] leaves its codes and divides its scale.
 */
convrot_status convrot_fold_row_scales(float* s_row, const float* smooth, int n,
                                       convrot_stream_t stream);

/*
 * Weight-only path ("Matmul" row of the MOSS-Image card's file table: the
 * weight can also be dequantised for a bf16 matmul).  The stored weight is
 * ConvRot-rotated, so instead of rotating the weight back the activation is
 * rotated by the same Hadamard and kept in bf16 (no activation quantisation):
 *   Xr[m,k] = bf16_rn(r * (x * (1 + norm_w)) * R)      convrot_rotate_act_bf16
 *             (norm_w NULL: no RMSNorm, r = 1; group 256, 16 or 0)
 *   Y[m,n]  = bf16_rn(s_row[n] * sum_k Xr[m,k] * Wq[n,k])   convrot_weight_only_linear
 * The int8 codes are expanded to bf16 (exactly) into tensor memory and
 * multiplied on the tensor cores (bf16 inputs, fp32 accumulation), so Y
 * approximates x W^T with the weight's int8 rounding only.
 * x bf16 [M, K], Xr bf16 [M, K], Wq int8 [N, K], s_row fp32 [N], Y bf16 [M, N];
 * K % 16 == 0, N % 8 == 0; all 16-byte aligned.
 * workspace: at least convrot_weight_only_workspace_bytes(M, N, K) bytes
 * (0: may be NULL), with the rules of convrot_int8_linear.  Some shapes
 * split the K range of some output tiles over two CTAs; their fp32 partial
 * sums meet there, added at L2.  A tile never has more than two parts, and
 * 0 + a + b is the same in either order, so results do not depend on timing.
 * convrot_weight_only_gemm_f32 writes the raw fp32 accumulators instead
 * (acc fp32 [M, N]) for accuracy checks.
 */
convrot_status convrot_rotate_act_bf16(const void* x, int M, int K, int group,
                                       const float* norm_w, float eps, void* Xr,
                                       convrot_stream_t stream);
size_t convrot_weight_only_workspace_bytes(int M, int N, int K);
convrot_status convrot_weight_only_linear(const void* Xr, const int8_t* Wq, const float* s_row,
                                          int M, int N, int K, void* Y, void* workspace,
                                          size_t workspace_bytes, convrot_stream_t stream);
convrot_status convrot_weight_only_gemm_f32(const void* Xr, const int8_t* Wq, int M, int N, int K,
                                            float* acc, void* workspace, size_t workspace_bytes,
                                            convrot_stream_t stream);

/*
 * Allocation-free W8A8 linear.  The model cards have no counterpart: this is
 * an interface addition for callers that cannot allocate device memory where
 * they run the layer (plugins without an allocator, runtimes whose device
 * memory is fixed after start-up, paths where an allocation would stall the
 * device).  It computes exactly what convrot_int8_linear computes, with the
 * same kernels, but takes the split-tile workspace from a fixed 24 MiB array
 * inside the library instead of from the caller; it calls no allocator.
 *  - Every GPU that loads the library holds that array until the process exits.
 *  - The first call on a device looks up the array's device address
 *    (set-up, once per device); make that first call before any stream capture.
 *  - Shapes whose workspace exceeds 24 MiB are rejected with
 *    CONVROT_ERR_WORKSPACE (on a 148-SM B200 every M <= 128 fits; larger M
 *    with tiles split across CTAs does not - use convrot_int8_linear).
 *  - All calls on a device share the array and it keeps the last call's
 *    contents.  What must start at zero (split-tile counters and partial
 *    sums) is cleared at set-up, left zero by every call that completes, and
 *    cleared again by the first call after convrot_device_status reported
 *    CONVROT_ERR_DEVICE_TIMEOUT.  Calls that overlap on the GPU race on it.
 * Arguments, layouts and return codes otherwise as convrot_int8_linear.
 */
convrot_status convrot_int8_linear_noalloc(const int8_t* Xq, const float* s_tok, const int8_t* Wq,
                                           const float* s_row, int M, int N, int K, void* Y,
                                           convrot_stream_t stream);

/*
 * Raw int32 accumulators of the same tensor-core kernels and work schedule
 * (including stream-K partial tiles), for exactness checks:
 * acc[m,n] = sum_k Xq[m,k] * Wq[n,k]   (int32 [M, N] out, 16-byte aligned).
 * Workspace rules as for convrot_int8_linear (same size query).
 */
convrot_status convrot_int8_gemm_s32(const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                                     int32_t* acc, void* workspace, size_t workspace_bytes,
                                     convrot_stream_t stream);
convrot_status convrot_w4a8_gemm_s32(const int8_t* Xq, const uint8_t* Wq4, int M, int N, int K,
                                     int32_t* acc, void* workspace, size_t workspace_bytes,
                                     convrot_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H */
