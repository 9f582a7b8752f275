/*
 * sage_b200.h -- C ABI of the quantized attention forward pass on NVIDIA B200
 * (sm_100a).
 *
 * The call follows the SageAttention package's statement of its interface
 * ("sageattention" package page, skillfed.io, section "Quickstart"):
 *     sageattn(q, k, v, tensor_layout="HND", is_causal=False, smooth_k=True)
 * with head dimension 64, 96 or 128, Nq != Nkv allowed, and group-query
 * attention (same page, section "What it is and what it does").  The pass
 * (same page; closerAI ComfyUI blog, part 2; "SageAttention2: Technical
 * report", section 2):
 *   1. smoothing: subtract the per-channel mean of K over all tokens
 *      (smooth_k); optionally subtract per-block Q means (smooth_q) and V
 *      channel means (smooth_v), with their exact correction terms;
 *   2. quantisation: symmetric INT8 Q with one fp32 scale per token and K
 *      with one per block of 32 tokens (the pages' per-block / per-thread
 *      granularity: closerAI blog, part 4; "SageAttention2: Technical
 *      report", section 1); V to FP8 e4m3 with per-channel scales.  On
 *      request (qk_bits = 4) Q and K take INT4 codes in [-7, 7] on the same
 *      blocks instead: the report's 4-bit variant (section 1), which its
 *      section 3 applies to all but the most sensitive layers;
 *   3. a flash-style kernel: INT8 Q K^T with exact int32 accumulation,
 *      dequantisation, online softmax in base 2 with the row's running max
 *      m raised to every 128-key tile's max and the running sum rescaled
 *      with it, P quantised to FP8 e4m3 as 448 * exp2(s - m) (at most 448,
 *      e4m3's largest finite value), FP8 P V with fp32 accumulation;
 *   4. epilogue: divide by the row sum, rescale by the V channel scale (and
 *      add the V mean back), round to the input's 16-bit type.
 *
 * Conventions shared by every entry point:
 *   - The library allocates nothing and keeps no state between calls.  All
 *     device memory (inputs, output, workspace) is owned by the caller.
 *   - Calls that take a stream are asynchronous on that stream; argument
 *     errors are returned before anything is enqueued.  No C++ exception
 *     crosses this interface.
 *   - Every internal wait of the kernels is bounded (about one second).  A
 *     wait that runs out records SAGE_ERR_DEVICE_TIMEOUT in the workspace's
 *     status word and the kernel returns early; read it with
 *     sage_get_device_status() after the stream has finished.  A pre-pass
 *     kernel whose shared memory is not 128-byte aligned (not expected)
 *     records SAGE_ERR_ALIGNMENT there and does nothing.
 *   - Sizes: B * Hq * Nq and B * Hkv * Nkv, with Nq and Nkv rounded up to
 *     128, and B * Hkv * D must stay below 2^31 (32-bit tensor-map
 *     coordinates and kernel indices); larger problems are rejected with
 *     SAGE_ERR_UNSUPPORTED.
 */
#ifndef SAGE_B200_H
#define SAGE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SAGE_ABI_VERSION 5

/* A CUDA stream handle (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st *sage_stream_t;

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1,     /* shapes, flags or pointers out of contract */
  SAGE_ERR_UNSUPPORTED = 2,     /* head_dim, dtype, or a device that is not sm_100 */
  SAGE_ERR_ALIGNMENT = 3,       /* a pointer or stride breaks the 16-byte rule */
  SAGE_ERR_CUDA = 4,            /* a CUDA runtime call failed (launch, copy, query) */
  SAGE_ERR_DEVICE_TIMEOUT = 5,  /* a bounded wait inside a kernel ran out */
  SAGE_ERR_WORKSPACE = 6        /* workspace missing, too small or misaligned */
} sage_status_t;

typedef enum {
  SAGE_LAYOUT_HND = 0,          /* [B, H, N, D] ("HND" on the Quickstart page) */
  SAGE_LAYOUT_NHD = 1           /* [B, N, H, D] */
} sage_layout_t;

typedef enum { SAGE_F16 = 0, SAGE_BF16 = 1 } sage_dtype_t;

/*
 * One attention call.
 *   q      [B, Hq,  Nq,  D] (HND) or [B, Nq,  Hq,  D] (NHD), dtype `dtype`
 *   k, v   [B, Hkv, Nkv, D] (HND) or [B, Nkv, Hkv, D] (NHD), dtype `dtype`
 *   out    same shape, layout and dtype as q; written by sage_attn_fwd
 * Strides are in elements, listed in the layout's own order (HND: b, h, n, d;
 * NHD: b, n, h, d).  The last stride must be 1; every other stride and every
 * base pointer must be a multiple of 16 bytes (8 elements); tensors may not
 * overlap `out`.  Query head h reads kv head h / (Hq / Hkv); Hq % Hkv == 0.
 * D is 64, 96 or 128.  Nq >= 0, Nkv >= 1 (when Nq > 0); B, Hq, Hkv >= 1.
 * With Nq == 0 the compute calls return SAGE_OK without reading any pointer.
 * is_causal masks key j for query i when j > i (top-left alignment, as in
 * scaled_dot_product_attention).  sm_scale <= 0 selects 1/sqrt(D).
 * The workspace holds the quantised tensors, scales and means; its size
 * comes from sage_workspace_size() and it must be 256-byte aligned.
 * Precondition of the exact fixed-point means: |x| * N < 2^39 for every
 * smoothed input x (e.g. |x| < 2^24 at N = 32768).  Inputs must be finite.
 */
typedef struct {
  const void *q, *k, *v;
  void *out;
  int32_t B, Hq, Hkv, Nq, Nkv, D;
  int64_t q_strides[4], k_strides[4], v_strides[4], o_strides[4];
  int32_t layout;               /* sage_layout_t */
  int32_t dtype;                /* sage_dtype_t */
  int32_t is_causal, smooth_k, smooth_q, smooth_v;
  float sm_scale;
  void *workspace;
  size_t workspace_bytes;
  /* Variable-length batch (both null for the batched layout): host arrays of
   * B + 1 non-decreasing token offsets starting at 0.  Sequence b owns
   * tokens [cu_seqlens_q[b], cu_seqlens_q[b+1]) of q and out and tokens
   * [cu_seqlens_kv[b], cu_seqlens_kv[b+1]) of k and v: the B sequences are
   * packed along the token axis of one tensor per input, and the batch
   * strides are ignored.  Nq and Nkv are then bounds on the sequence lengths
   * (they size the workspace); a sequence with queries needs at least one
   * key.  Each sequence is its own problem (its own smoothing means and V
   * scales; causal masking top-left within it).  The arrays are copied
   * during the call. */
  const int32_t *cu_seqlens_q, *cu_seqlens_kv;
  /* Bits of the Q and K codes: 8 (or 0) for INT8 codes in [-127, 127], 4 for
   * INT4 codes in [-7, 7] (scale = amax / 7 per block).  INT4 codes are held
   * in the same int8 workspace buffers and multiplied on the INT8 tensor
   * path, which computes their products exactly; V and P stay FP8.  Any
   * other value is SAGE_ERR_INVALID_ARG. */
  int32_t qk_bits;
} sage_attn_params_t;

/* Where the quantised tensors live inside the workspace (tests, debugging).
 * Rows are padded: Nq_pad = Nq rounded up to 128, Nkv_pad likewise; the
 * INT8 row length Dp is 64 for D = 64 and 128 otherwise (zero padded).
 * Padding rows and columns hold zero codes. */
typedef struct {
  int8_t *q8;        /* [B*Hq ][Nq_pad ][Dp]  INT8 (or INT4) codes of Q (or Q - mq) */
  int8_t *k8;        /* [B*Hkv][Nkv_pad][Dp]  INT8 (or INT4) codes of K - mean_k */
  uint8_t *v8t;      /* [B*Hkv][D][Nkv_pad]   FP8 e4m3 codes of V (- mean_v), transposed */
  float *q_scale;    /* [B*Hq ][Nq_pad]       one per query token (0 past Nq)    */
  float *k_scale;    /* [B*Hkv][Nkv_pad/32]   one per 32 keys                    */
  float *v_scale;    /* [B*Hkv][D]                                               */
  float *mean_k;     /* [B*Hkv][D]   (zeros when smooth_k == 0)                  */
  float *mean_v;     /* [B*Hkv][D]   (zeros when smooth_v == 0)                  */
  float *mq;         /* [B*Hq][Nq_pad/128][D]; NULL unless smooth_q              */
  float *dsk;        /* [B*Hq][Nq_pad/128][Nkv_pad] = (mq . K'_j) * sm_scale * log2(e); NULL unless smooth_q */
  int32_t *status;   /* device status word (sage_status_t of the last device failure) */
  int32_t Dp, Nq_pad, Nkv_pad;
} sage_workspace_view_t;

/* Version of this interface (SAGE_ABI_VERSION). */
int32_t sage_abi_version(void);

/* Human-readable name of a status code (static storage). */
const char *sage_status_string(sage_status_t status);

/* Workspace bytes needed for `p` (its pointers and workspace fields are not
 * read).  Returns SAGE_ERR_INVALID_ARG / SAGE_ERR_UNSUPPORTED for shapes the
 * call would reject. */
sage_status_t sage_workspace_size(const sage_attn_params_t *p, size_t *bytes);

/* Sub-buffer pointers of p->workspace (host-side arithmetic only). */
sage_status_t sage_workspace_view(const sage_attn_params_t *p, sage_workspace_view_t *view);

/* The whole pass: smoothing + quantisation pre-pass, then the attention
 * kernel, enqueued on `stream`.  Writes p->out.  Also resets the device
 * status word at its start. */
sage_status_t sage_attn_fwd(const sage_attn_params_t *p, sage_stream_t stream);

/* The two halves of sage_attn_fwd, exposed so that their device time can be
 * measured apart; calling sage_attn_fwd_prepass and then
 * sage_attn_fwd_attention with the same parameters and workspace is
 * equivalent to sage_attn_fwd (they are sage_quantize and
 * sage_attn_quantized).  The pre-pass half resets the device status word.
 * Errors as for sage_attn_fwd. */
sage_status_t sage_attn_fwd_prepass(const sage_attn_params_t *p, sage_stream_t stream);
sage_status_t sage_attn_fwd_attention(const sage_attn_params_t *p, sage_stream_t stream);

/* Pre-pass only (steps 1-2): fills the workspace from q, k, v. */
sage_status_t sage_quantize(const sage_attn_params_t *p, sage_stream_t stream);

/* Attention only (steps 3-4) on a workspace that sage_quantize() filled for
 * the same parameters.  Writes p->out. */
sage_status_t sage_attn_quantized(const sage_attn_params_t *p, sage_stream_t stream);

/* sage_attn_fwd for callers that cannot allocate device memory.  Some hosts
 * hand this library a fixed memory budget and forbid allocations once they
 * have started (serving runtimes with pre-planned pools, plug-in hosts that
 * own the device heap), and some call from latency-critical loops where a
 * cudaMalloc would synchronise the device and stall the caller.  Those
 * callers cannot provide the workspace.
 * This entry point ignores p->workspace / p->workspace_bytes and uses a
 * library-owned scratch area instead: a static device array of
 * SAGE_NOALLOC_MAX_WORKSPACE_BYTES (64 MiB) that every GPU which loads this
 * library holds until the process exits.  The caller still passes q, k, v and
 * out.  Problems whose workspace (sage_workspace_size) exceeds that limit are
 * rejected with SAGE_ERR_WORKSPACE before anything is enqueued.  The first
 * call on each device looks up the array's device address (with that device
 * current); make that first call before any stream capture.  Nothing here
 * allocates.  All calls share the one array and it keeps the last call's
 * contents; each call clears what must start at zero.  Calls that overlap on
 * the GPU (other streams, other threads) race on the array and must be
 * serialised by the caller.  sage_get_device_status does not see this
 * array; read it with sage_noalloc_device_status.
 * The SageAttention pages have no counterpart of this call. */
#define SAGE_NOALLOC_MAX_WORKSPACE_BYTES (64ull << 20)
sage_status_t sage_attn_fwd_noalloc(const sage_attn_params_t *p, sage_stream_t stream);

/* Synchronously read the device status word that the last
 * sage_attn_fwd_noalloc call with the same shapes and flags left in the
 * library scratch of the current device (SAGE_OK when no kernel recorded a
 * failure).  p's workspace fields are ignored.  No counterpart on the pages. */
sage_status_t sage_noalloc_device_status(const sage_attn_params_t *p, int32_t *code);

/* Debug: the attention half of the pass (as sage_attn_quantized, on a
 * workspace that sage_quantize filled; it writes p->out too) in a build of
 * the attention kernel that also copies the int32 tile S = q8 k8^T of query
 * tile `qtile` (128 rows) and key tile `ktile` (128 keys) of (batch b, query
 * head h), as its softmax warps read it from tensor memory, row-major to the
 * device buffer s_out[128*128].  Key tiles a causal query tile skips are not
 * computed (s_out is then left untouched).  Not for variable-length batches. */
sage_status_t sage_debug_dump_s(const sage_attn_params_t *p, int32_t b, int32_t h, int32_t qtile,
                                int32_t ktile, int32_t *s_out, sage_stream_t stream);

/* Debug: O = P V for one 128x128 FP8 P tile given row-major on the device
 * (p8[128*128], e4m3 codes) and key tile `ktile` of kv head (b, hkv) of a
 * filled workspace; O is fp32 [128][D] row-major in o_out.  Same shared
 * memory layout, descriptors and FP8 tensor-core path as the kernel. */
sage_status_t sage_debug_pv(const sage_attn_params_t *p, int32_t b, int32_t hkv, int32_t ktile,
                            const uint8_t *p8, float *o_out, sage_stream_t stream);

/* Debug: the kernel's fp32 -> FP8 e4m3 conversion (round to nearest even,
 * saturating to +-448) applied to n device floats, in the kernel's byte
 * order (element 2i in the low byte of each packed pair). */
sage_status_t sage_debug_e4m3(const float *in, uint8_t *out, int64_t n, sage_stream_t stream);

/* Debug: back-to-back 8-bit tensor-core MMAs (128x256x32 each, operands
 * resident in shared memory; kind 0 = INT8 -> S32, kind 1 = FP8 e4m3 -> F32)
 * on `ctas` CTAs for `iters` iterations; used to measure the attainable
 * 8-bit MMA rate.  `sink` is a device int32 buffer of ctas + 1 entries: one
 * value per CTA, then a status word the waits use. */
sage_status_t sage_debug_mma_loop(int32_t ctas, int32_t iters, int32_t kind, int32_t *sink,
                                  sage_stream_t stream);

/* Debug: the attention kernel's exp2 (the hardware ex2.approx.ftz.f32)
 * applied to n device floats; used to measure its error against fp64. */
sage_status_t sage_debug_ex2(const float *in, float *out, int64_t n, sage_stream_t stream);

/* Debug: one thread waits on a shared-memory barrier that nothing completes,
 * through the same bounded wait every kernel uses; after about one second the
 * wait gives up and writes SAGE_ERR_DEVICE_TIMEOUT into status[0] (a device
 * int32 the caller zeroes).  Exercises failure reporting without a fault. */
sage_status_t sage_debug_wait_timeout(int32_t *status, sage_stream_t stream);

/* Synchronously read the device status word of p->workspace into *code
 * (SAGE_OK when no kernel recorded a failure since the last reset). */
sage_status_t sage_get_device_status(const sage_attn_params_t *p, int32_t *code);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_B200_H */
