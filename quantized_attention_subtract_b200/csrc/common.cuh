// common.cuh -- constants and kernel parameter blocks of the CUDA path.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace sage {

// Quantisation granularity and tiling.  The SageAttention pages fix
// "per-block" quantisation of Q and K without block sizes ("sageattention"
// package page, "What it is") and name finer, per-thread granularity for
// SageAttention2 (closerAI ComfyUI blog, part 4; "SageAttention2: Technical
// report", section 1).  The reading taken: one INT8 scale per query token
// (one softmax thread owns one query row), one per block of 32 keys (one per
// 32-key section of that thread's exponent loop); query tiles and KV tiles
// of 128 (one tensor-core M tile / N tile); Q's smoothing mean per 128-token
// query tile.
constexpr int kQTile = 128;
constexpr int kKBlk = 32;
constexpr int kKVTile = 128;

// Online softmax, the plain rule: a row's running max m is raised to every
// tile's max, and P is quantised as e4m3(448 * 2^(s - m)) <= 448, e4m3's
// largest finite value.  kLog2P8 = fp32(log2(448)).
constexpr float kLog2P8 = 8.807354927062988281f;        // 0x410CEAED
constexpr float kLog2e = 1.44269502162933349609375f;    // fp32(log2 e), 0x3FB8AA3B

// Fixed-point means: sum of rint(x * 2^24) in int64.
constexpr float kFixScale = 16777216.0f;

// Workspace sub-buffers (device pointers), derived on the host.
struct Workspace {
  int8_t *q8;
  int8_t *k8;
  uint8_t *v8t;
  float *q_scale, *k_scale, *v_scale;
  float *mean_k, *mean_v;
  float *v_inv;                  // 448 / amax per V channel (0 for an all-zero channel)
  float *mq, *dsk;
  long long *k_sum, *v_sum;      // fixed-point channel sums [B*Hkv][D]
  unsigned *v_max, *v_min;       // order-preserving keys of V channel max/min
  int *status;
  int Dp, Nq_pad, Nkv_pad, nqb, nkb;  // nqb: 128-row query tiles; nkb: 32-key K blocks
};

// Shapes / flags / strides of one call, as the kernels see them.
struct Problem {
  const uint16_t *q, *k, *v;
  void *out;
  int B, Hq, Hkv, Nq, Nkv, D;
  // element strides of (batch, head, token) for each tensor; the channel
  // stride is 1
  long long qs_b, qs_h, qs_n, ks_b, ks_h, ks_n, vs_b, vs_h, vs_n, os_b, os_h, os_n;
  int bf16;
  int is_causal, smooth_k, smooth_q, smooth_v;
  float sm_scale;
  float K2;  // fp32(sm_scale * fp32(log2 e))
  // largest code of the Q and K quantisation: 127 (INT8) or 7 (INT4)
  float qmax;
  // Variable-length batches: batch entry b is sequence b with tokens
  // [cu_q[b], cu_q[b+1]) of the packed q (and cu_kv of k, v); Nq / Nkv are
  // then the maximum lengths and the batch strides are unused.  Null for
  // the batched layout.  Device copies in the workspace.
  const int *cu_q, *cu_kv;
  // Variable-length batches only: running totals over the sequences of the
  // work units that exist -- 128-row query tiles, 64-token and 128-token key
  // chunks -- (B + 1 entries each, device), and their grand totals, so that
  // kernels enumerate only units inside a sequence.
  const int *pc_q128, *pc_kv64, *pc_kv128, *pc_q256;
  int tot_q128, tot_kv64, tot_kv128, tot_q256;
  // Pre-pass loads of inputs whose tokens are strided (NHD, packed
  // variable-length batches, padded rows): 1 when the pre-pass reads that
  // tensor through the tensor maps of InputMaps (one box per unit) instead of
  // one bulk copy per row; *_hn: map dimension order (D, H, N, B) instead of
  // (D, N, H, B).  A variable-length batch's map spans all packed tokens with
  // a batch extent of 1.
  int k_map, v_map, q_map;
  int k_hn, v_hn, q_hn;
  // Debug only (the S-dump instantiation of the attention kernel): the int32
  // S tile of query tile dump_qt, KV tile dump_kt of (batch, head) dump_bh is
  // copied row-major to s_dump[128 * 128] as the softmax warps read it.
  int32_t *s_dump;
  int dump_bh, dump_qt, dump_kt;
};

// Tensor maps of the caller's 16-bit inputs for the pre-pass: boxes of D
// channels x 64 tokens (kv_stats) and x 128 tokens (quantize) of one head.
struct InputMaps {
  CUtensorMap k64, v64, k128, v128, q128;
};

// Sequence b with pc[b] * mul <= x < pc[b + 1] * mul (pc non-decreasing,
// pc[0] = 0, x < pc[B] * mul): binary search over the B + 1 running totals.
__device__ __forceinline__ int seq_of(const int *pc, int B, long long mul, long long x) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)pc[mid] * mul <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Unit x of a variable-length enumeration with `heads` heads per sequence:
// sequence b, head h, unit index t within (b, h) (per-sequence unit counts
// pc[b + 1] - pc[b]).
__device__ __forceinline__ void seq_unit(const int *pc, int B, int heads, long long x, int &b, int &h,
                                         int &t) {
  b = seq_of(pc, B, heads, x);
  const int n = pc[b + 1] - pc[b];
  const int r = int(x - (long long)pc[b] * heads);  // unit counts stay below 2^31
  h = r / n;
  t = r % n;
}

// Per batch entry: query / key counts, and the element offset of (token 0,
// head 0) of q, k, v and out.
__device__ __forceinline__ int nq_of(const Problem &pb, int b) {
  return pb.cu_q ? pb.cu_q[b + 1] - pb.cu_q[b] : pb.Nq;
}
__device__ __forceinline__ int nkv_of(const Problem &pb, int b) {
  return pb.cu_kv ? pb.cu_kv[b + 1] - pb.cu_kv[b] : pb.Nkv;
}
__device__ __forceinline__ long long q_off(const Problem &pb, int b) {
  return pb.cu_q ? (long long)pb.cu_q[b] * pb.qs_n : (long long)b * pb.qs_b;
}
__device__ __forceinline__ long long o_off(const Problem &pb, int b) {
  return pb.cu_q ? (long long)pb.cu_q[b] * pb.os_n : (long long)b * pb.os_b;
}
__device__ __forceinline__ long long k_off(const Problem &pb, int b) {
  return pb.cu_kv ? (long long)pb.cu_kv[b] * pb.ks_n : (long long)b * pb.ks_b;
}
__device__ __forceinline__ long long v_off(const Problem &pb, int b) {
  return pb.cu_kv ? (long long)pb.cu_kv[b] * pb.vs_n : (long long)b * pb.vs_b;
}

// ---- integer codes of the pre-pass
constexpr float kTinyAmax = 0x1p-64f;  // blocks below this quantise to zero

// A code is rint(fl(x * inv)), round half to even: adding 1.5 * 2^23 in fp32
// to fl(x * inv) rounds it to an integer exactly that way and leaves it (two's
// complement) in the low mantissa bits; |fl(x * inv)| is at most
// qmax * (1 + 2^-24), so the code stays in [-qmax, qmax].
// The scalar __fmul_rn / __fadd_rn are never contracted into a fused
// multiply-add; an f32x2 multiply followed by an f32x2 add can be (measured:
// codes of exact ties moved), so codes are formed with scalar ops.

// Pack the low bytes of four such code words (first in bits [0, 8)).
__device__ __forceinline__ uint32_t pack4_lo(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Host-side launchers (defined in prepass.cu / attn_fwd.cu).
cudaError_t launch_prepass(const Problem &pb, const Workspace &ws, const InputMaps &im,
                           cudaStream_t stream);
cudaError_t launch_attention(const Problem &pb, const Workspace &ws, const CUtensorMap &tm_q,
                             const CUtensorMap &tm_k, const CUtensorMap &tm_v, cudaStream_t stream);
cudaError_t launch_attention_dump(const Problem &pb, const Workspace &ws, const CUtensorMap &tm_q,
                                  const CUtensorMap &tm_k, const CUtensorMap &tm_v, cudaStream_t stream);
cudaError_t launch_debug_pv(const Problem &pb, const Workspace &ws, const CUtensorMap &tm_v,
                            int b, int hkv, int ktile, const uint8_t *p8, float *o_out,
                            cudaStream_t stream);
cudaError_t launch_debug_e4m3(const float *in, uint8_t *out, int64_t n, cudaStream_t stream);
cudaError_t launch_mma_loop(int ctas, int iters, int kind, int32_t *sink, cudaStream_t stream);
cudaError_t launch_debug_ex2(const float *in, float *out, int64_t n, cudaStream_t stream);
cudaError_t launch_wait_timeout(int *status, cudaStream_t stream);

}  // namespace sage
