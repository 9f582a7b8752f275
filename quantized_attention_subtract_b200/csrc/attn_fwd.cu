// attn_fwd.cu -- the quantized attention kernel for sm_100a.
//
// Computes, per (batch, query head, pair of 128-row query tiles), the
// flash-style pass the SageAttention pages describe (INT8 Q K^T, FP8 P V;
// closerAI ComfyUI blog, part 2; "sageattention" package page, "What it is"):
//   S = q8 k8^T                    exact int32, tensor cores (kind::i8)
//   s = S * q_scale[row] * k_scale[32-key block] * sm_scale * log2(e)
//       (+ dS for smoothed Q)
//   online softmax in base 2: the row's running max m is raised to every
//   tile's max; O and l are rescaled by 2^(m_old - m_new) when it grows
//   P8 = e4m3(448 * 2^(s - m))     FP8 probabilities (<= 448)
//   O += P8 v8                     fp32 accumulation, tensor cores (kind::f8f6f4)
//   out = O * v_scale / l (+ mean_v), rounded to bf16 / fp16
//
// One CTA (512 threads, four warpgroups) per SM owns two query tiles, A and
// B, of one (batch, head), and streams the head's K and V tiles once for both.
//   warps 0-3   softmax of tile A, warps 4-7 softmax of tile B: one query row
//               per thread (TMEM lane).  S_j is read with tcgen05.ld (which
//               frees S_j's columns for S_{j+1} at once), the row's rescale
//               factor goes to shared memory, and the FP8 P_j is written to
//               its own TMEM columns (head dims 64 and 96) or to shared memory
//               with the 128-byte swizzle (head dim 128, where S and O fill
//               the 512 TMEM columns).  The two warpgroups take turns for their
//               exponentials (A's tile j, B's tile j, A's tile j + 1, ...), so
//               that each has the exp2 units to itself while the other loads
//               S and takes its max.
//   warps 8-11  correction: multiply a tile's O rows in TMEM by the rescale
//               factor (after P V_{j-1}, before P V_j), then the epilogue
//   warp 12     TMA producer: Q_A, Q_B once, then K_0, K_1, V_0, K_2, V_1, ...
//               into a shared-memory ring (order = MMA consumption order)
//   warp 13     allocates the 512 TMEM columns and issues the MMAs, per KV
//               tile j: S_A(j+1), S_B(j+1) as soon as the softmax warps have
//               read S(j), then O_A += P_A(j) V_j, O_B += P_B(j) V_j; it runs
//               its loop with the whole warp and issues from one elected lane
//   warps 14-15 idle
// TMEM: S_A at columns [0, 128), S_B at [128, 256), O_A and O_B from 256 (D
// columns each, 128 apart for D = 128), P_A and P_B (32 columns each) after
// them for D < 128.
// Causal tiles past the diagonal are skipped; keys >= Nkv and (causal) keys
// > query are masked; rows >= Nq are computed but not stored.
// Template flags: smoothed Q (dS added to the logits), variable-length
// batches (per-sequence lengths and offsets; only query-tile pairs inside a
// sequence are launched), S dump (a debug instantiation that copies one S
// tile to global memory as the softmax warps read it).
// Every tcgen05.ld / st here runs under warp-uniform control flow
// (.sync.aligned), and every wait is bounded (about one second).
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cfloat>

#include "common.cuh"
#include "ptx.cuh"

namespace sage {
namespace {

template <int D>
struct Cfg {
  static constexpr int Dp = D == 64 ? 64 : 128;       // INT8 row length in smem / workspace
  static constexpr int kQKSteps = D / 32;             // K = 32 bytes per 8-bit MMA
  static constexpr bool kPTmem = D < 128;             // FP8 P in TMEM (else shared memory)
  static constexpr int kQBytes = 128 * Dp;
  static constexpr int kKBytes = 128 * Dp;
  static constexpr int kVBytes = D * 128;
  static constexpr int kPBytes = 128 * 128;           // one tile's P, 128 rows x 128 keys
  static constexpr int kStageBytes = kKBytes > kVBytes ? kKBytes : kVBytes;
  static constexpr int kStages = D == 64 ? 8 : 6;     // 3-4 KV tiles in flight
  static constexpr int kOffQ = 0;                     // Q_A, Q_B
  static constexpr int kOffRing = kOffQ + 2 * kQBytes;
  static constexpr int kOffP = kOffRing + kStages * kStageBytes;  // P_A, P_B (D = 128)
  static constexpr int kOffBar = kOffP + (kPTmem ? 0 : 2 * kPBytes);
  static constexpr int kBarBytes = 512;
  static constexpr int kOffAlpha = kOffBar + kBarBytes;  // float [2][128] rescale factors
  static constexpr int kOffL = kOffAlpha + 1024;         // float [2][128] row sums
  static constexpr int kOffMisc = kOffL + 1024;          // TMEM base, status snapshot
  static constexpr int kSmem = kOffMisc + 64 + 1024;     // +1024: base alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kThreads = 512;
  // TMEM columns of tile X's S, O and (D < 128) P
  static __device__ __forceinline__ uint32_t col_s(int X) { return 128u * uint32_t(X); }
  static __device__ __forceinline__ uint32_t col_o(int X) {
    return 256u + uint32_t(D == 128 ? 128 : D) * uint32_t(X);
  }
  static __device__ __forceinline__ uint32_t col_p(int X) { return 256u + 2u * D + 32u * uint32_t(X); }
};
static_assert(256 + 2 * 96 + 64 <= 512 && 256 + 2 * 64 + 64 <= 512, "TMEM columns");
static_assert(Cfg<128>::kSmem <= 227 * 1024, "shared memory");

// Register split of the attention CTA (512 threads launched at 128 registers
// each, the whole register file): the helper warpgroup (TMA producer, MMA
// issuer, two idle warps) and the correction warpgroup give registers back,
// the two softmax warpgroups take them.
constexpr uint32_t kLaunchRegs = 128, kSoftmaxRegs = 184, kCorrRegs = 96, kHelperRegs = 48;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kCorrRegs + 128 * kHelperRegs == kLaunchRegs * 512,
              "register split");

// Barrier slots (8 bytes each) inside the barrier area.  [X] = tile A / B.
enum Bar {
  kBarQ = 0,
  kBarFull = 1,      // + stage (8)   TMA bytes
  kBarEmpty = 9,     // + stage (8)   tcgen05.commit
  kBarSFull = 17,    // + X           tcgen05.commit: S_X(j) in TMEM
  kBarSEmpty = 19,   // + X           4 softmax warps: S_X(j) read into registers
  kBarPReady = 21,   // + X           4 softmax warps: P_X(j) written
  kBarAlpha = 23,    // + X           4 softmax warps: rescale factors of tile j in smem
  kBarOReady = 25,   // + X           4 correction warps: O_X ready for P V_j
  kBarLReady = 27,   // + X           4 softmax warps: row sums in smem (once)
  kBarTurn = 29,     // + X           4 warps of the other softmax warpgroup: X's turn for exp2
  kBarPVDone = 31,   // + X           tcgen05.commit: P V_j of tile X complete
  kBarFinal = 33,
  kNumBars = 34
};
static_assert(kNumBars * 8 <= 512, "barrier area");

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int *status) {
  const bool ok = mbar_wait(bar, parity, status);
  return __all_sync(0xffffffffu, ok);
}
// The same with the suspend-time hint (the single-issuer roles' waits).
__device__ __forceinline__ bool warp_wait_h(uint32_t bar, uint32_t parity, int *status,
                                            bool honor_abort = true) {
  const bool ok = mbar_wait_h(bar, parity, status, honor_abort);
  return __all_sync(0xffffffffu, ok);
}

constexpr float kBias = 12582912.0f;  // 1.5 * 2^23

// One query row's share of one KV tile (128 keys), first part: s[] holds the
// int32 S row from TMEM.  Without smoothed Q it is converted in place to
// fp32 (exact: |S| <= 127^2 * 128 < 2^24); with smoothed Q it becomes the
// logits x = S * c + dsk (S biased to the fp32 bit pattern of 1.5 * 2^23 + S,
// which is exact, then unbiased in the FMA).  Keys k >= lim (only when
// kMasked) are set to -inf.  c[q] is the dequantisation factor of keys
// 32 q .. 32 q + 31.  Returns the tile max of the logits over the valid keys
// (-inf if none).
template <bool kMasked, bool kSmoothQ>
__device__ __forceinline__ float tile_max(uint32_t (&s)[128], const float (&c)[4],
                                          const float *dsk_tile, int lim) {
#define X(k) __uint_as_float(s[k])
  if (!kSmoothQ) {
#pragma unroll
    for (int k = 0; k < 128; ++k) s[k] = __float_as_uint(__int2float_rn(int(s[k])));
  } else {
    const float2 nb = make_float2(-kBias, -kBias);
#pragma unroll
    for (int k = 0; k < 128; ++k) s[k] += 0x4B400000u;
#pragma unroll
    for (int k = 0; k < 128; k += 4) {
      const float4 d4 = __ldg(reinterpret_cast<const float4 *>(dsk_tile + k));
      const float2 c2 = make_float2(c[k / 32], c[k / 32]);
      const float2 x01 = __ffma2_rn(__fadd2_rn(make_float2(X(k), X(k + 1)), nb), c2, make_float2(d4.x, d4.y));
      const float2 x23 = __ffma2_rn(__fadd2_rn(make_float2(X(k + 2), X(k + 3)), nb), c2, make_float2(d4.z, d4.w));
      s[k] = __float_as_uint(x01.x);
      s[k + 1] = __float_as_uint(x01.y);
      s[k + 2] = __float_as_uint(x23.x);
      s[k + 3] = __float_as_uint(x23.y);
    }
  }
  // keys k >= lim become -inf in place: they drop out of the max here and
  // give 2^-inf = 0 in tile_exp
  if (kMasked) {
#pragma unroll
    for (int k = 0; k < 128; ++k) s[k] = k < lim ? s[k] : 0xFF800000u;
  }
  // two independent 3-input max chains per 32-key section
  float h[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) h[q] = -INFINITY;
#pragma unroll
  for (int sec = 0; sec < 4; ++sec)
#pragma unroll
    for (int k = 32 * sec; k < 32 * sec + 32; k += 4) {
      h[2 * sec] = fmax3(h[2 * sec], X(k), X(k + 1));
      h[2 * sec + 1] = fmax3(h[2 * sec + 1], X(k + 2), X(k + 3));
    }
  float r = -INFINITY;
#pragma unroll
  for (int sec = 0; sec < 4; ++sec) {
    const float hs = fmaxf(h[2 * sec], h[2 * sec + 1]);
    // max_k fl(S_k * c) == fl(max_k S_k * c) since c >= 0
    if (kSmoothQ) r = fmaxf(r, hs);
    else r = fmaxf(r, hs == -INFINITY ? -INFINITY : __fmul_rn(hs, c[sec]));
  }
  return r;
#undef X
}

// The exponent arguments t = x * c - mb (mb = m - log2(448), so a key at the
// row max gets t = log2(448)), in place, with smoothed Q t = x - mb (x
// already holds the logit).  Computed before the warpgroup's turn for the
// exponentials, so that the turn holds only the exp2 and what depends on it.
template <bool kSmoothQ>
__device__ __forceinline__ void tile_args(uint32_t (&s)[128], const float (&c)[4], float nmb) {
#define X(k) __uint_as_float(s[k])
  const float2 nmb2 = make_float2(nmb, nmb);
#pragma unroll
  for (int sec = 0; sec < 4; ++sec) {
    // A scale product of exactly 0 means an all-zero Q row or K block, so
    // S = 0 there; the smallest normal float in its place leaves S * c = 0
    // and keeps masked keys at -inf * c = -inf instead of NaN.
    const float ce = c[sec] == 0.f ? FLT_MIN : c[sec];
    const float2 c2 = make_float2(ce, ce);
#pragma unroll
    for (int k = 32 * sec; k < 32 * sec + 32; k += 2) {
      const float2 x = make_float2(X(k), X(k + 1));
      const float2 t = kSmoothQ ? __fadd2_rn(x, nmb2) : __ffma2_rn(x, c2, nmb2);
      s[k] = __float_as_uint(t.x);
      s[k + 1] = __float_as_uint(t.y);
    }
  }
#undef X
}

// Second part: probabilities 2^t of the arguments tile_args left in s[],
// their sum (returned) and their FP8 codes, stored one 32-key section at a
// time: kPTmem -- to the row's TMEM lane at columns pdst .. pdst + 31 (keys
// 4 w .. 4 w + 3 in column w; stores issued, the caller waits); otherwise to
// the row's 128 bytes of a shared-memory P tile at pdst with the 128-byte
// swizzle (16-byte unit u at u ^ (row % 8)).  Pairs of keys go through f32x2
// ops; every lane of a packed op rounds like its scalar counterpart.
template <bool kPTmem>
__device__ __forceinline__ float tile_exp(const uint32_t (&s)[128], uint32_t pdst, uint32_t rx) {
#define X(k) __uint_as_float(s[k])
  float2 acc01 = make_float2(0.f, 0.f), acc23 = make_float2(0.f, 0.f);
#pragma unroll
  for (int sec = 0; sec < 4; ++sec) {
    uint32_t pk[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int k = 32 * sec + 4 * q;
      const float2 p01 = make_float2(ex2_approx(X(k)), ex2_approx(X(k + 1)));
      const float2 p23 = make_float2(ex2_approx(X(k + 2)), ex2_approx(X(k + 3)));
      acc01 = __fadd2_rn(acc01, p01);
      acc23 = __fadd2_rn(acc23, p23);
      pk[q] = e4m3x4(p01.x, p01.y, p23.x, p23.y);
    }
    if constexpr (kPTmem) {
      tmem_st8_issue(pdst + 8u * uint32_t(sec), pk);
    } else {
      // keys 32 sec .. 32 sec + 31 are the 16-byte units 2 sec and 2 sec + 1 of the row
      sts128(pdst + ((32u * sec) ^ rx), pk[0], pk[1], pk[2], pk[3]);
      sts128(pdst + ((32u * sec + 16u) ^ rx), pk[4], pk[5], pk[6], pk[7]);
    }
  }
  return (acc01.x + acc01.y) + (acc23.x + acc23.y);
#undef X
}

// Multiply this thread's O row (TMEM lane, D fp32 columns at tO) by a, 32
// columns at a time.
template <int D>
__device__ __forceinline__ void rescale_row(uint32_t tO, float a) {
  const float2 a2 = make_float2(a, a);
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + 32 * c, o);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
      o[e] = __float_as_uint(v.x);
      o[e + 1] = __float_as_uint(v.y);
    }
    tmem_st32_issue(tO + 32 * c, o);
  }
  tmem_st_wait();
}

// Epilogue of one row: out = O * v_scale / l (+ mean_v) as bf16 / fp16,
// stored when the row is a real query (store == true).
template <int D>
__device__ __forceinline__ void store_row(uint32_t tO, float l, const float *vs, const float *mv,
                                          bool smooth_v, bool bf16, uint8_t *orow, bool store) {
  const float inv_l = 1.0f / l;
  // one 32-column chunk at a time (not unrolled: the correction warps run at
  // a small register budget)
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(tO + 32 * c, r);
    uint32_t packed[16];
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      // channel scales (and means) four at a time: the per-head arrays are
      // 256-byte aligned and 32 c + e is a multiple of 4
      const float4 s4 = __ldg(reinterpret_cast<const float4 *>(vs + 32 * c + e));
      float o[4] = {__uint_as_float(r[e]) * (s4.x * inv_l), __uint_as_float(r[e + 1]) * (s4.y * inv_l),
                    __uint_as_float(r[e + 2]) * (s4.z * inv_l), __uint_as_float(r[e + 3]) * (s4.w * inv_l)};
      if (smooth_v) {
        const float4 m4 = __ldg(reinterpret_cast<const float4 *>(mv + 32 * c + e));
        o[0] += m4.x;
        o[1] += m4.y;
        o[2] += m4.z;
        o[3] += m4.w;
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        if (bf16) {
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(o[2 * h2], o[2 * h2 + 1]);
          packed[e / 2 + h2] = *reinterpret_cast<const uint32_t *>(&v2);
        } else {
          const __half2 v2 = __floats2half2_rn(o[2 * h2], o[2 * h2 + 1]);
          packed[e / 2 + h2] = *reinterpret_cast<const uint32_t *>(&v2);
        }
      }
    }
    if (store) {
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4)
        *reinterpret_cast<uint4 *>(orow + 64 * c + 16 * v4) =
            make_uint4(packed[4 * v4], packed[4 * v4 + 1], packed[4 * v4 + 2], packed[4 * v4 + 3]);
    }
  }
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}


template <int D, bool kSmoothQ, bool kVarlen, bool kDump>
__global__ void __maxnreg__(128)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const Problem pb, const Workspace ws) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  // the shared base, the warp index and (below) the TMEM base go through a
  // shuffle from lane 0, so the compiler knows them warp-uniform and keeps
  // the barrier and TMEM addresses built from them in uniform registers
  const uint32_t s_base = __shfl_sync(0xffffffffu, smem_u32(smem), 0);
  const uint32_t sQ = s_base + C::kOffQ, sRing = s_base + C::kOffRing, bars = s_base + C::kOffBar;
  const uint32_t sP = s_base + C::kOffP;
  auto bar = [&](int i) { return bars + 8u * uint32_t(i); };
  float *alpha_s = reinterpret_cast<float *>(smem + C::kOffAlpha);
  float *l_s = reinterpret_cast<float *>(smem + C::kOffL);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
  int *status_snap = reinterpret_cast<int *>(smem + C::kOffMisc + 4);

  const int warp = __shfl_sync(0xffffffffu, int(threadIdx.x / 32), 0), lane = threadIdx.x % 32;
  int *status = ws.status;

  // ---- work item: (b, h, pair of query tiles 2 pr, 2 pr + 1); causal runs
  // the longest pairs first
  const int npair = (ws.nqb + 1) / 2, bhq = pb.B * pb.Hq;
  int pr, bh;
  if (kVarlen) {
    // only the pairs inside a sequence are launched
    int sb, sh;
    seq_unit(pb.pc_q256, pb.B, pb.Hq, blockIdx.x, sb, sh, pr);
    bh = sb * pb.Hq + sh;
  } else if (pb.is_causal) {
    pr = npair - 1 - int(blockIdx.x / bhq);
    bh = int(blockIdx.x % bhq);
  } else {
    pr = int(blockIdx.x % npair);
    bh = int(blockIdx.x / npair);
  }
  const int b = bh / pb.Hq, h = bh % pb.Hq;
  const int hk = h / (pb.Hq / pb.Hkv), bhk = b * pb.Hkv + hk;
  const int Nq_b = kVarlen ? nq_of(pb, b) : pb.Nq, Nkv_b = kVarlen ? nkv_of(pb, b) : pb.Nkv;
  const int q0A = 2 * kQTile * pr, q0B = q0A + kQTile;
  // tile B takes part only if it holds a query of this entry
  const bool hasB = q0B < Nq_b;
  const int nkt_all = (Nkv_b + kKVTile - 1) / kKVTile;
  auto tiles_of = [&](int q0) {
    return pb.is_causal ? min(nkt_all, min(q0 + kQTile - 1, Nq_b - 1) / kKVTile + 1) : nkt_all;
  };
  const int TA = tiles_of(q0A), TB = hasB ? tiles_of(q0B) : 0;
  const int T = max(TA, TB);

  if (threadIdx.x == 0) {
    // four warps (of the softmax or correction warpgroups) arrive on the
    // S-empty ... turn barriers; TMA bytes or a single tcgen05.commit
    // complete the others
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), (i >= kBarSEmpty && i < kBarPVDone) ? 4 : 1);
    fence_mbar_init();
    // one read of the status word decides for every warp whether an earlier
    // CTA already failed
    *status_snap = *(volatile int *)status;
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  const bool skip_all = *status_snap != 0;

  if (warp >= 12) {
    reg_dealloc<kHelperRegs>();
    if (warp == 12 && !skip_all) {
      // ================================================= TMA producer
      // The whole warp runs the loop; the elected lane issues the copies.
      const bool leader = elect_one();
      if (leader) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        mbar_arrive_expect_tx(bar(kBarQ), uint32_t(C::kQBytes) * (hasB ? 2u : 1u));
        tma_load_2d(sQ, &tm_q, bar(kBarQ), 0, bh * ws.Nq_pad + q0A);
        if (hasB) tma_load_2d(sQ + C::kQBytes, &tm_q, bar(kBarQ), 0, bh * ws.Nq_pad + q0B);
      }
      __syncwarp();
      int n = 0;
      bool ok = true;
      const int krow0 = bhk * ws.Nkv_pad, vrow0 = bhk * D;
      auto load = [&](bool isV, int j) {
        if (!ok) return;
        const int st = n % C::kStages;
        if (!warp_wait_h(bar(kBarEmpty + st), ((n / C::kStages) & 1) ^ 1, status)) {
          ok = false;
          return;
        }
        if (leader) {
          const uint32_t dst = sRing + st * C::kStageBytes, full = bar(kBarFull + st);
          if (!isV) {
            mbar_arrive_expect_tx(full, C::kKBytes);
            tma_load_2d(dst, &tm_k, full, 0, krow0 + j * kKVTile);
          } else {
            mbar_arrive_expect_tx(full, C::kVBytes);
            tma_load_2d(dst, &tm_v, full, j * kKVTile, vrow0);
          }
        }
        __syncwarp();
        ++n;
      };
      // K_0, K_1, V_0, K_2, V_1, ..., V_{T-1}
      load(false, 0);
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) load(false, j + 1);
        load(true, j);
      }
      // Before leaving, make sure every copy issued has landed (bounded).
      warp_wait_h(bar(kBarQ), 0, status, false);
      for (int m = (n > C::kStages ? n - C::kStages : 0); m < n; ++m)
        warp_wait_h(bar(kBarFull + m % C::kStages), (m / C::kStages) & 1, status, false);
    } else if (warp == 13 && !skip_all) {
      // ================================================= MMA issuer
      // The whole warp runs the loop (warp-uniform control flow, so that the
      // descriptors stay in uniform registers); the elected lane issues the
      // MMAs and commits.  Ring-stage descriptors differ only in their
      // start-address field (16-byte units, bits [0, 14)).
      const bool leader = elect_one();
      constexpr uint32_t id_s = idesc_i8(128, 128);
      constexpr uint32_t id_o = idesc_e4m3_f32(128, D);
      constexpr uint64_t kStageStep = uint64_t(C::kStageBytes) >> 4;
      const uint64_t dQ0 = smem_desc_kmajor(sQ, C::Dp);
      const uint64_t dQ1 = smem_desc_kmajor(sQ + C::kQBytes, C::Dp);
      const uint64_t dK0 = smem_desc_kmajor(sRing, C::Dp);
      const uint64_t dV0 = smem_desc_kmajor(sRing, 128);
      const uint64_t dP0 = smem_desc_kmajor(sP, 128);
      int n = 0;
      bool ok = warp_wait_h(bar(kBarQ), 0, status);
      auto wait_stage = [&]() -> uint32_t {
        const int st = n % C::kStages;
        if (ok && !warp_wait_h(bar(kBarFull + st), (n / C::kStages) & 1, status)) ok = false;
        ++n;
        return uint32_t(st);
      };
      // S_X = Q_X K^T from ring stage st, committed to S-full[X]
      auto issue_s = [&](int X, uint32_t st) {
        const uint64_t dK = dK0 + st * kStageStep, dQ = X ? dQ1 : dQ0;
        if (leader) {
#pragma unroll
          for (int k = 0; k < C::kQKSteps; ++k)
            mma_i8_ss(tmem + C::col_s(X), dQ + 2 * k, dK + 2 * k, id_s, k > 0 ? 1u : 0u);
          mma_commit(bar(kBarSFull + X));
        }
        __syncwarp();
      };
      if (ok) {
        const uint32_t stK = wait_stage();
        if (ok) {
          tc_fence_after();
          issue_s(0, stK);
          if (TB > 0) issue_s(1, stK);
          if (leader) mma_commit(bar(kBarEmpty + stK));
          __syncwarp();
        }
      }
      for (int j = 0; ok && j < T; ++j) {
        // S(j+1) of both tiles, each once its softmax warps have read S(j)
        if (j + 1 < T) {
          const uint32_t stK = wait_stage();
#pragma unroll
          for (int X = 0; X < 2; ++X) {
            if (!ok || j + 1 >= (X ? TB : TA)) continue;
            if (!warp_wait_h(bar(kBarSEmpty + X), j & 1, status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(X, stK);
          }
          if (!ok) break;
          if (leader) mma_commit(bar(kBarEmpty + stK));
          __syncwarp();
        }
        // O_X += P_X(j) V_j once P_X(j) is written and O_X corrected
        const uint32_t stV = wait_stage();
        if (!ok) break;
        const uint64_t dV = dV0 + stV * kStageStep;
#pragma unroll
        for (int X = 0; X < 2; ++X) {
          if (j >= (X ? TB : TA)) continue;
          if (!warp_wait_h(bar(kBarPReady + X), j & 1, status) ||
              !warp_wait_h(bar(kBarOReady + X), j & 1, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if constexpr (C::kPTmem)
                mma_f8_ts(tmem + C::col_o(X), tmem + C::col_p(X) + 8u * k, dV + 2 * k, id_o,
                          (j > 0 || k > 0) ? 1u : 0u);
              else
                mma_f8_ss(tmem + C::col_o(X), dP0 + uint64_t(X) * (uint64_t(C::kPBytes) >> 4) + 2 * k,
                          dV + 2 * k, id_o, (j > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(bar(kBarPVDone + X));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (leader) mma_commit(bar(kBarEmpty + stV));
        __syncwarp();
      }
      // every MMA issued by the elected lane has finished before teardown
      if (leader) mma_commit(bar(kBarFinal));
      __syncwarp();
      warp_wait_h(bar(kBarFinal), 0, status, false);
    }
  } else if (warp >= 8) {
    reg_dealloc<kCorrRegs>();
    // ================================================= correction / epilogue
    const int wq = warp & 3, row = 32 * wq + lane;
    const uint32_t lane_off = uint32_t(32 * wq) << 16;
    bool ok = !skip_all;
    for (int j = 0; ok && j < T; ++j) {
#pragma unroll
      for (int X = 0; X < 2; ++X) {
        const int TX = X ? TB : TA;
        if (j >= TX) continue;
        if (!warp_wait(bar(kBarAlpha + X), j & 1, status)) {
          ok = false;
          break;
        }
        const float a = alpha_s[X * 128 + row];
        // the first tile overwrites O; later ones rescale when a row's max grew
        if (j > 0 && __any_sync(0xffffffffu, a != 1.f)) {
          if (!warp_wait(bar(kBarPVDone + X), (j - 1) & 1, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          rescale_row<D>(tmem + lane_off + C::col_o(X), a);
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarOReady + X));
      }
    }
    // ---- epilogue: out = O * v_scale / l (+ mean_v)
#pragma unroll
    for (int X = 0; X < 2; ++X) {
      const int TX = X ? TB : TA;
      if (!ok || TX == 0) continue;
      if (!warp_wait(bar(kBarLReady + X), 0, status) ||
          !warp_wait(bar(kBarPVDone + X), (TX - 1) & 1, status)) {
        ok = false;
        continue;
      }
      tc_fence_after();
      const int i = (X ? q0B : q0A) + row;
      uint8_t *orow = reinterpret_cast<uint8_t *>(pb.out) +
                      2 * ((kVarlen ? o_off(pb, b) : b * pb.os_b) + h * pb.os_h + (long long)i * pb.os_n);
      store_row<D>(tmem + lane_off + C::col_o(X), l_s[X * 128 + row], ws.v_scale + (long long)bhk * D,
                   ws.mean_v + (long long)bhk * D, pb.smooth_v != 0, pb.bf16 != 0, orow, i < Nq_b);
    }
  } else {
    reg_alloc<kSoftmaxRegs>();
    // ================================================= softmax
    const int X = warp >> 2, wq = warp & 3;
    const int row = 32 * wq + lane;            // row within the query tile (TMEM lane)
    const int q0 = X ? q0B : q0A, TX = X ? TB : TA;
    const int i = q0 + row;                    // query index
    const uint32_t lane_off = uint32_t(32 * wq) << 16;
    const uint32_t tS = tmem + lane_off + C::col_s(X);
    // where this row's FP8 P goes: its TMEM lane at the tile's P columns, or
    // its 128 bytes of the tile's shared-memory P buffer (row-major, swizzled)
    const uint32_t pdst = C::kPTmem ? tmem + lane_off + C::col_p(X)
                                    : sP + uint32_t(X) * C::kPBytes + uint32_t(row) * 128u;
    const uint32_t rx = uint32_t(row & 7) << 4;
    if (!skip_all && TX > 0) {
      const float qs = ws.q_scale[(long long)bh * ws.Nq_pad + i];
      const float *ksc = ws.k_scale + (long long)bhk * (ws.Nkv_pad / kKBlk);
      const float *dsk = kSmoothQ ? ws.dsk + ((long long)bh * ws.nqb + q0 / kQTile) * ws.Nkv_pad : nullptr;
      float m_run = -INFINITY, l = 0.f;
      bool ok = true;
      float4 ks = __ldg(reinterpret_cast<const float4 *>(ksc));  // K block scales, one tile ahead
      for (int j = 0; j < TX; ++j) {
        const int kb = j * kKVTile;
        float c[4];
        c[0] = __fmul_rn(__fmul_rn(qs, ks.x), pb.K2);
        c[1] = __fmul_rn(__fmul_rn(qs, ks.y), pb.K2);
        c[2] = __fmul_rn(__fmul_rn(qs, ks.z), pb.K2);
        c[3] = __fmul_rn(__fmul_rn(qs, ks.w), pb.K2);
        if (j + 1 < TX) ks = __ldg(reinterpret_cast<const float4 *>(ksc + 4 * (j + 1)));
        if (!warp_wait(bar(kBarSFull + X), j & 1, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[128];
        tmem_ld64x2(tS, s);
        // S_X(j) is in registers: its columns are free for S_X(j + 1)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarSEmpty + X));
        if constexpr (kDump) {
          if (bh == pb.dump_bh && q0 / kQTile == pb.dump_qt && j == pb.dump_kt)
            for (int k = 0; k < 128; ++k) pb.s_dump[row * 128 + k] = int32_t(s[k]);
        }
        // valid keys of this tile for this row form the prefix [0, lim)
        int lim = min(kKVTile, Nkv_b - kb);
        if (pb.is_causal) lim = min(lim, i - kb + 1);
        const float *dsk_tile = kSmoothQ ? dsk + kb : nullptr;
        const float m_tile = lim < kKVTile ? tile_max<true, kSmoothQ>(s, c, dsk_tile, lim)
                                           : tile_max<false, kSmoothQ>(s, c, dsk_tile, lim);
        // (rows of a diagonal or ragged tile took different branches above;
        // the TMEM stores below need the whole warp converged)
        __syncwarp();
        // the plain running max; the rescale factor of this tile goes to the
        // correction warps (1 when the max did not grow)
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = (m_new > m_run && m_run != -INFINITY) ? ex2_approx(__fsub_rn(m_run, m_new)) : 1.f;
        // P V_{j-1} has completed: the MMA warp has taken O-ready of tile j - 1,
        // so the correction warps are done with tile j - 1's factors (the slot
        // and the alpha / O-ready barrier phases can move on), and P_X(j - 1)
        // has been read (its buffer can take P_X(j))
        if (j > 0 && !warp_wait(bar(kBarPVDone + X), (j - 1) & 1, status)) {
          ok = false;
          break;
        }
        alpha_s[X * 128 + row] = alpha;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarAlpha + X));
        m_run = m_new;
        const float nmb = m_run == -INFINITY ? 0.f : -__fsub_rn(m_run, kLog2P8);
        tile_args<kSmoothQ>(s, c, nmb);
        // The two softmax warpgroups take turns for their exponentials (A's
        // tile j, B's tile j, A's tile j + 1, ...).
        if (X == 0 ? (j >= 1 && j - 1 < TB) : (j < TA)) {
          if (!warp_wait(bar(kBarTurn + X), (X == 0 ? j - 1 : j) & 1, status)) {
            ok = false;
            break;
          }
        }
        const float lsum = tile_exp<C::kPTmem>(s, pdst, rx);
        if (X == 0 ? j < TB : j + 1 < TA) {
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarTurn + (1 - X)));
        }
        l = __fmaf_rn(l, alpha, lsum);
        // the P stores complete (TMEM) or become visible to the tensor core's
        // async proxy (shared memory), then P_j is handed to the MMA warp
        if constexpr (C::kPTmem) tmem_st_wait();
        else fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarPReady + X));
      }
      if (ok) {
        l_s[X * 128 + row] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarLReady + X));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------ debug: one P V tile
// 128 threads; P from global (row-major 128x128 e4m3) written into shared
// memory with the 128-byte swizzle; V tile by TMA; O = P V (kind::f8f6f4,
// both operands from shared memory): a check of the FP8 tensor-core path's
// fp32 accumulation.
template <int D>
__global__ void __launch_bounds__(128, 1)
debug_pv_kernel(const __grid_constant__ CUtensorMap tm_v, const Problem pb, const Workspace ws,
                int b, int hkv, int ktile, const uint8_t *p8, float *o_out) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  const uint32_t sP = smem_u32(smem), sV = sP + 128 * 128;
  const uint32_t bar0 = sV + C::kVBytes, bar1 = bar0 + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 128 * 128 + C::kVBytes + 16);
  const int warp = threadIdx.x / 32;
  const int row = threadIdx.x;
  if (threadIdx.x == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar1, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  for (int cc = 0; cc < 8; ++cc)
    *reinterpret_cast<uint4 *>(smem + swz_offset(row, 16 * cc, 128)) =
        *reinterpret_cast<const uint4 *>(p8 + row * 128 + 16 * cc);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar0, C::kVBytes);
    tma_load_2d(sV, &tm_v, bar0, ktile * 128, (b * pb.Hkv + hkv) * D);
    ok = mbar_wait(bar0, 0, ws.status);
    if (ok) {
      tc_fence_after();
      const uint64_t dP = smem_desc_kmajor(sP, 128), dV = smem_desc_kmajor(sV, 128);
      for (int k = 0; k < 4; ++k)
        mma_f8_ss(tmem, dP + 2 * k, dV + 2 * k, idesc_e4m3_f32(128, D), k > 0 ? 1u : 0u);
      mma_commit(bar1);
    }
  }
  if (__syncthreads_and(ok ? 1 : 0) && warp_wait(bar1, 0, ws.status)) {
    tc_fence_after();
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + 32 * c, r);
      for (int e = 0; e < 32; ++e) o_out[row * D + 32 * c + e] = __uint_as_float(r[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------ debug: e4m3, ex2
__global__ void debug_e4m3_kernel(const float *in, uint8_t *out, int64_t n) {
  const int64_t i = 2 * (int64_t(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float lo = in[i], hi = (i + 1 < n) ? in[i + 1] : 0.f;
  const uint32_t pr = e4m3x2(lo, hi);
  out[i] = uint8_t(pr & 0xFF);
  if (i + 1 < n) out[i + 1] = uint8_t(pr >> 8);
}

// The attention kernel's exp2 (ex2.approx.ftz.f32) applied elementwise.
__global__ void debug_ex2_kernel(const float *in, float *out, int64_t n) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) out[i] = ex2_approx(in[i]);
}

// ------------------------------------------------------------ debug: MMA loop
// Back-to-back 8-bit MMAs 128x256x32 from resident shared-memory operands:
// kind::i8 (kind 0) or kind::f8f6f4 e4m3 (kind 1).
__global__ void __launch_bounds__(128, 1) mma_loop_kernel(int iters, int kind, int32_t *sink, int *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  const uint32_t sA = smem_u32(smem), sB = sA + 128 * 128;
  const uint32_t bar0 = sB + 256 * 128;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 128 * 128 + 256 * 128 + 16);
  const int warp = threadIdx.x / 32;
  for (int o = 4 * threadIdx.x; o < 384 * 128; o += 4 * blockDim.x)
    *reinterpret_cast<uint32_t *>(smem + o) = 0x01010101u * ((o >> 7) & 3);
  if (threadIdx.x == 0) {
    mbar_init(bar0, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    const uint64_t dA = smem_desc_kmajor(sA, 128), dB = smem_desc_kmajor(sB, 128);
    if (kind == 0) {
      const uint32_t id = idesc_i8(128, 256);
      for (int it = 0; it < iters; ++it)
#pragma unroll
        for (int k = 0; k < 4; ++k) mma_i8_ss(tmem, dA + 2 * k, dB + 2 * k, id, (it | k) ? 1u : 0u);
    } else {
      const uint32_t id = idesc_e4m3_f32(128, 256);
      for (int it = 0; it < iters; ++it)
#pragma unroll
        for (int k = 0; k < 4; ++k) mma_f8_ss(tmem, dA + 2 * k, dB + 2 * k, id, (it | k) ? 1u : 0u);
    }
    mma_commit(bar0);
    mbar_wait(bar0, 0, status);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    uint32_t r[32];
    tmem_ld32(tmem, r);
    if (threadIdx.x == 0) sink[blockIdx.x] = int32_t(r[0]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------ debug: bounded wait
__global__ void wait_timeout_kernel(int *status) {
  __shared__ __align__(8) uint64_t b;
  const uint32_t bar = smem_u32(&b);
  mbar_init(bar, 1);
  fence_mbar_init();
  mbar_wait(bar, 0, status, false);  // nothing arrives: gives up after the limit
}

template <int D, bool SQ, bool VL, bool DUMP>
cudaError_t launch_attention_dq(const Problem &pb, const Workspace &ws, const CUtensorMap &tq,
                                const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t stream) {
  using C = Cfg<D>;
  // The warpgroup register split adds up to exactly the launch allocation of
  // kLaunchRegs per thread; with any other count the softmax warpgroups'
  // setmaxnreg.inc could not be satisfied, so such a build is refused.
  static const int launch_regs = [] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, attn_fwd_kernel<D, SQ, VL, DUMP>) == cudaSuccess ? fa.numRegs : -1;
  }();
  if (launch_regs != int(kLaunchRegs)) return cudaErrorInvalidKernelImage;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, SQ, VL, DUMP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const unsigned grid = VL ? unsigned(pb.Hq) * unsigned(pb.tot_q256)
                           : unsigned(pb.B) * unsigned(pb.Hq) * unsigned((ws.nqb + 1) / 2);
  if (grid == 0) return cudaSuccess;
  attn_fwd_kernel<D, SQ, VL, DUMP><<<grid, C::kThreads, C::kSmem, stream>>>(tq, tk, tv, pb, ws);
  return cudaGetLastError();
}

template <int D, bool DUMP>
cudaError_t launch_attention_d(const Problem &pb, const Workspace &ws, const CUtensorMap &tq,
                               const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t stream) {
  if (pb.cu_q)
    return pb.smooth_q ? launch_attention_dq<D, true, true, DUMP>(pb, ws, tq, tk, tv, stream)
                       : launch_attention_dq<D, false, true, DUMP>(pb, ws, tq, tk, tv, stream);
  return pb.smooth_q ? launch_attention_dq<D, true, false, DUMP>(pb, ws, tq, tk, tv, stream)
                     : launch_attention_dq<D, false, false, DUMP>(pb, ws, tq, tk, tv, stream);
}

template <int D>
cudaError_t launch_debug_pv_d(const Problem &pb, const Workspace &ws, const CUtensorMap &tv, int b,
                              int hkv, int kt, const uint8_t *p8, float *o, cudaStream_t stream) {
  using C = Cfg<D>;
  const int smem = 128 * 128 + C::kVBytes + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(debug_pv_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  debug_pv_kernel<D><<<1, 128, smem, stream>>>(tv, pb, ws, b, hkv, kt, p8, o);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Problem &pb, const Workspace &ws, const CUtensorMap &tq,
                             const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t stream) {
  switch (pb.D) {
    case 64: return launch_attention_d<64, false>(pb, ws, tq, tk, tv, stream);
    case 96: return launch_attention_d<96, false>(pb, ws, tq, tk, tv, stream);
    case 128: return launch_attention_d<128, false>(pb, ws, tq, tk, tv, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attention_dump(const Problem &pb, const Workspace &ws, const CUtensorMap &tq,
                                  const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t stream) {
  switch (pb.D) {
    case 64: return launch_attention_d<64, true>(pb, ws, tq, tk, tv, stream);
    case 96: return launch_attention_d<96, true>(pb, ws, tq, tk, tv, stream);
    case 128: return launch_attention_d<128, true>(pb, ws, tq, tk, tv, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_debug_pv(const Problem &pb, const Workspace &ws, const CUtensorMap &tv, int b,
                            int hkv, int kt, const uint8_t *p8, float *o, cudaStream_t stream) {
  switch (pb.D) {
    case 64: return launch_debug_pv_d<64>(pb, ws, tv, b, hkv, kt, p8, o, stream);
    case 96: return launch_debug_pv_d<96>(pb, ws, tv, b, hkv, kt, p8, o, stream);
    case 128: return launch_debug_pv_d<128>(pb, ws, tv, b, hkv, kt, p8, o, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_debug_e4m3(const float *in, uint8_t *out, int64_t n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int64_t pairs = (n + 1) / 2;
  debug_e4m3_kernel<<<unsigned((pairs + 255) / 256), 256, 0, stream>>>(in, out, n);
  return cudaGetLastError();
}

cudaError_t launch_debug_ex2(const float *in, float *out, int64_t n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  debug_ex2_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(in, out, n);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout(int *status, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 1, 0, stream>>>(status);
  return cudaGetLastError();
}

cudaError_t launch_mma_loop(int ctas, int iters, int kind, int32_t *sink, cudaStream_t stream) {
  const int smem = 384 * 128 + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(mma_loop_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem);
  if (e != cudaSuccess) return e;
  // the sink doubles as the status word location after the per-CTA outputs
  mma_loop_kernel<<<ctas, 128, smem, stream>>>(iters, kind, sink, reinterpret_cast<int *>(sink + ctas));
  return cudaGetLastError();
}

}  // namespace sage
