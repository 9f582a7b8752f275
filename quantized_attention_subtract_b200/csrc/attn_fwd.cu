// attn_fwd.cu -- the quantized attention kernel for sm_100a.
//
// Computes, per (batch, query head, 128-row query tile), the flash-style
// pass the SageAttention pages describe (INT8 Q K^T, FP8 P V; closerAI
// ComfyUI blog, part 2; "sageattention" package page, "What it is"):
//   S = q8 k8^T                    exact int32, tensor cores (kind::i8)
//   s = S * q_scale * k_scale * sm_scale * log2(e)   (+ dS for smoothed Q)
//   online softmax in base 2 with a lazily raised reference max m (raised
//   only past m + 1) and sum l
//   P8 = e4m3(224 * 2^(s - m))     FP8 probabilities (<= 448 since s <= m + 1)
//   O += P8 v8                     fp32 accumulation, tensor cores (kind::f8f6f4)
//   out = O * v_scale / l (+ mean_v), rounded to bf16 / fp16
//
// One CTA (256 threads, two warpgroups) owns one query tile; two CTAs share
// an SM, so the tensor core alternates between them while each runs its
// softmax.  The helper warpgroup gives registers to the softmax warpgroup
// (setmaxnreg).
//   warp 0      TMA producer: Q once, then K_0, K_1, V_0, K_2, V_1, ... into a
//               3-stage shared-memory ring (order = MMA consumption order)
//   warp 1      allocates 256 TMEM columns and issues the MMAs:
//               S_{j+1} = Q K_{j+1}^T as soon as softmax has read S_j, then
//               O += P_j V_j once P_j is in shared memory
//               (both roles run their loop with the whole warp and issue from
//               one elected lane; their waits carry a suspend-time hint)
//   warps 2-3   idle
//   warps 4-7   softmax: one query row per thread (TMEM lane), reads S with
//               tcgen05.ld, writes P_j (swizzled, double-buffered) to shared
//               memory 32 keys at a time, rescales its O row in TMEM when the
//               reference max moves (overlapped with the exponentials), and
//               runs the epilogue
// TMEM: S at columns [0,128), O at [128, 128 + D).
// Causal tiles past the diagonal are skipped; keys >= Nkv and (causal)
// keys > query are masked; rows >= Nq are computed but not stored.
// Template flags: smoothed Q (dS added to the logits), fused Q (the CTA
// quantises its own Q tile from the 16-bit input before the roles split),
// variable-length batches (per-sequence lengths and offsets; only query tiles
// inside a sequence are launched).
// Every tcgen05.ld / st here runs under warp-uniform control flow (.sync.aligned).
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
  static constexpr int kQKSteps = D / 32;             // K=32 bytes per 8-bit MMA
  static constexpr int kStages = 3;
  static constexpr int kQBytes = 128 * Dp;
  static constexpr int kKBytes = 128 * Dp;
  static constexpr int kVBytes = D * 128;
  static constexpr int kStageBytes = kKBytes > kVBytes ? kKBytes : kVBytes;
  static constexpr int kPBytes = 128 * 128;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kOffQ + kQBytes;
  static constexpr int kOffP = kOffRing + kStages * kStageBytes;
  static constexpr int kOffBar = kOffP + 2 * kPBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = kOffBar + kBarBytes + 1024;   // +1024: base alignment slack
  static constexpr uint32_t kTmemCols = 256;
  static constexpr int kThreads = 256;
};

// Register split of the attention CTA (256 threads launched at 128 registers
// each): the helper warpgroup (TMA producer, MMA issuer, two idle warps)
// gives registers back, the softmax warpgroup takes them.  56 * 128 + 200 *
// 128 == 256 * 128, the block's whole allocation.
constexpr uint32_t kLaunchRegs = 128, kHelperRegs = 56, kSoftmaxRegs = 200;
static_assert(kHelperRegs * 128 + kSoftmaxRegs * 128 == kLaunchRegs * 256, "register split");

// Barrier slots (8 bytes each) inside the barrier area.
enum Bar {
  kBarQ = 0,
  kBarFull = 1,    // + stage (3)
  kBarEmpty = 4,   // + stage (3)
  kBarSFull = 7,
  kBarSEmpty = 8,
  kBarPFull = 9,   // + buffer (2)
  kBarPVDone = 11, // + buffer (2)
  kBarFinal = 13,
  kNumBars = 14
};

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

// One query row's share of one KV tile (128 keys), in two parts around the
// lazy reference-max update.
//
// tile_max: s[] holds the int32 S row from TMEM and is biased in place to the
// fp32 bit patterns of 1.5 * 2^23 + S (exact for |S| < 2^22, same order as
// S); with smoothed Q it then holds the logits x = S * c_half + dsk.  Keys
// k >= lim (only when kMasked) are set to -inf.  Returns the tile max of the
// logits over the valid keys [0, lim) (-inf if none).
template <bool kMasked, bool kSmoothQ>
__device__ __forceinline__ float tile_max(uint32_t (&s)[128], float c0, float c1,
                                          const float *dsk_tile, int lim) {
  constexpr float kBias = 12582912.0f;
#define X(k) __uint_as_float(s[k])
#pragma unroll
  for (int k = 0; k < 128; ++k) s[k] += 0x4B400000u;
  if (kSmoothQ) {
    const float2 nb = make_float2(-kBias, -kBias);
#pragma unroll
    for (int k = 0; k < 128; k += 4) {
      const float4 d4 = __ldg(reinterpret_cast<const float4 *>(dsk_tile + k));
      const float c = k < 64 ? c0 : c1;
      const float2 c2 = make_float2(c, c);
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
  // eight independent 3-input max chains keep the dependency depth at 8
  float h[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) h[q] = -INFINITY;
#pragma unroll
  for (int k = 0; k < 64; k += 8) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k0 = k + 2 * q, k1 = k0 + 64;
      h[q] = fmax3(h[q], X(k0), X(k0 + 1));
      h[q + 4] = fmax3(h[q + 4], X(k1), X(k1 + 1));
    }
  }
  const float h0 = fmaxf(h[0], h[1]), h1 = fmaxf(h[2], h[3]);
  const float h2 = fmaxf(h[4], h[5]), h3 = fmaxf(h[6], h[7]);
  const float lo = fmaxf(h0, h1), hi = fmaxf(h2, h3);
  if (kSmoothQ) return fmaxf(lo, hi);
  // max_j fl(S_j * c) == fl(max_j S_j * c) since c >= 0; the biased max
  // minus the bias is max_j S_j exactly
  return fmaxf(lo == -INFINITY ? -INFINITY : __fmul_rn(__fsub_rn(lo, kBias), c0),
               hi == -INFINITY ? -INFINITY : __fmul_rn(__fsub_rn(hi, kBias), c1));
#undef X
}

// tile_exp: probabilities 2^(x - m_used + log2 224) of the valid keys, their
// sum (returned) and their FP8 codes, stored to this row of the swizzled P
// buffer 32 keys at a time.  With `rescale` (warp-uniform) the O row is
// multiplied by `alpha` (1 for rows whose reference max did not move) in
// 32-column TMEM chunks, chunk c's load in flight behind the exponentials of
// keys 32 (c + 1) .. 32 (c + 1) + 31.  Pairs of keys go through f32x2 ops; every lane of a packed
// op rounds like its scalar counterpart.
template <int D, bool kSmoothQ>
__device__ __forceinline__ float tile_exp(const uint32_t (&s)[128], float c0, float c1, float nmb,
                                          uint32_t prow_s, uint32_t rx, bool rescale, float alpha,
                                          uint32_t tO) {
  constexpr float kBias = 12582912.0f;
  constexpr int kChunks = D / 32;
#define X(k) __uint_as_float(s[k])
  uint32_t o[32];
  float2 acc01 = make_float2(0.f, 0.f), acc23 = make_float2(0.f, 0.f);
  const float2 nmb2 = make_float2(nmb, nmb), nb2 = make_float2(-kBias, -kBias);
  const float2 a2 = make_float2(alpha, alpha);
  // A scale product of exactly 0 means an all-zero Q or K block, so S = 0
  // there; the smallest normal float in its place leaves S * c = 0 and keeps
  // masked keys at -inf * c = -inf instead of NaN.
  const float c0e = c0 == 0.f ? FLT_MIN : c0, c1e = c1 == 0.f ? FLT_MIN : c1;
  const float2 c02 = make_float2(c0e, c0e), c12 = make_float2(c1e, c1e);
#pragma unroll
  for (int sec = 0; sec < 4; ++sec) {
    // O chunk sec - 1 is rescaled while the exponentials of keys 32 sec ..
    // 32 sec + 31 are computed (register pressure peaks in section 0)
    const int ch = sec - 1;
    if (ch >= 0 && ch < kChunks && rescale) tmem_ld32_issue(tO + 32 * ch, o);
    uint32_t pk[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int k = 32 * sec + 4 * q;
      float2 t01, t23;
      const float2 x01 = make_float2(X(k), X(k + 1)), x23 = make_float2(X(k + 2), X(k + 3));
      if (kSmoothQ) {
        t01 = __fadd2_rn(x01, nmb2);
        t23 = __fadd2_rn(x23, nmb2);
      } else {
        const float2 c2 = k < 64 ? c02 : c12;
        t01 = __ffma2_rn(__fadd2_rn(x01, nb2), c2, nmb2);
        t23 = __ffma2_rn(__fadd2_rn(x23, nb2), c2, nmb2);
      }
      const float2 p01 = make_float2(ex2_approx(t01.x), ex2_approx(t01.y));
      const float2 p23 = make_float2(ex2_approx(t23.x), ex2_approx(t23.y));
      acc01 = __fadd2_rn(acc01, p01);
      acc23 = __fadd2_rn(acc23, p23);
      pk[q] = e4m3x4(p01.x, p01.y, p23.x, p23.y);
    }
    // keys 32 sec .. 32 sec + 31 are the 16-byte units 2 sec and 2 sec + 1 of the row
    sts128(prow_s + ((32u * sec) ^ rx), pk[0], pk[1], pk[2], pk[3]);
    sts128(prow_s + ((32u * sec + 16u) ^ rx), pk[4], pk[5], pk[6], pk[7]);
    if (ch >= 0 && ch < kChunks && rescale) {
      tmem_ld32_wait(o);
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float2 o2 = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
        o[e] = __float_as_uint(o2.x);
        o[e + 1] = __float_as_uint(o2.y);
      }
      tmem_st32_issue(tO + 32 * ch, o);
    }
  }
  if (kChunks == 4 && rescale) {
    tmem_ld32_issue(tO + 96, o);
    tmem_ld32_wait(o);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float2 o2 = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
      o[e] = __float_as_uint(o2.x);
      o[e + 1] = __float_as_uint(o2.y);
    }
    tmem_st32_issue(tO + 96, o);
  }
  if (rescale) tmem_st_wait();
  return (acc01.x + acc01.y) + (acc23.x + acc23.y);
#undef X
}

// Fused Q quantisation (no smoothing of Q), run by all 256 threads of the
// CTA before the warp roles split: the CTA's 16-bit Q tile is in shared
// memory at `qin` as D/32 boxes of [128 rows][32 channels] with the 64-byte
// swizzle (rows past Nq are zero).  Thread (row, half) reads the half's
// 16-channel units of its row, the eight warps agree on the block amax (one
// CTA barrier), and every thread writes its units' INT8 codes into the
// swizzled Q operand tile `sq` and into the workspace copy `q8_row` (half 1
// also writes the zero padding units when D < Dp).  The same arithmetic as
// the pre-pass: scale = amax / 127, code = rint(fl(x * (127 / amax))).
// Returns the block scale.  With ok == false the tile is not read and the
// codes are zero.
template <int D>
__device__ __forceinline__ float fused_quantize_q(const uint8_t *qin, uint8_t *sq, uint8_t *q8_row,
                                                  float *xw, bool ok, bool bf16, int row, int half) {
  constexpr int Dp = Cfg<D>::Dp, kMine = D / 32;  // 16-channel units per half row
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int u0 = half * kMine;
  uint32_t w[8 * kMine];  // 16-bit channel pairs (channel 2i in the low half)
#pragma unroll
  for (int t = 0; t < kMine; ++t) {
    const int u = u0 + t;  // unit u = chunks 2 (u % 2), +1 of box u / 2
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (ok) v = *reinterpret_cast<const uint4 *>(qin + 8192 * (u >> 1) + swz_offset(row, 32 * (u & 1) + 16 * c, 64));
      w[8 * t + 4 * c] = v.x;
      w[8 * t + 4 * c + 1] = v.y;
      w[8 * t + 4 * c + 2] = v.z;
      w[8 * t + 4 * c + 3] = v.w;
    }
  }
  // |x| of a finite 16-bit float orders like its bit pattern with the sign
  // cleared; four independent max chains
  uint32_t m4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int e = 0; e < 8 * kMine; ++e) m4[e & 3] = __vmaxu2(m4[e & 3], w[e] & 0x7FFF7FFFu);
  const uint32_t m2 = __vmaxu2(__vmaxu2(m4[0], m4[1]), __vmaxu2(m4[2], m4[3]));
  const uint32_t mb = max(m2 & 0xFFFFu, m2 >> 16);
  float amax = bf16 ? __uint_as_float(mb << 16) : __half2float(__ushort_as_half((unsigned short)mb));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) xw[warp] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(fmaxf(xw[0], xw[1]), fmaxf(xw[2], xw[3])), fmaxf(fmaxf(xw[4], xw[5]), fmaxf(xw[6], xw[7])));
  float scale = 0.f, inv = 0.f;
  if (amax >= kTinyAmax) {
    scale = __fdiv_rn(amax, 127.0f);
    inv = __fdiv_rn(127.0f, amax);
  }
#pragma unroll
  for (int t = 0; t < kMine; ++t) {
    uint32_t cw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w0 = w[8 * t + 2 * q], w1 = w[8 * t + 2 * q + 1];
      float2 x01, x23;
      if (bf16) {
        x01 = make_float2(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xFFFF0000u));
        x23 = make_float2(__uint_as_float(w1 << 16), __uint_as_float(w1 & 0xFFFF0000u));
      } else {
        x01 = __half22float2(*reinterpret_cast<const __half2 *>(&w0));
        x23 = __half22float2(*reinterpret_cast<const __half2 *>(&w1));
      }
      // scalar int8_bits: its separately rounded multiply and add must not be
      // contracted into one fused multiply-add (packed f32x2 forms may be)
      cw[q] = pack4_lo(int8_bits(x01.x, inv), int8_bits(x01.y, inv), int8_bits(x23.x, inv),
                       int8_bits(x23.y, inv));
    }
    const int u = u0 + t;
    const uint4 c4 = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    *reinterpret_cast<uint4 *>(sq + swz_offset(row, 16 * u, Dp)) = c4;
    *reinterpret_cast<uint4 *>(q8_row + 16 * u) = c4;
  }
  if (half == 1) {
#pragma unroll
    for (int u = D / 16; u < Dp / 16; ++u) {
      *reinterpret_cast<uint4 *>(sq + swz_offset(row, 16 * u, Dp)) = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4 *>(q8_row + 16 * u) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  return scale;
}

// One K or V tile load of the producer thread into ring stage n % kStages
// (after the stage's previous contents were consumed; bounded wait), in the
// MMA's consumption order; advances n.  ok turns false on a timeout.
template <int D>
__device__ __forceinline__ void issue_kv(bool isK, int j, int &n, bool &ok, uint32_t bars,
                                         uint32_t sRing, const CUtensorMap *tm_k,
                                         const CUtensorMap *tm_v, int krow0, int vrow0, int *status) {
  using C = Cfg<D>;
  if (!ok) return;
  const int st = n % C::kStages;
  const uint32_t ph = (n / C::kStages) & 1;
  if (!mbar_wait_h(bars + 8u * uint32_t(kBarEmpty + st), ph ^ 1, status)) {
    ok = false;
    return;
  }
  const uint32_t dst = sRing + st * C::kStageBytes, full = bars + 8u * uint32_t(kBarFull + st);
  if (isK) {
    mbar_arrive_expect_tx(full, C::kKBytes);
    tma_load_2d(dst, tm_k, full, 0, krow0 + j * kKVTile);
  } else {
    mbar_arrive_expect_tx(full, C::kVBytes);
    tma_load_2d(dst, tm_v, full, j * kKVTile, vrow0);
  }
  ++n;
}

// The same issued by a whole warp (warp-uniform control flow, so that the
// coordinates stay in uniform registers): every lane waits for the stage,
// the elected lane arms its barrier and issues the copy.
template <int D>
__device__ __forceinline__ void issue_kv_warp(bool isK, int j, int &n, bool &ok, bool leader,
                                              uint32_t bars, uint32_t sRing, const CUtensorMap *tm_k,
                                              const CUtensorMap *tm_v, int krow0, int vrow0,
                                              int *status) {
  using C = Cfg<D>;
  if (!ok) return;
  const int st = n % C::kStages;
  const uint32_t ph = (n / C::kStages) & 1;
  if (!warp_wait_h(bars + 8u * uint32_t(kBarEmpty + st), ph ^ 1, status)) {
    ok = false;
    return;
  }
  const uint32_t dst = sRing + st * C::kStageBytes, full = bars + 8u * uint32_t(kBarFull + st);
  if (leader) {
    if (isK) {
      mbar_arrive_expect_tx(full, C::kKBytes);
      tma_load_2d(dst, tm_k, full, 0, krow0 + j * kKVTile);
    } else {
      mbar_arrive_expect_tx(full, C::kVBytes);
      tma_load_2d(dst, tm_v, full, j * kKVTile, vrow0);
    }
  }
  __syncwarp();
  ++n;
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int D, bool kSmoothQ, bool kFuseQ, bool kVarlen>
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
  const uint32_t sQ = s_base + C::kOffQ, sRing = s_base + C::kOffRing, sP = s_base + C::kOffP;
  const uint32_t bars = s_base + C::kOffBar;
  auto bar = [&](int i) { return bars + 8u * uint32_t(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffBar + 8 * kNumBars);

  const int warp = __shfl_sync(0xffffffffu, int(threadIdx.x / 32), 0), lane = threadIdx.x % 32;
  int *status = ws.status;

  // ---- work item: (b, h, query tile); causal runs the longest tiles first
  const int nq = ws.nqb, bhq = pb.B * pb.Hq;
  int qt, bh;
  if (kVarlen) {
    // only the query tiles inside a sequence are launched
    int sb, sh;
    seq_unit(pb.pc_q128, pb.B, pb.Hq, blockIdx.x, sb, sh, qt);
    bh = sb * pb.Hq + sh;
  } else if (pb.is_causal) {
    qt = nq - 1 - int(blockIdx.x / bhq);
    bh = int(blockIdx.x % bhq);
  } else {
    qt = int(blockIdx.x % nq);
    bh = int(blockIdx.x / nq);
  }
  const int b = bh / pb.Hq, h = bh % pb.Hq;
  const int hk = h / (pb.Hq / pb.Hkv), bhk = b * pb.Hkv + hk;
  const int q0 = qt * kQBlk;
  // this entry's lengths (a sequence of a variable-length batch may be
  // shorter than the padded maximum: its surplus query tiles do nothing)
  const int Nq_b = kVarlen ? nq_of(pb, b) : pb.Nq, Nkv_b = kVarlen ? nkv_of(pb, b) : pb.Nkv;
  if (kVarlen && q0 >= Nq_b) return;
  const int nkt_all = (Nkv_b + kKVTile - 1) / kKVTile;
  int T = nkt_all;
  if (pb.is_causal) T = min(nkt_all, min(q0 + kQBlk - 1, Nq_b - 1) / kKVTile + 1);

  if (threadIdx.x == 0) {
    // the softmax warps (4) arrive on S-empty and P-full; TMA bytes or a
    // single tcgen05.commit complete the others
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(bar(i), (i == kBarSEmpty || i == kBarPFull || i == kBarPFull + 1) ? 4 : 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  const bool skip_all = *(volatile int *)status != 0;  // an earlier CTA already failed

  // ---- producer (thread 0) state: with fused Q the first ring loads are
  // issued before the roles split, so that they land while Q is quantised;
  // n_carry of them, which the producer loop then skips
  int n_carry = 0;
  if constexpr (kFuseQ) {
    if (threadIdx.x == 0 && !skip_all) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      // the 16-bit Q tile into the P buffers (free until the first P_j):
      // D/32 boxes of 32 channels x 128 rows, zero past Nq
      mbar_arrive_expect_tx(bar(kBarQ), 128 * D * 2);
#pragma unroll
      for (int bx = 0; bx < D / 32; ++bx) {
        if (pb.q_map_hn)
          tma_load_4d(sP + 8192 * bx, &tm_q, bar(kBarQ), 32 * bx, h, q0, b);
        else
          tma_load_4d(sP + 8192 * bx, &tm_q, bar(kBarQ), 32 * bx, q0, h, b);
      }
      // the first stages (fresh: no wait) in consumption order K_0, K_1, V_0
      bool ok = true;
      issue_kv<D>(true, 0, n_carry, ok, bars, sRing, &tm_k, &tm_v, bhk * ws.Nkv_pad, bhk * D, status);
      if (T > 1) issue_kv<D>(true, 1, n_carry, ok, bars, sRing, &tm_k, &tm_v, bhk * ws.Nkv_pad, bhk * D, status);
      issue_kv<D>(false, 0, n_carry, ok, bars, sRing, &tm_k, &tm_v, bhk * ws.Nkv_pad, bhk * D, status);
    }
  }
  float qs_fused = 0.f;
  if constexpr (kFuseQ) {
    // ---- every thread: quantise the Q tile (thread = (row, half)); the
    // generic writes of the INT8 tile are made visible to the tensor core's
    // async proxy before the barrier that precedes the first MMA
    const bool qok = !skip_all && mbar_wait(bar(kBarQ), 0, status);
    const int qrow = threadIdx.x & 127, qhalf = threadIdx.x >> 7;
    float *xw = reinterpret_cast<float *>(smem + C::kOffBar + 8 * kNumBars + 16);
    uint8_t *q8_row = reinterpret_cast<uint8_t *>(ws.q8) + ((long long)bh * ws.Nq_pad + q0 + qrow) * C::Dp;
    qs_fused = fused_quantize_q<D>(smem + C::kOffP, smem + C::kOffQ, q8_row, xw, qok, pb.bf16 != 0,
                                   qrow, qhalf);
    if (qok && threadIdx.x == 0) ws.q_scale[(long long)bh * nq + qt] = qs_fused;
    fence_proxy_async_smem();
    __syncthreads();
  }

  if (warp < 4) {
  reg_dealloc<kHelperRegs>();
  if (warp == 0) {
    // ================================================= TMA producer
    // The whole warp runs the loop; the elected lane issues the copies.
    if (!skip_all) {
      const bool leader = elect_one();
      if constexpr (!kFuseQ) {
        if (leader) {
          tma_prefetch_desc(&tm_q);
          tma_prefetch_desc(&tm_k);
          tma_prefetch_desc(&tm_v);
          mbar_arrive_expect_tx(bar(kBarQ), C::kQBytes);
          tma_load_2d(sQ, &tm_q, bar(kBarQ), 0, bh * ws.Nq_pad + q0);
        }
        __syncwarp();
      }
      // (thread 0 issued the first n_carry loads before the roles split)
      const int carried = kFuseQ ? __shfl_sync(0xffffffffu, n_carry, 0) : 0;
      int n = carried;
      bool ok = true;
      // K_0, K_1, V_0, K_2, V_1, ... skipping the loads issued early
      int pos = 0;
      auto issue = [&](bool isK, int j) {
        if constexpr (kFuseQ) {
          if (pos++ < carried) return;
        }
        issue_kv_warp<D>(isK, j, n, ok, leader, bars, sRing, &tm_k, &tm_v, bhk * ws.Nkv_pad, bhk * D,
                         status);
      };
      issue(true, 0);
      for (int j = 0; j < T; ++j) {
        if (j + 1 < T) issue(true, j + 1);
        issue(false, j);
      }
      // Before leaving, make sure every copy issued has landed (bounded).
      warp_wait_h(bar(kBarQ), 0, status, false);
      for (int m = (n > C::kStages ? n - C::kStages : 0); m < n; ++m)
        warp_wait_h(bar(kBarFull + m % C::kStages), (m / C::kStages) & 1, status, false);
    }
  } else if (warp == 1) {
    // ================================================= MMA issuer
    // The whole warp runs the loop (warp-uniform control flow, so that the
    // descriptors stay in uniform registers); the elected lane issues the
    // MMAs and commits.  Descriptors of the ring stages and P buffers differ
    // only in their start-address field (16-byte units, bits [0, 14)).
    if (!skip_all) {
      const bool leader = elect_one();
      const uint32_t tS = tmem, tO = tmem + 128;
      constexpr uint32_t id_s = idesc_i8(128, 128);
      constexpr uint32_t id_o = idesc_e4m3_f32(128, D);
      constexpr uint64_t kStageStep = uint64_t(C::kStageBytes) >> 4, kPStep = uint64_t(C::kPBytes) >> 4;
      const uint64_t dQ = smem_desc_kmajor(sQ, C::Dp);
      const uint64_t dK0 = smem_desc_kmajor(sRing, C::Dp);
      const uint64_t dV0 = smem_desc_kmajor(sRing, 128);
      const uint64_t dP0 = smem_desc_kmajor(sP, 128);
      int n = 0;
      // with fused Q the INT8 tile was published by the barrier above
      bool ok = kFuseQ ? true : warp_wait_h(bar(kBarQ), 0, status);
      auto wait_stage = [&]() -> uint32_t {
        const int st = n % C::kStages;
        if (ok && !warp_wait_h(bar(kBarFull + st), (n / C::kStages) & 1, status)) ok = false;
        return uint32_t(st);
      };
      auto issue_s = [&](uint32_t st) {
        const uint64_t dK = dK0 + st * kStageStep;
        if (leader) {
#pragma unroll
          for (int k = 0; k < C::kQKSteps; ++k)
            mma_i8_ss(tS, dQ + 2 * k, dK + 2 * k, id_s, k > 0 ? 1u : 0u);
          mma_commit(bar(kBarSFull));
          mma_commit(bar(kBarEmpty + st));
        }
        __syncwarp();
        ++n;
      };
      if (ok) {
        const uint32_t st = wait_stage();
        tc_fence_after();
        if (ok) issue_s(st);
      }
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) {
          const uint32_t st = wait_stage();
          if (ok && !warp_wait_h(bar(kBarSEmpty), j & 1, status)) ok = false;
          if (!ok) break;
          tc_fence_after();
          issue_s(st);
        }
        const uint32_t st = wait_stage();
        if (ok && !warp_wait_h(bar(kBarPFull + (j & 1)), (j >> 1) & 1, status)) ok = false;
        if (!ok) break;
        tc_fence_after();
        const uint64_t dP = dP0 + uint64_t(j & 1) * kPStep;
        const uint64_t dV = dV0 + st * kStageStep;
        if (leader) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_f8_ss(tO, dP + 2 * k, dV + 2 * k, id_o, (j > 0 || k > 0) ? 1u : 0u);
          mma_commit(bar(kBarPVDone + (j & 1)));
          mma_commit(bar(kBarEmpty + st));
        }
        __syncwarp();
        ++n;
      }
      // every MMA issued by the elected lane has finished before teardown
      if (leader) mma_commit(bar(kBarFinal));
      __syncwarp();
      warp_wait_h(bar(kBarFinal), 0, status, false);
    }
  }
  } else {
    reg_alloc<kSoftmaxRegs>();
    // ================================================= softmax / correction / epilogue
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int row = 32 * wq + lane;          // row within the query tile
    const int i = q0 + row;                  // query index
    const uint32_t lane_off = uint32_t(32 * wq) << 16;
    const uint32_t tS = tmem + lane_off, tO = tmem + lane_off + 128;
    const float qs = kFuseQ ? qs_fused : ws.q_scale[(long long)bh * nq + qt];
    const uint32_t prow_rx = uint32_t(row & 7) << 4;   // swizzle of this row's 16-byte units
    const float *ksc = ws.k_scale + (long long)bhk * (ws.Nkv_pad / kKBlk);
    const float *dsk = kSmoothQ ? ws.dsk + ((long long)bh * nq + qt) * ws.Nkv_pad : nullptr;
    float m_run = -INFINITY, l = 0.f;
    bool ok = !skip_all;
    float ks0 = ksc[0], ks1 = ksc[1];   // K block scales of the tile, one tile ahead
    for (int j = 0; ok && j < T; ++j) {
      const int kb = j * kKVTile;
      const float c0 = __fmul_rn(__fmul_rn(qs, ks0), pb.K2);
      const float c1 = __fmul_rn(__fmul_rn(qs, ks1), pb.K2);
      if (j + 1 < T) {
        ks0 = ksc[2 * j + 2];
        ks1 = ksc[2 * j + 3];
      }
      if (!warp_wait(bar(kBarSFull), j & 1, status)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[128];
      tmem_ld64x2(tS, s);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarSEmpty));

      // valid keys of this tile for this row form the prefix [0, lim)
      int lim = min(kKVTile, Nkv_b - kb);
      if (pb.is_causal) lim = min(lim, i - kb + 1);
      const bool masked = lim < kKVTile;
      const float *dsk_tile = kSmoothQ ? dsk + kb : nullptr;
      const float m_tile = masked ? tile_max<true, kSmoothQ>(s, c0, c1, dsk_tile, lim)
                                  : tile_max<false, kSmoothQ>(s, c0, c1, dsk_tile, lim);
      // lazy reference max: raised (to the tile max) only when the tile max
      // exceeds it by more than kLazyLog2
      float alpha = 1.f;
      bool need = false;
      if (m_tile != -INFINITY && (m_run == -INFINITY || m_tile > __fadd_rn(m_run, kLazyLog2))) {
        if (m_run != -INFINITY) {
          alpha = ex2_approx(__fsub_rn(m_run, m_tile));
          need = true;
        } else {
          alpha = 0.f;
        }
        m_run = m_tile;
      }
      const float nmb = m_run == -INFINITY ? 0.f : -__fsub_rn(m_run, kLog2P8Scale);
      const bool rescale = __any_sync(0xffffffffu, need);
      // P_j goes to shared buffer j & 1, free once P V_{j-2} is done; a
      // rescale of O needs P V_{j-1} done, which implies P V_{j-2}
      if (rescale) {
        if (!warp_wait(bar(kBarPVDone + ((j - 1) & 1)), ((j - 1) >> 1) & 1, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
      } else if (j >= 2 && !warp_wait(bar(kBarPVDone + (j & 1)), ((j - 2) >> 1) & 1, status)) {
        ok = false;
        break;
      }
      // this row of P_j's buffer (128 bytes; 16-byte units XOR-swizzled by row % 8)
      const uint32_t prow_s = sP + uint32_t(j & 1) * C::kPBytes + uint32_t(row) * 128u;
      const float a_row = need ? alpha : 1.f;
      const float lsum = tile_exp<D, kSmoothQ>(s, c0, c1, nmb, prow_s, prow_rx, rescale, a_row, tO);
      l = __fmaf_rn(l, alpha, lsum);
      // P stores visible to the tensor core (async proxy), TMEM writes ordered,
      // then P_j is handed to the MMA warp
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarPFull + (j & 1)));
    }

    // ---- epilogue: out = O * v_scale / l (+ mean_v)
    if (ok && warp_wait(bar(kBarPVDone + ((T - 1) & 1)), ((T - 1) >> 1) & 1, status)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const float *vs = ws.v_scale + (long long)bhk * D;
      const float *mv = ws.mean_v + (long long)bhk * D;
      uint8_t *orow = reinterpret_cast<uint8_t *>(pb.out) +
                      2 * ((kVarlen ? o_off(pb, b) : b * pb.os_b) + h * pb.os_h + (long long)i * pb.os_n);
#pragma unroll
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
          if (pb.smooth_v) {
            const float4 m4 = __ldg(reinterpret_cast<const float4 *>(mv + 32 * c + e));
            o[0] += m4.x;
            o[1] += m4.y;
            o[2] += m4.z;
            o[3] += m4.w;
          }
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            if (pb.bf16) {
              const __nv_bfloat162 v2 = __floats2bfloat162_rn(o[2 * h2], o[2 * h2 + 1]);
              packed[e / 2 + h2] = *reinterpret_cast<const uint32_t *>(&v2);
            } else {
              const __half2 v2 = __floats2half2_rn(o[2 * h2], o[2 * h2 + 1]);
              packed[e / 2 + h2] = *reinterpret_cast<const uint32_t *>(&v2);
            }
          }
        }
        if (i < Nq_b) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            *reinterpret_cast<uint4 *>(orow + 64 * c + 16 * v4) =
                make_uint4(packed[4 * v4], packed[4 * v4 + 1], packed[4 * v4 + 2], packed[4 * v4 + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------ debug: one S tile
// 128 threads.  S = q8[qtile] k8[ktile]^T through TMA + tcgen05 kind::i8.
template <int D>
__global__ void __launch_bounds__(128, 1)
dump_s_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const Problem pb, const Workspace ws, int b, int h, int qtile, int ktile,
              int32_t *s_out) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  const uint32_t sQ = smem_u32(smem), sK = sQ + C::kQBytes;
  const uint32_t bar0 = sK + C::kKBytes, bar1 = bar0 + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kQBytes + C::kKBytes + 16);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar1, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int hk = h / (pb.Hq / pb.Hkv);
  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar0, C::kQBytes + C::kKBytes);
    tma_load_2d(sQ, &tm_q, bar0, 0, (b * pb.Hq + h) * ws.Nq_pad + qtile * 128);
    tma_load_2d(sK, &tm_k, bar0, 0, (b * pb.Hkv + hk) * ws.Nkv_pad + ktile * 128);
    ok = mbar_wait(bar0, 0, ws.status);
    if (ok) {
      tc_fence_after();
      const uint64_t dQ = smem_desc_kmajor(sQ, C::Dp), dK = smem_desc_kmajor(sK, C::Dp);
      for (int k = 0; k < C::kQKSteps; ++k)
        mma_i8_ss(tmem, dQ + 2 * k, dK + 2 * k, idesc_i8(128, 128), k > 0 ? 1u : 0u);
      mma_commit(bar1);
    }
  }
  if (__syncthreads_and(ok ? 1 : 0) && warp_wait(bar1, 0, ws.status)) {
    tc_fence_after();
    const int row = 32 * warp + lane;
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + 32 * c, r);
      for (int e = 0; e < 32; ++e) s_out[row * 128 + 32 * c + e] = int32_t(r[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------ debug: one P V tile
// 128 threads; P from global (row-major 128x128 e4m3) written into shared
// memory with the kernel's swizzle; V tile by TMA; O = P V (kind::f8f6f4).
template <int D>
__global__ void __launch_bounds__(128, 1)
debug_pv_kernel(const __grid_constant__ CUtensorMap tm_v, const Problem pb, const Workspace ws,
                int b, int hkv, int ktile, const uint8_t *p8, float *o_out) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  const uint32_t sP = smem_u32(smem), sV = sP + C::kPBytes;
  const uint32_t bar0 = sV + C::kVBytes, bar1 = bar0 + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kPBytes + C::kVBytes + 16);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
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

// ------------------------------------------------------------ debug: e4m3
__global__ void debug_e4m3_kernel(const float *in, uint8_t *out, int64_t n) {
  const int64_t i = 2 * (int64_t(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float lo = in[i], hi = (i + 1 < n) ? in[i + 1] : 0.f;
  const uint32_t pr = e4m3x2(lo, hi);
  out[i] = uint8_t(pr & 0xFF);
  if (i + 1 < n) out[i + 1] = uint8_t(pr >> 8);
}

// ------------------------------------------------------------ debug: MMA loop
// Back-to-back INT8 MMAs 128x256x32 from resident shared-memory operands.
__global__ void __launch_bounds__(128, 1) mma_loop_kernel(int iters, int32_t *sink, int *status) {
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
    const uint32_t id = idesc_i8(128, 256);
    for (int it = 0; it < iters; ++it)
#pragma unroll
      for (int k = 0; k < 4; ++k) mma_i8_ss(tmem, dA + 2 * k, dB + 2 * k, id, (it | k) ? 1u : 0u);
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

template <int D, bool SQ, bool FQ, bool VL>
cudaError_t launch_attention_dq(const Problem &pb, const Workspace &ws, const CUtensorMap &tq,
                                const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t stream) {
  using C = Cfg<D>;
  // The warpgroup register split adds up to exactly the launch allocation of
  // kLaunchRegs per thread; with any other count the softmax warpgroup's
  // setmaxnreg.inc could not be satisfied, so such a build is refused.
  static const int launch_regs = [] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, attn_fwd_kernel<D, SQ, FQ, VL>) == cudaSuccess ? fa.numRegs : -1;
  }();
  if (launch_regs != int(kLaunchRegs)) return cudaErrorInvalidKernelImage;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, SQ, FQ, VL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const unsigned grid = VL ? unsigned(pb.Hq) * unsigned(pb.tot_q128)
                           : unsigned(pb.B) * unsigned(pb.Hq) * unsigned(ws.nqb);
  if (grid == 0) return cudaSuccess;
  attn_fwd_kernel<D, SQ, FQ, VL><<<grid, C::kThreads, C::kSmem, stream>>>(tq, tk, tv, pb, ws);
  return cudaGetLastError();
}

// ------------------------------------------------------------ debug: bounded wait
__global__ void wait_timeout_kernel(int *status) {
  __shared__ __align__(8) uint64_t b;
  const uint32_t bar = smem_u32(&b);
  mbar_init(bar, 1);
  fence_mbar_init();
  mbar_wait(bar, 0, status, false);  // nothing arrives: gives up after the limit
}

template <int D>
cudaError_t launch_attention_d(const Problem &pb, const Workspace &ws, const CUtensorMap &tq,
                               const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t stream) {
  // Q is fused only without Q smoothing (the smoothed path needs the
  // pre-pass's block means and its Delta S rows)
  // (variable-length batches are never fused)
  if (pb.cu_q)
    return pb.smooth_q ? launch_attention_dq<D, true, false, true>(pb, ws, tq, tk, tv, stream)
                       : launch_attention_dq<D, false, false, true>(pb, ws, tq, tk, tv, stream);
  if (pb.smooth_q) return launch_attention_dq<D, true, false, false>(pb, ws, tq, tk, tv, stream);
  return pb.q_fused ? launch_attention_dq<D, false, true, false>(pb, ws, tq, tk, tv, stream)
                    : launch_attention_dq<D, false, false, false>(pb, ws, tq, tk, tv, stream);
}

template <int D>
cudaError_t launch_dump_s_d(const Problem &pb, const Workspace &ws, const CUtensorMap &tq,
                            const CUtensorMap &tk, int b, int h, int qt, int kt, int32_t *s,
                            cudaStream_t stream) {
  using C = Cfg<D>;
  const int smem = C::kQBytes + C::kKBytes + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(dump_s_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dump_s_kernel<D><<<1, 128, smem, stream>>>(tq, tk, pb, ws, b, h, qt, kt, s);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_debug_pv_d(const Problem &pb, const Workspace &ws, const CUtensorMap &tv, int b,
                              int hkv, int kt, const uint8_t *p8, float *o, cudaStream_t stream) {
  using C = Cfg<D>;
  const int smem = C::kPBytes + C::kVBytes + 64 + 1024;
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
    case 64: return launch_attention_d<64>(pb, ws, tq, tk, tv, stream);
    case 96: return launch_attention_d<96>(pb, ws, tq, tk, tv, stream);
    case 128: return launch_attention_d<128>(pb, ws, tq, tk, tv, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_dump_s(const Problem &pb, const Workspace &ws, const CUtensorMap &tq,
                          const CUtensorMap &tk, int b, int h, int qt, int kt, int32_t *s,
                          cudaStream_t stream) {
  switch (pb.D) {
    case 64: return launch_dump_s_d<64>(pb, ws, tq, tk, b, h, qt, kt, s, stream);
    case 96: return launch_dump_s_d<96>(pb, ws, tq, tk, b, h, qt, kt, s, stream);
    case 128: return launch_dump_s_d<128>(pb, ws, tq, tk, b, h, qt, kt, s, stream);
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

cudaError_t launch_wait_timeout(int *status, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 1, 0, stream>>>(status);
  return cudaGetLastError();
}

cudaError_t launch_mma_loop(int ctas, int iters, int32_t *sink, cudaStream_t stream) {
  const int smem = 384 * 128 + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(mma_loop_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem);
  if (e != cudaSuccess) return e;
  // the sink doubles as the status word location after the per-CTA outputs
  mma_loop_kernel<<<ctas, 128, smem, stream>>>(iters, sink, reinterpret_cast<int *>(sink + ctas));
  return cudaGetLastError();
}

}  // namespace sage
