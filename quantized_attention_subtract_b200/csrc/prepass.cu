// prepass.cu -- smoothing + quantisation pre-pass (HBM-bandwidth bound).
//
// Follows the SageAttention pages: K is smoothed by subtracting its
// per-channel mean over all tokens ("sageattention" package page,
// Quickstart: smooth_k), Q and V may be smoothed by subtracting channel means
// ("SageAttention2: Technical report", section 2), Q and K are quantised per
// block to INT8 and V to FP8 (closerAI ComfyUI blog, part 2).
//
// Four kernels on one stream:
//   kv_stats   persistent; contiguous runs of (b, kv head, 64-token chunk)
//              units per CTA: fixed-point channel sums of K (and V) and the V
//              channel max/min in registers, flushed with atomics when the run
//              changes head (integer addition is exact, so the order does not
//              matter);
//   kv_finalize per (b, kv head): mean_k, mean_v, V channel scale and its
//              reciprocal, once per channel;
//   quantize   persistent over 128-token tiles of K, V, then Q (K/V heads in
//              reverse so their second read hits L2): smoothing, block amax,
//              INT8 codes of K and Q stored from registers, FP8 codes of V
//              transposed through shared memory (keys contiguous), all in the
//              attention kernel's layout;
//   delta_s    (smooth_q only) the correction dS[blk][j] = mq[blk] . K'_j,
//              stored pre-multiplied by sm_scale * log2(e).
//
// Threads own 16-byte chunks (8 channels) of rows, so loads are 16-byte
// vectors and a warp covers whole rows.  Rows arrive in shared memory through
// copies on an mbarrier ring: one cp.async.bulk per unit when tokens are
// dense, one tensor-map box per unit when they are strided (NHD, packed
// variable-length batches, padded rows; one bulk copy per row if the driver
// rejects the map).  Variable-length batches enumerate only the units inside
// a sequence.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace sage {
namespace {


__device__ __forceinline__ void load8(const uint16_t *p, int bf16, float (&x)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t lo = w[i] & 0xFFFFu, hi = w[i] >> 16;
    if (bf16) {
      x[2 * i] = __uint_as_float(uint32_t(lo) << 16);
      x[2 * i + 1] = __uint_as_float(uint32_t(hi) << 16);
    } else {
      x[2 * i] = __half2float(__ushort_as_half(lo));
      x[2 * i + 1] = __half2float(__ushort_as_half(hi));
    }
  }
}

__device__ __forceinline__ unsigned float_key(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Exact fixed-point mean: (sum of rint(x * 2^24)) / (n * 2^24), fp64
// division, one rounding to fp32.
__device__ __forceinline__ float fixed_mean(long long sum, long long n) {
  return __double2float_rn(__ddiv_rn(double(sum), double(n) * 16777216.0));
}

__device__ __forceinline__ long long fixed_point(float x) {
  return __float2ll_rn(__fmul_rn(x, kFixScale));
}

// ------------------------------------------------------------ streaming
// Both streaming kernels are persistent: each block walks a list of units
// (128-token tiles or 64-token chunks) and keeps the rows of the next units in
// flight with cp.async.bulk copies into a ring of shared-memory stages, one
// 16-byte-aligned row per copy (HND and NHD alike), completed on an mbarrier.
constexpr int kStatChunk = 64;     // tokens per kv_stats unit

__device__ __forceinline__ void decode8(uint4 u, int bf16, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t lo = w[i] & 0xFFFFu, hi = w[i] >> 16;
    if (bf16) {
      x[2 * i] = __uint_as_float(uint32_t(lo) << 16);
      x[2 * i + 1] = __uint_as_float(uint32_t(hi) << 16);
    } else {
      x[2 * i] = __half2float(__ushort_as_half(lo));
      x[2 * i + 1] = __half2float(__ushort_as_half(hi));
    }
  }
}

// Issue the copies of one unit: rows [0, nrows) of a tensor starting at
// `src` with element stride `stride` between rows go to `dst` (row pitch
// `rowb` bytes).  Called by every thread.  Dense rows (stride == row length)
// are one copy by thread 0; otherwise thread t copies row t (many small
// copies are much slower than one large one).  Thread 0 arms the barrier
// with the unit's byte count.
__device__ __forceinline__ void issue_rows(uint32_t dst, const uint16_t *src, long long stride,
                                           int nrows, int rowb, uint32_t bar, bool arm,
                                           uint32_t total_bytes) {
  if (arm && threadIdx.x == 0) mbar_arrive_expect_tx(bar, total_bytes);
  if (stride * 2 == rowb) {
    // rows back to back in memory (dense tokens): one copy of the whole run
    if (threadIdx.x == 0 && nrows > 0) bulk_load(dst, src, uint32_t(nrows) * rowb, bar);
  } else if (int(threadIdx.x) < nrows) {
    bulk_load(dst + threadIdx.x * rowb, src + threadIdx.x * stride, rowb, bar);
  }
}

// Tensor-map load of one box (D channels x the map's token count) of head h
// of batch entry b, from token r0 of that entry on: a variable-length batch's
// map spans all packed tokens (entry b starts at token cu[b]) with a batch
// extent of 1.  x = 0, so the 16-byte rule on the innermost coordinate holds.
__device__ __forceinline__ void map_load(uint32_t dst, const CUtensorMap *m, uint32_t bar, int hn,
                                         const int *cu, int b, int h, int r0) {
  const int tok = (cu ? cu[b] : 0) + r0, bb = cu ? 0 : b;
  if (hn) tma_load_4d(dst, m, bar, 0, h, tok, bb);
  else tma_load_4d(dst, m, bar, 0, tok, h, bb);
}

// Thread 0 of a block: arm `bar` with `bytes` and load one box (out of line,
// so that the unit loop that calls it keeps its registers).
__device__ __noinline__ void map_issue(uint32_t dst, const CUtensorMap *m, uint32_t bar, uint32_t bytes,
                                       int hn, const int *cu, int b, int h, int r0) {
  mbar_arrive_expect_tx(bar, bytes);
  map_load(dst, m, bar, hn, cu, b, h, r0);
}

// Tensor-map boxes land at 128-byte aligned shared addresses: the dynamic
// shared array is declared 1024-byte aligned, and a block whose base is not
// 128-byte aligned reports SAGE_ERR_ALIGNMENT and does nothing (block-uniform,
// before any barrier exists).
__device__ __forceinline__ bool smem_misaligned(const uint8_t *base, int *status) {
  if ((smem_u32(base) & 127u) == 0) return false;
  if (threadIdx.x == 0) atomicCAS(status, 0, kStatusAlignment);
  return true;
}

// Block-wide bounded wait; every thread learns whether it succeeded.
__device__ __forceinline__ bool block_wait(uint32_t bar, uint32_t parity, int *status) {
  const bool ok = mbar_wait(bar, parity, status);
  return __syncthreads_and(ok ? 1 : 0) != 0;
}

// ------------------------------------------------------------ kv_stats
// Persistent, grid <= 2 per SM, block 256.  Units are 64-token chunks of one
// (b, kv head), numbered bh * nchunks + chunk; block i takes a contiguous run
// of units, so its partial sums stay in registers and are flushed (block
// reduction + integer / ordered-key atomics) only when the head changes.
// Stage: 64 K rows then 64 V rows (K only when smooth_k).
constexpr int kStatStages = 2;

__global__ void __launch_bounds__(256, 2) kv_stats_kernel(Problem pb, Workspace ws,
                                                          const __grid_constant__ CUtensorMap mk,
                                                          const __grid_constant__ CUtensorMap mv) {
  extern __shared__ __align__(1024) uint8_t sm_stats[];
  if (smem_misaligned(sm_stats, ws.status)) return;
  const int D = pb.D, C8 = D / 8, rowb = 2 * D;
  const int c8 = threadIdx.x % C8, rg = threadIdx.x / C8;   // 16 / 21 / 32 row groups
  const int ngroups = blockDim.x / C8;
  const int nchunk = (pb.Nkv + kStatChunk - 1) / kStatChunk;
  // variable-length batches enumerate only the chunks inside a sequence
  const long long nunits = pb.cu_kv ? (long long)pb.Hkv * pb.tot_kv64 : (long long)pb.B * pb.Hkv * nchunk;
  const long long u0 = nunits * blockIdx.x / gridDim.x, u1 = nunits * (blockIdx.x + 1) / gridDim.x;
  const int stage_bytes = 2 * kStatChunk * rowb;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm_stats + kStatStages * stage_bytes);
  long long *red = reinterpret_cast<long long *>(bars + 8);         // [ngroups][D]
  const uint32_t s_base = smem_u32(sm_stats), b_base = smem_u32(bars);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStatStages; ++i) mbar_init(b_base + 8 * i, 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto unit_src = [&](long long u, int &bh, int &j0, int &n) {
    if (pb.cu_kv) {
      int b, h, t;
      seq_unit(pb.pc_kv64, pb.B, pb.Hkv, u, b, h, t);
      bh = b * pb.Hkv + h;
      j0 = t * kStatChunk;
    } else {
      // unit counts stay below 2^31 (the host's size checks): 32-bit division
      const int ui = int(u);
      bh = ui / nchunk;
      j0 = (ui % nchunk) * kStatChunk;
    }
    n = min(kStatChunk, nkv_of(pb, bh / pb.Hkv) - j0);  // <= 0: past this sequence's end
  };
  auto issue = [&](long long u, int st) {
    int bh, j0, n;
    unit_src(u, bh, j0, n);
    const int b = bh / pb.Hkv, h = bh % pb.Hkv;
    const uint32_t dst = s_base + st * stage_bytes, bar = b_base + 8 * st;
    if (n <= 0) {
      // nothing to copy (past the sequence's end): complete the phase
      if (threadIdx.x == 0) mbar_arrive(bar);
      return;
    }
    // a tensor-map box always lands whole (rows past the tensor read as zero)
    const uint32_t kbytes = pb.smooth_k ? uint32_t(pb.k_map ? kStatChunk : n) * rowb : 0u;
    const uint32_t vbytes = uint32_t(pb.v_map ? kStatChunk : n) * rowb;
    if (threadIdx.x == 0) mbar_arrive_expect_tx(bar, kbytes + vbytes);
    const uint16_t *ksrc = pb.k + k_off(pb, b) + h * pb.ks_h + j0 * pb.ks_n;
    const uint16_t *vsrc = pb.v + v_off(pb, b) + h * pb.vs_h + j0 * pb.vs_n;
    // strided tokens with a tensor map: one box per tensor; dense tokens: one
    // copy per tensor; otherwise one per row (K rows by threads 0.., V rows by
    // threads ..127)
    if (pb.k_map) {
      if (pb.smooth_k && threadIdx.x == 0) map_load(dst, &mk, bar, pb.k_hn, pb.cu_kv, b, h, j0);
    } else if (pb.ks_n == D) {
      if (pb.smooth_k && threadIdx.x == 0) bulk_load(dst, ksrc, uint32_t(n) * rowb, bar);
    } else if (pb.smooth_k && int(threadIdx.x) < n) {
      bulk_load(dst + threadIdx.x * rowb, ksrc + threadIdx.x * pb.ks_n, rowb, bar);
    }
    if (pb.v_map) {
      if (threadIdx.x == 32) map_load(dst + kStatChunk * rowb, &mv, bar, pb.v_hn, pb.cu_kv, b, h, j0);
    } else if (pb.vs_n == D) {
      if (threadIdx.x == 127) bulk_load(dst + kStatChunk * rowb, vsrc, uint32_t(n) * rowb, bar);
    } else if (int(threadIdx.x) >= 128 - n && threadIdx.x < 128) {
      const int r = threadIdx.x - (128 - n);
      bulk_load(dst + (kStatChunk + r) * rowb, vsrc + r * pb.vs_n, rowb, bar);
    }
  };

  long long ksum[8], vsum[8];
  float vmax[8], vmin[8];
  auto reset = [&]() {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      ksum[e] = 0;
      vsum[e] = 0;
      vmax[e] = -INFINITY;
      vmin[e] = INFINITY;
    }
  };
  auto flush = [&](int bh) {
    const bool live = rg < ngroups;
    if (pb.smooth_k) {
      if (live)
#pragma unroll
        for (int e = 0; e < 8; ++e) red[rg * D + 8 * c8 + e] = ksum[e];
      __syncthreads();
      if (int(threadIdx.x) < D) {
        long long t = 0;
        for (int r = 0; r < ngroups; ++r) t += red[r * D + threadIdx.x];
        atomicAdd(reinterpret_cast<unsigned long long *>(ws.k_sum + (long long)bh * D + threadIdx.x),
                  (unsigned long long)t);
      }
      __syncthreads();
    }
    if (pb.smooth_v) {
      if (live)
#pragma unroll
        for (int e = 0; e < 8; ++e) red[rg * D + 8 * c8 + e] = vsum[e];
      __syncthreads();
      if (int(threadIdx.x) < D) {
        long long t = 0;
        for (int r = 0; r < ngroups; ++r) t += red[r * D + threadIdx.x];
        atomicAdd(reinterpret_cast<unsigned long long *>(ws.v_sum + (long long)bh * D + threadIdx.x),
                  (unsigned long long)t);
      }
      __syncthreads();
    }
    float *redf = reinterpret_cast<float *>(red);
    if (live)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        redf[rg * D + 8 * c8 + e] = vmax[e];
        redf[(ngroups + rg) * D + 8 * c8 + e] = vmin[e];
      }
    __syncthreads();
    if (int(threadIdx.x) < D) {
      float mx = -INFINITY, mn = INFINITY;
      for (int r = 0; r < ngroups; ++r) {
        mx = fmaxf(mx, redf[r * D + threadIdx.x]);
        mn = fminf(mn, redf[(ngroups + r) * D + threadIdx.x]);
      }
      atomicMax(ws.v_max + (long long)bh * D + threadIdx.x, float_key(mx));
      atomicMin(ws.v_min + (long long)bh * D + threadIdx.x, float_key(mn));
    }
    __syncthreads();
  };

  reset();
  for (int i = 0; i < kStatStages; ++i)
    if (u0 + i < u1) issue(u0 + i, i);
  int cur_bh = -1;
  bool ok = true;
  for (long long u = u0; u < u1; ++u) {
    const int it = int(u - u0), st = it % kStatStages;
    if (!block_wait(b_base + 8 * st, (it / kStatStages) & 1, ws.status)) { ok = false; break; }
    int bh, j0, n;
    unit_src(u, bh, j0, n);
    if (bh != cur_bh) {
      if (cur_bh >= 0) flush(cur_bh);
      reset();
      cur_bh = bh;
    }
    const uint8_t *stage = sm_stats + st * stage_bytes;
    if (rg < ngroups) {
      for (int r = rg; r < n; r += ngroups) {
        float x[8];
        if (pb.smooth_k) {
          decode8(*reinterpret_cast<const uint4 *>(stage + r * rowb + 16 * c8), pb.bf16, x);
#pragma unroll
          for (int e = 0; e < 8; ++e) ksum[e] += fixed_point(x[e]);
        }
        decode8(*reinterpret_cast<const uint4 *>(stage + (kStatChunk + r) * rowb + 16 * c8), pb.bf16, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          vmax[e] = fmaxf(vmax[e], x[e]);
          vmin[e] = fminf(vmin[e], x[e]);
          if (pb.smooth_v) vsum[e] += fixed_point(x[e]);
        }
      }
    }
    __syncthreads();  // stage consumed
    if (u + kStatStages < u1) issue(u + kStatStages, st);
  }
  if (ok && cur_bh >= 0) flush(cur_bh);
  if (!ok) {
    // wait (bounded) for every copy still in flight before leaving
    for (long long u = u0; u < u1 && u < u0 + kStatStages; ++u) {
      const int it = int(u - u0);
      mbar_wait(b_base + 8 * (it % kStatStages), (it / kStatStages) & 1, ws.status, false);
    }
  }
}

// ------------------------------------------------------------ kv_finalize
// grid B * Hkv, block D: the per-channel constants every K and V tile of a
// head uses, computed once: mean_k (exact fixed-point mean), mean_v, and the
// V channel scale amax/448 with its reciprocal 448/amax (IEEE fp32 division;
// amax = max |fl(v - mean_v)| taken from the channel max and min, which is
// exact because fl(v - mean) is monotone in v).
__global__ void kv_finalize_kernel(Problem pb, Workspace ws) {
  const int c = threadIdx.x;
  const long long ci = (long long)blockIdx.x * pb.D + c;
  if (c >= pb.D) return;
  const int n = nkv_of(pb, int(blockIdx.x) / pb.Hkv);
  if (n <= 0) {  // a sequence without keys: nothing reads these
    ws.mean_k[ci] = ws.mean_v[ci] = ws.v_scale[ci] = ws.v_inv[ci] = 0.f;
    return;
  }
  ws.mean_k[ci] = pb.smooth_k ? fixed_mean(ws.k_sum[ci], n) : 0.f;
  const float mv = pb.smooth_v ? fixed_mean(ws.v_sum[ci], n) : 0.f;
  ws.mean_v[ci] = mv;
  const float hi = __fsub_rn(key_float(ws.v_max[ci]), mv);
  const float lo = __fsub_rn(key_float(ws.v_min[ci]), mv);
  const float a = fmaxf(fabsf(hi), fabsf(lo));
  float sc = 0.f, inv = 0.f;
  if (a >= kTinyAmax) {
    sc = __fdiv_rn(a, 448.0f);
    inv = __fdiv_rn(448.0f, a);
  }
  ws.v_scale[ci] = sc;
  ws.v_inv[ci] = inv;
}

// Lanes per row group of quantize_kernel: a power of two >= D / 8 (16-byte
// chunks per row), so that a row group's lanes sit inside one warp and its
// reductions are warp shuffles.  With D = 96 four lanes of each group idle.
__host__ __device__ constexpr int quant_lanes(int D) { return D == 64 ? 8 : 16; }

// INT8 codes of a thread's four rows (4 rg .. +3) x eight channels (8 c8 ..
// +7), row r with reciprocal scale inv[r], straight to a [128][Dp] tile in
// global memory: the lanes of a row write its Dp bytes contiguously, lanes
// past the input's D / 8 chunks (not `live`) write the zero padding.
__device__ __forceinline__ void store_codes(uint8_t *dst, int Dp, int c8, int rg, bool live,
                                            const float (&x)[4][8], const float (&inv)[4]) {
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    uint32_t w0 = 0u, w1 = 0u;
    if (live) {
      uint32_t c[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) c[e] = __float_as_uint(__fadd_rn(__fmul_rn(x[r][e], inv[r]), 12582912.0f));
      w0 = pack4_lo(c[0], c[1], c[2], c[3]);
      w1 = pack4_lo(c[4], c[5], c[6], c[7]);
    }
    if (8 * c8 < Dp) *reinterpret_cast<uint2 *>(dst + (4 * rg + r) * Dp + 8 * c8) = make_uint2(w0, w1);
  }
}

// Integer scale and reciprocal of a block with absolute maximum a (IEEE fp32
// divisions): scale = a / qmax, inv = qmax / a (qmax = 127 for INT8 codes, 7
// for INT4); both 0 below kTinyAmax.
__device__ __forceinline__ void int_scale(float a, float qmax, float &scale, float &inv) {
  scale = 0.f;
  inv = 0.f;
  if (a >= kTinyAmax) {
    scale = __fdiv_rn(a, qmax);
    inv = __fdiv_rn(qmax, a);
  }
}

// ------------------------------------------------------------ quantize
// Persistent, grid <= 2 per SM, block 32 * L threads (L = quant_lanes(D)):
// thread t owns channels 8 * (t % L) .. +7 of the four consecutive rows
// 4 * (t / L) .. +3 of a 128-token tile.  Units: K and V tiles first, heads
// in reverse order (those kv_stats read last may still be in L2), then Q
// tiles; block i takes units i, i + grid, ...  Two input stages of 128 rows
// are kept in flight.
//   K tile: K' = K - mean_k; four INT8 blocks of 32 rows (8 row groups, a
//           whole number of warps each): block amax by warp shuffles and one
//           shared atomic per warp, one barrier.
//   Q tile: optional smoothing by the tile's channel mean; one INT8 scale per
//           row: row amax by shuffles among the row group's lanes, no barrier.
//   V tile: V' = V - mean_v, FP8 per channel, transposed through shared memory.
constexpr int kQuantStages = 2;

struct QUnit {
  int kind;  // 0 = K tile, 1 = V tile, 2 = Q tile
  int bh, t, b, h, r0, nvalid;
  const uint16_t *src;
  long long stride;
};

// Units of quantize_kernel: K and V tiles (both), then Q tiles; variable-length
// batches count only the tiles inside a sequence.
__host__ __device__ __forceinline__ long long quant_units(const Problem &pb, const Workspace &ws) {
  const long long nKV = pb.cu_kv ? (long long)pb.Hkv * pb.tot_kv128
                                 : (long long)pb.B * pb.Hkv * (ws.Nkv_pad / kKVTile);
  const long long nQ = pb.cu_q ? (long long)pb.Hq * pb.tot_q128 : (long long)pb.B * pb.Hq * ws.nqb;
  return 2 * nKV + nQ;
}

// kVarlen: the unit numbering of a variable-length batch (only the tiles inside
// a sequence); a template parameter so that the batched kernel, whose thread 0
// decodes a unit on the path to every unit's barrier, carries none of it.
// (out of line: the variable-length search would otherwise cost the unit loop
// registers)
__device__ __noinline__ int2 seq_unit_ht(const int *pc, int B, int heads, long long x) {
  int b, h, t;
  seq_unit(pc, B, heads, x, b, h, t);
  return make_int2(b * heads + h, t);
}

template <bool kVarlen>
__device__ __forceinline__ QUnit quant_unit(const Problem &pb, const Workspace &ws, long long u) {
  QUnit q{};
  const int nKt = ws.Nkv_pad / kKVTile;
  const long long nKV = kVarlen ? (long long)pb.Hkv * pb.tot_kv128 : (long long)pb.B * pb.Hkv * nKt;
  if (u < 2 * nKV) {
    q.kind = int(u & 1);
    const int kvi = int(nKV - 1 - (u >> 1));  // reverse head order (counts < 2^31)
    if (kVarlen) {
      const int2 bt = seq_unit_ht(pb.pc_kv128, pb.B, pb.Hkv, kvi);
      q.bh = bt.x;
      q.t = bt.y;
    } else {
      q.t = kvi % nKt;
      q.bh = kvi / nKt;
    }
    q.b = q.bh / pb.Hkv;
    q.h = q.bh % pb.Hkv;
    q.r0 = q.t * kKVTile;
    q.nvalid = max(0, min(kKVTile, nkv_of(pb, q.b) - q.r0));
    if (q.kind == 0) {
      q.src = pb.k + k_off(pb, q.b) + q.h * pb.ks_h + q.r0 * pb.ks_n;
      q.stride = pb.ks_n;
    } else {
      q.src = pb.v + v_off(pb, q.b) + q.h * pb.vs_h + q.r0 * pb.vs_n;
      q.stride = pb.vs_n;
    }
  } else {
    const int qi = int(u - 2 * nKV);
    q.kind = 2;
    if (kVarlen) {
      const int2 bt = seq_unit_ht(pb.pc_q128, pb.B, pb.Hq, qi);
      q.bh = bt.x;
      q.t = bt.y;
    } else {
      q.t = qi % ws.nqb;
      q.bh = qi / ws.nqb;
    }
    q.b = q.bh / pb.Hq;
    q.h = q.bh % pb.Hq;
    q.r0 = q.t * kQTile;
    q.nvalid = max(0, min(kQTile, nq_of(pb, q.b) - q.r0));
    q.src = pb.q + q_off(pb, q.b) + q.h * pb.qs_h + q.r0 * pb.qs_n;
    q.stride = pb.qs_n;
  }
  return q;
}

// kMaps: some input is read through a tensor map (a template parameter, so
// that the kernel for dense inputs carries none of it).
template <bool kVarlen, bool kMaps>
__global__ void __launch_bounds__(512, 2) quantize_kernel(Problem pb, Workspace ws,
                                                          const __grid_constant__ CUtensorMap mk,
                                                          const __grid_constant__ CUtensorMap mv,
                                                          const __grid_constant__ CUtensorMap mq) {
  extern __shared__ __align__(1024) uint8_t sm_q[];
  if (smem_misaligned(sm_q, ws.status)) return;
  const int D = pb.D, Dp = ws.Dp, C8 = D / 8, L = quant_lanes(D), rowb = 2 * D;
  const int c8 = threadIdx.x % L, rg = threadIdx.x / L;  // rows 4 rg .. 4 rg + 3
  const bool live = c8 < C8;                              // lane holds input channels
  const int stage_bytes = 128 * rowb;
  uint8_t *tile = sm_q + kQuantStages * stage_bytes;        // output codes [128][128]
  uint64_t *bars = reinterpret_cast<uint64_t *>(tile + 128 * 128);
  unsigned long long *colsum = reinterpret_cast<unsigned long long *>(bars + 4);
  float *chan = reinterpret_cast<float *>(colsum + 128);
  unsigned *mslot = reinterpret_cast<unsigned *>(chan + 128);  // [2 parities][4 K blocks]
  QUnit *desc = reinterpret_cast<QUnit *>(mslot + 8);        // [stages + 1]
  const uint32_t s_base = smem_u32(sm_q), b_base = smem_u32(bars);
  // K and V tiles, then Q tiles (skipped when the attention kernel quantises Q)
  const long long nunits = quant_units(pb, ws);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kQuantStages; ++i) mbar_init(b_base + 8 * i, 1);
    fence_mbar_init();
    for (int i = 0; i < 8; ++i) mslot[i] = 0u;
  }
  __syncthreads();
  // Unit descriptors are decoded once, by thread 0, into a ring of
  // kQuantStages + 1 shared slots: iteration it reads slot it % (S + 1) and
  // thread 0 fills slot (it + S) % (S + 1) -- the slot of iteration it - 1,
  // which every thread has finished reading by this iteration's first
  // barrier.
  constexpr int kSlots = kQuantStages + 1;
  auto issue = [&](const QUnit &q, int st) {
    if constexpr (kMaps) {
      const int use_map = q.kind == 0 ? pb.k_map : q.kind == 1 ? pb.v_map : pb.q_map;
      if (use_map) {
        // one box of 128 tokens (rows past nvalid are loaded but never used)
        if (threadIdx.x == 0)
          map_issue(s_base + st * stage_bytes, q.kind == 0 ? &mk : q.kind == 1 ? &mv : &mq,
                    b_base + 8 * st, uint32_t(stage_bytes),
                    q.kind == 0 ? pb.k_hn : q.kind == 1 ? pb.v_hn : pb.q_hn,
                    q.kind == 2 ? pb.cu_q : pb.cu_kv, q.b, q.h, q.r0);
        return;
      }
    }
    issue_rows(s_base + st * stage_bytes, q.src, q.stride, q.nvalid, rowb, b_base + 8 * st, true,
               uint32_t(q.nvalid) * rowb);
  };
  if (threadIdx.x == 0)
    for (int i = 0; i < kQuantStages; ++i)
      if (blockIdx.x + (long long)i * gridDim.x < nunits)
        desc[i] = quant_unit<kVarlen>(pb, ws, blockIdx.x + (long long)i * gridDim.x);
  static_assert(kQuantStages + 1 == kSlots, "descriptor ring");
  __syncthreads();
  for (int i = 0; i < kQuantStages; ++i)
    if (blockIdx.x + (long long)i * gridDim.x < nunits) issue(desc[i], i);

  float x[4][8];
  int it = 0;
  bool ok = true;
  for (long long u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
    const int st = it % kQuantStages;
    if (!block_wait(b_base + 8 * st, (it / kQuantStages) & 1, ws.status)) { ok = false; break; }
    const QUnit q = desc[it % kSlots];
    // K-block max slots: this unit uses parity it & 1; the other parity (last
    // read in iteration it - 1) is cleared for the next unit
    unsigned *mx = mslot + 4 * (it & 1);
    if (threadIdx.x < 4) mslot[4 * ((it + 1) & 1) + threadIdx.x] = 0u;
    const uint8_t *stage = sm_q + st * stage_bytes;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = 4 * rg + r;
      if (live && row < q.nvalid) decode8(*reinterpret_cast<const uint4 *>(stage + row * rowb + 16 * c8), pb.bf16, x[r]);
      else
#pragma unroll
        for (int e = 0; e < 8; ++e) x[r][e] = 0.f;
    }
    const long long un = u + (long long)kQuantStages * gridDim.x;
    QUnit *dn = desc + (it + kQuantStages) % kSlots;
    if (threadIdx.x == 0 && un < nunits) *dn = quant_unit<kVarlen>(pb, ws, un);
    __syncthreads();  // stage consumed; next descriptor visible
    if (un < nunits) issue(*dn, st);

    if (q.kind == 0) {
      // ---------------- K tile: K' = K - mean_k, four INT8 blocks of 32 rows
      float mean[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (live) {
        const float4 *mk4 = reinterpret_cast<const float4 *>(ws.mean_k + (long long)q.bh * D + 8 * c8);
        const float4 m0 = __ldg(mk4), m1 = __ldg(mk4 + 1);
        mean[0] = m0.x; mean[1] = m0.y; mean[2] = m0.z; mean[3] = m0.w;
        mean[4] = m1.x; mean[5] = m1.y; mean[6] = m1.z; mean[7] = m1.w;
      }
      float a = 0.f;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (live && 4 * rg + r < q.nvalid)
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const float2 d = __fadd2_rn(make_float2(x[r][e], x[r][e + 1]), make_float2(-mean[e], -mean[e + 1]));
            x[r][e] = d.x;
            x[r][e + 1] = d.y;
            a = fmaxf(a, fmaxf(fabsf(d.x), fabsf(d.y)));
          }
      // rows 32 k .. 32 k + 31 (row groups 8 k .. 8 k + 7) form block k; each
      // warp lies inside one block.  Non-negative floats order like their bits.
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      if ((threadIdx.x & 31) == 0) atomicMax(mx + rg / 8, __float_as_uint(a));
      __syncthreads();
      float inv[4], sc;
      int_scale(__uint_as_float(mx[rg / 8]), pb.qmax, sc, inv[0]);
      inv[1] = inv[2] = inv[3] = inv[0];
      if (threadIdx.x < 4) {
        float s4, i4;
        int_scale(__uint_as_float(mx[threadIdx.x]), pb.qmax, s4, i4);
        ws.k_scale[(long long)q.bh * (ws.Nkv_pad / kKBlk) + 4 * q.t + threadIdx.x] = s4;
      }
      store_codes(reinterpret_cast<uint8_t *>(ws.k8) + ((long long)q.bh * ws.Nkv_pad + q.r0) * Dp, Dp,
                  c8, rg, live, x, inv);
    } else if (q.kind == 1) {
      // ---------------- V tile: V' = V - mean_v, FP8 per channel, transposed
      float mean[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, inv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (live) {
        const float4 *mv4 = reinterpret_cast<const float4 *>(ws.mean_v + (long long)q.bh * D + 8 * c8);
        const float4 *iv4 = reinterpret_cast<const float4 *>(ws.v_inv + (long long)q.bh * D + 8 * c8);
        const float4 m0 = __ldg(mv4), m1 = __ldg(mv4 + 1), i0 = __ldg(iv4), i1 = __ldg(iv4 + 1);
        mean[0] = m0.x; mean[1] = m0.y; mean[2] = m0.z; mean[3] = m0.w;
        mean[4] = m1.x; mean[5] = m1.y; mean[6] = m1.z; mean[7] = m1.w;
        inv[0] = i0.x; inv[1] = i0.y; inv[2] = i0.z; inv[3] = i0.w;
        inv[4] = i1.x; inv[5] = i1.y; inv[6] = i1.z; inv[7] = i1.w;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (4 * rg + r < q.nvalid) {
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const float2 d = __fmul2_rn(__fadd2_rn(make_float2(x[r][e], x[r][e + 1]), make_float2(-mean[e], -mean[e + 1])),
                                     make_float2(inv[e], inv[e + 1]));
            x[r][e] = d.x;
            x[r][e + 1] = d.y;
          }
        }
      }
      // Transposed tile [D][128 keys] as 32 words per channel row; the word of
      // keys 4 rg .. 4 rg + 3 of channel c sits at position (rg + rot * c8) % 32,
      // which puts the 32 lanes of a warp on 32 different banks.
      const int rot = 32 / L;
      uint32_t *tw = reinterpret_cast<uint32_t *>(tile);
      if (live) {
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          uint32_t w_lo = 0, w_hi = 0;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint32_t pr = e4m3x2(x[r][e], x[r][e + 1]);
            w_lo |= (pr & 0xFFu) << (8 * r);
            w_hi |= (pr >> 8) << (8 * r);
          }
          const int pos = (rg + rot * c8) & 31;
          tw[(8 * c8 + e) * 32 + pos] = w_lo;
          tw[(8 * c8 + e + 1) * 32 + pos] = w_hi;
        }
      }
      __syncthreads();
      uint8_t *dst = ws.v8t + (long long)q.bh * D * ws.Nkv_pad + q.r0;
      for (int t = threadIdx.x; t < D * 8; t += blockDim.x) {
        const int c = t >> 3, qq = t & 7;  // channel row c, keys 16 qq .. 16 qq + 15
        const int sh = rot * (c >> 3);
        uint4 o;
        o.x = tw[c * 32 + ((4 * qq + 0 + sh) & 31)];
        o.y = tw[c * 32 + ((4 * qq + 1 + sh) & 31)];
        o.z = tw[c * 32 + ((4 * qq + 2 + sh) & 31)];
        o.w = tw[c * 32 + ((4 * qq + 3 + sh) & 31)];
        *reinterpret_cast<uint4 *>(dst + (long long)c * ws.Nkv_pad + 16 * qq) = o;
      }
    } else {
      // ---------------- Q tile: optional smoothing mean, one INT8 scale per row
      if (pb.smooth_q) {
        if (int(threadIdx.x) < D) colsum[threadIdx.x] = 0ull;
        __syncthreads();
        if (live) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            long long s = 0;
#pragma unroll
            for (int r = 0; r < 4; ++r)
              if (4 * rg + r < q.nvalid) s += fixed_point(x[r][e]);
            atomicAdd(&colsum[8 * c8 + e], (unsigned long long)s);
          }
        }
        __syncthreads();
        if (int(threadIdx.x) < D) {
          const float m = q.nvalid > 0 ? fixed_mean((long long)colsum[threadIdx.x], q.nvalid) : 0.f;
          chan[threadIdx.x] = m;
          ws.mq[((long long)q.bh * ws.nqb + q.t) * D + threadIdx.x] = m;
        }
        __syncthreads();
        if (live) {
#pragma unroll
          for (int r = 0; r < 4; ++r)
            if (4 * rg + r < q.nvalid)
#pragma unroll
              for (int e = 0; e < 8; e += 2) {
                const float2 d = __fadd2_rn(make_float2(x[r][e], x[r][e + 1]),
                                            make_float2(-chan[8 * c8 + e], -chan[8 * c8 + e + 1]));
                x[r][e] = d.x;
                x[r][e + 1] = d.y;
              }
        }
      }
      float a[4], inv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        a[r] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a[r] = fmaxf(a[r], fabsf(x[r][e]));
      }
      // row amax over the row group's L lanes (aligned inside the warp)
#pragma unroll
      for (int o = L / 2; o > 0; o >>= 1)
#pragma unroll
        for (int r = 0; r < 4; ++r) a[r] = fmaxf(a[r], __shfl_xor_sync(0xffffffffu, a[r], o));
      // lane c8 < 4 of the group divides for row 4 rg + c8 (IEEE divisions)
      // and stores its scale (0 past nvalid); the group's lanes take the four
      // reciprocals by shuffles
      float s_own, i_own;
      int_scale(c8 == 0 ? a[0] : c8 == 1 ? a[1] : c8 == 2 ? a[2] : a[3], pb.qmax, s_own, i_own);
      const int gbase = int(threadIdx.x & 31) & ~(L - 1);
#pragma unroll
      for (int r = 0; r < 4; ++r) inv[r] = __shfl_sync(0xffffffffu, i_own, gbase + r);
      if (c8 < 4) ws.q_scale[(long long)q.bh * ws.Nq_pad + q.r0 + 4 * rg + c8] = s_own;
      store_codes(reinterpret_cast<uint8_t *>(ws.q8) + ((long long)q.bh * ws.Nq_pad + q.r0) * Dp, Dp,
                  c8, rg, live, x, inv);
    }
    // The V transpose tile is rewritten only after the next unit's first
    // barrier, which every thread reaches after its reads of this one.
  }
  if (!ok) {
    // wait (bounded) for copies still in flight before leaving
    for (int i = 0; i < kQuantStages; ++i) {
      const long long u = blockIdx.x + (long long)(it + i) * gridDim.x;
      if (u < nunits) mbar_wait(b_base + 8 * ((it + i) % kQuantStages), ((it + i) / kQuantStages) & 1, ws.status, false);
    }
  }
}

// ------------------------------------------------------------ delta_s
// grid (Nkv_pad / 128, B * Hq), block 128: thread t owns key 128*kt + t.
// dsk[b,h][blk][j] = fp32(dS * K2), dS = sum_c mq[blk][c] * K'[j][c] (fp32 FMA).
constexpr int kDsChunk = 16;  // q blocks per shared-memory chunk of mq
__global__ void __launch_bounds__(128) delta_s_kernel(Problem pb, Workspace ws) {
  extern __shared__ float sm[];
  float *kpt = sm;                  // [D][128]  K' transposed
  float *mqs = sm + pb.D * 128;     // [kDsChunk][D]
  const int D = pb.D;
  const int kt = blockIdx.x, bh = blockIdx.y, b = bh / pb.Hq, h = bh % pb.Hq;
  const int hk = h / (pb.Hq / pb.Hkv), bhk = b * pb.Hkv + hk;
  const int t = threadIdx.x;
  // stage K' (recomputed from K and mean_k) for this 128-key tile
  for (int o = t; o < 128 * (D / 8); o += 128) {
    const int r = o / (D / 8), c8 = o % (D / 8), j = kt * 128 + r;
    float xv[8];
    if (j < nkv_of(pb, b)) {
      load8(pb.k + k_off(pb, b) + hk * pb.ks_h + (long long)j * pb.ks_n + 8 * c8, pb.bf16, xv);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        xv[e] = __fsub_rn(xv[e], ws.mean_k[(long long)bhk * D + 8 * c8 + e]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) xv[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) kpt[(8 * c8 + e) * 128 + r] = xv[e];
  }
  for (int q0 = 0; q0 < ws.nqb; q0 += kDsChunk) {
    const int nb = min(kDsChunk, ws.nqb - q0);
    __syncthreads();
    for (int o = t; o < nb * D; o += 128)
      mqs[o] = ws.mq[((long long)bh * ws.nqb + q0) * D + o];
    __syncthreads();
    for (int qb = 0; qb < nb; ++qb) {
      float acc = 0.f;
      for (int c = 0; c < D; ++c) acc = __fmaf_rn(mqs[qb * D + c], kpt[c * 128 + t], acc);
      ws.dsk[((long long)bh * ws.nqb + q0 + qb) * ws.Nkv_pad + kt * 128 + t] =
          __fmul_rn(acc, pb.K2);
    }
  }
}

}  // namespace

cudaError_t launch_prepass(const Problem &pb, const Workspace &ws, const InputMaps &im,
                           cudaStream_t stream) {
  const long long nch = (long long)pb.B * pb.Hkv * pb.D;
  // sums (int64) and max keys start at zero; min keys at all-ones
  cudaError_t e = cudaMemsetAsync(ws.k_sum, 0, nch * (2 * sizeof(long long) + sizeof(unsigned)),
                                  stream);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(ws.v_min, 0xFF, nch * sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // kv_stats: persistent, 2 blocks per SM
  const int rowb = 2 * pb.D;
  const int ngroups = 256 / (pb.D / 8);
  const size_t st_smem = kStatStages * 2 * kStatChunk * rowb + 64 + sizeof(long long) * ngroups * pb.D;
  e = cudaFuncSetAttribute(kv_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)st_smem);
  if (e != cudaSuccess) return e;
  const long long nchunk = (pb.Nkv + kStatChunk - 1) / kStatChunk;
  const long long su = pb.cu_kv ? (long long)pb.Hkv * pb.tot_kv64 : (long long)pb.B * pb.Hkv * nchunk;
  const unsigned g1 = (unsigned)std::min<long long>(su, 2LL * sms);
  if (g1 > 0) {  // (a variable-length batch may hold no keys at all)
    kv_stats_kernel<<<g1, 256, st_smem, stream>>>(pb, ws, im.k64, im.v64);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  kv_finalize_kernel<<<pb.B * pb.Hkv, 128, 0, stream>>>(pb, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // quantize: persistent, 2 blocks per SM
  // stages | output tile | 4 barriers | colsum[128] | chan[128] | K-block max slots[8] | desc[stages + 1]
  const size_t q_smem = kQuantStages * 128 * rowb + 128 * 128 + 32 + 128 * 8 + 128 * 4 + 8 * 4 +
                        (kQuantStages + 1) * sizeof(QUnit);
  const bool maps = pb.k_map || pb.v_map || pb.q_map;
  auto qk = pb.cu_q ? (maps ? quantize_kernel<true, true> : quantize_kernel<true, false>)
                    : (maps ? quantize_kernel<false, true> : quantize_kernel<false, false>);
  e = cudaFuncSetAttribute(qk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)q_smem);
  if (e != cudaSuccess) return e;
  const long long nblk = quant_units(pb, ws);
  const unsigned g2 = (unsigned)std::min<long long>(nblk, 2LL * sms);
  if (g2 > 0) {
    qk<<<g2, 32 * quant_lanes(pb.D), q_smem, stream>>>(pb, ws, im.k128, im.v128, im.q128);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (pb.smooth_q) {
    const size_t smem = sizeof(float) * (pb.D * 128 + kDsChunk * pb.D);
    e = cudaFuncSetAttribute(delta_s_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(sizeof(float) * (128 * 128 + kDsChunk * 128)));
    if (e != cudaSuccess) return e;
    delta_s_kernel<<<dim3(ws.Nkv_pad / 128, pb.B * pb.Hq), 128, smem, stream>>>(pb, ws);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace sage
