// prepass.cu -- smoothing + quantisation pre-pass (HBM-bandwidth bound).
//
// Follows the SageAttention pages: K is smoothed by subtracting its
// per-channel mean over all tokens ("sageattention" package page,
// Quickstart: smooth_k), Q and V may be smoothed by subtracting channel means
// ("SageAttention2: Technical report", section 2), Q and K are quantised per
// block to INT8 and V to FP8 (closerAI ComfyUI blog, part 2).
//
// Three kernels on one stream:
//   kv_stats   per (b, kv head, 256-token chunk): fixed-point channel sums of
//              K (and V) and the V channel max/min, combined with atomics
//              (integer addition is exact, so the order does not matter);
//   quantize   per 128-token tile of K, V or Q (in that order, K/V heads in
//              reverse so their second read hits L2): smoothing, block amax,
//              INT8/FP8 codes written through shared memory as whole
//              coalesced tiles in the attention kernel's layout (V
//              transposed so that keys are contiguous);
//   delta_s    (smooth_q only) the correction dS[blk][j] = mq[blk] . K'_j,
//              stored pre-multiplied by sm_scale * log2(e).
//
// Threads own 16-byte chunks (8 channels) of rows, so loads are 16-byte
// vectors and a warp covers whole rows.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace sage {
namespace {

constexpr int kRowsPerPass = 16;   // rows handled concurrently by one CTA
constexpr int kStatTokens = 256;   // tokens per kv_stats CTA
constexpr float kTinyAmax = 0x1p-64f;  // blocks below this quantise to zero

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

// ------------------------------------------------------------ kv_stats
// grid (ceil(Nkv / 256), B * Hkv), block 16 * (D / 8).  Each thread owns one
// 16-byte chunk (8 channels) and walks rows 16 apart, two rows per step so
// that four 16-byte loads are in flight before any arithmetic.
__global__ void __launch_bounds__(256, 2) kv_stats_kernel(Problem pb, Workspace ws) {
  const int C8 = pb.D / 8;
  const int c8 = threadIdx.x % C8, r0 = threadIdx.x / C8;
  const int bh = blockIdx.y, b = bh / pb.Hkv, h = bh % pb.Hkv;
  const int j0 = blockIdx.x * kStatTokens;
  const uint16_t *kb = pb.k + b * pb.ks_b + h * pb.ks_h + 8 * c8;
  const uint16_t *vb = pb.v + b * pb.vs_b + h * pb.vs_h + 8 * c8;

  long long ksum[8], vsum[8];
  float vmax[8], vmin[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    ksum[e] = 0;
    vsum[e] = 0;
    vmax[e] = -INFINITY;
    vmin[e] = INFINITY;
  }
  for (int rr = r0; rr < kStatTokens; rr += 2 * kRowsPerPass) {
    float xk[2][8], xv[2][8];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int j = j0 + rr + u * kRowsPerPass;
      if (j < pb.Nkv) {
        if (pb.smooth_k) load8(kb + j * pb.ks_n, pb.bf16, xk[u]);
        load8(vb + j * pb.vs_n, pb.bf16, xv[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int j = j0 + rr + u * kRowsPerPass;
      if (j < pb.Nkv) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (pb.smooth_k) ksum[e] += fixed_point(xk[u][e]);
          vmax[e] = fmaxf(vmax[e], xv[u][e]);
          vmin[e] = fminf(vmin[e], xv[u][e]);
          if (pb.smooth_v) vsum[e] += fixed_point(xv[u][e]);
        }
      }
    }
  }

  // Combine the 16 row groups per channel through shared memory.
  __shared__ long long red[kRowsPerPass][128];
  const int D = pb.D;
  const int tid = threadIdx.x;
  long long *ks_out = ws.k_sum + (long long)bh * D;
  long long *vs_out = ws.v_sum + (long long)bh * D;
  if (pb.smooth_k) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r0][8 * c8 + e] = ksum[e];
    __syncthreads();
    if (tid < D) {
      long long s = 0;
      for (int r = 0; r < kRowsPerPass; ++r) s += red[r][tid];
      atomicAdd(reinterpret_cast<unsigned long long *>(ks_out + tid), (unsigned long long)s);
    }
    __syncthreads();
  }
  if (pb.smooth_v) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r0][8 * c8 + e] = vsum[e];
    __syncthreads();
    if (tid < D) {
      long long s = 0;
      for (int r = 0; r < kRowsPerPass; ++r) s += red[r][tid];
      atomicAdd(reinterpret_cast<unsigned long long *>(vs_out + tid), (unsigned long long)s);
    }
    __syncthreads();
  }
  float *redf = reinterpret_cast<float *>(&red[0][0]);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    redf[r0 * 128 + 8 * c8 + e] = vmax[e];
    redf[kRowsPerPass * 128 + r0 * 128 + 8 * c8 + e] = vmin[e];
  }
  __syncthreads();
  if (tid < D) {
    float mx = -INFINITY, mn = INFINITY;
    for (int r = 0; r < kRowsPerPass; ++r) {
      mx = fmaxf(mx, redf[r * 128 + tid]);
      mn = fminf(mn, redf[kRowsPerPass * 128 + r * 128 + tid]);
    }
    atomicMax(ws.v_max + (long long)bh * D + tid, float_key(mx));
    atomicMin(ws.v_min + (long long)bh * D + tid, float_key(mn));
  }
}

// Block-wide max of two values (one per K half, or the same value twice);
// up to 32 warps.
__device__ __forceinline__ void block_max2(float &a, float &b, float *scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, o));
  }
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
  __syncthreads();
  if (lane == 0) {
    scratch[warp] = a;
    scratch[32 + warp] = b;
  }
  __syncthreads();
  a = scratch[0];
  b = scratch[32];
  for (int w = 1; w < nw; ++w) {
    a = fmaxf(a, scratch[w]);
    b = fmaxf(b, scratch[32 + w]);
  }
}

__device__ __forceinline__ uint32_t int8_code(float x, float inv) {
  int q = __float2int_rn(__fmul_rn(x, inv));
  q = q > 127 ? 127 : (q < -127 ? -127 : q);
  return uint32_t(q) & 0xFFu;
}

// Copy a finished [rows][row_bytes] tile from shared memory to a contiguous
// global destination with 16-byte stores.
__device__ __forceinline__ void store_tile(uint8_t *dst, const uint8_t *src, int bytes) {
  for (int o = 16 * threadIdx.x; o < bytes; o += 16 * blockDim.x)
    *reinterpret_cast<uint4 *>(dst + o) = *reinterpret_cast<const uint4 *>(src + o);
}

// ------------------------------------------------------------ quantize
// grid (nK + nV + nQ), block 32 * (D / 8): thread t owns channels
// 8 * (t % (D/8)) .. +7 of the four consecutive rows 4 * (t / (D/8)) .. +3 of
// one 128-token tile.  Block order: K and V tiles first, heads in reverse
// order (those kv_stats read last are still in L2), then Q blocks.
__global__ void __launch_bounds__(512, 2) quantize_kernel(Problem pb, Workspace ws) {
  __shared__ __align__(16) uint8_t tile[128 * 128];
  __shared__ unsigned long long colsum[128];
  __shared__ float chan[128];
  __shared__ float scratch[64];

  const int D = pb.D, Dp = ws.Dp, C8 = D / 8;
  const int c8 = threadIdx.x % C8, rg = threadIdx.x / C8;  // rows 4 rg .. 4 rg + 3
  const int nKt = ws.Nkv_pad / kKVTile;
  const int nKV = pb.B * pb.Hkv * nKt;
  int blk = blockIdx.x;
  float x[4][8];

  if (blk < 2 * nKV) {
    const int isV = blk & 1;
    const int kvi = nKV - 1 - (blk >> 1);  // reverse head order
    const int kt = kvi % nKt, bh = kvi / nKt, b = bh / pb.Hkv, h = bh % pb.Hkv;
    const int j0 = kt * kKVTile, nvalid = max(0, min(kKVTile, pb.Nkv - j0));
    if (!isV) {
      // ---------------- K tile: K' = K - mean_k, two INT8 blocks of 64
      const uint16_t *src = pb.k + b * pb.ks_b + h * pb.ks_h + 8 * c8;
      float mean[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        mean[e] = pb.smooth_k ? fixed_mean(ws.k_sum[(long long)bh * D + 8 * c8 + e], pb.Nkv) : 0.f;
      if (kt == 0 && rg == 0)
#pragma unroll
        for (int e = 0; e < 8; ++e) ws.mean_k[(long long)bh * D + 8 * c8 + e] = mean[e];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = 4 * rg + u;
        if (r < nvalid) load8(src + (long long)(j0 + r) * pb.ks_n, pb.bf16, x[u]);
      }
      float a = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (4 * rg + u < nvalid) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x[u][e] = __fsub_rn(x[u][e], mean[e]);
            a = fmaxf(a, fabsf(x[u][e]));
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) x[u][e] = 0.f;
        }
      }
      // rows 0..63 belong to block 2 kt, rows 64..127 to 2 kt + 1
      float a0 = rg < 16 ? a : 0.f, a1 = rg < 16 ? 0.f : a;
      block_max2(a0, a1, scratch);
      float inv0 = 0.f, inv1 = 0.f, s0 = 0.f, s1 = 0.f;
      if (a0 >= kTinyAmax) {
        s0 = __fdiv_rn(a0, 127.0f);
        inv0 = __fdiv_rn(127.0f, a0);
      }
      if (a1 >= kTinyAmax) {
        s1 = __fdiv_rn(a1, 127.0f);
        inv1 = __fdiv_rn(127.0f, a1);
      }
      if (threadIdx.x == 0) {
        ws.k_scale[(long long)bh * (ws.Nkv_pad / kKBlk) + 2 * kt] = s0;
        ws.k_scale[(long long)bh * (ws.Nkv_pad / kKBlk) + 2 * kt + 1] = s1;
      }
      const float inv = rg < 16 ? inv0 : inv1;
      if (Dp != D)
        for (int o = 4 * threadIdx.x; o < 128 * Dp; o += 4 * blockDim.x)
          *reinterpret_cast<uint32_t *>(tile + o) = 0u;
      __syncthreads();
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t w0 = 0, w1 = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          w0 |= int8_code(x[u][e], inv) << (8 * e);
          w1 |= int8_code(x[u][e + 4], inv) << (8 * e);
        }
        *reinterpret_cast<uint2 *>(tile + (4 * rg + u) * Dp + 8 * c8) = make_uint2(w0, w1);
      }
      __syncthreads();
      store_tile(reinterpret_cast<uint8_t *>(ws.k8) + ((long long)bh * ws.Nkv_pad + j0) * Dp, tile,
                 128 * Dp);
      return;
    }
    // ---------------- V tile: V' = V - mean_v, FP8 per channel, transposed
    const uint16_t *src = pb.v + b * pb.vs_b + h * pb.vs_h + 8 * c8;
    float mean[8], inv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const long long ci = (long long)bh * D + 8 * c8 + e;
      mean[e] = pb.smooth_v ? fixed_mean(ws.v_sum[ci], pb.Nkv) : 0.f;
      const float hi = __fsub_rn(key_float(ws.v_max[ci]), mean[e]);
      const float lo = __fsub_rn(key_float(ws.v_min[ci]), mean[e]);
      const float a = fmaxf(fabsf(hi), fabsf(lo));
      float sc = 0.f;
      inv[e] = 0.f;
      if (a >= kTinyAmax) {
        sc = __fdiv_rn(a, 448.0f);
        inv[e] = __fdiv_rn(448.0f, a);
      }
      if (kt == 0 && rg == 0) {
        ws.v_scale[ci] = sc;
        ws.mean_v[ci] = mean[e];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = 4 * rg + u;
      if (r < nvalid) {
        load8(src + (long long)(j0 + r) * pb.vs_n, pb.bf16, x[u]);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[u][e] = __fmul_rn(__fsub_rn(x[u][e], mean[e]), inv[e]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[u][e] = 0.f;
      }
    }
    // Transposed tile [D][128 keys] as 32 words per channel row; the word of
    // keys 4 rg .. 4 rg + 3 of channel c sits at position (rg + rot * c8) % 32,
    // which puts the 32 lanes of a warp on 32 different banks.
    const int rot = 32 / (C8 == 12 ? 16 : C8);
    uint32_t *tw = reinterpret_cast<uint32_t *>(tile);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      uint32_t w_lo = 0, w_hi = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t pr = e4m3x2(x[u][e], x[u][e + 1]);
        w_lo |= (pr & 0xFFu) << (8 * u);
        w_hi |= (pr >> 8) << (8 * u);
      }
      const int pos = (rg + rot * c8) & 31;
      tw[(8 * c8 + e) * 32 + pos] = w_lo;
      tw[(8 * c8 + e + 1) * 32 + pos] = w_hi;
    }
    __syncthreads();
    uint8_t *dst = ws.v8t + (long long)bh * D * ws.Nkv_pad + j0;
    for (int t = threadIdx.x; t < D * 8; t += blockDim.x) {
      const int c = t >> 3, q = t & 7;  // channel row c, keys 16 q .. 16 q + 15
      const int sh = rot * (c >> 3);
      uint4 o;
      o.x = tw[c * 32 + ((4 * q + 0 + sh) & 31)];
      o.y = tw[c * 32 + ((4 * q + 1 + sh) & 31)];
      o.z = tw[c * 32 + ((4 * q + 2 + sh) & 31)];
      o.w = tw[c * 32 + ((4 * q + 3 + sh) & 31)];
      *reinterpret_cast<uint4 *>(dst + (long long)c * ws.Nkv_pad + 16 * q) = o;
    }
    return;
  }
  blk -= 2 * nKV;
  {
    // ---------------- Q block: optional block mean, INT8 per block
    const int qb = blk % ws.nqb, bh = blk / ws.nqb, b = bh / pb.Hq, h = bh % pb.Hq;
    const int i0 = qb * kQBlk, nvalid = min(kQBlk, pb.Nq - i0);
    const uint16_t *src = pb.q + b * pb.qs_b + h * pb.qs_h + 8 * c8;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = 4 * rg + u;
      if (r < nvalid) load8(src + (long long)(i0 + r) * pb.qs_n, pb.bf16, x[u]);
      else
#pragma unroll
        for (int e = 0; e < 8; ++e) x[u][e] = 0.f;
    }
    if (pb.smooth_q) {
      if (threadIdx.x < D) colsum[threadIdx.x] = 0ull;
      __syncthreads();
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        long long s = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (4 * rg + u < nvalid) s += fixed_point(x[u][e]);
        atomicAdd(&colsum[8 * c8 + e], (unsigned long long)s);
      }
      __syncthreads();
      if (threadIdx.x < D) {
        const float m = fixed_mean((long long)colsum[threadIdx.x], nvalid);
        chan[threadIdx.x] = m;
        ws.mq[((long long)bh * ws.nqb + qb) * D + threadIdx.x] = m;
      }
      __syncthreads();
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (4 * rg + u < nvalid)
#pragma unroll
          for (int e = 0; e < 8; ++e) x[u][e] = __fsub_rn(x[u][e], chan[8 * c8 + e]);
    }
    float a = 0.f, unused = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(x[u][e]));
    block_max2(a, unused, scratch);
    float inv = 0.f, scale = 0.f;
    if (a >= kTinyAmax) {
      scale = __fdiv_rn(a, 127.0f);
      inv = __fdiv_rn(127.0f, a);
    }
    if (threadIdx.x == 0) ws.q_scale[(long long)bh * ws.nqb + qb] = scale;
    if (Dp != D)
      for (int o = 4 * threadIdx.x; o < 128 * Dp; o += 4 * blockDim.x)
        *reinterpret_cast<uint32_t *>(tile + o) = 0u;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t w0 = 0, w1 = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w0 |= int8_code(x[u][e], inv) << (8 * e);
        w1 |= int8_code(x[u][e + 4], inv) << (8 * e);
      }
      *reinterpret_cast<uint2 *>(tile + (4 * rg + u) * Dp + 8 * c8) = make_uint2(w0, w1);
    }
    __syncthreads();
    store_tile(reinterpret_cast<uint8_t *>(ws.q8) + ((long long)bh * ws.Nq_pad + i0) * Dp, tile,
               128 * Dp);
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
    if (j < pb.Nkv) {
      load8(pb.k + b * pb.ks_b + hk * pb.ks_h + (long long)j * pb.ks_n + 8 * c8, pb.bf16, xv);
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

cudaError_t launch_prepass(const Problem &pb, const Workspace &ws, cudaStream_t stream) {
  const long long nch = (long long)pb.B * pb.Hkv * pb.D;
  // sums (int64) and max keys start at zero; min keys at all-ones
  cudaError_t e = cudaMemsetAsync(ws.k_sum, 0, nch * (2 * sizeof(long long) + sizeof(unsigned)),
                                  stream);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(ws.v_min, 0xFF, nch * sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  dim3 g1((pb.Nkv + kStatTokens - 1) / kStatTokens, pb.B * pb.Hkv);
  kv_stats_kernel<<<g1, 16 * (pb.D / 8), 0, stream>>>(pb, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nKt = ws.Nkv_pad / kKVTile;
  const long long nblk = (long long)pb.B * pb.Hq * ws.nqb + 2LL * pb.B * pb.Hkv * nKt;
  quantize_kernel<<<dim3((unsigned)nblk), 32 * (pb.D / 8), 0, stream>>>(pb, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
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
