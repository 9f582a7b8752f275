// sage_host.cu -- the C ABI (include/sage_b200.h): argument validation,
// workspace layout, TMA descriptor creation and kernel launches.
//
// The call mirrors sageattn(q, k, v, tensor_layout, is_causal, smooth_k,
// sm_scale) as the "sageattention" package page states it ("Quickstart"):
// head_dim 64/96/128, Nq != Nkv and group-query attention.  Everything here
// is host code: it checks the request, derives the workspace sub-buffers and
// enqueues kernels; it never touches tensor data and allocates nothing.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/sage_b200.h"
#include "common.cuh"

using namespace sage;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
  size_t off_q8, off_k8, off_v8t, off_qs, off_ks, off_vs, off_mk, off_mv, off_mq, off_dsk;
  size_t off_ksum, off_vsum, off_vmax, off_vmin, off_vinv, off_status, off_cu, total;
  int Dp, Nq_pad, Nkv_pad, nqb, nkb;
};

bool is_flag(int32_t v) { return v == 0 || v == 1; }

// Shape and flag checks shared by every entry point (no pointers read).
sage_status_t check_shape(const sage_attn_params_t *p) {
  if (!p) return SAGE_ERR_INVALID_ARG;
  if (p->D != 64 && p->D != 96 && p->D != 128) return SAGE_ERR_UNSUPPORTED;
  if (p->dtype != SAGE_F16 && p->dtype != SAGE_BF16) return SAGE_ERR_UNSUPPORTED;
  if (p->layout != SAGE_LAYOUT_HND && p->layout != SAGE_LAYOUT_NHD) return SAGE_ERR_INVALID_ARG;
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->Nq < 0 || p->Nkv < 0) return SAGE_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return SAGE_ERR_INVALID_ARG;
  if (p->Nq > 0 && p->Nkv < 1) return SAGE_ERR_INVALID_ARG;
  if (!is_flag(p->is_causal) || !is_flag(p->smooth_k) || !is_flag(p->smooth_q) ||
      !is_flag(p->smooth_v))
    return SAGE_ERR_INVALID_ARG;
  if (!(p->sm_scale == p->sm_scale) || std::isinf(p->sm_scale)) return SAGE_ERR_INVALID_ARG;
  if (p->qk_bits != 0 && p->qk_bits != 8 && p->qk_bits != 4) return SAGE_ERR_INVALID_ARG;
  // TMA row coordinates and kernel indices are 32-bit
  const long long nq_pad = (p->Nq + 127LL) / 128 * 128, nkv_pad = (p->Nkv + 127LL) / 128 * 128;
  if ((long long)p->B * p->Hq * nq_pad >= (1LL << 31)) return SAGE_ERR_UNSUPPORTED;
  if ((long long)p->B * p->Hkv * nkv_pad >= (1LL << 31)) return SAGE_ERR_UNSUPPORTED;
  if ((long long)p->B * p->Hkv * p->D >= (1LL << 31)) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

bool is_varlen(const sage_attn_params_t *p) { return p->cu_seqlens_q != nullptr; }

// Offsets of a variable-length batch (host arrays, read here): both or
// neither given; start at 0, non-decreasing, each length within its bound,
// at least one key for a sequence with queries.
sage_status_t check_varlen(const sage_attn_params_t *p) {
  if ((p->cu_seqlens_q == nullptr) != (p->cu_seqlens_kv == nullptr)) return SAGE_ERR_INVALID_ARG;
  if (!is_varlen(p)) return SAGE_OK;
  const int32_t *cq = p->cu_seqlens_q, *ck = p->cu_seqlens_kv;
  if (cq[0] != 0 || ck[0] != 0) return SAGE_ERR_INVALID_ARG;
  for (int b = 0; b < p->B; ++b) {
    const long long lq = (long long)cq[b + 1] - cq[b], lk = (long long)ck[b + 1] - ck[b];
    if (lq < 0 || lq > p->Nq || lk < 0 || lk > p->Nkv) return SAGE_ERR_INVALID_ARG;
    if (lq > 0 && lk < 1) return SAGE_ERR_INVALID_ARG;
  }
  return SAGE_OK;
}

Layout make_layout(const sage_attn_params_t *p) {
  Layout L{};
  L.Dp = p->D == 64 ? 64 : 128;
  L.Nq_pad = int((p->Nq + 127) / 128 * 128);
  L.Nkv_pad = int((p->Nkv + 127) / 128 * 128);
  L.nqb = L.Nq_pad / 128;
  L.nkb = L.Nkv_pad / kKBlk;
  const size_t BHq = size_t(p->B) * p->Hq, BHk = size_t(p->B) * p->Hkv, D = size_t(p->D);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, kAlign);
    return at;
  };
  L.off_q8 = take(BHq * L.Nq_pad * L.Dp);
  L.off_k8 = take(BHk * L.Nkv_pad * L.Dp);
  L.off_v8t = take(BHk * D * L.Nkv_pad);
  L.off_qs = take(BHq * L.Nq_pad * sizeof(float));   // one scale per query token
  L.off_ks = take(BHk * L.nkb * sizeof(float));      // one per 32 keys
  L.off_vs = take(BHk * D * sizeof(float));
  L.off_mk = take(BHk * D * sizeof(float));
  L.off_mv = take(BHk * D * sizeof(float));
  // k_sum, v_sum, v_max are contiguous (one memset clears them), then v_min
  L.off_ksum = o;
  o += BHk * D * sizeof(long long);
  L.off_vsum = o;
  o += BHk * D * sizeof(long long);
  L.off_vmax = o;
  o = align_up(o + BHk * D * sizeof(unsigned), kAlign);
  L.off_vmin = take(BHk * D * sizeof(unsigned));
  L.off_vinv = take(BHk * D * sizeof(float));
  L.off_status = take(16);
  // offsets and running unit totals of a variable-length batch: 6 x (B + 1)
  L.off_cu = is_varlen(p) ? take(6 * (size_t(p->B) + 1) * sizeof(int32_t)) : 0;
  if (p->smooth_q) {
    L.off_mq = take(BHq * L.nqb * D * sizeof(float));
    L.off_dsk = take(BHq * L.nqb * size_t(L.Nkv_pad) * sizeof(float));
  } else {
    L.off_mq = L.off_dsk = 0;
  }
  L.total = o;
  return L;
}

Workspace make_workspace(const sage_attn_params_t *p, const Layout &L) {
  uint8_t *w = static_cast<uint8_t *>(p->workspace);
  Workspace ws{};
  ws.q8 = reinterpret_cast<int8_t *>(w + L.off_q8);
  ws.k8 = reinterpret_cast<int8_t *>(w + L.off_k8);
  ws.v8t = w + L.off_v8t;
  ws.q_scale = reinterpret_cast<float *>(w + L.off_qs);
  ws.k_scale = reinterpret_cast<float *>(w + L.off_ks);
  ws.v_scale = reinterpret_cast<float *>(w + L.off_vs);
  ws.mean_k = reinterpret_cast<float *>(w + L.off_mk);
  ws.mean_v = reinterpret_cast<float *>(w + L.off_mv);
  ws.mq = p->smooth_q ? reinterpret_cast<float *>(w + L.off_mq) : nullptr;
  ws.dsk = p->smooth_q ? reinterpret_cast<float *>(w + L.off_dsk) : nullptr;
  ws.k_sum = reinterpret_cast<long long *>(w + L.off_ksum);
  ws.v_sum = reinterpret_cast<long long *>(w + L.off_vsum);
  ws.v_max = reinterpret_cast<unsigned *>(w + L.off_vmax);
  ws.v_min = reinterpret_cast<unsigned *>(w + L.off_vmin);
  ws.v_inv = reinterpret_cast<float *>(w + L.off_vinv);
  ws.status = reinterpret_cast<int *>(w + L.off_status);
  ws.Dp = L.Dp;
  ws.Nq_pad = L.Nq_pad;
  ws.Nkv_pad = L.Nkv_pad;
  ws.nqb = L.nqb;
  ws.nkb = L.nkb;
  return ws;
}

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

sage_status_t check_tensor(const void *ptr, const int64_t *st) {
  if (!ptr) return SAGE_ERR_INVALID_ARG;
  if (st[3] != 1) return SAGE_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (st[i] < 0) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(ptr)) return SAGE_ERR_ALIGNMENT;
  for (int i = 0; i < 3; ++i)
    if (st[i] % 8 != 0) return SAGE_ERR_ALIGNMENT;
  return SAGE_OK;
}

sage_status_t check_workspace(const sage_attn_params_t *p, const Layout &L) {
  if (!p->workspace) return SAGE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(p->workspace) % kAlign != 0) return SAGE_ERR_WORKSPACE;
  if (p->workspace_bytes < L.total) return SAGE_ERR_WORKSPACE;
  return SAGE_OK;
}

// The library's kernels are built for sm_100a only.
sage_status_t check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SAGE_ERR_CUDA;
  if (major != 10 || minor != 0) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

// (batch, head, token) element strides of a tensor given in layout order.
void bhn_strides(const sage_attn_params_t *p, const int64_t *st, long long &sb, long long &sh,
                 long long &sn) {
  sb = st[0];
  if (p->layout == SAGE_LAYOUT_HND) {
    sh = st[1];
    sn = st[2];
  } else {
    sn = st[1];
    sh = st[2];
  }
}

Problem make_problem(const sage_attn_params_t *p) {
  Problem pb{};
  pb.q = static_cast<const uint16_t *>(p->q);
  pb.k = static_cast<const uint16_t *>(p->k);
  pb.v = static_cast<const uint16_t *>(p->v);
  pb.out = p->out;
  pb.B = p->B;
  pb.Hq = p->Hq;
  pb.Hkv = p->Hkv;
  pb.Nq = p->Nq;
  pb.Nkv = p->Nkv;
  pb.D = p->D;
  bhn_strides(p, p->q_strides, pb.qs_b, pb.qs_h, pb.qs_n);
  bhn_strides(p, p->k_strides, pb.ks_b, pb.ks_h, pb.ks_n);
  bhn_strides(p, p->v_strides, pb.vs_b, pb.vs_h, pb.vs_n);
  bhn_strides(p, p->o_strides, pb.os_b, pb.os_h, pb.os_n);
  pb.bf16 = p->dtype == SAGE_BF16;
  pb.is_causal = p->is_causal;
  pb.smooth_k = p->smooth_k;
  pb.smooth_q = p->smooth_q;
  pb.smooth_v = p->smooth_v;
  // sm_scale <= 0 selects 1/sqrt(D); both roundings are IEEE fp32
  pb.sm_scale = p->sm_scale > 0.f ? p->sm_scale : 1.0f / std::sqrt(float(p->D));
  volatile float l2e = kLog2e;  // keep the product a single fp32 rounding
  pb.K2 = pb.sm_scale * l2e;
  pb.qmax = p->qk_bits == 4 ? 7.0f : 127.0f;
  return pb;
}

// ---- TMA descriptors (driver entry point fetched through the runtime)
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D byte tensor [rows][cols] (row pitch = cols bytes), box [box_rows][box_cols].
bool make_map(CUtensorMap *m, void *base, uint64_t cols, uint64_t rows, uint32_t box_cols,
              uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw =
      box_cols == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Maps {
  CUtensorMap q, k, v;
};

// Tensor map of a caller's 16-bit input (element strides s_b, s_h, s_n; the
// channel stride is 1) for the pre-pass: dimensions (D, N, H, B), or
// (D, H, N, B) when the head stride is the smaller one, so the strides
// increase; box D channels x `rows` tokens of one head, no swizzle, zero fill
// past N.  A variable-length batch passes the packed token count as N and
// B = 1.  Returns false when the driver rejects the map (the pre-pass then
// copies rows one by one).
bool make_input_map(const uint16_t *base, int bf16, int D, long long s_b, long long s_h,
                    long long s_n, long long H, long long N, long long B, uint32_t rows,
                    CUtensorMap *m, int *hn) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || N <= 0 || H <= 0 || B <= 0) return false;
  const bool head_inner = s_h < s_n;
  *hn = head_inner ? 1 : 0;
  const long long sb = B == 1 ? (head_inner ? N * s_n : H * s_h) : s_b;
  const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(head_inner ? H : N),
                              cuuint64_t(head_inner ? N : H), cuuint64_t(B)};
  const cuuint64_t strides[3] = {cuuint64_t(2 * (head_inner ? s_h : s_n)),
                                 cuuint64_t(2 * (head_inner ? s_n : s_h)), cuuint64_t(2 * sb)};
  const cuuint32_t box[4] = {cuuint32_t(D), head_inner ? 1u : rows, head_inner ? rows : 1u, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
            const_cast<uint16_t *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Input maps for every input the pre-pass reads whose tokens are not dense
// (token stride != D); dense inputs keep one bulk copy per unit.  nq_tot /
// nkv_tot: packed token counts of a variable-length batch (0 otherwise).
void make_input_maps(Problem &pb, InputMaps &im, long long nq_tot, long long nkv_tot) {
  const bool vl = pb.cu_q != nullptr;
  const long long Bm = vl ? 1 : pb.B;
  const long long Nk = vl ? nkv_tot : pb.Nkv, Nq = vl ? nq_tot : pb.Nq;
  int hn0 = 0, hn1 = 0;
  if (pb.ks_n != pb.D && pb.smooth_k &&
      make_input_map(pb.k, pb.bf16, pb.D, pb.ks_b, pb.ks_h, pb.ks_n, pb.Hkv, Nk, Bm, 64, &im.k64, &hn0) &&
      make_input_map(pb.k, pb.bf16, pb.D, pb.ks_b, pb.ks_h, pb.ks_n, pb.Hkv, Nk, Bm, 128, &im.k128, &hn1)) {
    pb.k_map = 1;
    pb.k_hn = hn0;
  } else if (pb.ks_n != pb.D && !pb.smooth_k &&
             make_input_map(pb.k, pb.bf16, pb.D, pb.ks_b, pb.ks_h, pb.ks_n, pb.Hkv, Nk, Bm, 128, &im.k128, &hn1)) {
    pb.k_map = 1;  // kv_stats does not read K without smooth_k
    pb.k_hn = hn1;
  }
  if (pb.vs_n != pb.D &&
      make_input_map(pb.v, pb.bf16, pb.D, pb.vs_b, pb.vs_h, pb.vs_n, pb.Hkv, Nk, Bm, 64, &im.v64, &hn0) &&
      make_input_map(pb.v, pb.bf16, pb.D, pb.vs_b, pb.vs_h, pb.vs_n, pb.Hkv, Nk, Bm, 128, &im.v128, &hn1)) {
    pb.v_map = 1;
    pb.v_hn = hn0;
  }
  if (pb.qs_n != pb.D &&
      make_input_map(pb.q, pb.bf16, pb.D, pb.qs_b, pb.qs_h, pb.qs_n, pb.Hq, Nq, Bm, 128, &im.q128, &hn0)) {
    pb.q_map = 1;
    pb.q_hn = hn0;
  }
}

bool make_maps(const sage_attn_params_t *p, const Workspace &ws, Maps &m) {
  const uint64_t BHq = uint64_t(p->B) * p->Hq, BHk = uint64_t(p->B) * p->Hkv;
  return make_map(&m.q, ws.q8, ws.Dp, BHq * ws.Nq_pad, ws.Dp, 128) &&
         make_map(&m.k, ws.k8, ws.Dp, BHk * ws.Nkv_pad, ws.Dp, 128) &&
         make_map(&m.v, ws.v8t, ws.Nkv_pad, BHk * p->D, 128, p->D);
}

// Full validation for calls that read tensors / the workspace.
sage_status_t validate(const sage_attn_params_t *p, bool need_inputs, bool need_out, Layout &L) {
  sage_status_t s = check_shape(p);
  if (s != SAGE_OK) return s;
  if ((s = check_varlen(p)) != SAGE_OK) return s;
  if (need_inputs) {
    if ((s = check_tensor(p->q, p->q_strides)) != SAGE_OK) return s;
    if ((s = check_tensor(p->k, p->k_strides)) != SAGE_OK) return s;
    if ((s = check_tensor(p->v, p->v_strides)) != SAGE_OK) return s;
  }
  if (need_out && (s = check_tensor(p->out, p->o_strides)) != SAGE_OK) return s;
  L = make_layout(p);
  if ((s = check_workspace(p, L)) != SAGE_OK) return s;
  return check_device();
}

// pre / attn: which half of the pass to enqueue (both for sage_attn_fwd).
sage_status_t run(const sage_attn_params_t *p, sage_stream_t stream, bool pre, bool attn) {
  // No queries: nothing to compute and no pointer is read (empty tensors
  // may have null data pointers).
  sage_status_t s = check_shape(p);
  if (s != SAGE_OK) return s;
  if (p->Nq == 0) return SAGE_OK;
  Layout L;
  s = validate(p, pre, attn, L);
  if (s != SAGE_OK) return s;
  const Workspace ws = make_workspace(p, L);
  Problem pb = make_problem(p);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  long long nq_tot = 0, nkv_tot = 0;  // packed token counts (variable-length batches)
  if (is_varlen(p)) {
    // The kernels read the (validated) sequence offsets from the workspace,
    // with the running totals of each sequence's query tiles (128 rows),
    // query-tile pairs (256 rows) and key chunks (64 and 128 tokens), so that
    // they enumerate only units inside a sequence.
    const int B = p->B;
    std::vector<int32_t> h(6 * size_t(B + 1), 0);
    int32_t *cq = h.data(), *ck = cq + B + 1, *pq = ck + B + 1, *p64 = pq + B + 1, *p128 = p64 + B + 1,
            *p256 = p128 + B + 1;
    for (int b = 0; b <= B; ++b) {
      cq[b] = p->cu_seqlens_q[b];
      ck[b] = p->cu_seqlens_kv[b];
    }
    for (int b = 0; b < B; ++b) {
      const int lq = cq[b + 1] - cq[b], lk = ck[b + 1] - ck[b];
      pq[b + 1] = pq[b] + (lq + 127) / 128;
      p64[b + 1] = p64[b] + (lk + 63) / 64;
      p128[b + 1] = p128[b] + (lk + 127) / 128;
      p256[b + 1] = p256[b] + ((lq + 127) / 128 + 1) / 2;  // pairs of query tiles
    }
    int32_t *d = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(p->workspace) + L.off_cu);
    // pageable source: the copy has read h before the call returns
    if (cudaMemcpyAsync(d, h.data(), h.size() * sizeof(int32_t), cudaMemcpyHostToDevice, st) != cudaSuccess)
      return SAGE_ERR_CUDA;
    pb.cu_q = d;
    pb.cu_kv = d + (B + 1);
    pb.pc_q128 = d + 2 * (B + 1);
    pb.pc_kv64 = d + 3 * (B + 1);
    pb.pc_kv128 = d + 4 * (B + 1);
    pb.pc_q256 = d + 5 * (B + 1);
    pb.tot_q256 = p256[B];
    pb.tot_q128 = pq[B];
    pb.tot_kv64 = p64[B];
    pb.tot_kv128 = p128[B];
    nq_tot = cq[B];
    nkv_tot = ck[B];
  }
  Maps m;
  if (pre && cudaMemsetAsync(ws.status, 0, sizeof(int), st) != cudaSuccess) return SAGE_ERR_CUDA;
  if (pre) {
    InputMaps im;
    std::memset(&im, 0, sizeof(im));
    make_input_maps(pb, im, nq_tot, nkv_tot);
    if (launch_prepass(pb, ws, im, st) != cudaSuccess) return SAGE_ERR_CUDA;
  }
  if (attn) {
    if (!make_maps(p, ws, m)) return SAGE_ERR_CUDA;
    if (launch_attention(pb, ws, m.q, m.k, m.v, st) != cudaSuccess) return SAGE_ERR_CUDA;
  }
  return SAGE_OK;
}

// Library-owned scratch for sage_attn_fwd_noalloc (see the header): one
// array per device that loads the library, alive until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SAGE_NOALLOC_MAX_WORKSPACE_BYTES];

// Device address of g_noalloc_scratch, looked up with the device current and
// cached per device ordinal together with the context it was looked up in:
// after a device reset the module is loaded again (possibly elsewhere) in a
// new primary context, so a changed context triggers a fresh lookup.  In host
// code the array's name is only a host-side stand-in, never a device address.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CtxGetCurrentFn ctx_get_current_fn() {
  static std::once_flag once;
  static CtxGetCurrentFn fn = nullptr;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

sage_status_t noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SAGE_ERR_UNSUPPORTED;
  // a first lookup lets the runtime create or bind the device's primary
  // context; the context is read after it
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  CUcontext ctx = nullptr;
  CtxGetCurrentFn get = ctx_get_current_fn();
  if (g_noalloc_ptr[dev]) {
    if (!get || get(&ctx) != CUDA_SUCCESS) return SAGE_ERR_CUDA;
    if (ctx == g_noalloc_ctx[dev]) {
      *out = g_noalloc_ptr[dev];
      return SAGE_OK;
    }
  }
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return SAGE_ERR_CUDA;
  if (!get || get(&ctx) != CUDA_SUCCESS || !ctx) return SAGE_ERR_CUDA;
  g_noalloc_ptr[dev] = ptr;
  g_noalloc_ctx[dev] = ctx;
  *out = ptr;
  return SAGE_OK;
}

// The params of a call redirected to the library scratch.
sage_status_t noalloc_params(const sage_attn_params_t *p, sage_attn_params_t *q) {
  sage_status_t s = check_shape(p);
  if (s != SAGE_OK) return s;
  if (make_layout(p).total > SAGE_NOALLOC_MAX_WORKSPACE_BYTES) return SAGE_ERR_WORKSPACE;
  if ((s = check_device()) != SAGE_OK) return s;
  void *scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != SAGE_OK) return s;
  *q = *p;
  q->workspace = scratch;
  q->workspace_bytes = SAGE_NOALLOC_MAX_WORKSPACE_BYTES;
  return SAGE_OK;
}

}  // namespace

extern "C" {

int32_t sage_abi_version(void) { return SAGE_ABI_VERSION; }

const char *sage_status_string(sage_status_t s) {
  switch (s) {
    case SAGE_OK: return "SAGE_OK";
    case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
    case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
    case SAGE_ERR_ALIGNMENT: return "SAGE_ERR_ALIGNMENT";
    case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
    case SAGE_ERR_DEVICE_TIMEOUT: return "SAGE_ERR_DEVICE_TIMEOUT";
    case SAGE_ERR_WORKSPACE: return "SAGE_ERR_WORKSPACE";
  }
  return "SAGE_ERR_UNKNOWN";
}

sage_status_t sage_workspace_size(const sage_attn_params_t *p, size_t *bytes) {
  if (!bytes) return SAGE_ERR_INVALID_ARG;
  const sage_status_t s = check_shape(p);
  if (s != SAGE_OK) return s;
  *bytes = make_layout(p).total;
  return SAGE_OK;
}

sage_status_t sage_workspace_view(const sage_attn_params_t *p, sage_workspace_view_t *v) {
  if (!v) return SAGE_ERR_INVALID_ARG;
  sage_status_t s = check_shape(p);
  if (s != SAGE_OK) return s;
  const Layout L = make_layout(p);
  if ((s = check_workspace(p, L)) != SAGE_OK) return s;
  const Workspace ws = make_workspace(p, L);
  v->q8 = ws.q8;
  v->k8 = ws.k8;
  v->v8t = ws.v8t;
  v->q_scale = ws.q_scale;
  v->k_scale = ws.k_scale;
  v->v_scale = ws.v_scale;
  v->mean_k = ws.mean_k;
  v->mean_v = ws.mean_v;
  v->mq = ws.mq;
  v->dsk = ws.dsk;
  v->status = ws.status;
  v->Dp = ws.Dp;
  v->Nq_pad = ws.Nq_pad;
  v->Nkv_pad = ws.Nkv_pad;
  return SAGE_OK;
}

sage_status_t sage_attn_fwd(const sage_attn_params_t *p, sage_stream_t stream) {
  return run(p, stream, true, true);
}

sage_status_t sage_attn_fwd_prepass(const sage_attn_params_t *p, sage_stream_t stream) {
  return run(p, stream, true, false);
}

sage_status_t sage_attn_fwd_attention(const sage_attn_params_t *p, sage_stream_t stream) {
  return run(p, stream, false, true);
}

sage_status_t sage_attn_fwd_noalloc(const sage_attn_params_t *p, sage_stream_t stream) {
  sage_attn_params_t q;
  const sage_status_t s = noalloc_params(p, &q);
  if (s != SAGE_OK) return s;
  return run(&q, stream, true, true);
}

sage_status_t sage_noalloc_device_status(const sage_attn_params_t *p, int32_t *code) {
  if (!code) return SAGE_ERR_INVALID_ARG;
  sage_attn_params_t q;
  const sage_status_t s = noalloc_params(p, &q);
  if (s != SAGE_OK) return s;
  return sage_get_device_status(&q, code);
}

sage_status_t sage_quantize(const sage_attn_params_t *p, sage_stream_t stream) {
  return run(p, stream, true, false);
}

sage_status_t sage_attn_quantized(const sage_attn_params_t *p, sage_stream_t stream) {
  return run(p, stream, false, true);
}

sage_status_t sage_debug_dump_s(const sage_attn_params_t *p, int32_t b, int32_t h, int32_t qtile,
                                int32_t ktile, int32_t *s_out, sage_stream_t stream) {
  sage_status_t s = check_shape(p);
  if (s != SAGE_OK) return s;
  if (p->Nq == 0 || is_varlen(p)) return SAGE_ERR_INVALID_ARG;
  Layout L;
  if ((s = validate(p, false, true, L)) != SAGE_OK) return s;
  if (!s_out || b < 0 || b >= p->B || h < 0 || h >= p->Hq || qtile < 0 || qtile >= L.nqb ||
      ktile < 0 || ktile >= L.Nkv_pad / 128)
    return SAGE_ERR_INVALID_ARG;
  const Workspace ws = make_workspace(p, L);
  Maps m;
  if (!make_maps(p, ws, m)) return SAGE_ERR_CUDA;
  Problem pb = make_problem(p);
  pb.s_dump = s_out;
  pb.dump_bh = b * p->Hq + h;
  pb.dump_qt = qtile;
  pb.dump_kt = ktile;
  return launch_attention_dump(pb, ws, m.q, m.k, m.v, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_pv(const sage_attn_params_t *p, int32_t b, int32_t hkv, int32_t ktile,
                            const uint8_t *p8, float *o_out, sage_stream_t stream) {
  Layout L;
  sage_status_t s = validate(p, false, false, L);
  if (s != SAGE_OK) return s;
  if (!p8 || !o_out || !aligned16(p8) || b < 0 || b >= p->B || hkv < 0 || hkv >= p->Hkv ||
      ktile < 0 || ktile >= L.Nkv_pad / 128)
    return SAGE_ERR_INVALID_ARG;
  const Workspace ws = make_workspace(p, L);
  Maps m;
  if (!make_maps(p, ws, m)) return SAGE_ERR_CUDA;
  return launch_debug_pv(make_problem(p), ws, m.v, b, hkv, ktile, p8, o_out,
                         reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_e4m3(const float *in, uint8_t *out, int64_t n, sage_stream_t stream) {
  if (n < 0 || (n > 0 && (!in || !out))) return SAGE_ERR_INVALID_ARG;
  sage_status_t s = check_device();
  if (s != SAGE_OK) return s;
  return launch_debug_e4m3(in, out, n, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_mma_loop(int32_t ctas, int32_t iters, int32_t kind, int32_t *sink,
                                  sage_stream_t stream) {
  if (ctas < 1 || iters < 1 || (kind != 0 && kind != 1) || !sink) return SAGE_ERR_INVALID_ARG;
  sage_status_t s = check_device();
  if (s != SAGE_OK) return s;
  return launch_mma_loop(ctas, iters, kind, sink, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_ex2(const float *in, float *out, int64_t n, sage_stream_t stream) {
  if (n < 0 || (n > 0 && (!in || !out))) return SAGE_ERR_INVALID_ARG;
  sage_status_t s = check_device();
  if (s != SAGE_OK) return s;
  return launch_debug_ex2(in, out, n, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_wait_timeout(int32_t *status, sage_stream_t stream) {
  if (!status) return SAGE_ERR_INVALID_ARG;
  sage_status_t s = check_device();
  if (s != SAGE_OK) return s;
  return launch_wait_timeout(status, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

sage_status_t sage_get_device_status(const sage_attn_params_t *p, int32_t *code) {
  if (!code) return SAGE_ERR_INVALID_ARG;
  sage_status_t s = check_shape(p);
  if (s != SAGE_OK) return s;
  const Layout L = make_layout(p);
  if ((s = check_workspace(p, L)) != SAGE_OK) return s;
  int32_t v = 0;
  if (cudaMemcpy(&v, static_cast<uint8_t *>(p->workspace) + L.off_status, sizeof(v),
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return SAGE_ERR_CUDA;
  *code = v;
  return SAGE_OK;
}

}  // extern "C"
