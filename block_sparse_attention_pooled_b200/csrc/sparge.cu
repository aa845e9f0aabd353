// Host side of the C ABI declared in include/sparge.h: argument checks,
// workspace carving, TMA descriptors and kernel launches. All kernels of the
// library are compiled in this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "sparge.h"
#include "ptx.cuh"
#include "mask.cuh"
#include "attn.cuh"
#include "linear.cuh"
#include "lin_out.cuh"
#include "quant.cuh"
#include "attn_q8.cuh"
#include "attn_bwd.cuh"
#include "lin_bwd.cuh"
#include "selftest.cuh"

namespace {

using namespace sparge;

constexpr int kMaxNkb = 4096;

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Dims {
  int64_t BH, nqb, nkb;
};

// Shape checks shared by every entry point. Returns OK / INVALID / UNSUPPORTED.
sparge_status check_shape(const sparge_shape* s, Dims* out) {
  if (s == nullptr) return SPARGE_ERR_INVALID_ARG;
  if (s->B <= 0 || s->H <= 0 || s->N <= 0 || s->d <= 0 || s->bq <= 0 || s->bk <= 0) return SPARGE_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return SPARGE_ERR_UNSUPPORTED;
  if (s->bq != 64 && s->bq != 128) return SPARGE_ERR_UNSUPPORTED;
  if (s->bk != 64 && s->bk != 128) return SPARGE_ERR_UNSUPPORTED;
  out->BH = (int64_t)s->B * s->H;
  out->nqb = ceil_div(s->N, s->bq);
  out->nkb = ceil_div(s->N, s->bk);
  if (out->nkb > kMaxNkb) return SPARGE_ERR_UNSUPPORTED;
  if (out->BH * out->nqb > INT32_MAX || out->BH > INT32_MAX) return SPARGE_ERR_UNSUPPORTED;
  return SPARGE_OK;
}

sparge_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SPARGE_OK;
  (void)cudaGetLastError();  // clear the sticky-free launch error
  return SPARGE_ERR_CUDA;
}

// The mask's scratch: pooled Q and K (double [BH, Nqb | Nkb, d]) and the
// scaled scores (double [BH, Nqb, Nkb]) that the selection turns into
// probabilities.
struct MaskWs {
  size_t qbar, kbar, z, total;
};

MaskWs mask_ws(const sparge_shape* s, const Dims& d) {
  MaskWs w;
  w.qbar = 0;
  w.kbar = w.qbar + align256((size_t)d.BH * d.nqb * s->d * 8);
  w.z = w.kbar + align256((size_t)d.BH * d.nkb * s->d * 8);
  w.total = w.z + align256((size_t)d.BH * d.nqb * d.nkb * 8);
  return w;
}

// The router's scratch: the mask's, then the projected blocks q^ and k^
// (double, sized for the widest supported router width).
constexpr int kMaxRouterDim = 128;

struct RouterWs {
  MaskWs mask;
  size_t qhat, khat, total;
};

RouterWs router_ws(const sparge_shape* s, const Dims& d) {
  RouterWs w;
  w.mask = mask_ws(s, d);
  w.qhat = w.mask.total;
  w.khat = w.qhat + align256((size_t)d.BH * d.nqb * kMaxRouterDim * 8);
  w.total = w.khat + align256((size_t)d.BH * d.nkb * kMaxRouterDim * 8);
  return w;
}

// ---------------------------------------------------------------------------
// TMA descriptors through the driver entry point (no link-time libcuda).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 map over [BH][N][d] with a (64 columns x rows x 1) box, 128-byte
// swizzle, zero fill outside the tensor.
bool make_map_bhnd(CUtensorMap* m, const void* base, int64_t BH, int N, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Raises a kernel's dynamic shared memory limit once per device. Any host
// thread may launch: the fast path reads an atomic table, and the attribute
// is only ever raised (to the largest size asked for so far) under a lock, so
// a thread asking for less cannot lower a limit another thread relies on.
template <typename K>
cudaError_t ensure_smem(K kernel, int bytes, int slot) {
  static std::atomic<int> done[64][32];  // [device][slot]: one slot per kernel
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || slot < 0 || slot >= 32)
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (done[dev][slot].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  std::lock_guard<std::mutex> lock(mu);
  const int have = done[dev][slot].load(std::memory_order_relaxed);
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[dev][slot].store(bytes, std::memory_order_release);
  return e;
}

// Launch order of the query tiles (tile_order_kernel): heads in groups whose
// K and V (2 N d bf16 each) fit in 64 MB of L2, heaviest tiles first. When not
// even two heads fit, the grid stays head-major (sorting inside one head
// measured slower: it breaks the locality of neighbouring query blocks, which
// keep mostly the same key blocks), and *order is set to null.
cudaError_t launch_tile_order(const int32_t* kv_cnt, const sparge_shape* s, const Dims& dm, int32_t** order,
                              cudaStream_t st) {
  const int64_t per_head = 4 * (int64_t)s->N * s->d;
  const int64_t G = std::min<int64_t>(dm.BH, (int64_t(64) << 20) / per_head);
  if (G < 2) {
    *order = nullptr;
    return cudaSuccess;
  }
  tile_order_kernel<<<(unsigned)ceil_div(dm.BH, G), kOrderThreads, tile_order_smem_bytes((int)dm.nkb), st>>>(
      kv_cnt, dm.BH, (int)dm.nqb, (int)dm.nkb, (int)G, *order);
  return cudaGetLastError();
}

inline size_t order_bytes(const Dims& d) { return align256((size_t)d.BH * d.nqb * 4); }

// Scaled scores of DD-wide pooled (or projected) vectors into Z.
template <int DD>
cudaError_t launch_scores(const double* a, const double* b, const Dims& dm, double* Z, cudaStream_t st) {
  const double scale = 1.0 / std::sqrt((double)DD);
  const int ssm = score_smem_bytes<DD>();
  cudaError_t e = ensure_smem(score_kernel<DD>, ssm, DD == 64 ? 0 : 1);
  if (e != cudaSuccess) return e;
  const int64_t tiles = dm.BH * ceil_div(dm.nqb, kScoreRows) * ceil_div(dm.nkb, kScoreTileJ);
  score_kernel<DD><<<(unsigned)tiles, 128, ssm, st>>>(a, b, (int)dm.nqb, (int)dm.nkb, scale, Z);
  return cudaGetLastError();
}

// Router projections of the pooled vectors (DR output columns).
template <int D, int DR>
cudaError_t launch_projection(const double* qbar, const double* kbar, const Dims& dm, int H, const float* Wq,
                              const float* Wk, double* qhat, double* khat, cudaStream_t st) {
  const unsigned gq = (unsigned)(ceil_div(dm.nqb, kProjRows) * dm.BH);
  const unsigned gk = (unsigned)(ceil_div(dm.nkb, kProjRows) * dm.BH);
  constexpr int psm = project_smem_bytes<D>();
  project_kernel<D, DR><<<gq, 128, psm, st>>>(qbar, dm.nqb, H, Wq, qhat);
  project_kernel<D, DR><<<gk, 128, psm, st>>>(kbar, dm.nkb, H, Wk, khat);
  return cudaGetLastError();
}

// Pool, (project,) score, select. Wq / Wk null: no router.
template <int D>
sparge_status launch_mask(const void* Q, const void* K, const sparge_shape* s, const Dims& dm, int kc, double topp,
                          int32_t* kv_idx, int32_t* kv_cnt, float* row_thresh, float* probs, uint8_t* ws,
                          cudaStream_t st, const float* Wq = nullptr, const float* Wk = nullptr, int dr = 0,
                          double* qhat = nullptr, double* khat = nullptr) {
  const MaskWs w = mask_ws(s, dm);
  double* qbar = reinterpret_cast<double*>(ws + w.qbar);
  double* kbar = reinterpret_cast<double*>(ws + w.kbar);
  double* Z = reinterpret_cast<double*>(ws + w.z);
  constexpr int per_cta = 128 / (D / 8);
  const int64_t gq = ceil_div(dm.BH * dm.nqb, per_cta), gk = ceil_div(dm.BH * dm.nkb, per_cta);
  pool_kernel<D><<<(unsigned)(gq + gk), 128, 0, st>>>(static_cast<const __nv_bfloat16*>(Q),
                                                     static_cast<const __nv_bfloat16*>(K), dm.BH, s->N, s->bq,
                                                     s->bk, gq, qbar, kbar);
  const int64_t tiles = dm.BH * ceil_div(dm.nqb, kScoreRows) * ceil_div(dm.nkb, kScoreTileJ);
  if (tiles > INT32_MAX) return SPARGE_ERR_UNSUPPORTED;
  cudaError_t e;
  if (Wq != nullptr) {
    if (dr == 64) {
      e = launch_projection<D, 64>(qbar, kbar, dm, s->H, Wq, Wk, qhat, khat, st);
      if (e == cudaSuccess) e = launch_scores<64>(qhat, khat, dm, Z, st);
    } else {
      e = launch_projection<D, 128>(qbar, kbar, dm, s->H, Wq, Wk, qhat, khat, st);
      if (e == cudaSuccess) e = launch_scores<128>(qhat, khat, dm, Z, st);
    }
  } else {
    e = launch_scores<D>(qbar, kbar, dm, Z, st);
  }
  if (e != cudaSuccess) return cuda_status(e);
  if (dm.nkb <= kSelWarpMaxNkb) {  // one warp per row
    const int sel_sm = select_warp_smem_bytes((int)dm.nkb);
    e = ensure_smem(select_warp_kernel, sel_sm, 17);
    if (e != cudaSuccess) return cuda_status(e);
    select_warp_kernel<<<(unsigned)ceil_div(dm.BH * dm.nqb, kSelWarpRows), kSelWarpRows * 32, sel_sm, st>>>(
        Z, dm.BH * dm.nqb, (int)dm.nkb, kc, topp, kv_idx, kv_cnt, row_thresh, probs);
    return cuda_status(cudaGetLastError());
  }
  const int sel_sm = select_smem_bytes((int)dm.nkb);
  e = ensure_smem(select_kernel, sel_sm, 2);
  if (e != cudaSuccess) return cuda_status(e);
  select_kernel<<<(unsigned)(dm.BH * dm.nqb), kSelectThreads, sel_sm, st>>>(Z, dm.BH * dm.nqb, (int)dm.nkb, kc, topp,
                                                                           kv_idx, kv_cnt, row_thresh, probs);
  return cuda_status(cudaGetLastError());
}

// 3-D map over one-byte codes [BH][N][128] with a (128 x rows x 1) box,
// 128-byte swizzle, zero fill outside the tensor.
bool make_map_u8(CUtensorMap* m, const void* base, int64_t BH, int N, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {128, (cuuint64_t)N * 128};
  cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Workspace of the backward: D_i per row, the transposed mask (query-block
// lists per key block and their lengths).
struct BwdWs {
  size_t dsum, qidx, qcnt, order, total;
};

BwdWs bwd_ws(const sparge_shape* s, const Dims& d) {
  BwdWs w;
  w.dsum = 0;
  w.qidx = w.dsum + align256((size_t)d.BH * s->N * 4);
  w.qcnt = w.qidx + align256((size_t)d.BH * d.nkb * d.nqb * 4);
  w.order = w.qcnt + align256((size_t)d.BH * d.nkb * 4);
  w.total = w.order + order_bytes(d);
  return w;
}

constexpr int kMaxTransposeSmem = 200 * 1024;

sparge_status launch_bwd(const void* Q, const void* K, const void* V, const sparge_shape* s, const Dims& dm,
                         const int32_t* kv_idx, const int32_t* kv_cnt, const void* O, const float* lse,
                         const void* dO, void* dQ, void* dK, void* dV, uint8_t* ws, cudaStream_t st) {
  constexpr int D = 128;
  CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv;
  if (!make_map_bhnd(&mq, Q, dm.BH, s->N, D, kTileQ) || !make_map_bhnd(&mk, K, dm.BH, s->N, D, kTileK) ||
      !make_map_bhnd(&mv, V, dm.BH, s->N, D, kTileK) || !make_map_bhnd(&mdo, dO, dm.BH, s->N, D, kTileQ) ||
      !make_map_bhnd(&mdq, dQ, dm.BH, s->N, D, s->bq) || !make_map_bhnd(&mdk, dK, dm.BH, s->N, D, kTileK) ||
      !make_map_bhnd(&mdv, dV, dm.BH, s->N, D, kTileK))
    return SPARGE_ERR_CUDA;
  const BwdWs w = bwd_ws(s, dm);
  float* dsum = reinterpret_cast<float*>(ws + w.dsum);
  int32_t* q_idx = reinterpret_cast<int32_t*>(ws + w.qidx);
  int32_t* q_cnt = reinterpret_cast<int32_t*>(ws + w.qcnt);
  const int64_t rows = dm.BH * s->N;
  bwd_dot_kernel<D><<<(unsigned)ceil_div(rows, 256 / (D / 8)), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), rows, dsum);
  const int tsm = transpose_smem_bytes((int)dm.nqb);
  cudaError_t e = ensure_smem(mask_transpose_kernel, tsm, 10);
  if (e != cudaSuccess) return cuda_status(e);
  mask_transpose_kernel<<<(unsigned)(dm.BH * ceil_div(dm.nkb, kTrCols)), kTrCols, tsm, st>>>(
      kv_idx, kv_cnt, (int)dm.nqb, (int)dm.nkb, q_idx, q_cnt);
  BwdParams p;
  p.lse = lse;
  p.dsum = dsum;
  p.N = s->N;
  p.nqb = (int)dm.nqb;
  p.nkb = (int)dm.nkb;
  p.bq = s->bq;
  p.bk = s->bk;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.scale = (float)(1.0 / std::sqrt((double)D));
  int32_t* order = reinterpret_cast<int32_t*>(ws + w.order);
  e = launch_tile_order(kv_cnt, s, dm, &order, st);
  if (e != cudaSuccess) return cuda_status(e);
  p.order = order;
  p.lst = kv_idx;
  p.cnt = kv_cnt;
  const BwdLinParams lp{};
  e = ensure_smem(attn_bwd_dq_kernel<D, false>, BwdQSmem<D, false>::kBytes, 11);
  if (e != cudaSuccess) return cuda_status(e);
  attn_bwd_dq_kernel<D, false><<<(unsigned)(dm.BH * dm.nqb), bwd_q_threads<false>(), BwdQSmem<D, false>::kBytes,
                                 st>>>(
      mq, mk, mv, mdo, mdq, mq, p, lp);
  p.order = nullptr;
  p.lst = q_idx;
  p.cnt = q_cnt;
  const BwdKVLin lk{};
  e = ensure_smem(attn_bwd_dkdv_kernel<D, 0>, BwdKVSmem<D>::kBytes, 12);
  if (e != cudaSuccess) return cuda_status(e);
  attn_bwd_dkdv_kernel<D, 0><<<(unsigned)(dm.BH * ceil_div(s->N, kTileK)), kAttnThreads, BwdKVSmem<D>::kBytes, st>>>(
      mq, mk, mv, mdo, mdk, mdv, p, lk);
  return cuda_status(cudaGetLastError());
}

// Workspace of the low-bit sparse branch: codes and scales of Q, K, V.
struct Q8Ws {
  size_t q8, k8, v8, sq, sk, sv, vpart, order, total;
};

Q8Ws q8_ws(const sparge_shape* s, const Dims& d) {
  Q8Ws w;
  const size_t codes = align256((size_t)d.BH * s->N * s->d);
  const int64_t nch = ceil_div(s->N, kVChunk);
  w.q8 = 0;
  w.k8 = w.q8 + codes;
  w.v8 = w.k8 + codes;
  w.sq = w.v8 + codes;
  w.sk = w.sq + align256((size_t)d.BH * d.nqb * 4);
  w.sv = w.sk + align256((size_t)d.BH * d.nkb * 4);
  w.vpart = w.sv + align256((size_t)d.BH * s->d * 4);
  w.order = w.vpart + align256((size_t)d.BH * nch * s->d * 4);
  w.total = w.order + order_bytes(d);
  return w;
}

sparge_status launch_q8(const void* Q, const void* K, const void* V, const sparge_shape* s, const Dims& dm,
                        const int32_t* kv_idx, const int32_t* kv_cnt, void* O, uint8_t* ws, cudaStream_t st) {
  const Q8Ws w = q8_ws(s, dm);
  int8_t* q8 = reinterpret_cast<int8_t*>(ws + w.q8);
  int8_t* k8 = reinterpret_cast<int8_t*>(ws + w.k8);
  uint8_t* v8 = ws + w.v8;
  float* sq = reinterpret_cast<float*>(ws + w.sq);
  float* sk = reinterpret_cast<float*>(ws + w.sk);
  float* sv = reinterpret_cast<float*>(ws + w.sv);
  float* vpart = reinterpret_cast<float*>(ws + w.vpart);
  const int64_t q_ctas = dm.BH * dm.nqb, k_ctas = dm.BH * dm.nkb, nch = ceil_div(s->N, kVChunk);
  const int64_t total = q_ctas + k_ctas + dm.BH * nch;
  if (total > INT32_MAX) return SPARGE_ERR_UNSUPPORTED;
  const __nv_bfloat16* Qb = static_cast<const __nv_bfloat16*>(Q);
  const __nv_bfloat16* Kb = static_cast<const __nv_bfloat16*>(K);
  const __nv_bfloat16* Vb = static_cast<const __nv_bfloat16*>(V);
  quant_qk_vmax_kernel<128><<<(unsigned)total, kQuantThreads, 0, st>>>(Qb, Kb, Vb, dm.BH, s->N, s->bq, s->bk, q_ctas,
                                                                       k_ctas, q8, sq, k8, sk, vpart);
  quant_v_kernel<128><<<(unsigned)(dm.BH * nch), kQuantThreads, 0, st>>>(Vb, s->N, vpart, v8, sv);
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_u8(&mq, q8, dm.BH, s->N, kTileQ) || !make_map_u8(&mk, k8, dm.BH, s->N, kTileK) ||
      !make_map_u8(&mv, v8, dm.BH, s->N, kTileK) || !make_map_bhnd(&mo, O, dm.BH, s->N, 128, s->bq))
    return SPARGE_ERR_CUDA;
  int32_t* order = reinterpret_cast<int32_t*>(ws + w.order);
  cudaError_t eo = launch_tile_order(kv_cnt, s, dm, &order, st);
  if (eo != cudaSuccess) return cuda_status(eo);
  Q8Params p;
  p.kv_idx = kv_idx;
  p.kv_cnt = kv_cnt;
  p.order = order;
  p.sq = sq;
  p.sk = sk;
  p.sv = sv;
  p.N = s->N;
  p.nqb = (int)dm.nqb;
  p.nkb = (int)dm.nkb;
  p.bq = s->bq;
  p.bk = s->bk;
  p.c0 = (float)(1.4426950408889634 / std::sqrt(128.0));
  cudaError_t e = ensure_smem(attn_q8_kernel, Q8Smem::kBytes, 9);
  if (e != cudaSuccess) return cuda_status(e);
  attn_q8_kernel<<<(unsigned)(dm.BH * dm.nqb), kQ8Threads, Q8Smem::kBytes, st>>>(mq, mk, mv, mo, p);
  return cuda_status(cudaGetLastError());
}

struct Sla2Ws {
  size_t phik, s_all, z_all, z_tile, partial, order, total;
};

Sla2Ws sla2_ws(const sparge_shape* s, const Dims& d) {
  Sla2Ws w;
  w.phik = 0;
  w.s_all = w.phik + align256((size_t)d.BH * s->N * s->d * 2);
  w.z_all = w.s_all + align256((size_t)d.BH * s->d * s->d * 4);
  w.z_tile = w.z_all + align256((size_t)d.BH * s->d * 4);
  w.partial = w.z_tile + align256((size_t)d.BH * ceil_div(s->N, 64) * s->d * 4);
  w.order = w.partial + align256((size_t)(lin_grid(d.BH, s->N) + d.BH) * kLinPartial * 4);
  w.total = w.order + order_bytes(d);
  return w;
}

template <int D, bool MIX>
sparge_status launch_attn(const void* Q, const void* K, const void* V, const sparge_shape* s, const Dims& dm,
                          const int32_t* kv_idx, const int32_t* kv_cnt, void* O, float* lse, const float* alpha,
                          cudaStream_t st, const int32_t* order = nullptr) {
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_bhnd(&mq, Q, dm.BH, s->N, D, kTileQ) || !make_map_bhnd(&mk, K, dm.BH, s->N, D, kTileK) ||
      !make_map_bhnd(&mv, V, dm.BH, s->N, D, kTileK) || !make_map_bhnd(&mo, O, dm.BH, s->N, D, s->bq))
    return SPARGE_ERR_CUDA;
  AttnParams p;
  p.alpha = alpha;
  p.H = s->H;
  p.kv_idx = kv_idx;
  p.kv_cnt = kv_cnt;
  p.order = order;
  p.lse = lse;
  p.N = s->N;
  p.nqb = (int)dm.nqb;
  p.nkb = (int)dm.nkb;
  p.bq = s->bq;
  p.bk = s->bk;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  const int smem = AttnSmem<D, MIX>::kBytes;
  cudaError_t e = ensure_smem(attn_fwd_kernel<D, MIX>, smem, MIX ? 5 : (D == 64 ? 3 : 4));
  if (e != cudaSuccess) return cuda_status(e);
  attn_fwd_kernel<D, MIX><<<(unsigned)(dm.BH * dm.nqb), kAttnThreads, smem, st>>>(mq, mk, mv, mo, p);
  return cuda_status(cudaGetLastError());
}

// (1 - alpha_h) O_linear into O, one CTA per query block (d = 128).
sparge_status launch_linear_out(const void* Q, const void* V, const sparge_shape* s, const Dims& dm,
                                const int32_t* kv_idx, const int32_t* kv_cnt, const void* phik, const float* s_all,
                                const float* z_all, const float* z_tile, const float* alpha, void* O,
                                cudaStream_t st, float* den_out = nullptr, void* sc_out = nullptr,
                                float* zc_out = nullptr) {
  CUtensorMap mq, mv, mp, mo, msc;
  if (!make_map_bhnd(&mq, Q, dm.BH, s->N, 128, 128) || !make_map_bhnd(&mv, V, dm.BH, s->N, 128, 64) ||
      !make_map_bhnd(&mp, phik, dm.BH, s->N, 128, 64) || !make_map_bhnd(&mo, O, dm.BH, s->N, 128, s->bq) ||
      !make_map_bhnd(&msc, sc_out != nullptr ? sc_out : O, sc_out != nullptr ? dm.BH * dm.nqb : dm.BH,
                     sc_out != nullptr ? 128 : s->N, 128, 128))
    return SPARGE_ERR_CUDA;
  LoParams p;
  p.kv_idx = kv_idx;
  p.kv_cnt = kv_cnt;
  p.s_all = s_all;
  p.z_all = z_all;
  p.z_tile = z_tile;
  p.alpha = alpha;
  p.den_out = den_out;
  p.zc_out = zc_out;
  p.store_sc = sc_out != nullptr;
  p.H = s->H;
  p.N = s->N;
  p.ntiles = (int)ceil_div(s->N, 64);
  p.nqb = (int)dm.nqb;
  p.nkb = (int)dm.nkb;
  p.bq = s->bq;
  p.bk = s->bk;
  cudaError_t e = ensure_smem(linear_out_kernel, LoSmem::kBytes, 7);
  if (e != cudaSuccess) return cuda_status(e);
  const int64_t pairs = dm.BH * ceil_div(dm.nqb, 2);  // two neighbouring query blocks per CTA
  linear_out_kernel<<<(unsigned)pairs, kLoThreads, LoSmem::kBytes, st>>>(mq, mv, mp, mo, msc, p);
  return cuda_status(cudaGetLastError());
}

sparge_status launch_summaries(const void* K, const void* V, const sparge_shape* s, const Dims& dm, void* phik,
                               float* partial, float* s_all, float* z_all, float* z_tile, cudaStream_t st,
                               const float* row_scale = nullptr, const float* row_w = nullptr,
                               void* v_scaled = nullptr) {
  CUtensorMap mk, mv, mp, mvs;
  if (!make_map_bhnd(&mk, K, dm.BH, s->N, 128, 64) || !make_map_bhnd(&mv, V, dm.BH, s->N, 128, 64) ||
      !make_map_bhnd(&mp, phik, dm.BH, s->N, 128, 64) ||
      !make_map_bhnd(&mvs, v_scaled != nullptr ? v_scaled : phik, dm.BH, s->N, 128, 64))
    return SPARGE_ERR_CUDA;
  LinParams p;
  p.partial = partial;
  p.z_tile = z_tile;
  p.row_scale = row_scale;
  p.row_w = row_w;
  p.N = s->N;
  p.ntiles = (int)ceil_div(s->N, 64);
  p.total = dm.BH * p.ntiles;
  const int64_t grid = lin_grid(dm.BH, s->N);
  p.per_cta = ceil_div(p.total, grid);
  cudaError_t e;
  if (row_scale != nullptr) {  // the backward's G_all / g_all (K -> Q, V -> dO)
    e = ensure_smem(linear_summary_kernel<true>, LinSmem::kBytes, 13);
    if (e != cudaSuccess) return cuda_status(e);
    linear_summary_kernel<true><<<(unsigned)grid, kLinThreads, LinSmem::kBytes, st>>>(mk, mv, mp, mvs, p);
  } else {
    e = ensure_smem(linear_summary_kernel<false>, LinSmem::kBytes, 6);
    if (e != cudaSuccess) return cuda_status(e);
    linear_summary_kernel<false><<<(unsigned)grid, kLinThreads, LinSmem::kBytes, st>>>(mk, mv, mp, mp, p);
  }
  dim3 rgrid((unsigned)ceil_div(kLinPartial, 256), (unsigned)dm.BH);
  linear_reduce_kernel<<<rgrid, 256, 0, st>>>(partial, p.ntiles, p.per_cta, s_all, z_all);
  return cuda_status(cudaGetLastError());
}

// Workspace of the SLA2 backward: the forward's linear summaries and the
// recomputed branch outputs, the row pass, the gradient summaries, the
// transposed mask and the fp32 sparse partials of dK and dV.
struct Sla2BwdWs {
  Sla2Ws f;  // phi(K), S_all, z_all, z_tile, summary partials
  size_t sc, zc, os, lse, ol, den, alpha0, dsum, cw, fw, ew, dpart, phiq, cdo, g, gall, gtile, qidx, qcnt, dkp,
      dvp, total;
};

inline int sla2_row_chunks(int N) { return (int)ceil_div(N, kRowsPerCta); }

Sla2BwdWs sla2_bwd_ws(const sparge_shape* s, const Dims& d) {
  Sla2BwdWs w;
  w.f = sla2_ws(s, d);
  const size_t tens = align256((size_t)d.BH * s->N * s->d * 2), rows = align256((size_t)d.BH * s->N * 4);
  const size_t mat32 = align256((size_t)d.BH * s->d * s->d * 4);
  w.sc = w.f.total;
  w.zc = w.sc + align256((size_t)d.BH * d.nqb * s->d * s->d * 2);
  w.os = w.zc + align256((size_t)d.BH * d.nqb * s->d * 4);
  w.lse = w.os + tens;
  w.ol = w.lse + rows;
  w.den = w.ol + tens;
  w.alpha0 = w.den + rows;
  w.dsum = w.alpha0 + align256((size_t)s->H * 4);
  w.cw = w.dsum + rows;
  w.fw = w.cw + rows;
  w.ew = w.fw + rows;
  w.dpart = w.ew + rows;
  w.phiq = w.dpart + align256((size_t)d.BH * sla2_row_chunks(s->N) * 4);
  w.cdo = w.phiq + tens;
  w.g = w.cdo + tens;
  w.gall = w.g + mat32;
  w.gtile = w.gall + align256((size_t)d.BH * s->d * 4);
  w.qidx = w.gtile + align256((size_t)d.BH * ceil_div(s->N, 64) * s->d * 4);
  w.qcnt = w.qidx + align256((size_t)d.BH * d.nkb * d.nqb * 4);
  w.dkp = w.qcnt + align256((size_t)d.BH * d.nkb * 4);
  w.dvp = w.dkp + align256((size_t)d.BH * s->N * s->d * 4);
  w.total = w.dvp + align256((size_t)d.BH * s->N * s->d * 4);
  return w;
}

sparge_status launch_sla2_bwd(const void* Q, const void* K, const void* V, const sparge_shape* s, const Dims& dm,
                              const int32_t* kv_idx, const int32_t* kv_cnt, const float* alpha, const void* dO,
                              void* dQ, void* dK, void* dV, float* dalpha, uint8_t* ws, cudaStream_t st) {
  constexpr int D = 128;
  const Sla2BwdWs w = sla2_bwd_ws(s, dm);
  auto at = [&](size_t off) { return static_cast<void*>(ws + off); };
  auto fat = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  // 1. The forward's pieces: summaries, O_l unscaled with its denominators
  //    (alpha = 0 gives weight 1) and each query block's S_c (bf16) and z_c,
  //    the sparse branch with lse.
  sparge_status r = launch_summaries(K, V, s, dm, at(w.f.phik), fat(w.f.partial), fat(w.f.s_all), fat(w.f.z_all),
                                     fat(w.f.z_tile), st);
  if (r != SPARGE_OK) return r;
  cudaError_t e = cudaMemsetAsync(at(w.alpha0), 0, (size_t)s->H * 4, st);
  if (e != cudaSuccess) return cuda_status(e);
  int32_t* order = reinterpret_cast<int32_t*>(ws + w.f.order);
  e = launch_tile_order(kv_cnt, s, dm, &order, st);
  if (e != cudaSuccess) return cuda_status(e);
  r = launch_linear_out(Q, V, s, dm, kv_idx, kv_cnt, at(w.f.phik), fat(w.f.s_all), fat(w.f.z_all), fat(w.f.z_tile),
                        fat(w.alpha0), at(w.ol), st, fat(w.den), at(w.sc), fat(w.zc));
  if (r != SPARGE_OK) return r;
  r = launch_attn<D, false>(Q, K, V, s, dm, kv_idx, kv_cnt, at(w.os), fat(w.lse), nullptr, st, order);
  if (r != SPARGE_OK) return r;
  // 2. Row pass and dalpha.
  const int chunks = sla2_row_chunks(s->N);
  sla2_bwd_rows_kernel<D><<<(unsigned)(dm.BH * chunks), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(at(w.os)), static_cast<const __nv_bfloat16*>(at(w.ol)),
      static_cast<const __nv_bfloat16*>(dO), fat(w.den), alpha, s->H, s->N, chunks, fat(w.dsum), fat(w.cw),
      fat(w.fw), fat(w.ew), fat(w.dpart));
  sla2_dalpha_kernel<<<1, 128, 0, st>>>(fat(w.dpart), s->B, s->H, chunks, dalpha);
  // 3. G_all, g_all, g_tile, phi(Q) and c_i dO_i (the summary kernel on Q
  //    and dO with c_i, e_i).
  r = launch_summaries(Q, dO, s, dm, at(w.phiq), fat(w.f.partial), fat(w.g), fat(w.gall), fat(w.gtile), st,
                       fat(w.cw), fat(w.ew), at(w.cdo));
  if (r != SPARGE_OK) return r;
  // 4. Transposed mask.
  int32_t* q_idx = reinterpret_cast<int32_t*>(ws + w.qidx);
  int32_t* q_cnt = reinterpret_cast<int32_t*>(ws + w.qcnt);
  const int tsm = transpose_smem_bytes((int)dm.nqb);
  e = ensure_smem(mask_transpose_kernel, tsm, 10);
  if (e != cudaSuccess) return cuda_status(e);
  mask_transpose_kernel<<<(unsigned)(dm.BH * ceil_div(dm.nkb, kTrCols)), kTrCols, tsm, st>>>(
      kv_idx, kv_cnt, (int)dm.nqb, (int)dm.nkb, q_idx, q_cnt);
  // 5. dQ (sparse + linear), then dK and dV: sparse part into fp32 partials,
  //    linear part and the combination into bf16.
  CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv, mpk, msc, mpq64, mcdo;
  if (!make_map_bhnd(&mq, Q, dm.BH, s->N, D, kTileQ) || !make_map_bhnd(&mk, K, dm.BH, s->N, D, kTileK) ||
      !make_map_bhnd(&mv, V, dm.BH, s->N, D, kTileK) || !make_map_bhnd(&mdo, dO, dm.BH, s->N, D, kTileQ) ||
      !make_map_bhnd(&mdq, dQ, dm.BH, s->N, D, s->bq) || !make_map_bhnd(&mdk, dK, dm.BH, s->N, D, kTileK) ||
      !make_map_bhnd(&mdv, dV, dm.BH, s->N, D, kTileK) ||
      !make_map_bhnd(&mpk, at(w.f.phik), dm.BH, s->N, D, kTileK) ||
      !make_map_bhnd(&msc, at(w.sc), dm.BH * dm.nqb, D, D, kTileQ) ||
      !make_map_bhnd(&mpq64, at(w.phiq), dm.BH, s->N, D, 64) || !make_map_bhnd(&mcdo, at(w.cdo), dm.BH, s->N, D, 64))
    return SPARGE_ERR_CUDA;
  BwdParams p;
  p.lse = fat(w.lse);
  p.dsum = fat(w.dsum);
  p.N = s->N;
  p.nqb = (int)dm.nqb;
  p.nkb = (int)dm.nkb;
  p.bq = s->bq;
  p.bk = s->bk;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.scale = (float)(1.0 / std::sqrt((double)D));
  p.order = order;
  p.lst = kv_idx;
  p.cnt = kv_cnt;
  BwdLinParams lp;
  lp.alpha = alpha;
  lp.cw = fat(w.cw);
  lp.fw = fat(w.fw);
  lp.zc = fat(w.zc);
  lp.H = s->H;
  e = ensure_smem(attn_bwd_dq_kernel<D, true>, BwdQSmem<D, true>::kBytes, 14);
  if (e != cudaSuccess) return cuda_status(e);
  attn_bwd_dq_kernel<D, true><<<(unsigned)(dm.BH * dm.nqb), bwd_q_threads<true>(), BwdQSmem<D, true>::kBytes,
                                st>>>(
      mq, mk, mv, mdo, mdq, msc, p, lp);
  p.order = nullptr;
  p.lst = q_idx;
  p.cnt = q_cnt;
  BwdKVLin lk;
  lk.alpha = alpha;
  lk.dk_part = fat(w.dkp);
  lk.dv_part = fat(w.dvp);
  lk.H = s->H;
  const unsigned kgrid = (unsigned)(dm.BH * ceil_div(s->N, kTileK));
  e = ensure_smem(attn_bwd_dkdv_kernel<D, 1>, BwdKVSmem<D>::kBytes, 15);
  if (e != cudaSuccess) return cuda_status(e);
  attn_bwd_dkdv_kernel<D, 1><<<kgrid, kAttnThreads, BwdKVSmem<D>::kBytes, st>>>(mq, mk, mv, mdo, mdk, mdv, p, lk);
  LbParams lb;
  lb.q_idx = q_idx;
  lb.q_cnt = q_cnt;
  lb.g_all = fat(w.g);
  lb.g_vec = fat(w.gall);
  lb.g_tile = fat(w.gtile);
  lb.dk_part = fat(w.dkp);
  lb.dv_part = fat(w.dvp);
  lb.dK = static_cast<__nv_bfloat16*>(dK);
  lb.dV = static_cast<__nv_bfloat16*>(dV);
  lb.N = s->N;
  lb.ntiles = (int)ceil_div(s->N, 64);
  lb.nqb = (int)dm.nqb;
  lb.nkb = (int)dm.nkb;
  lb.bq = s->bq;
  lb.bk = s->bk;
  e = ensure_smem(linear_dkdv_kernel, LbSmem::kBytes, 18);
  if (e != cudaSuccess) return cuda_status(e);
  const int64_t kpairs = dm.BH * ceil_div(lb.ntiles, 2);  // two neighbouring key tiles per CTA
  linear_dkdv_kernel<<<(unsigned)kpairs, kLoThreads, LbSmem::kBytes, st>>>(mpq64, mcdo, mpk, mv, lb);
  return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// Scratch for sparge_mask_noalloc: a fixed array in device memory, part of
// the loaded module, so that entry point needs no allocation at all. Every
// device that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device. Host code may
// not use the array's name as an address; cudaGetSymbolAddress is called once
// per device (with that device current) and the result is cached.
sparge_status noalloc_scratch(uint8_t** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cuda_status(cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return cuda_status(e == cudaSuccess ? cudaErrorInvalidSymbol : e);
    addr[dev] = p;
  }
  *out = static_cast<uint8_t*>(addr[dev]);
  return SPARGE_OK;
}

}  // namespace

extern "C" {

size_t sparge_workspace_bytes(int op, const sparge_shape* shape) {
  Dims dm;
  if (check_shape(shape, &dm) != SPARGE_OK) return 0;
  switch (op) {
    case SPARGE_OP_MASK:
      return mask_ws(shape, dm).total;
    case SPARGE_OP_ATTN:
      return order_bytes(dm);
    case SPARGE_OP_SLA2:
      return shape->d == 128 ? sla2_ws(shape, dm).total : 0;
    case SPARGE_OP_ATTN_Q8:
      return shape->d == 128 ? q8_ws(shape, dm).total : 0;
    case SPARGE_OP_MASK_ROUTER:
      return router_ws(shape, dm).total;
    case SPARGE_OP_ATTN_BWD:
      return shape->d == 128 ? bwd_ws(shape, dm).total : 0;
    case SPARGE_OP_SLA2_BWD:
      return shape->d == 128 ? sla2_bwd_ws(shape, dm).total : 0;
    default:
      return 0;
  }
}

sparge_status sparge_mask(const void* Q, const void* K, const sparge_shape* shape, double topk_frac, double topp,
                          int32_t* kv_idx, int32_t* kv_cnt, float* row_thresh, float* probs, void* workspace,
                          size_t workspace_bytes, void* stream) {
  Dims dm;
  sparge_status st = check_shape(shape, &dm);
  if (st != SPARGE_OK) return st;
  if (!Q || !K || !kv_idx || !kv_cnt) return SPARGE_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || (probs && !aligned16(probs))) return SPARGE_ERR_INVALID_ARG;
  if (!(topk_frac >= 0.0 && topk_frac <= 1.0) || !(topp >= 0.0 && topp <= 1.0)) return SPARGE_ERR_INVALID_ARG;
  const size_t need = mask_ws(shape, dm).total;
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPARGE_ERR_WORKSPACE;
  int kc = 0;
  if (topk_frac > 0.0) {
    const double c = std::ceil(topk_frac * (double)dm.nkb - 1e-9);
    kc = (int)std::min<double>(std::max<double>(c, 0.0), (double)dm.nkb);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (shape->d == 64) return launch_mask<64>(Q, K, shape, dm, kc, topp, kv_idx, kv_cnt, row_thresh, probs, ws, s);
  return launch_mask<128>(Q, K, shape, dm, kc, topp, kv_idx, kv_cnt, row_thresh, probs, ws, s);
}

sparge_status sparge_mask_router(const void* Q, const void* K, const sparge_shape* shape, const float* Wq,
                                 const float* Wk, int dr, double topk_frac, double topp, int32_t* kv_idx,
                                 int32_t* kv_cnt, float* row_thresh, float* probs, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  Dims dm;
  sparge_status st = check_shape(shape, &dm);
  if (st != SPARGE_OK) return st;
  if (!Q || !K || !Wq || !Wk || !kv_idx || !kv_cnt) return SPARGE_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || (probs && !aligned16(probs))) return SPARGE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Wq) & 3u) || (reinterpret_cast<uintptr_t>(Wk) & 3u)) return SPARGE_ERR_INVALID_ARG;
  if (!(topk_frac >= 0.0 && topk_frac <= 1.0) || !(topp >= 0.0 && topp <= 1.0)) return SPARGE_ERR_INVALID_ARG;
  if (dr != 64 && dr != 128) return SPARGE_ERR_UNSUPPORTED;
  const RouterWs w = router_ws(shape, dm);
  if (workspace == nullptr || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPARGE_ERR_WORKSPACE;
  int kc = 0;
  if (topk_frac > 0.0) {
    const double c = std::ceil(topk_frac * (double)dm.nkb - 1e-9);
    kc = (int)std::min<double>(std::max<double>(c, 0.0), (double)dm.nkb);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* qhat = reinterpret_cast<double*>(ws + w.qhat);
  double* khat = reinterpret_cast<double*>(ws + w.khat);
  if (shape->d == 64)
    return launch_mask<64>(Q, K, shape, dm, kc, topp, kv_idx, kv_cnt, row_thresh, probs, ws, s, Wq, Wk, dr, qhat,
                           khat);
  return launch_mask<128>(Q, K, shape, dm, kc, topp, kv_idx, kv_cnt, row_thresh, probs, ws, s, Wq, Wk, dr, qhat,
                          khat);
}

sparge_status sparge_mask_noalloc(const void* Q, const void* K, const sparge_shape* shape, double topk_frac,
                                  double topp, int32_t* kv_idx, int32_t* kv_cnt, float* row_thresh, float* probs,
                                  void* stream) {
  Dims dm;
  sparge_status st = check_shape(shape, &dm);
  if (st != SPARGE_OK) return st;
  if (!Q || !K || !kv_idx || !kv_cnt) return SPARGE_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || (probs && !aligned16(probs))) return SPARGE_ERR_INVALID_ARG;
  if (!(topk_frac >= 0.0 && topk_frac <= 1.0) || !(topp >= 0.0 && topp <= 1.0)) return SPARGE_ERR_INVALID_ARG;
  // Pooled Q and K and the score rows live in the scratch.
  if (mask_ws(shape, dm).total > kNoAllocScratchBytes) return SPARGE_ERR_WORKSPACE;
  uint8_t* ws = nullptr;
  st = noalloc_scratch(&ws);
  if (st != SPARGE_OK) return st;
  int kc = 0;
  if (topk_frac > 0.0) {
    const double c = std::ceil(topk_frac * (double)dm.nkb - 1e-9);
    kc = (int)std::min<double>(std::max<double>(c, 0.0), (double)dm.nkb);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (shape->d == 64) return launch_mask<64>(Q, K, shape, dm, kc, topp, kv_idx, kv_cnt, row_thresh, probs, ws, s);
  return launch_mask<128>(Q, K, shape, dm, kc, topp, kv_idx, kv_cnt, row_thresh, probs, ws, s);
}

sparge_status sparge_attn_fwd(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                              const int32_t* kv_idx, const int32_t* kv_cnt, void* O, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream) {
  Dims dm;
  sparge_status st = check_shape(shape, &dm);
  if (st != SPARGE_OK) return st;
  if (!Q || !K || !V || !O || !kv_idx || !kv_cnt) return SPARGE_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SPARGE_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < order_bytes(dm) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPARGE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* order = static_cast<int32_t*>(workspace);
  cudaError_t e = launch_tile_order(kv_cnt, shape, dm, &order, s);
  if (e != cudaSuccess) return cuda_status(e);
  if (shape->d == 64)
    return launch_attn<64, false>(Q, K, V, shape, dm, kv_idx, kv_cnt, O, lse, nullptr, s, order);
  return launch_attn<128, false>(Q, K, V, shape, dm, kv_idx, kv_cnt, O, lse, nullptr, s, order);
}

sparge_status sparge_attn_fwd_q8(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                                 const int32_t* kv_idx, const int32_t* kv_cnt, void* O, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  Dims dm;
  sparge_status st = check_shape(shape, &dm);
  if (st != SPARGE_OK) return st;
  if (!Q || !K || !V || !O || !kv_idx || !kv_cnt) return SPARGE_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SPARGE_ERR_INVALID_ARG;
  if (shape->d != 128 || dm.BH > 65535) return SPARGE_ERR_UNSUPPORTED;
  const Q8Ws w = q8_ws(shape, dm);
  if (workspace == nullptr || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPARGE_ERR_WORKSPACE;
  return launch_q8(Q, K, V, shape, dm, kv_idx, kv_cnt, O, static_cast<uint8_t*>(workspace),
                   static_cast<cudaStream_t>(stream));
}

sparge_status sla2_attn_fwd(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                            const int32_t* kv_idx, const int32_t* kv_cnt, const float* alpha, void* O,
                            void* workspace, size_t workspace_bytes, void* stream) {
  Dims dm;
  sparge_status st = check_shape(shape, &dm);
  if (st != SPARGE_OK) return st;
  if (!Q || !K || !V || !O || !kv_idx || !kv_cnt || !alpha) return SPARGE_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SPARGE_ERR_INVALID_ARG;
  if (shape->d != 128 || dm.BH > 65535) return SPARGE_ERR_UNSUPPORTED;
  const Sla2Ws w = sla2_ws(shape, dm);
  if (workspace == nullptr || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPARGE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* phik = ws + w.phik;
  float* s_all = reinterpret_cast<float*>(ws + w.s_all);
  float* z_all = reinterpret_cast<float*>(ws + w.z_all);
  float* z_tile = reinterpret_cast<float*>(ws + w.z_tile);
  float* partial = reinterpret_cast<float*>(ws + w.partial);
  int32_t* order = reinterpret_cast<int32_t*>(ws + w.order);
  cudaError_t e = launch_tile_order(kv_cnt, shape, dm, &order, s);
  if (e != cudaSuccess) return cuda_status(e);
  st = launch_summaries(K, V, shape, dm, phik, partial, s_all, z_all, z_tile, s);
  if (st != SPARGE_OK) return st;
  st = launch_linear_out(Q, V, shape, dm, kv_idx, kv_cnt, phik, s_all, z_all, z_tile, alpha, O, s);
  if (st != SPARGE_OK) return st;
  return launch_attn<128, true>(Q, K, V, shape, dm, kv_idx, kv_cnt, O, nullptr, alpha, s, order);
}

sparge_status sparge_attn_bwd(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                              const int32_t* kv_idx, const int32_t* kv_cnt, const void* O, const float* lse,
                              const void* dO, void* dQ, void* dK, void* dV, void* workspace, size_t workspace_bytes,
                              void* stream) {
  Dims dm;
  sparge_status st = check_shape(shape, &dm);
  if (st != SPARGE_OK) return st;
  if (!Q || !K || !V || !O || !lse || !dO || !dQ || !dK || !dV || !kv_idx || !kv_cnt) return SPARGE_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(dQ) ||
      !aligned16(dK) || !aligned16(dV))
    return SPARGE_ERR_INVALID_ARG;
  if (shape->d != 128 || transpose_smem_bytes((int)dm.nqb) > kMaxTransposeSmem) return SPARGE_ERR_UNSUPPORTED;
  if ((int64_t)dm.BH * ceil_div(shape->N, kTileK) > INT32_MAX) return SPARGE_ERR_UNSUPPORTED;
  const BwdWs w = bwd_ws(shape, dm);
  if (workspace == nullptr || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPARGE_ERR_WORKSPACE;
  return launch_bwd(Q, K, V, shape, dm, kv_idx, kv_cnt, O, lse, dO, dQ, dK, dV, static_cast<uint8_t*>(workspace),
                    static_cast<cudaStream_t>(stream));
}

sparge_status sla2_attn_bwd(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                            const int32_t* kv_idx, const int32_t* kv_cnt, const float* alpha, const void* dO, void* dQ,
                            void* dK, void* dV, float* dalpha, void* workspace, size_t workspace_bytes, void* stream) {
  Dims dm;
  sparge_status st = check_shape(shape, &dm);
  if (st != SPARGE_OK) return st;
  if (!Q || !K || !V || !dO || !dQ || !dK || !dV || !dalpha || !kv_idx || !kv_cnt || !alpha)
    return SPARGE_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dO) || !aligned16(dQ) || !aligned16(dK) ||
      !aligned16(dV))
    return SPARGE_ERR_INVALID_ARG;
  if (shape->d != 128 || dm.BH > 65535 || transpose_smem_bytes((int)dm.nqb) > kMaxTransposeSmem)
    return SPARGE_ERR_UNSUPPORTED;
  if ((int64_t)dm.BH * ceil_div(shape->N, kTileK) > INT32_MAX) return SPARGE_ERR_UNSUPPORTED;
  const Sla2BwdWs w = sla2_bwd_ws(shape, dm);
  if (workspace == nullptr || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPARGE_ERR_WORKSPACE;
  return launch_sla2_bwd(Q, K, V, shape, dm, kv_idx, kv_cnt, alpha, dO, dQ, dK, dV, dalpha,
                         static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
}

sparge_status sparge_selftest_wait(int32_t limit_us, int32_t* gave_up, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return SPARGE_ERR_INVALID_ARG;
  if (gave_up != nullptr && (reinterpret_cast<uintptr_t>(gave_up) & 3u)) return SPARGE_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>((unsigned long long)limit_us * 1000ull,
                                                                         gave_up);
  return cuda_status(cudaGetLastError());
}

sparge_status sparge_device_status(void* stream, int32_t* code) {
  if (code == nullptr) return SPARGE_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_status(e);
  unsigned int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, sparge::g_device_error, sizeof v);
  if (e != cudaSuccess) return cuda_status(e);
  e = cudaMemcpyToSymbol(sparge::g_device_error, &zero, sizeof zero);
  if (e != cudaSuccess) return cuda_status(e);
  *code = (int32_t)v;
  return v ? SPARGE_ERR_DEVICE_TIMEOUT : SPARGE_OK;
}

const char* sparge_status_string(sparge_status status) {
  switch (status) {
    case SPARGE_OK: return "ok";
    case SPARGE_ERR_INVALID_ARG: return "invalid argument";
    case SPARGE_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case SPARGE_ERR_WORKSPACE: return "workspace missing or too small";
    case SPARGE_ERR_CUDA: return "CUDA error";
    case SPARGE_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

}  // extern "C"
