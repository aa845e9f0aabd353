// Block-mask kernels: pooling, pooled block importance and hybrid Top-k /
// Top-p selection (SpargeAttention2 article, arXiv:2602.13515, sections 1
// and 4: a pooling pre-filter scores blocks cheaply, a hybrid Top-k / Top-p
// rule selects them, and the result is a block-level mask).
//
// The selection is an integer decision taken from floating point. These
// kernels fix the operation order so the decision is reproducible:
//   pool : fp32 sum over a block's valid rows in row order, then divide by
//          the number of valid rows;
//   score: fp32 fused multiply-add over channels 0..d-1 in order, then times
//          (float)(1/sqrt(d));
//   prob : expf(z - rowmax) / rowsum;
//   order: probability descending, block index ascending for ties;
//   Top-p: running sum of the ordered probabilities in double, first prefix
//          whose sum is >= p.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparge {

// ----------------------------------------------------------------------------
// Pool: out[g, c] = mean over the valid rows of block g of X[., c].
// X: [BH, N, d] bf16. Each thread owns 8 consecutive channels of one block and
// walks its rows in order (16-byte loads, 8 fp32 accumulators).
// ----------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const __nv_bfloat16* __restrict__ Q,
                                                   const __nv_bfloat16* __restrict__ K, int64_t BH, int N, int bq,
                                                   int bk, int64_t q_ctas, float* __restrict__ qbar,
                                                   float* __restrict__ kbar) {
  constexpr int TPB = D / 8;            // threads per block-row
  constexpr int BLOCKS_PER_CTA = 128 / TPB;
  // CTAs [0, q_ctas) pool Q blocks, the rest pool K blocks.
  const bool is_q = blockIdx.x < q_ctas;
  const __nv_bfloat16* X = is_q ? Q : K;
  float* out = is_q ? qbar : kbar;
  const int blk = is_q ? bq : bk;
  const int64_t cta = is_q ? blockIdx.x : blockIdx.x - q_ctas;
  const int nb = (N + blk - 1) / blk;
  const int64_t g = cta * BLOCKS_PER_CTA + threadIdx.x / TPB;  // flat (bh, block)
  if (g >= BH * nb) return;
  const int c8 = (threadIdx.x % TPB) * 8;
  const int64_t bh = g / nb;
  const int I = (int)(g % nb);
  const int r0 = I * blk;
  const int r1 = min(N, r0 + blk);
  const uint4* src = reinterpret_cast<const uint4*>(X + (bh * N + r0) * D + c8);
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
  const int rows = r1 - r0;
  auto add_row = [&](uint4 v) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __bfloat1622float2(h[j]);
      acc[2 * j] = __fadd_rn(acc[2 * j], f.x);
      acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], f.y);
    }
  };
  int r = 0;
  for (; r + 16 <= rows; r += 16) {  // 16 rows in flight per thread, added in order
    uint4 v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = __ldg(src + (int64_t)(r + u) * (D / 8));
#pragma unroll
    for (int u = 0; u < 16; ++u) add_row(v[u]);
  }
  for (; r < rows; ++r) add_row(__ldg(src + (int64_t)r * (D / 8)));
  const float cnt = (float)rows;
  float4* dst = reinterpret_cast<float4*>(out + g * D + c8);
  dst[0] = make_float4(__fdiv_rn(acc[0], cnt), __fdiv_rn(acc[1], cnt), __fdiv_rn(acc[2], cnt),
                       __fdiv_rn(acc[3], cnt));
  dst[1] = make_float4(__fdiv_rn(acc[4], cnt), __fdiv_rn(acc[5], cnt), __fdiv_rn(acc[6], cnt),
                       __fdiv_rn(acc[7], cnt));
}

// ----------------------------------------------------------------------------
// Learnt router (SLA2 article, arXiv:2602.12675, section 2: a router with two
// learnable projection matrices maps the query and key features into a space
// suited to the routing decision): pooled block vectors are projected,
//   out[g, c'] = sum_c in[g, c] * W_h[c, c'],  W_h = W + h * D * DR,
// each entry a sequential fused multiply-add over c in order. One CTA = up to
// 32 pooled blocks of one (b, h) (CTA = bh * chunks + chunk), so every row uses
// the same W_h; thread t computes column t % DR for rows t / DR, t / DR + G,
// ... (G = 128 / DR row groups), reading each W_h entry once per CTA.
// ----------------------------------------------------------------------------
constexpr int kProjRows = 32;

template <int D, int DR>
__global__ void __launch_bounds__(128) project_kernel(const float* __restrict__ in, int64_t nb, int H,
                                                      const float* __restrict__ W, float* __restrict__ out) {
  constexpr int G = 128 / DR, RPT = kProjRows / G;  // row groups, rows per thread
  __shared__ __align__(16) float sx[kProjRows][D];
  const int64_t chunks = (nb + kProjRows - 1) / kProjRows;
  const int64_t bh = blockIdx.x / chunks;
  const int64_t r0 = (blockIdx.x % chunks) * kProjRows;
  const int nr = (int)(nb - r0 < kProjRows ? nb - r0 : kProjRows);
  const float* src = in + (bh * nb + r0) * D;
  for (int e = threadIdx.x; e < kProjRows * (D / 4); e += 128) {
    const int r = e / (D / 4), c4 = (e % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < nr) v = *reinterpret_cast<const float4*>(src + (int64_t)r * D + c4);
    *reinterpret_cast<float4*>(&sx[r][c4]) = v;
  }
  __syncthreads();
  const int col = threadIdx.x % DR, grp = threadIdx.x / DR;
  const float* w = W + (bh % H) * D * DR + col;
  float acc[RPT];
#pragma unroll
  for (int k = 0; k < RPT; ++k) acc[k] = 0.0f;
#pragma unroll 4
  for (int c = 0; c < D; ++c) {
    const float wc = __ldg(w + c * DR);
#pragma unroll
    for (int k = 0; k < RPT; ++k) acc[k] = __fmaf_rn(sx[grp + k * G][c], wc, acc[k]);
  }
  float* dst = out + (bh * nb + r0) * DR + col;
#pragma unroll
  for (int k = 0; k < RPT; ++k)
    if (grp + k * G < nr) dst[(int64_t)(grp + k * G) * DR] = acc[k];
}

// ----------------------------------------------------------------------------
// Scaled scores z[I, J] = (q̄_I . k̄_J) * (float)(1/sqrt(d)). One CTA = 32
// query-block rows x 64 key blocks of one (b,h); each thread owns 4 rows x 4
// key blocks (8 shared-memory vector loads per 64 fused multiply-adds) and
// runs their fused multiply-add chains over channels in order.
// Pooled K rows are padded by 4 floats in shared memory so that the 16-byte
// loads of different rows fall in different banks. The row softmax happens
// in the selection kernel, which reads the whole row anyway.
// ----------------------------------------------------------------------------
constexpr int kScoreRows = 32;
constexpr int kScoreTileJ = 64;

template <int D>
__host__ __device__ constexpr int score_smem_bytes() {
  return (kScoreRows * D + kScoreTileJ * (D + 4)) * 4;
}

template <int D>
__global__ void __launch_bounds__(128) score_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                                                    int nqb, int nkb, float scale, float* __restrict__ Z) {
  extern __shared__ __align__(16) float sm[];
  float* sq = sm;                                   // [32][D]
  float* sk = sq + kScoreRows * D;                  // [64][D+4]
  const int tiles_q = (nqb + kScoreRows - 1) / kScoreRows;
  const int tiles_j = (nkb + kScoreTileJ - 1) / kScoreTileJ;
  const int64_t cta = blockIdx.x;
  const int64_t bh = cta / ((int64_t)tiles_q * tiles_j);
  const int rem = (int)(cta % ((int64_t)tiles_q * tiles_j));
  const int I0 = (rem / tiles_j) * kScoreRows;
  const int J0 = (rem % tiles_j) * kScoreTileJ;
  const int nrows = min(kScoreRows, nqb - I0);
  const int nj = min(kScoreTileJ, nkb - J0);
  const int tid = threadIdx.x;
  // Every load of the tile is issued before the first store (unrolled), so
  // the CTA waits for one round trip to L2 rather than one per 128 vectors.
  constexpr int kQVec = kScoreRows * (D / 4) / 128, kKVec = kScoreTileJ * (D / 4) / 128;
  float4 vq[kQVec], vk[kKVec];
#pragma unroll
  for (int u = 0; u < kQVec; ++u) {
    const int e = tid + 128 * u, i = e / (D / 4), c4 = (e % (D / 4)) * 4;
    vq[u] = i < nrows ? *reinterpret_cast<const float4*>(qbar + (bh * nqb + I0 + i) * D + c4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int u = 0; u < kKVec; ++u) {
    const int e = tid + 128 * u, j = e / (D / 4), c4 = (e % (D / 4)) * 4;
    vk[u] = j < nj ? *reinterpret_cast<const float4*>(kbar + (bh * nkb + J0 + j) * D + c4)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int u = 0; u < kQVec; ++u) {
    const int e = tid + 128 * u, i = e / (D / 4), c4 = (e % (D / 4)) * 4;
    *reinterpret_cast<float4*>(sq + i * D + c4) = vq[u];
  }
#pragma unroll
  for (int u = 0; u < kKVec; ++u) {
    const int e = tid + 128 * u, j = e / (D / 4), c4 = (e % (D / 4)) * 4;
    *reinterpret_cast<float4*>(sk + j * (D + 4) + c4) = vk[u];
  }
  __syncthreads();
  const int jl = tid % 16;   // key blocks jl, jl+16, jl+32, jl+48 of the tile
  const int ig = tid / 16;   // query rows 4*ig .. 4*ig+3
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
#pragma unroll 2
  for (int c = 0; c < D; c += 4) {
    float4 q[4], k[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) q[a] = *reinterpret_cast<const float4*>(sq + (4 * ig + a) * D + c);
#pragma unroll
    for (int b = 0; b < 4; ++b) k[b] = *reinterpret_cast<const float4*>(sk + (jl + 16 * b) * (D + 4) + c);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        acc[a][b] = __fmaf_rn(q[a].x, k[b].x, acc[a][b]);
        acc[a][b] = __fmaf_rn(q[a].y, k[b].y, acc[a][b]);
        acc[a][b] = __fmaf_rn(q[a].z, k[b].z, acc[a][b]);
        acc[a][b] = __fmaf_rn(q[a].w, k[b].w, acc[a][b]);
      }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = jl + 16 * b;
      if (j < nj && 4 * ig + a < nrows)
        Z[(bh * nqb + I0 + 4 * ig + a) * (int64_t)nkb + J0 + j] = __fmul_rn(acc[a][b], scale);
    }
}

// ----------------------------------------------------------------------------
// Softmax + selection. One CTA of 256 threads per query-block row:
//   0. P = expf(z - rowmax) / rowsum, the row sum taken as 32 interleaved
//      partial sums (partial l adds the terms l, l+32, ... in turn) combined
//      pairwise at distances 16, 8, 4, 2, 1; P is written back over z.
//   1. Key of block j = the bit pattern of P_j (ordered like P for P >= 0);
//      weight of block j = P_j in 64-bit fixed point (2^62 = 1), exact for
//      P >= 2^-39 and truncated below, so running sums are exact integers
//      whatever the summation order.
//   2. Top-p: radix select (four 8-bit digits, most significant first) of the
//      key at which the descending running weight first reaches p; ties at
//      that key all weigh the same, so the count needed follows by division.
//   3. m = max(kc, pc, 1). When m = pc the m-th largest key is the Top-p key
//      just found; otherwise a second radix select (counting) finds it.
//      Blocks above it are kept, and of the blocks at it the lowest indices
//      fill the remaining places.
//   4. Kept flags are compacted in block order (block-wide scans) into the
//      ascending kept list.
// ----------------------------------------------------------------------------
constexpr int kSelectThreads = 256;
constexpr int kSelectMaxPer = 16;  // blocks per thread: Nkb <= 4096

__host__ __device__ constexpr int select_smem_bytes(int nkb) {
  // z / P row (4 B per block) + keys (4 B per block) + histograms + scratch
  return ((nkb + 3) / 4 * 4) * 8 + 256 * 12 + 1024;
}

__device__ __forceinline__ unsigned long long p_fixed62(unsigned int bits) {
  const int e = (int)((bits >> 23) & 0xFFu);
  if (e == 0) return 0ull;  // zero or subnormal: below 2^-126
  const unsigned long long mant = (unsigned long long)((bits & 0x7FFFFFu) | 0x800000u);
  const int sh = e - 88;    // value = mant * 2^(e - 150); times 2^62
  if (sh >= 0) return mant << sh;
  return (-sh >= 64) ? 0ull : (mant >> (-sh));
}

// Block-wide exclusive scan of one int per thread (256 threads).
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[wid] = x;
  __syncthreads();
  int base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kSelectThreads / 32; ++w) {
    const int s = scratch[w];
    if (w < wid) base += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return base + x - v;
}

// One radix-select pass. Candidates are keys whose bits above `shift + 8`
// equal `prefix`. Buckets are digits (key >> shift) & 255 taken from the top
// (largest key) down. With weights (by_weight) it finds the bucket where the
// running weight, starting from *above_w, first reaches `target`; otherwise
// the bucket where the running count, starting from *above_c, first reaches
// it. Updates prefix / above_w / above_c. Called by all 256 threads.
__device__ void radix_pass(const unsigned int* keys, int nkb, int shift, unsigned int hi_mask, bool by_weight,
                           unsigned long long target, unsigned int* prefix, unsigned long long* above_w,
                           int* above_c, unsigned int* hcnt, unsigned long long* hsum, unsigned int* bc) {
  const int tid = threadIdx.x;
  hcnt[tid] = 0u;
  hsum[tid] = 0ull;
  __syncthreads();
  const unsigned int pre = *prefix;
  for (int j = tid; j < nkb; j += kSelectThreads) {
    const unsigned int k = keys[j];
    if ((k & hi_mask) == pre) {
      const unsigned int d = (k >> shift) & 255u;
      atomicAdd(&hcnt[d], 1u);
      if (by_weight) atomicAdd(&hsum[d], p_fixed62(k));
    }
  }
  __syncthreads();
  if (tid < 32) {
    // Lane l owns buckets 255-8l ... 248-8l (descending).
    unsigned long long lw = 0ull;
    unsigned int lc = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int b = 255 - 8 * tid - i;
      lw += hsum[b];
      lc += hcnt[b];
    }
    unsigned long long xw = lw;
    unsigned int xc = lc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long yw = __shfl_up_sync(0xffffffffu, xw, o);
      const unsigned int yc = __shfl_up_sync(0xffffffffu, xc, o);
      if (tid >= o) {
        xw += yw;
        xc += yc;
      }
    }
    const unsigned long long aw = *above_w + xw - lw;  // running value before this lane's buckets
    const unsigned int ac = (unsigned int)*above_c + xc - lc;
    const bool reach = by_weight ? (aw + lw >= target) : ((unsigned long long)(ac + lc) >= target);
    const unsigned int ballot = __ballot_sync(0xffffffffu, reach);
    const int first = __ffs(ballot) - 1;  // first lane (from the top) whose buckets reach the target
    if (tid == first) {
      unsigned long long w = aw;
      unsigned int c = ac;
      int bsel = 255 - 8 * tid - 7;
      for (int i = 0; i < 8; ++i) {
        const int b = 255 - 8 * tid - i;
        const bool hit = by_weight ? (w + hsum[b] >= target) : ((unsigned long long)(c + hcnt[b]) >= target);
        if (hit) {
          bsel = b;
          break;
        }
        w += hsum[b];
        c += hcnt[b];
      }
      bc[0] = (unsigned int)bsel;
      bc[1] = c;
      *reinterpret_cast<unsigned long long*>(bc + 2) = w;
    }
  }
  __syncthreads();
  *prefix = pre | (bc[0] << shift);
  *above_c = (int)bc[1];
  *above_w = *reinterpret_cast<unsigned long long*>(bc + 2);
  __syncthreads();
}

__global__ void __launch_bounds__(kSelectThreads) select_kernel(float* __restrict__ P, int64_t rows, int nkb,
                                                                 int kc, double topp, int32_t* __restrict__ kv_idx,
                                                                 int32_t* __restrict__ kv_cnt,
                                                                 float* __restrict__ row_thresh) {
  extern __shared__ __align__(16) unsigned char smraw[];
  const int npad = (nkb + 3) / 4 * 4;
  float* ev = reinterpret_cast<float*>(smraw);                                  // [npad]
  unsigned int* keys = reinterpret_cast<unsigned int*>(smraw + npad * 4);        // [npad]
  unsigned long long* hsum = reinterpret_cast<unsigned long long*>(smraw + npad * 8);  // [256]
  unsigned int* hcnt = reinterpret_cast<unsigned int*>(smraw + npad * 8 + 2048);       // [256]
  unsigned int* bc = hcnt + 256;                                                  // [4]
  float* red = reinterpret_cast<float*>(bc + 4);                                  // [16]
  int* scratch = reinterpret_cast<int*>(red + 16);                                // [8]
  const int64_t row = blockIdx.x;
  if (row >= rows) return;
  const int tid = threadIdx.x;
  float* prow = P + row * (int64_t)nkb;

  // 0. Row softmax.
  float mx = -INFINITY;
  for (int j = tid; j < nkb; j += kSelectThreads) {
    const float z = prow[j];
    ev[j] = z;
    mx = fmaxf(mx, z);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < kSelectThreads / 32; ++w) mx = fmaxf(mx, red[w]);
  for (int j = tid; j < nkb; j += kSelectThreads) ev[j] = expf(__fsub_rn(ev[j], mx));
  __syncthreads();
  if (tid < 32) {
    float part = 0.0f;
    for (int j = tid; j < nkb; j += 32) part = __fadd_rn(part, ev[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part = __fadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
    if (tid == 0) red[8] = part;
  }
  __syncthreads();
  const float rsum = red[8];
  for (int j = tid; j < nkb; j += kSelectThreads) {
    const float pj = __fdiv_rn(ev[j], rsum);
    prow[j] = pj;
    keys[j] = __float_as_uint(pj);
  }
  __syncthreads();

  // 2. Top-p count.
  int pc = 0;
  unsigned int p_key = 0u;  // key of the pc-th largest block, when the Top-p select ran
  int p_above = 0;          // blocks above that key
  bool have_p = false;
  if (topp > 0.0) {
    const unsigned long long target = (unsigned long long)ceil(topp * 4611686018427387904.0);  // p * 2^62
    unsigned long long tot = 0ull;  // total weight (exact integer sum)
    for (int j = tid; j < nkb; j += kSelectThreads) tot += p_fixed62(keys[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    if ((tid & 31) == 0) hsum[tid >> 5] = tot;
    __syncthreads();
    tot = 0ull;
#pragma unroll
    for (int w = 0; w < kSelectThreads / 32; ++w) tot += hsum[w];
    __syncthreads();
    if (tot < target) {
      pc = nkb;  // never reached
    } else {
      unsigned int prefix = 0u;
      unsigned long long above_w = 0ull;
      int above_c = 0;
      for (int shift = 24; shift >= 0; shift -= 8) {
        const unsigned int hi_mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
        radix_pass(keys, nkb, shift, hi_mask, true, target, &prefix, &above_w, &above_c, hcnt, hsum, bc);
      }
      // All blocks with key == prefix weigh the same.
      const unsigned long long wt = p_fixed62(prefix);
      const unsigned long long need = target - above_w;  // > 0 by construction
      const unsigned long long c = wt ? (need + wt - 1) / wt : 0ull;
      pc = above_c + (int)c;
      p_key = prefix;
      p_above = above_c;
      have_p = true;
    }
  }
  const int m = min(nkb, max(max(kc, pc), 1));

  // 3. Key of the m-th largest block, and how many of its ties are kept.
  unsigned int tkey = p_key;
  int above_m = p_above;
  if (!(have_p && m == pc)) {
    unsigned int prefix = 0u;
    unsigned long long above_w = 0ull;
    int above_c = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
      const unsigned int hi_mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
      radix_pass(keys, nkb, shift, hi_mask, false, (unsigned long long)m, &prefix, &above_w, &above_c, hcnt, hsum,
                 bc);
    }
    tkey = prefix;
    above_m = above_c;
  }
  const int ties_kept = m - above_m;

  // 4. Compaction in block order: each thread owns a contiguous chunk.
  const int per = (nkb + kSelectThreads - 1) / kSelectThreads;
  const int j0 = min(nkb, tid * per), j1 = min(nkb, j0 + per);
  int nt = 0;
  for (int j = j0; j < j1; ++j) nt += keys[j] == tkey;
  int tie_tot;
  int tie_rank = block_excl_scan(nt, scratch, &tie_tot);
  int nk = 0;
  {
    int tr = tie_rank;
    for (int j = j0; j < j1; ++j) {
      const unsigned int k = keys[j];
      if (k > tkey || (k == tkey && tr++ < ties_kept)) ++nk;
    }
  }
  int kept_tot;
  int pos = block_excl_scan(nk, scratch, &kept_tot);
  int32_t* out = kv_idx + row * (int64_t)nkb;
  {
    int tr = tie_rank;
    for (int j = j0; j < j1; ++j) {
      const unsigned int k = keys[j];
      if (k > tkey || (k == tkey && tr++ < ties_kept)) out[pos++] = j;
    }
  }
  if (tid == 0) {
    kv_cnt[row] = m;
    if (row_thresh) row_thresh[row] = __uint_as_float(tkey);
  }
}

// ----------------------------------------------------------------------------
// The same selection with one warp per row (eight rows per CTA), for rows of
// at most kSelWarpMaxNkb blocks: every step is the arithmetic of
// select_kernel (the softmax's 32 interleaved partial sums are exactly one
// warp's lanes; the running weights are exact integers; the radix passes
// walk the same 8-bit digits), but the row's steps synchronise with warp
// barriers instead of block barriers. Each warp owns its row's P (then keys)
// and a 256-bucket histogram in shared memory.
// ----------------------------------------------------------------------------
constexpr int kSelWarpRows = 8;
constexpr int kSelWarpMaxNkb = 2048;

__host__ __device__ constexpr int select_warp_bytes(int nkb) { return (nkb + 3) / 4 * 16 + 256 * 12 + 16; }
__host__ __device__ constexpr int select_warp_smem_bytes(int nkb) { return kSelWarpRows * select_warp_bytes(nkb); }

// One radix pass of the warp version (see radix_pass): returns the selected
// digit and updates prefix / above_w / above_c; called by all 32 lanes.
__device__ __forceinline__ void radix_pass_warp(const unsigned int* keys, int nkb, int shift, unsigned int hi_mask,
                                                bool by_weight, unsigned long long target, unsigned int* prefix,
                                                unsigned long long* above_w, int* above_c, unsigned int* hcnt,
                                                unsigned long long* hsum) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    hcnt[lane * 8 + i] = 0u;
    hsum[lane * 8 + i] = 0ull;
  }
  __syncwarp();
  const unsigned int pre = *prefix;
  for (int j = lane; j < nkb; j += 32) {
    const unsigned int k = keys[j];
    if ((k & hi_mask) == pre) {
      const unsigned int d = (k >> shift) & 255u;
      atomicAdd(&hcnt[d], 1u);
      if (by_weight) atomicAdd(&hsum[d], p_fixed62(k));
    }
  }
  __syncwarp();
  // Lane l owns buckets 255-8l ... 248-8l (descending).
  unsigned long long lw = 0ull;
  unsigned int lc = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int b = 255 - 8 * lane - i;
    lw += hsum[b];
    lc += hcnt[b];
  }
  unsigned long long xw = lw;
  unsigned int xc = lc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long yw = __shfl_up_sync(0xffffffffu, xw, o);
    const unsigned int yc = __shfl_up_sync(0xffffffffu, xc, o);
    if (lane >= o) {
      xw += yw;
      xc += yc;
    }
  }
  const unsigned long long aw = *above_w + xw - lw;
  const unsigned int ac = (unsigned int)*above_c + xc - lc;
  const bool reach = by_weight ? (aw + lw >= target) : ((unsigned long long)(ac + lc) >= target);
  const unsigned int ballot = __ballot_sync(0xffffffffu, reach);
  const int first = __ffs(ballot) - 1;
  unsigned long long w = aw;
  unsigned int c = ac;
  int bsel = 255 - 8 * lane - 7;
  if (lane == first) {
    for (int i = 0; i < 8; ++i) {
      const int b = 255 - 8 * lane - i;
      const bool hit = by_weight ? (w + hsum[b] >= target) : ((unsigned long long)(c + hcnt[b]) >= target);
      if (hit) {
        bsel = b;
        break;
      }
      w += hsum[b];
      c += hcnt[b];
    }
  }
  bsel = __shfl_sync(0xffffffffu, bsel, first);
  c = __shfl_sync(0xffffffffu, c, first);
  w = __shfl_sync(0xffffffffu, w, first);
  *prefix = pre | ((unsigned int)bsel << shift);
  *above_c = (int)c;
  *above_w = w;
  __syncwarp();
}

__global__ void __launch_bounds__(kSelWarpRows * 32) select_warp_kernel(float* __restrict__ P, int64_t rows, int nkb,
                                                                        int kc, double topp,
                                                                        int32_t* __restrict__ kv_idx,
                                                                        int32_t* __restrict__ kv_cnt,
                                                                        float* __restrict__ row_thresh) {
  extern __shared__ __align__(16) unsigned char smraw[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * kSelWarpRows + wid;
  if (row >= rows) return;  // whole warps only: no block barrier follows
  unsigned char* mine = smraw + wid * select_warp_bytes(nkb);
  float* ev = reinterpret_cast<float*>(mine);                                      // [nkb], then the keys
  unsigned int* keys = reinterpret_cast<unsigned int*>(mine);
  unsigned long long* hsum = reinterpret_cast<unsigned long long*>(mine + (nkb + 3) / 4 * 16);  // [256]
  unsigned int* hcnt = reinterpret_cast<unsigned int*>(hsum + 256);                // [256]
  float* prow = P + row * (int64_t)nkb;

  // 0. Row softmax: max, exponentials, lane l's partial sum over l, l+32, ...
  float mx = -INFINITY;
  for (int j = lane; j < nkb; j += 32) {
    const float z = prow[j];
    ev[j] = z;
    mx = fmaxf(mx, z);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float part = 0.0f;
  for (int j = lane; j < nkb; j += 32) {
    const float e = expf(__fsub_rn(ev[j], mx));
    ev[j] = e;
    part = __fadd_rn(part, e);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part = __fadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
  const float rsum = part;
  unsigned long long tot = 0ull;  // total weight (exact integer sum)
  for (int j = lane; j < nkb; j += 32) {
    const float pj = __fdiv_rn(ev[j], rsum);
    prow[j] = pj;
    keys[j] = __float_as_uint(pj);
    tot += p_fixed62(__float_as_uint(pj));
  }
  __syncwarp();
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);

  // 2. Top-p count.
  int pc = 0;
  unsigned int p_key = 0u;
  int p_above = 0;
  bool have_p = false;
  if (topp > 0.0) {
    const unsigned long long target = (unsigned long long)ceil(topp * 4611686018427387904.0);  // p * 2^62
    if (tot < target) {
      pc = nkb;
    } else {
      unsigned int prefix = 0u;
      unsigned long long above_w = 0ull;
      int above_c = 0;
      for (int shift = 24; shift >= 0; shift -= 8) {
        const unsigned int hi_mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
        radix_pass_warp(keys, nkb, shift, hi_mask, true, target, &prefix, &above_w, &above_c, hcnt, hsum);
      }
      const unsigned long long wt = p_fixed62(prefix);
      const unsigned long long need = target - above_w;
      const unsigned long long c = wt ? (need + wt - 1) / wt : 0ull;
      pc = above_c + (int)c;
      p_key = prefix;
      p_above = above_c;
      have_p = true;
    }
  }
  const int m = min(nkb, max(max(kc, pc), 1));

  // 3. Key of the m-th largest block, and how many of its ties are kept.
  unsigned int tkey = p_key;
  int above_m = p_above;
  if (!(have_p && m == pc)) {
    unsigned int prefix = 0u;
    unsigned long long above_w = 0ull;
    int above_c = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
      const unsigned int hi_mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
      radix_pass_warp(keys, nkb, shift, hi_mask, false, (unsigned long long)m, &prefix, &above_w, &above_c, hcnt,
                      hsum);
    }
    tkey = prefix;
    above_m = above_c;
  }
  const int ties_kept = m - above_m;

  // 4. Compaction in block order, 32 blocks per round: ties at the threshold
  //    key are kept lowest index first.
  int32_t* out = kv_idx + row * (int64_t)nkb;
  const unsigned int lt = (1u << lane) - 1u;
  int ties_before = 0, kept_before = 0;
  for (int j0 = 0; j0 < nkb; j0 += 32) {
    const int j = j0 + lane;
    const unsigned int k = j < nkb ? keys[j] : 0u;
    const bool tie = j < nkb && k == tkey;
    const unsigned int tb = __ballot_sync(0xffffffffu, tie);
    const bool keep = j < nkb && (k > tkey || (tie && ties_before + __popc(tb & lt) < ties_kept));
    const unsigned int kb = __ballot_sync(0xffffffffu, keep);
    if (keep) out[kept_before + __popc(kb & lt)] = j;
    ties_before += __popc(tb);
    kept_before += __popc(kb);
  }
  if (lane == 0) {
    kv_cnt[row] = m;
    if (row_thresh) row_thresh[row] = __uint_as_float(tkey);
  }
}

// ----------------------------------------------------------------------------
// Launch order of the query tiles for the kernels that walk a tile's kept
// blocks (their work is proportional to the kept count, which varies several
// times over between tiles). Heads go in groups of G, so the K and V of a
// group stay resident in L2 while its tiles run; inside a group the tiles
// with more kept blocks come first, so the last wave of the grid holds the
// lightest tiles. order[] is a permutation of [0, BH * Nqb); one CTA sorts
// one group by counting (kept counts are at most Nkb). The order of equal
// counts depends on scheduling; the kernels' results do not depend on the
// order at all.
// ----------------------------------------------------------------------------
constexpr int kOrderThreads = 1024;

__host__ __device__ constexpr int tile_order_smem_bytes(int nkb) { return (nkb + 1) * 4 + 32 * 4; }

__global__ void __launch_bounds__(kOrderThreads) tile_order_kernel(const int32_t* __restrict__ kv_cnt, int64_t BH,
                                                                   int nqb, int nkb, int G,
                                                                   int32_t* __restrict__ order) {
  extern __shared__ int hist[];  // [nkb + 1] bins (descending kept count), then 32 warp totals
  int* wsum = hist + nkb + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t h0 = (int64_t)blockIdx.x * G;
  const int nh = (int)(BH - h0 < G ? BH - h0 : G);
  const int n = nh * nqb;
  const int64_t t0 = h0 * nqb;
  for (int b = tid; b <= nkb; b += kOrderThreads) hist[b] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kOrderThreads) {
    const int c = min(max(__ldg(kv_cnt + t0 + i), 0), nkb);
    atomicAdd(&hist[nkb - c], 1);
  }
  __syncthreads();
  // Exclusive scan of the bins: each thread owns a run of `per` bins.
  const int per = (nkb + 1 + kOrderThreads - 1) / kOrderThreads;
  const int b0 = tid * per, b1 = min(nkb + 1, b0 + per);
  int run = 0;
  for (int b = b0; b < b1; ++b) run += hist[b];
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += v;
    }
    wsum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int off = incl - run + (warp > 0 ? wsum[warp - 1] : 0);
  for (int b = b0; b < b1; ++b) {
    const int c = hist[b];
    hist[b] = off;
    off += c;
  }
  __syncthreads();
  for (int i = tid; i < n; i += kOrderThreads) {
    const int c = min(max(__ldg(kv_cnt + t0 + i), 0), nkb);
    const int pos = atomicAdd(&hist[nkb - c], 1);
    order[t0 + pos] = (int32_t)(t0 + i);
  }
}

}  // namespace sparge
