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
  for (; r + 8 <= rows; r += 8) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(src + (int64_t)(r + u) * (D / 8));
#pragma unroll
    for (int u = 0; u < 8; ++u) add_row(v[u]);  // rows in order
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
// Scaled scores z[I, J] = (q̄_I . k̄_J) * (float)(1/sqrt(d)). One CTA = 16
// query-block rows x 64 key blocks of one (b,h); each thread owns 2 rows x 4
// key blocks and runs their fused multiply-add chains over channels in order.
// Pooled K rows are padded by 4 floats in shared memory so that the 16-byte
// loads of different rows fall in different banks. The row softmax happens
// in the selection kernel, which reads the whole row anyway.
// ----------------------------------------------------------------------------
constexpr int kScoreRows = 16;
constexpr int kScoreTileJ = 64;

template <int D>
__host__ __device__ constexpr int score_smem_bytes() {
  return (kScoreRows * D + kScoreTileJ * (D + 4)) * 4;
}

template <int D>
__global__ void __launch_bounds__(128) score_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                                                    int nqb, int nkb, float scale, float* __restrict__ Z) {
  extern __shared__ __align__(16) float sm[];
  float* sq = sm;                                   // [16][D]
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
  for (int e = tid; e < kScoreRows * (D / 4); e += 128) {
    const int i = e / (D / 4), c4 = (e % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < nrows) v = *reinterpret_cast<const float4*>(qbar + (bh * nqb + I0 + i) * D + c4);
    *reinterpret_cast<float4*>(sq + i * D + c4) = v;
  }
  for (int e = tid; e < kScoreTileJ * (D / 4); e += 128) {
    const int j = e / (D / 4), c4 = (e % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < nj) v = *reinterpret_cast<const float4*>(kbar + (bh * nkb + J0 + j) * D + c4);
    *reinterpret_cast<float4*>(sk + j * (D + 4) + c4) = v;
  }
  __syncthreads();
  const int jl = tid % 16;   // key blocks jl, jl+16, jl+32, jl+48 of the tile
  const int ig = tid / 16;   // query rows 2*ig, 2*ig+1
  float acc[2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
#pragma unroll 4
  for (int c = 0; c < D; c += 4) {
    float4 q[2], k[4];
#pragma unroll
    for (int a = 0; a < 2; ++a) q[a] = *reinterpret_cast<const float4*>(sq + (2 * ig + a) * D + c);
#pragma unroll
    for (int b = 0; b < 4; ++b) k[b] = *reinterpret_cast<const float4*>(sk + (jl + 16 * b) * (D + 4) + c);
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        acc[a][b] = __fmaf_rn(q[a].x, k[b].x, acc[a][b]);
        acc[a][b] = __fmaf_rn(q[a].y, k[b].y, acc[a][b]);
        acc[a][b] = __fmaf_rn(q[a].z, k[b].z, acc[a][b]);
        acc[a][b] = __fmaf_rn(q[a].w, k[b].w, acc[a][b]);
      }
  }
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = jl + 16 * b;
      if (j < nj && 2 * ig + a < nrows)
        Z[(bh * nqb + I0 + 2 * ig + a) * (int64_t)nkb + J0 + j] = __fmul_rn(acc[a][b], scale);
    }
}

// ----------------------------------------------------------------------------
// Softmax + selection. One CTA of 256 threads per query-block row:
//   0. P = expf(z - rowmax) / rowsum, the row sum taken as 32 interleaved
//      partial sums (partial l adds z-terms l, l+32, ... in turn) combined
//      pairwise at distances 16, 8, 4, 2, 1; P is written back over z;
//   1. keys (~bits(P) << 32 | J): ascending order = P descending, J ascending;
//   2. bitonic sort in shared memory (padded to a power of two);
//   3. running sums of the sorted P in double -> pc = first prefix >= topp;
//   4. m = max(kc, pc, 1); flag the first m blocks; compact the flags in block
//      order to emit the kept list ascending.
// ----------------------------------------------------------------------------
constexpr int kSelectThreads = 256;

__host__ __device__ constexpr int select_pad(int nkb) {
  int n = 32;
  while (n < nkb) n <<= 1;
  return n;
}

__host__ __device__ constexpr int select_smem_bytes(int nkb) {
  // keys (8 B each) + flags/scan (4 B each) + per-thread sums (8 B each)
  return select_pad(nkb) * 8 + select_pad(nkb) * 4 + kSelectThreads * 8 + 64;
}

__global__ void __launch_bounds__(kSelectThreads) select_kernel(float* __restrict__ P, int64_t rows,
                                                                 int nkb, int kc, double topp,
                                                                 int32_t* __restrict__ kv_idx,
                                                                 int32_t* __restrict__ kv_cnt,
                                                                 float* __restrict__ row_thresh) {
  extern __shared__ __align__(16) unsigned char smraw[];
  const int n = select_pad(nkb);
  unsigned long long* key = reinterpret_cast<unsigned long long*>(smraw);
  int* flag = reinterpret_cast<int*>(smraw + (size_t)n * 8);
  double* tsum = reinterpret_cast<double*>(smraw + (size_t)n * 12);
  int* s_misc = reinterpret_cast<int*>(smraw + (size_t)n * 12 + kSelectThreads * 8);
  const int64_t row = blockIdx.x;
  if (row >= rows) return;
  const int tid = threadIdx.x;
  float* prow = P + row * (int64_t)nkb;
  float* ev = reinterpret_cast<float*>(flag);  // e-values, before the flags need the space
  float* red = reinterpret_cast<float*>(tsum);

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
    if (tid == 0) red[16] = part;
  }
  __syncthreads();
  const float rsum = red[16];
  for (int j = tid; j < n; j += kSelectThreads) {
    unsigned long long k = ~0ull;
    if (j < nkb) {
      const float pj = __fdiv_rn(ev[j], rsum);
      prow[j] = pj;
      k = ((unsigned long long)(0xFFFFFFFFu - __float_as_uint(pj)) << 32) | (unsigned int)j;
    }
    key[j] = k;
  }
  if (tid == 0) s_misc[0] = nkb;  // pc candidate (min), starts at "never reached"
  __syncthreads();

  // Bitonic sort, ascending.
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = tid; t < n / 2; t += kSelectThreads) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const unsigned long long a = key[lo], b = key[hi];
        if ((a > b) == up) {
          key[lo] = b;
          key[hi] = a;
        }
      }
      __syncthreads();
    }
  }

  // Top-p: each thread sums a contiguous chunk of the sorted order in double,
  // an exclusive scan over the chunk sums gives each chunk's start, then each
  // thread finds the first crossing inside its chunk.
  int pc = 0;
  if (topp > 0.0) {
    const int chunk = (nkb + kSelectThreads - 1) / kSelectThreads;
    const int s0 = min(nkb, tid * chunk), s1 = min(nkb, s0 + chunk);
    double local = 0.0;
    for (int s = s0; s < s1; ++s)
      local += (double)__uint_as_float(0xFFFFFFFFu - (unsigned int)(key[s] >> 32));
    tsum[tid] = local;
    __syncthreads();
    // Hillis-Steele inclusive scan over 256 doubles.
    for (int off = 1; off < kSelectThreads; off <<= 1) {
      const double v = (tid >= off) ? tsum[tid - off] : 0.0;
      __syncthreads();
      tsum[tid] += v;
      __syncthreads();
    }
    double run = tsum[tid] - local;  // exclusive prefix
    for (int s = s0; s < s1; ++s) {
      run += (double)__uint_as_float(0xFFFFFFFFu - (unsigned int)(key[s] >> 32));
      if (run >= topp) {
        atomicMin(&s_misc[0], s + 1);
        break;
      }
    }
    __syncthreads();
    pc = s_misc[0];
  }
  const int m = max(max(kc, pc), 1);

  // Flag kept blocks, then compact in block-index order.
  for (int j = tid; j < n; j += kSelectThreads) flag[j] = 0;
  __syncthreads();
  for (int s = tid; s < m; s += kSelectThreads) flag[(int)(key[s] & 0xFFFFFFFFu)] = 1;
  __syncthreads();
  // Block-wide exclusive scan of flags, each thread owning a contiguous chunk.
  const int chunk = n / kSelectThreads > 0 ? n / kSelectThreads : 1;
  const int c0 = tid * chunk, c1 = min(n, c0 + chunk);
  int cnt = 0;
  for (int j = c0; j < c1; ++j) cnt += flag[j];
  int* tcnt = reinterpret_cast<int*>(tsum);
  tcnt[tid] = cnt;
  __syncthreads();
  for (int off = 1; off < kSelectThreads; off <<= 1) {
    const int v = (tid >= off) ? tcnt[tid - off] : 0;
    __syncthreads();
    tcnt[tid] += v;
    __syncthreads();
  }
  int pos = tcnt[tid] - cnt;
  int32_t* out = kv_idx + row * (int64_t)nkb;
  for (int j = c0; j < c1; ++j)
    if (flag[j]) out[pos++] = j;
  if (tid == 0) {
    kv_cnt[row] = m;
    if (row_thresh) row_thresh[row] = __uint_as_float(0xFFFFFFFFu - (unsigned int)(key[m - 1] >> 32));
  }
}

}  // namespace sparge
