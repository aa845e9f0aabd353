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
__global__ void __launch_bounds__(128) pool_kernel(const __nv_bfloat16* __restrict__ X, int64_t BH, int N,
                                                   int blk, float* __restrict__ out) {
  constexpr int TPB = D / 8;            // threads per block-row
  constexpr int BLOCKS_PER_CTA = 128 / TPB;
  const int nb = (N + blk - 1) / blk;
  const int64_t g = (int64_t)blockIdx.x * BLOCKS_PER_CTA + threadIdx.x / TPB;  // flat (bh, block)
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
  int r = 0;
  for (; r + 4 <= rows; r += 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(src + (int64_t)(r + u) * (D / 8));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f = __bfloat1622float2(h[j]);
        acc[2 * j] = __fadd_rn(acc[2 * j], f.x);
        acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], f.y);
      }
    }
  }
  for (; r < rows; ++r) {
    uint4 v = __ldg(src + (int64_t)r * (D / 8));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __bfloat1622float2(h[j]);
      acc[2 * j] = __fadd_rn(acc[2 * j], f.x);
      acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], f.y);
    }
  }
  const float cnt = (float)rows;
  float4* dst = reinterpret_cast<float4*>(out + g * D + c8);
  dst[0] = make_float4(__fdiv_rn(acc[0], cnt), __fdiv_rn(acc[1], cnt), __fdiv_rn(acc[2], cnt),
                       __fdiv_rn(acc[3], cnt));
  dst[1] = make_float4(__fdiv_rn(acc[4], cnt), __fdiv_rn(acc[5], cnt), __fdiv_rn(acc[6], cnt),
                       __fdiv_rn(acc[7], cnt));
}

// ----------------------------------------------------------------------------
// Scores + row softmax. One CTA = 16 query-block rows of one (b,h) against all
// Nkb key blocks. Pooled K is staged through shared memory 64 blocks at a time
// (rows padded by 4 floats so that 16-byte loads of different rows fall in
// different banks); each thread owns 2 rows x 4 key blocks and runs their
// fused multiply-add chains over channels in order. The scaled scores are
// written to the output rows, which the same CTA then turns into
// probabilities in place (the rows stay in L2 between the two passes).
// ----------------------------------------------------------------------------
constexpr int kScoreRows = 16;
constexpr int kScoreTileJ = 64;

template <int D>
__host__ __device__ constexpr int score_smem_bytes() {
  return (kScoreRows * D + kScoreTileJ * (D + 4)) * 4;
}

template <int D>
__global__ void __launch_bounds__(128) score_softmax_kernel(const float* __restrict__ qbar,
                                                            const float* __restrict__ kbar, int64_t BH,
                                                            int nqb, int nkb, float scale,
                                                            float* __restrict__ P) {
  extern __shared__ __align__(16) float sm[];
  float* sq = sm;                                   // [16][D]
  float* sk = sq + kScoreRows * D;                  // [64][D+4]
  const int tiles_per_bh = (nqb + kScoreRows - 1) / kScoreRows;
  const int64_t bh = blockIdx.x / tiles_per_bh;
  const int I0 = (blockIdx.x % tiles_per_bh) * kScoreRows;
  const int nrows = min(kScoreRows, nqb - I0);
  const int tid = threadIdx.x;

  for (int e = tid; e < kScoreRows * D; e += 128) {
    const int i = e / D;
    sq[e] = (i < nrows) ? qbar[(bh * nqb + I0 + i) * D + (e % D)] : 0.0f;
  }
  const int jl = tid % 16;   // key blocks jl, jl+16, jl+32, jl+48 of the tile
  const int ig = tid / 16;   // query rows 2*ig, 2*ig+1
  const float* kb_head = kbar + bh * (int64_t)nkb * D;
  for (int J0 = 0; J0 < nkb; J0 += kScoreTileJ) {
    __syncthreads();
    const int nj = min(kScoreTileJ, nkb - J0);
    for (int e = tid; e < kScoreTileJ * (D / 4); e += 128) {
      const int j = e / (D / 4), c4 = (e % (D / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < nj) v = *reinterpret_cast<const float4*>(kb_head + (int64_t)(J0 + j) * D + c4);
      *reinterpret_cast<float4*>(sk + j * (D + 4) + c4) = v;
    }
    __syncthreads();
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
          P[(bh * nqb + I0 + 2 * ig + a) * (int64_t)nkb + J0 + j] = __fmul_rn(acc[a][b], scale);
      }
  }
  __syncthreads();
  // Softmax: warp w handles rows w, w+4, w+8, w+12.
  const int warp = tid / 32, lane = tid % 32;
  for (int i = warp; i < nrows; i += 4) {
    float* z = P + (bh * nqb + I0 + i) * (int64_t)nkb;
    float mx = -INFINITY;
    for (int j = lane; j < nkb; j += 32) mx = fmaxf(mx, z[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.0f;
    for (int j = lane; j < nkb; j += 32) {
      const float e = expf(__fsub_rn(z[j], mx));
      z[j] = e;
      sum = __fadd_rn(sum, e);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, o));
    for (int j = lane; j < nkb; j += 32) z[j] = __fdiv_rn(z[j], sum);
  }
}

// ----------------------------------------------------------------------------
// Selection. One CTA of 256 threads per query-block row:
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

__global__ void __launch_bounds__(kSelectThreads) select_kernel(const float* __restrict__ P, int64_t rows,
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
  const float* prow = P + row * (int64_t)nkb;

  for (int j = tid; j < n; j += kSelectThreads) {
    unsigned long long k = ~0ull;
    if (j < nkb) {
      const unsigned int bits = __float_as_uint(prow[j]);
      k = ((unsigned long long)(0xFFFFFFFFu - bits) << 32) | (unsigned int)j;
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
