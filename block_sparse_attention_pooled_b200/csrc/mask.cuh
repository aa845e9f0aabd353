// Block-mask kernels: pooling, pooled block importance and hybrid Top-k /
// Top-p selection (SpargeAttention2 article, arXiv:2602.13515, sections 1
// and 4: a pooling pre-filter scores blocks cheaply, a hybrid Top-k / Top-p
// rule selects them, and the result is a block-level mask).
//
// The selection is an integer decision taken from floating point, so every
// step that feeds it runs in double precision:
//   pool : exact double sums of a block's valid bf16 rows, divided by the
//          number of valid rows;
//   score: double fused multiply-adds over the channels, times 1/sqrt(d);
//   prob : exp(z - rowmax) times the reciprocal of the row sum, in double;
//   order: probability descending, block index ascending for ties, on the
//          64-bit patterns of the double probabilities;
//   Top-p: running sums of the ordered probabilities in 2^-62 fixed point
//          (exact integer sums), first prefix whose sum is >= p.
// The result therefore differs from the exact real-number decision only
// where two probabilities, or a running sum and p, lie within a few units in
// the last place of a double of each other.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparge {

// ----------------------------------------------------------------------------
// Pool: out[g, c] = mean over the valid rows of block g of X[., c], in double.
// X: [BH, N, d] bf16. Each thread owns 8 consecutive channels of one block and
// walks its rows (16-byte loads, 8 double accumulators). A bf16 value has 8
// significant bits, so a block's sum of up to 128 of them is exact in double
// whenever their exponents span less than 38 binades; the mean is then the
// exact sum with one rounding.
// ----------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const __nv_bfloat16* __restrict__ Q,
                                                   const __nv_bfloat16* __restrict__ K, int64_t BH, int N, int bq,
                                                   int bk, int64_t q_ctas, double* __restrict__ qbar,
                                                   double* __restrict__ kbar) {
  constexpr int TPB = D / 8;            // threads per block-row
  constexpr int BLOCKS_PER_CTA = 128 / TPB;
  // CTAs [0, q_ctas) pool Q blocks, the rest pool K blocks.
  const bool is_q = blockIdx.x < q_ctas;
  const __nv_bfloat16* X = is_q ? Q : K;
  double* out = is_q ? qbar : kbar;
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
  double acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.0;
  const int rows = r1 - r0;
  auto add_row = [&](uint4 v) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __bfloat1622float2(h[j]);
      acc[2 * j] = __dadd_rn(acc[2 * j], (double)f.x);
      acc[2 * j + 1] = __dadd_rn(acc[2 * j + 1], (double)f.y);
    }
  };
  int r = 0;
  for (; r + 16 <= rows; r += 16) {  // 16 rows in flight per thread
    uint4 v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = __ldg(src + (int64_t)(r + u) * (D / 8));
#pragma unroll
    for (int u = 0; u < 16; ++u) add_row(v[u]);
  }
  for (; r < rows; ++r) add_row(__ldg(src + (int64_t)r * (D / 8)));
  const double cnt = (double)rows;
  double2* dst = reinterpret_cast<double2*>(out + g * D + c8);
#pragma unroll
  for (int j = 0; j < 4; ++j) dst[j] = make_double2(__ddiv_rn(acc[2 * j], cnt), __ddiv_rn(acc[2 * j + 1], cnt));
}

// ----------------------------------------------------------------------------
// Learnt router (SLA2 article, arXiv:2602.12675, section 2: a router with two
// learnable projection matrices maps the query and key features into a space
// suited to the routing decision): pooled block vectors are projected,
//   out[g, c'] = sum_c in[g, c] * W_h[c, c'],  W_h = W + h * D * DR,
// in double (the fp32 weights widened exactly). One CTA = up to 32 pooled
// blocks of one (b, h) (CTA = bh * chunks + chunk), so every row uses the
// same W_h; thread t computes column t % DR for rows t / DR, t / DR + G, ...
// (G = 128 / DR row groups), reading each W_h entry once per CTA.
// ----------------------------------------------------------------------------
constexpr int kProjRows = 32;

template <int D>
__host__ __device__ constexpr int project_smem_bytes() {
  return kProjRows * D * 8;
}

template <int D, int DR>
__global__ void __launch_bounds__(128) project_kernel(const double* __restrict__ in, int64_t nb, int H,
                                                      const float* __restrict__ W, double* __restrict__ out) {
  constexpr int G = 128 / DR, RPT = kProjRows / G;  // row groups, rows per thread
  extern __shared__ __align__(16) double sx[];        // [kProjRows][D]
  const int64_t chunks = (nb + kProjRows - 1) / kProjRows;
  const int64_t bh = blockIdx.x / chunks;
  const int64_t r0 = (blockIdx.x % chunks) * kProjRows;
  const int nr = (int)(nb - r0 < kProjRows ? nb - r0 : kProjRows);
  const double* src = in + (bh * nb + r0) * D;
  for (int e = threadIdx.x; e < kProjRows * (D / 2); e += 128) {
    const int r = e / (D / 2), c2 = (e % (D / 2)) * 2;
    double2 v = make_double2(0.0, 0.0);
    if (r < nr) v = *reinterpret_cast<const double2*>(src + (int64_t)r * D + c2);
    *reinterpret_cast<double2*>(&sx[r * D + c2]) = v;
  }
  __syncthreads();
  const int col = threadIdx.x % DR, grp = threadIdx.x / DR;
  const float* w = W + (bh % H) * D * DR + col;
  double acc[RPT];
#pragma unroll
  for (int k = 0; k < RPT; ++k) acc[k] = 0.0;
#pragma unroll 4
  for (int c = 0; c < D; ++c) {
    const double wc = (double)__ldg(w + c * DR);
#pragma unroll
    for (int k = 0; k < RPT; ++k) acc[k] = __fma_rn(sx[(grp + k * G) * D + c], wc, acc[k]);
  }
  double* dst = out + (bh * nb + r0) * DR + col;
#pragma unroll
  for (int k = 0; k < RPT; ++k)
    if (grp + k * G < nr) dst[(int64_t)(grp + k * G) * DR] = acc[k];
}

// ----------------------------------------------------------------------------
// Scaled scores z[I, J] = (q̄_I . k̄_J) * (1/sqrt(d)), in double, on the fp64
// tensor cores (mma.sync m8n8k4 .f64: each instruction is 256 fused
// multiply-adds of one warp, its operands one double per lane). One CTA =
// 64 query-block rows x 64 key blocks of one (b,h); warp w owns rows
// 32 (w / 2) .. + 31 and key blocks 32 (w % 2) .. + 31 as 4 x 4 tiles of 8 x 8.
// The pooled vectors pass through shared memory 32 channels at a time in a
// two-stage cp.async ring; rows are padded to 36 doubles, so the 8 rows x 4
// channels a fragment load touches fill the banks twice (256 bytes, the
// minimum of two wavefronts). Rows past the tile's end are zero-filled.
// The row softmax happens in the selection kernel, which reads the whole row
// anyway.
// ----------------------------------------------------------------------------
constexpr int kScoreRows = 64;     // query-block rows per CTA
constexpr int kScoreTileJ = 64;    // key blocks per CTA
constexpr int kScoreChunk = 32;    // channels per stage
constexpr int kScorePitch = 36;    // doubles per staged row

template <int D>
__host__ __device__ constexpr int score_smem_bytes() {
  return 2 * (kScoreRows + kScoreTileJ) * kScorePitch * 8;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void dmma_884(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

template <int D>
__global__ void __launch_bounds__(128) score_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar,
                                                    int nqb, int nkb, double scale, double* __restrict__ Z) {
  extern __shared__ __align__(16) double smd[];
  constexpr int kStage = (kScoreRows + kScoreTileJ) * kScorePitch;  // doubles per stage
  constexpr int kChunks = D / kScoreChunk;
  const int tiles_q = (nqb + kScoreRows - 1) / kScoreRows;
  const int tiles_j = (nkb + kScoreTileJ - 1) / kScoreTileJ;
  const int64_t cta = blockIdx.x;
  const int64_t bh = cta / ((int64_t)tiles_q * tiles_j);
  const int rem = (int)(cta % ((int64_t)tiles_q * tiles_j));
  const int I0 = (rem / tiles_j) * kScoreRows;
  const int J0 = (rem % tiles_j) * kScoreTileJ;
  const int nrows = min(kScoreRows, nqb - I0);
  const int nj = min(kScoreTileJ, nkb - J0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double* qsrc = qbar + (bh * nqb + I0) * D;
  const double* ksrc = kbar + (bh * nkb + J0) * D;
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smd);

  // Stage `st` takes channels [ch * 32, ch * 32 + 32) of the tile's 64 + 64
  // rows: 128 rows x 16 pieces of 16 bytes (2 doubles), 16 pieces per thread.
  auto load_stage = [&](int st, int ch) {
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int e = tid + 128 * u;          // 0 .. 2047
      const int r = e >> 4, piece = e & 15;  // row 0 .. 127 (q rows, then k rows), piece 0 .. 15
      const bool is_q = r < kScoreRows;
      const int rr = is_q ? r : r - kScoreRows;
      const bool valid = rr < (is_q ? nrows : nj);
      const double* src = (is_q ? qsrc : ksrc) + (int64_t)(valid ? rr : 0) * D + ch * kScoreChunk + piece * 2;
      const uint32_t dst = sbase + (uint32_t)((st * kStage + r * kScorePitch + piece * 2) * 8);
      cp_async16(dst, src, valid ? 16 : 0);
    }
  };

  double acc[4][4][2];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = 0.0;
  const int wr = 32 * (warp >> 1), wj = 32 * (warp & 1);
  const int fr = lane >> 2, fc = lane & 3;  // fragment row (A row / B column) and channel

  load_stage(0, 0);
  cp_async_commit();
#pragma unroll 1
  for (int ch = 0; ch < kChunks; ++ch) {
    if (ch + 1 < kChunks) {
      load_stage((ch + 1) & 1, ch + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const double* sq = smd + (ch & 1) * kStage;
    const double* sk = sq + kScoreRows * kScorePitch;
#pragma unroll
    for (int kk = 0; kk < kScoreChunk / 4; ++kk) {
      double a[4], b[4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) a[mt] = sq[(wr + 8 * mt + fr) * kScorePitch + 4 * kk + fc];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) b[nt] = sk[(wj + 8 * nt + fr) * kScorePitch + 4 * kk + fc];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) dmma_884(acc[mt][nt][0], acc[mt][nt][1], a[mt], b[nt]);
    }
    __syncthreads();  // the stage is refilled two chunks later
  }
  // Accumulator (c0, c1) of tile (mt, nt) sits at row 8 mt + lane / 4,
  // columns 8 nt + 2 (lane % 4) + {0, 1}.
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const int i = wr + 8 * mt + fr;
    if (i >= nrows) continue;
    double* zrow = Z + (bh * nqb + I0 + i) * (int64_t)nkb + J0;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int j = wj + 8 * nt + 2 * fc;
      if (j < nj) zrow[j] = __dmul_rn(acc[mt][nt][0], scale);
      if (j + 1 < nj) zrow[j + 1] = __dmul_rn(acc[mt][nt][1], scale);
    }
  }
}

// ----------------------------------------------------------------------------
// Softmax + selection. Keys are the 64-bit patterns of the double
// probabilities (ordered like P for P >= 0); the weight of a block is its
// probability in 64-bit fixed point (2^62 = 1), exact for P >= 2^-9 and
// truncated to a multiple of 2^-62 below, so running sums are exact integers
// whatever the summation order (the truncation moves a row's total by less
// than Nkb * 2^-62).
//   0. P = exp(z - rowmax) * (1 / rowsum) (double; within a rounding unit of
//      the quotient, and equal scores still give equal probabilities).
//   1. Top-p: a radix select of the key at which the descending running
//      weight first reaches p. The first pass buckets the keys by binade
//      below the row's largest (bucket 255 - (e_top - e)); the next passes
//      take 8-bit digits of the mantissa inside the chosen binade. It stops
//      as soon as the bucket where p is reached holds a single block (its
//      index is recorded while the histogram is built). If the blocks left at
//      full resolution tie exactly, they weigh the same and the count needed
//      follows by division.
//   2. m = max(kc, pc, 1). When m = pc the threshold is the one just found;
//      otherwise a counting radix select finds the m-th largest key, stopping
//      as soon as the bucket where the count is reached holds one block, or
//      is kept whole (its smallest key is then the threshold).
//   3. The threshold is a full key T and a number t of the blocks equal to T
//      that are kept (lowest indices first): a block is kept if its key
//      exceeds T, or equals T and fewer than t lower-indexed blocks do.
//      Kept flags are compacted in block order into the ascending kept list.
// ----------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long p_fixed62(unsigned long long bits) {
  const int e = (int)((bits >> 52) & 0x7FFull);
  if (e == 0) return 0ull;  // zero or subnormal: below 2^-1022
  const unsigned long long mant = (bits & 0xFFFFFFFFFFFFFull) | (1ull << 52);
  const int sh = e - 1013;  // value = mant * 2^(e - 1075); times 2^62
  if (sh >= 0) return mant << sh;  // sh <= 10 for P <= 1
  return (-sh >= 64) ? 0ull : (mant >> (-sh));
}

constexpr int kSelectThreads = 256;
constexpr unsigned long long kWeightOne = 1ull << 62;
constexpr int kAllTies = 1 << 30;  // "every block equal to the threshold key is kept"

// The threshold of a row: see step 3 above.
struct RowThreshold {
  unsigned long long key;
  int ties_kept;
  int count;  // blocks kept when this threshold alone decides (pc or m)
};

__device__ __forceinline__ bool keep_key(unsigned long long k, const RowThreshold& t, int tie_rank) {
  return k > t.key || (k == t.key && tie_rank < t.ties_kept);
}

// State of a radix select between passes.
struct RadixState {
  unsigned long long prefix;   // resolved bits of the selected class
  unsigned long long mask;     // which bits are resolved
  unsigned long long above_w;  // weight of the keys above the selected class
  int above_c;                 // count of the keys above the selected class
  int bucket_c;                // count of the keys in the selected class
  int bsel;                    // selected bucket of the last pass
  int bidx;                    // index of a key of that bucket (the key when bucket_c == 1)
};

// Bucket of key k in one pass: shift < 0 is the binade pass (every key is a
// candidate; bucket 255 holds the binade of the row's largest key, bucket 0
// everything 255 or more binades below, zeros included); otherwise the 8-bit
// digit at `shift` of the keys in the selected class.
__device__ __forceinline__ bool key_bucket(unsigned long long k, int shift, int e_top, const RadixState& st,
                                           unsigned int* d) {
  if (shift < 0) {
    const int e = (int)((k >> 52) & 0x7FFull);
    *d = 255u - (unsigned int)min(255, e_top - e);
    return true;
  }
  *d = (unsigned int)(k >> shift) & 255u;
  return (k & st.mask) == st.prefix;
}

// Finds, among 256 buckets held by lanes (lane l owns buckets 255-8l ...
// 248-8l, descending), the first (from the largest key down) where the
// running weight (by_weight) or count, starting from st's totals, reaches
// `target`. Called by the 32 lanes of one warp; every lane gets the result.
__device__ __forceinline__ RadixState radix_scan_warp(const unsigned int* hcnt, const unsigned long long* hsum,
                                                      const unsigned int* hidx, bool by_weight,
                                                      unsigned long long target, int shift, RadixState st) {
  const int lane = threadIdx.x & 31;
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
  const unsigned long long aw = st.above_w + xw - lw;  // running value before this lane's buckets
  const unsigned int ac = (unsigned int)st.above_c + xc - lc;
  const bool reach = by_weight ? (aw + lw >= target) : ((unsigned long long)(ac + lc) >= target);
  const unsigned int ballot = __ballot_sync(0xffffffffu, reach);
  const int first = __ffs(ballot) - 1;  // first lane (from the top) whose buckets reach the target
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
  st.bsel = bsel;
  st.above_c = (int)c;
  st.above_w = w;
  st.bucket_c = (int)hcnt[bsel];
  st.bidx = (int)hidx[bsel];
  if (shift >= 0) {
    st.prefix |= (unsigned long long)bsel << shift;
    st.mask |= 255ull << shift;
  }
  return st;
}

// Radix select over one row's keys. pass(shift, e_top, by_weight, target,
// state) builds one histogram and scans it; class_min(state) returns the
// smallest key of the selected class; key_at(j) reads key j. by_weight:
// Top-p (target = p in fixed point; *count receives pc); otherwise the
// target-th largest key (*count = target).
template <typename Pass, typename ClassMin, typename KeyAt>
__device__ __forceinline__ RowThreshold radix_select(Pass pass, ClassMin class_min, KeyAt key_at, int e_top,
                                                     bool by_weight, unsigned long long target) {
  RadixState st{0ull, 0ull, 0ull, 0, 0, 0, 0};
  st = pass(-1, e_top, by_weight, target, st);  // binade pass
  // Mantissa digits inside one binade (shifts 44, 36, ..., 4, then 0: the
  // last digit overlaps the one before, whose bits are already resolved);
  // the full key's digits (56, 48, ..., 0) when the chosen bucket mixes
  // binades (255 or more below the largest key, zeros).
  const bool mixed = st.bsel == 0;
  int n = 0;
  if (st.bucket_c != 1) {
    if (mixed) {
      st = RadixState{0ull, 0ull, 0ull, 0, 0, 0, 0};
    } else {
      st.prefix = (unsigned long long)(e_top - (255 - st.bsel)) << 52;  // sign 0 and the binade's exponent
      st.mask = 0xFFFull << 52;
    }
  }
  for (;;) {
    if (st.bucket_c == 1) {  // one block left in the class: it is the threshold
      return RowThreshold{key_at(st.bidx), 1, st.above_c + 1};
    }
    const int need_c = (int)target - st.above_c;
    if (!by_weight && need_c == st.bucket_c) {  // the whole class is kept (never right after a reset: 0 < need_c)
      return RowThreshold{class_min(st), kAllTies, (int)target};
    }
    if (n == (mixed ? 8 : 7)) break;  // full key resolved
    st = pass(mixed ? 56 - 8 * n : max(44 - 8 * n, 0), e_top, by_weight, target, st);
    ++n;
  }
  // Every key of the class equals st.prefix: ties.
  int need = (int)target - st.above_c;
  if (by_weight) {
    const unsigned long long wt = p_fixed62(st.prefix);
    const unsigned long long rem = target - st.above_w;  // > 0 by construction
    need = wt ? (int)((rem + wt - 1) / wt) : st.bucket_c;
  }
  need = max(1, min(need, st.bucket_c));
  return RowThreshold{st.prefix, need, st.above_c + need};
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}
__device__ __forceinline__ unsigned long long umin64(unsigned long long a, unsigned long long b) {
  return a < b ? a : b;
}

__host__ __device__ constexpr int select_smem_bytes(int nkb) {
  // P / keys row (8 B per block) + histograms (weights, counts, one index per
  // bucket) + scratch
  return ((nkb + 1) / 2 * 2) * 8 + 256 * 16 + 1024;
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

// Block-wide maximum / minimum of one 64-bit value per thread (256 threads).
template <bool MAX>
__device__ __forceinline__ unsigned long long block_ext64(unsigned long long v, unsigned long long* scratch) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, v, o);
    v = MAX ? umax64(v, y) : umin64(v, y);
  }
  if (lane == 0) scratch[wid] = v;
  __syncthreads();
  v = scratch[0];
#pragma unroll
  for (int w = 1; w < kSelectThreads / 32; ++w) v = MAX ? umax64(v, scratch[w]) : umin64(v, scratch[w]);
  __syncthreads();
  return v;
}

// Selection with one CTA (256 threads) per row, for rows longer than the
// warp kernel takes.
__global__ void __launch_bounds__(kSelectThreads) select_kernel(const double* __restrict__ Z, int64_t rows, int nkb,
                                                                 int kc, double topp, int32_t* __restrict__ kv_idx,
                                                                 int32_t* __restrict__ kv_cnt,
                                                                 float* __restrict__ row_thresh,
                                                                 float* __restrict__ probs) {
  extern __shared__ __align__(16) unsigned char smraw[];
  const int npad = (nkb + 1) / 2 * 2;
  double* ev = reinterpret_cast<double*>(smraw);                                       // [npad], then the keys
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smraw);
  unsigned long long* hsum = reinterpret_cast<unsigned long long*>(smraw + npad * 8);  // [256]
  unsigned int* hcnt = reinterpret_cast<unsigned int*>(hsum + 256);                   // [256]
  unsigned int* hidx = hcnt + 256;                                                     // [256]
  RadixState* shared_st = reinterpret_cast<RadixState*>(hidx + 256);                   // [1]
  double* red = reinterpret_cast<double*>(shared_st + 1);                             // [8]
  unsigned long long* ured = reinterpret_cast<unsigned long long*>(red + 8);          // [8]
  int* scratch = reinterpret_cast<int*>(ured + 8);                                    // [8]
  const int64_t row = blockIdx.x;
  if (row >= rows) return;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const double* zrow = Z + row * (int64_t)nkb;

  // 0. Row softmax.
  double mx = -INFINITY;
  for (int j = tid; j < nkb; j += kSelectThreads) {
    const double z = zrow[j];
    ev[j] = z;
    mx = fmax(mx, z);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[wid] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < kSelectThreads / 32; ++w) mx = fmax(mx, red[w]);
  __syncthreads();
  double part = 0.0;
  for (int j = tid; j < nkb; j += kSelectThreads) {
    const double e = exp(__dsub_rn(ev[j], mx));
    ev[j] = e;
    part = __dadd_rn(part, e);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part = __dadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
  if (lane == 0) red[wid] = part;
  __syncthreads();
  double rsum = 0.0;
#pragma unroll
  for (int w = 0; w < kSelectThreads / 32; ++w) rsum = __dadd_rn(rsum, red[w]);
  unsigned long long tot = 0ull, kmax = 0ull;  // total weight (exact integer sum), largest key
  const double rinv = __drcp_rn(rsum);
  for (int j = tid; j < nkb; j += kSelectThreads) {
    const double pj = __dmul_rn(ev[j], rinv);
    if (probs) probs[row * (int64_t)nkb + j] = (float)pj;
    const unsigned long long k = (unsigned long long)__double_as_longlong(pj);
    keys[j] = k;
    tot += p_fixed62(k);
    kmax = umax64(kmax, k);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  if (lane == 0) ured[wid] = tot;
  __syncthreads();
  tot = 0ull;
#pragma unroll
  for (int w = 0; w < kSelectThreads / 32; ++w) tot += ured[w];
  __syncthreads();
  kmax = block_ext64<true>(kmax, ured);
  const int e_top = (int)((kmax >> 52) & 0x7FFull);

  auto pass = [&](int shift, int etop, bool by_weight, unsigned long long target, RadixState st) {
    hcnt[tid] = 0u;
    hsum[tid] = 0ull;
    __syncthreads();
    for (int j = tid; j < nkb; j += kSelectThreads) {
      const unsigned long long k = keys[j];
      unsigned int d;
      if (key_bucket(k, shift, etop, st, &d)) {
        atomicAdd(&hcnt[d], 1u);
        if (by_weight) atomicAdd(&hsum[d], p_fixed62(k));
        hidx[d] = (unsigned int)j;
      }
    }
    __syncthreads();
    if (tid < 32) {
      const RadixState s2 = radix_scan_warp(hcnt, hsum, hidx, by_weight, target, shift, st);
      if (tid == 0) *shared_st = s2;
    }
    __syncthreads();
    st = *shared_st;
    __syncthreads();
    return st;
  };
  auto class_min = [&](const RadixState& st) {
    unsigned long long v = ~0ull;
    for (int j = tid; j < nkb; j += kSelectThreads) {
      const unsigned long long k = keys[j];
      if ((k & st.mask) == st.prefix) v = umin64(v, k);
    }
    return block_ext64<false>(v, ured);
  };
  auto key_at = [&](int j) { return keys[j]; };

  // 1. Top-p count.
  int pc = 0;
  bool have_p = false;
  RowThreshold thr{0ull, 0, 0};
  if (topp > 0.0) {
    const unsigned long long target = (unsigned long long)ceil(topp * (double)kWeightOne);
    if (tot < target) {
      pc = nkb;  // never reached
    } else {
      thr = radix_select(pass, class_min, key_at, e_top, true, target);
      pc = thr.count;
      have_p = true;
    }
  }
  const int m = min(nkb, max(max(kc, pc), 1));
  // 2. Threshold of the m-th largest block.
  if (!(have_p && m == pc)) thr = radix_select(pass, class_min, key_at, e_top, false, (unsigned long long)m);

  // 3. Compaction in block order: each thread owns a contiguous chunk.
  const int per = (nkb + kSelectThreads - 1) / kSelectThreads;
  const int j0 = min(nkb, tid * per), j1 = min(nkb, j0 + per);
  int nt = 0;
  for (int j = j0; j < j1; ++j) nt += keys[j] == thr.key;
  int tie_tot;
  const int tie_rank = block_excl_scan(nt, scratch, &tie_tot);
  int nk = 0;
  {
    int tr = tie_rank;
    for (int j = j0; j < j1; ++j) {
      const unsigned long long k = keys[j];
      nk += keep_key(k, thr, tr);
      tr += k == thr.key;
    }
  }
  int kept_tot;
  int pos = block_excl_scan(nk, scratch, &kept_tot);
  int32_t* out = kv_idx + row * (int64_t)nkb;
  {
    int tr = tie_rank;
    for (int j = j0; j < j1; ++j) {
      const unsigned long long k = keys[j];
      if (keep_key(k, thr, tr)) out[pos++] = j;
      tr += k == thr.key;
    }
  }
  if (tid == 0) {
    kv_cnt[row] = m;
    if (row_thresh) row_thresh[row] = (float)__longlong_as_double((long long)thr.key);
  }
}

// ----------------------------------------------------------------------------
// The same selection with one warp per row (eight rows per CTA), for rows of
// at most kSelWarpMaxNkb blocks: every step is the arithmetic of
// select_kernel, but the row's steps synchronise with warp barriers instead
// of block barriers. Each warp owns its row's P (then keys) and a 256-bucket
// histogram in shared memory.
// ----------------------------------------------------------------------------
constexpr int kSelWarpRows = 8;
constexpr int kSelWarpMaxNkb = 2048;

__host__ __device__ constexpr int select_warp_bytes(int nkb) { return (nkb + 1) / 2 * 16 + 256 * 16; }
__host__ __device__ constexpr int select_warp_smem_bytes(int nkb) { return kSelWarpRows * select_warp_bytes(nkb); }

__global__ void __launch_bounds__(kSelWarpRows * 32) select_warp_kernel(const double* __restrict__ Z, int64_t rows,
                                                                        int nkb, int kc, double topp,
                                                                        int32_t* __restrict__ kv_idx,
                                                                        int32_t* __restrict__ kv_cnt,
                                                                        float* __restrict__ row_thresh,
                                                                        float* __restrict__ probs) {
  extern __shared__ __align__(16) unsigned char smraw[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * kSelWarpRows + wid;
  if (row >= rows) return;  // whole warps only: no block barrier follows
  unsigned char* mine = smraw + wid * select_warp_bytes(nkb);
  double* ev = reinterpret_cast<double*>(mine);  // [nkb], then the keys
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(mine);
  unsigned long long* hsum = reinterpret_cast<unsigned long long*>(mine + (nkb + 1) / 2 * 16);  // [256]
  unsigned int* hcnt = reinterpret_cast<unsigned int*>(hsum + 256);                           // [256]
  unsigned int* hidx = hcnt + 256;                                                             // [256]
  const double* zrow = Z + row * (int64_t)nkb;

  // 0. Row softmax.
  double mx = -INFINITY;
  for (int j = lane; j < nkb; j += 32) {
    const double z = zrow[j];
    ev[j] = z;
    mx = fmax(mx, z);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  double part = 0.0;
  for (int j = lane; j < nkb; j += 32) {
    const double e = exp(__dsub_rn(ev[j], mx));
    ev[j] = e;
    part = __dadd_rn(part, e);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part = __dadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
  const double rsum = part;
  unsigned long long tot = 0ull, kmax = 0ull;  // total weight (exact integer sum), largest key
  const double rinv = __drcp_rn(rsum);
  for (int j = lane; j < nkb; j += 32) {
    const double pj = __dmul_rn(ev[j], rinv);
    if (probs) probs[row * (int64_t)nkb + j] = (float)pj;
    const unsigned long long k = (unsigned long long)__double_as_longlong(pj);
    keys[j] = k;
    tot += p_fixed62(k);
    kmax = umax64(kmax, k);
  }
  __syncwarp();
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
    kmax = umax64(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  const int e_top = (int)((kmax >> 52) & 0x7FFull);

  auto pass = [&](int shift, int etop, bool by_weight, unsigned long long target, RadixState st) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      hcnt[lane * 8 + i] = 0u;
      hsum[lane * 8 + i] = 0ull;
    }
    __syncwarp();
    for (int j = lane; j < nkb; j += 32) {
      const unsigned long long k = keys[j];
      unsigned int d;
      if (key_bucket(k, shift, etop, st, &d)) {
        atomicAdd(&hcnt[d], 1u);
        if (by_weight) atomicAdd(&hsum[d], p_fixed62(k));
        hidx[d] = (unsigned int)j;
      }
    }
    __syncwarp();
    st = radix_scan_warp(hcnt, hsum, hidx, by_weight, target, shift, st);
    __syncwarp();
    return st;
  };
  auto class_min = [&](const RadixState& st) {
    unsigned long long v = ~0ull;
    for (int j = lane; j < nkb; j += 32) {
      const unsigned long long k = keys[j];
      if ((k & st.mask) == st.prefix) v = umin64(v, k);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = umin64(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
  };
  auto key_at = [&](int j) { return keys[j]; };

  // 1. Top-p count.
  int pc = 0;
  bool have_p = false;
  RowThreshold thr{0ull, 0, 0};
  if (topp > 0.0) {
    const unsigned long long target = (unsigned long long)ceil(topp * (double)kWeightOne);
    if (tot < target) {
      pc = nkb;
    } else {
      thr = radix_select(pass, class_min, key_at, e_top, true, target);
      pc = thr.count;
      have_p = true;
    }
  }
  const int m = min(nkb, max(max(kc, pc), 1));
  // 2. Threshold of the m-th largest block.
  if (!(have_p && m == pc)) thr = radix_select(pass, class_min, key_at, e_top, false, (unsigned long long)m);

  // 3. Compaction in block order, 32 blocks per round: ties at the threshold
  //    are kept lowest index first.
  int32_t* out = kv_idx + row * (int64_t)nkb;
  const unsigned int lt = (1u << lane) - 1u;
  int ties_before = 0, kept_before = 0;
  for (int j0 = 0; j0 < nkb; j0 += 32) {
    const int j = j0 + lane;
    const unsigned long long k = j < nkb ? keys[j] : 0ull;
    const bool tie = j < nkb && k == thr.key;
    const unsigned int tb = __ballot_sync(0xffffffffu, tie);
    const bool keep = j < nkb && keep_key(k, thr, ties_before + __popc(tb & lt));
    const unsigned int kb = __ballot_sync(0xffffffffu, keep);
    if (keep) out[kept_before + __popc(kb & lt)] = j;
    ties_before += __popc(tb);
    kept_before += __popc(kb);
  }
  if (lane == 0) {
    kv_cnt[row] = m;
    if (row_thresh) row_thresh[row] = (float)__longlong_as_double((long long)thr.key);
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
