// Block-sparse attention backward on the 5th-generation tensor cores.
//
// What it computes (SpargeAttention2 article, arXiv:2602.13515, section 1:
// the sparse attention is trainable, so its gradients flow through the kept
// blocks; section 4: each block is either fully computed or fully skipped).
// For the sparse forward O_i = sum_{j kept} P_ij v_j, P_ij = softmax_j(s_ij),
// s_ij = q_i . k_j / sqrt(d), and dL/dO = dO:
//   D_i   = dO_i . O_i
//   P_ij  = exp(s_ij - lse_i)                 (lse from the forward)
//   dP_ij = dO_i . v_j,   dS_ij = P_ij (dP_ij - D_i)
//   dQ_i  = sum_j dS_ij k_j / sqrt(d)          (kept keys of i's block)
//   dK_j  = sum_i dS_ij q_i / sqrt(d),  dV_j = sum_i P_ij dO_i
//                                              (rows whose block keeps j's)
//
// Four or five launches, no atomics (bit-reproducible):
//   bwd_dot_kernel         D_i for every row;
//   mask_transpose_kernel  for every key block, the ascending list of query
//                          blocks that keep it;
//   tile_order_kernel      the query tiles' launch order (as the forward's),
//                          when groups of heads fit in L2;
//   attn_bwd_dq_kernel     one CTA per query tile, walking its kept key tiles
//                          (the forward's structure): S = Q K^T and
//                          dP = dO V^T into TMEM, dS written back over S as
//                          bf16, dQ += dS K with dS read from TMEM;
//   attn_bwd_dkdv_kernel   one CTA per 64-key tile, walking the query tiles
//                          that keep it: S and dP as above; P and dS staged
//                          as bf16 in shared memory; dV^T += dO^T P and
//                          dK^T += Q^T dS accumulate in TMEM with the head
//                          dimension on the lanes (M = d = 128), so the MMAs
//                          keep M = 128 for 64-key blocks.
// Warp roles as in the forward: warp 0 TMA producer, warp 1 MMA issuer and
// TMEM owner, then one row (TMEM lane) per thread in warpgroups of four
// warps (three in the dQ kernel, one in the dK/dV kernel). d = 128.
#pragma once
#include <cuda.h>
#include <cstdint>
#include <cuda_bf16.h>

#include "attn.cuh"
#include "ptx.cuh"

namespace sparge {

enum : unsigned int {
  kErrBwdIn = 0x700, kErrBwdKFull, kErrBwdVFull, kErrBwdKEmpty, kErrBwdVEmpty, kErrBwdSFull, kErrBwdPFull,
  kErrBwdFinal, kErrBwdDrain, kErrBwdStage, kErrBwdInEmpty, kErrBwdKV
};

struct BwdParams {
  const int32_t* lst;  // dQ: kv_idx [BH, nqb, nkb]; dK/dV: query-block lists [BH, nkb, nqb]
  const int32_t* cnt;  // dQ: kv_cnt [BH, nqb];       dK/dV: list lengths [BH, nkb]
  const int32_t* order;  // dQ: launch order of the query tiles (as the forward's), or null
  const float* lse;    // [BH, N], natural log, from the forward
  const float* dsum;   // [BH, N], D_i = dO_i . O_i
  int N;
  int nqb;
  int nkb;
  int bq;
  int bk;
  float scale_log2;  // log2(e) / sqrt(d)
  float scale;       // 1 / sqrt(d)
};

// ---------------------------------------------------------------------------
// D_i = sum_c dO_ic O_ic in fp32 (bf16 inputs); each thread takes 8 channels,
// the row's threads combine by shuffles in a fixed order.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_dot_kernel(const __nv_bfloat16* __restrict__ O,
                                                      const __nv_bfloat16* __restrict__ dO, int64_t rows,
                                                      float* __restrict__ dsum) {
  constexpr int TPR = D / 8;
  const int64_t g = (int64_t)blockIdx.x * (256 / TPR) + threadIdx.x / TPR;
  const int c8 = (threadIdx.x % TPR) * 8;
  float acc = 0.0f;
  if (g < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(O + g * D + c8);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + g * D + c8);
    const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 x = __bfloat1622float2(ha[j]), y = __bfloat1622float2(hb[j]);
      acc = __fmaf_rn(x.x, y.x, acc);
      acc = __fmaf_rn(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (g < rows && threadIdx.x % TPR == 0) dsum[g] = acc;
}

// ---------------------------------------------------------------------------
// Transposed mask: for key block J of head bh, the query blocks I whose kept
// list holds J, ascending. One CTA = one head x 256 key blocks: a bit matrix
// [Nqb][256] in shared memory is filled from the kept lists, then thread t
// walks column t in query-block order. Entries outside [0, Nkb) are ignored.
// ---------------------------------------------------------------------------
constexpr int kTrCols = 256;

__host__ __device__ constexpr int transpose_smem_bytes(int nqb) { return nqb * (kTrCols / 8); }

__global__ void __launch_bounds__(kTrCols) mask_transpose_kernel(const int32_t* __restrict__ kv_idx,
                                                                 const int32_t* __restrict__ kv_cnt, int nqb,
                                                                 int nkb, int32_t* __restrict__ q_idx,
                                                                 int32_t* __restrict__ q_cnt) {
  extern __shared__ uint32_t bits[];  // [nqb][kTrCols / 32]
  constexpr int W = kTrCols / 32;
  const int chunks = (nkb + kTrCols - 1) / kTrCols;
  const int64_t bh = blockIdx.x / chunks;
  const int j0 = (int)(blockIdx.x % chunks) * kTrCols;
  for (int e = threadIdx.x; e < nqb * W; e += kTrCols) bits[e] = 0u;
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int I = warp; I < nqb; I += kTrCols / 32) {
    const int64_t row = bh * nqb + I;
    const int c = min(max(__ldg(kv_cnt + row), 0), nkb);
    const int32_t* lst = kv_idx + row * nkb;
    for (int e = lane; e < c; e += 32) {
      const int J = __ldg(lst + e) - j0;
      if (J >= 0 && J < kTrCols) atomicOr(&bits[I * W + (J >> 5)], 1u << (J & 31));
    }
  }
  __syncthreads();
  const int J = j0 + threadIdx.x;
  if (J < nkb) {
    const int w = threadIdx.x >> 5;
    const uint32_t m = 1u << (threadIdx.x & 31);
    int32_t* out = q_idx + (bh * nkb + J) * (int64_t)nqb;
    int n = 0;
    for (int I = 0; I < nqb; ++I)
      if (bits[I * W + w] & m) out[n++] = I;
    q_cnt[bh * nkb + J] = n;
  }
}

// ---------------------------------------------------------------------------
// Row pass of the SLA2 backward (SLA2 article, arXiv:2602.12675, section 2:
// O = alpha_h O_s + (1 - alpha_h) O_l). Row i of head bh, h = bh % H:
//   D_i = alpha_h dO_i . O_s,i     (the sparse backward's D for dO -> alpha_h dO)
//   f_i = dO_i . O_l,i,  c_i = (1 - alpha_h) / den_i (0 where the linear
//   branch is off, den_i = 0), e_i = c_i f_i,
//   and dO_i . (O_s,i - O_l,i), the row's share of dalpha_h.
// One CTA = kRowsPerCta rows of one (bh), 16 threads per row; each CTA's
// dalpha share goes to part[] and sla2_dalpha_kernel adds them in order.
// ---------------------------------------------------------------------------
constexpr int kRowsPerCta = 256;

template <int D>
__global__ void __launch_bounds__(256)
    sla2_bwd_rows_kernel(const __nv_bfloat16* __restrict__ Os, const __nv_bfloat16* __restrict__ Ol,
                         const __nv_bfloat16* __restrict__ dO, const float* __restrict__ den,
                         const float* __restrict__ alpha, int H, int N, int chunks, float* __restrict__ dsum,
                         float* __restrict__ cw, float* __restrict__ fw, float* __restrict__ ew,
                         float* __restrict__ part) {
  constexpr int TPR = D / 8, RPP = 256 / TPR;
  __shared__ float red[8];
  const int64_t bh = blockIdx.x / chunks;
  const int r0 = (int)(blockIdx.x % chunks) * kRowsPerCta;
  const float a = __ldg(alpha + bh % H);
  const int c8 = (threadIdx.x % TPR) * 8;
  float acc = 0.0f;
  for (int k = 0; k < kRowsPerCta / RPP; ++k) {
    const int r = r0 + k * RPP + threadIdx.x / TPR;
    float ds = 0.0f, dl = 0.0f;
    if (r < N) {
      const int64_t g = (bh * N + r) * D + c8;
      const uint4 uo = *reinterpret_cast<const uint4*>(Os + g);
      const uint4 ul = *reinterpret_cast<const uint4*>(Ol + g);
      const uint4 ud = *reinterpret_cast<const uint4*>(dO + g);
      const __nv_bfloat162* ho = reinterpret_cast<const __nv_bfloat162*>(&uo);
      const __nv_bfloat162* hl = reinterpret_cast<const __nv_bfloat162*>(&ul);
      const __nv_bfloat162* hd = reinterpret_cast<const __nv_bfloat162*>(&ud);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 xo = __bfloat1622float2(ho[j]), xl = __bfloat1622float2(hl[j]), xd = __bfloat1622float2(hd[j]);
        ds = __fmaf_rn(xd.x, xo.x, ds);
        ds = __fmaf_rn(xd.y, xo.y, ds);
        dl = __fmaf_rn(xd.x, xl.x, dl);
        dl = __fmaf_rn(xd.y, xl.y, dl);
      }
    }
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) {
      ds += __shfl_xor_sync(0xffffffffu, ds, o);
      dl += __shfl_xor_sync(0xffffffffu, dl, o);
    }
    if (r < N && threadIdx.x % TPR == 0) {
      const int64_t row = bh * N + r;
      const float dn = __ldg(den + row);
      const float c = dn > 0.0f ? (1.0f - a) / dn : 0.0f;
      dsum[row] = a * ds;
      fw[row] = dl;
      cw[row] = c;
      ew[row] = c * dl;
      acc += ds - dl;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w];
    part[blockIdx.x] = t;
  }
}

// dalpha_h = the row shares of every batch of head h, in (batch, chunk) order.
__global__ void __launch_bounds__(128) sla2_dalpha_kernel(const float* __restrict__ part, int B, int H, int chunks,
                                                          float* __restrict__ dalpha) {
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    float acc = 0.0f;
    for (int b = 0; b < B; ++b)
      for (int k = 0; k < chunks; ++k) acc += part[(int64_t)(b * H + h) * chunks + k];
    dalpha[h] = acc;
  }
}

// ---------------------------------------------------------------- shared pieces
// The row's 64 values of a TMEM block (S or dP) into registers.
__device__ __forceinline__ void load_row64(uint32_t taddr, float (&s)[kTileK]) { load_scores(taddr, s); }

// P_j = 2^(s_j * scale_log2 - lse2); pp = a P, pds = dS = P (a dP - D) (a:
// the branch weight alpha_h of the SLA2 mix, 1 for the sparse branch alone);
// keys at or past N (and rows the caller marks invalid) give zeros.
__device__ __forceinline__ void p_and_ds(const float (&s)[kTileK], const float (&dp)[kTileK], float scale_log2,
                                         float lse2, float Di, float a, int key0, int N, bool row_ok,
                                         uint32_t (&pp)[kTileK / 2], uint32_t (&pds)[kTileK / 2]) {
  const uint64_t sc2 = f2(scale_log2, scale_log2), nl2 = f2(-lse2, -lse2), nd2 = f2(-Di, -Di), a2 = f2(a, a);
  const bool tail = key0 + kTileK > N;
#pragma unroll
  for (int k = 0; k < kTileK / 2; ++k) {
    const float2 x = f2_split(fma2(f2(s[2 * k], s[2 * k + 1]), sc2, nl2));
    float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
    if (!row_ok || (tail && key0 + 2 * k >= N)) p0 = 0.0f;
    if (!row_ok || (tail && key0 + 2 * k + 1 >= N)) p1 = 0.0f;
    const float2 g = f2_split(fma2(f2(dp[2 * k], dp[2 * k + 1]), a2, nd2));
    pp[k] = pack_bf16x2(a * p0, a * p1);
    pds[k] = pack_bf16x2(p0 * g.x, p1 * g.y);
  }
}

// Entries of a block list, 32 at a time, one per lane, a chunk ahead of use,
// so no tile waits on a global load. The whole warp calls get() with the
// same non-decreasing entry index.
struct ListChunks {
  int cur, nxt, chunk;
  __device__ __forceinline__ ListChunks(const int32_t* lst, int n, int lane) : chunk(0) {
    cur = lane < n ? __ldg(lst + lane) : 0;
    nxt = 32 + lane < n ? __ldg(lst + 32 + lane) : 0;
  }
  __device__ __forceinline__ int get(const int32_t* lst, int n, int e, int lane) {
    while ((e >> 5) != chunk) {
      ++chunk;
      cur = nxt;
      nxt = 32 * (chunk + 1) + lane < n ? __ldg(lst + 32 * (chunk + 1) + lane) : 0;
    }
    return __shfl_sync(0xffffffffu, cur, e & 31);
  }
};

// ---------------------------------------------------------------------------
// dQ: one CTA per (bh, query block), the forward's walk over kept key tiles.
// TMEM columns: S(b) [64b, 64b+64) and dP(b) [192 + 64b, ...) for the three
// tile buffers b = t % 3, dQ [384, 512); dS(t) (bf16 pairs) over the first
// 32 columns of S(t)'s buffer. One CTA per SM (512 columns) with three dS
// warpgroups: warpgroup w takes the tiles t = w mod 3 (and buffer w), and a
// run of the dQ columns in the epilogue. The MMA warp computes S and dP two
// tiles ahead, so a warpgroup that finishes a tile finds its next one ready.
//
// SLA2 = true adds the linear branch's query gradient (SLA2 article,
// arXiv:2602.12675, sections 1 and 2). With c_i = (1 - alpha_h) / den_i,
// f_i = dO_i . O_l,i (den_i, O_l from the forward's linear branch) and the
// complement of i's kept keys,
//   dphi(q_i) = c_i sum_{j not kept} (dP_ij - f_i) phi(k_j) = c_i (S_c dO_i - f_i z_c)
// with S_c, z_c the complement summaries of i's query block, which
// linear_out_kernel forms anyway (it stores them for the backward: S_c as a
// bf16 [128][128] tile per block). After the last dQ product the MMA warp
// adds L = dO S_c^T (one M 128, N 128, K 128 product) into the S columns
// [0, 128), which every dQ product has read by then, and the epilogue forms
//   dq_i = scale * dQ_i + c_i (L_i - f_i z_c) * phi'(q_i).
// The sparse part uses alpha_h dO: dS = P (alpha_h dP - D_i), D_i = alpha_h dO_i . O_s,i.
// ---------------------------------------------------------------------------
// dS warpgroups of the dQ kernel: three (each takes every third tile and owns
// one of the three S / dP buffers; dS is formed half a tile at a time so 448
// threads fit the register file).
template <bool SLA2>
__host__ __device__ constexpr int bwd_q_wgs() { return 3; }
template <bool SLA2>
__host__ __device__ constexpr int bwd_q_threads() { return 64 + 128 * bwd_q_wgs<SLA2>(); }

// dS = P (a dP - D) for 32 keys (half a tile) of the sparse branch, read
// from TMEM at the given S and dP columns; 16 bf16 pairs out. a = 1, or
// alpha_h in the SLA2 backward.
__device__ __forceinline__ void ds_half(uint32_t ts, uint32_t tp, float scale_log2, float lse2, float Di, float a,
                                        int key0, int N, bool row_ok, uint32_t (&pds)[16]) {
  uint32_t sv[2][16], pv[2][16];
  tmem_ld16(ts, sv[0]);
  tmem_ld16(ts + 16, sv[1]);
  tmem_ld16(tp, pv[0]);
  tmem_ld16(tp + 16, pv[1]);
  tmem_ld_wait();
  const uint64_t sc2 = f2(scale_log2, scale_log2), nl2 = f2(-lse2, -lse2), nd2 = f2(-Di, -Di), a2 = f2(a, a);
  const bool tail = key0 + 32 > N;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int h = k / 8, c = (2 * k) % 16;
    const float2 x = f2_split(fma2(f2(__uint_as_float(sv[h][c]), __uint_as_float(sv[h][c + 1])), sc2, nl2));
    float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
    if (!row_ok || (tail && key0 + 2 * k >= N)) p0 = 0.0f;
    if (!row_ok || (tail && key0 + 2 * k + 1 >= N)) p1 = 0.0f;
    const float2 g = f2_split(fma2(f2(__uint_as_float(pv[h][c]), __uint_as_float(pv[h][c + 1])), a2, nd2));
    pds[k] = pack_bf16x2(p0 * g.x, p1 * g.y);
  }
}

template <int D, bool SLA2>
struct BwdQSmem {
  // K(t) is held until dQ(t) has read it, one softmax period after S(t): a
  // four-slot K ring keeps its loads two tiles ahead. V(t) frees after dP(t).
  // SLA2: the query block's bf16 S_c tile sits after dO.
  static constexpr int NB = 3;
  static constexpr int NSK = 4, NSV = 2;
  static constexpr int kQBytes = kTileQ * D * 2;
  static constexpr int kKBytes = kTileK * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kOffQ + kQBytes;
  static constexpr int kOffSc = kOffDO + kQBytes;
  static constexpr int kOffK = kOffSc + (SLA2 ? kQBytes : 0);
  static constexpr int kOffV = kOffK + NSK * kKBytes;
  static constexpr int kOffBar = kOffV + NSV * kKBytes;
  static constexpr int kBarIn = 0, kBarKFull = 1, kBarKEmpty = 1 + NSK, kBarVFull = 1 + 2 * NSK,
                       kBarVEmpty = 1 + 2 * NSK + NSV, kBarSFull = 1 + 2 * NSK + 2 * NSV,
                       kBarPFull = kBarSFull + NB, kBarFinal = kBarPFull + NB, kBarDrain = kBarFinal + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffTmem + 16 + 1024;  // + room to align the base to 1024
  static constexpr int kTmemCols = 512;
};

// Per-row inputs of the SLA2 backward (null for the sparse branch alone).
struct BwdLinParams {
  const float* alpha;  // [H]
  const float* cw;     // [BH, N] c_i
  const float* fw;     // [BH, N] f_i
  const float* zc;     // [BH * nqb, d] z_c of each query block
  int H;
};

template <int D, bool SLA2>
__global__ void __launch_bounds__(bwd_q_threads<SLA2>(), 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmSc,
                       const BwdParams p, const BwdLinParams lp) {
  using L = BwdQSmem<D, SLA2>;
  constexpr int NSK = L::NSK, NSV = L::NSV, NB = L::NB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t sQ = sbase + L::kOffQ, sDO = sbase + L::kOffDO, sK = sbase + L::kOffK, sV = sbase + L::kOffV;
  const uint32_t sSc = sbase + L::kOffSc;
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffTmem + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = p.order ? __ldg(p.order + blockIdx.x) : (int)blockIdx.x;  // (bh, query block)
  const int bh = tile / p.nqb;
  const int q0 = (tile % p.nqb) * p.bq;
  const int tiles_per_block = p.bk / kTileK;
  const int cnt = min(max(__ldg(p.cnt + tile), 0), p.nkb);
  const int T = cnt * tiles_per_block;
  const int32_t* lst = p.lst + (int64_t)tile * p.nkb;
  const bool work = T > 0 || SLA2;  // the linear branch has a term even when nothing is kept

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarIn), 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(bar(L::kBarKFull + s), 1);
      mbar_init(bar(L::kBarKEmpty + s), 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(bar(L::kBarVFull + s), 1);
      mbar_init(bar(L::kBarVEmpty + s), 1);
    }
    for (int s = 0; s < NB; ++s) {
      mbar_init(bar(L::kBarSFull + s), 1);
      mbar_init(bar(L::kBarPFull + s), 128);
    }
    mbar_init(bar(L::kBarFinal), 1);
    mbar_init(bar(L::kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::kOffTmem, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 64 * NB, tQ = tmem + 128 * NB;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp walks the list (indices by shuffle); lane 0 waits and issues.
    if (work) {
      int nk = 0, nv = 0;
      bool ok = true;
      if (lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        mbar_arrive_expect_tx(bar(L::kBarIn), (SLA2 ? 3 : 2) * L::kQBytes);
        for (int b = 0; b < D / 64; ++b) {
          tma_load_3d(sQ + b * (kTileQ * 128), &tmQ, bar(L::kBarIn), b * 64, q0, bh);
          tma_load_3d(sDO + b * (kTileQ * 128), &tmDO, bar(L::kBarIn), b * 64, q0, bh);
          if (SLA2) tma_load_3d(sSc + b * (kTileQ * 128), &tmSc, bar(L::kBarIn), b * 64, 0, tile);
        }
      }
      ListChunks lc(lst, cnt, lane);
      for (int t = 0; t < T; ++t) {
        const int key0 = lc.get(lst, cnt, t / tiles_per_block, lane) * p.bk + (t % tiles_per_block) * kTileK;
        if (lane == 0) {
          const int ks = t % NSK, vs = t % NSV;
          // V(t) feeds dP(t) only, so its slot frees early; K(t) also feeds dQ(t).
          ok = t < NSV || role_wait(bar(L::kBarVEmpty + vs), (t / NSV - 1) & 1, kErrBwdVEmpty, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(bar(L::kBarVFull + vs), L::kKBytes);
            for (int b = 0; b < D / 64; ++b)
              tma_load_3d(sV + vs * L::kKBytes + b * (kTileK * 128), &tmV, bar(L::kBarVFull + vs), b * 64, key0,
                          bh);
            ++nv;
            ok = t < NSK || role_wait(bar(L::kBarKEmpty + ks), (t / NSK - 1) & 1, kErrBwdKEmpty, abort_flag);
          }
          if (ok) {
            mbar_arrive_expect_tx(bar(L::kBarKFull + ks), L::kKBytes);
            for (int b = 0; b < D / 64; ++b)
              tma_load_3d(sK + ks * L::kKBytes + b * (kTileK * 128), &tmK, bar(L::kBarKFull + ks), b * 64, key0,
                          bh);
            ++nk;
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      // Never leave with copies in flight.
      if (lane == 0) {
        mbar_wait(bar(L::kBarIn), 0, kErrBwdIn);
        for (int t = (nk > NSK ? nk - NSK : 0); t < nk; ++t)
          mbar_wait(bar(L::kBarKFull + t % NSK), (t / NSK) & 1, kErrBwdKFull);
        for (int t = (nv > NSV ? nv - NSV : 0); t < nv; ++t)
          mbar_wait(bar(L::kBarVFull + t % NSV), (t / NSV) & 1, kErrBwdVFull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (work) {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_bf16_f32(kTileQ, kTileK, false, false);
      constexpr uint32_t idQ = idesc_bf16_f32(kTileQ, D, false, true);
      constexpr uint32_t idL = idesc_bf16_f32(kTileQ, D, false, false);
      const uint64_t dQd = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dDO = sdesc_sw128(sDO, 16, 1024);
      const uint64_t dSc = sdesc_sw128(sSc, 16, 1024);               // K-major B (row = feature)
      const uint64_t dK = sdesc_sw128(sK, 16, 1024);                // K-major (S = Q K^T)
      const uint64_t dKmn = sdesc_sw128(sK, kTileK * 128, 1024);    // MN-major (dQ += dS K)
      const uint64_t dV = sdesc_sw128(sV, 16, 1024);                // K-major (dP = dO V^T)
      auto warp_wait = [&](int b, uint32_t parity, unsigned int site) {
        return __all_sync(0xffffffffu, role_wait(bar(b), parity, site, abort_flag));
      };
      bool ok = warp_wait(L::kBarIn, 0, kErrBwdIn);
      tc_fence_after();
      // S(t) and dP(t) run NB - 1 tiles ahead of dQ(t): buffer t % NB was last
      // read by dQ(t - NB), issued (and its dS written) before.
      for (int t = 0; ok && t < T + NB - 1; ++t) {
        if (t < T) {
          const int ks = t % NSK, vs = t % NSV, b = t % NB;
          ok = warp_wait(L::kBarKFull + ks, (t / NSK) & 1, kErrBwdKFull) &&
               warp_wait(L::kBarVFull + vs, (t / NSV) & 1, kErrBwdVFull);
          if (!ok) break;
          tc_fence_after();
          if (leader) {
            const uint64_t dKs = dK + (uint64_t)((ks * L::kKBytes) >> 4);
            const uint64_t dVs = dV + (uint64_t)((vs * L::kKBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t qo = ((kk >> 2) * (kTileQ * 128) + (kk & 3) * 32) >> 4;
              const uint32_t ko = ((kk >> 2) * (kTileK * 128) + (kk & 3) * 32) >> 4;
              mma_ss(tS + b * 64, dQd + qo, dKs + ko, idS, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t qo = ((kk >> 2) * (kTileQ * 128) + (kk & 3) * 32) >> 4;
              const uint32_t ko = ((kk >> 2) * (kTileK * 128) + (kk & 3) * 32) >> 4;
              mma_ss(tP + b * 64, dDO + qo, dVs + ko, idS, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar(L::kBarSFull + b));
            mma_commit(bar(L::kBarVEmpty + vs));
          }
          __syncwarp();
        }
        if (t >= NB - 1) {
          const int u = t - (NB - 1), ks = u % NSK, b = u % NB;
          ok = warp_wait(L::kBarPFull + b, (u / NB) & 1, kErrBwdPFull);
          if (!ok) break;
          tc_fence_after();
          if (leader) {
            const uint64_t dKm = dKmn + (uint64_t)((ks * L::kKBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk)  // 16 keys = 2048 bytes of K = 8 packed dS columns
              mma_ts(tQ, tS + b * 64 + kk * 8, dKm + kk * 128, idQ, (u > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar(L::kBarKEmpty + ks));
            if (!SLA2 && u == T - 1) mma_commit(bar(L::kBarFinal));
          }
          __syncwarp();
        }
      }
      if (SLA2 && ok) {
        // L = dO S_c^T into the S columns [0, 128): every dS there has been
        // read by a dQ product issued before this one.
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qo = ((kk >> 2) * (kTileQ * 128) + (kk & 3) * 32) >> 4;
            mma_ss(tS, dDO + qo, dSc + qo, idL, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(L::kBarFinal));
        }
        __syncwarp();
      }
      if (leader) mma_commit(bar(L::kBarDrain));
      __syncwarp();
      mbar_wait(bar(L::kBarDrain), 0, kErrBwdDrain);
    }
  } else {
    // ------------------------------------------------------------ dS + epilogue
    constexpr int WG = bwd_q_wgs<SLA2>();
    const int wg = (warp - 2) >> 2;  // takes tiles wg, wg + WG, ...
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool row_ok = r < p.bq && q0 + r < p.N;
    const int64_t grow = (int64_t)bh * p.N + q0 + r;
    const float lse2 = row_ok ? __ldg(p.lse + grow) * 1.4426950408889634f : 0.0f;
    const float Di = row_ok ? __ldg(p.dsum + grow) : 0.0f;
    const float a_h = SLA2 ? __ldg(lp.alpha + (bh % lp.H)) : 1.0f;
    const float fi = SLA2 && row_ok ? __ldg(lp.fw + grow) : 0.0f;
    const float ci = SLA2 && row_ok ? __ldg(lp.cw + grow) : 0.0f;
    bool ok = true;
    ListChunks lc(lst, cnt, lane);
    for (int t = wg; t < T; t += WG) {
      const int b = t % NB;
      const int key0 = lc.get(lst, cnt, t / tiles_per_block, lane) * p.bk + (t % tiles_per_block) * kTileK;
      ok = __all_sync(0xffffffffu, role_wait(bar(L::kBarSFull + b), (t / NB) & 1, kErrBwdSFull, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // Half a tile at a time; the half written back (columns 16h..16h+15 of
      // S) holds S values already read.
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pds[16];
        ds_half(tS + lane_off + b * 64 + 32 * h, tP + lane_off + b * 64 + 32 * h, p.scale_log2, lse2, Di, a_h,
                key0 + 32 * h, p.N, row_ok, pds);
        tmem_st16(tS + lane_off + b * 64 + 16 * h, pds);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarPFull + b));
    }
    if (ok && work) {
      ok = __all_sync(0xffffffffu, role_wait(bar(L::kBarFinal), 0, kErrBwdFinal, abort_flag));
      tc_fence_after();
    }
    // Epilogue: scale * dQ (+ the linear term) -> bf16 -> Q buffer (free: every
    // MMA is done) -> TMA store; warpgroup wg takes a run of 16-column groups.
    constexpr int kCols = (D / 16 + WG - 1) / WG * 16;
#pragma unroll 1
    for (int c = wg * kCols; c < min(D, (wg + 1) * kCols); c += 16) {
      uint32_t v[16];
      if (T > 0 && ok) {
        tmem_ld16(tQ + lane_off + c, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
      float o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = __uint_as_float(v[j]) * p.scale;
      if (SLA2) {
        uint32_t l[16];
        if (ok) {
          tmem_ld16(tS + lane_off + c, l);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) l[j] = 0u;
        }
        float qv[16];
        read_row16(sQ, r, c, qv);
        const float* z = lp.zc + (int64_t)tile * D + c;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float dphi = ci * (__uint_as_float(l[j]) - fi * __ldg(z + j));
          o[j] += dphi * (qv[j] > 0.0f ? 1.0f : __expf(qv[j]));
        }
      }
      stage_row16(sQ, r, c, o);
    }
    fence_async_smem();
    asm volatile("bar.sync 1, %0;" ::"n"(128 * WG) : "memory");
    if (warp == 2 && lane == 0) {
      for (int b = 0; b < D / 64; ++b) tma_store_3d(&tmDQ, sQ + b * (kTileQ * 128), b * 64, q0, bh);
      tma_store_commit();
      tma_store_wait_read0();  // the staging tile has been read: the CTA may end
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// dK, dV: one CTA per (bh, 64-key tile), walking the query blocks that keep
// the tile's block (lists from mask_transpose_kernel). Per query tile u:
//   S(u) = Q_u K^T, dP(u) = dO_u V^T             (M = 128 query rows, N = 64)
//   P(u), dS(u) -> bf16 staging tiles [128 rows][64 keys] (shared memory)
//   dV^T += dO_u^T P(u), dK^T += Q_u^T dS(u)     (M = 128 channels, N = 64, K = 128 rows)
// TMEM columns: S(b) [64b, 64b+64), dP(b) [128+64b, 192+64b), dV^T [256, 320),
// dK^T [320, 384). One CTA per SM (512 columns).
//
// MODE 0: the sparse branch alone; bf16 dK, dV.
// MODE 1: the sparse part of the SLA2 backward: dV stages alpha_h P, dS uses
//         alpha_h dP (D_i already carries alpha_h); fp32 partials out.
// (linear_dkdv_kernel then adds the linear branch's dK, dV to the MODE 1
// partials.)
// ---------------------------------------------------------------------------
template <int D>
struct BwdKVSmem {
  static constexpr int NS = 2;
  static constexpr int kQBytes = kTileQ * D * 2;   // Q_u or dO_u
  static constexpr int kKBytes = kTileK * D * 2;   // K or V of the key tile
  static constexpr int kSlot = 2 * kQBytes;        // Q_u then dO_u
  static constexpr int kStBytes = kTileQ * kTileK * 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKBytes;
  static constexpr int kOffRing = kOffV + kKBytes;
  static constexpr int kOffP = kOffRing + NS * kSlot;
  static constexpr int kOffDS = kOffP + kStBytes;  // P and dS staging: together one [128][128] tile
  static constexpr int kOffBar = kOffDS + kStBytes;
  // Q_u and dO_u have their own barriers: dO_u frees after dV(u), Q_u after
  // dK(u), so the next loads into the slot start as early as possible.
  static constexpr int kBarKV = 0, kBarQFull = 1, kBarDOFull = 1 + NS, kBarQEmpty = 1 + 2 * NS,
                       kBarDOEmpty = 1 + 3 * NS, kBarSFull = 1 + 4 * NS, kBarPReady = 3 + 4 * NS,
                       kBarStage = 4 + 4 * NS, kBarFinal = 5 + 4 * NS, kBarDrain = 6 + 4 * NS;
  static constexpr int kNumBars = 7 + 4 * NS;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffTmem + 16 + 1024;
  static constexpr int kTmemCols = 512;
};

// 64 bf16 (pairs in pk) as row r of a [128 rows][64 columns] tile with the
// 128-byte swizzle: the MN-major operand layout of a 64-wide N.
__device__ __forceinline__ void stage_row64(uint32_t tile, int r, const uint32_t (&pk)[kTileK / 2]) {
  const uint32_t row_addr = tile + r * 128;
#pragma unroll
  for (int ch = 0; ch < 8; ++ch)
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_addr + ((ch ^ (r & 7)) * 16)),
                 "r"(pk[4 * ch]), "r"(pk[4 * ch + 1]), "r"(pk[4 * ch + 2]), "r"(pk[4 * ch + 3])
                 : "memory");
}

// Column c of a [64 keys][D] bf16 tile in TMA layout (64-column boxes of 64
// rows, 128-byte swizzle) from the thread's 64 values, scaled by f.
template <int D>
__device__ __forceinline__ void stage_col64(uint32_t tile, int c, const float (&v)[kTileK], float f) {
  const uint32_t base = tile + (c / 64) * (kTileK * 128) + (c % 8) * 2;
  const int cc = (c % 64) / 8;
#pragma unroll
  for (int j = 0; j < kTileK; ++j) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v[j] * f);
    const uint16_t u = *reinterpret_cast<const uint16_t*>(&h);
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(base + j * 128 + ((cc ^ (j & 7)) * 16)), "h"(u) : "memory");
  }
}

// Element (row j, column c) of such a tile, as float.
__device__ __forceinline__ float tile_at(const uint8_t* tile, int j, int c) {
  const int cc = (c % 64) / 8;
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
      tile + (c / 64) * (kTileK * 128) + j * 128 + ((cc ^ (j & 7)) * 16) + (c % 8) * 2));
}

// Inputs and outputs of the SLA2 mode of the dK/dV kernel.
struct BwdKVLin {
  const float* alpha;   // [H] (MODE 1)
  float* dk_part;       // [BH, N, d] fp32: MODE 1 writes scale * dK_sparse
  float* dv_part;       // [BH, N, d] fp32: MODE 1 writes dV_sparse
  int H;
};

template <int D, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                         const BwdParams p, const BwdKVLin lk) {
  using L = BwdKVSmem<D>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t sK = sbase + L::kOffK, sV = sbase + L::kOffV, sRing = sbase + L::kOffRing;
  const uint32_t sP = sbase + L::kOffP, sDS = sbase + L::kOffDS;
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffTmem + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nkt = (p.N + kTileK - 1) / kTileK;
  const int bh = blockIdx.x / nkt;               // head-major: consecutive CTAs share a head's Q and dO
  const int kt = blockIdx.x % nkt;
  const int key0 = kt * kTileK;
  const int64_t jrow = (int64_t)bh * p.nkb + key0 / p.bk;  // (bh, key block)
  const int T = min(max(__ldg(p.cnt + jrow), 0), p.nqb);
  const int32_t* lst = p.lst + jrow * p.nqb;
  const bool work = T > 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarKV), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::kBarQFull + s), 1);
      mbar_init(bar(L::kBarDOFull + s), 1);
      mbar_init(bar(L::kBarQEmpty + s), 1);
      mbar_init(bar(L::kBarDOEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) mbar_init(bar(L::kBarSFull + s), 1);
    mbar_init(bar(L::kBarPReady), 128);
    mbar_init(bar(L::kBarStage), 1);
    mbar_init(bar(L::kBarFinal), 1);
    mbar_init(bar(L::kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::kOffTmem, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 128, tDV = tmem + 256, tDK = tmem + 320;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp walks the list (indices by shuffle); lane 0 waits and issues.
    if (work) {
      int n_in = 0;
      bool ok = true;
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmDO);
        mbar_arrive_expect_tx(bar(L::kBarKV), 2 * L::kKBytes);
        for (int b = 0; b < D / 64; ++b) {
          tma_load_3d(sK + b * (kTileK * 128), &tmK, bar(L::kBarKV), b * 64, key0, bh);
          tma_load_3d(sV + b * (kTileK * 128), &tmV, bar(L::kBarKV), b * 64, key0, bh);
        }
      }
      ListChunks lc(lst, T, lane);
      int n_do = 0;
      for (int t = 0; t < T; ++t) {
        const int q0 = lc.get(lst, T, t, lane) * p.bq;
        if (lane == 0) {
          const int slot = t % NS, round = t / NS;
          const uint32_t dst = sRing + slot * L::kSlot;
          ok = t < NS || role_wait(bar(L::kBarDOEmpty + slot), (round - 1) & 1, kErrBwdInEmpty, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(bar(L::kBarDOFull + slot), L::kQBytes);
            for (int b = 0; b < D / 64; ++b)
              tma_load_3d(dst + L::kQBytes + b * (kTileQ * 128), &tmDO, bar(L::kBarDOFull + slot), b * 64, q0, bh);
            ++n_do;
            ok = t < NS || role_wait(bar(L::kBarQEmpty + slot), (round - 1) & 1, kErrBwdInEmpty, abort_flag);
          }
          if (ok) {
            mbar_arrive_expect_tx(bar(L::kBarQFull + slot), L::kQBytes);
            for (int b = 0; b < D / 64; ++b)
              tma_load_3d(dst + b * (kTileQ * 128), &tmQ, bar(L::kBarQFull + slot), b * 64, q0, bh);
            ++n_in;
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      if (lane == 0) {
        mbar_wait(bar(L::kBarKV), 0, kErrBwdKV);
        for (int t = (n_in > NS ? n_in - NS : 0); t < n_in; ++t)
          mbar_wait(bar(L::kBarQFull + t % NS), (t / NS) & 1, kErrBwdIn);
        for (int t = (n_do > NS ? n_do - NS : 0); t < n_do; ++t)
          mbar_wait(bar(L::kBarDOFull + t % NS), (t / NS) & 1, kErrBwdIn);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (work) {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_bf16_f32(kTileQ, kTileK, false, false);
      constexpr uint32_t idT = idesc_bf16_f32(D, kTileK, true, true);
      const uint64_t dRingK = sdesc_sw128(sRing, 16, 1024);               // Q_u, dO_u as K-major A
      const uint64_t dRingM = sdesc_sw128(sRing, kTileQ * 128, 1024);     // Q_u, dO_u as MN-major A
      const uint64_t dK = sdesc_sw128(sK, 16, 1024);
      const uint64_t dV = sdesc_sw128(sV, 16, 1024);
      const uint64_t dPst = sdesc_sw128(sP, kTileQ * 128, 1024);          // MN-major B, one 64-wide atom
      const uint64_t dDSst = sdesc_sw128(sDS, kTileQ * 128, 1024);
      auto warp_wait = [&](int b, uint32_t parity, unsigned int site) {
        return __all_sync(0xffffffffu, role_wait(bar(b), parity, site, abort_flag));
      };
      // dP(t) and S(t) for tile t into TMEM buffer t & 1.
      auto issue_sdp = [&](int t) -> bool {
        const int slot = t % NS, b = t & 1;
        const uint32_t so = (uint32_t)((slot * L::kSlot) >> 4);
        const uint32_t doo = (uint32_t)((slot * L::kSlot + L::kQBytes) >> 4);
        if (!warp_wait(L::kBarDOFull + slot, (t / NS) & 1, kErrBwdIn)) return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qo = ((kk >> 2) * (kTileQ * 128) + (kk & 3) * 32) >> 4;
            const uint32_t ko = ((kk >> 2) * (kTileK * 128) + (kk & 3) * 32) >> 4;
            mma_ss(tP + b * 64, dRingK + doo + qo, dV + ko, idS, kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
        if (!warp_wait(L::kBarQFull + slot, (t / NS) & 1, kErrBwdIn)) return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qo = ((kk >> 2) * (kTileQ * 128) + (kk & 3) * 32) >> 4;
            const uint32_t ko = ((kk >> 2) * (kTileK * 128) + (kk & 3) * 32) >> 4;
            mma_ss(tS + b * 64, dRingK + so + qo, dK + ko, idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(L::kBarSFull + b));
        }
        __syncwarp();
        return true;
      };
      bool ok = warp_wait(L::kBarKV, 0, kErrBwdKV);
      tc_fence_after();
      // S and dP run two tiles ahead; dV(u) and dK(u) are issued as soon as
      // P(u) and dS(u) are staged, before the loads of tile u + 2 are awaited.
      for (int t = 0; ok && t < T && t < 2; ++t) ok = issue_sdp(t);
      for (int u = 0; ok && u < T; ++u) {
        const int slot = u % NS;
        if (!warp_wait(L::kBarPReady, u & 1, kErrBwdPFull)) break;
        tc_fence_after();
        if (leader) {
          const uint32_t so = (uint32_t)((slot * L::kSlot) >> 4);
          const uint32_t doo = (uint32_t)((slot * L::kSlot + L::kQBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kTileQ / 16; ++kk)  // 16 query rows = 2048 bytes of each operand
            mma_ss(tDV, dRingM + doo + kk * 128, dPst + kk * 128, idT, (u > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::kBarDOEmpty + slot));
#pragma unroll
          for (int kk = 0; kk < kTileQ / 16; ++kk)
            mma_ss(tDK, dRingM + so + kk * 128, dDSst + kk * 128, idT, (u > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::kBarQEmpty + slot));
          mma_commit(bar(L::kBarStage));
          if (u == T - 1) mma_commit(bar(L::kBarFinal));
        }
        __syncwarp();
        if (u + 2 < T) ok = issue_sdp(u + 2);
      }
      if (leader) mma_commit(bar(L::kBarDrain));
      __syncwarp();
      mbar_wait(bar(L::kBarDrain), 0, kErrBwdDrain);
    }
  } else {
    // ------------------------------------------------------------ staging + epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;  // query row of the tile; in the epilogue, the channel
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float a_h = MODE == 1 ? __ldg(lk.alpha + (bh % lk.H)) : 1.0f;
    bool ok = true;
    ListChunks lc(lst, T, lane);
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      const int q0 = lc.get(lst, T, t, lane) * p.bq;
      const bool row_ok = r < p.bq && q0 + r < p.N;
      const int64_t grow = (int64_t)bh * p.N + q0 + r;
      // lse and D of the row.
      const float x0 = row_ok ? __ldg(p.lse + grow) : 0.0f;
      const float x1 = row_ok ? __ldg(p.dsum + grow) : 0.0f;
      ok = __all_sync(0xffffffffu, role_wait(bar(L::kBarSFull + b), (t >> 1) & 1, kErrBwdSFull, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float s[kTileK], dp[kTileK];
      load_row64(tS + lane_off + b * 64, s);
      load_row64(tP + lane_off + b * 64, dp);
      uint32_t pp[kTileK / 2], pds[kTileK / 2];
      p_and_ds(s, dp, p.scale_log2, x0 * 1.4426950408889634f, x1, a_h, key0, p.N, row_ok, pp, pds);
      // The staging tiles are free once the MMAs of the previous tile have
      // read them.
      if (t > 0) {
        ok = __all_sync(0xffffffffu, role_wait(bar(L::kBarStage), (t - 1) & 1, kErrBwdStage, abort_flag));
        if (!ok) break;
      }
      stage_row64(sP, r, pp);
      stage_row64(sDS, r, pds);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(L::kBarPReady));
    }
    if (ok && work) {
      ok = __all_sync(0xffffffffu, role_wait(bar(L::kBarFinal), 0, kErrBwdFinal, abort_flag));
      tc_fence_after();
    }
    // Epilogue: lane r holds channel r of dV^T and dK^T (keys along the columns).
    const uint32_t sOutV = sRing, sOutK = sRing + L::kKBytes;
    float v[kTileK];
    if (work && ok) {
      load_row64(tDV + lane_off, v);
    } else {
#pragma unroll
      for (int j = 0; j < kTileK; ++j) v[j] = 0.0f;
    }
    const int64_t obase = ((int64_t)bh * p.N + key0) * D + r;
    const int nvalid = min(kTileK, p.N - key0);
    if (MODE == 1) {
#pragma unroll
      for (int j = 0; j < kTileK; ++j)
        if (j < nvalid) lk.dv_part[obase + (int64_t)j * D] = v[j];
    } else {
      stage_col64<D>(sOutV, r, v, 1.0f);
    }
    if (work && ok) {
      load_row64(tDK + lane_off, v);
    } else {
#pragma unroll
      for (int j = 0; j < kTileK; ++j) v[j] = 0.0f;
    }
    if (MODE == 1) {
#pragma unroll
      for (int j = 0; j < kTileK; ++j)
        if (j < nvalid) lk.dk_part[obase + (int64_t)j * D] = v[j] * p.scale;
    } else {
      stage_col64<D>(sOutK, r, v, p.scale);
    }
    if (MODE == 0) {
      fence_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (warp == 2 && lane == 0) {
        for (int b = 0; b < D / 64; ++b) {
          tma_store_3d(&tmDV, sOutV + b * (kTileK * 128), b * 64, key0, bh);
          tma_store_3d(&tmDK, sOutK + b * (kTileK * 128), b * 64, key0, bh);
        }
        tma_store_commit();
        tma_store_wait_read0();  // the staging tile has been read: the CTA may end
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace sparge
