// Block-sparse attention forward on the 5th-generation tensor cores.
//
// What it computes (SpargeAttention2 article, arXiv:2602.13515, section 4:
// attention runs block by block and each block is either fully computed or
// fully skipped; SLA2 article, arXiv:2602.12675, section 2: the sparse branch
// is renormalised over the kept region only):
//   O[i] = sum_{j in kept keys of block(i)} softmax_j(q_i . k_j / sqrt(d)) v_j
//
// One CTA owns one 128-row query tile of one (batch, head) and walks only the
// key tiles (64 keys each) of that tile's kept blocks:
//   warp 0      TMA producer: Q once, then K and V tiles into two 2-slot rings;
//   warp 1      MMA issuer and TMEM owner: S = Q K^T into a double-buffered
//               TMEM S, then O += P V with P read back from TMEM;
//   warps 2..5  softmax: one query row per thread (TMEM lane), fp32 online
//               softmax with lazy rescaling, P written to TMEM as bf16 over
//               its own S columns; then the epilogue (O / l -> bf16 -> TMA
//               store, optional log-sum-exp).
// TMEM columns: S0 [0,64), S1 [64,128), O [128,128+D); P(t) (bf16, two per
// 32-bit column) is written over the first 32 columns of S(t)'s buffer.
//
// With MIX = true the kernel finishes the sparse + linear mix of the SLA2
// article (arXiv:2602.12675, section 2), O = alpha_h O_sparse +
// (1 - alpha_h) O_linear: linear_out_kernel has already written
// (1 - alpha_h) O_linear into O (bf16); the producer loads that tile into the
// Q buffer once the last S MMA has read Q, and the epilogue adds
// alpha_h O_sparse before storing the tile back.
#pragma once
#include <cuda.h>
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparge {

constexpr int kAttnThreads = 192;
constexpr int kTileQ = 128;   // query rows per MMA tile
constexpr int kTileK = 64;    // keys per MMA tile
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8
// Of the 64 exponentials per row and full key tile, 2 * kPolyPairs run on the
// FMA and integer pipes (exp2_poly2) and the rest on the MUFU (ex2.approx).
// The MUFU's 16 results per clock and SM take as long per tile as the tile's
// two MMAs, but moving 16 or 24 of the 64 to the polynomial measured no faster
// on B200 (the softmax chain is bound by latency as much as by the MUFU), so
// the default keeps them all on the MUFU. Tail tiles (keys past N, scores
// -inf) always use the MUFU.
#ifndef SPARGE_POLY_PAIRS
#define SPARGE_POLY_PAIRS 0
#endif
constexpr int kPolyPairs = SPARGE_POLY_PAIRS;

// Error site codes recorded in g_device_error by the attention kernel.
enum : unsigned int {
  kErrAttnQ = 0x100, kErrAttnKFull, kErrAttnVFull, kErrAttnKEmpty, kErrAttnVEmpty, kErrAttnSFull,
  kErrAttnPFull, kErrAttnODone, kErrAttnOFinal, kErrAttnDrain, kErrAttnOl
};

struct AttnParams {
  const int32_t* kv_idx;  // [BH, nqb, nkb]
  const int32_t* kv_cnt;  // [BH, nqb]
  const int32_t* order;   // [BH * nqb] launch order of the tiles, or null (head-major)
  float* lse;             // [BH, N] or null
  const float* alpha;     // MIX: [H]
  int H;
  int N;
  int nqb;
  int nkb;
  int bq;                 // 64 or 128: rows of the query block that share a mask row
  int bk;                 // 64 or 128: keys per mask block (bk / 64 key tiles each)
  float scale_log2;       // log2(e) / sqrt(d)
};

template <int D, bool MIX>
struct AttnSmem {
  // K / V ring depth: two slots keep the kernel small enough for two CTAs per SM.
  static constexpr int NS = 2;
  static constexpr int kQBytes = kTileQ * D * 2;
  static constexpr int kKBytes = kTileK * D * 2;
  static constexpr int kVBytes = kTileK * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + NS * kKBytes;
  static constexpr int kOffBar = kOffV + NS * kVBytes;
  // Barrier slots: K full / V full / K empty / V empty rings, S full and
  // P full pairs, then single barriers.
  static constexpr int kBarQ = 0, kBarKFull = 1, kBarVFull = 1 + NS, kBarKEmpty = 1 + 2 * NS,
                       kBarVEmpty = 1 + 3 * NS, kBarSFull = 1 + 4 * NS, kBarPFull = 3 + 4 * NS,
                       kBarODone = 5 + 4 * NS, kBarOFinal = 6 + 4 * NS, kBarDrain = 7 + 4 * NS,
                       kBarOl = 8 + 4 * NS;
  static constexpr int kNumBars = 9 + 4 * NS;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kUsed = kOffTmem + 16;
  // Pad so that at most two CTAs fit on an SM: two CTAs x 256 TMEM columns
  // use the SM's 512 columns exactly, and a third would block in alloc.
  static constexpr int kBytes = (kUsed + 1024 > 80 * 1024 ? kUsed + 1024 : 80 * 1024);
  static constexpr int kTmemCols = 256;
};

// ---------------------------------------------------------------- softmax tile
// One thread = one query row (its TMEM lane); a tile = 64 keys.

// The row's 64 scores of S from TMEM (taddr includes the warp's lane offset).
__device__ __forceinline__ void load_scores(uint32_t taddr, float (&s)[kTileK]) {
  uint32_t v[4][16];
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld16(taddr + 16 * c, v[c]);
  tmem_ld_wait();
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int j = 0; j < 16; ++j) s[16 * c + j] = __uint_as_float(v[c][j]);
}

// Keys at or past N score -inf.
__device__ __forceinline__ void mask_tail(float (&s)[kTileK], int key0, int N) {
  if (key0 + kTileK > N) {
#pragma unroll
    for (int j = 0; j < kTileK; ++j)
      if (key0 + j >= N) s[j] = -INFINITY;
  }
}

// Three-operand max tree: 36 instructions, depth 4.
__device__ __forceinline__ float row_max64(const float (&s)[kTileK]) {
  float m8[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    m8[j] = fmax3(fmax3(s[j], s[8 + j], s[16 + j]), fmax3(s[24 + j], s[32 + j], s[40 + j]), fmaxf(s[48 + j], s[56 + j]));
  return fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
}

// Multiplies the row's D accumulator columns at taddr by f.
template <int D>
__device__ __forceinline__ void rescale_row(uint32_t taddr, float f) {
  uint32_t v[16];
#pragma unroll 1
  for (int c = 0; c < D; c += 16) {
    tmem_ld16(taddr + c, v);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
    tmem_st16(taddr + c, v);
  }
  tmem_st_wait();
}

// p_j = 2^(s_j * scale_log2 - m) packed as bf16 pairs into pk; returns the
// sum of the p_j in fp32. Pair instructions throughout but the MUFU; the
// first 2 * NPOLY values take the polynomial exp2 instead.
template <int NPOLY>
__device__ __forceinline__ float exp_pack(const float (&s)[kTileK], float scale_log2, float m,
                                          uint32_t (&pk)[kTileK / 2]) {
  const uint64_t scale2 = f2(scale_log2, scale_log2), negm2 = f2(-m, -m);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};  // four pair sums: short dependency chains
#pragma unroll
  for (int k = 0; k < kTileK / 2; ++k) {
    const uint64_t x = fma2(f2(s[2 * k], s[2 * k + 1]), scale2, negm2);
    uint64_t e;
    if (k < NPOLY) {
      e = exp2_poly2(x);
    } else {
      const float2 xv = f2_split(x);
      e = f2(ex2_approx(xv.x), ex2_approx(xv.y));
    }
    acc[k & 3] = add2(acc[k & 3], e);
    const float2 ev = f2_split(e);
    pk[k] = pack_bf16x2(ev.x, ev.y);
  }
  const float2 a = f2_split(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])));
  return a.x + a.y;
}

// P (bf16 pairs) into the first 32 columns of its S buffer.
__device__ __forceinline__ void store_p(uint32_t taddr, const uint32_t (&pk)[kTileK / 2]) {
  tmem_st16(taddr, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
  tmem_st16(taddr + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
  tmem_st_wait();
}

// Writes 16 values of row r (columns c..c+15) as bf16 into a tile of
// 128-row, 64-column boxes with the 128-byte swizzle (the TMA layout).
__device__ __forceinline__ void stage_row16(uint32_t tile, int r, int c, const float (&o)[16]) {
  uint32_t w[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) w[j] = pack_bf16x2(o[2 * j], o[2 * j + 1]);
  const int box = c / 64, cc = c % 64;
  const uint32_t row_addr = tile + box * (kTileQ * 128) + r * 128;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int chunk = (cc / 8 + h) ^ (r & 7);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_addr + chunk * 16), "r"(w[4 * h]),
                 "r"(w[4 * h + 1]), "r"(w[4 * h + 2]), "r"(w[4 * h + 3])
                 : "memory");
  }
}

// Reads 16 bf16 values of row r (columns c..c+15) from such a tile.
__device__ __forceinline__ void read_row16(uint32_t tile, int r, int c, float (&o)[16]) {
  const int box = c / 64, cc = c % 64;
  const uint32_t row_addr = tile + box * (kTileQ * 128) + r * 128;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t x[4];
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3])
                 : "r"(row_addr + (((cc / 8 + h) ^ (r & 7)) * 16))
                 : "memory");
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&x[k]));
      o[8 * h + 2 * k] = f.x;
      o[8 * h + 2 * k + 1] = f.y;
    }
  }
}

// First key of key tile t of a query tile whose kept-block list is `lst`.
__device__ __forceinline__ int tile_key0(const int32_t* lst, int t, int tiles_per_block, int bk) {
  const int e = t / tiles_per_block;
  return __ldg(lst + e) * bk + (t % tiles_per_block) * kTileK;
}

template <int D, bool MIX>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const AttnParams p) {
  using L = AttnSmem<D, MIX>;
  constexpr int NS = L::NS;
  constexpr int kBarQ = L::kBarQ, kBarKFull = L::kBarKFull, kBarVFull = L::kBarVFull, kBarKEmpty = L::kBarKEmpty,
                kBarVEmpty = L::kBarVEmpty, kBarSFull = L::kBarSFull, kBarPFull = L::kBarPFull,
                kBarODone = L::kBarODone, kBarOFinal = L::kBarOFinal, kBarDrain = L::kBarDrain, kBarOl = L::kBarOl;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t sQ = sbase + L::kOffQ, sK = sbase + L::kOffK, sV = sbase + L::kOffV;
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffTmem + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = p.order ? __ldg(p.order + blockIdx.x) : (int)blockIdx.x;  // (bh, query block)
  const int bh = tile / p.nqb;
  const int qb = tile % p.nqb;
  const int q0 = qb * p.bq;                    // first query row of the tile
  const int tiles_per_block = p.bk / kTileK;
  const int cnt = min(max(__ldg(p.kv_cnt + tile), 0), p.nkb);  // a bad count cannot walk past the list
  const int T = cnt * tiles_per_block;         // key tiles to visit
  const int32_t* lst = p.kv_idx + (int64_t)tile * p.nkb;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarPFull + s), 128);
    }
    mbar_init(bar(kBarODone), 1);
    mbar_init(bar(kBarOFinal), 1);
    mbar_init(bar(kBarDrain), 1);
    mbar_init(bar(kBarOl), 1);
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
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && (T > 0 || MIX)) {
      int nk = 0, nv = 0;  // K and V tiles issued
      bool ok = true;
      if (T > 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        mbar_arrive_expect_tx(bar(kBarQ), L::kQBytes);
        for (int b = 0; b < D / 64; ++b) tma_load_3d(sQ + b * (kTileQ * 128), &tmQ, bar(kBarQ), b * 64, q0, bh);
        int key_next = tile_key0(lst, 0, tiles_per_block, p.bk);
        for (int t = 0; t < T; ++t) {
          const int slot = t % NS, round = t / NS;
          const int key0 = key_next;
          if (t + 1 < T) key_next = tile_key0(lst, t + 1, tiles_per_block, p.bk);  // latency hidden by the waits
          if (t >= NS && !role_wait(bar(kBarKEmpty + slot), (round - 1) & 1, kErrAttnKEmpty, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(kBarKFull + slot), L::kKBytes);
          for (int b = 0; b < D / 64; ++b)
            tma_load_3d(sK + slot * L::kKBytes + b * (kTileK * 128), &tmK, bar(kBarKFull + slot), b * 64, key0, bh);
          ++nk;
          if (t >= NS && !role_wait(bar(kBarVEmpty + slot), (round - 1) & 1, kErrAttnVEmpty, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(kBarVFull + slot), L::kVBytes);
          for (int b = 0; b < D / 64; ++b)
            tma_load_3d(sV + slot * L::kVBytes + b * (kTileK * 128), &tmV, bar(kBarVFull + slot), b * 64, key0, bh);
          ++nv;
        }
      }
      bool ol_issued = false;
      if (MIX && ok) {
        // The Q buffer takes the (1 - alpha) O_linear tile once S(T-1), the
        // last MMA that reads Q, has completed. (S(T-3) completed before
        // K(T-1) was loaded, so that barrier is at most one phase behind.)
        if (T == 0 || role_wait(bar(kBarSFull + ((T - 1) & 1)), ((T - 1) >> 1) & 1, kErrAttnSFull, abort_flag)) {
          mbar_arrive_expect_tx(bar(kBarOl), (D / 64) * p.bq * 128);
          for (int b = 0; b < D / 64; ++b) tma_load_3d(sQ + b * (kTileQ * 128), &tmO, bar(kBarOl), b * 64, q0, bh);
          ol_issued = true;
        }
      }
      // Never leave with copies in flight: wait for the last loads issued to
      // land (they normally have; this only matters when a role gave up).
      if (T > 0) mbar_wait(bar(kBarQ), 0, kErrAttnQ);
      for (int t = (nk > NS ? nk - NS : 0); t < nk; ++t)
        mbar_wait(bar(kBarKFull + t % NS), (t / NS) & 1, kErrAttnKFull);
      for (int t = (nv > NS ? nv - NS : 0); t < nv; ++t)
        mbar_wait(bar(kBarVFull + t % NS), (t / NS) & 1, kErrAttnVFull);
      if (ol_issued) mbar_wait(bar(kBarOl), 0, kErrAttnOl);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop (waits, descriptor arithmetic), so every
    // MMA operand is warp-uniform; one elected lane issues the MMAs and the
    // commits. Shared-memory descriptors are formed once: their address field
    // counts 16-byte units, so a byte offset o inside the tile is + (o >> 4).
    if (T > 0) {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_bf16_f32(kTileQ, kTileK, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kTileQ, D, false, true);
      const uint64_t dQ = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dK = sdesc_sw128(sK, 16, 1024);
      const uint64_t dV = sdesc_sw128(sV, kTileK * 128, 1024);
      auto warp_wait = [&](int b, uint32_t parity, unsigned int site) {
        return __all_sync(0xffffffffu, role_wait(bar(b), parity, site, abort_flag));
      };
      bool ok = warp_wait(kBarQ, 0, kErrAttnQ);
      tc_fence_after();
      for (int t = 0; ok && t <= T; ++t) {
        if (t < T) {
          const int slot = t % NS;
          if (!warp_wait(kBarKFull + slot, (t / NS) & 1, kErrAttnKFull)) break;
          tc_fence_after();
          if (leader) {
            const uint64_t dKs = dK + (uint64_t)((slot * L::kKBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              // 16 bf16 = 32 bytes along K inside a 128-byte swizzle row; 64 columns per box.
              const uint32_t qo = ((kk >> 2) * (kTileQ * 128) + (kk & 3) * 32) >> 4;
              const uint32_t ko = ((kk >> 2) * (kTileK * 128) + (kk & 3) * 32) >> 4;
              mma_ss(tS + (t & 1) * 64, dQ + qo, dKs + ko, idS, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar(kBarSFull + (t & 1)));
            mma_commit(bar(kBarKEmpty + slot));
          }
          __syncwarp();
        }
        if (t >= 1) {
          const int u = t - 1, vs = u % NS;
          if (!warp_wait(kBarVFull + vs, (u / NS) & 1, kErrAttnVFull)) break;
          tc_fence_after();
          const uint64_t dVs = dV + (uint64_t)((vs * L::kVBytes) >> 4);
          if (!warp_wait(kBarPFull + (u & 1), (u >> 1) & 1, kErrAttnPFull)) break;
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk)  // 16 keys = 2048 bytes of V = 8 packed P columns
              mma_ts(tO, tS + (u & 1) * 64 + kk * 8, dVs + kk * 128, idPV, (u > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar(kBarVEmpty + vs));
            mma_commit(bar(kBarODone));
            if (u == T - 1) mma_commit(bar(kBarOFinal));
          }
          __syncwarp();
        }
      }
      // Drain: every MMA the leader issued has completed before TMEM is freed.
      if (leader) mma_commit(bar(kBarDrain));
      __syncwarp();
      mbar_wait(bar(kBarDrain), 0, kErrAttnDrain);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;             // row of the query tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    // Kept-block indices arrive 32 at a time, one per lane, a chunk ahead of
    // use; each tile takes its index with a shuffle, so no tile waits on a
    // global load.
    int idx_cur = lane < cnt ? __ldg(lst + lane) : 0;
    int idx_nxt = 32 + lane < cnt ? __ldg(lst + 32 + lane) : 0;
    for (int t = 0; t < T; ++t) {
      const int pb = t & 1;  // S / P buffer of this tile
      const int e = t / tiles_per_block, sub = t % tiles_per_block;  // kept-list entry, tile within it
      if (e > 0 && (e & 31) == 0 && sub == 0) {
        idx_cur = idx_nxt;
        idx_nxt = e + 32 + lane < cnt ? __ldg(lst + e + 32 + lane) : 0;
      }
      const int key0 = __shfl_sync(0xffffffffu, idx_cur, e & 31) * p.bk + sub * kTileK;
      ok = __all_sync(0xffffffffu, role_wait(bar(kBarSFull + pb), (t >> 1) & 1, kErrAttnSFull, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float s[kTileK];
      load_scores(tS + lane_off + pb * 64, s);
      mask_tail(s, key0, p.N);
      const float m_new = fmaxf(m_run, row_max64(s) * p.scale_log2);
      if (t == 0) {
        m_run = m_new;
      } else if (__any_sync(0xffffffffu, m_new > m_run + kRescaleThreshold)) {
        // O holds sum_j 2^(s_j - m_run) v_j; move it to the new reference.
        // The decision is warp-wide (TMEM loads and stores are warp
        // collectives); each row scales by its own factor (1 if its max held).
        ok = __all_sync(0xffffffffu, role_wait(bar(kBarODone), (t - 1) & 1, kErrAttnODone, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const float f = ex2_approx(m_run - m_new);
        rescale_row<D>(tO + lane_off, f);
        l_run *= f;
        m_run = m_new;
      }
      uint32_t pk[kTileK / 2];
      if (key0 + kTileK <= p.N)  // the same for every row of the tile
        l_run += exp_pack<kPolyPairs>(s, p.scale_log2, m_run, pk);
      else
        l_run += exp_pack<0>(s, p.scale_log2, m_run, pk);
      store_p(tS + lane_off + pb * 64, pk);
      tc_fence_before();
      mbar_arrive(bar(kBarPFull + pb));
    }
    if (ok && T > 0) {
      ok = __all_sync(0xffffffffu, role_wait(bar(kBarOFinal), 0, kErrAttnOFinal, abort_flag));
      tc_fence_after();
    }
    const float inv_l = (T > 0 && l_run > 0.0f) ? 1.0f / l_run : 0.0f;
    // MIX: the Q buffer holds (1 - alpha_h) O_linear for this tile.
    if (MIX && ok) ok = __all_sync(0xffffffffu, role_wait(bar(kBarOl), 0, kErrAttnOl, abort_flag));
    const float w_s = (MIX ? __ldg(p.alpha + (bh % p.H)) : 1.0f) * inv_l;
    // Epilogue: w_s O (+ the linear tile) -> bf16 -> Q buffer -> TMA store.
#pragma unroll 1
    for (int c = 0; c < D; c += 16) {
      uint32_t v[16];
      if (T > 0 && ok) {
        tmem_ld16(tO + lane_off + c, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
      float o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = __uint_as_float(v[j]) * w_s;
      if (MIX && ok) {
        float ol[16];
        read_row16(sQ, r, c, ol);
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] += ol[j];
      }
      stage_row16(sQ, r, c, o);
    }
    if (p.lse != nullptr && r < p.bq && q0 + r < p.N) {
      const float lse = (T > 0 && l_run > 0.0f) ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      p.lse[(int64_t)bh * p.N + q0 + r] = lse;
    }
    fence_async_smem();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (warp == 2 && lane == 0) {
      for (int b = 0; b < D / 64; ++b) tma_store_3d(&tmO, sQ + b * (kTileQ * 128), b * 64, q0, bh);
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

}  // namespace sparge
