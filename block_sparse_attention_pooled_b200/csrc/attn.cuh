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
//   warp 0      TMA producer: Q once, then K and V tiles into two rings (2 slots;
//               3 for the LIN variant, which runs one CTA per SM);
//   warp 1      MMA issuer and TMEM owner: S = Q K^T into a double-buffered
//               TMEM S, then O += P V with P read back from TMEM;
//   warps 2..5  softmax: one query row per thread (TMEM lane), fp32 online
//               softmax with lazy rescaling, P written to TMEM as bf16 over
//               its own S columns; then the epilogue (O / l -> bf16 -> TMA
//               store, optional log-sum-exp).
// TMEM columns: S0 [0,64), S1 [64,128), O [128,128+D).
//
// With LIN = true the same kernel also produces the sparse + linear mix of
// the SLA2 article (arXiv:2602.12675, sections 1 and 2):
//   O = alpha_h * O_sparse + (1 - alpha_h) * O_linear,
//   O_linear[i] = phi(q_i)^T S_c / phi(q_i) . z_c  over the blocks NOT kept,
// where S_c = S_all - S_kept and z_c = z_all - z_kept. S_all / z_all come from
// linear_summary_kernel; S_kept = sum over the kept key tiles of
// phi(K_t)^T [V_t | 1] is accumulated here with one more MMA per tile (A =
// the phi(K) tile, B = the V tile followed by a ones block, both already in
// shared memory), into TMEM columns [256, 400). The epilogue writes
// [S_c | z_c] as bf16 into shared memory, turns the Q tile into phi(Q) in
// place and runs one more MMA, phi(Q) [S_c | z_c], whose column 128 is the
// denominator.
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
// Of the 64 exponentials per row and tile, this many run on the FMA pipe
// (exp2_poly) and the rest on the MUFU (ex2.approx).
constexpr int kPolyExp = 0;

// Error site codes recorded in g_device_error by the attention kernel.
enum : unsigned int {
  kErrAttnQ = 0x100, kErrAttnKFull, kErrAttnVFull, kErrAttnKEmpty, kErrAttnVEmpty, kErrAttnSFull,
  kErrAttnPFull, kErrAttnODone, kErrAttnOFinal, kErrAttnDrain, kErrAttnLin
};

struct AttnParams {
  const int32_t* kv_idx;  // [BH, nqb, nkb]
  const int32_t* kv_cnt;  // [BH, nqb]
  float* lse;             // [BH, N] or null
  const float* s_all;     // LIN: [BH, 128, 128] fp32
  const float* z_all;     // LIN: [BH, 128] fp32
  const float* alpha;     // LIN: [H]
  int H;
  int N;
  int nqb;
  int nkb;
  int bq;                 // 64 or 128: rows of the query block that share a mask row
  int bk;                 // 64 or 128: keys per mask block (bk / 64 key tiles each)
  float scale_log2;       // log2(e) / sqrt(d)
};

template <int D, bool LIN>
struct AttnSmem {
  // K / V (/ phi(K)) ring depth. Two slots keep the plain kernel small enough
  // for two CTAs per SM; the LIN kernel runs one CTA per SM and uses three.
  static constexpr int NS = LIN ? 3 : 2;
  static constexpr int kQBytes = kTileQ * D * 2;
  static constexpr int kKBytes = kTileK * D * 2;
  static constexpr int kVData = kTileK * D * 2;
  static constexpr int kVBytes = kVData + (LIN ? 8192 : 0);   // LIN: ones block after V
  static constexpr int kPBytes = LIN ? kTileK * D * 2 : 0;     // phi(K) tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + NS * kKBytes;
  static constexpr int kOffP = kOffV + NS * kVBytes;
  static constexpr int kOffBar = kOffP + NS * kPBytes;
  // Barrier slots: K full / V full / K empty / V empty rings, S full and
  // P full pairs, then single barriers.
  static constexpr int kBarQ = 0, kBarKFull = 1, kBarVFull = 1 + NS, kBarKEmpty = 1 + 2 * NS,
                       kBarVEmpty = 1 + 3 * NS, kBarSFull = 1 + 4 * NS, kBarPFull = 3 + 4 * NS,
                       kBarODone = 5 + 4 * NS, kBarOFinal = 6 + 4 * NS, kBarDrain = 7 + 4 * NS,
                       kBarLin = 8 + 4 * NS;
  static constexpr int kNumBars = 9 + 4 * NS;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kUsed = kOffTmem + 16;
  // Pad so that at most two CTAs fit on an SM: two CTAs x 256 TMEM columns
  // use the SM's 512 columns exactly, and a third would block in alloc.
  // LIN needs all 512 columns and is one CTA per SM by its size.
  static constexpr int kBytes = (kUsed + 1024 > 80 * 1024 ? kUsed + 1024 : 80 * 1024);
  static constexpr int kTmemCols = LIN ? 512 : 256;
  // LIN epilogue: [S_c | z_c] staged over the (then idle) K and V rings.
  static constexpr int kOffStage = kOffK;
  static_assert(!LIN || kOffStage + 3 * 128 * 128 <= kOffV + kVData, "stage must not reach the ones block");
};


// Waits on an mbarrier unless another role already gave up; gives up itself
// (and tells the others through *abort) after the global time limit.
__device__ __forceinline__ bool role_wait(uint32_t bar, uint32_t parity, unsigned int site,
                                          volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      record_error(site);
      *abort = 1;
      return false;
    }
  }
  return true;
}

// First key of key tile t of a query tile whose kept-block list is `lst`.
__device__ __forceinline__ int tile_key0(const int32_t* lst, int t, int tiles_per_block, int bk) {
  const int e = t / tiles_per_block;
  return __ldg(lst + e) * bk + (t % tiles_per_block) * kTileK;
}

__device__ __forceinline__ float phi_attn(float x) { return x > 0.0f ? x + 1.0f : __expf(x); }

template <int D, bool LIN>
__global__ void __launch_bounds__(kAttnThreads, LIN ? 1 : 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmPhiK, const AttnParams p) {
  static_assert(!LIN || D == 128, "the linear branch is built for d = 128");
  using L = AttnSmem<D, LIN>;
  constexpr int NS = L::NS;
  constexpr int kBarQ = L::kBarQ, kBarKFull = L::kBarKFull, kBarVFull = L::kBarVFull, kBarKEmpty = L::kBarKEmpty,
                kBarVEmpty = L::kBarVEmpty, kBarSFull = L::kBarSFull, kBarPFull = L::kBarPFull,
                kBarODone = L::kBarODone, kBarOFinal = L::kBarOFinal, kBarDrain = L::kBarDrain, kBarLin = L::kBarLin;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t sQ = sbase + L::kOffQ, sK = sbase + L::kOffK, sV = sbase + L::kOffV, sP = sbase + L::kOffP;
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffTmem + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x;                 // (bh, query block), head-major
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
    mbar_init(bar(kBarLin), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (LIN) {
    // Ones block after each V slot: the 16 extra B columns that yield z.
    for (int sl = 0; sl < NS; ++sl) {
      uint4* ones = reinterpret_cast<uint4*>(sgen + L::kOffV + sl * L::kVBytes + L::kVData);
      for (int u = threadIdx.x; u < 8192 / 16; u += kAttnThreads)
        ones[u] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    }
    fence_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::kOffTmem, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128, tL = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && (T > 0 || LIN)) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar(kBarQ), L::kQBytes);
      for (int b = 0; b < D / 64; ++b) tma_load_3d(sQ + b * (kTileQ * 128), &tmQ, bar(kBarQ), b * 64, q0, bh);
      int nk = 0, nv = 0;  // K and V tiles issued
      int key_next = tile_key0(lst, 0, tiles_per_block, p.bk);
      for (int t = 0; t < T; ++t) {
        const int slot = t % NS, round = t / NS;
        const int key0 = key_next;
        if (t + 1 < T) key_next = tile_key0(lst, t + 1, tiles_per_block, p.bk);  // latency hidden by the waits
        if (t >= NS && !role_wait(bar(kBarKEmpty + slot), (round - 1) & 1, kErrAttnKEmpty, abort_flag)) break;
        mbar_arrive_expect_tx(bar(kBarKFull + slot), L::kKBytes);
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(sK + slot * L::kKBytes + b * (kTileK * 128), &tmK, bar(kBarKFull + slot), b * 64, key0, bh);
        ++nk;
        if (t >= NS && !role_wait(bar(kBarVEmpty + slot), (round - 1) & 1, kErrAttnVEmpty, abort_flag)) break;
        mbar_arrive_expect_tx(bar(kBarVFull + slot), L::kVData + L::kPBytes);
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(sV + slot * L::kVBytes + b * (kTileK * 128), &tmV, bar(kBarVFull + slot), b * 64, key0, bh);
        if (LIN)
          for (int b = 0; b < D / 64; ++b)
            tma_load_3d(sP + slot * L::kPBytes + b * (kTileK * 128), &tmPhiK, bar(kBarVFull + slot), b * 64, key0, bh);
        ++nv;
      }
      // Never leave with copies in flight: wait for the last loads issued to
      // land (they normally have; this only matters when a role gave up).
      mbar_wait(bar(kBarQ), 0, kErrAttnQ);
      for (int t = (nk > NS ? nk - NS : 0); t < nk; ++t)
        mbar_wait(bar(kBarKFull + t % NS), (t / NS) & 1, kErrAttnKFull);
      for (int t = (nv > NS ? nv - NS : 0); t < nv; ++t)
        mbar_wait(bar(kBarVFull + t % NS), (t / NS) & 1, kErrAttnVFull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kTileQ, kTileK, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kTileQ, D, false, true);
      bool ok = role_wait(bar(kBarQ), 0, kErrAttnQ, abort_flag);
      tc_fence_after();
      for (int t = 0; ok && t <= T; ++t) {
        if (t < T) {
          const int slot = t % NS;
          if (!role_wait(bar(kBarKFull + slot), (t / NS) & 1, kErrAttnKFull, abort_flag)) break;
          tc_fence_after();
          const uint32_t kbase = sK + slot * L::kKBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32u;  // 16 bf16 = 32 bytes along K inside the swizzle row
            const uint64_t a = sdesc_sw128(sQ + (kk >> 2) * (kTileQ * 128) + off, 16, 1024);
            const uint64_t b = sdesc_sw128(kbase + (kk >> 2) * (kTileK * 128) + off, 16, 1024);
            mma_ss(tS + (t & 1) * 64, a, b, idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(kBarSFull + (t & 1)));
          mma_commit(bar(kBarKEmpty + slot));
        }
        if (t >= 1) {
          const int u = t - 1, vs = u % NS;
          if (!role_wait(bar(kBarVFull + vs), (u / NS) & 1, kErrAttnVFull, abort_flag)) break;
          tc_fence_after();
          const uint32_t vbase = sV + vs * L::kVBytes;
          if (LIN) {
            // S_kept[feature, 0..143] += phi(K_u)^T [V_u | 1]; independent of
            // the softmax, so it is queued before waiting for P_u.
            constexpr uint32_t idL = idesc_bf16_f32(128, 144, true, true);
            const uint32_t pbase = sP + vs * L::kPBytes;
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk) {
              const uint64_t a = sdesc_sw128(pbase + kk * (16 * 128), kTileK * 128, 1024);
              const uint64_t b = sdesc_sw128(vbase + kk * (16 * 128), kTileK * 128, 1024);
              mma_ss(tL, a, b, idL, (u > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (!role_wait(bar(kBarPFull + (u & 1)), (u >> 1) & 1, kErrAttnPFull, abort_flag)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk) {
            const uint64_t b = sdesc_sw128(vbase + kk * (16 * 128), kTileK * 128, 1024);
            mma_ts(tO, tS + (u & 1) * 64 + kk * 8, b, idPV, (u > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(kBarVEmpty + vs));
          mma_commit(bar(kBarODone));
          if (u == T - 1) mma_commit(bar(kBarOFinal));
        }
      }
      // Drain: every MMA this thread issued has completed before TMEM is freed.
      mma_commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, kErrAttnDrain);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;             // row of the query tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float m_run = -INFINITY, l_run = 0.0f;
    int kept_keys = 0;  // valid keys in the kept tiles (LIN: the complement is empty when this is N)
    bool ok = true;
    // The block index of tile t+1 is requested while tile t is processed, so
    // its global-load latency stays off the softmax's critical path.
    int key_next = T > 0 ? tile_key0(lst, 0, tiles_per_block, p.bk) : 0;
    for (int t = 0; t < T; ++t) {
      const int slot = t & 1;
      const int key0 = key_next;
      if (t + 1 < T) key_next = tile_key0(lst, t + 1, tiles_per_block, p.bk);
      ok = __all_sync(0xffffffffu, role_wait(bar(kBarSFull + slot), (t >> 1) & 1, kErrAttnSFull, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float s[kTileK];
      {
        uint32_t v[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld16(tS + lane_off + slot * 64 + 16 * c, v[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 16; ++j) s[16 * c + j] = __uint_as_float(v[c][j]);
      }
      kept_keys += max(0, min(kTileK, p.N - key0));
      if (key0 + kTileK > p.N) {
#pragma unroll
        for (int j = 0; j < kTileK; ++j)
          if (key0 + j >= p.N) s[j] = -INFINITY;
      }
      float mx;  // tree reduction: depth 6 instead of a 64-long chain
      {
        float m8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          m8[j] = fmaxf(fmaxf(fmaxf(s[j], s[8 + j]), fmaxf(s[16 + j], s[24 + j])),
                        fmaxf(fmaxf(s[32 + j], s[40 + j]), fmaxf(s[48 + j], s[56 + j])));
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      }
      const float m_new = fmaxf(m_run, mx * p.scale_log2);
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
        uint32_t v[16];
#pragma unroll 1
        for (int c = 0; c < D; c += 16) {
          tmem_ld16(tO + lane_off + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
          tmem_st16(tO + lane_off + c, v);
        }
        tmem_st_wait();
        l_run *= f;
        m_run = m_new;
      }
      const float neg_m = -m_run;
      float ps[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums: short dependency chains
      uint32_t pk[kTileK / 2];
#pragma unroll
      for (int j = 0; j < kTileK; j += 2) {
        const float xa = fmaf(s[j], p.scale_log2, neg_m), xb = fmaf(s[j + 1], p.scale_log2, neg_m);
        const float a = (j < kPolyExp) ? exp2_poly(xa) : ex2_approx(xa);
        const float b = (j < kPolyExp) ? exp2_poly(xb) : ex2_approx(xb);
        ps[(j >> 1) & 3] += a + b;
        pk[j / 2] = pack_bf16x2(a, b);
      }
      l_run += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      // P (bf16) overwrites the first 32 columns of this S buffer.
      tmem_st16(tS + lane_off + slot * 64, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
      tmem_st16(tS + lane_off + slot * 64 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(kBarPFull + slot));
    }
    if (ok && T > 0) {
      ok = __all_sync(0xffffffffu, role_wait(bar(kBarOFinal), 0, kErrAttnOFinal, abort_flag));
      tc_fence_after();
    }
    const float inv_l = (T > 0 && l_run > 0.0f) ? 1.0f / l_run : 0.0f;
    // Writes 16 output values of row r (columns c..c+15) as bf16 into the
    // Q buffer, laid out the way the 128-byte-swizzled O tensor map expects.
    auto stage_out16 = [&](int c, const float (&o)[16]) {
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) w[j] = pack_bf16x2(o[2 * j], o[2 * j + 1]);
      const int box = c / 64, cc = c % 64;
      const uint32_t row_addr = sQ + box * (kTileQ * 128) + r * 128;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int chunk = (cc / 8 + h) ^ (r & 7);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_addr + chunk * 16), "r"(w[4 * h]),
                     "r"(w[4 * h + 1]), "r"(w[4 * h + 2]), "r"(w[4 * h + 3])
                     : "memory");
      }
    };
    if constexpr (!LIN) {
      // Epilogue: O / l -> bf16 -> Q buffer -> TMA store.
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
        for (int j = 0; j < 16; ++j) o[j] = __uint_as_float(v[j]) * inv_l;
        stage_out16(c, o);
      }
    } else {
      // 1. Q is needed as phi(Q): wait for it when no key tile was visited.
      if (ok && T == 0) ok = __all_sync(0xffffffffu, role_wait(bar(kBarQ), 0, kErrAttnQ, abort_flag));
      // 2. [S_c | z_c] for feature a = r: S_all - S_kept, z_all - z_kept, as
      //    bf16 into the stage, MN-major with 128-byte swizzle (row a, three
      //    64-column boxes; column 128 = z_c, the rest of box 2 zero).
      const uint32_t sStage = sbase + L::kOffStage;
      const float* srow = p.s_all + ((int64_t)bh * 128 + r) * 128;
#pragma unroll 1
      for (int c = 0; c < 144; c += 16) {
        uint32_t v[16];
        if (T > 0 && ok) {
          tmem_ld16(tL + lane_off + c, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0u;
        }
        float sc[16];
        if (c < 128) {
#pragma unroll
          for (int j = 0; j < 16; ++j) sc[j] = __ldg(srow + c + j) - __uint_as_float(v[j]);
        } else {
          sc[0] = __ldg(p.z_all + (int64_t)bh * 128 + r) - __uint_as_float(v[0]);
#pragma unroll
          for (int j = 1; j < 16; ++j) sc[j] = 0.0f;
        }
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = pack_bf16x2(sc[2 * j], sc[2 * j + 1]);
        const int box = c / 64, cc = c % 64;
        const uint32_t row_addr = sStage + box * (128 * 128) + r * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int chunk = (cc / 8 + h) ^ (r & 7);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_addr + chunk * 16), "r"(w[4 * h]),
                       "r"(w[4 * h + 1]), "r"(w[4 * h + 2]), "r"(w[4 * h + 3])
                       : "memory");
        }
      }
      {  // zero the rest of box 2 (columns 144..191), which the MMA does not read but keep defined
        const uint32_t row_addr = sStage + 2 * (128 * 128) + r * 128;
#pragma unroll
        for (int ch = 2; ch < 8; ++ch)
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(row_addr + ((ch ^ (r & 7)) * 16)), "r"(0u)
                       : "memory");
      }
      // 3. phi(Q) in place over this thread's row of the Q tile (elementwise,
      //    so the swizzle does not matter).
#pragma unroll
      for (int b = 0; b < D / 64; ++b) {
        uint4* row = reinterpret_cast<uint4*>(sgen + L::kOffQ + b * (kTileQ * 128) + r * 128);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint4 x = row[ch];
          __nv_bfloat162* hx = reinterpret_cast<__nv_bfloat162*>(&x);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float2 f = __bfloat1622float2(hx[j]);
            hx[j] = __floats2bfloat162_rn(phi_attn(f.x), phi_attn(f.y));
          }
          row[ch] = x;
        }
      }
      fence_async_smem();
      tc_fence_before();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // 4. O_lin numerator and denominator: phi(Q) [S_c | z_c] -> TMEM [256, 400).
      if (warp == 2 && lane == 0 && ok) {
        tc_fence_after();
        constexpr uint32_t idF = idesc_bf16_f32(kTileQ, 144, false, true);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sdesc_sw128(sQ + (kk >> 2) * (kTileQ * 128) + (kk & 3) * 32u, 16, 1024);
          const uint64_t b = sdesc_sw128(sStage + kk * (16 * 128), 128 * 128, 1024);
          mma_ss(tL, a, b, idF, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(kBarLin));
      }
      if (ok) ok = __all_sync(0xffffffffu, role_wait(bar(kBarLin), 0, kErrAttnLin, abort_flag));
      tc_fence_after();
      // 5. Mix and stage the output row.
      const float a_h = __ldg(p.alpha + (bh % p.H));
      float inv_den = 0.0f;
      if (ok) {
        uint32_t v[16];
        tmem_ld16(tL + lane_off + 128, v);
        tmem_ld_wait();
        const float den = __uint_as_float(v[0]);
        inv_den = (kept_keys < p.N && den > 0.0f) ? 1.0f / den : 0.0f;
      }
      const float ws = a_h * inv_l, wl = (1.0f - a_h) * inv_den;
#pragma unroll 1
      for (int c = 0; c < D; c += 16) {
        uint32_t vo[16], vl[16];
        if (ok) {
          if (T > 0) tmem_ld16(tO + lane_off + c, vo);
          tmem_ld16(tL + lane_off + c, vl);
          tmem_ld_wait();
        }
        float o[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float os = (ok && T > 0) ? __uint_as_float(vo[j]) : 0.0f;
          const float ol = ok ? __uint_as_float(vl[j]) : 0.0f;
          o[j] = ws * os + wl * ol;
        }
        stage_out16(c, o);
      }
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
      tma_store_wait0();
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
