// Linear-branch dK and dV of the sparse + linear mix (SLA2 article,
// arXiv:2602.12675, sections 1 and 2: O = alpha * O_sparse +
// (1 - alpha) * O_linear, both branches trained), and their sum with the
// sparse branch's fp32 partials.
//
// For key j and the query rows i whose block does NOT keep j's block
// (c_i = (1 - alpha_h) / den_i, f_i and e_i = c_i f_i from the row pass):
//   dphi(k_j) = sum_i c_i (dO_i . v_j - f_i) phi(q_i) = G_c v_j - g_c
//   dv_j      = sum_i c_i (phi(q_i) . phi(k_j)) dO_i = G_c^T phi(k_j)
// with, over those rows, G_c = sum_i phi(q_i) (c_i dO_i)^T and
// g_c = sum_i e_i phi(q_i). The rows whose block keeps j's are the
// complement's complement, so per 64-key tile J
//   G_c(J) = G_all - sum_{u keeps J} phi(Q_u)^T cdO_u
//   g_c(J) = g_all - sum_{u keeps J} (the g_tile sums of u's rows)
// (G_all, g_all, g_tile, phi(Q) and cdO = c_i dO_i from the summary kernel's
// GRAD pass), and then
//   dK_J = dK_sparse + (G_c V_J^T - g_c)^T * phi'(K_J),  phi'(k) = min(phi(k), 1)
//   dV_J = dV_sparse + (G_c^T phi(K_J)^T)^T
// The kept share costs one MMA per kept (query block, key tile) pair, with
// no elementwise work between products.
//
// One CTA takes two neighbouring key tiles, A = 2c and B = 2c + 1 of one
// (batch, head) (A alone for the last tile of an odd count); neighbouring
// key blocks are kept by mostly the same query blocks, so the CTA walks the
// ascending union of the two query-block lists (the transposed mask) and
// loads each phi(Q)/cdO tile of it once. As in linear_out_kernel, with X the
// tile whose list is the shorter and Y the other, D_base = sum over X's
// list and D_diff = (Y's sum) - (X's sum) (+ the rows only Y's list holds,
// - the rows only X's list holds, by the MMA's negate-A bit).
//
// 192 threads:
//   warp 0      TMA producer: the union's phi(Q) and cdO tiles (64 rows each)
//               into a three-slot ring (32 KB a slot); then phi(K_A), V_A into
//               the slot the next tile would take and phi(K_B), V_B into the
//               slot of the last tile;
//   warp 1      MMA issuer and TMEM owner: D_base / D_diff [feature, 0..127]
//               +/-= phi(Q_u)^T cdO_u (M 128, N 128, K 64 rows per tile, both
//               operands MN-major), in TMEM columns 0..127 (D0) and 128..255
//               (D1); then per key tile dphiK^T = G_c V^T (M 128 features,
//               N 64 keys, K 128 value dims) and dV^T = G_c^T phi(K)^T (M 128
//               value dims, N 64 keys, K 128 features) into that tile's
//               columns;
//   warps 2..5  while the MMAs run, the g_tile sums of both lists (thread r =
//               feature r) and the loads of row r of G_all; then the epilogue,
//               TMEM lane r being feature r (dphiK^T, G_c) or value dim r
//               (dV^T): G_c,X = G_all - D_base and G_c,Y = G_c,X - D_diff in
//               fp32 over the accumulators (D0 then holds G_c,A, D1 G_c,B);
//               G_c,A as bf16 into the staging slot; once A's products are
//               done, G_c,B the same way, and A's dK, dV rows are formed and
//               written; then B's.
#pragma once
#include <cuda.h>
#include <climits>
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "attn.cuh"
#include "lin_out.cuh"

namespace sparge {

enum : unsigned int {
  kErrLbFull = 0x900, kErrLbEmpty, kErrLbKept, kErrLbKV, kErrLbStage, kErrLbOut, kErrLbDrain
};

struct LbSmem {
  static constexpr int NS = 3;
  static constexpr int kTile = 64 * 128 * 2;  // a 64-row, 128-column bf16 tile: two 64-column boxes
  static constexpr int kSlot = 2 * kTile;     // [phi(Q) | cdO] in the ring, [phi(K) | V] after it
  static constexpr int kOffBar = NS * kSlot;
  static constexpr int kBarFull = 0, kBarEmpty = NS, kBarKept = 2 * NS, kBarKV0 = 2 * NS + 1,
                       kBarKV1 = 2 * NS + 2, kBarStage0 = 2 * NS + 3, kBarStage1 = 2 * NS + 4,
                       kBarOut0 = 2 * NS + 5, kBarOut1 = 2 * NS + 6, kBarDrain = 2 * NS + 7;
  static constexpr int kNumBars = 2 * NS + 8;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // TMEM base, abort flag, union tile count, written sums
  static constexpr int kBytes = kOffMisc + 16 + 1024;     // + alignment slack: two CTAs per SM
  static_assert(kSlot == 2 * 128 * 128, "G_c (128 x 128 bf16) fills one slot");
};

struct LbParams {
  const int32_t* q_idx;   // [BH, nkb, nqb] query blocks keeping each key block, ascending
  const int32_t* q_cnt;   // [BH, nkb]
  const float* g_all;     // [BH, 128, 128] fp32 G_all, row = feature
  const float* g_vec;     // [BH, 128] g_all
  const float* g_tile;    // [BH, ntiles, 128] sums of e_i phi(q_i) over 64-row tiles
  const float* dk_part;   // [BH, N, 128] fp32 scale * dK_sparse
  const float* dv_part;   // [BH, N, 128] fp32 dV_sparse
  __nv_bfloat16* dK;      // [BH, N, 128]
  __nv_bfloat16* dV;      // [BH, N, 128]
  int N;
  int ntiles;             // ceil(N / 64): key tiles and 64-row query tiles
  int nqb;
  int nkb;
  int bq;
  int bk;
};

__global__ void __launch_bounds__(kLoThreads, 2)
    linear_dkdv_kernel(const __grid_constant__ CUtensorMap tmPhiQ, const __grid_constant__ CUtensorMap tmCdo,
                       const __grid_constant__ CUtensorMap tmPhiK, const __grid_constant__ CUtensorMap tmV,
                       const LbParams p) {
  using L = LbSmem;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffMisc + 4);
  volatile int* tiles_slot = reinterpret_cast<volatile int*>(sgen + L::kOffMisc + 8);
  volatile int* sums_slot = reinterpret_cast<volatile int*>(sgen + L::kOffMisc + 12);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int npairs = (p.ntiles + 1) / 2;
  const int bh = (int)(blockIdx.x / (unsigned)npairs);
  const int ka = 2 * (int)(blockIdx.x % (unsigned)npairs);  // key tile A; B = ka + 1
  const bool has_b = ka + 1 < p.ntiles;
  const int key0a = ka * 64, key0b = key0a + 64;
  const int64_t jb_a = (int64_t)bh * p.nkb + key0a / p.bk, jb_b = (int64_t)bh * p.nkb + key0b / p.bk;
  const int cnt_a = min(max(__ldg(p.q_cnt + jb_a), 0), p.nqb);
  const int cnt_b = has_b ? min(max(__ldg(p.q_cnt + jb_b), 0), p.nqb) : 0;
  const int32_t* lst_a = p.q_idx + jb_a * p.nqb;
  const int32_t* lst_b = p.q_idx + jb_b * p.nqb;
  const int tiles_per_block = p.bq / 64;
  const bool base_is_a = cnt_a <= cnt_b;  // X = the shorter list
  const uint32_t col_base = base_is_a ? 0u : 128u, col_diff = 128u - col_base;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::kBarFull + s), 1);
      mbar_init(bar(L::kBarEmpty + s), 1);
    }
    mbar_init(bar(L::kBarKept), 2);  // the MMA issuer's arrive (with the tile count) and its commit
    mbar_init(bar(L::kBarKV0), 1);
    mbar_init(bar(L::kBarKV1), 1);
    mbar_init(bar(L::kBarStage0), 128);
    mbar_init(bar(L::kBarStage1), 128);
    mbar_init(bar(L::kBarOut0), 1);
    mbar_init(bar(L::kBarOut1), 1);
    mbar_init(bar(L::kBarDrain), 1);
    *abort_flag = 0;
    *tiles_slot = 0;
    *sums_slot = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::kOffMisc, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto warp_wait = [&](int b, uint32_t parity, unsigned int site) {
    return __all_sync(0xffffffffu, role_wait(bar(b), parity, site, abort_flag));
  };
  // Slots after the union walk, given its tile count T: k = 0 phi(K_A), V_A;
  // k = 1 the staged G_c; k = 2 phi(K_B), V_B.
  auto slot_addr = [&](int T, int k) { return sbase + (uint32_t)(((T + k) % NS) * L::kSlot); };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tmPhiQ);
      tma_prefetch_desc(&tmCdo);
      tma_prefetch_desc(&tmPhiK);
      tma_prefetch_desc(&tmV);
    }
    KeptCursor ca, cb;
    ca.init(lst_a, cnt_a, lane);
    cb.init(lst_b, cnt_b, lane);
    int t = 0, issued = 0, qb;
    bool in_a, in_b, ok = true;
    while (union_next(ca, cb, lane, qb, in_a, in_b)) {
      for (int sub = 0; sub < tiles_per_block; ++sub, ++t) {
        const int slot = t % NS;
        if (ok && t >= NS) ok = warp_wait(L::kBarEmpty + slot, (t / NS - 1) & 1, kErrLbEmpty);
        if (!ok) continue;  // keep counting: T fixes the epilogue's slots
        if (leader) {
          const uint32_t sq = sbase + slot * L::kSlot, sd = sq + L::kTile;
          const int row0 = qb * p.bq + sub * 64;
          mbar_arrive_expect_tx(bar(L::kBarFull + slot), L::kSlot);
          for (int b = 0; b < 2; ++b) {
            tma_load_3d(sq + b * 8192, &tmPhiQ, bar(L::kBarFull + slot), b * 64, row0, bh);
            tma_load_3d(sd + b * 8192, &tmCdo, bar(L::kBarFull + slot), b * 64, row0, bh);
          }
        }
        __syncwarp();
        ++issued;
      }
    }
    const int T = t;
    // phi(K_A), V_A go to slot T % NS, as a tile T would: once tile T - NS's
    // product (if any) has read it; phi(K_B), V_B to slot (T - 1) % NS, once
    // the last tile's product has read it.
    bool a_issued = false, b_issued = false;
    if (ok && (T < NS || warp_wait(L::kBarEmpty + T % NS, (T / NS - 1) & 1, kErrLbEmpty))) {
      if (leader) {
        const uint32_t sk = slot_addr(T, 0);
        mbar_arrive_expect_tx(bar(L::kBarKV0), L::kSlot);
        for (int b = 0; b < 2; ++b) {
          tma_load_3d(sk + b * 8192, &tmPhiK, bar(L::kBarKV0), b * 64, key0a, bh);
          tma_load_3d(sk + L::kTile + b * 8192, &tmV, bar(L::kBarKV0), b * 64, key0a, bh);
        }
      }
      a_issued = true;
    } else {
      ok = false;
    }
    if (has_b && ok && (T < 1 || warp_wait(L::kBarEmpty + (T - 1) % NS, ((T - 1) / NS) & 1, kErrLbEmpty))) {
      if (leader) {
        const uint32_t sk = slot_addr(T, 2);
        mbar_arrive_expect_tx(bar(L::kBarKV1), L::kSlot);
        for (int b = 0; b < 2; ++b) {
          tma_load_3d(sk + b * 8192, &tmPhiK, bar(L::kBarKV1), b * 64, key0b, bh);
          tma_load_3d(sk + L::kTile + b * 8192, &tmV, bar(L::kBarKV1), b * 64, key0b, bh);
        }
      }
      b_issued = true;
    }
    // Never leave with copies in flight.
    if (leader) {
      for (int u = (issued > NS ? issued - NS : 0); u < issued; ++u)
        mbar_wait(bar(L::kBarFull + u % NS), (u / NS) & 1, kErrLbFull);
      if (a_issued) mbar_wait(bar(L::kBarKV0), 0, kErrLbKV);
      if (b_issued) mbar_wait(bar(L::kBarKV1), 0, kErrLbKV);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    constexpr uint32_t idKept = idesc_bf16_f32(128, 128, true, true);
    constexpr uint32_t idKeptNeg = idKept | (1u << 13);  // negate A: -phi(Q_u)^T cdO_u
    constexpr uint32_t idGK = idesc_bf16_f32(128, 64, false, false);  // G_c V^T: both K-major
    constexpr uint32_t idGtK = idesc_bf16_f32(128, 64, true, false);  // G_c^T phi(K)^T: A MN-major
    const uint64_t dRing = sdesc_sw128(sbase, 64 * 128, 1024);       // MN-major, 64-row boxes
    KeptCursor ca, cb;
    ca.init(lst_a, cnt_a, lane);
    cb.init(lst_b, cnt_b, lane);
    int t = 0, qb;
    bool in_a, in_b, ok = true, started_base = false, started_diff = false;
    while (union_next(ca, cb, lane, qb, in_a, in_b)) {
      const bool in_x = base_is_a ? in_a : in_b, in_y = base_is_a ? in_b : in_a;
      for (int sub = 0; sub < tiles_per_block; ++sub, ++t) {
        const int slot = t % NS;
        if (ok) ok = warp_wait(L::kBarFull + slot, (t / NS) & 1, kErrLbFull);
        if (ok) {
          tc_fence_after();
          if (leader) {
            const uint64_t dA = dRing + (uint64_t)((slot * L::kSlot) >> 4);
            const uint64_t dB = dA + (uint64_t)(L::kTile >> 4);
            if (in_x) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)  // 16 rows = 2048 bytes of each operand
                mma_ss(tmem + col_base, dA + kk * 128, dB + kk * 128, idKept, (started_base || kk > 0) ? 1u : 0u);
            }
            if (in_x != in_y) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem + col_diff, dA + kk * 128, dB + kk * 128, in_x ? idKeptNeg : idKept,
                       (started_diff || kk > 0) ? 1u : 0u);
            }
            mma_commit(bar(L::kBarEmpty + slot));
          }
          __syncwarp();
        }
        started_base = started_base || in_x;
        started_diff = started_diff || in_x != in_y;
      }
    }
    const int T = t;
    if (leader) {
      *tiles_slot = T;
      *sums_slot = (started_base ? 1 : 0) | (started_diff ? 2 : 0);
      mbar_arrive(bar(L::kBarKept));  // publishes T and which sums were written
      mma_commit(bar(L::kBarKept));   // every kept-share MMA (none when T = 0) has completed
    }
    __syncwarp();
    const uint32_t sG = slot_addr(T, 1);
    const uint64_t dGk = sdesc_sw128(sG, 16, 1024);         // G_c as K-major A (128-row boxes)
    const uint64_t dGm = sdesc_sw128(sG, 128 * 128, 1024);  // G_c^T as MN-major A
    // Products of one key tile into TMEM columns col .. col + 127:
    // dphiK^T at col, dV^T at col + 64.
    auto tile_products = [&](uint32_t sKV, uint32_t col) {
      const uint64_t dPk = sdesc_sw128(sKV, 16, 1024);             // phi(K) as K-major B (64-row boxes)
      const uint64_t dVk = sdesc_sw128(sKV + L::kTile, 16, 1024);  // V as K-major B
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {  // K = 128 value dims, 16 at a time
        const uint32_t go = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
        const uint32_t ko = ((kk >> 2) * (64 * 128) + (kk & 3) * 32) >> 4;
        mma_ss(tmem + col, dGk + go, dVk + ko, idGK, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {  // K = 128 features, 16 at a time
        const uint32_t ko = ((kk >> 2) * (64 * 128) + (kk & 3) * 32) >> 4;
        mma_ss(tmem + col + 64, dGm + kk * 128, dPk + ko, idGtK, kk > 0 ? 1u : 0u);
      }
    };
    if (ok) ok = warp_wait(L::kBarStage0, 0, kErrLbStage);
    if (ok) ok = warp_wait(L::kBarKV0, 0, kErrLbKV);
    if (ok) {
      tc_fence_after();
      if (leader) {
        tile_products(slot_addr(T, 0), 0u);
        mma_commit(bar(L::kBarOut0));
      }
      __syncwarp();
    }
    if (has_b && ok) ok = warp_wait(L::kBarStage1, 0, kErrLbStage);
    if (has_b && ok) ok = warp_wait(L::kBarKV1, 0, kErrLbKV);
    if (has_b && ok) {
      tc_fence_after();
      if (leader) {
        tile_products(slot_addr(T, 2), 128u);
        mma_commit(bar(L::kBarOut1));
      }
      __syncwarp();
    }
    if (leader) mma_commit(bar(L::kBarDrain));
    __syncwarp();
    mbar_wait(bar(L::kBarDrain), 0, kErrLbDrain);
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;       // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;  // feature (G_c, g_c, dK) / value dim (dV)
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t tD0 = tmem + lane_off, tD1 = tmem + lane_off + 128;
    // Kept share of g for one list: the g_tile sums of its blocks' 64-row
    // tiles (a last 128-row block may hold one tile), four loads in flight.
    const float* gt = p.g_tile + (int64_t)bh * p.ntiles * 128 + r;
    auto g_kept = [&](const int32_t* lst, int cnt) {
      auto gtile = [&](int tt) {
        const int tile64 = __ldg(lst + tt / tiles_per_block) * tiles_per_block + tt % tiles_per_block;
        return tile64 < p.ntiles ? __ldg(gt + (int64_t)tile64 * 128) : 0.0f;
      };
      const int T1 = cnt * tiles_per_block;
      float gk = 0.0f;
      int t = 0;
      for (; t + 4 <= T1; t += 4) {
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = gtile(t + u);
        gk += (v[0] + v[1]) + (v[2] + v[3]);
      }
      for (; t < T1; ++t) gk += gtile(t);
      return gk;
    };
    const float g_r = __ldg(p.g_vec + (int64_t)bh * 128 + r);
    const float gc_a = g_r - g_kept(lst_a, cnt_a);
    const float gc_b = has_b ? g_r - g_kept(lst_b, cnt_b) : 0.0f;
    // Row r (feature r) of G_all: all 32 loads in flight at once, issued
    // while the products still run.
    float4 ga[32];
    {
      const float4* grow = reinterpret_cast<const float4*>(p.g_all + ((int64_t)bh * 128 + r) * 128);
#pragma unroll
      for (int k = 0; k < 32; ++k) ga[k] = __ldg(grow + k);
    }
    bool ok = warp_wait(L::kBarKept, 0, kErrLbKept);
    tc_fence_after();
    const int T = *tiles_slot;
    const uint32_t sG = slot_addr(T, 1);
    const int sums = *sums_slot;
    const bool has_base = ok && (sums & 1), has_diff = ok && (sums & 2);
    const uint32_t tBase = tD0 + col_base, tDiff = tD0 + col_diff;
    // 1. G_c,X = G_all - D_base and G_c,Y = G_c,X - D_diff for row r (an
    //    accumulator no product wrote counts as 0), in fp32 back over the
    //    two accumulators: D0 then holds G_c,A and D1 G_c,B.
#pragma unroll
    for (int c = 0; c < 128; c += 16) {
      uint32_t v[16];
      if (has_base) {
        tmem_ld16(tBase + c, v);
        tmem_ld_wait_regs(v);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
      uint32_t gx[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 a = ga[c / 4 + j];
        gx[4 * j] = __float_as_uint(a.x - __uint_as_float(v[4 * j]));
        gx[4 * j + 1] = __float_as_uint(a.y - __uint_as_float(v[4 * j + 1]));
        gx[4 * j + 2] = __float_as_uint(a.z - __uint_as_float(v[4 * j + 2]));
        gx[4 * j + 3] = __float_as_uint(a.w - __uint_as_float(v[4 * j + 3]));
      }
      if (has_diff) {
        tmem_ld16(tDiff + c, v);
        tmem_ld_wait_regs(v);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(gx[j]) - __uint_as_float(v[j]));
      tmem_st16(tBase + c, gx);
      tmem_st16(tDiff + c, v);
    }
    tmem_st_wait();
    // G_c of one tile (D0 or D1) as bf16 into the staging slot: row r,
    // two 64-column boxes of 128 rows with the 128-byte swizzle (K-major
    // G_c and MN-major G_c^T at once).
    auto stage_g = [&](uint32_t tD) {
#pragma unroll 1
      for (int c = 0; c < 128; c += 16) {
        uint32_t v[16];
        if (ok) {
          tmem_ld16(tD + c, v);
          tmem_ld_wait_regs(v);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0u;
        }
        float g[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) g[j] = __uint_as_float(v[j]);
        stage_row16(sG, r, c, g);
      }
      fence_async_smem();
      tc_fence_before();
    };
    stage_g(tD0);
    mbar_arrive(bar(L::kBarStage0));
    // dK and dV rows of one key tile: lane r is feature r of dphiK^T (columns
    // col .. col + 63) and value dim r of dV^T (col + 64 ..); key j's phi(k)
    // comes from the phi(K) tile in shared memory.
    auto finish_tile = [&](uint32_t col, uint32_t sKV, int key0, float gc) {
      const int nvalid = min(64, p.N - key0);
      const int64_t base = ((int64_t)bh * p.N + key0) * 128 + r;
      const uint8_t* phik = sgen + (sKV - sbase);
#pragma unroll 1
      for (int c = 0; c < 64; c += 16) {
        uint32_t vk[16], vv[16];
        if (ok) {
          tmem_ld16(tmem + lane_off + col + c, vk);
          tmem_ld16(tmem + lane_off + col + 64 + c, vv);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) vk[j] = vv[j] = 0u;
        }
        float pk[16], pv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const bool in = c + j < nvalid;
          pk[j] = in ? __ldg(p.dk_part + base + (int64_t)(c + j) * 128) : 0.0f;
          pv[j] = in ? __ldg(p.dv_part + base + (int64_t)(c + j) * 128) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (c + j < nvalid) {
            const float dphi = __uint_as_float(vk[j]) - gc;
            const float dk = pk[j] + dphi * fminf(tile_at(phik, c + j, r), 1.0f);
            const float dv = pv[j] + __uint_as_float(vv[j]);
            p.dK[base + (int64_t)(c + j) * 128] = __float2bfloat16_rn(dk);
            p.dV[base + (int64_t)(c + j) * 128] = __float2bfloat16_rn(dv);
          }
        }
      }
    };
    // 2. A's products done: the staging slot takes G_c,B, then A's rows.
    if (ok) ok = warp_wait(L::kBarOut0, 0, kErrLbOut);
    tc_fence_after();
    if (has_b) {
      stage_g(tD1);
      mbar_arrive(bar(L::kBarStage1));
    }
    if (ok) ok = warp_wait(L::kBarKV0, 0, kErrLbKV);
    finish_tile(0u, slot_addr(T, 0), key0a, gc_a);
    if (has_b) {
      if (ok) ok = warp_wait(L::kBarOut1, 0, kErrLbOut);
      if (ok) ok = warp_wait(L::kBarKV1, 0, kErrLbKV);
      tc_fence_after();
      finish_tile(128u, slot_addr(T, 2), key0b, gc_b);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace sparge
