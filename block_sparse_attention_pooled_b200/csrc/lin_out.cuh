// Linear-branch output of the sparse + linear mix (SLA2 article,
// arXiv:2602.12675, section 1: the less important pairs go through linear
// attention; section 2: O = alpha * O_sparse + (1 - alpha) * O_linear).
//
// Per query tile (bq rows of one (batch, head), computed as a 128-row tile):
//   S_kept      = sum over the tile's kept key tiles t of phi(K_t)^T V_t
//   z_kept      = sum over the same tiles of z_tile[t]
//   [S_c | z_c] = [S_all - S_kept | z_all - z_kept]      (the blocks NOT kept)
//   O_linear[i] = phi(q_i)^T S_c / phi(q_i) . z_c
// and the tile of O is written as (1 - alpha_h) O_linear in bf16. The
// attention kernel (attn_fwd_kernel<128, true>) then reads that tile in its
// epilogue and adds alpha_h O_sparse, so O_linear is rounded once and
// O_sparse never before the mix.
//
// phi(x) = elu(x) + 1. phi(K) comes precomputed in bf16 from
// linear_summary_kernel, the same values S_all, z_all and z_tile were built
// from, so the complements are the sums over the blocks not kept up to fp32
// rounding.
//
// 192 threads:
//   warp 0      TMA producer (whole warp, one elected lane issues): phi(K)
//               and V tiles of the kept blocks into a three-slot ring, then
//               the Q tile into the slot the next tile would take, as soon
//               as that slot is free;
//   warp 1      MMA issuer (whole warp, one elected lane issues) and TMEM
//               owner: D[feature, 0..127] += phi(K_t)^T V_t (M 128, N 128,
//               K 64 per tile, both operands MN-major), starting from zero,
//               which leaves D = S_kept; then phi(Q) S_c into the same columns;
//   warps 2..5  while the MMAs run, z_kept (thread r adds z_tile[t][r] over
//               the kept tiles) and the loads of row r of S_all; then the
//               epilogue: TMEM lane r is feature r for S_c = S_all - S_kept
//               (bf16, staged in shared memory as the MN-major B operand) and
//               query row r for the output, whose denominator phi(q_r) . z_c
//               they take in fp32.
// Shared memory: ring slot s = [phi(K) 16 KB | V 16 KB]. With T kept tiles the
// Q tile (32 KB) goes to slot T % 3 (free once tile T - 3's product is done)
// and becomes phi(Q) and then the output; S_c (two 128-row boxes, 32 KB) goes
// to slot (T + 1) % 3 after the last product. Three slots keep two CTAs per
// SM, six tiles in flight per SM.
#pragma once
#include <cuda.h>
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "attn.cuh"

namespace sparge {

constexpr int kLoThreads = 192;

enum : unsigned int {
  kErrLoFull = 0x300, kErrLoEmpty, kErrLoKept, kErrLoQ, kErrLoStage, kErrLoOut, kErrLoDrain
};

#ifndef SPARGE_LO_SLOTS
#define SPARGE_LO_SLOTS 3
#endif

struct LoSmem {
  static constexpr int NS = SPARGE_LO_SLOTS;
  static constexpr int kTile = 64 * 128 * 2;         // phi(K) or V tile: two 64-column boxes of 64 keys
  static constexpr int kSlot = 2 * kTile;            // 32 KB
  static constexpr int kOffX = NS * kSlot;           // zc[128] (fp32)
  static constexpr int kOffBar = kOffX + 128 * 4;
  static constexpr int kBarFull = 0, kBarEmpty = NS, kBarKept = 2 * NS, kBarQ = 2 * NS + 1,
                       kBarStage = 2 * NS + 2, kBarOut = 2 * NS + 3, kBarDrain = 2 * NS + 4;
  static constexpr int kNumBars = 2 * NS + 5;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffTmem + 16 + 1024;  // + alignment slack: two CTAs per SM
  static_assert(kSlot == 2 * 128 * 128, "the Q tile and S_c each fill one ring slot");
  static_assert(NS >= 2, "Q and S_c take two different slots");
};

struct LoParams {
  const int32_t* kv_idx;  // [BH, nqb, nkb]
  const int32_t* kv_cnt;  // [BH, nqb]
  const int32_t* order;   // [BH * nqb] launch order of the tiles, or null (head-major)
  const float* s_all;     // [BH, 128, 128] fp32, row = feature
  const float* z_all;     // [BH, 128] fp32
  const float* z_tile;    // [BH, ntiles, 128] fp32
  const float* alpha;     // [H]
  float* den_out;         // [BH, N] or null: phi(q) . z_c per row (0 where the branch is off)
  int H;
  int N;
  int ntiles;             // ceil(N / 64)
  int nqb;
  int nkb;
  int bq;
  int bk;
};



__global__ void __launch_bounds__(kLoThreads, 2)
    linear_out_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmPhiK, const __grid_constant__ CUtensorMap tmO,
                      const LoParams p) {
  using L = LoSmem;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const int tile_ = p.order ? __ldg(p.order + blockIdx.x) : (int)blockIdx.x;
  const int cnt_ = min(max(__ldg(p.kv_cnt + tile_), 0), p.nkb);
  const int T_ = cnt_ * (p.bk / 64);
  // Q in the slot the next tile would take, S_c in the one after.
  const uint32_t sQ = sbase + (T_ % NS) * L::kSlot, sStage = sbase + ((T_ + 1) % NS) * L::kSlot;
  const int q_off = (T_ % NS) * L::kSlot;
  float* zc = reinterpret_cast<float*>(sgen + L::kOffX);  // [128] z_c
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffTmem + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = tile_;  // (bh, query block)
  const int bh = tile / p.nqb;
  const int qb = tile % p.nqb;
  const int q0 = qb * p.bq;
  const int tiles_per_block = p.bk / 64;
  const int cnt = cnt_;
  const int T = T_;
  const int32_t* lst = p.kv_idx + (int64_t)tile * p.nkb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::kBarFull + s), 1);
      mbar_init(bar(L::kBarEmpty + s), 1);
    }
    mbar_init(bar(L::kBarKept), 1);
    mbar_init(bar(L::kBarQ), 1);
    mbar_init(bar(L::kBarStage), 128);
    mbar_init(bar(L::kBarOut), 1);
    mbar_init(bar(L::kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::kOffTmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto warp_wait = [&](int b, uint32_t parity, unsigned int site) {
    return __all_sync(0xffffffffu, role_wait(bar(b), parity, site, abort_flag));
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tmPhiK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmQ);
    }
    // Kept-block indices, 32 at a time, one per lane, a chunk ahead of use.
    int idx_cur = lane < cnt ? __ldg(lst + lane) : 0;
    int idx_nxt = 32 + lane < cnt ? __ldg(lst + 32 + lane) : 0;
    int issued = 0;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int slot = t % NS;
      const int e = t / tiles_per_block, sub = t % tiles_per_block;
      if (e > 0 && (e & 31) == 0 && sub == 0) {
        idx_cur = idx_nxt;
        idx_nxt = e + 32 + lane < cnt ? __ldg(lst + e + 32 + lane) : 0;
      }
      const int key0 = __shfl_sync(0xffffffffu, idx_cur, e & 31) * p.bk + sub * 64;
      if (t >= NS && !warp_wait(L::kBarEmpty + slot, (t / NS - 1) & 1, kErrLoEmpty)) {
        ok = false;
        break;
      }
      if (leader) {
        const uint32_t sp = sbase + slot * L::kSlot, sv = sp + L::kTile;
        mbar_arrive_expect_tx(bar(L::kBarFull + slot), L::kSlot);
        for (int b = 0; b < 2; ++b) {
          tma_load_3d(sp + b * 8192, &tmPhiK, bar(L::kBarFull + slot), b * 64, key0, bh);
          tma_load_3d(sv + b * 8192, &tmV, bar(L::kBarFull + slot), b * 64, key0, bh);
        }
      }
      __syncwarp();
      ++issued;
    }
    // Q goes to slot T % NS, as a tile T would: once tile T - NS's product
    // (if any) has read that slot.
    bool q_issued = false;
    if (ok && (T < NS || warp_wait(L::kBarEmpty + T % NS, (T / NS - 1) & 1, kErrLoEmpty))) {
      if (leader) {
        mbar_arrive_expect_tx(bar(L::kBarQ), 2 * 128 * 128);
        for (int b = 0; b < 2; ++b) tma_load_3d(sQ + b * (128 * 128), &tmQ, bar(L::kBarQ), b * 64, q0, bh);
      }
      q_issued = true;
    }
    // Never leave with copies in flight.
    if (leader) {
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        mbar_wait(bar(L::kBarFull + t % NS), (t / NS) & 1, kErrLoFull);
      if (q_issued) mbar_wait(bar(L::kBarQ), 0, kErrLoQ);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    constexpr uint32_t idKept = idesc_bf16_f32(128, 128, true, true);
    constexpr uint32_t idOut = idesc_bf16_f32(128, 128, false, true);
    const uint64_t dRing = sdesc_sw128(sbase, 64 * 128, 1024);     // MN-major, 64-row boxes
    const uint64_t dQ = sdesc_sw128(sQ, 16, 1024);                 // K-major, 128-row boxes
    const uint64_t dStage = sdesc_sw128(sStage, 128 * 128, 1024);  // MN-major, 128-row boxes
    bool ok = true;
    for (int t = 0; ok && t < T; ++t) {
      const int slot = t % NS;
      if (!warp_wait(L::kBarFull + slot, (t / NS) & 1, kErrLoFull)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (leader) {
        const uint64_t dP = dRing + (uint64_t)((slot * L::kSlot) >> 4);
        const uint64_t dV = dP + (uint64_t)(L::kTile >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 16 keys = 2048 bytes of each operand
          mma_ss(tmem, dP + kk * 128, dV + kk * 128, idKept, (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(L::kBarEmpty + slot));
      }
      __syncwarp();
    }
    if (leader) mma_commit(bar(L::kBarKept));  // every S_kept MMA (none when T = 0) has completed
    __syncwarp();
    if (ok && warp_wait(L::kBarStage, 0, kErrLoStage)) {
      tc_fence_after();
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t qo = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
          mma_ss(tmem, dQ + qo, dStage + kk * 128, idOut, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::kBarOut));
      }
      __syncwarp();
    }
    if (leader) mma_commit(bar(L::kBarDrain));
    __syncwarp();
    mbar_wait(bar(L::kBarDrain), 0, kErrLoDrain);
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;            // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;       // feature (S_c, z_c) / query row (output)
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    // z_kept[r] over the kept tiles, four loads in flight at a time. A last
    // 128-key block may hold a single 64-key tile: its second tile lies past
    // N, has no z_tile entry and adds nothing.
    float zk = 0.0f;
    {
      const float* zt = p.z_tile + (int64_t)bh * p.ntiles * 128 + r;
      auto ztile = [&](int tt) {
        const int tile64 = (__ldg(lst + tt / tiles_per_block) * p.bk + (tt % tiles_per_block) * 64) / 64;
        return tile64 < p.ntiles ? __ldg(zt + (int64_t)tile64 * 128) : 0.0f;
      };
      int t = 0;
      for (; t + 4 <= T; t += 4) {
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = ztile(t + u);
        zk += (v[0] + v[1]) + (v[2] + v[3]);
      }
      for (; t < T; ++t) zk += ztile(t);
    }
    // Row r (feature r) of S_all: all 32 loads in flight at once, issued
    // while the products still run.
    float4 sa[32];
    {
      const float4* srow = reinterpret_cast<const float4*>(p.s_all + ((int64_t)bh * 128 + r) * 128);
#pragma unroll
      for (int k = 0; k < 32; ++k) sa[k] = __ldg(srow + k);
    }
    bool ok = warp_wait(L::kBarKept, 0, kErrLoKept);
    tc_fence_after();
    // 1. S_c row a = r (S_all - D; D = 0 when nothing is kept) as bf16,
    //    MN-major for the last MMA (two 64-column boxes of 128 rows,
    //    128-byte swizzle).
#pragma unroll
    for (int c = 0; c < 128; c += 16) {
      uint32_t v[16];
      if (ok && T > 0) {
        tmem_ld16(tmem + lane_off + c, v);
        tmem_ld_wait_regs(v);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
      float sc[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 a = sa[c / 4 + j];
        sc[4 * j] = a.x - __uint_as_float(v[4 * j]);
        sc[4 * j + 1] = a.y - __uint_as_float(v[4 * j + 1]);
        sc[4 * j + 2] = a.z - __uint_as_float(v[4 * j + 2]);
        sc[4 * j + 3] = a.w - __uint_as_float(v[4 * j + 3]);
      }
      stage_row16(sStage, r, c, sc);
    }
    // 2. z_c, then phi(Q) in place. phi is elementwise, so the tile is
    //    walked as a flat array of 16-byte units, consecutive threads on
    //    consecutive units (no bank conflicts).
    zc[r] = __ldg(p.z_all + (int64_t)bh * 128 + r) - zk;
    if (ok) ok = warp_wait(L::kBarQ, 0, kErrLoQ);
    if (ok) {
      // Sixteen 16-byte units per thread: every load in flight before the
      // first conversion, every store after the last.
      constexpr int kUnits = (2 * 128 * 128) / 16 / 128;
      uint4* qt = reinterpret_cast<uint4*>(sgen + q_off);
      uint4 x[kUnits];
#pragma unroll
      for (int k = 0; k < kUnits; ++k) x[k] = qt[r + 128 * k];
#pragma unroll
      for (int k = 0; k < kUnits; ++k) {
        __nv_bfloat162* hx = reinterpret_cast<__nv_bfloat162*>(&x[k]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(hx[j]);
          hx[j] = __floats2bfloat162_rn(phi_elu1(f.x), phi_elu1(f.y));
        }
      }
#pragma unroll
      for (int k = 0; k < kUnits; ++k) qt[r + 128 * k] = x[k];
    }
    fence_async_smem();
    tc_fence_before();
    mbar_arrive(bar(L::kBarStage));
    asm volatile("bar.sync 1, 128;" ::: "memory");  // z_c complete
    // 3. Denominator phi(q_r) . z_c in fp32; every block kept: the
    //    complement is empty and the linear branch is 0.
    float den = 0.0f;
#pragma unroll 1
    for (int c = 0; c < 128; c += 16) {
      float qv[16];
      read_row16(sQ, r, c, qv);
#pragma unroll
      for (int j = 0; j < 16; ++j) den = fmaf(qv[j], zc[c + j], den);
    }
    const float a_h = __ldg(p.alpha + (bh % p.H));
    const float wl = (cnt < p.nkb && den > 0.0f) ? (1.0f - a_h) / den : 0.0f;
    if (p.den_out != nullptr && r < p.bq && q0 + r < p.N)
      p.den_out[(int64_t)bh * p.N + q0 + r] = (cnt < p.nkb && den > 0.0f) ? den : 0.0f;
    if (ok) ok = warp_wait(L::kBarOut, 0, kErrLoOut);
    tc_fence_after();
    // 4. O tile = (1 - alpha_h) numerator / denominator, bf16, TMA store.
#pragma unroll 1
    for (int c = 0; c < 128; c += 16) {
      uint32_t v[16];
      if (ok) {
        tmem_ld16(tmem + lane_off + c, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
      float o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = wl * __uint_as_float(v[j]);
      stage_row16(sQ, r, c, o);
    }
    fence_async_smem();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (warp == 2 && lane == 0) {
      for (int b = 0; b < 2; ++b) tma_store_3d(&tmO, sQ + b * (128 * 128), b * 64, q0, bh);
      tma_store_commit();
      tma_store_wait_read0();  // the staging tile has been read: the CTA may end
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
