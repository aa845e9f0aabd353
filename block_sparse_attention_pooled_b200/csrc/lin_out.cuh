// Linear-branch output of the sparse + linear mix (SLA2 article,
// arXiv:2602.12675, section 1: the less important pairs go through linear
// attention; section 2: O = alpha * O_sparse + (1 - alpha) * O_linear).
//
// Per query tile (bq rows of one (batch, head), computed as a 128-row tile):
//   S_kept      = sum over the tile's kept key tiles t of phi(K_t)^T [V_t | 1]
//   [S_c | z_c] = [S_all - S_kept | z_all - z_kept]      (the blocks NOT kept)
//   O_linear[i] = phi(q_i)^T S_c / phi(q_i) . z_c
// and the tile of O is written as (1 - alpha_h) O_linear in bf16. The
// attention kernel (attn_fwd_kernel<128, true>) then reads that tile in its
// epilogue and adds alpha_h O_sparse, so O_linear is rounded once and
// O_sparse never before the mix.
//
// phi(x) = elu(x) + 1. phi(K) comes precomputed in bf16 from
// linear_summary_kernel, the same values S_all and z_all were built from, so
// the complement S_all - S_kept is exactly the sum over the blocks not kept
// up to fp32 rounding.
//
// 192 threads:
//   warp 0      TMA producer: phi(K) and V tiles of the kept blocks into a
//               two-slot ring; then the Q tile, once the ring is idle;
//   warp 1      MMA issuer (whole warp, one elected lane issues) and TMEM
//               owner: S_kept[feature, 0..143] += phi(K_t)^T [V_t | 1]
//               (M 128, N 144, K 64 per tile; both operands MN-major; the
//               ones block after each V slot yields z_kept in column 128);
//               then phi(Q) [S_c | z_c] into the same TMEM columns;
//   warps 2..5  epilogue: TMEM lane r is feature r for [S_c | z_c] (bf16,
//               staged in shared memory as the MN-major B operand) and query
//               row r for the output.
// Shared memory: ring slot s = [phi(K) 16 KB | V 16 KB | ones 8 KB]; after the
// last MMA of the ring the same bytes hold [S_c | z_c] (three 128-row boxes,
// 48 KB) and the Q tile (32 KB), which becomes phi(Q) and then the output.
#pragma once
#include <cuda.h>
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparge {

constexpr int kLoThreads = 192;

enum : unsigned int {
  kErrLoFull = 0x300, kErrLoEmpty, kErrLoKept, kErrLoQ, kErrLoStage, kErrLoOut, kErrLoDrain
};

struct LoSmem {
  static constexpr int NS = 2;
  static constexpr int kPhiK = 64 * 128 * 2;        // phi(K) tile: two 64-column boxes of 64 keys
  static constexpr int kV = 64 * 128 * 2;           // V tile, same layout
  static constexpr int kOnes = 8192;                // B columns 128..191 of the tile (16 used)
  static constexpr int kSlot = kPhiK + kV + kOnes;  // 40 KB
  static constexpr int kOffStage = 0;               // epilogue: [S_c | z_c], three boxes of 128 rows
  static constexpr int kOffQ = 3 * 128 * 128;       // epilogue: Q tile -> phi(Q) -> output
  static constexpr int kOffBar = NS * kSlot;
  static constexpr int kBarFull = 0, kBarEmpty = NS, kBarKept = 2 * NS, kBarQ = 2 * NS + 1,
                       kBarStage = 2 * NS + 2, kBarOut = 2 * NS + 3, kBarDrain = 2 * NS + 4;
  static constexpr int kNumBars = 2 * NS + 5;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffTmem + 16 + 1024;  // + alignment slack: two CTAs per SM
  static_assert(kOffQ + 2 * 128 * 128 <= kOffBar, "epilogue tiles must fit in the ring");
};

struct LoParams {
  const int32_t* kv_idx;  // [BH, nqb, nkb]
  const int32_t* kv_cnt;  // [BH, nqb]
  const float* s_all;     // [BH, 128, 128] fp32, row = feature
  const float* z_all;     // [BH, 128] fp32
  const float* alpha;     // [H]
  int H;
  int N;
  int nqb;
  int nkb;
  int bq;
  int bk;
};

__device__ __forceinline__ float phi_lin(float x) { return x > 0.0f ? x + 1.0f : __expf(x); }

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
  const uint32_t sStage = sbase + L::kOffStage, sQ = sbase + L::kOffQ;
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffTmem + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x;  // (bh, query block), head-major
  const int bh = tile / p.nqb;
  const int qb = tile % p.nqb;
  const int q0 = qb * p.bq;
  const int tiles_per_block = p.bk / 64;
  const int cnt = min(max(__ldg(p.kv_cnt + tile), 0), p.nkb);
  const int T = cnt * tiles_per_block;
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
  for (int s = 0; s < NS; ++s) {
    uint4* ones = reinterpret_cast<uint4*>(sgen + s * L::kSlot + L::kPhiK + L::kV);
    for (int u = threadIdx.x; u < L::kOnes / 16; u += kLoThreads)
      ones[u] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  }
  fence_async_smem();
  if (warp == 1) {
    tmem_alloc(sbase + L::kOffTmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmPhiK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmQ);
      int issued = 0;
      bool ok = true;
      for (int t = 0; t < T; ++t) {
        const int slot = t % NS;
        const int key0 = __ldg(lst + t / tiles_per_block) * p.bk + (t % tiles_per_block) * 64;
        if (t >= NS && !role_wait(bar(L::kBarEmpty + slot), (t / NS - 1) & 1, kErrLoEmpty, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t sp = sbase + slot * L::kSlot, sv = sp + L::kPhiK;
        mbar_arrive_expect_tx(bar(L::kBarFull + slot), L::kPhiK + L::kV);
        for (int b = 0; b < 2; ++b) {
          tma_load_3d(sp + b * 8192, &tmPhiK, bar(L::kBarFull + slot), b * 64, key0, bh);
          tma_load_3d(sv + b * 8192, &tmV, bar(L::kBarFull + slot), b * 64, key0, bh);
        }
        ++issued;
      }
      // Q goes where the ring was, once every MMA that reads the ring is done.
      bool q_issued = false;
      if (ok && role_wait(bar(L::kBarKept), 0, kErrLoKept, abort_flag)) {
        mbar_arrive_expect_tx(bar(L::kBarQ), 2 * 128 * 128);
        for (int b = 0; b < 2; ++b) tma_load_3d(sQ + b * (128 * 128), &tmQ, bar(L::kBarQ), b * 64, q0, bh);
        q_issued = true;
      }
      // Never leave with copies in flight.
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        mbar_wait(bar(L::kBarFull + t % NS), (t / NS) & 1, kErrLoFull);
      if (q_issued) mbar_wait(bar(L::kBarQ), 0, kErrLoQ);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    constexpr uint32_t idKept = idesc_bf16_f32(128, 144, true, true);
    constexpr uint32_t idOut = idesc_bf16_f32(128, 144, false, true);
    const uint64_t dRing = sdesc_sw128(sbase, 64 * 128, 1024);        // MN-major, 64-row boxes
    const uint64_t dQ = sdesc_sw128(sQ, 16, 1024);                    // K-major, 128-row boxes
    const uint64_t dStage = sdesc_sw128(sStage, 128 * 128, 1024);     // MN-major, 128-row boxes
    auto warp_wait = [&](int b, uint32_t parity, unsigned int site) {
      return __all_sync(0xffffffffu, role_wait(bar(b), parity, site, abort_flag));
    };
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int slot = t % NS;
      if (!warp_wait(L::kBarFull + slot, (t / NS) & 1, kErrLoFull)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (leader) {
        const uint64_t dP = dRing + (uint64_t)((slot * L::kSlot) >> 4);
        const uint64_t dV = dP + (uint64_t)(L::kPhiK >> 4);
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
    const int r = q * 32 + lane;       // feature (phase 1) / query row (phase 2)
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    auto warp_wait = [&](int b, uint32_t parity, unsigned int site) {
      return __all_sync(0xffffffffu, role_wait(bar(b), parity, site, abort_flag));
    };
    bool ok = warp_wait(L::kBarKept, 0, kErrLoKept);
    tc_fence_after();
    // 1. [S_c | z_c] row r as bf16, MN-major with the 128-byte swizzle
    //    (three 64-column boxes; column 128 = z_c, the rest of box 2 zero).
    const float* srow = p.s_all + ((int64_t)bh * 128 + r) * 128;
#pragma unroll 1
    for (int c = 0; c < 144; c += 16) {
      uint32_t v[16];
      if (ok && T > 0) {
        tmem_ld16(tmem + lane_off + c, v);
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
    {  // columns 144..191 of box 2: not read by the MMA (N = 144), kept defined
      const uint32_t row_addr = sStage + 2 * (128 * 128) + r * 128;
#pragma unroll
      for (int ch = 2; ch < 8; ++ch)
        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(row_addr + ((ch ^ (r & 7)) * 16)), "r"(0u)
                     : "memory");
    }
    // 2. phi(Q) in place over query row r (elementwise: the swizzle does not matter).
    if (ok) ok = warp_wait(L::kBarQ, 0, kErrLoQ);
    if (ok) {
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint4* row = reinterpret_cast<uint4*>(sgen + L::kOffQ + b * (128 * 128) + r * 128);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint4 x = row[ch];
          __nv_bfloat162* hx = reinterpret_cast<__nv_bfloat162*>(&x);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(hx[j]);
            hx[j] = __floats2bfloat162_rn(phi_lin(f.x), phi_lin(f.y));
          }
          row[ch] = x;
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    mbar_arrive(bar(L::kBarStage));
    // 3. O tile = (1 - alpha_h) * numerator / denominator, bf16, TMA store.
    if (ok) ok = warp_wait(L::kBarOut, 0, kErrLoOut);
    tc_fence_after();
    const float a_h = __ldg(p.alpha + (bh % p.H));
    float wl = 0.0f;
    if (ok) {
      uint32_t v[16];
      tmem_ld16(tmem + lane_off + 128, v);
      tmem_ld_wait();
      const float den = __uint_as_float(v[0]);
      // Every block kept: the complement is empty and the linear branch is 0.
      wl = (cnt < p.nkb && den > 0.0f) ? (1.0f - a_h) / den : 0.0f;
    }
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
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        w[j] = pack_bf16x2(wl * __uint_as_float(v[2 * j]), wl * __uint_as_float(v[2 * j + 1]));
      const int box = c / 64, cc = c % 64;
      const uint32_t row_addr = sQ + box * (128 * 128) + r * 128;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int chunk = (cc / 8 + h) ^ (r & 7);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_addr + chunk * 16), "r"(w[4 * h]),
                     "r"(w[4 * h + 1]), "r"(w[4 * h + 2]), "r"(w[4 * h + 3])
                     : "memory");
      }
    }
    fence_async_smem();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (warp == 2 && lane == 0) {
      for (int b = 0; b < 2; ++b) tma_store_3d(&tmO, sQ + b * (128 * 128), b * 64, q0, bh);
      tma_store_commit();
      tma_store_wait0();
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
