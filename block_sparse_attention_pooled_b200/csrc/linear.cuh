// Linear-attention summaries for the sparse + linear mix (SLA2 article,
// arXiv:2602.12675, section 1: the less important pairs go through linear
// attention; phi(x) = elu(x) + 1 is this library's feature map).
//
// Per (batch, head) this kernel produces
//   phiK  = phi(K)                         bf16 [N, d]   (kept for the attention kernel)
//   S_all = sum_j phi(k_j) v_j^T           fp32 [d, d]   (row = feature, column = value dim)
//   z_all = sum_j phi(k_j)                 fp32 [d]
//   z_tile[t] = sum of phi(k_j) over the 64 keys of tile t, from the bf16
//               phi(K) values (fp32 [ceil(N / 64), d])
// The attention kernel subtracts the kept blocks' share of S_all and z_all to
// get the complement's summaries.
//
// With GRAD = true the same kernel gives the summaries the backward of the
// linear branch needs (rows are query rows then, with per-row weights c_i and
// e_i from the backward's row pass):
//   phiQ  = phi(Q)                         bf16 [N, d]
//   cdO   = c_i dO_i                       bf16 [N, d]
//   G_all = sum_i phi(q_i) (c_i dO_i)^T     fp32 [d, d]
//   g_all = sum_i e_i phi(q_i)              fp32 [d]
//   g_tile[t] = sum of e_i phi(q_i) over the 64 rows of tile t
// (K -> Q, V -> dO with row i scaled by c_i, the column sums weighted by e_i).
//
// The flattened (head, 64-key tile) range is split evenly over a persistent
// grid of kLinCtas CTAs (two per SM on 148 SMs); CTA c takes the tiles
// [c W, (c + 1) W) in order, W = ceil(tiles / grid), so every CTA does the
// same work and the grid ends in one wave. 192 threads:
//   warp 0      TMA producer: K and V tiles of the range into a three-slot
//               ring (32 KB a slot);
//   warp 1      TMEM owner and issuer (one elected lane): for each tile, once
//               the compute warps have applied phi, a TMA store of the phi(K)
//               tile (GRAD: and of the scaled V tile) and four MMAs D[feature, 0..127] += phi(K)^T V (M 128,
//               N 128, K 64, both operands MN-major in shared memory); two
//               accumulators (TMEM columns 0..127 and 128..255) alternate
//               between the head segments of the range;
//   warps 2..5  compute: phi in place on the K tile (rows past N zeroed),
//               then thread a (= feature) sums column a of the tile for
//               z_tile; at the end of a head segment they write the
//               accumulator and the segment's z sum out as one partial
//               summary [128][129].
// A slot is reused once the compute warps have read it, its MMAs have
// completed and the phi(K) store has read it. The partial of CTA c and head h
// goes to slot c + h (strictly increasing in (c, h), so no two collide), and
// linear_reduce_kernel adds each head's partials in CTA order: the result
// does not depend on scheduling.
//
// GRAD: V rows are scaled by c_i in place before the MMAs (and the scaled
// tile is stored too), and the column sums are those of e_i phi(q_i) (e_i
// staged per tile in shared memory): per 64-row tile into z_tile, per
// segment into the partial.
#pragma once
#include <cuda.h>
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparge {

constexpr int kLinThreads = 192;
constexpr int kLinCtas = 296;           // persistent grid: two CTAs on each of 148 SMs
constexpr int kLinPartial = 128 * 129;  // per (CTA, head) segment: [feature][128 value columns + z]

enum : unsigned int { kErrLinFull = 0x200, kErrLinMma, kErrLinDrain, kErrLinReady, kErrLinEmpty, kErrLinAcc };

struct LinSmem {
  static constexpr int NS = 3;
  static constexpr int kTile = 64 * 128 * 2;     // K / phi(K) or V tile: two 64-column boxes of 64 rows
  static constexpr int kSlot = 2 * kTile;        // 32 KB
  static constexpr int kOffE = NS * kSlot;       // GRAD: e_i of each slot's 64 rows (fp32)
  static constexpr int kOffBar = kOffE + NS * 64 * 4;
  static constexpr int kBarFull = 0, kBarReady = NS, kBarEmpty = 2 * NS, kBarAccFull = 3 * NS,
                       kBarAccFree = 3 * NS + 2, kBarDrain = 3 * NS + 4;
  static constexpr int kNumBars = 3 * NS + 5;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffTmem + 16 + 1024;  // + alignment slack: two CTAs per SM
};

struct LinParams {
  float* partial;  // [grid + BH][128][129]: partial of (CTA c, head h) at slot c + h
  float* z_tile;   // [BH, ntiles, 128] per-tile column sums, or null
  const float* row_scale;  // GRAD: c_i [BH, N]
  const float* row_w;      // GRAD: e_i [BH, N]
  int N;
  int ntiles;      // ceil(N / 64)
  int64_t total;   // BH * ntiles
  int64_t per_cta; // W = ceil(total / grid)
};

// Grid of the summary kernel for BH heads of N rows.
inline int64_t lin_grid(int64_t BH, int N) {
  const int64_t total = BH * ((N + 63) / 64);
  return total < kLinCtas ? total : kLinCtas;
}

// Applies phi to 8 packed bf16 values.
__device__ __forceinline__ uint4 phi8(uint4 v) {
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float2 f = __bfloat1622float2(h[j]);
    h[j] = __floats2bfloat162_rn(phi_elu1(f.x), phi_elu1(f.y));
  }
  return v;
}

// Waits until at most one of this thread's bulk store groups still reads
// shared memory.
__device__ __forceinline__ void bulk_store_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// Element (row, col) of a swizzled 64-row, 64-column bf16 box (128-byte rows).
__device__ __forceinline__ float box_at(const uint8_t* box, int row, int col) {
  return __bfloat162float(
      *reinterpret_cast<const __nv_bfloat16*>(box + row * 128 + ((((col >> 3) ^ (row & 7)) << 4) | ((col & 7) << 1))));
}

template <bool GRAD>
__global__ void __launch_bounds__(kLinThreads, 2)
    linear_summary_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmPhiK, const __grid_constant__ CUtensorMap tmVs,
                          const LinParams p) {
  using L = LinSmem;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffTmem + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t f0 = (int64_t)blockIdx.x * p.per_cta;
  const int64_t f1 = min(p.total, f0 + p.per_cta);
  const int n = f1 > f0 ? (int)(f1 - f0) : 0;  // tiles of this CTA
  // Tile i of the range: head and tile within the head; a segment ends where
  // the head changes or the range ends.
  auto head_of = [&](int i) { return (int)((f0 + i) / p.ntiles); };
  auto tile_of = [&](int i) { return (int)((f0 + i) % p.ntiles); };
  auto seg_last = [&](int i) { return i + 1 == n || tile_of(i) + 1 == p.ntiles; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::kBarFull + s), 1);
      mbar_init(bar(L::kBarReady + s), 128);
      mbar_init(bar(L::kBarEmpty + s), 130);  // compute threads, the MMA commit, the store-read arrive
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(L::kBarAccFull + a), 1);
      mbar_init(bar(L::kBarAccFree + a), 128);
    }
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
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    int issued = 0;
    for (int i = 0; i < n; ++i) {
      const int slot = i % NS;
      if (i >= NS && !warp_wait(L::kBarEmpty + slot, (i / NS - 1) & 1, kErrLinEmpty)) break;
      if (leader) {
        const uint32_t sk = sbase + slot * L::kSlot, sv = sk + L::kTile;
        const int key0 = tile_of(i) * 64, bh = head_of(i);
        mbar_arrive_expect_tx(bar(L::kBarFull + slot), L::kSlot);
        for (int b = 0; b < 2; ++b) {
          tma_load_3d(sk + b * 8192, &tmK, bar(L::kBarFull + slot), b * 64, key0, bh);
          tma_load_3d(sv + b * 8192, &tmV, bar(L::kBarFull + slot), b * 64, key0, bh);
        }
      }
      __syncwarp();
      ++issued;
    }
    // Never leave with copies in flight.
    if (leader)
      for (int u = (issued > NS ? issued - NS : 0); u < issued; ++u)
        mbar_wait(bar(L::kBarFull + u % NS), (u / NS) & 1, kErrLinFull);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA and phi(K) store issuer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tmPhiK);
      if (GRAD) tma_prefetch_desc(&tmVs);
    }
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128, true, true);
    bool ok = true;
    int seg = 0;          // segment index of tile i
    bool seg_start = true;
    for (int i = 0; ok && i < n; ++i) {
      const int slot = i % NS, acc = seg & 1;
      if (seg_start && seg >= 2) ok = warp_wait(L::kBarAccFree + acc, ((seg >> 1) - 1) & 1, kErrLinAcc);
      if (ok) ok = warp_wait(L::kBarReady + slot, (i / NS) & 1, kErrLinReady);
      if (!ok) break;
      tc_fence_after();
      const bool last = seg_last(i);
      if (leader) {
        const uint32_t sk = sbase + slot * L::kSlot, sv = sk + L::kTile;
        const int key0 = tile_of(i) * 64, bh = head_of(i);
        for (int b = 0; b < 2; ++b) {
          tma_store_3d(&tmPhiK, sk + b * 8192, b * 64, key0, bh);
          if (GRAD) tma_store_3d(&tmVs, sv + b * 8192, b * 64, key0, bh);  // c_i dO_i
        }
        tma_store_commit();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 keys = 2048 bytes of each operand
          const uint64_t a = sdesc_sw128(sk + kk * 2048, 8192, 1024);
          const uint64_t b = sdesc_sw128(sv + kk * 2048, 8192, 1024);
          mma_ss(tmem + acc * 128, a, b, idesc, (!seg_start || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(L::kBarEmpty + slot));
        if (last) mma_commit(bar(L::kBarAccFull + acc));
        // The previous tile's phi(K) store has read its slot.
        if (i > 0) {
          bulk_store_wait_read1();
          mbar_arrive(bar(L::kBarEmpty + (i - 1) % NS));
        }
      }
      __syncwarp();
      seg_start = last;
      if (last) ++seg;
    }
    if (leader) {
      tma_store_wait_read0();  // every phi(K) tile has been read from shared memory: the CTA may end
      mma_commit(bar(L::kBarDrain));
    }
    __syncwarp();
    mbar_wait(bar(L::kBarDrain), 0, kErrLinDrain);
  } else {
    // ------------------------------------------------------------ compute warps
    const int ct = threadIdx.x - 64;  // 0..127: feature of the column sums
    const int q = warp & 3;           // TMEM lane quadrant of this warp
    const int a = q * 32 + lane;      // feature of this thread's TMEM lane
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float* sE = reinterpret_cast<float*>(sgen + L::kOffE);
    bool ok = true;
    int seg = 0;
    float zacc = 0.0f;  // column-a sum of the segment (feature ct)
    for (int i = 0; i < n; ++i) {
      const int slot = i % NS, bh = head_of(i), key0 = tile_of(i) * 64;
      if (ok) ok = warp_wait(L::kBarFull + slot, (i / NS) & 1, kErrLinFull);
      uint8_t* sk = sgen + slot * L::kSlot;
      if (ok) {
        // phi in place; rows past N become zero so they add nothing.
        uint4* tile = reinterpret_cast<uint4*>(sk);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int u = ct + 128 * j;               // 16-byte unit of the 16 KB tile
          const int row = (u * 16 % 8192) / 128;     // key row inside the box
          tile[u] = (key0 + row < p.N) ? phi8(tile[u]) : make_uint4(0u, 0u, 0u, 0u);
        }
        if (GRAD) {
          // dO rows scaled by c_i (zero past N); e_i staged for the column sums.
          uint4* vt = reinterpret_cast<uint4*>(sk + L::kTile);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int u = ct + 128 * j;
            const int row = (u * 16 % 8192) / 128;
            const float c = key0 + row < p.N ? __ldg(p.row_scale + (int64_t)bh * p.N + key0 + row) : 0.0f;
            uint4 v = vt[u];
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = __bfloat1622float2(h[k]);
              h[k] = __floats2bfloat162_rn(f.x * c, f.y * c);
            }
            vt[u] = v;
          }
          if (ct < 64) sE[slot * 64 + ct] = key0 + ct < p.N ? __ldg(p.row_w + (int64_t)bh * p.N + key0 + ct) : 0.0f;
        }
      }
      fence_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the whole tile is phi(K) (and scaled V)
      mbar_arrive(bar(L::kBarReady + slot));
      // Column ct of the phi(K) tile: z_tile (or, with GRAD, sum_i e_i phi(q_i)).
      float cs = 0.0f;
      if (ok) {
        const uint8_t* box = sk + (ct >> 6) * 8192;
        const int col = ct & 63;
        float part[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 16
        for (int row = 0; row < 64; ++row) {
          const float v = box_at(box, row, col);
          part[row & 3] = GRAD ? fmaf(sE[slot * 64 + row], v, part[row & 3]) : part[row & 3] + v;
        }
        cs = (part[0] + part[1]) + (part[2] + part[3]);
      }
      if (p.z_tile != nullptr) p.z_tile[((int64_t)bh * p.ntiles + tile_of(i)) * 128 + ct] = cs;
      zacc += cs;
      mbar_arrive(bar(L::kBarEmpty + slot));
      if (seg_last(i)) {
        // The segment's accumulator -> partial slot (blockIdx.x + bh): row a
        // from this thread's TMEM lane; column 128 = the column sum of
        // feature ct.
        const int acc = seg & 1;
        if (ok) ok = warp_wait(L::kBarAccFull + acc, (seg >> 1) & 1, kErrLinMma);
        tc_fence_after();
        float* prow = p.partial + (((int64_t)blockIdx.x + bh) * 128 + a) * 129;
#pragma unroll 1
        for (int c = 0; c < 128; c += 16) {
          uint32_t v[16];
          if (ok) {
            tmem_ld16(tmem + lane_off + acc * 128 + c, v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0u;
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) prow[c + j] = __uint_as_float(v[j]);
        }
        p.partial[(((int64_t)blockIdx.x + bh) * 128 + ct) * 129 + 128] = zacc;
        zacc = 0.0f;
        tc_fence_before();
        mbar_arrive(bar(L::kBarAccFree + acc));
        ++seg;
      }
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

// S_all / z_all of each head = the sum of its partials, in CTA order: head h
// was covered by the CTAs c = floor(h ntiles / W) .. floor(((h + 1) ntiles - 1) / W),
// whose partials sit at slots c + h. One thread per element of the
// [128][129] summary.
__global__ void __launch_bounds__(256) linear_reduce_kernel(const float* __restrict__ partial, int ntiles,
                                                            int64_t per_cta, float* __restrict__ s_all,
                                                            float* __restrict__ z_all) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= kLinPartial) return;
  const int64_t c0 = (int64_t)bh * ntiles / per_cta, c1 = ((int64_t)bh * ntiles + ntiles - 1) / per_cta;
  float acc = 0.0f;
  for (int64_t c = c0; c <= c1; ++c) acc += partial[(c + bh) * kLinPartial + e];
  const int a = e / 129, c = e % 129;
  if (c < 128)
    s_all[((int64_t)bh * 128 + a) * 128 + c] = acc;
  else
    z_all[(int64_t)bh * 128 + a] = acc;
}

}  // namespace sparge
