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
//   G_all = sum_i phi(q_i) (c_i dO_i)^T     fp32 [d, d]
//   g_all = sum_i e_i phi(q_i)              fp32 [d]
// (K -> Q, V -> dO with row i scaled by c_i, the ones column -> e_i; no z_tile).
//
// One CTA handles a run of 64-key tiles of one head: TMA loads K and V tiles,
// the 128 threads apply phi to the K tile in place in shared memory (rows past
// N are zeroed), a TMA store writes the phi(K) tile out, and one thread issues
// tcgen05 MMAs D[feature, 0..143] += phi(K)^T [V | 1] with both operands
// MN-major in shared memory (the ones block after V yields z). At the end
// the 128 TMEM lanes (one per feature) are written out as this CTA's partial
// summary; linear_reduce_kernel then adds the partials of each head in a
// fixed order, so the result does not depend on scheduling.
#pragma once
#include <cuda.h>
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparge {

constexpr int kLinThreads = 128;
constexpr int kLinTilesPerCta = 64;   // 4096 keys per CTA
constexpr int kLinN = 144;            // 128 value columns + the ones block (16 used)

enum : unsigned int { kErrLinFull = 0x200, kErrLinMma, kErrLinDrain };

struct LinSmem {
  static constexpr int kK = 64 * 128 * 2;          // K / phi(K) tile: two 64-column boxes
  static constexpr int kV = 64 * 128 * 2 + 8192;   // V tile + ones block (next MN block)
  static constexpr int kSlot = kK + kV;
  static constexpr int kOffBar = 2 * kSlot;
  static constexpr int kOffTmem = kOffBar + 64;
  static constexpr int kBytes = kOffTmem + 16 + 1024;
};

constexpr int kLinPartial = 128 * 129;  // per CTA: [feature][128 value columns + z]

struct LinParams {
  float* partial;  // [BH, ctas_per_head, 128, 129]
  float* z_tile;   // [BH, ntiles, 128] (null with GRAD)
  const float* row_scale;  // GRAD: c_i [BH, N]
  const float* row_w;      // GRAD: e_i [BH, N]
  int N;
  int ntiles;         // ceil(N / 64)
  int ctas_per_head;
};


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

template <bool GRAD>
__global__ void __launch_bounds__(kLinThreads)
    linear_summary_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmPhiK, const LinParams p) {
  using L = LinSmem;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_mma = [&](int s) { return bar0 + 16u + 8u * s; };
  const uint32_t bar_drain = bar0 + 32u;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffTmem);

  const int tid = threadIdx.x, warp = tid / 32;
  const int bh = blockIdx.x / p.ctas_per_head;
  const int t0 = (blockIdx.x % p.ctas_per_head) * kLinTilesPerCta;
  const int t1 = min(p.ntiles, t0 + kLinTilesPerCta);
  const int n = t1 - t0;

  // Ones blocks (the 16 value columns after V of each slot) never change.
  for (int s = 0; s < 2; ++s) {
    uint4* ones = reinterpret_cast<uint4*>(sgen + s * L::kSlot + L::kK + 64 * 128 * 2);
    for (int u = tid; u < 8192 / 16; u += kLinThreads) ones[u] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  }
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_mma(s), 1);
    }
    mbar_init(bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(sbase + L::kOffTmem, 256);
    tmem_relinquish();
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto issue_load = [&](int i) {
    const int slot = i & 1, key0 = (t0 + i) * 64;
    const uint32_t sk = sbase + slot * L::kSlot, sv = sk + L::kK;
    mbar_arrive_expect_tx(bar_full(slot), 2 * 64 * 128 * 2);
    for (int b = 0; b < 2; ++b) {
      tma_load_3d(sk + b * 8192, &tmK, bar_full(slot), b * 64, key0, bh);
      tma_load_3d(sv + b * 8192, &tmV, bar_full(slot), b * 64, key0, bh);
    }
  };
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmPhiK);
    for (int i = 0; i < min(2, n); ++i) issue_load(i);
  }
  constexpr uint32_t idesc = idesc_bf16_f32(128, kLinN, true, true);
  bool ok = true;
  bool stalled = false;  // thread 0 gave up waiting for a slot to drain
  for (int i = 0; i < n; ++i) {
    const int slot = i & 1, key0 = (t0 + i) * 64;
    const uint32_t sk = sbase + slot * L::kSlot, sv = sk + L::kK;
    const bool got = !stalled && mbar_wait(bar_full(slot), (i >> 1) & 1, kErrLinFull);
    if (!__syncthreads_and(got)) {
      ok = false;
      break;
    }
    // phi in place; rows past N become zero so they add nothing.
    uint4* tile = reinterpret_cast<uint4*>(sgen + slot * L::kSlot);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int u = tid + kLinThreads * j;           // 16-byte unit of the 16 KB tile
      const int row = (u * 16 % 8192) / 128;          // key row inside the box
      tile[u] = (key0 + row < p.N) ? phi8(tile[u]) : make_uint4(0u, 0u, 0u, 0u);
    }
    if (GRAD) {
      // dO rows scaled by c_i (zero past N); the ones column carries e_i.
      uint4* vt = reinterpret_cast<uint4*>(sgen + slot * L::kSlot + L::kK);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int u = tid + kLinThreads * j;
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
      if (tid < 64) {
        const float e = key0 + tid < p.N ? __ldg(p.row_w + (int64_t)bh * p.N + key0 + tid) : 0.0f;
        uint8_t* ones = sgen + slot * L::kSlot + L::kK + 64 * 128 * 2;
        *reinterpret_cast<__nv_bfloat16*>(ones + tid * 128 + ((tid & 7) << 4)) = __float2bfloat16_rn(e);
      }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      for (int b = 0; b < 2; ++b) tma_store_3d(&tmPhiK, sk + b * 8192, b * 64, key0, bh);
      tma_store_commit();
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t a = sdesc_sw128(sk + kk * 2048, 8192, 1024);
        const uint64_t b = sdesc_sw128(sv + kk * 2048, 8192, 1024);
        mma_ss(tmem, a, b, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(bar_mma(slot));
    }
    if (!GRAD) {
      // z_tile: thread = feature; column sum over the tile's 64 rows of the
      // swizzled phi(K) tile (a warp reads 64 contiguous bytes per row).
      const int a = tid, col = a & 63;
      const uint8_t* tb = sgen + slot * L::kSlot + (a >> 6) * 8192;
      float zs = 0.0f;
#pragma unroll 8
      for (int row = 0; row < 64; ++row)
        zs += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
            tb + row * 128 + ((((col >> 3) ^ (row & 7)) << 4) | ((col & 7) << 1))));
      p.z_tile[((int64_t)bh * p.ntiles + t0 + i) * 128 + a] = zs;
    }
    if (i + 2 < n) {
      __syncthreads();  // every thread has finished reading the slot
      if (tid == 0) {
        // The slot is reused once its MMAs and its phi(K) store have read it.
        stalled = !mbar_wait(bar_mma(slot), (i >> 1) & 1, kErrLinMma);
        tma_store_wait_read0();
        if (!stalled) issue_load(i + 2);
      }
    }
  }
  if (tid == 0) {
    mma_commit(bar_drain);
    mbar_wait(bar_drain, 0, kErrLinDrain);
    tma_store_wait_read0();  // the phi(K) tiles have been read from shared memory: the CTA may end
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  {
    // Lane = feature a of this thread's warp quadrant: row a of this CTA's
    // partial [S | z] (zeros if the CTA gave up, so the reduction stays defined).
    const int a = warp * 32 + (tid % 32);
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float* prow = p.partial + ((int64_t)blockIdx.x * 128 + a) * 129;
#pragma unroll 1
    for (int c = 0; c < 144; c += 16) {
      uint32_t v[16];
      if (ok && n > 0) {
        tmem_ld16(tmem + lane_off + c, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (c + j < 129) prow[c + j] = __uint_as_float(v[j]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// S_all / z_all of each head = the sum of its CTAs' partials, in CTA order.
// One thread per element of the [128][129] summary.
// s_bf16 (optional): a bf16 copy of S_all, [BH, 128, 128] row-major.
__global__ void __launch_bounds__(256) linear_reduce_kernel(const float* __restrict__ partial, int ctas_per_head,
                                                            float* __restrict__ s_all, float* __restrict__ z_all,
                                                            __nv_bfloat16* __restrict__ s_bf16) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= kLinPartial) return;
  const float* src = partial + (int64_t)bh * ctas_per_head * kLinPartial + e;
  float acc = 0.0f;
  for (int k = 0; k < ctas_per_head; ++k) acc += src[(int64_t)k * kLinPartial];
  const int a = e / 129, c = e % 129;
  if (c < 128) {
    s_all[((int64_t)bh * 128 + a) * 128 + c] = acc;
    if (s_bf16 != nullptr) s_bf16[((int64_t)bh * 128 + a) * 128 + c] = __float2bfloat16_rn(acc);
  } else
    z_all[(int64_t)bh * 128 + a] = acc;
}

}  // namespace sparge
