// Low-bit block-sparse attention forward (SLA2 article, arXiv:2602.12675,
// section 3: the sparse branch computes with its queries, keys, attention
// probabilities and values in a low-bit format, scaled into the format's
// range and back).
//
// Operands come from quant.cuh: int8 codes of Q and K with one scale per
// block, e4m3 codes of V with one scale per channel. For one query row i of
// query block I and the kept key tiles (64 keys, ascending) of its block:
//   S_j = q8_i . k8_j                     exact int32, tcgen05 kind::i8
//   x_j = float(S_j) * c_IJ,              c_IJ = c0 / (s_q[I] * s_k[J]) in fp32,
//                                         c0 = log2(e) / sqrt(d)
//   m   = an integer reference: ceil(max_j x_j) of the first tile, moved up
//         to a tile's ceil(max_j x_j) only when that exceeds m + 2 (O and l
//         then scaled by the exact 2^(m_old - m_new)), so max_j x_j <= m + 2
//   e_j = 2^(x_j - (m - 6)),  l += e_j,  p_j = e4m3(e_j)   (e_j <= 2^8 < 448)
//   O  += p_j v8_j                        fp32 in TMEM, tcgen05 kind::f8f6f4
// and O_i = O / (l * s_v) per channel. P is thereby scaled into e4m3's range:
// the row's largest code lies in (2^5, 2^8]. The library's definition puts
// it in (2^7, 2^8] (reference ceil of the max over every kept key, minus 8);
// since the references are integers and e4m3 rounding commutes with powers
// of two above its subnormals, the two differ only in the codes of keys more
// than 12 binades below the row's max.
//
// Same warp roles and pipeline as the bf16 kernel (attn.cuh): warp 0 TMA
// producer, warp 1 MMA issuer (whole warp, one elected lane issues), warps
// 2..5 softmax and epilogue; two CTAs per SM. 8-bit operands halve the shared
// memory per tile (Q 16 KB, K and V 8 KB each) and the MMA instructions per
// tile (four for S, K = 32 bytes each; two for P V).
// TMEM columns: S0 [0,64), S1 [64,128) (int32), O [128,256) (fp32); the 64
// e4m3 codes of P(t), four per 32-bit column, go over the first 16 columns
// of S(t)'s buffer.
#pragma once
#include <cuda.h>
#include <climits>
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "attn.cuh"
#include "quant.cuh"

namespace sparge {

constexpr int kQ8Threads = 192;

enum : unsigned int {
  kErrQ8Q = 0x500, kErrQ8KFull, kErrQ8VFull, kErrQ8KEmpty, kErrQ8VEmpty, kErrQ8SFull, kErrQ8PFull, kErrQ8ODone,
  kErrQ8OFinal, kErrQ8Drain
};

struct Q8Params {
  const int32_t* kv_idx;  // [BH, nqb, nkb]
  const int32_t* kv_cnt;  // [BH, nqb]
  const int32_t* order;   // [BH * nqb] launch order of the tiles, or null (head-major)
  const float* sq;        // [BH, nqb]
  const float* sk;        // [BH, nkb]
  const float* sv;        // [BH, 128]
  int N;
  int nqb;
  int nkb;
  int bq;
  int bk;
  float c0;               // log2(e) / sqrt(128), in fp32
};

struct Q8Smem {
  static constexpr int NS = 2;
  static constexpr int kQBytes = kTileQ * 128;  // 128 rows x 128 one-byte codes
  static constexpr int kKBytes = kTileK * 128;
  static constexpr int kVBytes = kTileK * 128;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + NS * kKBytes;
  static constexpr int kOffO = kOffV + NS * kVBytes;  // bf16 output staging (two 64-column boxes)
  static constexpr int kOffBar = kOffO + kTileQ * 128 * 2;
  static constexpr int kBarQ = 0, kBarKFull = 1, kBarVFull = 1 + NS, kBarKEmpty = 1 + 2 * NS,
                       kBarVEmpty = 1 + 3 * NS, kBarSFull = 1 + 4 * NS, kBarPFull = 3 + 4 * NS,
                       kBarODone = 5 + 4 * NS, kBarOFinal = 6 + 4 * NS, kBarDrain = 7 + 4 * NS;
  static constexpr int kNumBars = 8 + 4 * NS;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kUsed = kOffTmem + 16;
  // At most two CTAs per SM: two CTAs x 256 TMEM columns fill the SM's 512.
  static constexpr int kBytes = (kUsed + 1024 > 80 * 1024 ? kUsed + 1024 : 80 * 1024);
};

// Instruction descriptors (kind::i8 and kind::f8f6f4): D format bits 4-5
// (1 = f32, 2 = s32), A and B formats bits 7-9 / 10-12 (s8 = 1; e4m3 = 0),
// B major bit 16 (1 = MN-major), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem desc] * B[smem desc], int8 operands, int32 accumulator.
__device__ __forceinline__ void mma_ss_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], fp8 operands, fp32 accumulator.
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// int32 -> float, exact for |v| < 2^22: the integer is placed in the mantissa
// of 1.5 * 2^23 and the offset taken off again (integer add, float subtract).
__device__ __forceinline__ float i2f_small(int v) {
  return __fsub_rn(__uint_as_float((uint32_t)v + 0x4B400000u), 12582912.0f);
}

// Largest of the row's 64 scores: eight independent chains, then a tree.
__device__ __forceinline__ int row_max64_i(const int (&s)[kTileK]) {
  int m8[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    m8[j] = max(max(max(s[j], s[8 + j]), max(s[16 + j], s[24 + j])),
                max(max(s[32 + j], s[40 + j]), max(s[48 + j], s[56 + j])));
  return max(max(max(m8[0], m8[1]), max(m8[2], m8[3])), max(max(m8[4], m8[5]), max(m8[6], m8[7])));
}

__global__ void __launch_bounds__(kQ8Threads, 2)
    attn_q8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const Q8Params p) {
  using L = Q8Smem;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t sQ = sbase + L::kOffQ, sK = sbase + L::kOffK, sV = sbase + L::kOffV, sO = sbase + L::kOffO;
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffTmem + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = p.order ? __ldg(p.order + blockIdx.x) : (int)blockIdx.x;  // (bh, query block)
  const int bh = tile / p.nqb;
  const int qb = tile % p.nqb;
  const int q0 = qb * p.bq;
  const int tiles_per_block = p.bk / kTileK;
  const int cnt = min(max(__ldg(p.kv_cnt + tile), 0), p.nkb);
  const int T = cnt * tiles_per_block;
  const int32_t* lst = p.kv_idx + (int64_t)tile * p.nkb;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarQ), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::kBarKFull + s), 1);
      mbar_init(bar(L::kBarVFull + s), 1);
      mbar_init(bar(L::kBarKEmpty + s), 1);
      mbar_init(bar(L::kBarVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::kBarSFull + s), 1);
      mbar_init(bar(L::kBarPFull + s), 128);
    }
    mbar_init(bar(L::kBarODone), 1);
    mbar_init(bar(L::kBarOFinal), 1);
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
  const uint32_t tS = tmem, tO = tmem + 128;
  auto warp_wait = [&](int b, uint32_t parity, unsigned int site) {
    return __all_sync(0xffffffffu, role_wait(bar(b), parity, site, abort_flag));
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && T > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar(L::kBarQ), L::kQBytes);
      tma_load_3d(sQ, &tmQ, bar(L::kBarQ), 0, q0, bh);
      int nk = 0, nv = 0;
      int key_next = tile_key0(lst, 0, tiles_per_block, p.bk);
      for (int t = 0; t < T; ++t) {
        const int slot = t % NS, round = t / NS;
        const int key0 = key_next;
        if (t + 1 < T) key_next = tile_key0(lst, t + 1, tiles_per_block, p.bk);
        if (t >= NS && !role_wait(bar(L::kBarKEmpty + slot), (round - 1) & 1, kErrQ8KEmpty, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::kBarKFull + slot), L::kKBytes);
        tma_load_3d(sK + slot * L::kKBytes, &tmK, bar(L::kBarKFull + slot), 0, key0, bh);
        ++nk;
        if (t >= NS && !role_wait(bar(L::kBarVEmpty + slot), (round - 1) & 1, kErrQ8VEmpty, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::kBarVFull + slot), L::kVBytes);
        tma_load_3d(sV + slot * L::kVBytes, &tmV, bar(L::kBarVFull + slot), 0, key0, bh);
        ++nv;
      }
      mbar_wait(bar(L::kBarQ), 0, kErrQ8Q);
      for (int t = (nk > NS ? nk - NS : 0); t < nk; ++t)
        mbar_wait(bar(L::kBarKFull + t % NS), (t / NS) & 1, kErrQ8KFull);
      for (int t = (nv > NS ? nv - NS : 0); t < nv; ++t)
        mbar_wait(bar(L::kBarVFull + t % NS), (t / NS) & 1, kErrQ8VFull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (T > 0) {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_s8_s32(kTileQ, kTileK);
      constexpr uint32_t idPV = idesc_e4m3_f32(kTileQ, 128, true);
      const uint64_t dQ = sdesc_sw128(sQ, 16, 1024);            // K-major, one 128-byte atom per row
      const uint64_t dK = sdesc_sw128(sK, 16, 1024);
      const uint64_t dV = sdesc_sw128(sV, kTileK * 128, 1024);  // MN-major: 128 codes per key row
      bool ok = warp_wait(L::kBarQ, 0, kErrQ8Q);
      tc_fence_after();
      for (int t = 0; ok && t <= T; ++t) {
        if (t < T) {
          const int slot = t % NS;
          if (!warp_wait(L::kBarKFull + slot, (t / NS) & 1, kErrQ8KFull)) break;
          tc_fence_after();
          if (leader) {
            const uint64_t dKs = dK + (uint64_t)((slot * L::kKBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // 32 one-byte codes = 32 bytes along K per MMA
              mma_ss_i8(tS + (t & 1) * 64, dQ + kk * 2, dKs + kk * 2, idS, kk > 0 ? 1u : 0u);
            mma_commit(bar(L::kBarSFull + (t & 1)));
            mma_commit(bar(L::kBarKEmpty + slot));
          }
          __syncwarp();
        }
        if (t >= 1) {
          const int u = t - 1, vs = u % NS;
          if (!warp_wait(L::kBarVFull + vs, (u / NS) & 1, kErrQ8VFull)) break;
          if (!warp_wait(L::kBarPFull + (u & 1), (u >> 1) & 1, kErrQ8PFull)) break;
          tc_fence_after();
          if (leader) {
            const uint64_t dVs = dV + (uint64_t)((vs * L::kVBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)  // 32 keys: 8 TMEM columns of P, 4096 bytes of V
              mma_ts_f8(tO, tS + (u & 1) * 64 + kk * 8, dVs + kk * 256, idPV, (u > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar(L::kBarVEmpty + vs));
            mma_commit(bar(L::kBarODone));
            if (u == T - 1) mma_commit(bar(L::kBarOFinal));
          }
          __syncwarp();
        }
      }
      if (leader) mma_commit(bar(L::kBarDrain));
      __syncwarp();
      mbar_wait(bar(L::kBarDrain), 0, kErrQ8Drain);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    const float sqv = __ldg(p.sq + tile);
    const float* skh = p.sk + (int64_t)bh * p.nkb;
    // Kept-block indices and their score factors c = c0 / (s_q * s_k), 32
    // at a time, one per lane, a chunk ahead (the division runs once per
    // entry, in parallel across the lanes).
    auto factor = [&](int J) { return __fdiv_rn(p.c0, __fmul_rn(sqv, __ldg(skh + J))); };
    int idx_cur = lane < cnt ? __ldg(lst + lane) : 0;
    int idx_nxt = 32 + lane < cnt ? __ldg(lst + 32 + lane) : 0;
    float c_cur = factor(idx_cur), c_nxt = factor(idx_nxt);
    for (int t = 0; t < T; ++t) {
      const int pb = t & 1;
      const int e = t / tiles_per_block, sub = t % tiles_per_block;
      if (e > 0 && (e & 31) == 0 && sub == 0) {
        idx_cur = idx_nxt;
        c_cur = c_nxt;
        idx_nxt = e + 32 + lane < cnt ? __ldg(lst + e + 32 + lane) : 0;
        c_nxt = factor(idx_nxt);
      }
      const int key0 = __shfl_sync(0xffffffffu, idx_cur, e & 31) * p.bk + sub * kTileK;
      const float c = __shfl_sync(0xffffffffu, c_cur, e & 31);
      ok = warp_wait(L::kBarSFull + pb, (t >> 1) & 1, kErrQ8SFull);
      if (!ok) break;
      tc_fence_after();
      int s[kTileK];
      {
        uint32_t v[4][16];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_ld16(tS + lane_off + pb * 64 + 16 * cc, v[cc]);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int j = 0; j < 16; ++j) s[16 * cc + j] = (int)v[cc][j];
      }
      const bool full_tile = key0 + kTileK <= p.N;  // the same for every row of the tile
      const int nvalid = full_tile ? kTileK : p.N - key0;
      if (!full_tile) {  // keys past N (zero-filled K rows) must not win the max
#pragma unroll
        for (int j = 0; j < kTileK; ++j)
          if (j >= nvalid) s[j] = INT_MIN;
      }
      const int smax = row_max64_i(s);
      // A tile wholly past N (the second tile of a ragged 128-key block) has
      // no valid key: it leaves m as it is and contributes nothing.
      const float cm = nvalid > 0 ? ceilf(__fmul_rn(i2f_small(smax), c)) : m_run;
      // Each row moves its reference only past a margin of 2 binades (its
      // own decision, so the result does not depend on the other rows of the
      // warp).
      const float m_new = (t == 0 || cm > m_run + 2.0f) ? cm : m_run;
      if (t == 0) {
        m_run = m_new;
      } else if (__any_sync(0xffffffffu, m_new > m_run)) {
        // Exact rescale by 2^(m_run - m_new), an integer power of two; rows
        // whose reference held scale by 1.
        ok = warp_wait(L::kBarODone, (t - 1) & 1, kErrQ8ODone);
        if (!ok) break;
        tc_fence_after();
        const int sh = (int)(m_run - m_new);  // <= 0
        const float f = sh < -126 ? 0.0f : __int_as_float((127 + sh) << 23);
        rescale_row<128>(tO + lane_off, f);
        l_run *= f;
        m_run = m_new;
      }
      // e = 2^(x - (m - 6)), x = float(S) * c; codes e4m3(e); l += e.
      const float negref = 6.0f - m_run;
      const uint64_t c2 = f2(c, c), negm2 = f2(negref, negref), magic2 = f2(12582912.0f, 12582912.0f);
      uint64_t acc[2] = {0ull, 0ull};
      uint32_t pw[kTileK / 4];
#pragma unroll
      for (int k = 0; k < kTileK / 2; ++k) {
        const uint64_t sf = sub2(f2(__uint_as_float((uint32_t)s[2 * k] + 0x4B400000u),
                                    __uint_as_float((uint32_t)s[2 * k + 1] + 0x4B400000u)),
                                 magic2);
        const uint64_t y = add2(fma2(sf, c2, 0ull), negm2);
        const float2 yv = f2_split(y);
        float ea = ex2_approx(yv.x), eb = ex2_approx(yv.y);
        if (!full_tile) {
          if (2 * k >= nvalid) ea = 0.0f;
          if (2 * k + 1 >= nvalid) eb = 0.0f;
        }
        acc[k & 1] = add2(acc[k & 1], f2(ea, eb));
        const uint32_t code = e4m3x2(eb, ea);  // key 2k in the low byte
        if (k & 1)
          pw[k >> 1] |= code << 16;
        else
          pw[k >> 1] = code;
      }
      {
        const float2 a = f2_split(add2(acc[0], acc[1]));
        l_run += a.x + a.y;
      }
      tmem_st16(tS + lane_off + pb * 64, pw);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarPFull + pb));
    }
    if (ok && T > 0) {
      ok = warp_wait(L::kBarOFinal, 0, kErrQ8OFinal);
      tc_fence_after();
    }
    const float inv_l = (T > 0 && l_run > 0.0f) ? 1.0f / l_run : 0.0f;
    const float* svh = p.sv + (int64_t)bh * 128;
#pragma unroll 1
    for (int cc = 0; cc < 128; cc += 16) {
      uint32_t v[16];
      if (T > 0 && ok) {
        tmem_ld16(tO + lane_off + cc, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
      float o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = __uint_as_float(v[j]) * inv_l / __ldg(svh + cc + j);
      stage_row16(sO, r, cc, o);
    }
    fence_async_smem();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (warp == 2 && lane == 0) {
      for (int b = 0; b < 2; ++b) tma_store_3d(&tmO, sO + b * (kTileQ * 128), b * 64, q0, bh);
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
