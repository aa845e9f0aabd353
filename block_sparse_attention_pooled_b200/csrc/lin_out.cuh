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
// One CTA takes two neighbouring query blocks, A = 2c and B = 2c + 1 of one
// (batch, head) (A alone for the last block of an odd count). Neighbouring
// query blocks keep mostly the same key blocks, so the CTA walks the
// ascending union of the two kept lists and loads each phi(K)/V tile of it
// once. Two accumulators hold the two sums without multiplying a shared tile
// twice: with X the block whose list is the shorter and Y the other,
//   D_base = S_kept,X                 (the tiles X keeps)
//   D_diff = S_kept,Y - S_kept,X      (+ the tiles only Y keeps,
//                                      - the tiles only X keeps, by the MMA's
//                                      negate-A bit)
// and S_kept,Y = D_base + D_diff. A tile both keep costs one product, a tile
// only X keeps two, a tile only Y keeps one. On the video workloads that is
// about 1.2 products per union tile against the 1.5 the two blocks need on
// their own, and one operand load per union tile instead of 1.5.
//
// 192 threads:
//   warp 0      TMA producer (whole warp, one elected lane issues): the union's
//               phi(K) and V tiles into a three-slot ring; then Q_A into the
//               slot the next tile would take and Q_B into the slot of the
//               last tile, each as soon as its slot is free;
//   warp 1      MMA issuer (whole warp, one elected lane issues) and TMEM
//               owner: D_base / D_diff [feature, 0..127] +/-= phi(K_t)^T V_t
//               (M 128, N 128, K 64 per tile, both operands MN-major), each
//               starting from zero, in TMEM columns 0..127 (D0) and
//               128..255 (D1); then phi(Q_A) S_c,A into D0 and phi(Q_B) S_c,B
//               into D1;
//   warps 2..5  while the MMAs run, z_kept of both blocks (thread r adds
//               z_tile[t][r] over each kept list) and the loads of row r of
//               S_all; then the epilogue, TMEM lane r being feature r for
//               S_c = S_all - S_kept and query row r for the outputs:
//                 1. S_c,A and S_c,B in fp32 over the accumulators (D0 and
//                    D1), so that row r of S_all is read once; S_c,A as bf16
//                    into the staging slot (the MN-major B operand);
//                 2. phi(Q_A) in place; the output product of A may start;
//                    phi(Q_B) in place and both denominators
//                    phi(q_r) . z_c in fp32 while it runs;
//                 3. once A's product is done: S_c,B from D1 into the staging
//                    slot (B's product may start), then O_A from D0 to
//                    shared memory and out by TMA; then O_B the same way.
// Shared memory: ring slot s = [phi(K) 16 KB | V 16 KB]. With T union tiles,
// Q_A (32 KB) goes to slot T % 3 (free once tile T - 3's product is done),
// Q_B to slot (T + 2) % 3 (tile T - 1's) and the staged S_c (two 128-row
// boxes, 32 KB) to slot (T + 1) % 3; each Q slot then holds phi(Q) and then
// the output. Three slots keep two CTAs per SM, six tiles in flight per SM.
#pragma once
#include <cuda.h>
#include <climits>
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "attn.cuh"

namespace sparge {

constexpr int kLoThreads = 192;

enum : unsigned int {
  kErrLoFull = 0x300, kErrLoEmpty, kErrLoKept, kErrLoQ, kErrLoStage, kErrLoOut, kErrLoDrain
};

struct LoSmem {
  static constexpr int NS = 3;
  static constexpr int kTile = 64 * 128 * 2;         // phi(K) or V tile: two 64-column boxes of 64 keys
  static constexpr int kSlot = 2 * kTile;            // 32 KB
  static constexpr int kOffZ = NS * kSlot;           // z_c of A and of B: [2][128] fp32
  static constexpr int kOffBar = kOffZ + 2 * 128 * 4;
  static constexpr int kBarFull = 0, kBarEmpty = NS, kBarKept = 2 * NS, kBarQ0 = 2 * NS + 1,
                       kBarQ1 = 2 * NS + 2, kBarStage0 = 2 * NS + 3, kBarStage1 = 2 * NS + 4,
                       kBarOut0 = 2 * NS + 5, kBarOut1 = 2 * NS + 6, kBarDrain = 2 * NS + 7;
  static constexpr int kNumBars = 2 * NS + 8;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // TMEM base, abort flag, union tile count, written sums
  static constexpr int kBytes = kOffMisc + 16 + 1024;     // + alignment slack: two CTAs per SM
  static_assert(kSlot == 2 * 128 * 128, "a Q tile and S_c each fill one ring slot");
};

struct LoParams {
  const int32_t* kv_idx;  // [BH, nqb, nkb]
  const int32_t* kv_cnt;  // [BH, nqb]
  const float* s_all;     // [BH, 128, 128] fp32, row = feature
  const float* z_all;     // [BH, 128] fp32
  const float* z_tile;    // [BH, ntiles, 128] fp32
  const float* alpha;     // [H]
  float* den_out;         // [BH, N] or null: phi(q) . z_c per row (0 where the branch is off)
  float* zc_out;          // [BH * nqb, 128] or null: z_c per query block
  int store_sc;           // nonzero: S_c per query block as bf16 [BH * nqb, 128, 128] through tmSc
  int H;
  int N;
  int ntiles;             // ceil(N / 64)
  int nqb;
  int nkb;
  int bq;
  int bk;
};

// A warp's cursor over an ascending kept-block list: lane i holds entry
// (pos & ~31) + i in `cur` and the one 32 further in `nxt`, so the next chunk
// is in flight a chunk ahead of use. Every lane calls head() and step() with
// the same pos.
struct KeptCursor {
  const int32_t* lst;
  int cnt, pos, cur, nxt;
  __device__ __forceinline__ void init(const int32_t* l, int c, int lane) {
    lst = l;
    cnt = c;
    pos = 0;
    cur = lane < c ? __ldg(l + lane) : 0;
    nxt = 32 + lane < c ? __ldg(l + 32 + lane) : 0;
  }
  __device__ __forceinline__ int head() const {
    const int v = __shfl_sync(0xffffffffu, cur, pos & 31);
    return pos < cnt ? v : INT_MAX;
  }
  __device__ __forceinline__ void step(int lane) {
    ++pos;
    if ((pos & 31) == 0) {
      cur = nxt;
      nxt = pos + 32 + lane < cnt ? __ldg(lst + pos + 32 + lane) : 0;
    }
  }
};

// Next key block of the union of two ascending lists: returns false at the
// end, else the block and whether list a and list b hold it.
__device__ __forceinline__ bool union_next(KeptCursor& a, KeptCursor& b, int lane, int& kb, bool& in_a,
                                           bool& in_b) {
  const int ha = a.head(), hb = b.head();
  kb = min(ha, hb);
  if (kb == INT_MAX) return false;
  in_a = ha == kb;
  in_b = hb == kb;
  if (in_a) a.step(lane);
  if (in_b) b.step(lane);
  return true;
}

__global__ void __launch_bounds__(kLoThreads, 2)
    linear_out_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmPhiK, const __grid_constant__ CUtensorMap tmO,
                      const __grid_constant__ CUtensorMap tmSc, const LoParams p) {
  using L = LoSmem;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  float* zc = reinterpret_cast<float*>(sgen + L::kOffZ);  // [2][128] z_c of A, of B
  const uint32_t bar0 = sbase + L::kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kOffMisc + 4);
  volatile int* tiles_slot = reinterpret_cast<volatile int*>(sgen + L::kOffMisc + 8);
  volatile int* sums_slot = reinterpret_cast<volatile int*>(sgen + L::kOffMisc + 12);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int npairs = (p.nqb + 1) / 2;
  const int bh = (int)(blockIdx.x / (unsigned)npairs);
  const int qa = 2 * (int)(blockIdx.x % (unsigned)npairs);  // query block A; B = qa + 1
  const bool has_b = qa + 1 < p.nqb;
  const int64_t tile_a = (int64_t)bh * p.nqb + qa;
  const int cnt_a = min(max(__ldg(p.kv_cnt + tile_a), 0), p.nkb);
  const int cnt_b = has_b ? min(max(__ldg(p.kv_cnt + tile_a + 1), 0), p.nkb) : 0;
  const int32_t* lst_a = p.kv_idx + tile_a * p.nkb;
  const int32_t* lst_b = lst_a + p.nkb;
  const int q0a = qa * p.bq, q0b = q0a + p.bq;
  const int tiles_per_block = p.bk / 64;
  // The shorter list is X (the base sum): A when cnt_a <= cnt_b.
  const bool base_is_a = cnt_a <= cnt_b;
  const uint32_t col_base = base_is_a ? 0u : 128u, col_diff = 128u - col_base;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::kBarFull + s), 1);
      mbar_init(bar(L::kBarEmpty + s), 1);
    }
    mbar_init(bar(L::kBarKept), 2);  // the MMA issuer's arrive (with the tile count) and its commit
    mbar_init(bar(L::kBarQ0), 1);
    mbar_init(bar(L::kBarQ1), 1);
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
  // Slots of the epilogue, given the union's tile count T.
  auto slot_addr = [&](int T, int k) { return sbase + (uint32_t)(((T + k) % NS) * L::kSlot); };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tmPhiK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmQ);
    }
    KeptCursor ca, cb;
    ca.init(lst_a, cnt_a, lane);
    cb.init(lst_b, cnt_b, lane);
    int t = 0, issued = 0, kb;
    bool in_a, in_b, ok = true;
    while (union_next(ca, cb, lane, kb, in_a, in_b)) {
      for (int sub = 0; sub < tiles_per_block; ++sub, ++t) {
        const int slot = t % NS;
        if (ok && t >= NS) ok = warp_wait(L::kBarEmpty + slot, (t / NS - 1) & 1, kErrLoEmpty);
        if (!ok) continue;  // keep counting: T fixes the epilogue's slots
        if (leader) {
          const uint32_t sp = sbase + slot * L::kSlot, sv = sp + L::kTile;
          const int key0 = kb * p.bk + sub * 64;
          mbar_arrive_expect_tx(bar(L::kBarFull + slot), L::kSlot);
          for (int b = 0; b < 2; ++b) {
            tma_load_3d(sp + b * 8192, &tmPhiK, bar(L::kBarFull + slot), b * 64, key0, bh);
            tma_load_3d(sv + b * 8192, &tmV, bar(L::kBarFull + slot), b * 64, key0, bh);
          }
        }
        __syncwarp();
        ++issued;
      }
    }
    const int T = t;
    // Q_A goes to slot T % NS, as a tile T would: once tile T - NS's product
    // (if any) has read that slot. Q_B goes to slot (T + 2) % NS = (T - 1) % NS,
    // once the last tile's product has read it.
    bool qa_issued = false, qb_issued = false;
    if (ok && (T < NS || warp_wait(L::kBarEmpty + T % NS, (T / NS - 1) & 1, kErrLoEmpty))) {
      if (leader) {
        const uint32_t sq = slot_addr(T, 0);
        mbar_arrive_expect_tx(bar(L::kBarQ0), 2 * 128 * 128);
        for (int b = 0; b < 2; ++b) tma_load_3d(sq + b * (128 * 128), &tmQ, bar(L::kBarQ0), b * 64, q0a, bh);
      }
      qa_issued = true;
    } else {
      ok = false;
    }
    if (has_b && ok && (T < 1 || warp_wait(L::kBarEmpty + (T - 1) % NS, ((T - 1) / NS) & 1, kErrLoEmpty))) {
      if (leader) {
        const uint32_t sq = slot_addr(T, 2);
        mbar_arrive_expect_tx(bar(L::kBarQ1), 2 * 128 * 128);
        for (int b = 0; b < 2; ++b) tma_load_3d(sq + b * (128 * 128), &tmQ, bar(L::kBarQ1), b * 64, q0b, bh);
      }
      qb_issued = true;
    }
    // Never leave with copies in flight.
    if (leader) {
      for (int u = (issued > NS ? issued - NS : 0); u < issued; ++u)
        mbar_wait(bar(L::kBarFull + u % NS), (u / NS) & 1, kErrLoFull);
      if (qa_issued) mbar_wait(bar(L::kBarQ0), 0, kErrLoQ);
      if (qb_issued) mbar_wait(bar(L::kBarQ1), 0, kErrLoQ);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    constexpr uint32_t idKept = idesc_bf16_f32(128, 128, true, true);
    constexpr uint32_t idKeptNeg = idKept | (1u << 13);  // negate A: -phi(K_t)^T V_t
    constexpr uint32_t idOut = idesc_bf16_f32(128, 128, false, true);
    const uint64_t dRing = sdesc_sw128(sbase, 64 * 128, 1024);  // MN-major, 64-row boxes
    KeptCursor ca, cb;
    ca.init(lst_a, cnt_a, lane);
    cb.init(lst_b, cnt_b, lane);
    int t = 0, kb;
    bool in_a, in_b, ok = true, started_base = false, started_diff = false;
    while (union_next(ca, cb, lane, kb, in_a, in_b)) {
      const bool in_x = base_is_a ? in_a : in_b, in_y = base_is_a ? in_b : in_a;
      for (int sub = 0; sub < tiles_per_block; ++sub, ++t) {
        const int slot = t % NS;
        if (ok) ok = warp_wait(L::kBarFull + slot, (t / NS) & 1, kErrLoFull);
        if (ok) {
          tc_fence_after();
          if (leader) {
            const uint64_t dP = dRing + (uint64_t)((slot * L::kSlot) >> 4);
            const uint64_t dV = dP + (uint64_t)(L::kTile >> 4);
            if (in_x) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)  // 16 keys = 2048 bytes of each operand
                mma_ss(tmem + col_base, dP + kk * 128, dV + kk * 128, idKept, (started_base || kk > 0) ? 1u : 0u);
            }
            if (in_x != in_y) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem + col_diff, dP + kk * 128, dV + kk * 128, in_x ? idKeptNeg : idKept,
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
      mma_commit(bar(L::kBarKept));   // every S_kept MMA (none when T = 0) has completed
    }
    __syncwarp();
    const uint64_t dStage = sdesc_sw128(slot_addr(T, 1), 128 * 128, 1024);  // MN-major, 128-row boxes
    if (ok) ok = warp_wait(L::kBarStage0, 0, kErrLoStage);
    if (ok) {
      tc_fence_after();
      if (leader) {
        const uint64_t dQ = sdesc_sw128(slot_addr(T, 0), 16, 1024);  // K-major, 128-row boxes
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t qo = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
          mma_ss(tmem, dQ + qo, dStage + kk * 128, idOut, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::kBarOut0));
      }
      __syncwarp();
    }
    if (has_b && ok) ok = warp_wait(L::kBarStage1, 0, kErrLoStage);
    if (has_b && ok) {
      tc_fence_after();
      if (leader) {
        const uint64_t dQ = sdesc_sw128(slot_addr(T, 2), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t qo = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
          mma_ss(tmem + 128, dQ + qo, dStage + kk * 128, idOut, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::kBarOut1));
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
    const uint32_t tD0 = tmem + lane_off, tD1 = tmem + lane_off + 128;
    // z_kept[r] of one list, four loads in flight at a time. A last 128-key
    // block may hold a single 64-key tile: its second tile lies past N, has
    // no z_tile entry and adds nothing.
    const float* zt = p.z_tile + (int64_t)bh * p.ntiles * 128 + r;
    auto z_kept = [&](const int32_t* lst, int cnt) {
      auto ztile = [&](int tt) {
        const int tile64 = (__ldg(lst + tt / tiles_per_block) * p.bk + (tt % tiles_per_block) * 64) / 64;
        return tile64 < p.ntiles ? __ldg(zt + (int64_t)tile64 * 128) : 0.0f;
      };
      const int T1 = cnt * tiles_per_block;
      float zk = 0.0f;
      int t = 0;
      for (; t + 4 <= T1; t += 4) {
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = ztile(t + u);
        zk += (v[0] + v[1]) + (v[2] + v[3]);
      }
      for (; t < T1; ++t) zk += ztile(t);
      return zk;
    };
    const float zk_a = z_kept(lst_a, cnt_a);
    const float zk_b = has_b ? z_kept(lst_b, cnt_b) : 0.0f;
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
    const int T = *tiles_slot;
    const uint32_t sQa = slot_addr(T, 0), sStage = slot_addr(T, 1), sQb = slot_addr(T, 2);
    const int sums = *sums_slot;
    const bool has_base = ok && (sums & 1), has_diff = ok && (sums & 2);
    const uint32_t tBase = tD0 + col_base, tDiff = tD0 + col_diff;
    // 1. S_c,X = S_all - D_base and S_c,Y = S_c,X - D_diff for row r (an
    //    accumulator no product wrote counts as 0), in fp32 back over the
    //    two accumulators: then D0 holds S_c,A and D1 S_c,B, whichever block
    //    is X, and row r of S_all has been read once.
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
      uint32_t sx[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 a = sa[c / 4 + j];
        sx[4 * j] = __float_as_uint(a.x - __uint_as_float(v[4 * j]));
        sx[4 * j + 1] = __float_as_uint(a.y - __uint_as_float(v[4 * j + 1]));
        sx[4 * j + 2] = __float_as_uint(a.z - __uint_as_float(v[4 * j + 2]));
        sx[4 * j + 3] = __float_as_uint(a.w - __uint_as_float(v[4 * j + 3]));
      }
      if (has_diff) {
        tmem_ld16(tDiff + c, v);
        tmem_ld_wait_regs(v);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(sx[j]) - __uint_as_float(v[j]));
      tmem_st16(tBase + c, sx);
      tmem_st16(tDiff + c, v);
    }
    tmem_st_wait();
    //    S_c,A as bf16, MN-major for A's output product (two 64-column
    //    boxes of 128 rows, 128-byte swizzle), into the staging slot.
#pragma unroll 1
    for (int c = 0; c < 128; c += 16) {
      uint32_t v[16];
      tmem_ld16(tD0 + c, v);
      tmem_ld_wait_regs(v);
      float sc[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) sc[j] = __uint_as_float(v[j]);
      stage_row16(sStage, r, c, sc);
    }
    // 2. z_c of both blocks, then phi(Q_A) in place. phi is elementwise, so
    //    the tile is walked as a flat array of 16-byte units, consecutive
    //    threads on consecutive units (no bank conflicts).
    const float z_all_r = __ldg(p.z_all + (int64_t)bh * 128 + r);
    zc[r] = z_all_r - zk_a;
    zc[128 + r] = z_all_r - zk_b;
    auto phi_in_place = [&](uint32_t tile) {
      // Sixteen 16-byte units per thread: every load in flight before the
      // first conversion, every store after the last.
      constexpr int kUnits = (2 * 128 * 128) / 16 / 128;
      uint4* qt = reinterpret_cast<uint4*>(sgen + (tile - sbase));
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
    };
    if (ok) ok = warp_wait(L::kBarQ0, 0, kErrLoQ);
    if (ok) phi_in_place(sQa);
    fence_async_smem();
    tc_fence_before();
    mbar_arrive(bar(L::kBarStage0));
    asm volatile("bar.sync 1, 128;" ::: "memory");  // z_c and phi(Q_A) complete
    // For the backward: S_c,A (staged above) and both z_c out.
    if (p.store_sc && warp == 2 && lane == 0) {
      for (int b = 0; b < 2; ++b) tma_store_3d(&tmSc, sStage + b * (128 * 128), b * 64, 0, (int)tile_a);
      tma_store_commit();
    }
    if (p.zc_out != nullptr) {
      p.zc_out[tile_a * 128 + r] = zc[r];
      if (has_b) p.zc_out[(tile_a + 1) * 128 + r] = zc[128 + r];
    }
    // Denominator phi(q_r) . z_c in fp32; every block kept: the complement
    // is empty and the linear branch is 0.
    const float a_h = __ldg(p.alpha + (bh % p.H));
    auto row_weight = [&](uint32_t tile, const float* z, int cnt, int q0) {
      float den = 0.0f;
#pragma unroll 1
      for (int c = 0; c < 128; c += 16) {
        float qv[16];
        read_row16(tile, r, c, qv);
#pragma unroll
        for (int j = 0; j < 16; ++j) den = fmaf(qv[j], z[c + j], den);
      }
      const bool on = cnt < p.nkb && den > 0.0f;
      if (p.den_out != nullptr && r < p.bq && q0 + r < p.N) p.den_out[(int64_t)bh * p.N + q0 + r] = on ? den : 0.0f;
      return on ? (1.0f - a_h) / den : 0.0f;
    };
    const float wl_a = row_weight(sQa, zc, cnt_a, q0a);
    float wl_b = 0.0f;
    if (has_b) {
      if (ok) ok = warp_wait(L::kBarQ1, 0, kErrLoQ);
      if (ok) phi_in_place(sQb);
      asm volatile("bar.sync 1, 128;" ::: "memory");  // phi(Q_B) complete
      wl_b = row_weight(sQb, zc + 128, cnt_b, q0b);
    }
    // 3. A's product done: the staging slot is free for S_c,B (once the
    //    store of S_c,A, if any, has read it).
    if (ok) ok = warp_wait(L::kBarOut0, 0, kErrLoOut);
    tc_fence_after();
    if (p.store_sc && has_b) {
      if (warp == 2 && lane == 0) tma_store_wait_read0();
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
    if (has_b) {
#pragma unroll
      for (int c = 0; c < 128; c += 16) {
        uint32_t v[16];
        if (ok) {
          tmem_ld16(tD1 + c, v);
          tmem_ld_wait_regs(v);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0u;
        }
        float sc[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) sc[j] = __uint_as_float(v[j]);
        stage_row16(sStage, r, c, sc);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(L::kBarStage1));
    }
    // O tile = (1 - alpha_h) numerator / denominator, bf16, TMA store.
    auto store_output = [&](uint32_t tD, uint32_t tile, float wl, int q0) {
#pragma unroll 1
      for (int c = 0; c < 128; c += 16) {
        uint32_t v[16];
        if (ok) {
          tmem_ld16(tD + c, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0u;
        }
        float o[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] = wl * __uint_as_float(v[j]);
        stage_row16(tile, r, c, o);
      }
      fence_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (warp == 2 && lane == 0) {
        for (int b = 0; b < 2; ++b) tma_store_3d(&tmO, tile + b * (128 * 128), b * 64, q0, bh);
        tma_store_commit();
      }
    };
    store_output(tD0, sQa, wl_a, q0a);
    if (p.store_sc && has_b && warp == 2 && lane == 0) {  // S_c,B staged before the barrier in store_output
      for (int b = 0; b < 2; ++b) tma_store_3d(&tmSc, sStage + b * (128 * 128), b * 64, 0, (int)(tile_a + 1));
      tma_store_commit();
    }
    if (has_b) {
      if (ok) ok = warp_wait(L::kBarOut1, 0, kErrLoOut);
      tc_fence_after();
      store_output(tD1, sQb, wl_b, q0b);
    }
    if (warp == 2 && lane == 0) tma_store_wait_read0();  // the staging tiles have been read: the CTA may end
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
