// Operand codes for the low-bit sparse branch (SLA2 article, arXiv:2602.12675,
// section 3: the sparse branch's queries, keys, probabilities and values are
// mapped into a low-bit range with a scale, multiplied there, and scaled back).
//
// The article fixes neither the formats nor the scale granularity. Readings:
//   Q, K : int8, symmetric, one scale per (batch, head, block of bq / bk rows):
//          s = 127 / max|x| over the block (1 when the block is all zero),
//          code = rint(x * s) (ties to even) clamped to [-127, 127]; scale
//          and product in fp32.
//   V    : fp8 e4m3, one scale per (batch, head, channel) over every key:
//          s = 448 / max|v| (1 for an all-zero channel), code = e4m3(v * s)
//          rounded to nearest even, saturating; product in fp32.
// (P is coded inside the attention kernel.)
//
// Launch 1 (quant_qk_vmax_kernel): CTAs [0, q_ctas) code Q blocks,
// [q_ctas, q_ctas + k_ctas) code K blocks, the rest take the channel maxima
// of V over chunks of kVChunk rows. Launch 2 (quant_v_kernel): each CTA
// reduces its head's chunk maxima into the channel scales and codes one
// chunk of V.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparge {

constexpr int kQuantThreads = 128;
constexpr int kVChunk = 1024;  // rows of V per CTA

// Two floats to two e4m3 codes (hi, lo), rounded to nearest even, saturating.
__device__ __forceinline__ uint16_t e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ int8_t i8_code(float x, float s) {
  const int v = __float2int_rn(__fmul_rn(x, s));
  return (int8_t)max(-127, min(127, v));
}

// Largest value of v over the CTA's threads (all of them call it).
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  return m;
}

template <int D>
__global__ void __launch_bounds__(kQuantThreads)
    quant_qk_vmax_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                         const __nv_bfloat16* __restrict__ V, int64_t BH, int N, int bq, int bk, int64_t q_ctas,
                         int64_t k_ctas, int8_t* __restrict__ q8, float* __restrict__ sq, int8_t* __restrict__ k8,
                         float* __restrict__ sk, float* __restrict__ vpart) {
  __shared__ float red[kQuantThreads / 32];
  constexpr int TPR = D / 8;  // threads per row, 8 channels each
  constexpr int RPP = kQuantThreads / TPR;  // rows per pass
  const int tid = threadIdx.x, lr = tid / TPR, c0 = (tid % TPR) * 8;
  const int64_t cta = blockIdx.x;
  if (cta < q_ctas + k_ctas) {
    const bool is_q = cta < q_ctas;
    const int blk = is_q ? bq : bk;
    const int64_t nb = (N + blk - 1) / blk;
    const int64_t g = is_q ? cta : cta - q_ctas;  // bh * nb + block
    const int64_t bh = g / nb;
    const int r0 = (int)(g % nb) * blk, r1 = min(N, r0 + blk);
    const __nv_bfloat16* X = (is_q ? Q : K) + bh * (int64_t)N * D;
    float amax = 0.0f;
    for (int r = r0 + lr; r < r1; r += RPP) {
      const uint4 u = *reinterpret_cast<const uint4*>(X + (int64_t)r * D + c0);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h[j]);
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    amax = block_max(amax, red);
    const float s = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 1.0f;
    if (tid == 0) (is_q ? sq : sk)[g] = s;
    int8_t* out = (is_q ? q8 : k8) + bh * (int64_t)N * D;
    for (int r = r0 + lr; r < r1; r += RPP) {
      const uint4 u = *reinterpret_cast<const uint4*>(X + (int64_t)r * D + c0);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h[j]);
        const uint32_t lo = (uint8_t)i8_code(f.x, s), hi = (uint8_t)i8_code(f.y, s);
        w[j / 2] |= (lo | (hi << 8)) << (16 * (j % 2));
      }
      *reinterpret_cast<uint2*>(out + (int64_t)r * D + c0) = make_uint2(w[0], w[1]);
    }
    return;
  }
  // Channel maxima of V over one chunk of rows: each thread takes 8
  // channels of every RPP-th row (16-byte loads), then the row groups are
  // combined through shared memory.
  __shared__ float vm[RPP][D];
  const int64_t nch = (N + kVChunk - 1) / kVChunk;
  const int64_t g = cta - q_ctas - k_ctas;  // bh * nch + chunk
  const int64_t bh = g / nch;
  const int r0 = (int)(g % nch) * kVChunk, r1 = min(N, r0 + kVChunk);
  const __nv_bfloat16* X = V + bh * (int64_t)N * D;
  float m8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int r = r0 + lr; r < r1; r += RPP) {
    const uint4 u = *reinterpret_cast<const uint4*>(X + (int64_t)r * D + c0);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h[j]);
      m8[2 * j] = fmaxf(m8[2 * j], fabsf(f.x));
      m8[2 * j + 1] = fmaxf(m8[2 * j + 1], fabsf(f.y));
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) vm[lr][c0 + j] = m8[j];
  __syncthreads();
  if (tid < D) {
    float amax = 0.0f;
#pragma unroll
    for (int k = 0; k < RPP; ++k) amax = fmaxf(amax, vm[k][tid]);
    vpart[g * D + tid] = amax;
  }
}

template <int D>
__global__ void __launch_bounds__(kQuantThreads)
    quant_v_kernel(const __nv_bfloat16* __restrict__ V, int N, const float* __restrict__ vpart,
                   uint8_t* __restrict__ v8, float* __restrict__ sv) {
  __shared__ float s_sh[D];
  const int tid = threadIdx.x;
  const int64_t nch = (N + kVChunk - 1) / kVChunk;
  const int64_t g = blockIdx.x, bh = g / nch;
  const int r0 = (int)(g % nch) * kVChunk, r1 = min(N, r0 + kVChunk);
  if (tid < D) {
    float amax = 0.0f;
    for (int64_t k = 0; k < nch; ++k) amax = fmaxf(amax, vpart[(bh * nch + k) * D + tid]);
    const float s = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
    s_sh[tid] = s;
    if (g % nch == 0) sv[bh * D + tid] = s;
  }
  __syncthreads();
  constexpr int TPR = D / 8, RPP = kQuantThreads / TPR;
  const int lr = tid / TPR, c0 = (tid % TPR) * 8;
  const __nv_bfloat16* X = V + bh * (int64_t)N * D;
  uint8_t* out = v8 + bh * (int64_t)N * D;
  for (int r = r0 + lr; r < r1; r += RPP) {
    const uint4 u = *reinterpret_cast<const uint4*>(X + (int64_t)r * D + c0);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
    uint32_t w[2];
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      const float2 a = __bfloat1622float2(h[j]), b = __bfloat1622float2(h[j + 1]);
      const uint32_t lo = e4m3x2(__fmul_rn(a.y, s_sh[c0 + 2 * j + 1]), __fmul_rn(a.x, s_sh[c0 + 2 * j]));
      const uint32_t hi = e4m3x2(__fmul_rn(b.y, s_sh[c0 + 2 * j + 3]), __fmul_rn(b.x, s_sh[c0 + 2 * j + 2]));
      w[j / 2] = lo | (hi << 16);
    }
    *reinterpret_cast<uint2*>(out + (int64_t)r * D + c0) = make_uint2(w[0], w[1]);
  }
}

}  // namespace sparge
