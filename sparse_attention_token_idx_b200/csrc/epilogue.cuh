// The score epilogue shared by every scoring kernel ("Index scores" page:
// score equation S^I and the fp8_index docstring — ReLU of each head's logit,
// times the head weight, summed over the 64 heads, times the key scale).
//
// A thread owns one key (one TMEM lane) of an accumulator tile whose columns
// are the 64 heads of one query row.  It copies the row's 64 fp32 logits from
// TMEM into registers (load_logits), then reduces them (relu_head_sum).  Every kernel uses this one routine, so all of them
// produce the same fp32 score bit for bit: head pair p (heads 2p, 2p+1) goes
// into packed accumulator p mod 4 in increasing p with one packed FMA, then
// ((a0 + a1) + (a2 + a3)) with each ai the sum of its two lanes, then × scale.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace idx {

// The 64 logits of TMEM lane (lane_base's lane quadrant + this thread) at
// columns col … col+63, both halves in flight before one wait.
__device__ __forceinline__ void load_logits(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_ld32_nowait(taddr, r);
  tmem_ld32_nowait(taddr + 32, r + 32);
  tmem_wait();
  tmem_regs_ready(r);
  tmem_regs_ready(r + 32);
}

// Σ_h w_h · max(L_h, 0) · ks for the logits r[0..63]; weights in registers as
// packed pairs (wp[p] = {w_2p, w_2p+1}).
__device__ __forceinline__ float relu_head_sum(const uint32_t (&r)[64], const unsigned long long (&wp)[32],
                                               float ks) {
  unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int p = 0; p < 32; ++p)
    fma2(acc[p & 3], pack2(fmaxf(__uint_as_float(r[2 * p]), 0.f), fmaxf(__uint_as_float(r[2 * p + 1]), 0.f)), wp[p]);
  const float2 p0 = unpack2(acc[0]), p1 = unpack2(acc[1]), p2 = unpack2(acc[2]), p3 = unpack2(acc[3]);
  return (((p0.x + p0.y) + (p1.x + p1.y)) + ((p2.x + p2.y) + (p3.x + p3.y))) * ks;
}

// The same with the 64 weights read from shared memory (16-byte aligned),
// four at a time by broadcast loads.
__device__ __forceinline__ float relu_head_sum(const uint32_t (&r)[64], const float* w64, float ks) {
  unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
  const float4* wv = reinterpret_cast<const float4*>(w64);
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const float4 w4 = wv[q];
    fma2(acc[(2 * q) & 3],
         pack2(fmaxf(__uint_as_float(r[4 * q]), 0.f), fmaxf(__uint_as_float(r[4 * q + 1]), 0.f)), pack2(w4.x, w4.y));
    fma2(acc[(2 * q + 1) & 3],
         pack2(fmaxf(__uint_as_float(r[4 * q + 2]), 0.f), fmaxf(__uint_as_float(r[4 * q + 3]), 0.f)),
         pack2(w4.z, w4.w));
  }
  const float2 p0 = unpack2(acc[0]), p1 = unpack2(acc[1]), p2 = unpack2(acc[2]), p3 = unpack2(acc[3]);
  return (((p0.x + p0.y) + (p1.x + p1.y)) + ((p2.x + p2.y) + (p3.x + p3.y))) * ks;
}

}  // namespace idx
