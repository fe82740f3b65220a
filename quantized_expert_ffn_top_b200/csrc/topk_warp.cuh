// Top-k of one token's logits row by one warp, shared by the top-k kernels
// and the router kernels that pick in their epilogue.
//
// Selection is on the logits (softmax is monotone), the k largest in
// descending order with ties to the lower expert index; the k weights are
// the softmax over all E experts renormalised over the selected k, i.e.
// exp(L_j - L_0) / sum over the k picks.
#pragma once

#include <math.h>

#include "kernels.cuh"

namespace moe {

// Warp-wide maximum of a float (NaN inputs are never passed here: a row
// with a NaN is flagged before its picks are used) and minimum of a u32, one
// instruction each.
__device__ __forceinline__ float warp_max_f32(float v) {
  float m;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(v));
  return m;
}
__device__ __forceinline__ uint32_t warp_min_u32(uint32_t v) {
  uint32_t m;
  asm volatile("redux.sync.min.u32 %0, %1, 0xffffffff;" : "=r"(m) : "r"(v));
  return m;
}

// One warp picks the top k of one token's logits held in registers: J =
// ceil(E / 32) per lane, lane l holding logits l, l + 32, ... (entries at or
// past E are ignored).  Each round takes the largest not-yet-taken logit
// with a warp arg-max; lane 0 writes the index and exp(L - L_0); a final
// pass divides by the sum.  `bad` (any lane: a NaN was seen), or a row
// without a finite logit, raises the status word and writes indices 0..k-1
// with zero weights.
template <int J>
__device__ __forceinline__ void topk_select(const float (&v)[J], bool bad, int E, int k,
                                            int32_t* __restrict__ idx_row, float* __restrict__ w_row,
                                            int32_t* status) {
  const int lane = threadIdx.x & 31;
  uint32_t taken = 0u;
#pragma unroll
  for (int j = 0; j < J; ++j)
    if (lane + 32 * j >= E) taken |= 1u << j;
  float top = 0.0f, sum = 0.0f;
  bad = __any_sync(0xffffffffu, bad);
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int e = lane + 32 * j;
      if (!(taken & (1u << j)) && (v[j] > bv || (v[j] == bv && e < be))) {
        bv = v[j];
        be = e;
      }
    }
    // the warp's largest remaining logit, then the lowest expert holding it
    const float m = warp_max_f32(bv);
    const uint32_t bi = warp_min_u32((be != 0x7fffffff && bv == m) ? (uint32_t)be : 0xffffffffu);
    bv = m;
    be = bi == 0xffffffffu ? 0x7fffffff : (int)bi;
    if (be != 0x7fffffff && (be & 31) == lane) taken |= 1u << (be >> 5);
    if (r == 0) {
      top = bv;
      if (!(top > -INFINITY)) bad = true;
    }
    const float ex = expf(bv - top);
    sum += ex;
    if (lane == 0) {
      idx_row[r] = bad ? r : be;
      w_row[r] = bad ? 0.0f : ex;
    }
  }
  __syncwarp();
  if (bad) {
    if (lane == 0) raise_status(status, MOE_ERR_DEVICE_FAULT);
    return;
  }
  for (int r = lane; r < k; r += 32) w_row[r] = __fdiv_rn(w_row[r], sum);
}

// The same for a row in global memory that may arrive as nparts partial
// sums part_stride apart, added in part order; logits_out_row (nullable)
// receives the sums.  COHERENT: the row was written by other blocks of the
// running kernel, so it is read through L2 (ld.cg) rather than the
// read-only path.
template <int J, bool COHERENT>
__device__ __forceinline__ void topk_token(const float* __restrict__ L, int nparts, int64_t part_stride,
                                           float* __restrict__ logits_out_row, int E, int k,
                                           int32_t* __restrict__ idx_row, float* __restrict__ w_row,
                                           int32_t* status) {
  const int lane = threadIdx.x & 31;
  auto ld = [&](const float* p) { return COHERENT ? __ldcg(p) : __ldg(p); };
  float v[J];
  bool bad = false;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < E ? ld(L + e) : -INFINITY;
  }
  for (int p = 1; p < nparts; ++p) {
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int e = lane + 32 * j;
      if (e < E) v[j] += ld(L + p * part_stride + e);
    }
  }
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    if (e < E && isnan(v[j])) bad = true;
    if (e < E && logits_out_row) logits_out_row[e] = v[j];
  }
  topk_select<J>(v, bad, E, k, idx_row, w_row, status);
}

}  // namespace moe
