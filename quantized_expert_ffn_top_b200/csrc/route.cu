// Router: logits = x Wr^T (+ b) and top-k with renormalisation.
//
// The routed MoE layer picks k experts per token from a learned router (the
// MoE models the FreeToken upstream README lists under "About"; the router is
// also what the Domir6/FreeToken fork's "router lookahead" measures, "Changes
// in this fork").  Selection is on the logits -- softmax is monotone -- with
// ties to the lower expert index; the k weights are the softmax over all E
// experts renormalised over the selected k, i.e. exp(L_j - L_0) / sum.
#include <math.h>

#include "kernels.cuh"
#include "token_quant.cuh"
#include "topk_warp.cuh"

namespace moe {

// ------------------------------------------------------------ logits ------
// Small T (decode): one block of 8 warps per (expert, group of up to 8
// tokens).  Each thread takes 8 consecutive columns of every 2048-column
// stretch of H with 16-byte loads of the Wr row and the token rows, so the
// block issues all its loads at once; warp sums, then the 8 warps' partial
// sums are added in shared memory.
constexpr int kSmallTGroup = 8;
constexpr int kSmallThreads = 256;

// The logits of expert `e` for tokens t0 .. t0 + nt - 1 (nt <= 8), by one
// block of kSmallThreads threads, in the fixed order the header documents:
// thread p adds the 8 columns from 8p, then those 2048 further on, ...; the
// 32 threads of a warp are combined by an xor exchange; the 8 warp sums are
// added in order; then the bias.
__device__ __forceinline__ void small_logits_block(const uint16_t* __restrict__ x, int H,
                                                   const uint16_t* __restrict__ wr, const float* __restrict__ bias,
                                                   int E, int e, int64_t t0, int nt, float* __restrict__ logits,
                                                   float (*part)[kSmallTGroup]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[kSmallTGroup];
#pragma unroll
  for (int i = 0; i < kSmallTGroup; ++i) acc[i] = 0.0f;
  const uint16_t* wrow = wr + (int64_t)e * H;
  for (int h = threadIdx.x * 8; h < H; h += kSmallThreads * 8) {
    const uint4 wv = __ldg(reinterpret_cast<const uint4*>(wrow + h));
    uint4 xv[kSmallTGroup];
#pragma unroll
    for (int i = 0; i < kSmallTGroup; ++i)
      xv[i] = i < nt ? __ldg(reinterpret_cast<const uint4*>(x + (t0 + i) * H + h)) : make_uint4(0, 0, 0, 0);
    const uint32_t wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < kSmallTGroup; ++i) {
      const uint32_t xa[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[i] = fmaf(__uint_as_float(xa[q] << 16), __uint_as_float(wa[q] << 16), acc[i]);
        acc[i] = fmaf(__uint_as_float(xa[q] & 0xFFFF0000u), __uint_as_float(wa[q] & 0xFFFF0000u), acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kSmallTGroup; ++i) {
    const float v = warp_sum(acc[i]);
    if (lane == 0) part[warp][i] = v;
  }
  __syncthreads();
  if (threadIdx.x < nt) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kSmallThreads / 32; ++w) v += part[w][threadIdx.x];
    logits[(t0 + threadIdx.x) * E + e] = v + (bias ? __ldg(bias + e) : 0.0f);
  }
}

__global__ void __launch_bounds__(kSmallThreads) router_logits_small_kernel(const uint16_t* __restrict__ x, int64_t T,
                                                                           int H, const uint16_t* __restrict__ wr,
                                                                           const float* __restrict__ bias, int E,
                                                                           float* __restrict__ logits) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  __shared__ float part[kSmallThreads / 32][kSmallTGroup];
  const int64_t t0 = (int64_t)blockIdx.y * kSmallTGroup;
  const int nt = (int)((T - t0) < kSmallTGroup ? (T - t0) : kSmallTGroup);
  small_logits_block(x, H, wr, bias, E, blockIdx.x, t0, nt, logits, part);
}

// Larger T: 64 tokens x 64 experts per block, K in chunks of 32 staged in
// shared memory, 4 x 4 outputs per thread on the CUDA cores.
__global__ void __launch_bounds__(256) router_logits_tiled_kernel(const uint16_t* __restrict__ x, int64_t T, int H,
                                                                  const uint16_t* __restrict__ wr,
                                                                  const float* __restrict__ bias, int E,
                                                                  float* __restrict__ logits) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  __shared__ float xs[32][65];
  __shared__ float ws[32][65];
  const int tid = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * 64;
  const int e0 = blockIdx.y * 64;
  const int tr = tid / 16, tc = tid % 16;  // 16 x 16 threads, 4 x 4 each
  float acc[4][4] = {};
  for (int h0 = 0; h0 < H; h0 += 32) {
    // 64 rows x 32 columns of x and of Wr: 2048 values each, 8 per thread
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int idx = tid + i * 256;
      const int r = idx / 32, c = idx % 32;
      const int64_t t = t0 + r;
      const int e = e0 + r;
      const bool hin = h0 + c < H;
      xs[c][r] = (t < T && hin) ? bf16_to_f32(__ldg(x + t * H + h0 + c)) : 0.0f;
      ws[c][r] = (e < E && hin) ? bf16_to_f32(__ldg(wr + (int64_t)e * H + h0 + c)) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = xs[c][tr * 4 + i];
        b[i] = ws[c][tc * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + tr * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tc * 4 + j;
      if (e < E) logits[t * E + e] = acc[i][j] + (bias ? __ldg(bias + e) : 0.0f);
    }
  }
}

cudaError_t launch_router_logits(const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias, int E,
                                 float* logits, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (T <= 64 && H % 8 == 0) {
    dim3 grid((unsigned)E, (unsigned)((T + kSmallTGroup - 1) / kSmallTGroup));
    cudaError_t e = launch_pdl(router_logits_small_kernel, grid, dim3(kSmallThreads), 0, s, x, T, H, wr, bias, E, logits);
    if (e != cudaSuccess) return e;
  } else {
    dim3 grid((unsigned)((T + 63) / 64), (E + 63) / 64);
    cudaError_t e = launch_pdl(router_logits_tiled_kernel, grid, dim3(256), 0, s, x, T, H, wr, bias, E, logits);
    if (e != cudaSuccess) return e;
  }
  count_launches(1);
  return cudaGetLastError();
}

// -------------------------------------------------------------- top-k -----
// One warp per token; lane l holds logits l, l+32, ... in registers.  Each
// round picks the largest not-yet-taken logit (ties -> lower index) with a
// warp arg-max; lane 0 writes the index and exp(L - L_0); a final pass divides
// by the sum.  A NaN, or a row without a finite logit, raises the status word
// and writes indices 0..k-1 with zero weights.
// The logits may arrive as nparts partial sums (a router GEMM split along
// H), added here in part order; logits_out (nullable) receives the sums.
template <int J>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int nparts, int64_t part_stride,
                                                   float* __restrict__ logits_out, int64_t T, int E, int k,
                                                   int32_t* __restrict__ idx, float* __restrict__ w,
                                                   int32_t* status) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  topk_token<J, false>(logits + t * E, nparts, part_stride, logits_out ? logits_out + t * E : nullptr, E, k,
                       idx + t * k, w + t * k, status);
}

// The first kernel of the one-kernel forward at small batches (T <= 32):
// the logits exactly as router_logits_small_kernel computes them (the same
// fixed summation order), block (0, g) also quantises its token group into
// the gather layout (quant_token_gather), and the block that finishes last
// -- one ticket, reset by that block -- picks every token's top k.
template <int QFMT, int J>
__global__ void __launch_bounds__(kSmallThreads) router_decode_kernel(const uint16_t* __restrict__ x, int64_t T,
                                                                     int H, const uint16_t* __restrict__ wr,
                                                                     const float* __restrict__ bias, int E, int k,
                                                                     float* __restrict__ logits,
                                                                     int32_t* __restrict__ idx, float* __restrict__ w,
                                                                     int32_t* ticket, GatherQuant q,
                                                                     int32_t* status) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  __shared__ float part[kSmallThreads / 32][kSmallTGroup];
  __shared__ float r_tab[128];
  __shared__ int is_last;
  const int warp = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.y * kSmallTGroup;
  const int nt = (int)((T - t0) < kSmallTGroup ? (T - t0) : kSmallTGroup);
  small_logits_block(x, H, wr, bias, E, blockIdx.x, t0, nt, logits, part);
  if (blockIdx.x == 0) {
    constexpr int bs = QFMT == MOE_FMT_MXFP4 ? 32 : 16;
    const float scale = act_scale_of(QFMT, q.scale, q.amax);
    if (QFMT == MOE_FMT_NVFP4 && threadIdx.x < 128) r_tab[threadIdx.x] = nvfp4_multiplier(threadIdx.x, scale);
    __syncthreads();
    if (warp < nt) {
      const int64_t t = t0 + warp;
      quant_token_gather<QFMT>(x + t * H, H, scale, r_tab, q.xg + t * 8 * (H / 2), q.xsl + t * (H / (4 * bs)) * 16);
    }
  }
  // the block that finishes last picks the top k of every token
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(ticket, 1) == (int)(gridDim.x * gridDim.y) - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int64_t t = warp; t < T; t += kSmallThreads / 32)
    topk_token<J, true>(logits + t * E, 1, 0, nullptr, E, k, idx + t * k, w + t * k, status);
  if (threadIdx.x == 0) *ticket = 0;
}

cudaError_t launch_router_decode(int fmt, const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias,
                                 int E, int k, float* logits, int32_t* idx, float* w, int32_t* ticket,
                                 const GatherQuant& q, int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (T > kGatherMaxT || H % 256 != 0 || E > 256) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)E, (unsigned)((T + kSmallTGroup - 1) / kSmallTGroup));
  const int J = (E + 31) / 32;
  cudaError_t e = cudaErrorInvalidValue;
#define MOE_RD(F, JJ) \
  e = launch_pdl(router_decode_kernel<F, JJ>, grid, dim3(kSmallThreads), 0, s, x, T, H, wr, bias, E, k, logits, idx, w, \
                 ticket, q, status)
#define MOE_RD_J(F) \
  if (J <= 1) MOE_RD(F, 1); else if (J <= 2) MOE_RD(F, 2); else if (J <= 4) MOE_RD(F, 4); else MOE_RD(F, 8);
  if (fmt == MOE_FMT_NVFP4) {
    MOE_RD_J(MOE_FMT_NVFP4)
  } else if (fmt == MOE_FMT_MXFP4) {
    MOE_RD_J(MOE_FMT_MXFP4)
  } else {
    return cudaErrorInvalidValue;
  }
#undef MOE_RD_J
#undef MOE_RD
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int nparts, int64_t part_stride, float* logits_out, int64_t T, int E,
                        int k, int32_t* idx, float* w, int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((T + 7) / 8);
  const int J = (E + 31) / 32;
  cudaError_t e = cudaSuccess;
#define MOE_TOPK(JJ) \
  e = launch_pdl(topk_kernel<JJ>, dim3(grid), dim3(256), 0, s, logits, nparts, part_stride, logits_out, T, E, k, idx, w, status)
  if (J <= 1) MOE_TOPK(1);
  else if (J <= 2) MOE_TOPK(2);
  else if (J <= 4) MOE_TOPK(4);
  else if (J <= 8) MOE_TOPK(8);
  else if (J <= 16) MOE_TOPK(16);
  else MOE_TOPK(32);
#undef MOE_TOPK
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace moe
