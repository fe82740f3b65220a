// Weighted un-permute combine: out[t] = sum_{j<k} w[t,j] * y_perm[inv_perm[t*k+j]]
// (+ shared_y[t]), accumulated in fp32 in the order j = 0..k-1 and rounded
// once to bf16.  The always-on shared expert enters with weight 1.0 (the
// shared expert of the Domir6/FreeToken fork README, "Changes in this fork").
// Grid: token x stretch of 8 * blockDim.x columns; each thread owns 8
// columns (16-byte loads).  Every warp reads the token's slot indices and
// weights itself, 32 at a time into lane registers, and broadcasts them with
// shuffles, so no shared memory or block barrier is involved; a thread then
// issues up to eight row loads at once.
#include "kernels.cuh"

namespace moe {

constexpr int kCombineThreads = 256;
constexpr int kCombineMaxK = 1024;  // k <= E <= 1024

__global__ void __launch_bounds__(kCombineThreads, 4) combine_kernel(const uint16_t* __restrict__ y_perm,
                                                                  const int32_t* __restrict__ inv_perm,
                                                                  const float* __restrict__ w, int64_t T, int k,
                                                                  int H, const uint16_t* __restrict__ shared_y,
                                                                  uint16_t* __restrict__ out, int32_t* status) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  const int64_t t = blockIdx.x;
  const int64_t S = T * k;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.y * (blockDim.x * 8) + threadIdx.x * 8;
  const bool active = c < H;  // every lane takes part in the shuffles
  // an earlier kernel of the call gave up on a bounded wait: its outputs
  // are unspecified, so the layer's output is written as zeros
  if (status && __ldcg(status) == MOE_ERR_TIMEOUT) {
    if (active) *reinterpret_cast<uint4*>(out + t * H + c) = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  auto add = [&](const uint4& v, float wj) {
    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(wj, __uint_as_float(vv[i] << 16), acc[2 * i]);
      acc[2 * i + 1] = fmaf(wj, __uint_as_float(vv[i] & 0xFFFF0000u), acc[2 * i + 1]);
    }
  };
  for (int j0 = 0; j0 < k; j0 += 32) {
    const int nj = min(32, k - j0);
    int32_t pl = -1;
    float wl = 0.0f;
    if (lane < nj) {
      pl = __ldg(inv_perm + t * k + j0 + lane);
      wl = __ldg(w + t * k + j0 + lane);
      if (pl >= S) {
        if (blockIdx.y == 0 && threadIdx.x < 32) raise_status(status, MOE_ERR_DEVICE_FAULT);
        pl = -1;
      }
    }
    // slots j0 .. j0 + nj - 1, eight loads in flight, summed in slot order
    for (int jb = 0; jb < nj; jb += 8) {
      uint4 v[8];
      int32_t pj[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        pj[u] = __shfl_sync(0xffffffffu, pl, (jb + u) & 31);
        if (jb + u >= nj) pj[u] = -1;
        v[u] = (active && pj[u] >= 0) ? __ldcs(reinterpret_cast<const uint4*>(y_perm + (int64_t)pj[u] * H + c))
                                      : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float wj = __shfl_sync(0xffffffffu, wl, (jb + u) & 31);
        if (pj[u] >= 0) add(v[u], wj);
      }
    }
  }
  if (!active) return;
  if (shared_y) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(shared_y + t * H + c));
    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += __uint_as_float(vv[i] << 16);
      acc[2 * i + 1] += __uint_as_float(vv[i] & 0xFFFF0000u);
    }
  }
  uint4 o;
  uint32_t* po = &o.x;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    po[i] = (uint32_t)f32_to_bf16_rn(acc[2 * i]) | ((uint32_t)f32_to_bf16_rn(acc[2 * i + 1]) << 16);
  *reinterpret_cast<uint4*>(out + t * H + c) = o;
}

cudaError_t launch_combine(const uint16_t* y_perm, const int32_t* inv_perm, const float* w, int64_t T, int k, int H,
                           const uint16_t* shared_y, uint16_t* out, int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (k > kCombineMaxK) return cudaErrorInvalidValue;
  // narrower blocks for small H, so no warp is idle
  const int threads = min(kCombineThreads, ((H / 8) + 31) / 32 * 32);
  const dim3 grid((unsigned)T, (unsigned)((H + threads * 8 - 1) / (threads * 8)));
  cudaError_t e = launch_pdl(combine_kernel, grid, dim3(threads), 0, s, y_perm, inv_perm, w, T, k, H, shared_y, out,
                             status);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// The last step of a forward whose down projection added w * y into fp32
// rows (the combine in the down epilogue): out = bf16(out32), round to
// nearest even, eight values a thread.
__global__ void __launch_bounds__(256) round_rows_kernel(const float* __restrict__ out32, int64_t n8,
                                                         uint16_t* __restrict__ out, const int32_t* status) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();
  if (status && __ldcg(status) == MOE_ERR_TIMEOUT) {   // as in combine_kernel: zeros after a timeout
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x)
      reinterpret_cast<uint4*>(out)[i] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(out32) + 2 * i);
    const float4 b = __ldcs(reinterpret_cast<const float4*>(out32) + 2 * i + 1);
    uint4 o;
    o.x = (uint32_t)f32_to_bf16_rn(a.x) | ((uint32_t)f32_to_bf16_rn(a.y) << 16);
    o.y = (uint32_t)f32_to_bf16_rn(a.z) | ((uint32_t)f32_to_bf16_rn(a.w) << 16);
    o.z = (uint32_t)f32_to_bf16_rn(b.x) | ((uint32_t)f32_to_bf16_rn(b.y) << 16);
    o.w = (uint32_t)f32_to_bf16_rn(b.z) | ((uint32_t)f32_to_bf16_rn(b.w) << 16);
    reinterpret_cast<uint4*>(out)[i] = o;
  }
}

cudaError_t launch_round_rows(const float* out32, int64_t n, uint16_t* out, const int32_t* status, int num_sms,
                              cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (n % 8 != 0) return cudaErrorInvalidValue;
  const int64_t n8 = n / 8;
  const int64_t blocks = (n8 + 255) / 256;
  const int grid = (int)(blocks < (int64_t)num_sms * 8 ? blocks : (int64_t)num_sms * 8);
  cudaError_t e = launch_pdl(round_rows_kernel, dim3(grid), dim3(256), 0, s, out32, n8, out, status);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe
