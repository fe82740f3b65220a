// Weighted un-permute combine: out[t] = sum_{j<k} w[t,j] * y_perm[inv_perm[t*k+j]]
// (+ shared_y[t]), accumulated in fp32 in the order j = 0..k-1 and rounded
// once to bf16.  The always-on shared expert enters with weight 1.0 (the
// shared expert of the Domir6/FreeToken fork README, "Changes in this fork").
// Grid: token x 512-column stretch, 64 threads of 8 columns (16-byte loads)
// each.  The token's k slot indices and weights are staged in shared memory
// first, so every thread then issues its k row loads four at a time.
#include "kernels.cuh"

namespace moe {

constexpr int kCombineThreads = 64;
constexpr int kCombineCols = kCombineThreads * 8;
constexpr int kCombineMaxK = 1024;  // k <= E <= 1024

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const uint16_t* __restrict__ y_perm,
                                                                  const int32_t* __restrict__ inv_perm,
                                                                  const float* __restrict__ w, int64_t T, int k,
                                                                  int H, const uint16_t* __restrict__ shared_y,
                                                                  uint16_t* __restrict__ out, int32_t* status) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  __shared__ int32_t sp[kCombineMaxK];
  __shared__ float sw[kCombineMaxK];
  const int64_t t = blockIdx.x;
  const int64_t S = T * k;
  for (int j = threadIdx.x; j < k; j += kCombineThreads) {
    int32_t p = __ldg(inv_perm + t * k + j);
    if (p >= S) {
      if (blockIdx.y == 0) raise_status(status, MOE_ERR_DEVICE_FAULT);
      p = -1;
    }
    sp[j] = p;
    sw[j] = __ldg(w + t * k + j);
  }
  __syncthreads();
  const int c = blockIdx.y * kCombineCols + threadIdx.x * 8;
  if (c >= H) return;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  auto add = [&](const uint4& v, float wj) {
    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(wj, __uint_as_float(vv[i] << 16), acc[2 * i]);
      acc[2 * i + 1] = fmaf(wj, __uint_as_float(vv[i] & 0xFFFF0000u), acc[2 * i + 1]);
    }
  };
  int j = 0;
  for (; j + 4 <= k; j += 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int32_t p = sp[j + u];
      v[u] = p >= 0 ? __ldg(reinterpret_cast<const uint4*>(y_perm + (int64_t)p * H + c)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (sp[j + u] >= 0) add(v[u], sw[j + u]);
  }
  for (; j < k; ++j) {
    const int32_t p = sp[j];
    if (p >= 0) add(__ldg(reinterpret_cast<const uint4*>(y_perm + (int64_t)p * H + c)), sw[j]);
  }
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
  const dim3 grid((unsigned)T, (unsigned)((H + kCombineCols - 1) / kCombineCols));
  cudaError_t e = launch_pdl(combine_kernel, grid, dim3(kCombineThreads), 0, s, y_perm, inv_perm, w, T, k, H, shared_y,
                             out, status);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe
