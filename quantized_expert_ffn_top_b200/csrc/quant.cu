// Tensor amax and the canonical-layout block quantisers (moe_quantize), plus
// the fused quantise-and-dequantise of activation rows used by the GEMV path.
//
// The quantisation rules are those of the expert-weight formats the FreeToken
// upstream README names ("About": MXFP4, NVFP4, FP8, BF16) applied to activations
// for the W4A4 / W8A8 schemes (FreeToken commit 58f4b9ec0e: per-tensor FP8
// with a dynamic activation scale).  One thread owns one scale block, so the
// block maximum is a private loop and the codes of a block leave as one
// vector store.
#include "kernels.cuh"

namespace moe {

// ------------------------------------------------------------------ amax --
template <typename In>
__global__ void __launch_bounds__(256) amax_kernel(const In* __restrict__ x, int64_t n, float* __restrict__ out) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  float m = 0.0f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) m = fmaxf(m, fabsf(load_f32(x + i)));
  m = warp_max(m);
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
    m = warp_max(m);
    if (threadIdx.x == 0) atomic_max_nonneg(out, m);
  }
}

cudaError_t launch_amax(const void* x, int x_dtype, int64_t n, float* out, int num_sms, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float), s);
  if (e != cudaSuccess || n == 0) return e;
  int64_t blocks = (n + 255) / 256;
  int grid = (int)(blocks < (int64_t)num_sms * 8 ? blocks : (int64_t)num_sms * 8);
  if (x_dtype == 0)
    e = launch_pdl(amax_kernel<float>, dim3(grid), dim3(256), 0, s, static_cast<const float*>(x), n, out);
  else
    e = launch_pdl(amax_kernel<uint16_t>, dim3(grid), dim3(256), 0, s, static_cast<const uint16_t*>(x), n, out);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------- canonical quantisers --
// Tensor scale: the given one, or the one derived from the amax buffer.
__device__ __forceinline__ float resolve_scale(int fmt, const float* scale_in, const float* amax) {
  if (scale_in) return __ldg(scale_in);
  const float a = *amax;
  return fmt == MOE_FMT_NVFP4 ? nvfp4_tensor_scale(a) : fp8_tensor_scale(a);
}

template <typename In>
__global__ void __launch_bounds__(256) quantize_kernel(int fmt, const In* __restrict__ x, int64_t rows, int64_t K,
                                                       const float* __restrict__ scale_in, const float* amax,
                                                       uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                       float* __restrict__ scale_out) {
  const int bs = fmt == MOE_FMT_MXFP4 ? 32 : 16;
  const int64_t nblk = rows * (K / bs);
  const float scale = (fmt == MOE_FMT_MXFP4 || fmt == MOE_FMT_BF16) ? 1.0f : resolve_scale(fmt, scale_in, amax);
  if (scale_out && blockIdx.x == 0 && threadIdx.x == 0) *scale_out = scale;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
    const In* src = x + b * bs;
    float v[32];
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i < bs) {
        v[i] = load_f32(src + i);
        bmax = fmaxf(bmax, fabsf(v[i]));
      }
    }
    if (fmt == MOE_FMT_NVFP4) {
      uint32_t sc;
      float r;
      nvfp4_block_scale(bmax, scale, sc, r);
      *reinterpret_cast<uint2*>(codes + b * 8) = nvfp4_encode16(v, r);
      sf[b] = (uint8_t)sc;
    } else if (fmt == MOE_FMT_MXFP4) {
      uint32_t c;
      float inv;
      mxfp4_block_scale(bmax, c, inv);
      uint4 w;
      w.x = e2m1_encode8(v, inv);
      w.y = e2m1_encode8(v + 8, inv);
      w.z = e2m1_encode8(v + 16, inv);
      w.w = e2m1_encode8(v + 24, inv);
      *reinterpret_cast<uint4*>(codes + b * 16) = w;
      sf[b] = (uint8_t)c;
    } else if (fmt == MOE_FMT_BF16) {
      // bf16: round to nearest even, 16 values = 32 bytes
      uint32_t p[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        p[i] = (uint32_t)f32_to_bf16_rn(v[2 * i]) | ((uint32_t)f32_to_bf16_rn(v[2 * i + 1]) << 16);
      uint4* dst = reinterpret_cast<uint4*>(codes + b * 32);
      dst[0] = make_uint4(p[0], p[1], p[2], p[3]);
      dst[1] = make_uint4(p[4], p[5], p[6], p[7]);
    } else {
      const float inv = __frcp_rn(scale);
      uint4 w;
      uint32_t* pw = &w.x;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        pw[i] = e4m3x2_encode(__fmul_rn(v[4 * i], inv), __fmul_rn(v[4 * i + 1], inv)) |
                (e4m3x2_encode(__fmul_rn(v[4 * i + 2], inv), __fmul_rn(v[4 * i + 3], inv)) << 16);
      *reinterpret_cast<uint4*>(codes + b * 16) = w;
    }
  }
}

cudaError_t launch_quantize(int fmt, const void* x, int x_dtype, int64_t rows, int64_t K, const float* scale_in,
                            const float* amax, uint8_t* codes, uint8_t* sf, float* scale_out, int num_sms,
                            cudaStream_t s) {
  const int bs = fmt == MOE_FMT_MXFP4 ? 32 : 16;
  const int64_t nblk = rows * (K / bs);
  if (nblk == 0) return cudaSuccess;
  int64_t blocks = (nblk + 255) / 256;
  int grid = (int)(blocks < (int64_t)num_sms * 16 ? blocks : (int64_t)num_sms * 16);
  if (x_dtype == 0)
    quantize_kernel<float><<<grid, 256, 0, s>>>(fmt, static_cast<const float*>(x), rows, K, scale_in, amax, codes,
                                                sf, scale_out);
  else
    quantize_kernel<uint16_t><<<grid, 256, 0, s>>>(fmt, static_cast<const uint16_t*>(x), rows, K, scale_in, amax,
                                                   codes, sf, scale_out);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace moe
