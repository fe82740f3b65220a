// One-time repack of a CANONICAL expert bank into the PREPARED device layout
// (the load-time weight layout step the FreeToken upstream README calls the
// FTW fast weight format, "About"):
//  * W13 rows interleaved, prepared row 2i = gate row i, 2i + 1 = up row i,
//    so a gate/up pair lands in neighbouring accumulator rows;
//  * scale factors in the blocked 128-row x 4-column layout
//    (sf_blocked_offset), the order the tensor-core scale copy expects;
// and the load-time expansion of an FP4 / FP8 bank to bf16 (see below).
#include "kernels.cuh"

namespace moe {

__global__ void prepare_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int64_t E, int64_t R,
                                    int64_t row_bytes, bool interleave) {
  const int64_t vec = row_bytes / 16;
  const int64_t total = E * R * vec;
  const int64_t half = R / 2;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t v = i % vec;
    const int64_t r = (i / vec) % R;
    const int64_t e = i / (vec * R);
    const int64_t sr = interleave ? ((r & 1) ? half + (r >> 1) : (r >> 1)) : r;
    reinterpret_cast<uint4*>(dst)[i] = __ldg(reinterpret_cast<const uint4*>(src + (e * R + sr) * row_bytes) + v);
  }
}

__global__ void prepare_sf_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int64_t E, int64_t R,
                                  int64_t ncols, int64_t ncols_p, bool interleave) {
  const int64_t total = E * R * ncols_p;
  const int64_t half = R / 2;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % ncols_p;
    const int64_t r = (i / ncols_p) % R;
    const int64_t e = i / (ncols_p * R);
    const int64_t sr = interleave ? ((r & 1) ? half + (r >> 1) : (r >> 1)) : r;
    const uint8_t v = c < ncols ? __ldg(src + (e * R + sr) * ncols + c) : (uint8_t)0;
    dst[e * R * ncols_p + sf_blocked_offset(r, c, ncols_p)] = v;
  }
}

cudaError_t launch_prepare_rows(int fmt, const uint8_t* src, uint8_t* dst, int64_t E, int64_t R, int64_t row_bytes,
                                bool interleave, cudaStream_t s) {
  (void)fmt;
  const int64_t total = E * R * (row_bytes / 16);
  if (total == 0) return cudaSuccess;
  const int grid = (int)((total + 255) / 256 < 65535 ? (total + 255) / 256 : 65535);
  prepare_rows_kernel<<<grid, 256, 0, s>>>(src, dst, E, R, row_bytes, interleave);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_prepare_sf(const uint8_t* src, uint8_t* dst, int64_t E, int64_t R, int64_t ncols,
                              int64_t ncols_p, bool interleave, cudaStream_t s) {
  const int64_t total = E * R * ncols_p;
  if (total == 0) return cudaSuccess;
  const int grid = (int)((total + 255) / 256 < 65535 ? (total + 255) / 256 : 65535);
  prepare_sf_kernel<<<grid, 256, 0, s>>>(src, dst, E, R, ncols, ncols_p, interleave);
  count_launches(1);
  return cudaGetLastError();
}

// Dequantisation of a CANONICAL FP4 / FP8 expert tensor [E][R][K] to bf16,
// once at load time, for bf16-activation (W4A16 / W8A16) prefill on the bf16
// tensor cores: w = e2m1 * dec(e4m3) * g (NVFP4), e2m1 * 2^(c-127) (MXFP4),
// e4m3 * s (FP8), in fp32, then rounded to bf16 (nearest even).  The part
// scale of row r is gs[e * gstride + (r >= part_rows)] (gate / up parts of
// W13); gs NULL means 1.  One thread per 16 elements.
__global__ void dequant_bf16_kernel(int fmt, const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                    const float* __restrict__ gs, int gstride, int64_t part_rows, int64_t E,
                                    int64_t R, int64_t K, uint16_t* __restrict__ out) {
  const int64_t nb = K / 16;
  const int64_t total = E * R * nb;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c16 = i % nb;
    const int64_t row = i / nb;  // e * R + r
    const int64_t e = row / R, r = row % R;
    const float g = gs ? __ldg(gs + e * gstride + (r >= part_rows ? 1 : 0)) : 1.0f;
    float v[16];
    if (fmt == MOE_FMT_FP8) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(codes + row * K + c16 * 16));
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = e4m3_decode((ww[j / 4] >> (8 * (j % 4))) & 0xFFu) * g;
    } else {
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(codes + row * (K / 2) + c16 * 8));
      // e2m1 times the block scale is exact in fp32, so each weight is
      // rounded once, by the product with the global scale
      const float sc = fmt == MOE_FMT_NVFP4 ? e4m3_decode(__ldg(sf + row * nb + c16))
                                            : e8m0_decode(__ldg(sf + row * (K / 32) + c16 / 2));
      const float gg = fmt == MOE_FMT_NVFP4 ? g : 1.0f;
      const uint32_t ww[2] = {w.x, w.y};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 p = e2m1x2_decode((ww[j / 4] >> (8 * (j % 4))) & 0xFFu);
        v[2 * j] = (p.x * sc) * gg;
        v[2 * j + 1] = (p.y * sc) * gg;
      }
    }
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = (uint32_t)f32_to_bf16_rn(v[2 * j]) | ((uint32_t)f32_to_bf16_rn(v[2 * j + 1]) << 16);
    uint4* dst = reinterpret_cast<uint4*>(out + row * K + c16 * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

cudaError_t launch_dequant_bf16(int fmt, const uint8_t* codes, const uint8_t* sf, const float* gs, int gstride,
                                int64_t part_rows, int64_t E, int64_t R, int64_t K, uint16_t* out, cudaStream_t s) {
  const int64_t total = E * R * (K / 16);
  if (total == 0) return cudaSuccess;
  const int grid = (int)((total + 255) / 256 < 65535 ? (total + 255) / 256 : 65535);
  dequant_bf16_kernel<<<grid, 256, 0, s>>>(fmt, codes, sf, gs, gstride, part_rows, E, R, K, out);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace moe
