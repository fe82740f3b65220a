// One-time repack of a CANONICAL expert bank into the PREPARED device layout
// (the load-time weight layout step the FreeToken upstream README calls the
// FTW fast weight format, "About"):
//  * W13 rows interleaved, prepared row 2i = gate row i, 2i + 1 = up row i,
//    so a gate/up pair lands in neighbouring accumulator rows;
//  * scale factors in the blocked 128-row x 4-column layout
//    (sf_blocked_offset), the order the tensor-core scale copy expects.
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

}  // namespace moe
