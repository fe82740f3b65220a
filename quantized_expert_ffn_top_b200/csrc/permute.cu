// Token-to-expert histogram, offsets and stable permutation of the T*k slots,
// without global atomics.
//
// The permuted order is the expert-major "slot pool" of the
// atomicmilkshake/FreeToken fork README ("Known limits"): every expert's slots
// form one contiguous segment, so the grouped FFN reads each expert's weights
// for a dense block of rows.  Slots keep their flat order i = t*k + j inside a
// segment (stable), which makes the permutation unique and bit-comparable.
//
// Three passes over chunks of kChunk slots (8 warps x 256):
//   1. per chunk and expert, the count (warp-private counters fed by
//      __match_any_sync, one writer lane per expert and step);
//   2. one block: per expert the exclusive prefix over chunks, the totals, and
//      the exclusive prefix over experts -> offsets;
//   3. per chunk again: each warp's base = chunk base + earlier warps'
//      counts, and each slot's rank among equal experts earlier in its warp
//      step -> perm_token[p] = t, inv_perm[i] = p.
#include <mutex>

#include "kernels.cuh"

namespace moe {

constexpr int kPermWarps = 8;
constexpr int kSlotsPerWarp = 256;
constexpr int kChunk = kPermWarps * kSlotsPerWarp;

int permute_chunk_slots() { return kChunk; }

// Reads the expert of slot i, or -1 past the end / for an invalid index.
__device__ __forceinline__ int slot_expert(const int32_t* idx, int64_t S, int64_t i, int E, int32_t* status) {
  if (i >= S) return -1;
  const int e = __ldg(idx + i);
  if (e < 0 || e >= E) {
    raise_status(status, MOE_ERR_DEVICE_FAULT);
    return -1;
  }
  return e;
}

// Counts of each warp's 256-slot range into cnt[warp][e] (smem).
__device__ __forceinline__ void warp_counts(const int32_t* idx, int64_t S, int64_t base, int E, int32_t* cnt,
                                            int32_t* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* my = cnt + warp * E;
  for (int st = 0; st < kSlotsPerWarp / 32; ++st) {
    const int64_t i = base + (int64_t)warp * kSlotsPerWarp + st * 32 + lane;
    const int e = slot_expert(idx, S, i, E, status);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    if (e >= 0 && lane == leader) my[e] += __popc(peers);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kPermWarps * 32) perm_count_kernel(const int32_t* __restrict__ idx, int64_t S,
                                                                     int E, int32_t* __restrict__ chunk_counts,
                                                                     int32_t* status) {
  extern __shared__ int32_t cnt[];  // [kPermWarps][E]
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  warp_counts(idx, S, base, E, cnt, status);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t s = 0;
#pragma unroll
    for (int w = 0; w < kPermWarps; ++w) s += cnt[w * E + e];
    chunk_counts[(int64_t)blockIdx.x * E + e] = s;
  }
}

// One block of 1024 threads.  Turns chunk_counts[c][e] into the absolute base
// position of chunk c's first slot of expert e, and writes offsets[0..E].
__global__ void __launch_bounds__(1024) perm_scan_kernel(int32_t* __restrict__ chunk_counts, int nchunks, int E,
                                                         int32_t* __restrict__ offsets) {
  __shared__ int32_t tot[1024];
  __shared__ int32_t warp_tot[32];
  const int e = threadIdx.x;
  int32_t run = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {
      const int32_t v = chunk_counts[(int64_t)c * E + e];
      chunk_counts[(int64_t)c * E + e] = run;
      run += v;
    }
  }
  // exclusive scan of the totals over experts
  const int lane = e & 31, warp = e >> 5;
  int32_t incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t v = warp_tot[lane];
    int32_t vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += n;
    }
    warp_tot[lane] = vi - v;
  }
  __syncthreads();
  const int32_t excl = incl - run + warp_tot[warp];
  tot[e] = excl;
  if (e < E) offsets[e] = excl;
  if (e == E - 1) offsets[E] = excl + run;
  __syncthreads();
  if (e < E)
    for (int c = 0; c < nchunks; ++c) chunk_counts[(int64_t)c * E + e] += tot[e];
}

__global__ void __launch_bounds__(kPermWarps * 32) perm_scatter_kernel(const int32_t* __restrict__ idx, int64_t S,
                                                                       int k, int E,
                                                                       const int32_t* __restrict__ chunk_base,
                                                                       int32_t* __restrict__ perm_token,
                                                                       int32_t* __restrict__ inv_perm) {
  extern __shared__ int32_t cnt[];  // [kPermWarps][E]
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  warp_counts(idx, S, base, E, cnt, nullptr);
  __syncthreads();
  // exclusive prefix over warps per expert, offset by the chunk's base
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = chunk_base[(int64_t)blockIdx.x * E + e];
#pragma unroll
    for (int w = 0; w < kPermWarps; ++w) {
      const int32_t v = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* my = cnt + warp * E;
  for (int st = 0; st < kSlotsPerWarp / 32; ++st) {
    const int64_t i = base + (int64_t)warp * kSlotsPerWarp + st * 32 + lane;
    const int e = slot_expert(idx, S, i, E, nullptr);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    if (e >= 0) {
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int32_t p = my[e] + rank;
      perm_token[p] = (int32_t)(i / k);
      inv_perm[i] = p;
    } else if (i < S) {
      inv_perm[i] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == leader) my[e] += __popc(peers);
    __syncwarp();
  }
}

// Small batches (decode): the same three passes inside one block of 32
// warps, each warp owning a contiguous range of ceil(S/32) slots; the
// per-warp expert counters live in shared memory.  One launch instead of three.
constexpr int kSmallWarps = 32;
constexpr int64_t kSmallMaxS = 8192;

__global__ void __launch_bounds__(kSmallWarps * 32) perm_small_kernel(const int32_t* __restrict__ idx, int64_t S,
                                                                     int k, int E, int32_t* __restrict__ offsets,
                                                                     int32_t* __restrict__ perm_token,
                                                                     int32_t* __restrict__ inv_perm,
                                                                     int32_t* status) {
  extern __shared__ int32_t cnt[];  // [kSmallWarps][E], then [E] totals
  int32_t* tot = cnt + kSmallWarps * E;
  __shared__ int32_t warp_tot[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t per = ((S + kSmallWarps - 1) / kSmallWarps + 31) / 32 * 32;  // slots per warp, multiple of 32
  for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  int32_t* my = cnt + warp * E;
  const int64_t lo = warp * per, hi = min(S, lo + per);
  for (int64_t base = lo; base < hi; base += 32) {
    const int64_t i = base + lane;
    const int e = (i < hi) ? slot_expert(idx, S, i, E, status) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per expert: exclusive prefix over warps, total
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0;
    for (int w = 0; w < kSmallWarps; ++w) {
      const int32_t v = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += v;
    }
    tot[e] = run;
  }
  __syncthreads();
  // exclusive scan of the totals over experts (E <= 1024 = blockDim)
  const int e = threadIdx.x;
  const int32_t v = e < E ? tot[e] : 0;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int32_t wv = warp_tot[lane];
    int32_t wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_tot[lane] = wi - wv;
  }
  __syncthreads();
  const int32_t excl = incl - v + warp_tot[warp];
  __syncthreads();
  if (e < E) {
    tot[e] = excl;
    offsets[e] = excl;
  }
  if (e == E - 1) offsets[E] = excl + v;
  __syncthreads();
  for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) cnt[i] += tot[i % E];
  __syncthreads();
  for (int64_t base = lo; base < hi; base += 32) {
    const int64_t i = base + lane;
    const int ee = (i < hi) ? slot_expert(idx, S, i, E, nullptr) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, ee);
    if (ee >= 0) {
      const int32_t p = my[ee] + __popc(peers & ((1u << lane) - 1u));
      perm_token[p] = (int32_t)(i / k);
      inv_perm[i] = p;
    } else if (i < hi) {
      inv_perm[i] = -1;
    }
    __syncwarp();
    if (ee >= 0 && lane == __ffs(peers) - 1) my[ee] += __popc(peers);
    __syncwarp();
  }
}

cudaError_t launch_permute(const int32_t* idx, int64_t S, int k, int E, int32_t* offsets, int32_t* perm_token,
                           int32_t* inv_perm, PermuteScratch scratch, int32_t* status, cudaStream_t s) {
  const size_t small_smem = sizeof(int32_t) * (size_t)(kSmallWarps + 1) * E;
  if (S > 0 && S <= kSmallMaxS && small_smem <= 48 * 1024) {
    perm_small_kernel<<<1, kSmallWarps * 32, small_smem, s>>>(idx, S, k, E, offsets, perm_token, inv_perm, status);
    count_launches(1);
    return cudaGetLastError();
  }
  const int nchunks = (int)((S + kChunk - 1) / kChunk);
  if (nchunks == 0) {
    // no slots: offsets are all zero
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
  }
  const size_t smem = sizeof(int32_t) * kPermWarps * E;
  perm_count_kernel<<<nchunks, kPermWarps * 32, smem, s>>>(idx, S, E, scratch.chunk_counts, status);
  perm_scan_kernel<<<1, 1024, 0, s>>>(scratch.chunk_counts, nchunks, E, offsets);
  perm_scatter_kernel<<<nchunks, kPermWarps * 32, smem, s>>>(idx, S, k, E, scratch.chunk_counts, perm_token,
                                                              inv_perm);
  count_launches(3);
  return cudaGetLastError();
}

}  // namespace moe

// ---------------------------------------------------------------------------
// moe_permute without a workspace.
//
// Some callers cannot hand this library a workspace: a serving runtime that
// has already given all free device memory to its expert cache and KV pool,
// code that runs while a stream is being captured (cudaMalloc is not allowed
// there), or a host program with no device allocator of its own.  For them,
// the permutation's only scratch (the per-chunk expert counts) lives in the
// fixed array below, which every GPU that loads this library holds until the
// process exits.  The counts are fully rewritten by each call, so nothing has
// to be cleared first; calls that overlap on the GPU share the array and race.
// ---------------------------------------------------------------------------
namespace moe {
namespace {

constexpr int kFixedScratchInts = 65536;  // 256 KiB: nchunks * E <= 65536
static __device__ __align__(256) int32_t g_fixed_perm_scratch[kFixedScratchInts];

constexpr int kMaxDevices = 64;
int32_t* g_fixed_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_fixed_scratch_mu;

// Device address of the array on the current device, looked up once per device.
cudaError_t fixed_scratch_ptr(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_fixed_scratch_mu);
  if (!g_fixed_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fixed_perm_scratch);
    if (e != cudaSuccess) return e;
    g_fixed_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_fixed_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute_fixed_scratch(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E,
                                                int32_t* offsets, int32_t* perm_token, int32_t* inv_perm,
                                                int32_t* dev_status, moe_stream_t stream) {
  using namespace moe;
  if (T < 0 || k < 1 || E < 1 || E > 1024 || T * (int64_t)k > INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (!offsets || (T > 0 && (!topk_idx || !perm_token || !inv_perm))) return MOE_ERR_INVALID_ARG;
  const int64_t S = T * k;
  const int64_t nchunks = (S + kChunk - 1) / kChunk;
  if (nchunks * (int64_t)E > kFixedScratchInts) return MOE_ERR_WORKSPACE;  // beyond the fixed capacity
  int32_t* scratch = nullptr;
  if (fixed_scratch_ptr(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  PermuteScratch ps;
  ps.chunk_counts = scratch;
  ps.nchunks = (int)nchunks;
  return launch_permute(topk_idx, S, k, E, offsets, perm_token, inv_perm, ps, dev_status,
                        reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
