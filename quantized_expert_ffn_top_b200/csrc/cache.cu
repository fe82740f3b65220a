// Host -> HBM expert streaming: a pool of expert slots in HBM, managed least
// recently used, in front of an expert bank kept in page-locked host memory.
// This is the expert slot pool of the atomicmilkshake/FreeToken fork README
// ("Known limits") and the host-memory offload with a global LRU expert cache
// of the FreeToken upstream README ("About"), rebuilt so that the device
// decides and copies by itself: a forward through the cache needs no host
// synchronisation and can be captured in a CUDA graph.
//   admit  one block: marks the experts the batch routes to, keeps the slots
//          of those already resident, gives every other one the least
//          recently used slot that no expert of this batch holds (empty
//          slots first), and rewrites the top-k ids into slot ids;
//   fetch  copies the admitted experts from host memory into their slots
//          (loads of mapped, page-locked memory over PCIe);
// and the layer then runs on the pool as a bank of n_slots experts.
#include "kernels.cuh"

namespace moe {

// Cache state (int32 words in device memory):
//   [0] clock  [1] experts fetched by the last call  [2] total fetched
//   [3] total hits  then slot_of[E], expert_of[n], stamp[n], fetch_e[n], fetch_s[n]
struct CacheView {
  int32_t* head;
  int32_t* slot_of;
  int32_t* expert_of;
  int32_t* stamp;
  int32_t* fetch_e;
  int32_t* fetch_s;
};
__host__ __device__ inline CacheView cache_view(int32_t* st, int E, int n) {
  CacheView v;
  v.head = st;
  v.slot_of = st + 4;
  v.expert_of = v.slot_of + E;
  v.stamp = v.expert_of + n;
  v.fetch_e = v.stamp + n;
  v.fetch_s = v.fetch_e + n;
  return v;
}
size_t cache_state_words(int E, int n) { return 4 + (size_t)E + 4 * (size_t)n; }

constexpr int kAdmitThreads = 1024;   // E <= 1024 and n_slots <= 1024

__global__ void __launch_bounds__(kAdmitThreads) cache_admit_kernel(const int32_t* __restrict__ idx, int64_t S, int E,
                                                                    int n, int32_t* st, int32_t* __restrict__ idx_slot,
                                                                    int32_t* status) {
  pdl_wait();  // the top-k ids come from the previous kernel
  pdl_trigger();
  __shared__ int active[1024];
  __shared__ unsigned long long key[1024];
  __shared__ int nmiss, nhit;
  const CacheView c = cache_view(st, E, n);
  const int tid = threadIdx.x;
  const int clk = c.head[0] + 1;
  for (int e = tid; e < E; e += blockDim.x) active[e] = 0;
  if (tid == 0) nmiss = nhit = 0;
  __syncthreads();
  for (int64_t i = tid; i < S; i += blockDim.x) {
    const int e = idx[i];
    if (e >= 0 && e < E) active[e] = 1;
    else raise_status(status, MOE_ERR_DEVICE_FAULT);
  }
  __syncthreads();
  // slots sorted by (held by an expert of this batch, last use), empty slots
  // first: the first ones are the victims
  for (int s = tid; s < 1024; s += blockDim.x) {
    unsigned long long k = ~0ull;
    if (s < n) {
      const int e = c.expert_of[s];
      const bool hit = e >= 0 && e < E && active[e];
      if (hit) {
        c.stamp[s] = clk;
        atomicAdd(&nhit, 1);
      }
      const unsigned int rank = hit ? 0xFFFFFFFFu : (e < 0 ? 0u : (unsigned int)c.stamp[s] + 1u);
      k = ((unsigned long long)rank << 32) | (unsigned int)s;
    }
    key[s] = k;
  }
  __syncthreads();
  // bitonic sort of the 1024 keys, ascending
  for (int size = 2; size <= 1024; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < 1024; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const unsigned long long a = key[i], b = key[j];
          if ((a > b) == up) {
            key[i] = b;
            key[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // misses, in expert order, take the victims in order
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + tid;
    const bool miss = e < E && active[e] && c.slot_of[e] < 0;
    // rank among this pass's misses (experts e0 .. e0 + blockDim.x - 1): a block-wide count through shared memory
    __shared__ int wcount[32];
    const unsigned m = __ballot_sync(0xffffffffu, miss);
    if ((tid & 31) == 0) wcount[tid >> 5] = __popc(m);
    __syncthreads();
    int before = nmiss;
    for (int w = 0; w < (tid >> 5); ++w) before += wcount[w];
    const int r = before + __popc(m & ((1u << (tid & 31)) - 1u));
    if (miss) {
      const unsigned long long k = r < n ? key[r] : ~0ull;
      const int v = (int)(k & 0xFFFFFFFFull);
      if (r >= n || (k >> 32) == 0xFFFFFFFFull) {
        raise_status(status, MOE_ERR_DEVICE_FAULT);   // more experts than free slots
      } else {
        const int old = c.expert_of[v];
        if (old >= 0 && old < E) c.slot_of[old] = -1;
        c.expert_of[v] = e;
        c.slot_of[e] = v;
        c.stamp[v] = clk;
        c.fetch_e[r] = e;
        c.fetch_s[r] = v;
      }
    }
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += wcount[w];
      nmiss += tot;
    }
    __syncthreads();   // nmiss updated, wcount free for the next round
  }
  // the batch's top-k ids as slot ids
  for (int64_t i = tid; i < S; i += blockDim.x) {
    const int e = idx[i];
    idx_slot[i] = (e >= 0 && e < E) ? c.slot_of[e] : -1;
  }
  if (tid == 0) {
    const int m = nmiss < n ? nmiss : n;
    c.head[0] = clk;
    c.head[1] = m;
    c.head[2] += m;
    c.head[3] += nhit;
  }
}

// Copies the experts admitted by the last admit from host memory into their
// slots: every region of an expert is contiguous in the PREPARED layout.
__global__ void __launch_bounds__(256) cache_fetch_kernel(const int32_t* st, int E, int n, CacheCopy cc) {
  pdl_wait();  // the fetch list comes from the previous kernel
  pdl_trigger();
  const CacheView c = cache_view(const_cast<int32_t*>(st), E, n);
  const int m = c.head[1];
  int64_t vec_total = 0;
  for (int r = 0; r < cc.nregions; ++r) vec_total += cc.bytes[r] / 16;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int f = 0; f < m; ++f) {
    const int e = c.fetch_e[f], s = c.fetch_s[f];
    // four 16-byte vectors in flight per thread
    for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < vec_total; i0 += 4 * stride) {
      uint4 v[4];
      uint4* dst[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        int64_t i = i0 + u * stride;
        dst[u] = nullptr;
        if (i >= vec_total) continue;
        int r = 0;
        while (i >= cc.bytes[r] / 16) {
          i -= cc.bytes[r] / 16;
          ++r;
        }
        const uint4* src = reinterpret_cast<const uint4*>(cc.src[r] + (int64_t)e * cc.bytes[r]) + i;
        dst[u] = reinterpret_cast<uint4*>(cc.dst[r] + (int64_t)s * cc.bytes[r]) + i;
        v[u] = __ldcs(src);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (dst[u]) *dst[u] = v[u];
    }
    if (blockIdx.x == 0 && threadIdx.x < cc.ngs) {
      const int g = threadIdx.x;   // the expert's part scales
      cc.gs_dst[g][s * cc.gs_per[g] + 0] = cc.gs_src[g][e * cc.gs_per[g] + 0];
      if (cc.gs_per[g] > 1) cc.gs_dst[g][s * cc.gs_per[g] + 1] = cc.gs_src[g][e * cc.gs_per[g] + 1];
    }
  }
}

cudaError_t launch_cache_admit(const int32_t* idx, int64_t S, int E, int n, int32_t* state, int32_t* idx_slot,
                               int32_t* status, cudaStream_t s) {
  if (E > 1024 || n > 1024 || n < 1) return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(cache_admit_kernel, dim3(1), dim3(kAdmitThreads), 0, s, idx, S, E, n, state, idx_slot,
                             status);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_cache_fetch(const int32_t* state, int E, int n, const CacheCopy& cc, int num_sms, cudaStream_t s) {
  for (int r = 0; r < cc.nregions; ++r)
    if (cc.bytes[r] % 16 != 0) return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(cache_fetch_kernel, dim3(num_sms * 4), dim3(256), 0, s, state, E, n, cc);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe
