// Token-to-expert histogram, offsets and stable permutation of the T*k slots,
// with no atomic updates of the counts or positions (the result is
// deterministic).
//
// The permuted order is the expert-major "slot pool" of the
// atomicmilkshake/FreeToken fork README ("Known limits"): every expert's slots
// form one contiguous segment, so the grouped FFN reads each expert's weights
// for a dense block of rows.  Slots keep their flat order i = t*k + j inside a
// segment (stable), which makes the permutation unique and bit-comparable.
//
// Two passes over chunks of kChunk slots (8 warps x 256):
//   1. per chunk and expert, the count (warp-private counters fed by
//      __match_any_sync, one writer lane per expert and step);
//   2. per chunk again: every block reads all chunks' counts, so it knows
//      for each expert the slots in earlier chunks and the total; a scan of
//      the totals over experts gives the offsets (block 0 writes them and,
//      on request, the grouped FFN's tile plan); each warp's base = expert
//      offset + earlier chunks + earlier warps, and each slot's rank among
//      equal experts earlier in its warp step -> perm_token[p] = t,
//      inv_perm[i] = p.
// No block waits for another inside a kernel, and nothing is cleared first.
// Small batches run all three inside one block, which in the forward at up
// to 8 tokens also quantises x into the FFN's padded rows.
#include <string.h>

#include <mutex>

#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "token_quant.cuh"

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
  // the lane's eight slot experts are read up front, in one round trip
  int ev[kSlotsPerWarp / 32];
#pragma unroll
  for (int st = 0; st < kSlotsPerWarp / 32; ++st)
    ev[st] = slot_expert(idx, S, base + (int64_t)warp * kSlotsPerWarp + st * 32 + lane, E, status);
#pragma unroll
  for (int st = 0; st < kSlotsPerWarp / 32; ++st) {
    const int e = ev[st];
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    if (e >= 0 && lane == leader) my[e] += __popc(peers);
    __syncwarp();
  }
}

// Exclusive scan of v over the block's kPermWarps warps (256 threads);
// *total receives the sum.  Every thread calls it.
__device__ __forceinline__ int32_t scan256_excl(int32_t v, int32_t* warp_tot, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  __syncthreads();
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int32_t base = 0, sum = 0;
#pragma unroll
  for (int w = 0; w < kPermWarps; ++w) {
    base += w < warp ? warp_tot[w] : 0;
    sum += warp_tot[w];
  }
  *total = sum;
  return incl - v + base;
}

// Pass 1: per chunk and expert, the count.
__global__ void __launch_bounds__(kPermWarps * 32) perm_count_kernel(const int32_t* __restrict__ idx, int64_t S,
                                                                     int E, int32_t* __restrict__ chunk_counts,
                                                                     int32_t* status) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

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

// Pass 2 (see the file's head).  Dynamic shared memory: [kPermWarps][E]
// counters, then [E] totals and [E] earlier-chunk counts.
__global__ void __launch_bounds__(kPermWarps * 32) perm_scatter_kernel(const int32_t* __restrict__ idx, int64_t S,
                                                                       int k, int E,
                                                                       const int32_t* __restrict__ chunk_counts,
                                                                       int32_t* __restrict__ offsets, PlanOut plan,
                                                                       int32_t* __restrict__ perm_token,
                                                                       int32_t* __restrict__ inv_perm) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  extern __shared__ int32_t cnt[];
  int32_t* tot = cnt + kPermWarps * E;   // [E] slots of the expert in all chunks, then its offset
  int32_t* before = tot + E;             // [E] slots of the expert in earlier chunks
  __shared__ int32_t warp_tot[kPermWarps];
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) cnt[i] = 0;
  const int nchunks = gridDim.x, c = blockIdx.x;
  // every chunk's count of expert e, eight loads in flight
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0, pre = 0;
    for (int c0 = 0; c0 < nchunks; c0 += 8) {
      int32_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = c0 + u < nchunks ? __ldg(chunk_counts + (int64_t)(c0 + u) * E + e) : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (c0 + u == c) pre = run;
        run += v[u];
      }
    }
    tot[e] = run;
    before[e] = pre;
  }
  __syncthreads();
  const int64_t base = (int64_t)c * kChunk;
  warp_counts(idx, S, base, E, cnt, nullptr);
  // scans over experts: each thread owns a contiguous group of `per` experts
  const int per = (E + (int)blockDim.x - 1) / (int)blockDim.x;
  const int e0 = threadIdx.x * per;
  int32_t mine = 0, pad_mine = 0, til_mine = 0;
  const bool with_plan = c == 0 && plan.bn > 0;
  for (int e = e0; e < e0 + per && e < E; ++e) {
    mine += tot[e];
    pad_mine += (tot[e] + 127) / 128 * 128;
    if (with_plan) til_mine += (tot[e] + plan.bn - 1) / plan.bn;
  }
  int32_t total, pad_total = 0, til_total = 0;
  int32_t off = scan256_excl(mine, warp_tot, &total);
  int32_t pbase = 0, tbase = 0;
  if (with_plan) {
    pbase = scan256_excl(pad_mine, warp_tot, &pad_total);
    tbase = scan256_excl(til_mine, warp_tot, &til_total);
  }
  __syncthreads();
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int32_t n = tot[e];
    if (c == 0) offsets[e] = off;
    if (with_plan) {
      plan.poff[e] = pbase;
      const int til = (n + plan.bn - 1) / plan.bn;
      for (int j = 0; j < til && tbase + j < plan.max_tiles; ++j) {
        TileEntry te;
        te.e = e;
        te.row0 = pbase + j * plan.bn;
        te.nvalid = min(plan.bn, n - j * plan.bn);
        te.p0 = off + j * plan.bn;
        plan.tiles[tbase + j] = te;
      }
      pbase += (n + 127) / 128 * 128;
      tbase += til;
    }
    tot[e] = off;  // the expert's offset
    off += n;
  }
  if (c == 0 && threadIdx.x == 0) {
    offsets[E] = total;
    if (with_plan) {
      plan.poff[E] = pad_total;
      *plan.ntiles = min(til_total, plan.max_tiles);
    }
  }
  __syncthreads();
  // exclusive prefix over warps per expert, from the chunk's base
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = tot[e] + before[e];
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
  int ev[kSlotsPerWarp / 32];
#pragma unroll
  for (int st = 0; st < kSlotsPerWarp / 32; ++st)
    ev[st] = slot_expert(idx, S, base + (int64_t)warp * kSlotsPerWarp + st * 32 + lane, E, nullptr);
#pragma unroll
  for (int st = 0; st < kSlotsPerWarp / 32; ++st) {
    const int64_t i = base + (int64_t)warp * kSlotsPerWarp + st * 32 + lane;
    const int e = ev[st];
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

// Up to kBlockMaxS slots: the same passes inside one block of 32 warps,
// each warp owning a contiguous range of slots, the per-warp expert counters
// in shared memory -- one launch instead of three.  The block can also write
// the grouped FFN's tile plan (padded offsets and tile list), which needs the
// same per-expert counts.
constexpr int kBlockWarps = 32;
constexpr int64_t kBlockMaxS = 8192;   // beyond, one SM's scattered stores are the bottleneck
// x quantisation inside the block: a warp per token.  One SM then moves
// every token's bytes (about 12 KB a token at H = 2048, k = 8), so it pays
// only for the smallest batches: measured 2 us faster than the separate
// quantiser at T = 4 and 6 us slower at T = 32.
constexpr int64_t kBlockQuantMaxT = 8;
constexpr int kBlockQuantMaxE = 256;

// Exclusive scan of one value per thread over a 1024-thread block; *total
// receives the sum.  Every thread calls it.
__device__ __forceinline__ int32_t block_scan_excl(int32_t v, int32_t* warp_tot, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  __syncthreads();  // warp_tot free
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
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  *total = warp_tot[32];
  return incl - v + warp_tot[warp];
}

// The experts of a warp's next 4 x 32 slots, loaded together.
__device__ __forceinline__ void load4(const int32_t* idx, int64_t S, int64_t base, int64_t hi, int E, int32_t* status,
                                      int (&e)[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = base + u * 32 + lane;
    e[u] = (i < hi) ? slot_expert(idx, S, i, E, status) : -1;
  }
}

// Dynamic shared memory of the one-block kernel: the per-warp counters and
// the offsets ([kBlockWarps + 1][E] ints); with the x quantisation also the
// padded offsets ([E]), then, from the next 16-byte boundary, the warps'
// reorder buffers and the NVFP4 multiplier table.
constexpr size_t block_quant_buf_offset(int E) { return ((size_t)(kBlockWarps + 2) * E * 4 + 15) / 16 * 16; }
template <int QFMT>
constexpr size_t block_smem_bytes(int E) {
  return QFMT == 0 ? (size_t)(kBlockWarps + 1) * E * 4
                   : block_quant_buf_offset(E) + (size_t)kBlockWarps * TokenQuant<QFMT>::kWarpBuf * 16 + 128 * 4;
}

// QFMT != 0: after placing the slots, the block also quantises x (format
// QFMT) into the padded rows of the slots, as the per-token x quantiser does.
template <int QFMT>
__global__ void __launch_bounds__(kBlockWarps * 32) perm_block_kernel(const int32_t* __restrict__ idx, int64_t S,
                                                                     int k, int E, int32_t* __restrict__ offsets,
                                                                     int32_t* __restrict__ perm_token,
                                                                     int32_t* __restrict__ inv_perm,
                                                                     int32_t* status, PlanOut plan, SlotQuantOut q) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  extern __shared__ __align__(16) int32_t blk_smem[];
  int32_t* cnt = blk_smem;  // [kBlockWarps][E], then [E] offsets (then the quantisation's part)
  int32_t* tot = cnt + kBlockWarps * E;
  int32_t* pofs = tot + E;  // QFMT: [E] padded offsets
  __shared__ int32_t warp_tot[33];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t per = ((S + kBlockWarps - 1) / kBlockWarps + 127) / 128 * 128;  // slots per warp
  for (int i = threadIdx.x; i < kBlockWarps * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  int32_t* my = cnt + warp * E;
  const int64_t lo = warp * per, hi = min(S, lo + per);
  for (int64_t base = lo; base < hi; base += 128) {
    int ev[4];
    load4(idx, S, base, hi, E, status, ev);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const unsigned peers = __match_any_sync(0xffffffffu, ev[u]);
      if (ev[u] >= 0 && lane == __ffs(peers) - 1) my[ev[u]] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  // per expert: exclusive prefix over warps, total
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0;
    for (int w = 0; w < kBlockWarps; ++w) {
      const int32_t v = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += v;
    }
    tot[e] = run;
  }
  __syncthreads();
  // exclusive scan of the totals over experts (E <= 1024 = blockDim)
  const int e = threadIdx.x;
  const int32_t n_e = e < E ? tot[e] : 0;
  int32_t total;
  const int32_t excl = block_scan_excl(n_e, warp_tot, &total);
  if (e < E) {
    tot[e] = excl;
    offsets[e] = excl;
  }
  if (e == 0) offsets[E] = total;
  if (plan.bn > 0) {
    // padded offsets (segments start on multiples of 128 rows) and the tiles
    const int32_t pad = (n_e + 127) / 128 * 128;
    const int32_t til = (n_e + plan.bn - 1) / plan.bn;
    int32_t pad_total, til_total;
    const int32_t pbase = block_scan_excl(pad, warp_tot, &pad_total);
    const int32_t tbase = block_scan_excl(til, warp_tot, &til_total);
    if (e < E) {
      plan.poff[e] = pbase;
      if (QFMT != 0) pofs[e] = pbase;
      for (int j = 0; j < til && tbase + j < plan.max_tiles; ++j) {
        TileEntry te;
        te.e = e;
        te.row0 = pbase + j * plan.bn;
        te.nvalid = min(plan.bn, n_e - j * plan.bn);
        te.p0 = excl + j * plan.bn;
        plan.tiles[tbase + j] = te;
      }
    }
    if (e == 0) {
      plan.poff[E] = pad_total;
      *plan.ntiles = min(til_total, plan.max_tiles);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kBlockWarps * E; i += blockDim.x) cnt[i] += tot[i % E];
  __syncthreads();
  for (int64_t base = lo; base < hi; base += 128) {
    int ev[4];
    load4(idx, S, base, hi, E, nullptr, ev);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = base + u * 32 + lane;
      const int ee = ev[u];
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
  if constexpr (QFMT != 0) {
    using Q = TokenQuant<QFMT>;
    uint4* tbuf = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(cnt) + block_quant_buf_offset(E));
    float* r_tab = reinterpret_cast<float*>(tbuf + kBlockWarps * Q::kWarpBuf);
    const float scale = act_scale_of(QFMT, q.scale, q.amax);
    if (QFMT == MOE_FMT_NVFP4 && threadIdx.x < 128) r_tab[threadIdx.x] = nvfp4_multiplier(threadIdx.x, scale);
    for (int i = threadIdx.x; i < q.nzero; i += blockDim.x) q.zero[i] = 0;
    __syncthreads();  // inv_perm (global, this block's stores), padded offsets, table
    const int64_t T = S / k;
    for (int64_t t = warp; t < T; t += kBlockWarps) {
      // padded row of slot (t, j): the slot's rank in its expert past the
      // expert's first padded row
      auto row_of = [&](int j) -> int64_t {
        const int64_t i = t * k + j;
        const int32_t p = __ldcg(inv_perm + i);
        if (p < 0) return -1;
        const int e = __ldg(idx + i);
        if (e < 0 || e >= E) return -2;
        const int64_t row = (int64_t)pofs[e] + (p - tot[e]);
        return (row >= 0 && row < q.P) ? row : -2;
      };
      quant_token_slots<QFMT>(q.x + t * q.K, q.K, k, scale, r_tab, tbuf + warp * Q::kWarpBuf, row_of, q.codes,
                              q.sf, status);
    }
  }
}

bool permute_can_quantize(int64_t S, int64_t T, int E) {
  return S > 0 && S <= kBlockMaxS && T <= kBlockQuantMaxT && E <= kBlockQuantMaxE;
}

template <int QFMT>
cudaError_t launch_perm_block(const int32_t* idx, int64_t S, int k, int E, int32_t* offsets, int32_t* perm_token,
                              int32_t* inv_perm, int32_t* status, cudaStream_t s, const PlanOut& p,
                              const SlotQuantOut& q) {
  const size_t smem = block_smem_bytes<QFMT>(E);
  // E <= 1024 needs at most 132 KB without the quantisation, E <= 256 at
  // most 99 KB with it
  const size_t smem_max = block_smem_bytes<QFMT>(QFMT == 0 ? 1024 : kBlockQuantMaxE);
  cudaError_t e = cudaFuncSetAttribute(perm_block_kernel<QFMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_max);
  if (e != cudaSuccess) return e;
  e = launch_pdl(perm_block_kernel<QFMT>, dim3(1), dim3(kBlockWarps * 32), smem, s, idx, S, k, E, offsets,
                 perm_token, inv_perm, status, p, q);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_permute(const int32_t* idx, int64_t S, int k, int E, int32_t* offsets, int32_t* perm_token,
                           int32_t* inv_perm, PermuteScratch scratch, int32_t* status, cudaStream_t s,
                           const PlanOut* plan, bool* planned, const SlotQuantOut* quant, bool* quantized) {
  if (planned) *planned = false;
  if (quantized) *quantized = false;
  if (S > 0 && S <= kBlockMaxS) {
    PlanOut p;
    if (plan) {
      p = *plan;
    } else {
      memset(&p, 0, sizeof(p));
    }
    SlotQuantOut q;
    memset(&q, 0, sizeof(q));
    const bool with_q = quant && p.bn > 0 && quant->K % 64 == 0 && permute_can_quantize(S, S / k, E);
    if (with_q) q = *quant;
    cudaError_t e;
    switch (with_q ? q.fmt : 0) {
      case MOE_FMT_NVFP4:
        e = launch_perm_block<MOE_FMT_NVFP4>(idx, S, k, E, offsets, perm_token, inv_perm, status, s, p, q);
        break;
      case MOE_FMT_MXFP4:
        e = launch_perm_block<MOE_FMT_MXFP4>(idx, S, k, E, offsets, perm_token, inv_perm, status, s, p, q);
        break;
      case MOE_FMT_FP8:
        e = launch_perm_block<MOE_FMT_FP8>(idx, S, k, E, offsets, perm_token, inv_perm, status, s, p, q);
        break;
      default:
        e = launch_perm_block<0>(idx, S, k, E, offsets, perm_token, inv_perm, status, s, p, q);
        q.fmt = 0;
        break;
    }
    if (e != cudaSuccess) return e;
    if (planned && plan && plan->bn > 0) *planned = true;
    if (quantized) *quantized = with_q && q.fmt != 0;
    return cudaSuccess;
  }
  const int nchunks = (int)((S + kChunk - 1) / kChunk);
  if (nchunks == 0) {
    // no slots: offsets are all zero
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
  }
  PlanOut p;
  if (plan) {
    p = *plan;
  } else {
    memset(&p, 0, sizeof(p));
  }
  cudaError_t e = launch_pdl(perm_count_kernel, dim3(nchunks), dim3(kPermWarps * 32),
                             sizeof(int32_t) * kPermWarps * E, s, idx, S, E, scratch.chunk_counts, status);
  if (e != cudaSuccess) return e;
  e = launch_pdl(perm_scatter_kernel, dim3(nchunks), dim3(kPermWarps * 32), sizeof(int32_t) * (kPermWarps + 2) * E,
                 s, idx, S, k, E, (const int32_t*)scratch.chunk_counts, offsets, p, perm_token, inv_perm);
  if (e != cudaSuccess) return e;
  count_launches(2);
  if (planned && plan && plan->bn > 0) *planned = true;
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
                        reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
