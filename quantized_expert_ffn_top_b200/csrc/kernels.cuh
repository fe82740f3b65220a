// Kernel launchers of the B200 MoE layer (internal; the C ABI is in api.cu).
#pragma once

#include <string.h>

#include <utility>

#include "common.cuh"

namespace moe {

// Host-side count of kernel launches (moe_kernel_launch_count).
void count_launches(int n);

// Bound of every device wait in SM clocks (MOE_OPT_WAIT_CYCLES).
long long wait_cycles();

// Launch with programmatic dependent launch allowed (MOE_OPT_PDL, on by
// default): the kernel may begin while the previous kernel in the stream
// finishes; it calls pdl_wait() before reading that kernel's results.
bool pdl_enabled();
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

__device__ __forceinline__ float load_f32(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load_f32(const uint16_t* p) { return bf16_to_f32(__ldg(p)); }

// Blocked scale-factor layout of PREPARED banks and of the GEMM path's
// quantised activations: per 128 rows and per group of 4 consecutive scale
// columns, one 512-byte block in which row r's 4 scales sit at byte
// (r % 32) * 16 + ((r % 128) / 32) * 4 -- the order in which the tensor core
// scale-factor copy (tcgen05.cp 32x128b, replicated to the four lane
// quarters) lays 128 rows x 4 scales into tensor memory.
__host__ __device__ __forceinline__ int64_t sf_blocked_offset(int64_t row, int64_t col, int64_t ncols) {
  const int64_t groups = ncols / 4;  // scale columns are padded to a multiple of 4
  return ((row / 128) * groups + col / 4) * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4 + (col % 4);
}

// quant.cu
cudaError_t launch_amax(const void* x, int x_dtype, int64_t n, float* out, int num_sms, cudaStream_t s);
cudaError_t launch_quantize(int fmt, const void* x, int x_dtype, int64_t rows, int64_t K, const float* scale_in,
                            const float* amax, uint8_t* codes, uint8_t* sf, float* scale_out, int num_sms,
                            cudaStream_t s);

// Small batches: where and how x is quantised into the gather layout
// (quant_token_gather in token_quant.cuh): the static tensor scale or the
// amax it comes from (NVFP4), the codes [T][8][K/2] and the scale lines.
// Tokens a gathering batch may hold: a tile's scale lines serve rows below 32,
// and a token picks an expert at most once.
constexpr int kGatherMaxT = 32;
// Slots a gathering batch may hold: the one-kernel FFN keeps the token of
// every slot position in shared memory.
constexpr int kGatherMaxS = 256;
struct GatherQuant {
  const float* scale;
  const float* amax;
  uint8_t* xg;
  uint8_t* xsl;
  int32_t* zero;   // optional: nzero counters set to 0 (by block 0, after the wait)
  int nzero;
};

// route.cu
cudaError_t launch_router_logits(const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias, int E,
                                 float* logits, cudaStream_t s);
// logits: nparts partial sums part_stride apart (1 = plain logits); logits_out
// (nullable) receives their sum.
cudaError_t launch_topk(const float* logits, int nparts, int64_t part_stride, float* logits_out, int64_t T, int E,
                        int k, int32_t* idx, float* w, int32_t* status, cudaStream_t s);
// The one-kernel forward's router at T <= 32 (fmt NVFP4 or MXFP4, H % 256 ==
// 0, E <= 256): logits (the small-batch order), x into the gather layout, and
// the top k by the block that finishes last (`ticket`: zero on entry, left
// zero).
cudaError_t launch_router_decode(int fmt, const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias,
                                 int E, int k, float* logits, int32_t* idx, float* w, int32_t* ticket,
                                 const GatherQuant& q, int32_t* status, cudaStream_t s);

// permute.cu
struct PermuteScratch {
  int32_t* chunk_counts;   // [nchunks][E]
  int nchunks;
};
int permute_chunk_slots();
// Tile plan the permutation may write on the way (bn = 0: none).
struct PlanOut {
  int bn;
  int32_t* poff;                  // [E+1] padded offsets
  struct TileEntry* tiles;        // [max_tiles]
  int32_t* ntiles;
  int max_tiles;
};
// x quantisation (MATCH mode) the one-block permutation can run once it has
// placed the slots: every token row is quantised once into the padded rows
// of its slots (the plan's padded offsets, so it needs plan.bn > 0).
struct SlotQuantOut {
  int fmt;                 // MOE_FMT_NVFP4, MOE_FMT_MXFP4 or MOE_FMT_FP8
  const uint16_t* x;       // [T][K] bf16, T = S / k
  int K;                   // a multiple of 64
  int64_t P;               // padded rows allocated for the codes
  const float* scale;      // static per-tensor scale, or NULL
  const float* amax;       // dynamic: amax(x)
  uint8_t* codes;          // [P][K/2 | K]
  uint8_t* sf;             // blocked block scales
  int32_t* zero;           // optional: nzero counters set to 0
  int nzero;
};
// *planned (nullable) tells whether `plan` was written; if not, the caller
// runs the plan kernel itself.  *quantized (nullable) tells whether the x
// quantisation `quant` asked for was done.
cudaError_t launch_permute(const int32_t* idx, int64_t S, int k, int E, int32_t* offsets, int32_t* perm_token,
                           int32_t* inv_perm, PermuteScratch scratch, int32_t* status, cudaStream_t s,
                           const PlanOut* plan, bool* planned, const SlotQuantOut* quant = nullptr,
                           bool* quantized = nullptr);
// Whether launch_permute can quantise x in its one-block pass for S slots.
bool permute_can_quantize(int64_t S, int64_t T, int E);

// gemv.cu -- small-batch expert FFN (one pass over each active expert).
struct GemvArgs {
  int fmt, act, E, H, I;
  const uint8_t* w13;      // prepared
  const uint8_t* w13_sf;
  const float* w13_gs;
  const uint8_t* w2;
  const uint8_t* w2_sf;
  const float* w2_gs;
  const float* x_scale;    // MATCH: static scale (device) or nullptr
  const float* h_scale;
  const uint16_t* x;       // [T][H]
  int64_t T;
  int64_t S;               // slots: offsets must satisfy 0 <= offsets[e] <= offsets[e+1] <= S
  const int32_t* perm_token;
  const int32_t* offsets;
  float* x_amax;           // workspace scalars (dynamic scales)
  float* h_amax;
  float* h;                // [S][I] fp32
  uint16_t* y_perm;        // [S][H]
  const struct TileEntry* tiles;  // token groups of at most 8 slots per expert
  const int32_t* num_tiles;
  int32_t* status;
  long long wait_cycles;   // bound of every device wait (SM clocks)
};
constexpr int kGemvTokens = 8;  // token columns of one GEMV work item (the MMA n)
cudaError_t launch_gemv_up(const GemvArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_gemv_down(const GemvArgs& a, int num_sms, cudaStream_t s);

// combine.cu
cudaError_t launch_combine(const uint16_t* y_perm, const int32_t* inv_perm, const float* w, int64_t T, int k, int H,
                           const uint16_t* shared_y, uint16_t* out, int32_t* status, cudaStream_t s);
// out[i] = bf16(out32[i]) for n values (n % 8 == 0, 16-byte aligned).
cudaError_t launch_round_rows(const float* out32, int64_t n, uint16_t* out, const int32_t* status, int num_sms,
                              cudaStream_t s);

// cache.cu -- the HBM slot pool in front of a host-memory expert bank.
// An expert's regions (W13, its scales, W2, its scales) are contiguous in
// the PREPARED layout; src[r] + e * bytes[r] (device addresses of mapped
// host memory) goes to dst[r] + slot * bytes[r], and gs_per[g] fp32 part
// scales of gs_src[g] + e * gs_per[g] go to gs_dst[g] + slot * gs_per[g].
struct CacheCopy {
  const uint8_t* src[4];
  uint8_t* dst[4];
  int64_t bytes[4];
  int nregions;
  const float* gs_src[2];
  float* gs_dst[2];
  int gs_per[2];
  int ngs;
};
size_t cache_state_words(int E, int n_slots);
cudaError_t launch_cache_admit(const int32_t* idx, int64_t S, int E, int n_slots, int32_t* state, int32_t* idx_slot,
                               int32_t* status, cudaStream_t s);
cudaError_t launch_cache_fetch(const int32_t* state, int E, int n_slots, const CacheCopy& cc, int num_sms,
                               cudaStream_t s);

// prepare.cu
cudaError_t launch_prepare_rows(int fmt, const uint8_t* src, uint8_t* dst, int64_t E, int64_t R, int64_t row_bytes,
                                bool interleave, cudaStream_t s);
cudaError_t launch_dequant_bf16(int fmt, const uint8_t* codes, const uint8_t* sf, const float* gs, int gstride,
                                int64_t part_rows, int64_t E, int64_t R, int64_t K, uint16_t* out, cudaStream_t s);
cudaError_t launch_prepare_sf(const uint8_t* src, uint8_t* dst, int64_t E, int64_t R, int64_t ncols,
                              int64_t ncols_padded, bool interleave, cudaStream_t s);

}  // namespace moe
