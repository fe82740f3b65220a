// Internal interface of the tensor-core grouped GEMM path (gemm_tc.cu).
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

// One token tile of one expert: the padded row of its first token, the
// number of valid tokens (<= tile width) and the compact slot of its first
// token (offsets[e] + j * tile width).
struct TileEntry {
  int32_t e, row0, nvalid, p0;
};

enum { kEpiUpQuant = 0, kEpiUpF32 = 1, kEpiDown = 2, kEpiLogits = 3 };

// Operand type of the router GEMM (bf16 x and Wr) next to the moe_fmt values.
constexpr int kFmtBF16 = 4;

struct GemmArgs {
  int fmt, E, K, R;            // reduction length, weight rows per expert
  const uint8_t* w_sf;         // PREPARED blocked weight scales (NULL for FP8)
  const uint8_t* b_sf;         // blocked activation scales over padded rows
  const float* w_gs;           // [E][2] gate/up part scales, or [E] down scales
  const float* act_scale;      // static activation scale of the B operand, or NULL
  const float* act_amax;       // amax of the B operand's source (dynamic scale)
  const TileEntry* tiles;
  const int32_t* num_tiles;
  int I;                       // up: h row length
  uint8_t* hq;                 // up (quantised): h codes [padded rows][I/2]
  uint8_t* hsf;                //                 h scales, blocked
  const float* h_scale;        //                 static h scale (NVFP4)
  float* h32;                  // up (fp32): h [padded rows][I]
  float* h_amax;               //            amax of h
  uint16_t* y;                 // down: y_perm [y_rows][ldy] bf16
  int ldy;
  int64_t y_rows;
  // down, with the combine in the epilogue (out32 != NULL): out32[t][o] +=
  // w_perm[p] * y[p][o] for slot p of token t = perm_token[p] (w_perm NULL:
  // weight 1), fp32 reductions; t outside [0, out_rows) is a device fault
  float* out32;
  const int32_t* perm_token;
  const float* w_perm;
  int64_t out_rows;
  float* logits;               // router: logits [T][ldy] fp32 (+ bias)
  const float* bias;
  int ksplit;                  // router: K split over this many partial outputs,
  int64_t split_stride;        //         split s at logits + s * split_stride
  int64_t dense_rows;          // > 0: token tiles are plain row blocks (no tile list)
  // Early weight loads (programmatic launch): before waiting for the previous
  // kernel, the producer issues the weight tiles of its first stages.  Their
  // experts come from the tile list (1: written at least two kernels back,
  // so complete once this kernel runs) or from `offsets` (2: the tile list
  // is the previous kernel's output; offsets are older; E <= 256, else no
  // early loads).  0: off.
  int w_early;
  int w_early_l2;              // and this many further stages' weights prefetched to L2
  const int32_t* offsets;      // [E+1] compact expert offsets (w_early == 2; E <= 256)
  int max_tiles;               // entries allocated in `tiles`
  int32_t* status;
  long long wait_cycles;       // bound of every device wait (SM clocks)
};

struct QuantPaddedArgs {
  int E, K;
  int64_t S, T;
  int64_t P;                   // padded rows allocated (writes stay below)
  const int32_t* offsets;      // [E+1] compact
  const int32_t* poff;         // [E+1] padded
  const int32_t* perm_token;   // x source: token of each slot
  const int32_t* inv_perm;     // x source, optional: slot of each (token, j); then each
  int k;                       //   token is quantised once and written to its k slots
  const int32_t* slot_expert;  //   optional with it: expert of each (token, j) (top-k indices)
  const float* topk_w;         //   optional with it: weight of each (token, j); then
  float* w_perm;               //   w_perm[slot position] receives it
  PlanOut plan;                // per-slot x quantiser: also compute (and write) the tile plan
  int32_t* zero;               // optional: nzero counters set to 0 (by block 0, after the wait)
  int nzero;
  const uint16_t* x;           // [T][K] bf16
  const float* h32;            // or fp32 rows at padded positions
  const float* scale;          // static tensor scale or NULL
  const float* amax;           // dynamic: amax buffer
  uint8_t* codes;              // [padded rows][K/2 | K]
  uint8_t* sf;                 // blocked
  int32_t* status;
};

// The expert FFN as one persistent kernel (gate|up + SwiGLU + h quantisation,
// then down), for 64-token tiles: the CTAs take work items (every gate|up
// tile, then every down tile) from the counter `work` in increasing order; a
// down tile's token operand waits for the gate|up slices of its token tile,
// counted in tile_done.  The tile list comes from the offsets, or, when
// slot_expert is given, from the slots' expert ids: the top-k ids are then
// read before the wait on the previous kernel, so that kernel may be the one
// that writes the offsets.
struct FusedArgs {
  const int32_t* offsets;      // [E+1] compact (E <= 256)
  const int32_t* slot_expert;  // optional: [S] expert of each slot (flat top-k ids), all in [0, E)
  int64_t S;                   // slots: offsets[E]
  int64_t P;                   // padded rows allocated for x and h
  int32_t* tile_done;          // [max_tiles], zero on entry
  int32_t* work;               // item counter, zero on entry and set at least two launches before
                               // this kernel (it is read before the wait on the previous one)
  int static_items;            // 1: CTA b runs items b, b + grid, ... instead (for A/B measurement:
                               // it assumes every CTA is resident at once)
  int max_tiles;
  // Gather mode (small batches, at most kGatherMaxT slots per expert): the
  // gate|up token operand is copied row by row from the gather layout of x
  // (quant_token_gather), so nothing waits for a permutation.  The rows of
  // a tile are the slots of its expert in flat order; their tokens come from
  // perm_token (the grouped FFN) or, with slot_expert, from the slots
  // themselves (token = slot / k; the forward, which reads slot_expert only
  // after the wait on the previous kernel, the router).
  const uint8_t* xg;           // [T][8][K/2] codes, swizzled per row % 8
  const uint8_t* xsl;          // [T][K/(4 bs)][16] scale lines
  const int32_t* perm_token;   // [S] token of each slot position, or NULL
  int k;                       // slots per token (slot_expert mode)
  // the forward's combine in the down epilogue (slot_expert mode): out32
  // rows get topk_w[slot] * y (g2.out32 is set too); the CTA that finishes
  // last rounds them to bf16 into out
  const float* topk_w;
  uint16_t* out;
  int32_t* done;               // CTAs finished, zero on entry
  int64_t T;
};
constexpr int kFusedMaxE = 256;
cudaError_t launch_fused_ffn(const GemmArgs& g1, const GemmArgs& g2, const FusedArgs& f, const void* w13,
                             int64_t w13_rows, const void* w2, int64_t w2_rows, const void* xq, const void* hq,
                             int num_sms, cudaStream_t s);

// x of a small batch (T <= kGatherMaxT) into the gather layout the
// one-kernel FFN copies its token rows from (NVFP4 or MXFP4, K % 256 == 0).
cudaError_t launch_quant_gather(int fmt, const uint16_t* x, int64_t T, int K, const GatherQuant& q, cudaStream_t s);
cudaError_t launch_plan(const int32_t* offsets, int E, int64_t S, int bn, int32_t* poff, TileEntry* tiles,
                        int32_t* num_tiles, int max_tiles, int32_t* status, cudaStream_t s);
cudaError_t launch_quant_padded(const QuantPaddedArgs& a, bool src_x, int fmt, int num_sms, cudaStream_t s);
cudaError_t launch_grouped_gemm(const GemmArgs& g, int epi, int bn, const void* a_base, int64_t a_rows,
                                const void* b_base, int64_t b_rows, int num_sms, cudaStream_t s);
bool tensor_maps_available();
// The default bound of every device wait (about a second of SM clocks).
long long tc_default_wait_cycles();
// Early weight loads (MOE_OPT_EARLY_WEIGHTS): 0 off, 1 the ring's first pass,
// 2 also prefetch the next stages' weights to L2.
void set_early_weights(int mode);
int early_weights();
constexpr int kEarlyL2Stages = 16;
// CTA pairs (cta_group::2) for 192- and 256-token tiles whose weight rows
// divide by 256: 0 off, 1 on, 2 for long K loops only (the default).
void set_gemm_pairs(int mode);
// Router logits on the tensor cores, K split over ksplit partial outputs
// (logits_parts + s * part_stride, the bias in part 0; the top-k kernel adds
// them): E % 128 == 0, H % 64 == 0.  64-token tiles.
constexpr int kRouterBN = 64;
constexpr int kRouterMaxSplit = 4;
int router_ksplit(int64_t T, int E, int H, int num_sms);
// Router logits and top-k in one tcgen05 kernel (T >= 128; E a multiple of
// 16 up to 256; H % 64 == 0; k <= 16): 128 tokens per tile on the MMA's M
// side, every expert on its N side, the top-k kept per token in registers by
// the epilogue.  logits_out (nullable) receives the logits.
bool router_topk_fits(int64_t T, int E, int H, int k, int num_sms);
// Logits and top-k in one kernel, for batches whose 128-token tiles fill at
// least half the SMs (router_topk_fits).
cudaError_t launch_router_topk(const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias, int E,
                               int k, float* logits_out, int32_t* idx, float* w, int32_t* status, int num_sms,
                               cudaStream_t s);
cudaError_t launch_router_gemm(const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias, int E,
                               float* logits_parts, int64_t part_stride, int ksplit, int32_t* status, int num_sms,
                               cudaStream_t s);
}  // namespace moe
