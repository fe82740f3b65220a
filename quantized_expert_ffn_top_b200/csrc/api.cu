// C ABI of the B200 MoE layer (declared in include/moe_b200.h): argument
// checks on the host, workspace carving, path choice, and the launch
// sequence.  Every step of the layer runs in the kernels of this library.
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Sequential carving of the workspace (base == nullptr only measures).
struct Carver {
  char* base;
  size_t off;
  explicit Carver(void* b) : base(static_cast<char*>(b)), off(0) {}
  template <typename T>
  T* take(size_t count) {
    off = align_up(off, kAlign);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

struct Scalars {
  int32_t* status;
  float* x_amax;
  float* h_amax;
  float* sh_h_amax;
};

Scalars carve_head(Carver& c) {
  Scalars s;
  s.status = c.take<int32_t>(1);
  float* f = c.take<float>(8);
  s.x_amax = f;
  s.h_amax = f ? f + 1 : nullptr;
  s.sh_h_amax = f ? f + 2 : nullptr;
  return s;
}

int g_ffn_path = 0;  // MOE_OPT_FFN_PATH
static int g_fused_ffn = 1;  // MOE_OPT_FUSED_FFN
static int g_fused_combine = 0;  // MOE_OPT_FUSED_COMBINE
static int g_small_forward = 0;  // MOE_OPT_SMALL_BATCH_FORWARD
static int g_gather_x = 0;       // MOE_OPT_GATHER_X
static int g_router_topk = 1;    // MOE_OPT_ROUTER_TOPK
static int g_ffn_schedule = 0;   // MOE_OPT_FFN_SCHEDULE
static int g_perm_quant = 1;  // MOE_OPT_PERMUTE_QUANT

// Measurement hook (moe_set_stage_events).
cudaEvent_t g_stage_events[2 * MOE_STAGE_COUNT];
bool g_stage_on = false;
uint32_t g_stage_mask = 0;   // stages recorded since the hook was set

// External records, so that events captured into a CUDA graph stay readable
// by the caller after each replay.
void stage_mark(int stage, bool end, cudaStream_t s) {
  if (!g_stage_on) return;
  cudaEventRecordWithFlags(g_stage_events[2 * stage + (end ? 1 : 0)], s, cudaEventRecordExternal);
  g_stage_mask |= 1u << stage;
}

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = v > 0 ? v : 148;
  }
  return cached[dev];
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                          \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int block_size(int fmt) { return fmt == MOE_FMT_NVFP4 ? 16 : (fmt == MOE_FMT_MXFP4 ? 32 : 0); }
// bytes of one row of K weight or activation elements in a format
int64_t fmt_row_bytes(int fmt, int64_t K) {
  return fmt == MOE_FMT_FP8 ? K : (fmt == MOE_FMT_BF16 ? 2 * K : K / 2);
}

// Shape and pointer checks of a weight bank.
moe_status check_weights(const moe_weights* w, bool need_prepared) {
  if (!w) return MOE_ERR_INVALID_ARG;
  if (w->fmt != MOE_FMT_NVFP4 && w->fmt != MOE_FMT_MXFP4 && w->fmt != MOE_FMT_FP8 && w->fmt != MOE_FMT_BF16)
    return MOE_ERR_UNSUPPORTED;
  if (w->E < 1 || w->E > 1024 || w->H <= 0 || w->I <= 0) return MOE_ERR_INVALID_ARG;
  if (w->H % 128 != 0 || w->I % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (w->layout != MOE_LAYOUT_CANONICAL && w->layout != MOE_LAYOUT_PREPARED) return MOE_ERR_INVALID_ARG;
  if (need_prepared && w->layout != MOE_LAYOUT_PREPARED) return MOE_ERR_UNSUPPORTED;
  if (!w->w13 || !w->w2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->w13) || !aligned16(w->w2) || !aligned16(w->w13_sf) || !aligned16(w->w2_sf))
    return MOE_ERR_INVALID_ARG;
  if (block_size(w->fmt) && (!w->w13_sf || !w->w2_sf)) return MOE_ERR_INVALID_ARG;
  if ((w->fmt == MOE_FMT_NVFP4 || w->fmt == MOE_FMT_FP8) && (!w->w13_gs || !w->w2_gs)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// ---------------------------------------------------------------- layouts --
// Partial logits of the tensor-core router GEMM split along H: room for the
// largest split at every batch size, so that every scratch size below grows
// with T (a workspace sized for T serves every smaller batch).
constexpr int kRouterParts = kRouterMaxSplit;

// Router scratch: the (partial) logits.
struct RouteWs {
  Scalars head;
  float* parts;  // [nparts][T][E]
};
RouteWs carve_route(Carver& c, int64_t T, int E) {
  RouteWs r;
  r.head = carve_head(c);
  r.parts = c.take<float>((size_t)T * E * kRouterParts);
  return r;
}

struct PermWs {
  Scalars head;
  PermuteScratch scratch;
};
PermWs carve_perm(Carver& c, int64_t S, int E) {
  PermWs p;
  p.head = carve_head(c);
  p.scratch.nchunks = (int)((S + permute_chunk_slots() - 1) / permute_chunk_slots());
  p.scratch.chunk_counts = c.take<int32_t>((size_t)(p.scratch.nchunks > 0 ? p.scratch.nchunks : 1) * E);
  return p;
}

int g_gemm_bn = 0;  // token tile of the tensor-core path (MOE_OPT_GEMM_TILE_N); 0 = by batch size

int64_t padded_rows(int64_t S, int E) { return (int64_t)align_up((size_t)(S + (int64_t)E * 127), 128) + 256; }
// Tile list bound for the smallest token group (8 slots, the GEMV's MMA n).
int64_t max_tiles(int64_t S, int E) { return S / 8 + E + 1; }
// Bytes of the one-kernel FFN's counters (FfnScratch::counters).
size_t counters_bytes(int64_t S, int E) { return sizeof(int32_t) * (size_t)(4 + max_tiles(S, E)); }

// Scratch of the grouped FFN: GEMV path (h fp32 per compact slot) and tensor
// core path (padded, blocked quantised activations and the tile plan).
struct FfnScratch {
  float* h;          // GEMV: [S][I] fp32
  int32_t* poff;     // GEMM: [E+1] padded offsets
  TileEntry* tiles;  //       [max_tiles]
  int32_t* ntiles;
  uint8_t* xq;       //       [P][H/2 | H] codes of x in padded rows
  uint8_t* xsf;      //       [P * H/bs] blocked scales
  uint8_t* hq;       //       [P][I/2 | I]
  uint8_t* hsf;
  float* h32;        //       [P][I] fp32 h (dynamic h scale / FP8)
  // one-kernel FFN counters, cleared together: [0] the item counter, [1] CTAs
  // finished, [2] the decode router's ticket, [4 ..] gate|up slices finished
  // per token tile
  int32_t* counters;
  int32_t* work;
  int32_t* done;
  int32_t* ticket;
  int32_t* tile_done;  //     [max_tiles]
  float* w_perm;       //     [S] routing weight of each slot position (combine in the down epilogue)
  uint8_t* xg;         //     small batches: x in the gather layout, [min(S, 32)][8][H/2]
  uint8_t* xsl;        //     and its scale lines, [min(S, 32)][H / (4 bs)][16]
  int64_t P;
};
FfnScratch carve_ffn(Carver& c, int64_t S, const moe_weights* w) {
  FfnScratch f;
  const int bs = w->fmt == MOE_FMT_NVFP4 ? 16 : (w->fmt == MOE_FMT_MXFP4 ? 32 : 0);
  const int64_t rbh = fmt_row_bytes(w->fmt, w->H), rbi = fmt_row_bytes(w->fmt, w->I);
  f.P = padded_rows(S, w->E);
  f.h = c.take<float>((size_t)S * w->I);
  f.poff = c.take<int32_t>((size_t)w->E + 1);
  f.tiles = c.take<TileEntry>((size_t)max_tiles(S, w->E));
  f.ntiles = c.take<int32_t>(1);
  f.xq = c.take<uint8_t>((size_t)(f.P * rbh));
  f.xsf = bs ? c.take<uint8_t>((size_t)(f.P * (w->H / bs))) : nullptr;
  f.hq = c.take<uint8_t>((size_t)(f.P * rbi));
  f.hsf = bs ? c.take<uint8_t>((size_t)(f.P * (w->I / bs))) : nullptr;
  f.h32 = c.take<float>((size_t)(f.P * w->I));
  f.counters = c.take<int32_t>((size_t)(4 + max_tiles(S, w->E)));
  f.work = f.counters ? f.counters : nullptr;
  f.done = f.counters ? f.counters + 1 : nullptr;
  f.ticket = f.counters ? f.counters + 2 : nullptr;
  f.tile_done = f.counters ? f.counters + 4 : nullptr;
  f.w_perm = c.take<float>((size_t)S);
  // (T <= S: min(S, kGatherMaxT) rows cover every batch that gathers)
  const int64_t tg = S < kGatherMaxT ? S : kGatherMaxT;
  f.xg = bs ? c.take<uint8_t>((size_t)(tg * 8 * (w->H / 2))) : nullptr;
  f.xsl = bs ? c.take<uint8_t>((size_t)(tg * (w->H / (4 * bs)) * 16)) : nullptr;
  return f;
}

struct ForwardWs {
  Scalars head;
  float* logits;
  int32_t* idx;
  int32_t* idx_slot;   // forward through an expert cache: the top-k ids as slot ids
  float* w;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
  PermuteScratch pscratch;
  uint16_t* y_perm;
  float* out32;        // [T][H] fp32 output rows (combine in the down epilogue)
  FfnScratch ffn;
  int32_t* sh_offsets;
  int32_t* sh_perm;
  uint16_t* sh_y;
  FfnScratch sh_ffn;
};
ForwardWs carve_forward(Carver& c, int64_t T, int k, const moe_weights* routed, const moe_weights* shared) {
  ForwardWs f;
  const int E = routed->E;
  const int64_t S = T * k;
  f.head = carve_head(c);
  f.logits = c.take<float>((size_t)T * E * kRouterParts);
  f.idx = c.take<int32_t>((size_t)S);
  f.idx_slot = c.take<int32_t>((size_t)S);
  f.w = c.take<float>((size_t)S);
  f.offsets = c.take<int32_t>((size_t)E + 1);
  f.perm = c.take<int32_t>((size_t)S);
  f.inv = c.take<int32_t>((size_t)S);
  f.pscratch.nchunks = (int)((S + permute_chunk_slots() - 1) / permute_chunk_slots());
  f.pscratch.chunk_counts = c.take<int32_t>((size_t)(f.pscratch.nchunks > 0 ? f.pscratch.nchunks : 1) * E);
  f.y_perm = c.take<uint16_t>((size_t)S * routed->H);
  f.out32 = c.take<float>((size_t)T * routed->H);
  f.ffn = carve_ffn(c, S, routed);
  if (shared) {
    f.sh_offsets = c.take<int32_t>(2);
    f.sh_perm = c.take<int32_t>((size_t)T);
    f.sh_y = c.take<uint16_t>((size_t)T * routed->H);
    f.sh_ffn = carve_ffn(c, T, shared);
  } else {
    f.sh_offsets = f.sh_perm = nullptr;
    f.sh_y = nullptr;
    f.sh_ffn.h = nullptr;
  }
  return f;
}

// --------------------------------------------------------------- helpers --
__global__ void identity_routing_kernel(int64_t T, int32_t* offsets, int32_t* perm) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < T) perm[i] = (int32_t)i;
  if (i == 0) {
    offsets[0] = 0;
    offsets[1] = (int32_t)T;
  }
}

// Router logits into `parts`: *nparts partial sums T*E apart that the top-k
// kernel adds.  tcgen05 bf16 GEMM (split along H to fill the SMs) when the
// shapes allow it and the batch is large enough to matter, CUDA cores
// otherwise.
cudaError_t run_router(const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias, int E,
                       float* parts, int* nparts, int32_t* status, cudaStream_t s) {
  if (T >= 128 && E % 128 == 0 && H % 64 == 0 && tensor_maps_available()) {
    const int ks = router_ksplit(T, E, H, num_sms());   // at most kRouterParts
    *nparts = ks;
    return launch_router_gemm(x, T, H, wr, bias, E, parts, T * (int64_t)E, ks, status, num_sms(), s);
  }
  *nparts = 1;
  return launch_router_logits(x, T, H, wr, bias, E, parts, s);
}

// Logits and every token's top k.  Batches whose 128-token tiles fill at
// least half the SMs and whose E fits one MMA (E a multiple of 16 up to 256,
// k <= 16) take one kernel: the tensor cores with the top-k in their
// epilogue.  Otherwise the logits go to `parts` (the
// router GEMM's partial sums, or the CUDA-core sums) and topk_kernel picks.
// logits_out (nullable) receives the summed logits either way.
cudaError_t route_tokens(const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias, int E, int k,
                         float* parts, float* logits_out, int32_t* idx, float* w, int32_t* status, cudaStream_t s) {
  if (g_router_topk && router_topk_fits(T, E, H, k, num_sms()))
    return launch_router_topk(x, T, H, wr, bias, E, k, logits_out, idx, w, status, num_sms(), s);
  int nparts = 1;
  const cudaError_t e = run_router(x, T, H, wr, bias, E, parts, &nparts, status, s);
  if (e != cudaSuccess) return e;
  return launch_topk(parts, nparts, T * (int64_t)E, logits_out, T, E, k, idx, w, status, s);
}

bool gemm_shapes_ok(const moe_weights* w, int act) {
  // BF16 weights: bf16 activations in either mode
  if ((act != MOE_ACT_MATCH && w->fmt != MOE_FMT_BF16) || !tensor_maps_available()) return false;
  const int kb = w->fmt == MOE_FMT_FP8 ? 128 : (w->fmt == MOE_FMT_BF16 ? 64 : 256);
  return w->H % kb == 0 && w->I % kb == 0 && w->I % 64 == 0;
}

// Tensor cores whenever the activations are quantised and the shapes allow
// it; the weight-streaming GEMV for BF16 activations and other shapes.
bool use_gemm_path(const moe_weights* w, int64_t S, int act) {
  (void)S;
  if (g_ffn_path == 1 && w->fmt != MOE_FMT_BF16) return false;   // (no GEMV for BF16 weights)
  return gemm_shapes_ok(w, act);
}

// Token tile: 64 wide while the average expert holds fewer than 8 slots
// (decode: deep weight streaming, small B stages), 192 wide beyond (two
// accumulator buffers, so one tile's epilogue overlaps the next tile's MMAs;
// measured as fast as or faster than 256 up to the large prefill, with or
// without CTA pairs).  Arguments only, no device read-back.
int gemm_tile_n(int64_t S, int E) {
  if (g_gemm_bn) return g_gemm_bn;
  return S < 8 * (int64_t)E ? 64 : 192;
}

// The gate|up GEMM quantises h in its epilogue when h's scale needs no
// global reduction (MXFP4, or a static NVFP4 scale; BF16 h is not quantised).
bool h_in_epilogue(const moe_weights* w) {
  return w->fmt == MOE_FMT_MXFP4 || w->fmt == MOE_FMT_BF16 || (w->fmt == MOE_FMT_NVFP4 && w->a2_gs);
}

// Both projections as one kernel: block-scaled FP4 weights, h quantised in
// the epilogue, 64-token tiles, E <= 256.
bool ffn_one_kernel(const moe_weights* w, int64_t S) {
  return g_fused_ffn && h_in_epilogue(w) && (w->fmt == MOE_FMT_NVFP4 || w->fmt == MOE_FMT_MXFP4) &&
         gemm_tile_n(S, w->E) == 64 && w->E <= kFusedMaxE;
}

// The weighted combine in the down projection's epilogue
// (MOE_OPT_FUSED_COMBINE): the routed experts on the grouped GEMM (not the
// one-kernel FFN) behind the per-token x quantiser, which writes each slot's
// routing weight by position, and the shared expert, if any, on the grouped
// GEMM too.  Arguments only.
bool combine_in_down(const moe_weights* routed, const moe_weights* shared, int64_t T, int k, int act) {
  const int64_t S = T * k;
  if (!g_fused_combine || !use_gemm_path(routed, S, act) || ffn_one_kernel(routed, S)) return false;
  if (routed->fmt == MOE_FMT_BF16 || routed->H % 64 != 0) return false;
  if (shared && (!use_gemm_path(shared, T, act) || ffn_one_kernel(shared, T))) return false;
  return true;
}

// The GEMM arguments of the two projections: gate|up (+ SwiGLU, h in the
// epilogue when fused_h) over the quantised x rows, down over h.
void ffn_gemm_args(const moe_weights* w, const FfnScratch& f, int64_t S, float* x_amax, float* h_amax,
                   int32_t* status, bool fused_h, uint16_t* y_perm, GemmArgs& g, GemmArgs& d) {
  const int E = w->E, H = w->H, I = w->I;
  memset(&g, 0, sizeof(g));
  g.fmt = w->fmt;
  g.E = E;
  g.K = H;
  g.R = 2 * I;
  g.w_sf = w->w13_sf;
  g.b_sf = f.xsf;
  g.w_gs = w->w13_gs;
  g.act_scale = w->a13_gs;
  g.act_amax = x_amax;
  g.tiles = f.tiles;
  g.num_tiles = f.ntiles;
  g.I = I;
  g.hq = f.hq;
  g.hsf = f.hsf;
  g.h_scale = w->a2_gs;
  g.h32 = f.h32;
  g.h_amax = fused_h ? nullptr : h_amax;
  g.status = status;
  g.max_tiles = (int)max_tiles(S, E);
  g.wait_cycles = wait_cycles();
  memset(&d, 0, sizeof(d));
  d.fmt = w->fmt;
  d.E = E;
  d.K = I;
  d.R = H;
  d.w_sf = w->w2_sf;
  d.b_sf = f.hsf;
  d.w_gs = w->w2_gs;
  d.act_scale = w->a2_gs;
  d.act_amax = h_amax;
  d.tiles = f.tiles;
  d.num_tiles = f.ntiles;
  d.I = I;
  d.y = y_perm;
  d.ldy = H;
  d.y_rows = S;
  d.status = status;
  d.max_tiles = g.max_tiles;
  d.wait_cycles = g.wait_cycles;
}

// Small batches whose x goes to the gather layout (the one-kernel FFN copies
// its token rows from there, so no permutation is waited for).
bool gather_x(const moe_weights* w, int64_t T, int64_t S) {
  return g_gather_x && T <= kGatherMaxT && S <= kGatherMaxS && (w->fmt == MOE_FMT_NVFP4 || w->fmt == MOE_FMT_MXFP4) &&
         w->H % 256 == 0;
}

// x_ready: the permutation kernel has already quantised x into the padded
// rows (one_kernel only); the FFN then takes its tile list from the top-k ids
// (slot_expert).
moe_status run_gemm_ffn(const uint16_t* x, int64_t T, int64_t S, const int32_t* perm, const int32_t* offsets,
                        const int32_t* inv, int k, const int32_t* slot_expert, const moe_weights* w,
                        uint16_t* y_perm, const FfnScratch& f,
                        float* x_amax, float* h_amax, int32_t* status, cudaStream_t s, bool mark, bool planned,
                        bool x_ready, const float* topk_w, float* out32) {
  const int E = w->E, H = w->H, fmt = w->fmt;
  const int sms = num_sms();
  const int bn = gemm_tile_n(S, E);
  // gate|up projection + SwiGLU quantise h in the epilogue when its scale
  // needs no global reduction; with 64-token tiles the two projections then
  // run as one kernel
  const bool fused_h = h_in_epilogue(w);
  const bool one_kernel = ffn_one_kernel(w, S);
  // small batches on the one-kernel FFN: x in the gather layout
  const bool gather = one_kernel && !x_ready && gather_x(w, T, S);
  if (x_ready && (!one_kernel || !slot_expert || !planned)) return MOE_ERR_INVALID_ARG;
  if (out32 && one_kernel) return MOE_ERR_INVALID_ARG;
  if (out32 && topk_w && (!inv || fmt == MOE_FMT_BF16 || H % 64 != 0)) return MOE_ERR_INVALID_ARG;
  // (with x_ready the permutation kernel quantised x: no stage of its own)
  if (mark && !x_ready) stage_mark(MOE_STAGE_ACT_QUANT, false, s);
  // the x quantiser clears the one-kernel FFN's counters (with x_ready, the
  // permutation kernel did)
  const int ncounters = (int)(counters_bytes(S, E) / sizeof(int32_t));
  if (gather) {
    GatherQuant gq{w->a13_gs, x_amax, f.xg, f.xsl, one_kernel ? f.counters : nullptr, one_kernel ? ncounters : 0};
    MOE_TRY(launch_quant_gather(fmt, x, T, H, gq, s));
  } else {
    QuantPaddedArgs qa;
    memset(&qa, 0, sizeof(qa));
    qa.E = E;
    qa.K = H;
    qa.S = S;
    qa.T = T;
    qa.P = f.P;
    qa.offsets = offsets;
    qa.poff = f.poff;
    qa.perm_token = perm;
    qa.inv_perm = inv;
    qa.k = k;
    qa.slot_expert = slot_expert;
    // the combine in the down epilogue reads each slot's routing weight by
    // position; the token quantiser writes it on the way
    qa.topk_w = out32 ? topk_w : nullptr;
    qa.w_perm = out32 && topk_w ? f.w_perm : nullptr;
    if (!planned) {
      if (inv) {  // the token quantiser cannot write it
        MOE_TRY(launch_plan(offsets, E, S, bn, f.poff, f.tiles, f.ntiles, (int)max_tiles(S, E), status, s));
      } else {
        qa.plan.bn = bn;
        qa.plan.poff = f.poff;
        qa.plan.tiles = f.tiles;
        qa.plan.ntiles = f.ntiles;
        qa.plan.max_tiles = (int)max_tiles(S, E);
      }
    }
    qa.x = x;
    qa.scale = w->a13_gs;
    qa.amax = x_amax;
    qa.codes = f.xq;
    qa.sf = f.xsf;
    qa.status = status;
    qa.zero = one_kernel ? f.counters : nullptr;
    qa.nzero = one_kernel ? ncounters : 0;
    if (!x_ready) MOE_TRY(launch_quant_padded(qa, true, fmt, sms, s));
  }
  if (mark && !x_ready) stage_mark(MOE_STAGE_ACT_QUANT, true, s);
  GemmArgs g, d;
  ffn_gemm_args(w, f, S, x_amax, h_amax, status, fused_h, y_perm, g, d);
  // the tile list is two kernels back when the permutation or the plan kernel
  // wrote it; when the x quantiser just before writes it, the expert offsets
  // (older) name the experts of the early weight loads
  const int ew = early_weights();
  g.w_early = ew == 0 ? 0 : ((planned || inv) ? 1 : 2);
  g.w_early_l2 = ew == 2 ? kEarlyL2Stages : 0;
  g.offsets = offsets;
  d.w_early = ew == 0 ? 0 : 1;  // the tile list is at least two kernels back
  d.w_early_l2 = g.w_early_l2;
  d.out32 = out32;
  d.perm_token = perm;
  d.w_perm = out32 && topk_w ? f.w_perm : nullptr;
  d.out_rows = T;
  if (one_kernel) {
    // the weights are older than the quantiser: the first stages load before
    // the wait (the tile list comes from the offsets in the kernel)
    g.w_early = ew == 0 ? 0 : 1;
    FusedArgs fa;
    memset(&fa, 0, sizeof(fa));
    fa.offsets = offsets;
    fa.slot_expert = x_ready ? slot_expert : nullptr;   // the offsets are one kernel back then
    fa.S = S;
    fa.P = f.P;
    fa.tile_done = f.tile_done;
    fa.work = f.work;
    fa.static_items = g_ffn_schedule;
    fa.max_tiles = (int)max_tiles(S, E);
    if (gather) {
      fa.xg = f.xg;
      fa.xsl = f.xsl;
      fa.perm_token = perm;
      fa.k = k > 0 ? k : 1;
      fa.T = T;
    }
    if (mark) stage_mark(MOE_STAGE_FFN_UP, false, s);
    MOE_TRY(launch_fused_ffn(g, d, fa, w->w13, (int64_t)E * 2 * w->I, w->w2, (int64_t)E * H, f.xq, f.hq, sms, s));
    if (mark) stage_mark(MOE_STAGE_FFN_UP, true, s);   // both projections: no separate down stage
    return MOE_OK;
  }
  if (mark) stage_mark(MOE_STAGE_FFN_UP, false, s);
  if (!fused_h) MOE_TRY(cudaMemsetAsync(h_amax, 0, sizeof(float), s));
  MOE_TRY(launch_grouped_gemm(g, fused_h ? kEpiUpQuant : kEpiUpF32, bn, w->w13, (int64_t)E * 2 * w->I,
                              f.xq, f.P, sms, s));
  if (!fused_h) {
    QuantPaddedArgs qh;
    memset(&qh, 0, sizeof(qh));
    qh.E = E;
    qh.K = w->I;
    qh.S = S;
    qh.T = T;
    qh.P = f.P;
    qh.offsets = offsets;
    qh.poff = f.poff;
    qh.h32 = f.h32;
    qh.scale = w->a2_gs;
    qh.amax = h_amax;
    qh.codes = f.hq;
    qh.sf = f.hsf;
    qh.status = status;
    MOE_TRY(launch_quant_padded(qh, false, fmt, sms, s));
  }
  if (mark) stage_mark(MOE_STAGE_FFN_UP, true, s);
  if (mark) stage_mark(MOE_STAGE_FFN_DOWN, false, s);
  MOE_TRY(launch_grouped_gemm(d, kEpiDown, bn, w->w2, (int64_t)E * H, f.hq, f.P, sms, s));
  if (mark) stage_mark(MOE_STAGE_FFN_DOWN, true, s);
  return MOE_OK;
}

// Grouped FFN on already-validated arguments.  x_amax must hold amax(x) when
// the x scale is dynamic (MATCH, NVFP4/FP8, no a13_gs).
// inv (optional, with k = S / T) lets the tensor-core path quantise each
// token once for all its slots.
moe_status run_grouped_ffn(const uint16_t* x, int64_t T, int64_t S, const int32_t* perm, const int32_t* offsets,
                           const moe_weights* w, int act, uint16_t* y_perm, const FfnScratch& scratch,
                           float* x_amax, float* h_amax, int32_t* status, cudaStream_t s,
                           bool shared_stage = false, const int32_t* inv = nullptr, int k = 0,
                           const int32_t* slot_expert = nullptr, bool planned = false, bool x_ready = false,
                           const float* topk_w = nullptr, float* out32 = nullptr) {
  if (S == 0) return MOE_OK;
  const bool mark = !shared_stage;
  if (use_gemm_path(w, S, act))
    return run_gemm_ffn(x, T, S, perm, offsets, inv, k, slot_expert, w, y_perm, scratch, x_amax, h_amax, status, s,
                        mark, planned, x_ready, topk_w, out32);
  if (x_ready || out32) return MOE_ERR_INVALID_ARG;
  if (g_ffn_path == 2 || w->fmt == MOE_FMT_BF16) return MOE_ERR_UNSUPPORTED;   // the GEMV has no BF16 weights
  GemvArgs a;
  a.fmt = w->fmt;
  a.act = act;
  a.E = w->E;
  a.H = w->H;
  a.I = w->I;
  a.w13 = w->w13;
  a.w13_sf = w->w13_sf;
  a.w13_gs = w->w13_gs;
  a.w2 = w->w2;
  a.w2_sf = w->w2_sf;
  a.w2_gs = w->w2_gs;
  a.x_scale = w->a13_gs;
  a.h_scale = w->a2_gs;
  a.x = x;
  a.T = T;
  a.S = S;
  a.perm_token = perm;
  a.offsets = offsets;
  a.x_amax = x_amax;
  a.h_amax = (act == MOE_ACT_MATCH && w->fmt != MOE_FMT_MXFP4 && !w->a2_gs) ? h_amax : nullptr;
  a.h = scratch.h;
  a.y_perm = y_perm;
  a.tiles = scratch.tiles;
  a.num_tiles = scratch.ntiles;
  a.status = status;
  a.wait_cycles = wait_cycles();
  const int sms = num_sms();
  if (!planned)
    MOE_TRY(launch_plan(offsets, w->E, S, kGemvTokens, scratch.poff, scratch.tiles, scratch.ntiles,
                        (int)max_tiles(S, w->E), status, s));
  if (mark) stage_mark(MOE_STAGE_FFN_UP, false, s);
  MOE_TRY(launch_gemv_up(a, sms, s));
  if (mark) stage_mark(MOE_STAGE_FFN_UP, true, s);
  if (mark) stage_mark(MOE_STAGE_FFN_DOWN, false, s);
  MOE_TRY(launch_gemv_down(a, sms, s));
  if (mark) stage_mark(MOE_STAGE_FFN_DOWN, true, s);
  return MOE_OK;
}

// A side stream per device and a fork/join pair of events per call: work
// enqueued on `stream` after fork() depends on everything before it on the
// caller's stream, and the caller's stream waits for it at join().  Both are
// stream operations, so a graph capture of the caller's stream captures the
// fork and the join.  One side stream per device: concurrent forwards on one
// device serialise their shared experts (correctly, by their own events).
struct SideFork {
  cudaStream_t stream = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  bool forked = false;
  moe_status fork(cudaStream_t s) {
    static cudaStream_t side[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    {
      std::lock_guard<std::mutex> lk(mu);
      if (!side[dev] && cudaStreamCreateWithFlags(&side[dev], cudaStreamNonBlocking) != cudaSuccess)
        return MOE_ERR_CUDA;
      stream = side[dev];
    }
    if (cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaEventRecord(ev_fork, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamWaitEvent(stream, ev_fork, 0) != cudaSuccess) return MOE_ERR_CUDA;
    forked = true;
    return MOE_OK;
  }
  moe_status join(cudaStream_t s) {
    moe_status st = MOE_OK;
    if (forked) {
      if (cudaEventRecord(ev_join, stream) != cudaSuccess || cudaStreamWaitEvent(s, ev_join, 0) != cudaSuccess)
        st = MOE_ERR_CUDA;
      forked = false;
    }
    return st;
  }
  ~SideFork() {
    if (ev_fork) cudaEventDestroy(ev_fork);
    if (ev_join) cudaEventDestroy(ev_join);
  }
};

bool dynamic_x_scale(const moe_weights* w, int act) {
  return act == MOE_ACT_MATCH && (w->fmt == MOE_FMT_NVFP4 || w->fmt == MOE_FMT_FP8) && !w->a13_gs;
}

// Whether an activation's tensor scale is derived from the whole batch (x's
// with x scale a13, or h's), so that a token's result depends on the others.
bool batch_scaled(const moe_weights* w, const float* a13, int act) {
  return act == MOE_ACT_MATCH && (w->fmt == MOE_FMT_NVFP4 || w->fmt == MOE_FMT_FP8) && (!a13 || !w->a2_gs);
}

// The copy-in and copy-out streams of moe_forward_host, one pair per device.
moe_status copy_streams(cudaStream_t* in, cudaStream_t* out) {
  static cudaStream_t s_in[64], s_out[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(mu);
  if (!s_in[dev] && cudaStreamCreateWithFlags(&s_in[dev], cudaStreamNonBlocking) != cudaSuccess) return MOE_ERR_CUDA;
  if (!s_out[dev] && cudaStreamCreateWithFlags(&s_out[dev], cudaStreamNonBlocking) != cudaSuccess)
    return MOE_ERR_CUDA;
  *in = s_in[dev];
  *out = s_out[dev];
  return MOE_OK;
}

// Events of one moe_forward_host call, released when it returns (the driver
// frees a pending event's resources once it completes).
struct EventSet {
  cudaEvent_t ev[2 * MOE_MAX_HOST_SLICES + 3] = {};
  int n = 0;
  moe_status create(int count) {
    for (; n < count; ++n)
      if (cudaEventCreateWithFlags(&ev[n], cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  ~EventSet() {
    for (int i = 0; i < n; ++i) cudaEventDestroy(ev[i]);
  }
};

}  // namespace

static int g_pdl = 1;  // MOE_OPT_PDL
bool pdl_enabled() { return g_pdl != 0; }

static long long g_wait_cycles = tc_default_wait_cycles();  // MOE_OPT_WAIT_CYCLES
long long wait_cycles() { return g_wait_cycles; }

static uint64_t g_launches = 0;
static std::mutex g_launch_mu;
void count_launches(int n) {
  std::lock_guard<std::mutex> lk(g_launch_mu);
  g_launches += (uint64_t)n;
}
uint64_t launches_so_far() {
  std::lock_guard<std::mutex> lk(g_launch_mu);
  return g_launches;
}

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: unsupported format, layout or shape";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA launch or runtime error";
    case MOE_ERR_DEVICE_FAULT: return "MOE_ERR_DEVICE_FAULT: invalid data found on the device";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded device wait ran out";
  }
  return "unknown moe_status";
}

int32_t moe_version(void) { return 100; }

moe_status moe_set_option(int32_t option, int32_t value) {
  if (option == MOE_OPT_FFN_PATH) {
    if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
    g_ffn_path = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_GEMM_TILE_N) {
    if (value != 0 && value != 64 && value != 128 && value != 192 && value != 256) return MOE_ERR_INVALID_ARG;
    g_gemm_bn = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_PDL) {
    if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
    g_pdl = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_FUSED_FFN) {
    if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
    g_fused_ffn = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_PERMUTE_QUANT) {
    if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
    g_perm_quant = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_EARLY_WEIGHTS) {
    if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
    set_early_weights(value);
    return MOE_OK;
  }
  if (option == MOE_OPT_GATHER_X) {
    if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
    g_gather_x = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_ROUTER_TOPK) {
    if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
    g_router_topk = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_FFN_SCHEDULE) {
    if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
    g_ffn_schedule = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_SMALL_BATCH_FORWARD) {
    if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
    g_small_forward = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_FUSED_COMBINE) {
    if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
    g_fused_combine = value;
    return MOE_OK;
  }
  if (option == MOE_OPT_WAIT_CYCLES) {
    if (value < 0) return MOE_ERR_INVALID_ARG;
    g_wait_cycles = value == 0 ? tc_default_wait_cycles() : (long long)value;
    return MOE_OK;
  }
  if (option == MOE_OPT_GEMM_PAIR) {
    if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
    set_gemm_pairs(value);
    return MOE_OK;
  }
  return MOE_ERR_INVALID_ARG;
}

size_t moe_workspace_size(int64_t T, int32_t k, const moe_weights* routed, const moe_weights* shared, int32_t act) {
  if (T < 0 || k < 1 || check_weights(routed, false) != MOE_OK) return 0;
  if (shared && (check_weights(shared, false) != MOE_OK || shared->E != 1)) return 0;
  if (act != MOE_ACT_BF16 && act != MOE_ACT_MATCH) return 0;
  Carver c(nullptr);
  carve_forward(c, T, k, routed, shared);
  size_t need = c.off;
  Carver c2(nullptr);
  carve_head(c2);
  carve_ffn(c2, T * k, routed);
  need = need > c2.off ? need : c2.off;
  return align_up(need, kAlign);
}

size_t moe_prepared_weights_size(const moe_weights* w) {
  if (check_weights(w, false) != MOE_OK) return 0;
  const int64_t E = w->E, H = w->H, I = w->I;
  const int bs = block_size(w->fmt);
  const int64_t rb13 = fmt_row_bytes(w->fmt, H), rb2 = fmt_row_bytes(w->fmt, I);
  Carver c(nullptr);
  c.take<uint8_t>((size_t)(E * 2 * I * rb13));
  c.take<uint8_t>((size_t)(E * H * rb2));
  if (bs) {
    c.take<uint8_t>((size_t)(E * 2 * I * (H / bs)));
    c.take<uint8_t>((size_t)(E * H * (I / bs)));
  }
  return align_up(c.off, kAlign);
}

size_t moe_dequantized_weights_size(const moe_weights* w) {
  if (check_weights(w, false) != MOE_OK || w->fmt == MOE_FMT_BF16) return 0;
  Carver c(nullptr);
  c.take<uint16_t>((size_t)w->E * 2 * w->I * w->H);
  c.take<uint16_t>((size_t)w->E * w->H * w->I);
  return align_up(c.off, kAlign);
}

moe_status moe_dequantize_weights(const moe_weights* w, void* dst, size_t dst_bytes, moe_weights* out,
                                  moe_stream_t stream) {
  moe_status st = check_weights(w, false);
  if (st != MOE_OK) return st;
  if (w->fmt == MOE_FMT_BF16) return MOE_ERR_UNSUPPORTED;
  if (w->layout != MOE_LAYOUT_CANONICAL || !dst || !out) return MOE_ERR_INVALID_ARG;
  if (dst_bytes < moe_dequantized_weights_size(w)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t E = w->E, H = w->H, I = w->I;
  Carver c(dst);
  uint16_t* w13 = c.take<uint16_t>((size_t)(E * 2 * I * H));
  uint16_t* w2 = c.take<uint16_t>((size_t)(E * H * I));
  MOE_TRY(launch_dequant_bf16(w->fmt, w->w13, w->w13_sf, w->w13_gs, 2, I, E, 2 * I, H, w13, s));
  MOE_TRY(launch_dequant_bf16(w->fmt, w->w2, w->w2_sf, w->w2_gs, 1, H, E, H, I, w2, s));
  *out = *w;
  out->fmt = MOE_FMT_BF16;
  out->layout = MOE_LAYOUT_CANONICAL;
  out->w13 = reinterpret_cast<const uint8_t*>(w13);
  out->w2 = reinterpret_cast<const uint8_t*>(w2);
  out->w13_sf = out->w2_sf = nullptr;
  out->w13_gs = out->w2_gs = nullptr;
  out->a13_gs = out->a2_gs = nullptr;
  return MOE_OK;
}

moe_status moe_prepare_weights(const moe_weights* w, void* dst, size_t dst_bytes, moe_weights* prepared,
                               moe_stream_t stream) {
  moe_status st = check_weights(w, false);
  if (st != MOE_OK) return st;
  if (w->layout != MOE_LAYOUT_CANONICAL || !dst || !prepared) return MOE_ERR_INVALID_ARG;
  if (dst_bytes < moe_prepared_weights_size(w)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t E = w->E, H = w->H, I = w->I;
  const int bs = block_size(w->fmt);
  const int64_t rb13 = fmt_row_bytes(w->fmt, H), rb2 = fmt_row_bytes(w->fmt, I);
  Carver c(dst);
  uint8_t* w13 = c.take<uint8_t>((size_t)(E * 2 * I * rb13));
  uint8_t* w2 = c.take<uint8_t>((size_t)(E * H * rb2));
  uint8_t* sf13 = nullptr;
  uint8_t* sf2 = nullptr;
  if (bs) {
    sf13 = c.take<uint8_t>((size_t)(E * 2 * I * (H / bs)));
    sf2 = c.take<uint8_t>((size_t)(E * H * (I / bs)));
  }
  MOE_TRY(launch_prepare_rows(w->fmt, w->w13, w13, E, 2 * I, rb13, true, s));
  MOE_TRY(launch_prepare_rows(w->fmt, w->w2, w2, E, H, rb2, false, s));
  if (bs) {
    MOE_TRY(launch_prepare_sf(w->w13_sf, sf13, E, 2 * I, H / bs, H / bs, true, s));
    MOE_TRY(launch_prepare_sf(w->w2_sf, sf2, E, H, I / bs, I / bs, false, s));
  }
  *prepared = *w;
  prepared->layout = MOE_LAYOUT_PREPARED;
  prepared->w13 = w13;
  prepared->w2 = w2;
  prepared->w13_sf = sf13;
  prepared->w2_sf = sf2;
  return MOE_OK;
}

moe_status moe_quantize(int32_t fmt, const void* x, int32_t x_dtype, int64_t rows, int64_t K, const float* scale_in,
                        uint8_t* codes, uint8_t* sf, float* scale_out, void* ws, size_t ws_bytes,
                        moe_stream_t stream) {
  if (fmt != MOE_FMT_NVFP4 && fmt != MOE_FMT_MXFP4 && fmt != MOE_FMT_FP8 && fmt != MOE_FMT_BF16)
    return MOE_ERR_UNSUPPORTED;
  if (rows < 0 || K <= 0 || (x_dtype != 0 && x_dtype != 1)) return MOE_ERR_INVALID_ARG;
  const int bs = fmt == MOE_FMT_MXFP4 ? 32 : 16;
  if (K % bs != 0) return MOE_ERR_UNSUPPORTED;
  if (rows > 0 && (!x || !codes || (block_size(fmt) && !sf))) return MOE_ERR_INVALID_ARG;
  if (!aligned16(codes)) return MOE_ERR_INVALID_ARG;
  Carver c(ws);
  Scalars head = carve_head(c);
  if (!ws || ws_bytes < c.off) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (rows == 0) return MOE_OK;
  if ((fmt == MOE_FMT_NVFP4 || fmt == MOE_FMT_FP8) && !scale_in)
    MOE_TRY(launch_amax(x, x_dtype, rows * K, head.x_amax, num_sms(), s));
  return cuda_status(launch_quantize(fmt, x, x_dtype, rows, K, scale_in, head.x_amax, codes, sf, scale_out,
                                     num_sms(), s));
}

moe_status moe_route(const uint16_t* x, int64_t T, int32_t H, const uint16_t* wr, const float* bias, int32_t E,
                     int32_t k, float* logits, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                     moe_stream_t stream) {
  if (T < 0 || H <= 0 || H % 8 != 0 || E < 1 || E > 1024 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x || !wr || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(wr)) return MOE_ERR_INVALID_ARG;
  Carver c(ws);
  RouteWs r = carve_route(c, T, E);
  if (!ws || ws_bytes < c.off) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return cuda_status(route_tokens(x, T, H, wr, bias, E, k, r.parts, logits, topk_idx, topk_w, r.head.status, s));
}

moe_status moe_route_logits(const float* logits, int64_t T, int32_t E, int32_t k, int32_t* topk_idx, float* topk_w,
                            void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  Carver c(ws);
  Scalars head = carve_head(c);
  if (!ws || ws_bytes < c.off) return MOE_ERR_WORKSPACE;
  return cuda_status(launch_topk(logits, 1, 0, nullptr, T, E, k, topk_idx, topk_w, head.status,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E, int32_t* offsets,
                       int32_t* perm_token, int32_t* inv_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (T < 0 || k < 1 || E < 1 || E > 1024 || T * (int64_t)k > INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (!offsets || (T > 0 && (!topk_idx || !perm_token || !inv_perm))) return MOE_ERR_INVALID_ARG;
  Carver c(ws);
  PermWs p = carve_perm(c, T * k, E);
  if (!ws || ws_bytes < c.off) return MOE_ERR_WORKSPACE;
  return cuda_status(launch_permute(topk_idx, T * k, k, E, offsets, perm_token, inv_perm, p.scratch, p.head.status,
                                    reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr));
}

moe_status moe_grouped_ffn(const uint16_t* x, int64_t T, int32_t k, const int32_t* perm_token, const int32_t* offsets,
                           const moe_weights* w, int32_t act, uint16_t* y_perm, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
  moe_status st = check_weights(w, true);
  if (st != MOE_OK) return st;
  if (T < 0 || k < 1 || (act != MOE_ACT_BF16 && act != MOE_ACT_MATCH)) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x || !perm_token || !offsets || !y_perm)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y_perm)) return MOE_ERR_INVALID_ARG;
  const int64_t S = T * k;
  Carver c(ws);
  Scalars head = carve_head(c);
  FfnScratch f = carve_ffn(c, S, w);
  if (!ws || ws_bytes < c.off) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (S == 0) return MOE_OK;
  if (dynamic_x_scale(w, act)) {
    stage_mark(MOE_STAGE_ACT_QUANT, false, s);
    MOE_TRY(launch_amax(x, 1, T * w->H, head.x_amax, num_sms(), s));
    stage_mark(MOE_STAGE_ACT_QUANT, true, s);
  }
  return run_grouped_ffn(x, T, S, perm_token, offsets, w, act, y_perm, f, head.x_amax, head.h_amax, head.status, s);
}

moe_status moe_combine(const uint16_t* y_perm, const int32_t* inv_perm, const float* topk_w, int64_t T, int32_t k,
                       int32_t H, const uint16_t* shared_y, uint16_t* out, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  if (T < 0 || k < 1 || k > 1024 || H <= 0 || H % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!y_perm || !inv_perm || !topk_w || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(out) || !aligned16(shared_y)) return MOE_ERR_INVALID_ARG;
  Carver c(ws);
  Scalars head = carve_head(c);
  if (!ws || ws_bytes < c.off) return MOE_ERR_WORKSPACE;
  return cuda_status(launch_combine(y_perm, inv_perm, topk_w, T, k, H, shared_y, out, head.status,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_forward(const uint16_t* x, int64_t T, const uint16_t* wr, const float* bias, int32_t k,
                       const moe_weights* routed, const moe_weights* shared, int32_t act, uint16_t* out, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_weights(routed, true);
  if (st != MOE_OK) return st;
  if (shared) {
    st = check_weights(shared, true);
    if (st != MOE_OK) return st;
    if (shared->E != 1 || shared->H != routed->H || shared->fmt != routed->fmt) return MOE_ERR_INVALID_ARG;
  }
  const int E = routed->E, H = routed->H;
  if (T < 0 || k < 1 || k > E || (act != MOE_ACT_BF16 && act != MOE_ACT_MATCH)) return MOE_ERR_INVALID_ARG;
  if (T * (int64_t)k > INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x || !wr || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(wr) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  Carver c(ws);
  ForwardWs f = carve_forward(c, T, k, routed, shared);
  if (!ws || ws_bytes < c.off) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t S = T * k;
  // Small batches on the one-kernel FFN with no shared expert: two kernels.
  // The router computes the logits, quantises x into the gather layout and
  // picks every token's top k in its last block; the FFN takes its tiles from
  // the top-k ids (a tile's rows are its expert's slots in flat order, so no
  // permutation is needed), copies the token rows from the gather layout,
  // adds w * y into fp32 output rows in its down epilogue, and its last CTA
  // rounds them into `out`.
  const bool small2 = g_small_forward && !shared && act == MOE_ACT_MATCH && use_gemm_path(routed, S, act) &&
                      ffn_one_kernel(routed, S) && gather_x(routed, T, S) && H % 8 == 0;
  if (small2) {
    MOE_TRY(cudaMemsetAsync(f.ffn.counters, 0, counters_bytes(S, E), s));
    MOE_TRY(cudaMemsetAsync(f.out32, 0, sizeof(float) * (size_t)T * H, s));
    if (dynamic_x_scale(routed, act)) {
      stage_mark(MOE_STAGE_ACT_QUANT, false, s);
      MOE_TRY(launch_amax(x, 1, T * H, f.head.x_amax, num_sms(), s));
      stage_mark(MOE_STAGE_ACT_QUANT, true, s);
    }
    stage_mark(MOE_STAGE_ROUTE, false, s);
    const GatherQuant gq{routed->a13_gs, f.head.x_amax, f.ffn.xg, f.ffn.xsl};
    MOE_TRY(launch_router_decode(routed->fmt, x, T, H, wr, bias, E, k, f.logits, f.idx, f.w, f.ffn.ticket, gq,
                                 f.head.status, s));
    stage_mark(MOE_STAGE_ROUTE, true, s);
    GemmArgs g, d;
    ffn_gemm_args(routed, f.ffn, S, f.head.x_amax, f.head.h_amax, f.head.status, true, f.y_perm, g, d);
    g.w_early = early_weights() == 0 ? 0 : 1;
    d.w_early = g.w_early;
    d.out32 = f.out32;
    d.out_rows = T;
    FusedArgs fa;
    memset(&fa, 0, sizeof(fa));
    fa.offsets = f.offsets;
    fa.slot_expert = f.idx;
    fa.S = S;
    fa.P = f.ffn.P;
    fa.tile_done = f.ffn.tile_done;
    fa.work = f.ffn.work;
    fa.static_items = g_ffn_schedule;
    fa.max_tiles = (int)max_tiles(S, E);
    fa.xg = f.ffn.xg;
    fa.xsl = f.ffn.xsl;
    fa.k = k;
    fa.topk_w = f.w;
    fa.out = out;
    fa.done = f.ffn.done;
    fa.T = T;
    stage_mark(MOE_STAGE_FFN_UP, false, s);
    MOE_TRY(launch_fused_ffn(g, d, fa, routed->w13, (int64_t)E * 2 * routed->I, routed->w2, (int64_t)E * H,
                             f.ffn.xq, f.ffn.hq, num_sms(), s));
    stage_mark(MOE_STAGE_FFN_UP, true, s);
    return MOE_OK;
  }
  // Small batches on the one-kernel FFN: the one-block permutation also
  // quantises x, and the FFN takes its tile list from the top-k ids (two
  // kernels back), so its first weight loads go out while the permutation
  // runs.  The FFN's item counter is cleared here, before the router.
  const bool want_q = g_perm_quant && act == MOE_ACT_MATCH && use_gemm_path(routed, S, act) &&
                      ffn_one_kernel(routed, S) && H % 64 == 0 && permute_can_quantize(S, T, E);
  // The weighted combine in the down epilogues (routed and shared experts
  // add into fp32 rows, cleared here, before the fork), then one rounding pass.
  const bool fused_combine = combine_in_down(routed, shared, T, k, act);
  if (fused_combine) MOE_TRY(cudaMemsetAsync(f.out32, 0, sizeof(float) * (size_t)T * H, s));
  // 1. dynamic activation scale of x (shared by routed and shared experts)
  if (dynamic_x_scale(routed, act)) {
    stage_mark(MOE_STAGE_ACT_QUANT, false, s);
    MOE_TRY(launch_amax(x, 1, T * H, f.head.x_amax, num_sms(), s));
    stage_mark(MOE_STAGE_ACT_QUANT, true, s);
  }
  // 2. shared expert: every token, identity order, on a side stream forked
  // here and joined before the combine, so it overlaps routing and the
  // permutation; it reads the routed layer's x scale
  SideFork side;
  if (shared) {
    st = side.fork(s);
    if (st != MOE_OK) return st;
    cudaStream_t s2 = side.stream;
    stage_mark(MOE_STAGE_SHARED, false, s2);
    cudaError_t le = launch_pdl(identity_routing_kernel, dim3((unsigned)((T + 255) / 256)), dim3(256), 0, s2, T,
                                f.sh_offsets, f.sh_perm);
    count_launches(1);
    if (le == cudaSuccess) le = cudaGetLastError();
    st = le != cudaSuccess ? MOE_ERR_CUDA : MOE_OK;
    if (st == MOE_OK) {
      moe_weights sh = *shared;
      sh.a13_gs = routed->a13_gs;
      st = run_grouped_ffn(x, T, T, f.sh_perm, f.sh_offsets, &sh, act, f.sh_y, f.sh_ffn, f.head.x_amax,
                           f.head.sh_h_amax, f.head.status, s2, true, nullptr, 0, nullptr, false, false, nullptr,
                           fused_combine ? f.out32 : nullptr);
    }
    stage_mark(MOE_STAGE_SHARED, true, s2);
    if (st != MOE_OK) {
      side.join(s);
      return st;
    }
  }
  // 3. router
  stage_mark(MOE_STAGE_ROUTE, false, s);
  st = cuda_status(route_tokens(x, T, H, wr, bias, E, k, f.logits, nullptr, f.idx, f.w, f.head.status, s));
  stage_mark(MOE_STAGE_ROUTE, true, s);
  // 4. histogram + permutation; it also writes the routed FFN's tile plan
  PlanOut plan;
  plan.bn = use_gemm_path(routed, S, act) ? gemm_tile_n(S, E) : kGemvTokens;
  plan.poff = f.ffn.poff;
  plan.tiles = f.ffn.tiles;
  plan.ntiles = f.ffn.ntiles;
  plan.max_tiles = (int)max_tiles(S, E);
  SlotQuantOut q;
  memset(&q, 0, sizeof(q));
  if (want_q) {
    q.fmt = routed->fmt;
    q.x = x;
    q.K = H;
    q.P = f.ffn.P;
    q.scale = routed->a13_gs;
    q.amax = f.head.x_amax;
    q.codes = f.ffn.xq;
    q.sf = f.ffn.xsf;
    q.zero = f.ffn.counters;   // the one-kernel FFN's counters, cleared on the way
    q.nzero = (int)(counters_bytes(S, E) / sizeof(int32_t));
  }
  bool planned = false, x_ready = false;
  if (st == MOE_OK) {
    stage_mark(MOE_STAGE_PERMUTE, false, s);
    st = cuda_status(launch_permute(f.idx, S, k, E, f.offsets, f.perm, f.inv, f.pscratch, f.head.status, s, &plan,
                                    &planned, want_q ? &q : nullptr, &x_ready));
    stage_mark(MOE_STAGE_PERMUTE, true, s);
  }
  // 5. routed experts
  if (st == MOE_OK)
    st = run_grouped_ffn(x, T, S, f.perm, f.offsets, routed, act, f.y_perm, f.ffn, f.head.x_amax, f.head.h_amax,
                         f.head.status, s, false, f.inv, k, f.idx, planned, x_ready, f.w,
                         fused_combine ? f.out32 : nullptr);
  if (shared) {
    const moe_status js = side.join(s);
    if (st == MOE_OK) st = js;
  }
  if (st != MOE_OK) return st;
  // 6. combine (or, when the down epilogues did it, the rounding to bf16)
  stage_mark(MOE_STAGE_COMBINE, false, s);
  if (fused_combine)
    st = cuda_status(launch_round_rows(f.out32, T * (int64_t)H, out, f.head.status, num_sms(), s));
  else
    st = cuda_status(launch_combine(f.y_perm, f.inv, f.w, T, k, H, f.sh_y, out, f.head.status, s));
  stage_mark(MOE_STAGE_COMBINE, true, s);
  return st;
}

moe_status moe_forward_host(const uint16_t* x_host, int64_t T, const uint16_t* wr, const float* bias, int32_t k,
                            const moe_weights* routed, const moe_weights* shared, int32_t act, uint16_t* out_host,
                            uint16_t* x_dev, uint16_t* out_dev, int32_t n_slices, void* ws, size_t ws_bytes,
                            moe_stream_t stream) {
  moe_status st = check_weights(routed, true);
  if (st != MOE_OK) return st;
  if (shared) {
    st = check_weights(shared, true);
    if (st != MOE_OK) return st;
    if (shared->E != 1 || shared->H != routed->H || shared->fmt != routed->fmt) return MOE_ERR_INVALID_ARG;
  }
  const int64_t H = routed->H;
  if (T < 0 || k < 1 || k > routed->E || (act != MOE_ACT_BF16 && act != MOE_ACT_MATCH)) return MOE_ERR_INVALID_ARG;
  if (T * (int64_t)k > INT32_MAX || n_slices < 1 || n_slices > MOE_MAX_HOST_SLICES) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x_host || !out_host || !x_dev || !out_dev || !wr)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_dev) || !aligned16(out_dev) || !aligned16(wr) || (H * 2) % 16 != 0) return MOE_ERR_INVALID_ARG;
  // one slice when a tensor scale depends on the whole batch
  int64_t n = n_slices;
  if (batch_scaled(routed, routed->a13_gs, act) || (shared && batch_scaled(shared, routed->a13_gs, act))) n = 1;
  if (n > T) n = T > 0 ? T : 1;
  const int64_t Ts = T > 0 ? (T + n - 1) / n : 0;  // tokens per slice (the last may have fewer)
  n = T > 0 ? (T + Ts - 1) / Ts : 0;
  Carver c(nullptr);
  carve_forward(c, Ts, k, routed, shared);
  if (!ws || ws_bytes < c.off) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream), s_in = nullptr, s_out = nullptr;
  st = copy_streams(&s_in, &s_out);
  if (st != MOE_OK) return st;
  EventSet es;
  st = es.create((int)(2 * n + 3));
  if (st != MOE_OK) return st;
  cudaEvent_t ev_start = es.ev[0], ev_end = es.ev[1], ev_in_end = es.ev[2];
  cudaEvent_t* in_done = es.ev + 3;
  cudaEvent_t* fwd_done = es.ev + 3 + n;
  const size_t row = (size_t)H * sizeof(uint16_t);
  // the copy streams start after the work already on the caller's stream
  if (cudaEventRecord(ev_start, s) != cudaSuccess || cudaStreamWaitEvent(s_in, ev_start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(s_out, ev_start, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  // every slice's copy-in, back to back on the copy-in stream
  for (int64_t i = 0; i < n && st == MOE_OK; ++i) {
    const int64_t t0 = i * Ts, Ti = (T - t0) < Ts ? (T - t0) : Ts;
    if (cudaMemcpyAsync(x_dev + t0 * H, x_host + t0 * H, (size_t)Ti * row, cudaMemcpyHostToDevice, s_in) !=
            cudaSuccess ||
        cudaEventRecord(in_done[i], s_in) != cudaSuccess)
      st = MOE_ERR_CUDA;
  }
  // forwards on the caller's stream, each after its slice arrived; each
  // slice's copy-out after its forward
  for (int64_t i = 0; i < n && st == MOE_OK; ++i) {
    const int64_t t0 = i * Ts, Ti = (T - t0) < Ts ? (T - t0) : Ts;
    if (cudaStreamWaitEvent(s, in_done[i], 0) != cudaSuccess) {
      st = MOE_ERR_CUDA;
      break;
    }
    st = moe_forward(x_dev + t0 * H, Ti, wr, bias, k, routed, shared, act, out_dev + t0 * H, ws, ws_bytes, stream);
    if (st != MOE_OK) break;
    if (cudaEventRecord(fwd_done[i], s) != cudaSuccess || cudaStreamWaitEvent(s_out, fwd_done[i], 0) != cudaSuccess ||
        cudaMemcpyAsync(out_host + t0 * H, out_dev + t0 * H, (size_t)Ti * row, cudaMemcpyDeviceToHost, s_out) !=
            cudaSuccess)
      st = MOE_ERR_CUDA;
  }
  // the caller's stream waits for the last copy-in and the last copy-out
  // (also after an error, so that no copy of this call is left unordered
  // against later work on `stream`, and a capture of `stream` joins both
  // copy streams)
  const bool joined = cudaEventRecord(ev_in_end, s_in) == cudaSuccess &&
                      cudaEventRecord(ev_end, s_out) == cudaSuccess &&
                      cudaStreamWaitEvent(s, ev_in_end, 0) == cudaSuccess &&
                      cudaStreamWaitEvent(s, ev_end, 0) == cudaSuccess;
  if (st == MOE_OK && !joined) st = MOE_ERR_CUDA;
  return st;
}

size_t moe_expert_cache_bytes(const moe_weights* bank, int32_t n_slots) {
  if (check_weights(bank, true) != MOE_OK || n_slots < 1 || n_slots > bank->E || n_slots > 1024) return 0;
  moe_weights one = *bank;
  one.E = n_slots;
  one.layout = MOE_LAYOUT_CANONICAL;
  const size_t pool = moe_prepared_weights_size(&one);
  Carver c(nullptr);
  c.take<uint8_t>(pool);
  c.take<float>((size_t)n_slots * 2);
  c.take<float>((size_t)n_slots);
  c.take<int32_t>(cache_state_words(bank->E, n_slots));
  return align_up(c.off, kAlign);
}

moe_status moe_expert_cache_init(const moe_weights* bank, int32_t n_slots, void* dev, size_t dev_bytes,
                                 moe_expert_cache* cache, moe_stream_t stream) {
  moe_status st = check_weights(bank, true);
  if (st != MOE_OK) return st;
  if (!cache || !dev || n_slots < 1 || n_slots > bank->E || n_slots > 1024) return MOE_ERR_INVALID_ARG;
  if (dev_bytes < moe_expert_cache_bytes(bank, n_slots)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  moe_expert_cache cc;
  memset(&cc, 0, sizeof(cc));
  cc.bank = *bank;
  cc.n_slots = n_slots;
  // device addresses of the host arrays (they must be mapped)
  const void* host[6] = {bank->w13, bank->w13_sf, bank->w13_gs, bank->w2, bank->w2_sf, bank->w2_gs};
  for (int i = 0; i < 6; ++i) {
    if (!host[i]) continue;
    void* d = nullptr;
    if (cudaHostGetDevicePointer(&d, const_cast<void*>(host[i]), 0) != cudaSuccess || !d) {
      cudaGetLastError();   // clear the error this query leaves behind
      return MOE_ERR_INVALID_ARG;
    }
    cc.bank_dev[i] = d;
  }
  // the pool: a PREPARED bank of n_slots experts, then its part scales and the state
  const int64_t n = n_slots, H = bank->H, I = bank->I;
  const int bs = block_size(bank->fmt);
  const int64_t rb13 = fmt_row_bytes(bank->fmt, H), rb2 = fmt_row_bytes(bank->fmt, I);
  Carver c(dev);
  uint8_t* w13 = c.take<uint8_t>((size_t)(n * 2 * I * rb13));
  uint8_t* w2 = c.take<uint8_t>((size_t)(n * H * rb2));
  uint8_t* sf13 = bs ? c.take<uint8_t>((size_t)(n * 2 * I * (H / bs))) : nullptr;
  uint8_t* sf2 = bs ? c.take<uint8_t>((size_t)(n * H * (I / bs))) : nullptr;
  float* gs13 = c.take<float>((size_t)n * 2);
  float* gs2 = c.take<float>((size_t)n);
  int32_t* state = c.take<int32_t>(cache_state_words(bank->E, n_slots));
  cc.pool = *bank;
  cc.pool.E = n_slots;
  cc.pool.w13 = w13;
  cc.pool.w2 = w2;
  cc.pool.w13_sf = sf13;
  cc.pool.w2_sf = sf2;
  cc.pool.w13_gs = bank->w13_gs ? gs13 : nullptr;
  cc.pool.w2_gs = bank->w2_gs ? gs2 : nullptr;
  cc.state = state;
  // empty pool: clock and counters 0, slot_of / expert_of -1, stamps 0
  const size_t words = cache_state_words(bank->E, n_slots);
  MOE_TRY(cudaMemsetAsync(state, 0, words * sizeof(int32_t), s));
  MOE_TRY(cudaMemsetAsync(state + 4, 0xFF, ((size_t)bank->E + n_slots) * sizeof(int32_t), s));
  *cache = cc;
  return MOE_OK;
}

moe_status moe_forward_cached(const uint16_t* x, int64_t T, const uint16_t* wr, const float* bias, int32_t k,
                              const moe_expert_cache* cache, int32_t act, uint16_t* out, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
  if (!cache) return MOE_ERR_INVALID_ARG;
  moe_status st = check_weights(&cache->bank, true);
  if (st != MOE_OK) return st;
  st = check_weights(&cache->pool, true);
  if (st != MOE_OK) return st;
  const moe_weights* bank = &cache->bank;
  const moe_weights* pool = &cache->pool;
  const int E = bank->E, H = bank->H, n = cache->n_slots;
  if (T < 0 || k < 1 || k > E || (act != MOE_ACT_BF16 && act != MOE_ACT_MATCH)) return MOE_ERR_INVALID_ARG;
  if (T * (int64_t)k > INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x || !wr || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(wr) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  const int64_t S = T * k;
  if ((int64_t)n < (S < E ? S : E)) return MOE_ERR_INVALID_ARG;   // a batch must fit in the pool
  Carver c(ws);
  ForwardWs f = carve_forward(c, T, k, bank, nullptr);
  if (!ws || ws_bytes < c.off) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dynamic_x_scale(pool, act)) MOE_TRY(launch_amax(x, 1, T * H, f.head.x_amax, num_sms(), s));
  // route on the whole bank's router
  stage_mark(MOE_STAGE_ROUTE, false, s);
  MOE_TRY(route_tokens(x, T, H, wr, bias, E, k, f.logits, nullptr, f.idx, f.w, f.head.status, s));
  stage_mark(MOE_STAGE_ROUTE, true, s);
  // admit the batch's experts into slots and fetch the missing ones
  MOE_TRY(launch_cache_admit(f.idx, S, E, n, cache->state, f.idx_slot, f.head.status, s));
  CacheCopy cc;
  memset(&cc, 0, sizeof(cc));
  const int64_t I = bank->I;
  const int bs = block_size(bank->fmt);
  const int64_t rb13 = fmt_row_bytes(bank->fmt, H), rb2 = fmt_row_bytes(bank->fmt, I);
  cc.src[0] = static_cast<const uint8_t*>(cache->bank_dev[0]);
  cc.dst[0] = const_cast<uint8_t*>(pool->w13);
  cc.bytes[0] = 2 * I * rb13;
  cc.src[1] = static_cast<const uint8_t*>(cache->bank_dev[3]);
  cc.dst[1] = const_cast<uint8_t*>(pool->w2);
  cc.bytes[1] = H * rb2;
  cc.nregions = 2;
  if (bs) {
    cc.src[2] = static_cast<const uint8_t*>(cache->bank_dev[1]);
    cc.dst[2] = const_cast<uint8_t*>(pool->w13_sf);
    cc.bytes[2] = 2 * I * (H / bs);
    cc.src[3] = static_cast<const uint8_t*>(cache->bank_dev[4]);
    cc.dst[3] = const_cast<uint8_t*>(pool->w2_sf);
    cc.bytes[3] = H * (I / bs);
    cc.nregions = 4;
  }
  if (bank->w13_gs) {
    cc.gs_src[0] = static_cast<const float*>(cache->bank_dev[2]);
    cc.gs_dst[0] = const_cast<float*>(pool->w13_gs);
    cc.gs_per[0] = 2;
    cc.gs_src[1] = static_cast<const float*>(cache->bank_dev[5]);
    cc.gs_dst[1] = const_cast<float*>(pool->w2_gs);
    cc.gs_per[1] = 1;
    cc.ngs = 2;
  }
  MOE_TRY(launch_cache_fetch(cache->state, E, n, cc, num_sms(), s));
  // the layer on the pool: slot ids are the experts now
  stage_mark(MOE_STAGE_PERMUTE, false, s);
  PlanOut plan;
  plan.bn = use_gemm_path(pool, S, act) ? gemm_tile_n(S, n) : kGemvTokens;
  plan.poff = f.ffn.poff;
  plan.tiles = f.ffn.tiles;
  plan.ntiles = f.ffn.ntiles;
  plan.max_tiles = (int)max_tiles(S, n);
  bool planned = false;
  MOE_TRY(launch_permute(f.idx_slot, S, k, n, f.offsets, f.perm, f.inv, f.pscratch, f.head.status, s, &plan,
                         &planned));
  stage_mark(MOE_STAGE_PERMUTE, true, s);
  st = run_grouped_ffn(x, T, S, f.perm, f.offsets, pool, act, f.y_perm, f.ffn, f.head.x_amax, f.head.h_amax,
                       f.head.status, s, false, f.inv, k, f.idx_slot, planned, false);
  if (st != MOE_OK) return st;
  stage_mark(MOE_STAGE_COMBINE, false, s);
  st = cuda_status(launch_combine(f.y_perm, f.inv, f.w, T, k, H, nullptr, out, f.head.status, s));
  stage_mark(MOE_STAGE_COMBINE, true, s);
  return st;
}

moe_status moe_expert_cache_stats(const moe_expert_cache* cache, moe_stream_t stream, int64_t* stats) {
  if (!cache || !cache->state || !stats) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t h[4] = {0, 0, 0, 0};
  if (cudaMemcpyAsync(h, cache->state, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  for (int i = 0; i < 4; ++i) stats[i] = h[i];
  return MOE_OK;
}

moe_status moe_set_stage_events(void* const* events, int32_t n_events) {
  if (!events) {
    g_stage_on = false;   // the mask keeps what the hook recorded
    return MOE_OK;
  }
  g_stage_mask = 0;
  if (n_events < 2 * MOE_STAGE_COUNT) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 2 * MOE_STAGE_COUNT; ++i) {
    if (!events[i]) return MOE_ERR_INVALID_ARG;
    g_stage_events[i] = reinterpret_cast<cudaEvent_t>(events[i]);
  }
  g_stage_on = true;
  return MOE_OK;
}

uint32_t moe_stage_mask(void) { return g_stage_mask; }

uint64_t moe_kernel_launch_count(void) { return launches_so_far(); }

moe_status moe_get_device_status(void* ws, moe_stream_t stream, int32_t* host_status) {
  if (!ws || !host_status) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  *host_status = v;
  return MOE_OK;
}

}  // extern "C"
