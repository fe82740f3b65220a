/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) routed MoE expert FFN layer.
 *
 * The layer is the forward pass of a routed Mixture-of-Experts block as the
 * FreeToken engine serves it (FreeToken upstream README, "About": MoE serving
 * over MXFP4 / NVFP4 / FP8 / BF16 checkpoints):
 *
 *   logits = x Wr^T (+ b)                                    moe_route
 *   idx, w = top-k of softmax(logits), renormalised          moe_route(_logits)
 *   counts, offsets, stable permutation of the T*k slots     moe_permute
 *   y_p    = SwiGLU expert FFN of x[perm_token[p]] over the
 *            quantised weights of the slot's expert          moe_grouped_ffn
 *   out_t  = sum_j w[t,j] y_{inv_perm[t*k+j]} (+ shared_t)    moe_combine
 *   all of the above, enqueued as one call                   moe_forward
 *   the same from host buffers, copies overlapped            moe_forward_host
 *
 * Conventions shared by every entry point
 *  - Pointers marked (device) are CUDA device pointers; (host) are host
 *    pointers.  The caller owns every buffer.  No call allocates device
 *    memory: scratch space comes from the caller's workspace `ws` of
 *    `ws_bytes` bytes, sized by moe_workspace_size().
 *  - bf16 tensors are passed as uint16_t bit patterns; all tensors are
 *    row-major and contiguous.
 *  - Calls are asynchronous on `stream` (never the legacy default stream
 *    implicitly), perform no host synchronisation (except
 *    moe_get_device_status) and are safe to capture in a CUDA graph once the
 *    weights are prepared.
 *  - Argument errors are detected on the host before anything is enqueued and
 *    return MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED; outputs are then left
 *    untouched.  An unknown format is MOE_ERR_UNSUPPORTED, never a silent
 *    success with uninitialised output (the failure mode the
 *    atomicmilkshake/FreeToken fork README describes under "What else
 *    changed" for a kernel switch without a default).
 *  - Faults found on the device (an expert index out of range, a NaN or
 *    all -inf logit row) set a status word inside `ws`; the affected outputs
 *    are written with zeros (or the slot is dropped), never left
 *    uninitialised.  A bounded device wait that ran out (MOE_OPT_WAIT_CYCLES)
 *    sets the word to MOE_ERR_TIMEOUT: the kernel that gave up lets its
 *    copies in flight land, frees its tensor memory and returns, and the
 *    later kernels of the call still run.  The layer's output (moe_forward,
 *    moe_forward_host, moe_forward_cached, moe_combine) is then written as
 *    zeros -- the combine reads the word -- except after the two-kernel
 *    small-batch forward (MOE_OPT_SMALL_BATCH_FORWARD), whose output is then
 *    unspecified, like the other calls' intermediate outputs.  A word left
 *    at MOE_ERR_TIMEOUT by an earlier call zeroes the next combine on the
 *    same workspace too.  moe_get_device_status() reads and clears the word;
 *    the next call on the same workspace starts clean.
 *  - A launch failure returns MOE_ERR_CUDA.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_WORKSPACE = 3,
  MOE_ERR_CUDA = 4,
  MOE_ERR_DEVICE_FAULT = 5,
  MOE_ERR_TIMEOUT = 6
} moe_status;

/* Expert weight formats.
 *  NVFP4: e2m1 elements packed two per byte (element 2i in the low nibble),
 *         one e4m3 scale per 16 elements along K, one fp32 global scale per
 *         tensor part.
 *  MXFP4: e2m1 elements as above, one e8m0 scale per 32 elements along K
 *         (OCP Microscaling Formats v1.0).
 *  FP8:   e4m3 elements, one fp32 per-tensor scale per part: the per-tensor
 *         W8A8 scheme of FreeToken commit 58f4b9ec0e, where a fused
 *         projection keeps one scale per part and the parts' row ranges come
 *         from the load-time weight_scale run-lengths.
 *  BF16:  bf16 elements (bit patterns, 2 bytes), no scales: the BF16
 *         checkpoints of the upstream README ("About").  Activations are bf16
 *         in both activation modes (MATCH rounds h to bf16); always on the
 *         tensor cores (tcgen05 kind::f16). */
typedef enum { MOE_FMT_NVFP4 = 1, MOE_FMT_MXFP4 = 2, MOE_FMT_FP8 = 3, MOE_FMT_BF16 = 4 } moe_fmt;

/* Activation precision.
 *  BF16:  activations stay in bf16/fp32 (weight-only quantisation).
 *  MATCH: activations are quantised to the weights' format before each
 *         projection (W4A4 for NVFP4/MXFP4, W8A8 for FP8), the scheme of the
 *         fused FP8 projection path (FreeToken commit 58f4b9ec0e) and of the
 *         W4A8 decode kernel the atomicmilkshake fork names ("Known limits").
 *         x and h are quantised with the same rules as the weights; a tensor
 *         scale is static when given (a13_gs / a2_gs) and otherwise derived
 *         from the tensor's amax (NVFP4: amax/2688, FP8: amax/448). */
typedef enum { MOE_ACT_BF16 = 0, MOE_ACT_MATCH = 1 } moe_act;

/* Layout of a moe_weights bundle. CANONICAL is the layout documented below.
 * PREPARED is the device layout moe_prepare_weights() writes once at load
 * time (gate/up rows interleaved, scales blocked for the tensor cores);
 * only moe_prepare_weights() produces it. */
typedef enum { MOE_LAYOUT_CANONICAL = 0, MOE_LAYOUT_PREPARED = 1 } moe_layout;

/* One expert bank: E experts of one format, all tensors (device), read only.
 * Merged gate|up projection ("merged projections", atomicmilkshake fork
 * README, "What else changed") followed by the down projection
 * ("ffn_down_exps", same README, "Known limits").  CANONICAL layout:
 *   w13    [E][2I][H/2]  (FP8: [E][2I][H] bytes, BF16: [E][2I][H] bf16)
 *          rows 0..I-1 gate, I..2I-1 up
 *   w13_sf [E][2I][H/16] e4m3 (NVFP4) | [E][2I][H/32] e8m0 (MXFP4) | NULL (FP8, BF16)
 *   w13_gs [E][2] fp32   gate and up part scales (NVFP4, FP8); NULL for MXFP4, BF16
 *   w2     [E][H][I/2]   (FP8: [E][H][I] bytes, BF16: [E][H][I] bf16)
 *   w2_sf  [E][H][I/16] | [E][H][I/32] | NULL
 *   w2_gs  [E] fp32      (NVFP4, FP8); NULL for MXFP4, BF16
 *   a13_gs, a2_gs: one fp32 each, the static activation scale of x and of h
 *          in MATCH mode (NVFP4 global scale / FP8 per-tensor scale); NULL
 *          selects the dynamic amax-derived scale.  Unused for MXFP4.
 * The pointed-to memory must stay valid while calls that use it run. */
typedef struct {
  int32_t fmt, E, H, I, layout;
  const uint8_t* w13;
  const uint8_t* w13_sf;
  const float* w13_gs;
  const uint8_t* w2;
  const uint8_t* w2_sf;
  const float* w2_gs;
  const float* a13_gs;
  const float* a2_gs;
} moe_weights;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t moe_version(void);

/* Bytes of workspace every entry point of this header needs for a layer of
 * T tokens, top-k, the given routed bank and optional shared expert bank
 * (NULL), activation mode `act`.  One workspace of this size serves every
 * call below for that layer; returns 0 on invalid arguments. */
size_t moe_workspace_size(int64_t T, int32_t k, const moe_weights* routed, const moe_weights* shared,
                          int32_t act);

/* Bytes moe_prepare_weights() writes for a CANONICAL bank. */
size_t moe_prepared_weights_size(const moe_weights* canonical);

/* One-time, load-time repack of a CANONICAL bank into the device layout the
 * kernels read (the role the FTW "fast weight format" plays in the FreeToken
 * upstream README, "About"): gate/up rows interleaved (row 2i = gate i,
 * row 2i+1 = up i) and scale factors blocked per 128 rows x 4 scale columns.
 * Writes into `dst` (device, dst_bytes >= moe_prepared_weights_size()),
 * fills *prepared (host) with pointers into dst and into the canonical
 * bank's scalar arrays (w13_gs, w2_gs, a13_gs, a2_gs are shared, not copied).
 * Requires H % 64 == 0 and I % 64 == 0 (MXFP4: % 128).  Enqueued on `stream`. */
moe_status moe_prepare_weights(const moe_weights* canonical, void* dst, size_t dst_bytes,
                               moe_weights* prepared, moe_stream_t stream);

/* Bytes moe_dequantize_weights() writes for a CANONICAL NVFP4 / MXFP4 / FP8
 * bank: E*2I*H + E*H*I bf16 values (0 for a BF16 or invalid bank). */
size_t moe_dequantized_weights_size(const moe_weights* canonical);

/* Load-time expansion of a CANONICAL NVFP4 / MXFP4 / FP8 bank into a
 * CANONICAL BF16 bank, for bf16-activation (W4A16 / W8A16) prefill on the
 * bf16 tensor cores: each weight is decoded by its format's definition
 * (NVFP4 e2m1 * e4m3 * g, MXFP4 e2m1 * 2^(c-127), FP8 e4m3 * s) in fp32 and
 * rounded once to bf16 (nearest even).  The bank then runs like any BF16
 * bank (moe_prepare_weights, then the layer): it takes 4x the bytes of the
 * FP4 bank (2x FP8) in HBM and streams them at that size, so it pays at
 * prefill, where the layer is compute-bound, not at decode.  Writes into dst
 * (device, dst_bytes >= moe_dequantized_weights_size()), fills *bf16 (host)
 * with pointers into dst; static activation scales are dropped (BF16 has
 * none).  MOE_ERR_UNSUPPORTED for a BF16 bank, MOE_ERR_INVALID_ARG for a
 * PREPARED one.  Enqueued on `stream`. */
moe_status moe_dequantize_weights(const moe_weights* canonical, void* dst, size_t dst_bytes, moe_weights* bf16,
                                  moe_stream_t stream);

/* Quantise `rows` x `K` values into a CANONICAL-layout tensor of format
 * `fmt`, with the same rules the layer applies to activations:
 *   NVFP4: sc = e4m3(bmax/(6 g)), r = 1/(dec(sc) g), q = e2m1(x r)  (16-blocks)
 *   MXFP4: c = clamp(floor(log2 bmax) - 2 + 127, 0, 254), q = e2m1(x 2^(127-c))
 *   FP8:   q = e4m3(x * (1/s))
 *   BF16:  q = bf16(x)  (no scale; scale_out receives 1)
 * in fp32, round-to-nearest-even, saturating (BF16: overflowing to inf).  x (device) is fp32
 * (x_dtype 0) or bf16 bits (x_dtype 1).  scale_in (device, one fp32) is the
 * NVFP4 global scale g / FP8 scale s; NULL derives it from the amax of all
 * rows*K values (NVFP4 amax/2688, FP8 amax/448, 1 when the amax is 0).
 * scale_out (device, nullable) receives the scale used.  codes (device):
 * [rows][K/2] (FP8: [rows][K] bytes, BF16: [rows][K] bf16); sf (device):
 * [rows][K/16 | K/32], NULL for FP8 and BF16.  K % 16 (NVFP4, BF16) / 32
 * (MXFP4) == 0.  Used to quantise checkpoints on the
 * device, and the same device code quantises activations inside the layer. */
moe_status moe_quantize(int32_t fmt, const void* x, int32_t x_dtype, int64_t rows, int64_t K,
                        const float* scale_in, uint8_t* codes, uint8_t* sf, float* scale_out, void* ws,
                        size_t ws_bytes, moe_stream_t stream);

/* Router.  logits[t,e] = sum_h x[t,h] Wr[e,h] (+ bias[e]) in fp32;
 * idx[t, 0..k-1] = the k largest logits in descending order, ties to the
 * lower expert index; w[t,j] = exp(L_j - L_0) / sum_i exp(L_i - L_0) over the
 * selected k (softmax over E renormalised over the top k).
 *  x [T][H] bf16 (device), wr [E][H] bf16 (device), bias [E] fp32 (device,
 *  nullable), logits [T][E] fp32 (device, nullable output), topk_idx [T][k]
 *  int32 (device out), topk_w [T][k] fp32 (device out).
 * 1 <= k <= E <= 1024; T >= 0 (T == 0 enqueues nothing).  A row with a NaN
 * logit or no finite logit sets the device status word.
 * Summation order of the logits (all fp32; each product of two bf16 values
 * is exact, so only the sums round), the same on every launch:
 *  - T <= 64 and H % 8 == 0: 256 partial sums per logit; partial p adds the
 *    8 columns from 8p, then the 8 from 8p + 2048, 8p + 4096, ..., one
 *    column at a time; each group of 32 partials is combined by exchange
 *    (for d = 16, 8, 4, 2, 1 every partial q becomes q + (q xor d)), the
 *    group's sum being partial 32g; the 8 group sums are added in order onto
 *    0, then the bias (or 0).  A CPU replay of this order reproduces the
 *    logits, and so the routing, bit for bit.
 *  - T >= 128, H % 64 == 0 and either (a) ceil(T / 128) >= SMs / 2,
 *    E % 16 == 0, 16 <= E <= 256, k <= 16 (one kernel: all of H accumulated
 *    in one tensor-memory accumulator, the top k picked in its epilogue;
 *    MOE_OPT_ROUTER_TOPK) or (b) E % 128 == 0 (H split in up to 4 parts
 *    added in order, then the top-k kernel): the bf16 tensor cores
 *    (tcgen05), fp32 accumulation in their own order.
 *  - otherwise: one sequential sum over h = 0 .. H-1, then the bias (or 0). */
moe_status moe_route(const uint16_t* x, int64_t T, int32_t H, const uint16_t* wr, const float* bias, int32_t E,
                     int32_t k, float* logits, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                     moe_stream_t stream);

/* Top-k and renormalisation alone, from fp32 logits [T][E] (device). */
moe_status moe_route_logits(const float* logits, int64_t T, int32_t E, int32_t k, int32_t* topk_idx,
                            float* topk_w, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Token-to-expert histogram and stable permutation of the S = T*k slots
 * (slot i = t*k + j, expert topk_idx[i]):
 *   offsets[e]    exclusive prefix sum of the counts, offsets[E] = S   [E+1]
 *   perm_token[p] token of the slot at expert-major position p         [S]
 *   inv_perm[i]   position of slot i                                    [S]
 * Positions within one expert follow the flat slot index (stable).  The
 * expert segments are the "slot pool" rows the atomicmilkshake fork README
 * ("Known limits") indexes per expert.  All pointers device.  Counts and
 * positions need no atomic updates (per-chunk counts, a scan, then a rank
 * pass), so the result is deterministic.  An index outside [0, E) sets the
 * device status word (the slot is dropped). */
moe_status moe_permute(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E, int32_t* offsets,
                       int32_t* perm_token, int32_t* inv_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Grouped SwiGLU expert FFN over the permuted slots: for expert e and every
 * position p in [offsets[e], offsets[e+1]) with token t = perm_token[p]:
 *   [g | u] = act(x_t) W13_e^T,  h = g / (1 + exp(-g)) * u,
 *   y_perm[p] = act(h) W2_e^T                      (bf16 [S][H], device out)
 * act() is the identity (BF16) or the quantiser of the weights' format
 * (MATCH, see moe_act; the tensor amax of h is taken over all S slots; bf16
 * rounding for BF16 weights).  x [T][H] bf16, perm_token [S], offsets [E+1]
 * (device); w must be PREPARED.  With quantised activations (MATCH) and H, I
 * multiples of 256 (FP4) or 128 (FP8) the FFN runs as a tcgen05 block-scaled
 * grouped GEMM at every batch size -- 64-token tiles while T*k < 8E (decode:
 * each active expert's weights stream once; with NVFP4 and a static h scale
 * or MXFP4 both projections in one kernel, MOE_OPT_FUSED_FFN), 192-token
 * tiles beyond (prefill; CTA pairs for long K loops, MOE_OPT_GEMM_PAIR).  BF16
 * weights (H, I multiples of 64) always run the bf16 tcgen05 GEMM.  bf16
 * activations with FP4/FP8 weights and other shapes take a TMA-fed mma.sync
 * GEMV that streams each active expert's weights once (the decode split of
 * the atomicmilkshake fork README, "Quant types": MMVQ for decode, MMQ for
 * prefill); moe_dequantize_weights gives such layers the tensor cores at
 * prefill.  The choice is a host decision on the arguments, never a device
 * read-back. */
moe_status moe_grouped_ffn(const uint16_t* x, int64_t T, int32_t k, const int32_t* perm_token,
                           const int32_t* offsets, const moe_weights* w, int32_t act, uint16_t* y_perm, void* ws,
                           size_t ws_bytes, moe_stream_t stream);

/* Weighted un-permute: out[t] = sum_{j<k} w[t,j] y_perm[inv_perm[t*k+j]]
 * (+ shared_y[t]) accumulated in fp32 in order j = 0..k-1, rounded once to
 * bf16.  y_perm [T*k][H], shared_y [T][H] (nullable), out [T][H] bf16;
 * inv_perm [T*k], topk_w [T][k]; all device; 1 <= k <= 1024. */
moe_status moe_combine(const uint16_t* y_perm, const int32_t* inv_perm, const float* topk_w, int64_t T, int32_t k,
                       int32_t H, const uint16_t* shared_y, uint16_t* out, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/* The whole layer in one call: route -> permute -> grouped FFN -> (shared
 * expert, a dense SwiGLU FFN of the same format on every token with weight
 * 1.0, the always-on expert the Domir6/FreeToken fork README lists under
 * "Changes in this fork") -> combine.  x [T][H] bf16, wr [E][H] bf16,
 * bias [E] (nullable), out [T][H] bf16 (device).  routed and shared
 * (nullable, E == 1) must be PREPARED and of one format; the shared expert
 * reads the same x scale as the routed experts.  Intermediates live in `ws`.
 * The shared expert runs on a library-owned side stream forked from `stream`
 * after the x scale and joined before the combine (event record / wait, so a
 * graph capture of `stream` captures both branches); it overlaps routing and
 * the permutation.  Concurrent forwards on one device share that side stream
 * and serialise their shared experts. */
moe_status moe_forward(const uint16_t* x, int64_t T, const uint16_t* wr, const float* bias, int32_t k,
                       const moe_weights* routed, const moe_weights* shared, int32_t act, uint16_t* out, void* ws,
                       size_t ws_bytes, moe_stream_t stream);

/* moe_forward on host buffers, with the copies overlapped.  This entry point
 * is an engineering addition: the pages run the layer on activations already
 * on the device.  x_host and out_host ([T][H] bf16, host) are copied through
 * the caller's device staging buffers x_dev and out_dev ([T][H] bf16 each,
 * 16-byte aligned).  The batch is cut into n_slices (1 ..
 * MOE_MAX_HOST_SLICES) slices of ceil(T / n_slices) consecutive tokens.
 * Slice i is copied in on a library-owned copy stream, run through
 * moe_forward on `stream` once it has landed, and copied out on a second
 * copy stream once its forward is done.  The copies of one slice therefore
 * overlap the forward of another, provided the host buffers are page-locked
 * (pageable ones work but do not overlap).  `stream` waits for the last
 * copy-out, so synchronise `stream` before reading out_host.  The call
 * itself only enqueues.  Each token's result is that of a forward of its
 * slice:
 *  - When an activation's tensor scale is derived from the batch (MATCH with
 *    NVFP4 or FP8 weights and no a13_gs or no a2_gs), tokens are not
 *    independent, and the batch is run as one slice.
 *  - Otherwise a token's result equals its whole-batch result up to the
 *    router's summation order: the router may split its K loop differently
 *    at another batch size, which can flip a top-k choice whose logits tie
 *    to within rounding.
 * ws: at least moe_workspace_size(ceil(T / n_slices), k, routed, shared,
 * act) bytes (moe_workspace_size never decreases with T, so that size also
 * serves a shorter last slice); the slices' forwards reuse it one after the
 * other.  Argument errors return before anything is enqueued.  `stream`
 * waits for the last copy-in and the last copy-out, also after an error. */
#define MOE_MAX_HOST_SLICES 64
moe_status moe_forward_host(const uint16_t* x_host, int64_t T, const uint16_t* wr, const float* bias, int32_t k,
                            const moe_weights* routed, const moe_weights* shared, int32_t act, uint16_t* out_host,
                            uint16_t* x_dev, uint16_t* out_dev, int32_t n_slices, void* ws, size_t ws_bytes,
                            moe_stream_t stream);

/* Host -> HBM expert streaming: an LRU pool of `n_slots` expert slots in
 * HBM in front of an expert bank kept in page-locked host memory, for layers
 * whose experts do not all fit in HBM.  This is the expert slot pool of the
 * atomicmilkshake/FreeToken fork README ("Known limits") and the host-memory
 * expert offload with a global LRU expert cache of the FreeToken upstream
 * README ("About"), decided and copied on the device: a forward through the
 * cache performs no host synchronisation and can be captured in a CUDA
 * graph.  Per call, an admit kernel marks the experts the batch routes to,
 * keeps those already resident (hits), gives every other one the least
 * recently used slot that no expert of this batch holds (empty slots first)
 * and rewrites the top-k ids into slot ids; a fetch kernel copies the
 * admitted experts from host memory into their slots over PCIe; the layer
 * then runs on the pool as a bank of n_slots experts.  The result is the
 * layer's result on the whole bank.
 * Filled by moe_expert_cache_init; treat the fields as read-only. */
typedef struct {
  moe_weights bank;          /* the bank as given: PREPARED, page-locked host memory (a13_gs, a2_gs device) */
  moe_weights pool;          /* the slots: PREPARED, E = n_slots, device memory */
  const void* bank_dev[6];   /* device addresses of bank.w13, w13_sf, w13_gs, w2, w2_sf, w2_gs (or NULL) */
  int32_t* state;            /* device: clock, counters, slot and expert maps */
  int32_t n_slots;
} moe_expert_cache;

/* Device bytes moe_expert_cache_init needs for a pool of n_slots experts of
 * `bank` (0 on invalid arguments). */
size_t moe_expert_cache_bytes(const moe_weights* bank, int32_t n_slots);

/* Sets up a cache: `bank` is a PREPARED bank (moe_prepare_weights, then
 * copied to host memory) whose w13, w13_sf, w13_gs, w2, w2_sf and w2_gs live
 * in page-locked, device-mapped host memory (cudaHostAlloc / pinned torch
 * tensors) and whose a13_gs / a2_gs, if any, are device pointers.
 * 1 <= n_slots <= min(E, 1024).  `dev` (device, dev_bytes >=
 * moe_expert_cache_bytes) holds the pool and the state; the pool starts
 * empty.  Enqueued on `stream`.  MOE_ERR_INVALID_ARG when a host array is not
 * mapped into the device's address space. */
moe_status moe_expert_cache_init(const moe_weights* bank, int32_t n_slots, void* dev, size_t dev_bytes,
                                 moe_expert_cache* cache, moe_stream_t stream);

/* moe_forward with the routed experts streamed through `cache` (no shared
 * expert): route, admit, fetch, permute, grouped FFN on the pool, combine.
 * The pool must hold every expert one batch can route to: n_slots >=
 * min(E, T*k), else MOE_ERR_INVALID_ARG.  ws: moe_workspace_size(T, k,
 * &cache->bank, NULL, act) bytes.  Calls through one cache must not overlap
 * on the GPU (they share its slots). */
moe_status moe_forward_cached(const uint16_t* x, int64_t T, const uint16_t* wr, const float* bias, int32_t k,
                              const moe_expert_cache* cache, int32_t act, uint16_t* out, void* ws, size_t ws_bytes,
                              moe_stream_t stream);

/* Synchronises `stream` and reads the cache's counters: stats[0] calls so
 * far, [1] experts fetched by the last call, [2] experts fetched in all, [3]
 * hits in all (host, 4 values). */
moe_status moe_expert_cache_stats(const moe_expert_cache* cache, moe_stream_t stream, int64_t* stats);

/* Synchronises `stream`, copies the device status word of `ws` into
 * *host_status (a moe_status value: MOE_OK, MOE_ERR_DEVICE_FAULT or
 * MOE_ERR_TIMEOUT) and clears it.  Returns MOE_ERR_CUDA if the
 * synchronisation itself fails. */
moe_status moe_get_device_status(void* ws, moe_stream_t stream, int32_t* host_status);

/* Process-wide switches for A/B measurement (the pattern of the
 * FREETOKEN_FP8_ROWWISE_MM variable in FreeToken commit 58f4b9ec0e).
 *   MOE_OPT_FFN_PATH: 0 = heuristic (default), 1 = force the GEMV path
 *                     (BF16 weights keep the GEMM), 2 = force the tensor-core
 *                     GEMM path (returns MOE_ERR_UNSUPPORTED where the shapes
 *                     do not allow it).
 * Not thread-safe; set before enqueuing. */
/*   MOE_OPT_GEMM_TILE_N: token-tile width of the tensor-core path: 0 (default:
 *                     64 while T*k < 8E, else 192), 64 (four accumulators),
 *                     128 or 192 (two) or 256 (one, drained to registers).
 *   MOE_OPT_GEMM_PAIR: CTA pairs (tcgen05 cta_group::2, 256 weight rows per
 *                     tile, each CTA staging half of the token tile) for 192-
 *                     and 256-token tiles when the weight rows per expert
 *                     divide by 256: 0 never, 1 always, 2 (default) only for a
 *                     projection whose K loop has at least 12 stages (K >=
 *                     3072 for NVFP4 / MXFP4, 1536 for FP8).
 *   MOE_OPT_PDL:       1 (default) launches the layer's kernels with
 *                     programmatic dependent launch, so each one's setup
 *                     overlaps the previous kernel's tail; 0 launches them
 *                     plainly.
 *   MOE_OPT_EARLY_WEIGHTS: 1 (default) lets each tensor-core GEMM of the
 *                     expert FFN load the weight tiles of its first pipeline
 *                     stages before it waits for the previous kernel (the
 *                     weights are inputs of the call, so only the token
 *                     operand waits); 2 also prefetches the next stages'
 *                     weight tiles into L2; 0 loads every stage after the
 *                     wait.
 *   MOE_OPT_FUSED_FFN: 1 (default) runs the gate|up and down projections of a
 *                     64-token-tile batch (T*k < 8E; NVFP4 with a static h
 *                     scale, or MXFP4; E <= 256) as one persistent kernel
 *                     in which the down tiles of a token tile start as soon
 *                     as its gate|up tiles are stored; 0 launches the two
 *                     projections separately.
 *   MOE_OPT_PERMUTE_QUANT: 1 (default) lets moe_forward, when that one-kernel
 *                     FFN runs on quantised activations and T <= 8, E <= 256
 *                     and H % 64 == 0, quantise x inside the one-block
 *                     permutation kernel, and the FFN kernel then derives its
 *                     tile list from the top-k ids, so its first weight loads
 *                     overlap the permutation; 0 runs the x quantiser as a
 *                     kernel of its own.  Results are identical either way.
 *   MOE_OPT_WAIT_CYCLES: bound of every device wait, in SM clock cycles
 *                     (1 .. 2^31 - 1; 0 restores the default of 2e9, about
 *                     a second at 1.965 GHz).  A wait that runs past it gives
 *                     up with MOE_ERR_TIMEOUT (see the conventions above);
 *                     a small bound makes ordinary waits for memory run out,
 *                     which is how the timeout path is tested.
 *   MOE_OPT_FUSED_COMBINE: 1 lets moe_forward, when its routed (and
 *                     shared) experts run on the grouped tensor-core GEMM
 *                     (not the one-kernel FFN) and the weights are not BF16,
 *                     do the weighted combine in the down projection's
 *                     epilogue: each output row gets w * y added in fp32
 *                     (reductions in L2) and one pass rounds the rows to
 *                     bf16, so y_perm is neither written nor read back.  The
 *                     order of the k additions then varies from run to run
 *                     (results within fp32 rounding of each other); 0 keeps
 *                     bf16 y_perm and the ordered combine of moe_combine,
 *                     which is bit-reproducible (the default: the reductions
 *                     measured slower than the bf16 round trip).
 *   MOE_OPT_SMALL_BATCH_FORWARD: 1 (with MOE_OPT_GATHER_X = 1) runs
 *                     moe_forward at T <= 32 on the one-kernel FFN (NVFP4
 *                     with a static h scale, or
 *                     MXFP4; H % 256 == 0; E <= 256) with no shared expert as
 *                     two kernels: the router (logits, x quantised into a
 *                     layout the FFN copies token rows from, top-k in its
 *                     last block), then the FFN, which needs no permutation
 *                     (a tile's rows are its expert's slots in flat order),
 *                     adds w * y into fp32 output rows in its down epilogue
 *                     and rounds them to bf16 in the CTA that finishes last.
 *                     The logits and routing are those of moe_route; the
 *                     order of the k additions varies from run to run.  0
 *                     (default: measured slower than the permutation and
 *                     the ordered combine) keeps those.
 *   MOE_OPT_GATHER_X:  1 lets the one-kernel FFN of a batch of at most 32
 *                     tokens copy its token rows from a routing-independent
 *                     layout of the quantised x; 0 (default: measured
 *                     faster) keeps the quantised padded rows (and turns the
 *                     two-kernel small-batch forward off).
 *   MOE_OPT_ROUTER_TOPK: 1 (default) computes the logits and the top k in
 *                     one tensor-core kernel when the batch's 128-token tiles
 *                     number at least half the SMs, E % 16 == 0,
 *                     16 <= E <= 256, H % 64 == 0 and k <= 16; 0 keeps the
 *                     logits kernel and the separate top-k kernel.
 *   MOE_OPT_FFN_SCHEDULE: 0 (default) the one-kernel FFN's CTAs take work
 *                     items from a counter; 1 CTA b runs items b, b + grid,
 *                     ... -- for measurement only: a down item may then wait
 *                     on a CTA that is not resident (a concurrent kernel, MPS)
 *                     until the wait bound runs out. */
typedef enum {
  MOE_OPT_FFN_PATH = 1,
  MOE_OPT_GEMM_TILE_N = 2,
  MOE_OPT_GEMM_PAIR = 3,
  MOE_OPT_PDL = 4,
  MOE_OPT_EARLY_WEIGHTS = 5,
  MOE_OPT_FUSED_FFN = 6,
  MOE_OPT_PERMUTE_QUANT = 7,
  MOE_OPT_WAIT_CYCLES = 8,
  MOE_OPT_FUSED_COMBINE = 9,
  MOE_OPT_SMALL_BATCH_FORWARD = 10,
  MOE_OPT_GATHER_X = 11,
  MOE_OPT_FFN_SCHEDULE = 12,
  MOE_OPT_ROUTER_TOPK = 13
} moe_option;
moe_status moe_set_option(int32_t option, int32_t value);

/* moe_permute for callers that cannot allocate device memory (no workspace
 * argument).  This entry point is an engineering addition: the pages have no
 * counterpart to it.  It computes exactly what moe_permute computes.  Callers
 * that cannot provide a workspace -- a runtime that has handed all free device
 * memory to its own caches, code running during CUDA stream capture, where
 * cudaMalloc is not allowed, or a host program with no device allocator -- get
 * the permutation's scratch (per-chunk expert counts) from a fixed
 * 256 KiB array that every GPU loading this library holds until the process
 * exits.
 *  Limit: ceil(T*k / 2048) * E <= 65536 (e.g. T*k <= 1,048,576 slots for
 *  E = 128, 524,288 for E = 256); larger sizes return MOE_ERR_WORKSPACE and
 *  enqueue nothing.
 *  dev_status (device, nullable, one int32 the caller zeroes): raised to
 *  MOE_ERR_DEVICE_FAULT for an expert index outside [0, E).
 *  The first call on a device looks up the array's device address (once per
 *  device), so make that first call before any stream capture.  The array's
 *  contents are rewritten by every call, so nothing needs clearing, but calls
 *  that overlap on the GPU share the array and race: serialise them.  No
 *  device memory is allocated or freed. */
moe_status moe_permute_fixed_scratch(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E, int32_t* offsets,
                                     int32_t* perm_token, int32_t* inv_perm, int32_t* dev_status,
                                     moe_stream_t stream);

/* Measurement hooks.
 * moe_set_stage_events: when `events` is non-NULL it must hold
 * 2 * MOE_STAGE_COUNT cudaEvent_t handles; moe_forward and moe_grouped_ffn
 * then record events[2*s] before and events[2*s+1] after stage s on their
 * stream, so a caller can time each stage with cudaEventElapsedTime.  Stages
 * a call does not run are not recorded.  NULL turns the hook off.  Not
 * thread-safe; the handles must outlive the calls that record them.
 * moe_stage_mask: bit s is set when stage s has been recorded since events
 * were last installed (stages a call does not run stay clear; turning the
 * hook off keeps the mask).
 * moe_kernel_launch_count: number of kernels this library has launched in
 * the process so far (host-side count of kernel launches). */
typedef enum {
  MOE_STAGE_ROUTE = 0,      /* router logits + top-k */
  MOE_STAGE_PERMUTE = 1,    /* histogram, scan, permutation */
  MOE_STAGE_ACT_QUANT = 2,  /* activation amax / quantisation of x */
  MOE_STAGE_FFN_UP = 3,     /* gate|up projection + SwiGLU */
  MOE_STAGE_FFN_DOWN = 4,   /* down projection */
  MOE_STAGE_SHARED = 5,     /* shared expert (both projections) */
  MOE_STAGE_COMBINE = 6,    /* weighted un-permute */
  MOE_STAGE_COUNT = 7
} moe_stage;
moe_status moe_set_stage_events(void* const* events, int32_t n_events);
uint32_t moe_stage_mask(void);
uint64_t moe_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
