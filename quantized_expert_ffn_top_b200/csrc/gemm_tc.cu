// Tensor-core grouped expert GEMM for large batches (sm_100a tcgen05).
//
// The prefill half of the prefill/decode split the atomicmilkshake/FreeToken
// fork README describes ("Quant types": MMQ for prefill), rebuilt for B200:
// block-scaled tcgen05.mma (kind::mxf4nvf4 for NVFP4 / MXFP4, kind::f8f6f4
// for FP8 W8A8 -- the per-tensor FP8 projection of FreeToken commit
// 58f4b9ec0e) with accumulators in tensor memory, operands staged by TMA.
//
// Orientation ("swap AB"): the MMA's M side is 128 weight rows of one expert
// and its N side is a tile of that expert's tokens (the permuted slots).
// Weight rows always fill M = 128, while a ragged expert segment only pads N
// to a multiple of 16, so skewed routing wastes little work.
//
// Per CTA (persistent, one per SM), 2 + kEpiWarps warps:
//   warp 0   one thread issues TMA tile loads of A (weights) and B (quantised
//            activations) and bulk copies of their scale blocks into a ring of
//            shared-memory stages;
//   warp 1   allocates tensor memory; one thread copies each stage's scales
//            into tensor memory (tcgen05.cp) and issues the MMAs;
//   others   epilogue: read the accumulator from tensor memory (tcgen05.ld),
//            apply the tensor scales and write the result: SwiGLU and the
//            quantised h for the gate|up projection, bf16 y for the down
//            projection.
// Accumulators are double buffered in tensor memory so the epilogue of one
// tile overlaps the MMAs of the next.  Every wait is bounded: on timeout the
// kernel raises MOE_ERR_TIMEOUT, drains, frees its tensor memory and exits.
//
// Layouts (all prepared by the library):
//  * weights: PREPARED rows (W13: row 2i gate i, row 2i+1 up i), K-major;
//    scales blocked per 128 rows x 4 scale columns (sf_blocked_offset);
//  * activations: expert segments start on a multiple of 128 rows
//    ("padded" rows), K-major codes, scales blocked the same way.
#include <cuda.h>

#include <climits>
#include <cstdint>

#include "kernels.cuh"
#include "gemm_tc.cuh"
#include "tc_ptx.cuh"
#include "token_quant.cuh"
#include "topk_warp.cuh"

namespace moe {
namespace {

// one warp pair's [32 tokens][36] fp32 epilogue tile
constexpr int kEpiTileBytes = 32 * 36 * 4;

template <int FMT>
struct FmtTraits {
  // K elements per stage (128 bytes per row) and per MMA
  static constexpr int kBK = FMT == kFmtBF16 ? 64 : (FMT == MOE_FMT_FP8 ? 128 : 256);
  static constexpr int kMmaK = FMT == kFmtBF16 ? 16 : (FMT == MOE_FMT_FP8 ? 32 : 64);
  static constexpr int kSteps = kBK / kMmaK;                        // MMAs per stage
  static constexpr int kBs = FMT == MOE_FMT_NVFP4 ? 16 : (FMT == MOE_FMT_MXFP4 ? 32 : 0);
  static constexpr int kGroups = kBs ? kBK / (4 * kBs) : 0;         // 4-column scale groups per stage
};

// PAIR: a tile is 256 weight rows x BN (192 or 256) tokens computed by a cluster of two
// CTAs (cta_group::2): each CTA stages its 128 weight rows, half of the token
// rows and all BN tokens' scales, and owns its 128 rows of the accumulator.
template <int FMT, int EPI, int BN, bool PAIR = false>
struct Cfg {
  static_assert(BN == 64 || BN == 128 || BN == 192 || BN == 256, "token tile width");
  static_assert(!PAIR || BN == 256 || BN == 192, "CTA pairs run 192- or 256-token tiles");
  using F = FmtTraits<FMT>;
  // Scale blocks cover 128 token rows; a tile starts on a multiple of 64
  // rows, so a 192-wide tile may start half way into its first block and
  // spans two (see sfb_col_offset).
  static constexpr int kSfbBlocks = (BN + 127) / 128;
  static constexpr int kA = 128 * 128;
  static constexpr int kB = (PAIR ? BN / 2 : BN) * 128;
  static constexpr int kSFA = F::kGroups * 512;
  static constexpr int kSFB = F::kGroups * 512 * kSfbBlocks;
  static constexpr int kStage = ((kA + kB + kSFA + kSFB) + 1023) / 1024 * 1024;
  // epilogue shared memory: one [32 tokens][36] fp32 tile per warp pair (SwiGLU
  // transpose; 1 KB of it per warp stages the down projection's stores) and
  // the NVFP4 h multiplier table
  static constexpr int kEpiTile = kEpiTileBytes;
  static constexpr int kEpiBytes = (4 * (BN / 64) / 2) * kEpiTile + 512;
  static constexpr int kStages = (220 * 1024 - kEpiBytes - 2048) / kStage < 8
                                     ? (220 * 1024 - kEpiBytes - 2048) / kStage
                                     : 8;
  static constexpr int kAccStages = BN == 256 ? 1 : (BN >= 128 ? 2 : 4);
  // 64 accumulator columns per epilogue warp: BN / 64 warps per
  // tensor-memory lane quarter
  static constexpr int kEpiWarps = 4 * (BN / 64);
  static constexpr int kThreads = (2 + kEpiWarps) * 32;
  // arrivals that free an accumulator buffer: every epilogue warp of the tile
  static constexpr uint32_t kTemptyCount = kEpiWarps * (PAIR ? 2 : 1);
  static constexpr uint32_t kSfaCol = kAccStages * BN;
  static constexpr uint32_t kSfbCol = kSfaCol + F::kGroups * 4;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kSmem = kStages * kStage + 1024 /*align*/ + 1024 /*barriers etc.*/ + kEpiBytes;
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kSfbCol + F::kGroups * 4 * kSfbBlocks <= kTmemCols, "tensor memory overflow");
  // barriers (full, empty, tfull, tempty), the tensor-memory address and the
  // abort flag share the 1 KB control block
  static_assert((2 * kStages + 2 * kAccStages) * 8 + 8 <= 1024, "control block overflow");
  // the down projection double-buffers its store staging there: 2 KB per warp
  static_assert(kEpiWarps * 2048 <= kEpiBytes, "store staging");
};

// Tensor-memory column offset of a tile's first token inside its 128-row
// scale block: scales of token row r sit in column (r % 128) / 32 of the
// block's copy and consecutive blocks' copies are adjacent, so a tile
// starting half way into a block (64- and 192-wide tiles) reads its B scales
// two columns further on.
template <int BN>
__device__ __forceinline__ uint32_t sfb_col_offset(int row0) {
  return (BN == 64 || BN == 192) ? (uint32_t)((row0 & 127) >> 5) : 0u;
}

// Token-operand maps with box heights 16, 32, 64, 128, 256 rows: a tile
// loads only the rows it covers, rounded up to one of these.
struct TokenMaps {
  CUtensorMap m[5];
};

__device__ __forceinline__ int token_box_index(int rows) {
  return rows <= 16 ? 0 : (rows <= 32 ? 1 : (rows <= 64 ? 2 : (rows <= 128 ? 3 : 4)));
}

// The plan's tile list held in registers, derived from the compact offsets
// (or the per-expert counts) by one warp (E <= 256): lane l keeps
// offsets[8l .. 8l+8] and the tiles and
// padded rows of all experts before 8l.  Tile tt of the list is the same
// entry the plan kernels write: experts in order, ceil(n_e / bn) tiles each,
// expert segments starting on multiples of 128 padded rows.
struct WarpPlan {
  int lo0;          // offsets[8l]
  int hi[8];        // offsets[8l + j + 1] (held at the last offset past E)
  int tbase, pbase; // tiles and padded rows before expert 8l
  int ntiles;       // tiles of all experts
  bool ok;          // offsets[0] == 0, non-decreasing, offsets[E] == S (S >= 0), fits P and max_tiles

  __device__ __forceinline__ void load(const int32_t* offsets, int E, int bn, int64_t S, int64_t P, int max_tiles) {
    const int lane = threadIdx.x & 31, e0 = 8 * lane;
    lo0 = e0 <= E ? __ldcg(offsets + e0) : 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) hi[j] = e0 + j < E ? __ldcg(offsets + e0 + j + 1) : 0;
    bool good = !(lane == 0 && lo0 != 0);
    int prev = lo0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (e0 + j >= E) hi[j] = prev;
      if (hi[j] < prev) good = false;
      if (e0 + j == E - 1 && S >= 0 && (int64_t)hi[j] != S) good = false;
      prev = hi[j];
    }
    finish(bn, P, max_tiles, good);
  }
  // The same list from the per-expert slot counts cnt[0..E) (shared memory);
  // bad: a slot named no expert in [0, E).
  __device__ __forceinline__ void load_counts(const int32_t* cnt, bool bad, int E, int bn, int64_t S, int64_t P,
                                              int max_tiles) {
    const int lane = threadIdx.x & 31, e0 = 8 * lane;
    int sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      hi[j] = e0 + j < E ? cnt[e0 + j] : 0;
      sum += hi[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += a;
    }
    lo0 = incl - sum;
    int run = lo0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      run += hi[j];
      hi[j] = run;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    finish(bn, P, max_tiles, !bad && (S < 0 || (int64_t)total == S));
  }
  // tiles and padded rows before expert 8l, the totals, and the checks
  __device__ __forceinline__ void finish(int bn, int64_t P, int max_tiles, bool good) {
    const int lane = threadIdx.x & 31;
    int tsum = 0, psum = 0, prev = lo0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int nn = max(hi[j] - prev, 0);
      tsum += (nn + bn - 1) / bn;
      psum += (nn + 127) / 128 * 128;
      prev = hi[j];
    }
    int ti = tsum, pi = psum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, ti, o), b = __shfl_up_sync(0xffffffffu, pi, o);
      if (lane >= o) {
        ti += a;
        pi += b;
      }
    }
    tbase = ti - tsum;
    pbase = pi - psum;
    ntiles = __shfl_sync(0xffffffffu, ti, 31);
    const int prows = __shfl_sync(0xffffffffu, pi, 31);
    ok = __all_sync(0xffffffffu, good) && ntiles <= max_tiles && (int64_t)prows <= P;
  }
  // Padded row of slot p (0 <= p < offsets[E]), -1 if no expert holds it: whole warp.
  __device__ __forceinline__ int64_t row_of_slot(int p) const {
    int pr = pbase, prev = lo0, row = -1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = max(hi[j] - prev, 0);
      if (row < 0 && p >= prev && p < prev + n) row = pr + (p - prev);
      pr += (n + 127) / 128 * 128;
      prev = hi[j];
    }
    const unsigned m = __ballot_sync(0xffffffffu, row >= 0);
    return m ? (int64_t)__shfl_sync(0xffffffffu, row, __ffs(m) - 1) : -1;
  }
  // Entry tt (< ntiles): whole warp.
  __device__ __forceinline__ TileEntry at(int tt, int bn) const {
    const int lane = threadIdx.x & 31;
    int c = tbase, pr = pbase, prev = lo0;
    TileEntry te{-1, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = max(hi[j] - prev, 0);
      const int til = (n + bn - 1) / bn;
      if (te.e < 0 && tt >= c && tt < c + til) {
        const int jt = tt - c;
        te.e = 8 * lane + j;
        te.row0 = pr + jt * bn;
        te.nvalid = min(bn, n - jt * bn);
        te.p0 = prev + jt * bn;
      }
      c += til;
      pr += (n + 127) / 128 * 128;
      prev = hi[j];
    }
    const unsigned m = __ballot_sync(0xffffffffu, te.e >= 0);
    const int src = m ? __ffs(m) - 1 : 0;
    TileEntry r;
    r.e = m ? __shfl_sync(0xffffffffu, te.e, src) : -1;
    r.row0 = __shfl_sync(0xffffffffu, te.row0, src);
    r.nvalid = __shfl_sync(0xffffffffu, te.nvalid, src);
    r.p0 = __shfl_sync(0xffffffffu, te.p0, src);
    return r;
  }
};

// Quantises scale block b (bs values v) of padded row `row` and stores its
// codes and its scale (blocked layout, nb blocks per row of K values).
template <int FMT>
__device__ __forceinline__ void quant_block_store(const float* v, float scale, uint8_t* codes, uint8_t* sf,
                                                  int64_t row, int b, int nb, int K) {
  constexpr int bs = FMT == MOE_FMT_MXFP4 ? 32 : 16;
  if constexpr (FMT == kFmtBF16) {
    // bf16 activations: the 16 values (bf16 already) are stored as they are
    uint32_t p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      p[i] = (uint32_t)f32_to_bf16_rn(v[2 * i]) | ((uint32_t)f32_to_bf16_rn(v[2 * i + 1]) << 16);
    uint4* dst = reinterpret_cast<uint4*>(codes + row * (int64_t)K * 2 + b * 32);
    dst[0] = make_uint4(p[0], p[1], p[2], p[3]);
    dst[1] = make_uint4(p[4], p[5], p[6], p[7]);
    (void)scale;
    (void)sf;
    (void)nb;
    return;
  }
  float bmax = 0.0f;
#pragma unroll
  for (int i = 0; i < bs; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
  if constexpr (FMT == MOE_FMT_NVFP4) {
    uint32_t sc;
    float r;
    nvfp4_block_scale(bmax, scale, sc, r);
    *reinterpret_cast<uint2*>(codes + row * (K / 2) + b * 8) = nvfp4_encode16(v, r);
    sf[sf_blocked_offset(row, b, nb)] = (uint8_t)sc;
  } else if constexpr (FMT == MOE_FMT_MXFP4) {
    uint32_t c;
    float inv;
    mxfp4_block_scale(bmax, c, inv);
    uint4 w;
    w.x = e2m1_encode8(v, inv);
    w.y = e2m1_encode8(v + 8, inv);
    w.z = e2m1_encode8(v + 16, inv);
    w.w = e2m1_encode8(v + 24, inv);
    *reinterpret_cast<uint4*>(codes + row * (K / 2) + b * 16) = w;
    sf[sf_blocked_offset(row, b, nb)] = (uint8_t)c;
  } else {
    const float inv = __frcp_rn(scale);
    uint4 w;
    uint32_t* pw = &w.x;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      pw[i] = e4m3x2_encode(__fmul_rn(v[4 * i], inv), __fmul_rn(v[4 * i + 1], inv)) |
              (e4m3x2_encode(__fmul_rn(v[4 * i + 2], inv), __fmul_rn(v[4 * i + 3], inv)) << 16);
    *reinterpret_cast<uint4*>(codes + row * K + b * 16) = w;
  }
}

// bs bf16 values at src as floats
template <int bs>
__device__ __forceinline__ void load_bf16_block(const uint16_t* src, float* v) {
#pragma unroll
  for (int i = 0; i < bs; i += 8) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + i));
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[i + 2 * j] = __uint_as_float(ww[j] << 16);
      v[i + 2 * j + 1] = __uint_as_float(ww[j] & 0xFFFF0000u);
    }
  }
}

// Converts and stores an epilogue warp's slice of one tile: nch 16-column
// chunks of its 64 accumulator columns (from c_lo), in r0..r3.
template <int FMT, int EPI, int BN>
__device__ __forceinline__ void epilogue_slice(const GemmArgs& g, const CUtensorMap* tmap_y, const TileEntry& te,
                                               int mt, int split, int nch, int c_lo, int ew, int q, int lane,
                                               float gact, float g2, float* epi_tiles, const float* r_tab,
                                               uint16_t* y_stage, int ybufs, int& ypar, float& hmax,
                                               const uint32_t* r0, const uint32_t* r1, const uint32_t* r2,
                                               const uint32_t* r3, int ltok = -1, float lw = 0.0f) {
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    if (ch >= nch) break;  // both warps of a pair see the same ncol
    const uint32_t* rr = ch == 0 ? r0 : (ch == 1 ? r1 : (ch == 2 ? r2 : r3));
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(rr[j]);
    const int c0 = c_lo + ch * 16;
    if (EPI == kEpiLogits) {
      const int o = mt * 128 + q * 32 + lane;  // expert
      const float b = (g.bias && split == 0) ? __ldg(g.bias + o) : 0.0f;   // the bias joins split 0
      float* out = g.logits + (size_t)split * g.split_stride;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int tok = c0 + c;
        if (tok < te.nvalid) out[(size_t)(te.p0 + tok) * g.ldy + o] = v[c] + b;
      }
    } else if (EPI == kEpiDown) {
      const float sc = (FMT == MOE_FMT_MXFP4 || FMT == kFmtBF16) ? 1.0f : __ldg(g.w_gs + te.e) * gact;
      if (g.out32) {
        // the weighted un-permute in the epilogue: lanes 0..15 fetch the
        // chunk's tokens and routing weights; the warp's [tokens][32
        // outputs] block passes through its staging buffer (ybufs KB, 8
        // tokens per KB) so that each lane then adds 4 consecutive outputs
        // of one token with one vector reduction
        int tk = -1;
        float wt = 0.0f;
        if (!g.perm_token) {
          // rows below 32 (gather mode): lane r already holds row r's token and weight
          const int st = __shfl_sync(0xffffffffu, ltok, (c0 + lane) & 31);
          const float sw = __shfl_sync(0xffffffffu, lw, (c0 + lane) & 31);
          if (lane < 16 && c0 + lane < te.nvalid && c0 + lane < 32) {
            tk = st;
            wt = sw;
          }
        } else if (lane < 16 && c0 + lane < te.nvalid) {
          const int p = te.p0 + c0 + lane;
          tk = __ldg(g.perm_token + p);
          wt = g.w_perm ? __ldg(g.w_perm + p) : 1.0f;
        }
        if (tk >= g.out_rows || (lane < 16 && c0 + lane < te.nvalid && tk < 0)) {
          raise_status(g.status, MOE_ERR_DEVICE_FAULT);
          tk = -1;
        }
        float* sb = reinterpret_cast<float*>(y_stage) + ew * ybufs * 256;
        float* orow = g.out32 + mt * 128 + q * 32 + 4 * (lane & 7);
        const int nb = ybufs >= 2 ? 16 : 8;   // tokens per pass
#pragma unroll
        for (int h = 0; h < 16; h += 8) {
          if (h > 0 && nb == 16) break;     // one pass took all 16
          __syncwarp();                     // the previous pass has read the buffer
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (c >= h && c < h + nb) sb[(c - h) * 32 + lane] = v[c] * sc;
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (4 * i >= nb) break;                // uniform: lanes read tokens lane / 8 + 4i
            const int cc = (lane >> 3) + 4 * i;   // token of this read, within the pass
            const int t = __shfl_sync(0xffffffffu, tk, h + cc);
            const float ww = __shfl_sync(0xffffffffu, wt, h + cc);
            const float4 y4 = *reinterpret_cast<const float4*>(sb + cc * 32 + 4 * (lane & 7));
            if (t >= 0) tc::red_add_v4(orow + (size_t)t * g.ldy, ww * y4.x, ww * y4.y, ww * y4.z, ww * y4.w);
          }
        }
        continue;
      }
      if (c0 + 16 <= te.nvalid) {
        // a full chunk: stage [16 tokens][32 outputs] as bf16 in one of this
        // warp's ybufs 1 KB buffers and write it with one tensor store; with
        // two buffers the store of the previous chunk may still be reading
        uint16_t* stg = y_stage + (ew * ybufs + (ybufs == 2 ? ypar : 0)) * 512;
        if (lane == 0) {
          if (ybufs == 2) tc::bulk_wait_read_but1();   // the store from this buffer has read it
          else tc::bulk_wait_read();
        }
        ypar ^= 1;
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 16; ++c) stg[c * 32 + lane] = f32_to_bf16_rn(v[c] * sc);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc::tma_store_2d_keep(tmap_y, stg, mt * 128 + q * 32, te.p0 + c0, tc::l2_policy_evict_last());
          tc::bulk_commit();
        }
      } else {
        // the tile's last, partial chunk: the rows past nvalid belong to
        // the next expert's slots
        const int o = mt * 128 + q * 32 + lane;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int tok = c0 + c;
          if (tok < te.nvalid) g.y[(size_t)(te.p0 + tok) * g.ldy + o] = f32_to_bf16_rn(v[c] * sc);
        }
      }
    } else {
      // gate|up rows interleave (even lane gate, odd lane up): one shuffle
      // pairs them and SwiGLU runs on every lane.  Two chunks (32 tokens)
      // pass through the warp pair's shared-memory tile so that each of
      // the pair's 64 threads then owns 16 consecutive features of one
      // token -- one NVFP4 block, half an MXFP4 block -- for the block
      // maximum, the scale, the codes and 8-byte stores.
      if (ch & 1) continue;  // taken together with the even chunk
      const int part = lane & 1;
      const float sc = (FMT == MOE_FMT_MXFP4 || FMT == kFmtBF16) ? 1.0f : __ldg(g.w_gs + te.e * 2 + part) * gact;
      const int pp = q & 1;                                       // position in the warp pair
      float* tile = epi_tiles + (ew >> 1) * (kEpiTileBytes / 4);    // [32 tokens][36] of the pair
      const int fl = lane >> 1;                                   // feature within the warp's 16
      const int f_pair = mt * 64 + (q >> 1) * 32;                 // first feature of the pair
      const int bar = 1 + (ew >> 1);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        if (hf == 1 && ch + 1 >= nch) break;  // tokens past the tile: their rows are never stored
        const uint32_t* rh = hf == 0 ? rr : (ch == 0 ? r1 : r3);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float a = __uint_as_float(rh[2 * i]) * sc, b = __uint_as_float(rh[2 * i + 1]) * sc;
          const float recv = __shfl_xor_sync(0xffffffffu, part ? a : b, 1);
          const float gg = part ? recv : a;
          const float uu = part ? b : recv;
          tile[(hf * 16 + 2 * i + part) * 36 + pp * 16 + fl] = silu_fast(gg) * uu;
        }
      }
      asm volatile("bar.sync %0, 64;" ::"r"(bar) : "memory");
      const int tid = pp * 32 + lane;
      const int tl = tid >> 1, hh = tid & 1;
      const float4* src = reinterpret_cast<const float4*>(tile + tl * 36 + 16 * hh);
      float hv[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 f = src[j];
        hv[4 * j] = f.x;
        hv[4 * j + 1] = f.y;
        hv[4 * j + 2] = f.z;
        hv[4 * j + 3] = f.w;
      }
      const int tok = c0 + tl;
      const bool valid = tok < te.nvalid;
      const size_t row = (size_t)(te.row0 + tok);
      const int f0 = f_pair + 16 * hh;  // this thread's 16 features
      if (EPI == kEpiUpF32) {
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(g.h32 + row * g.I + f0);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = src[j];
#pragma unroll
          for (int j = 0; j < 16; ++j) hmax = fmaxf(hmax, fabsf(hv[j]));
        }
      } else if constexpr (FMT == kFmtBF16) {
        // bf16 weights: h in bf16, 16 features (32 bytes) per thread
        if (valid) {
          uint32_t p[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            p[j] = (uint32_t)f32_to_bf16_rn(hv[2 * j]) | ((uint32_t)f32_to_bf16_rn(hv[2 * j + 1]) << 16);
          uint4* dst = reinterpret_cast<uint4*>(g.hq + row * (int64_t)g.I * 2 + f0 * 2);
          dst[0] = make_uint4(p[0], p[1], p[2], p[3]);
          dst[1] = make_uint4(p[4], p[5], p[6], p[7]);
        }
      } else {
        float bmax = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(hv[j]));
        uint2 codes;
        uint32_t scode;
        if (FMT == MOE_FMT_NVFP4) {
          scode = nvfp4_scale_code(bmax, g2);
          codes = nvfp4_encode16(hv, r_tab[scode]);
        } else {
          bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));  // the 32-feature block
          float inv;
          mxfp4_block_scale(bmax, scode, inv);
          codes = make_uint2(e2m1_encode8(hv, inv), e2m1_encode8(hv + 8, inv));
        }
        if (valid) {
          *reinterpret_cast<uint2*>(g.hq + row * (g.I / 2) + f0 / 2) = codes;
          if (FMT == MOE_FMT_NVFP4)
            g.hsf[sf_blocked_offset((int64_t)row, f0 / 16, g.I / 16)] = (uint8_t)scode;
          if (FMT == MOE_FMT_MXFP4 && hh == 0)
            g.hsf[sf_blocked_offset((int64_t)row, f0 / 32, g.I / 32)] = (uint8_t)scode;
        }
      }
      asm volatile("bar.sync %0, 64;" ::"r"(bar) : "memory");
    }
  }
}

template <int FMT, int EPI, int BN, bool PAIR>
__global__ void __launch_bounds__(Cfg<FMT, EPI, BN, PAIR>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ TokenMaps tmaps_b,
                        const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                        const __grid_constant__ CUtensorMap tmap_y, const GemmArgs g) {
  using C = Cfg<FMT, EPI, BN, PAIR>;
  using F = FmtTraits<FMT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ctrl = smem + C::kStages * C::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + C::kAccStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + C::kAccStages);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_tiles = reinterpret_cast<float*>(ctrl + 1024);  // [kEpiWarps / 2][32 tokens][36]
  float* r_tab = epi_tiles + (C::kEpiWarps / 2) * (C::kEpiTile / 4);  // NVFP4 h: multiplier per scale code

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < C::kAccStages; ++a) {
      tc::mbar_init(&tfull[a], 1);
      tc::mbar_init(&tempty[a], C::kTemptyCount);
    }
    *abort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&tmap_a);
#pragma unroll
    for (int i = 0; i < 5; ++i) tc::prefetch_tmap(&tmaps_b.m[i]);
    if (PAIR && F::kBs) {
      tc::prefetch_tmap(&tmap_sfa);
      tc::prefetch_tmap(&tmap_sfb);
    }
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tc::tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tc::tmem_relinquish_pair();
    } else {
      tc::tmem_alloc(tmem_slot, C::kTmemCols);
      tc::tmem_relinquish();
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  // the peer's barriers must be initialised before either CTA signals them
  if constexpr (PAIR) tc::cluster_sync();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t rank = PAIR ? tc::cluster_rank() : 0u;
  // tiles: (token tile, weight-row block of 128 rows, or 256 for a pair)
  const int MT = g.R / (PAIR ? 256 : 128);
  const int nkb = g.K / F::kBK;
  const int ncols_w = F::kBs ? g.K / F::kBs : 0;  // scale columns per row (multiple of 4)
  // Early weight loads: the weights (and their scales) are inputs of the
  // layer, so while the previous kernel still runs the producer fills the
  // first pass of the ring with its first stages' weight tiles.  Each such
  // stage's barrier expects the weight bytes now, without an arrival; the
  // main loop arrives with the token bytes.  pre_e records the expert of
  // every early stage, checked against the tile list once it is readable.
  int n_pre = 0;
  int pre_e[C::kStages];
  if constexpr (!PAIR && EPI != kEpiLogits) {
    if (warp == 0 && g.w_early != 0 && (g.w_early == 1 || g.E <= 256)) {
      // past the ring, up to w_early_l2 more stages' weights go to L2
      const int budget = C::kStages + g.w_early_l2;
      const int nitems = min(32, (budget + nkb - 1) / nkb);
      // lane i: the expert of this CTA's i-th work item (-1: none), every
      // read in one round trip
      int e_i = -1;
      if (g.w_early == 1) {
        const int tt_i = (int)((blockIdx.x + (unsigned)lane * gridDim.x) / (unsigned)MT);
        const int nt = __ldcg(g.num_tiles);
        const int e = (lane < nitems && tt_i < g.max_tiles) ? __ldcg(&g.tiles[tt_i].e) : -1;
        e_i = tt_i < nt ? e : -1;
      } else {
        // the plan's tile list from the offsets
        WarpPlan wp;
        wp.load(g.offsets, g.E, BN, -1, INT64_MAX, INT_MAX);
        for (int i = 0; i < nitems; ++i) {
          const int tt = (int)((blockIdx.x + (unsigned)i * gridDim.x) / (unsigned)MT);
          const int e = tt < wp.ntiles ? wp.at(tt, BN).e : -1;
          if (lane == i) e_i = e;
        }
      }
      int n_l2 = 0;
      for (int i = 0; i < nitems && n_pre + n_l2 < budget; ++i) {
        const int e = __shfl_sync(0xffffffffu, e_i, i);
        if (e < 0 || e >= g.E) break;
        const int mt = (int)((blockIdx.x + (unsigned)i * gridDim.x) % (unsigned)MT);
        const uint8_t* sfa = F::kBs ? g.w_sf + (size_t)e * g.R * ncols_w + (size_t)mt * (ncols_w / 4) * 512 : nullptr;
        for (int kb = 0; kb < nkb && n_pre + n_l2 < budget; ++kb) {
          if (n_pre < C::kStages) {
            if (tc::elect_one()) {
              uint8_t* st = smem + n_pre * C::kStage;
              tc::mbar_expect_tx_only(&full[n_pre], C::kA + C::kSFA);
              tc::tma_load_2d(st, &tmap_a, &full[n_pre], kb * 128, e * g.R + mt * 128);
              if (F::kBs)
                tc::bulk_load(st + C::kA + C::kB, sfa + (size_t)kb * F::kGroups * 512, C::kSFA, &full[n_pre]);
            }
            __syncwarp();
            pre_e[n_pre++] = e;
          } else {
            if (tc::elect_one()) {
              tc::tma_prefetch_2d(&tmap_a, kb * 128, e * g.R + mt * 128);
              if (F::kBs) tc::bulk_prefetch_l2(sfa + (size_t)kb * F::kGroups * 512, C::kSFA);
            }
            __syncwarp();
            ++n_l2;
          }
        }
      }
    }
  }
  // the work above overlaps the previous kernel's tail (programmatic launch)
  pdl_wait();
  pdl_trigger();
  // The router GEMM may split K over ksplit CTAs per tile (partial logits
  // that the top-k kernel adds); work item t -> tile t / ksplit, split t % ksplit.
  const int ksplit = EPI == kEpiLogits ? g.ksplit : 1;
  // dense_rows > 0: the token tiles are the plain row blocks [i*BN, i*BN + BN)
  // of dense_rows rows (no tile list)
  auto tile_at = [&](int i) -> TileEntry {
    TileEntry te;
    if (g.dense_rows > 0) {
      te.e = 0;
      te.row0 = i * BN;
      te.nvalid = (int)min((int64_t)BN, g.dense_rows - (int64_t)i * BN);
      te.p0 = i * BN;
    } else {
      te = g.tiles[i];
    }
    return te;
  };
  const int ntok = g.dense_rows > 0 ? (int)((g.dense_rows + BN - 1) / BN) : __ldg(g.num_tiles);
  const int ntiles = ntok * MT * ksplit;
  const int t_first = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int t_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  // The producer and MMA warps run their loops with the whole warp, so the
  // loop state stays warp-uniform, and one elected lane issues the copies
  // and tensor-core instructions (a divergent single-thread loop issues them
  // at about half the rate).
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;  // stages issued by this loop; the first n_pre hold early weight loads
    // each tile's entry is read one tile ahead, off the critical path
    TileEntry te_next = t_first < ntiles ? tile_at((t_first / ksplit) / MT) : TileEntry{};
    for (int t = t_first; t < ntiles && !tc::aborted(abort); t += t_step) {
      const int tt = t / ksplit, split = t % ksplit;
      const int kb0 = split * nkb / ksplit, kb1 = (split + 1) * nkb / ksplit;
      const TileEntry te = te_next;
      if (t + t_step < ntiles) te_next = tile_at(((t + t_step) / ksplit) / MT);
      const int mt = PAIR ? (tt % MT) * 2 + (int)rank : tt % MT;   // this CTA's 128-row weight block
      const uint8_t* sfa = F::kBs ? g.w_sf + (size_t)te.e * g.R * ncols_w + (size_t)mt * (ncols_w / 4) * 512 : nullptr;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort, g.wait_cycles)) {
          if (lane == 0) raise_status(g.status, MOE_ERR_TIMEOUT);
          *abort = 1;
          break;
        }
        if (PAIR && tc::elect_one()) {
          // Both CTAs load their halves; the bytes complete on the leader's
          // barrier, which the leader alone arms with the pair's total.
          uint8_t* st = smem + stage * C::kStage;
          const int nh = min(BN, (te.nvalid + 31) & ~31) >> 1;      // token rows per CTA
          const int bi = token_box_index(nh);
          const uint32_t brows = min(16u << bi, (uint32_t)(BN / 2));   // the map's box height
          const int nblk = ((te.row0 & 127) + min(te.nvalid, BN) + 127) / 128;   // 128-row scale blocks in use
          const uint32_t cbar = tc::cluster_addr(&full[stage], 0);
          if (rank == 0)
            tc::mbar_expect_tx(&full[stage], 2u * (C::kA + brows * 128u + C::kSFA + nblk * F::kGroups * 512));
          tc::tma_load_2d_pair(st, &tmap_a, cbar, kb * 128, te.e * g.R + mt * 128);
          tc::tma_load_2d_pair(st + C::kA, &tmaps_b.m[bi], cbar, kb * 128, te.row0 + (int)rank * nh);
          if (F::kBs) {
            // scale maps: one 512-byte block per row
            const int wblk = (te.e * (g.R / 128) + mt) * (ncols_w / 4) + kb * F::kGroups;
            tc::tma_load_2d_pair(st + C::kA + C::kB, &tmap_sfa, cbar, 0, wblk);
            for (int nb = 0; nb < nblk; ++nb)
              tc::tma_load_2d_pair(st + C::kA + C::kB + C::kSFA + nb * F::kGroups * 512, &tmap_sfb, cbar, 0,
                                   (te.row0 / 128 + nb) * (ncols_w / 4) + kb * F::kGroups);
          }
        } else if (!PAIR && tc::elect_one()) {
          uint8_t* st = smem + stage * C::kStage;
          const int bi = token_box_index(min(te.nvalid, BN));
          const uint32_t brows = min(16u << bi, (uint32_t)BN);   // the map's box height
          const int nblk = ((te.row0 & 127) + min(te.nvalid, BN) + 127) / 128;   // 128-row scale blocks in use
          const bool early = issued < n_pre;   // weights already in flight (stage == issued)
          if (early && pre_e[issued] != te.e) raise_status(g.status, MOE_ERR_DEVICE_FAULT);
          tc::mbar_expect_tx(&full[stage], (early ? 0u : (uint32_t)(C::kA + C::kSFA)) + brows * 128u +
                                               nblk * F::kGroups * 512);
          if (!early) tc::tma_load_2d(st, &tmap_a, &full[stage], kb * 128, te.e * g.R + mt * 128);
          tc::tma_load_2d(st + C::kA, &tmaps_b.m[bi], &full[stage], kb * 128, te.row0);
          if (F::kBs) {
            if (!early) tc::bulk_load(st + C::kA + C::kB, sfa + (size_t)kb * F::kGroups * 512, C::kSFA, &full[stage]);
            for (int nb = 0; nb < nblk; ++nb) {
              const uint8_t* sfb =
                  g.b_sf + ((size_t)(te.row0 / 128 + nb) * (ncols_w / 4) + (size_t)kb * F::kGroups) * 512;
              tc::bulk_load(st + C::kA + C::kB + C::kSFA + nb * F::kGroups * 512, sfb, F::kGroups * 512,
                            &full[stage]);
            }
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // early weight loads that no tile consumed (a shorter tile list, or an
    // abort): arrive, so the barrier completes when they land, and wait for
    // that before the shared memory goes away
    for (int i = issued; i < n_pre; ++i) {
      if (tc::elect_one()) tc::mbar_arrive(&full[i]);
      __syncwarp();
      if (!tc::mbar_wait(&full[i], 0, abort, g.wait_cycles) && !tc::aborted(abort)) {
        if (lane == 0) raise_status(g.status, MOE_ERR_TIMEOUT);
        *abort = 1;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    // a pair's MMAs are issued by its leader (rank 0) alone
    // each tile's entry is read one tile ahead, off the critical path
    TileEntry te_next = t_first < ntiles ? tile_at((t_first / ksplit) / MT) : TileEntry{};
    for (int t = t_first; (!PAIR || rank == 0) && t < ntiles && !tc::aborted(abort); t += t_step) {
      const int tt = t / ksplit, split = t % ksplit;
      const int kb0 = split * nkb / ksplit, kb1 = (split + 1) * nkb / ksplit;
      const TileEntry te = te_next;
      if (t + t_step < ntiles) te_next = tile_at(((t + t_step) / ksplit) / MT);
      if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1u, abort, g.wait_cycles)) {
        if (lane == 0) raise_status(g.status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
      tc::fence_after_sync();
      // N: valid tokens rounded up to 16 (to 32 for a pair: each CTA holds N/2)
      const uint32_t n_mma = (uint32_t)min(BN, PAIR ? (te.nvalid + 31) & ~31 : (te.nvalid + 15) & ~15);
      const uint32_t d = tmem + acc * BN;
      const uint32_t sfb0 = tmem + C::kSfbCol + sfb_col_offset<BN>(te.row0);
      constexpr uint32_t kM = PAIR ? 256u : 128u;
      uint32_t idesc_nv = tc::idesc_mxf4(n_mma, false, 0, 0, kM), idesc_f8 = tc::idesc_f8(n_mma, kM),
               idesc_bf = tc::idesc_bf16(n_mma);
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!tc::mbar_wait(&full[stage], phase, abort, g.wait_cycles)) {
          if (lane == 0) raise_status(g.status, MOE_ERR_TIMEOUT);
          *abort = 1;
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (tc::elect_one()) {
          uint8_t* st = smem + stage * C::kStage;
          const uint32_t sa = tc::smem_u32(st), sb = tc::smem_u32(st + C::kA);
          if (F::kBs) {
            const uint64_t dsfa = tc::desc_sf(tc::smem_u32(st + C::kA + C::kB));
            const uint64_t dsfb = dsfa + (uint64_t)(C::kSFA >> 4);
#pragma unroll
            for (int grp = 0; grp < F::kGroups; ++grp) {
              if constexpr (PAIR) tc::sf_copy_pair(tmem + C::kSfaCol + 4 * grp, dsfa + (uint64_t)(grp * 32));
              else tc::sf_copy(tmem + C::kSfaCol + 4 * grp, dsfa + (uint64_t)(grp * 32));
#pragma unroll
              for (int nb = 0; nb < C::kSfbBlocks; ++nb)
                if (nb == 0 || (uint32_t)(te.row0 & 127) + n_mma > 128u) {  // second block only when the tile reaches it
                  const uint32_t ta = tmem + C::kSfbCol + grp * 4 * C::kSfbBlocks + nb * 4;
                  const uint64_t sd = dsfb + (uint64_t)((nb * F::kGroups + grp) * 32);
                  if constexpr (PAIR) tc::sf_copy_pair(ta, sd);
                  else tc::sf_copy(ta, sd);
                }
            }
          }
          const uint64_t da0 = tc::desc_sw128(sa), db0 = tc::desc_sw128(sb);
#pragma unroll
          for (int kk = 0; kk < F::kSteps; ++kk) {
            const uint64_t da = da0 + (uint64_t)(kk * 2);  // +32 bytes per MMA along K
            const uint64_t db = db0 + (uint64_t)(kk * 2);
            const uint32_t accum = (kb > kb0 || kk > 0) ? 1u : 0u;
            if (FMT == MOE_FMT_NVFP4) {
              const uint32_t sa_t = tmem + C::kSfaCol + 4 * kk, sb_t = sfb0 + kk * 4 * C::kSfbBlocks;
              if constexpr (PAIR) tc::mma_nvf4_pair(d, da, db, idesc_nv, sa_t, sb_t, accum);
              else tc::mma_nvf4(d, da, db, idesc_nv, sa_t, sb_t, accum);
            } else if (FMT == MOE_FMT_MXFP4) {
              const uint32_t id = (uint32_t)(kk & 1) * 2;  // two MMAs share one group of four e8m0 scales
              const uint32_t sa_t = tmem + C::kSfaCol + 4 * (kk >> 1), sb_t = sfb0 + (kk >> 1) * 4 * C::kSfbBlocks;
              if constexpr (PAIR) tc::mma_mxf4_pair(d, da, db, tc::idesc_mxf4(n_mma, true, id, id, kM), sa_t, sb_t, accum);
              else tc::mma_mxf4(d, da, db, tc::idesc_mxf4(n_mma, true, id, id), sa_t, sb_t, accum);
            } else if (FMT == MOE_FMT_FP8) {
              if constexpr (PAIR) tc::mma_f8_pair(d, da, db, idesc_f8, accum);
              else tc::mma_f8(d, da, db, idesc_f8, accum);
            } else {
              tc::mma_bf16(d, da, db, idesc_bf, accum);
            }
          }
          // frees the stage in both CTAs of a pair
          if constexpr (PAIR) tc::mma_commit_pair(&empty[stage], 0x3);
          else tc::mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (tc::elect_one()) {
        if constexpr (PAIR) tc::mma_commit_pair(&tfull[acc], 0x3);
        else tc::mma_commit(&tfull[acc]);
      }
      __syncwarp();
      if (++acc == C::kAccStages) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp drains its 64 accumulator columns into registers, hands the
    // tensor memory back to the MMA warp at once, then converts and stores.
    const int ew = warp - 2;
    const int q = warp & 3;                      // tensor-memory lane quarter of this warp
    const int cw = ew / 4;                       // which 64-column slice of the tile
    const float gact = act_scale_of(FMT, g.act_scale, g.act_amax);
    const float g2 = (EPI == kEpiUpQuant && FMT == MOE_FMT_NVFP4) ? act_scale_of(FMT, g.h_scale, nullptr) : 1.0f;
    if constexpr (EPI == kEpiUpQuant && FMT == MOE_FMT_NVFP4) {
      // r = 1 / (dec(sc) g) for every non-negative e4m3 code (0 for a zero scale)
      for (int c = ew * 32 + lane; c < 128; c += C::kEpiWarps * 32) r_tab[c] = nvfp4_multiplier((uint32_t)c, g2);
      asm volatile("bar.sync 15, %0;" ::"r"(C::kEpiWarps * 32) : "memory");
    }
    float hmax = 0.0f;
    int ypar = 0;   // down projection: the store-staging buffer in turn
    int acc = 0;
    uint32_t acc_phase = 0;
    // each tile's entry is read one tile ahead, off the critical path
    TileEntry te_next = t_first < ntiles ? tile_at((t_first / ksplit) / MT) : TileEntry{};
    for (int t = t_first; t < ntiles; t += t_step) {
      bool ok = tc::mbar_wait(&tfull[acc], acc_phase, abort, g.wait_cycles);
      // the two warps of a pair meet at named barriers in the SwiGLU
      // epilogue, so they go on, or give up, together
      if constexpr (EPI == kEpiUpQuant || EPI == kEpiUpF32) ok = tc::pair_all(ok, 1 + (ew >> 1));
      if (!ok) {
        if (lane == 0) raise_status(g.status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
      tc::fence_after_sync();
      const int tt = t / ksplit, split = t % ksplit;
      const TileEntry te = te_next;
      if (t + t_step < ntiles) te_next = tile_at(((t + t_step) / ksplit) / MT);
      const int mt = PAIR ? (tt % MT) * 2 + (int)rank : tt % MT;   // this CTA's 128 weight rows
      const int ncol = min(BN, (te.nvalid + 15) & ~15);
      const int c_lo = cw * 64;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN) + (uint32_t)c_lo;
      uint32_t r0[16], r1[16], r2[16], r3[16];
      // 16-column chunks of this warp's slice that hold valid tokens
      const int nch = c_lo < ncol ? min(4, (ncol - c_lo + 15) >> 4) : 0;
      if (nch > 0) {
        tc::tmem_ld16_async(tbase, r0);
        if (nch > 1) tc::tmem_ld16_async(tbase + 16, r1);
        if (nch > 2) tc::tmem_ld16_async(tbase + 32, r2);
        if (nch > 3) tc::tmem_ld16_async(tbase + 48, r3);
        tc::tmem_wait16(r0);
        if (nch > 1) tc::tmem_wait16(r1);
        if (nch > 2) tc::tmem_wait16(r2);
        if (nch > 3) tc::tmem_wait16(r3);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) tc::mbar_arrive_cluster(tc::cluster_addr(&tempty[acc], 0));   // the leader's MMA waits
        else tc::mbar_arrive(&tempty[acc]);
      }
      if (++acc == C::kAccStages) {
        acc = 0;
        acc_phase ^= 1u;
      }
      if (c_lo >= ncol) continue;  // both warps of a pair (same slice) skip together
      epilogue_slice<FMT, EPI, BN>(g, &tmap_y, te, mt, split, nch, c_lo, ew, q, lane, gact, g2, epi_tiles, r_tab,
                                   reinterpret_cast<uint16_t*>(epi_tiles), 2, ypar, hmax, r0, r1, r2, r3);
    }
    if (EPI == kEpiDown && lane == 0) tc::bulk_wait_all();   // stores done before the CTA exits
    if (EPI == kEpiUpF32 && g.h_amax) {
      hmax = warp_max(hmax);
      if (lane == 0) atomic_max_nonneg(g.h_amax, hmax);
    }
  }

  __syncwarp();
  __syncthreads();
  if (*abort) {
    // let copies and MMAs already in flight land before the memory goes away
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000LL) {
    }
  }
  // Neither CTA of a pair leaves while the other may still signal its
  // barriers or (leader's MMAs) read its shared memory.
  if constexpr (PAIR) tc::cluster_sync();
  tc::fence_after_sync();
  if (warp == 1) {
    if constexpr (PAIR) tc::tmem_dealloc_pair(tmem, C::kTmemCols);
    else tc::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------- fused expert FFN --
// gate|up + SwiGLU + h quantisation and the down projection in one
// persistent kernel (64-token tiles, NVFP4 / MXFP4 with an h scale that needs
// no global reduction).  Work item i is gate|up tile i for i < n1 = tiles *
// MT1, else down tile i - n1.  The CTAs take items from a counter in global
// memory, in increasing order, so every gate|up item is taken -- by a CTA
// that is running -- before any down item, and a CTA runs its items in the
// order it took them: a down item's wait for the gate|up items of its token
// tile always ends, whether or not all CTAs are resident at once (a kernel on
// another stream, MPS), and the work evens out across CTAs by itself.  Each
// epilogue warp counts its gate|up slice of token tile tt in tile_done[tt]
// after storing it; the producer issues a down item's token operand (h) once
// all MT1 * warps slices of its tile are counted.  The producer keeps two
// cursors: weight tiles go out as soon as a ring stage is free (the first
// item's first stages before the wait on the previous kernel), token tiles as
// their data is ready; the items it takes reach the MMA and epilogue warps
// through a queue in shared memory.
template <int FMT, int BN>
struct FusedCfg {
  using C = Cfg<FMT, kEpiUpQuant, BN, false>;
  // queue entries: the items between the epilogue and the weight cursor
  // (at most two rings of stages and the accumulators) fit with room to spare
  static constexpr int kQ = 32;
  static_assert(kQ >= 2 * C::kStages + C::kAccStages + 2, "item queue");
  // + the down store staging, the item queue, the expert counts (+ a flag),
  // the slot or token of every slot position of a gathering batch
  static constexpr int kSmem =
      C::kSmem + C::kEpiWarps * 1024 + kQ * (8 + 8 + 4) + (kFusedMaxE + 1) * 4 + kGatherMaxS * 2;
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

template <int FMT, int BN, bool GATHER>
__global__ void __launch_bounds__(Cfg<FMT, kEpiUpQuant, BN, false>::kThreads, 1)
    fused_ffn_kernel(const __grid_constant__ CUtensorMap tmap_w13, const __grid_constant__ TokenMaps tmaps_x,
                     const __grid_constant__ CUtensorMap tmap_w2, const __grid_constant__ TokenMaps tmaps_h,
                     const __grid_constant__ CUtensorMap tmap_y, const GemmArgs g1, const GemmArgs g2,
                     const FusedArgs f) {
  using C = Cfg<FMT, kEpiUpQuant, BN, false>;
  using F = FmtTraits<FMT>;
  using FC = FusedCfg<FMT, BN>;
  constexpr int kQ = FC::kQ;
  static_assert(F::kBs > 0, "block-scaled formats only");
  static_assert(C::kSfbBlocks == 1, "one scale block per token tile");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ctrl = smem + C::kStages * C::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + C::kAccStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + C::kAccStages);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_tiles = reinterpret_cast<float*>(ctrl + 1024);
  float* r_tab = epi_tiles + (C::kEpiWarps / 2) * (C::kEpiTile / 4);
  // the down projection's store staging, 1 KB per warp, apart from the
  // SwiGLU tiles (a warp may start its first down tile while its pair
  // partner still finishes the last gate|up tile)
  uint16_t* y_stage = reinterpret_cast<uint16_t*>(r_tab + 128);
  // item queue: entry j holds an item id (-1: no more items); q_full[j]
  // completes when the producer has written it, q_free[j] when the MMA warp
  // and every epilogue warp have read it
  uint64_t* q_full = reinterpret_cast<uint64_t*>(y_stage + C::kEpiWarps * 512);
  uint64_t* q_free = q_full + kQ;
  volatile int32_t* q_id = reinterpret_cast<volatile int32_t*>(q_free + kQ);
  int32_t* hist = const_cast<int32_t*>(q_id) + kQ;  // [kFusedMaxE] counts, bad flag
  // gather mode: the slot (forward) or token (grouped FFN) of every slot
  // position, experts in order, slots in flat order within an expert
  uint16_t* s_slot = reinterpret_cast<uint16_t*>(hist + kFusedMaxE + 1);
  // gather mode on the forward: the slots' experts come from the previous
  // kernel (the router), so everything waits for it
  const bool ids_from_prev = GATHER && f.slot_expert != nullptr;
  if (ids_from_prev) pdl_wait();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < C::kAccStages; ++a) {
      tc::mbar_init(&tfull[a], 1);
      tc::mbar_init(&tempty[a], C::kEpiWarps);
    }
    for (int j = 0; j < kQ; ++j) {
      tc::mbar_init(&q_full[j], 1);
      tc::mbar_init(&q_free[j], 1 + C::kEpiWarps);
    }
    *abort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&tmap_w13);
    tc::prefetch_tmap(&tmap_w2);
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      tc::prefetch_tmap(&tmaps_x.m[i]);
      tc::prefetch_tmap(&tmaps_h.m[i]);
    }
    tc::prefetch_tmap(&tmap_y);
  }
  if (warp == 0 && f.slot_expert) {
    // Slot counts per expert from the slots' expert ids: 32 slots per step,
    // the first lane of each group of equal ids adds the group's size.
    for (int e = lane; e <= kFusedMaxE; e += 32) hist[e] = 0;
    __syncwarp();
    bool bad = false;
    for (int64_t base = 0; base < f.S; base += 32 * 8) {
      int ev[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = base + 32 * u + lane;
        ev[u] = i < f.S ? __ldcg(f.slot_expert + i) : -1;
        if (i < f.S && (ev[u] < 0 || ev[u] >= g1.E)) {
          bad = true;
          ev[u] = -1;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const unsigned peers = __match_any_sync(0xffffffffu, ev[u]);
        if (ev[u] >= 0 && lane == __ffs(peers) - 1) hist[ev[u]] += __popc(peers);
        __syncwarp();
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) hist[kFusedMaxE] = 1;
    if (GATHER) {
      // the slots in expert-major order (a counting sort, stable in the flat
      // index): lane l holds the counts of experts 8l .. 8l + 7, turns them
      // into the exclusive prefix as cursors, places every slot, and puts
      // the counts back for the tile list
      __syncwarp();
      int cnt[8], run = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = 8 * lane + j < kFusedMaxE ? hist[8 * lane + j] : 0;
        run += cnt[j];
      }
      int incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += a;
      }
      int cur = incl - run;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (8 * lane + j < kFusedMaxE) hist[8 * lane + j] = cur;
        cur += cnt[j];
      }
      __syncwarp();
      for (int64_t base = 0; base < f.S && f.S <= kGatherMaxS; base += 32) {
        const int64_t i = base + lane;
        int e = i < f.S ? __ldcg(f.slot_expert + i) : -1;
        if (e >= g1.E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int pos = e >= 0 ? hist[e] + __popc(peers & ((1u << lane) - 1u)) : -1;
        __syncwarp();
        if (e >= 0) s_slot[pos] = (uint16_t)i;
        if (e >= 0 && lane == __ffs(peers) - 1) hist[e] += __popc(peers);
        __syncwarp();
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (8 * lane + j < kFusedMaxE) hist[8 * lane + j] = cnt[j];
    }
  }
  if (GATHER && warp == 0 && f.perm_token) {
    // the grouped FFN gives the token of every position (an input of the call)
    for (int64_t p = lane; p < f.S && f.S <= kGatherMaxS; p += 32) s_slot[p] = (uint16_t)__ldg(f.perm_token + p);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, C::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // Every warp derives the tile list itself, from the offsets or from the
  // slots' expert ids; either is older than the previous kernel (read before
  // waiting for it).
  WarpPlan plan;
  if (f.slot_expert)
    plan.load_counts(hist, hist[kFusedMaxE] != 0, g1.E, BN, f.S, f.P, f.max_tiles);
  else
    plan.load(f.offsets, g1.E, BN, f.S, f.P, f.max_tiles);
  const int ntok = plan.ok ? plan.ntiles : 0;
  if (!plan.ok && blockIdx.x == 0 && threadIdx.x == 0) raise_status(g1.status, MOE_ERR_DEVICE_FAULT);
  const int MT1 = g1.R / 128, MT2 = g2.R / 128;
  const int nkb1 = g1.K / F::kBK, nkb2 = g2.K / F::kBK;
  const int ncols1 = g1.K / F::kBs, ncols2 = g2.K / F::kBs;
  const int n1 = ntok * MT1, total = n1 + ntok * MT2;
  const int done_target = MT1 * C::kEpiWarps;
  const long long wait_lim = g1.wait_cycles;
  // item i: up (gate|up or down), token tile, weight-row block
  auto decode = [&](int i, bool& up, int& tt, int& mt) {
    up = i < n1;
    const int r = up ? i : i - n1, m = up ? MT1 : MT2;
    tt = r / m;
    mt = r % m;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Items are taken one ahead: lane 0 holds the counter's answer for the
    // next item while the current one's weights go out.
    int pending = 0, n_taken = 0;
    const bool dyn = !f.static_items;
    if (lane == 0 && !dyn) pending = (int)blockIdx.x;
    int pushed = 0;          // queue entries written (items, then the end mark)
    bool ended = false;      // the end mark is in the queue
    // weight cursor: item, stage within it, stage sequence number (ring slot
    // = seq % kStages)
    bool a_valid = false, a_up = false;
    int a_tt = 0, a_mt = 0, a_e = 0, kba = 0, seq_a = 0;
    // token cursor: queue position, stage within the item, sequence number
    int b_pos = 0, kbb = 0, seq_b = 0;
    bool b_have = false, b_up = false, b_ready = false;
    int b_tt = 0, b_mt = 0;
    TileEntry b_te{};
    int b_tok = -1;    // gather mode: lane r (< nvalid) holds the token of tile row r
    // token tiles whose gate|up slices are all stored: bit i of rdy is token
    // tile rdy_base + i (down items are taken in increasing token-tile order,
    // so one poll of 32 tiles ahead covers the next down items)
    uint32_t rdy = 0;
    int rdy_base = 0;
    // Moves the weight cursor to a newly taken item and queues it; false
    // when the queue has no room right now.
    auto take_next = [&]() -> bool {
      if (pushed - b_pos >= kQ) return false;   // the token cursor still reads that entry
      const int j = pushed % kQ;
      const uint32_t par = ((uint32_t)(pushed / kQ) & 1u) ^ 1u;
      if (__shfl_sync(0xffffffffu, (int)tc::mbar_test_wait(&q_free[j], par), 0) == 0) return false;
      int id = __shfl_sync(0xffffffffu, pending, 0);
      id = id < total ? id : -1;
      ++n_taken;
      if (lane == 0) {
        if (id >= 0) pending = f.static_items ? (int)blockIdx.x + n_taken * (int)gridDim.x : atomicAdd(f.work, 1);
        q_id[j] = id;
        tc::mbar_arrive(&q_full[j]);
      }
      __syncwarp();
      ++pushed;
      if (id < 0) {
        ended = true;
        a_valid = false;
        return true;
      }
      decode(id, a_up, a_tt, a_mt);
      a_e = plan.at(a_tt, BN).e;
      kba = 0;
      a_valid = true;
      return true;
    };
    auto issue_a = [&]() {
      const int st = seq_a % C::kStages;
      if (tc::elect_one()) {
        uint8_t* sp = smem + st * C::kStage;
        const int R = a_up ? g1.R : g2.R, nc = a_up ? ncols1 : ncols2;
        const uint8_t* sfa = (a_up ? g1.w_sf : g2.w_sf) + (size_t)a_e * R * nc + (size_t)a_mt * (nc / 4) * 512;
        tc::mbar_expect_tx_only(&full[st], C::kA + C::kSFA);
        tc::tma_load_2d(sp, a_up ? &tmap_w13 : &tmap_w2, &full[st], kba * 128, a_e * R + a_mt * 128);
        tc::bulk_load(sp + C::kA + C::kB, sfa + (size_t)kba * F::kGroups * 512, C::kSFA, &full[st]);
      }
      __syncwarp();
      ++seq_a;
      if (++kba == (a_up ? nkb1 : nkb2)) a_valid = false;
    };
    // Before the wait on the previous kernel (the x quantiser), at most
    // kPreStages weight stages of the first item are put in flight (the
    // ring's first pass needs no free slot): a deeper burst queues that
    // kernel's own reads behind it.
    constexpr int kPreStages = 3 < C::kStages ? 3 : C::kStages;
    if (!dyn) {
      take_next();
      if (g1.w_early != 0)
        while (a_valid && seq_a < kPreStages) issue_a();
    } else if (g1.w_early != 0 && (int)blockIdx.x < total) {
      // The counter is cleared by the kernel before this one, so items are
      // taken after the wait.  The first items go to the first CTAs to get
      // there, one each: CTA b prefetches item b's first stages into L2 for
      // whichever CTA takes it.
      bool up = false;
      int tt = 0, mt = 0;
      decode((int)blockIdx.x, up, tt, mt);
      const int e = plan.at(tt, BN).e;
      const int R = up ? g1.R : g2.R, nc = up ? ncols1 : ncols2, nkb = up ? nkb1 : nkb2;
      const uint8_t* sfa = (up ? g1.w_sf : g2.w_sf) + (size_t)e * R * nc + (size_t)mt * (nc / 4) * 512;
      if (tc::elect_one()) {
        for (int kb = 0; kb < kPreStages && kb < nkb; ++kb) {
          tc::tma_prefetch_2d(up ? &tmap_w13 : &tmap_w2, kb * 128, e * R + mt * 128);
          tc::bulk_prefetch_l2(sfa + (size_t)kb * F::kGroups * 512, C::kSFA);
        }
      }
      __syncwarp();
    }
    pdl_wait();
    pdl_trigger();
    if (dyn && lane == 0) pending = atomicAdd(f.work, 1);
    long long t_prog = clock64();
    while (true) {
      bool prog = false;
      // token tiles: every stage whose weights are out and whose data is
      // ready (a dependency poll at most once per pass)
      while (seq_b < seq_a) {
        if (!b_have) {
          const int id = q_id[b_pos % kQ];   // written by this warp, always an item here
          decode(id, b_up, b_tt, b_mt);
          b_te = plan.at(b_tt, BN);
          b_have = true;
          // gate|up token tiles come from the x quantiser before this kernel
          b_ready = b_up || (b_tt >= rdy_base && b_tt < rdy_base + 32 && ((rdy >> (b_tt - rdy_base)) & 1u));
          if (GATHER && b_up) {
            // the tile's rows are its expert's slots in flat order (one tile
            // per expert: at most kGatherMaxT slots; more means slots that
            // repeat a token, which the rows past 32 do not get)
            const int n = min(b_te.nvalid, kGatherMaxT);
            if (b_te.nvalid > kGatherMaxT && lane == 0) raise_status(g1.status, MOE_ERR_DEVICE_FAULT);
            const int v = lane < n && b_te.p0 + lane < f.S ? (int)s_slot[b_te.p0 + lane] : -1;
            b_tok = v < 0 ? -1 : (f.perm_token ? v : v / f.k);
            if (b_tok >= f.T) b_tok = -1;
          }
        }
        if (!b_ready) {
          // one round trip polls this token tile and the next 31
          if (b_tt < rdy_base || b_tt >= rdy_base + 32) {
            rdy = 0;
            rdy_base = b_tt;
          }
          const int tt_i = rdy_base + lane;
          const int v = tt_i < ntok ? tc::ld_acquire_gpu(f.tile_done + tt_i) : 0;
          rdy |= __ballot_sync(0xffffffffu, v >= done_target);
          if (!((rdy >> (b_tt - rdy_base)) & 1u)) break;
          tc::fence_proxy_async_global();   // for every token tile seen ready here
          b_ready = true;
        }
        const int st = seq_b % C::kStages;
        if (GATHER && b_up) {
          // x rows by bulk copies from the gather layout: lane r copies tile
          // row r's 128 code bytes (the variant swizzled for r % 8) and its
          // scale lines, one per 4-scale group of the stage
          uint8_t* sp = smem + st * C::kStage;
          const int n = min(b_te.nvalid, kGatherMaxT);
          if (tc::elect_one()) tc::mbar_expect_tx(&full[st], (uint32_t)n * (128u + F::kGroups * 16u));
          __syncwarp();
          const int t = b_tok >= 0 ? b_tok : 0;   // a bad slot still completes its bytes
          if (lane < n) {
            const uint8_t* src = f.xg + ((int64_t)t * 8 + (lane & 7)) * (g1.K / 2) + (int64_t)kbb * 128;
            tc::bulk_load(sp + C::kA + lane * 128, src, 128u, &full[st]);
            const uint8_t* lines = f.xsl + ((int64_t)t * (ncols1 / 4) + (int64_t)kbb * F::kGroups) * 16;
#pragma unroll
            for (int gi = 0; gi < F::kGroups; ++gi)
              tc::bulk_load(sp + C::kA + C::kB + C::kSFA + gi * 512 + lane * 16, lines + gi * 16, 16u, &full[st]);
          }
          __syncwarp();
        } else if (tc::elect_one()) {
          uint8_t* sp = smem + st * C::kStage;
          const int bi = token_box_index(min(b_te.nvalid, BN));
          const uint32_t brows = min(16u << bi, (uint32_t)BN);
          const int nc = b_up ? ncols1 : ncols2;
          tc::mbar_expect_tx(&full[st], brows * 128u + F::kGroups * 512);
          tc::tma_load_2d(sp + C::kA, b_up ? &tmaps_x.m[bi] : &tmaps_h.m[bi], &full[st], kbb * 128, b_te.row0);
          const uint8_t* sfb =
              (b_up ? g1.b_sf : g2.b_sf) + ((size_t)(b_te.row0 / 128) * (nc / 4) + (size_t)kbb * F::kGroups) * 512;
          tc::bulk_load(sp + C::kA + C::kB + C::kSFA, sfb, F::kGroups * 512, &full[st]);
        }
        __syncwarp();
        ++seq_b;
        if (++kbb == (b_up ? nkb1 : nkb2)) {
          kbb = 0;
          ++b_pos;
          b_have = false;
        }
        prog = true;
      }
      // weight tiles: every free ring slot, at most a ring ahead of the tokens
      while (seq_a < seq_b + C::kStages) {
        if (!a_valid) {
          if (ended || !take_next()) break;
          prog = true;
          if (!a_valid) break;   // the end mark
        }
        const int st = seq_a % C::kStages;
        const uint32_t par = (((uint32_t)(seq_a / C::kStages)) & 1u) ^ 1u;
        if (__shfl_sync(0xffffffffu, (int)tc::mbar_test_wait(&empty[st], par), 0) == 0) break;
        issue_a();
        prog = true;
      }
      if (ended && !a_valid && seq_b == seq_a) break;   // every item's stages are out
      if (prog) {
        t_prog = clock64();
      } else if (__any_sync(0xffffffffu, *abort != 0 || clock64() - t_prog > wait_lim)) {
        // neither cursor could move for the wait bound (all polls above are
        // non-blocking), or another warp gave up: the warp leaves as one
        if (lane == 0 && !*abort) raise_status(g1.status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
    }
    // weight tiles issued for stages whose token tiles were not (an abort):
    // arrive, so the barrier completes when they land, and wait for that
    for (int q = seq_b; q < seq_a; ++q) {
      const int st = q % C::kStages;
      if (tc::elect_one()) tc::mbar_arrive(&full[st]);
      __syncwarp();
      tc::mbar_wait(&full[st], ((uint32_t)(q / C::kStages)) & 1u, abort, wait_lim);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    pdl_wait();
    pdl_trigger();
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int k = 0; !tc::aborted(abort); ++k) {
      const int j = k % kQ;
      if (!tc::mbar_wait(&q_full[j], (uint32_t)(k / kQ) & 1u, abort, wait_lim)) {
        if (lane == 0) raise_status(g1.status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
      const int id = q_id[j];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&q_free[j]);
      if (id < 0) break;
      bool up = false;
      int tt = 0, mt = 0;
      decode(id, up, tt, mt);
      const TileEntry te = plan.at(tt, BN);
      if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1u, abort, wait_lim)) {
        if (lane == 0) raise_status(g1.status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
      tc::fence_after_sync();
      const uint32_t n_mma = (uint32_t)min(BN, (te.nvalid + 15) & ~15);
      const uint32_t d = tmem + acc * BN;
      // gathered rows start at tile row 0 of the stage; loaded ones at the
      // tile's padded row
      const uint32_t sfb0 = tmem + C::kSfbCol + ((GATHER && up) ? 0u : sfb_col_offset<BN>(te.row0));
      const uint32_t idesc_nv = tc::idesc_mxf4(n_mma, false, 0, 0);
      const int nkb = up ? nkb1 : nkb2;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!tc::mbar_wait(&full[stage], phase, abort, wait_lim)) {
          if (lane == 0) raise_status(g1.status, MOE_ERR_TIMEOUT);
          *abort = 1;
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (tc::elect_one()) {
          uint8_t* st = smem + stage * C::kStage;
          const uint64_t dsfa = tc::desc_sf(tc::smem_u32(st + C::kA + C::kB));
          const uint64_t dsfb = dsfa + (uint64_t)(C::kSFA >> 4);
#pragma unroll
          for (int grp = 0; grp < F::kGroups; ++grp) {
            tc::sf_copy(tmem + C::kSfaCol + 4 * grp, dsfa + (uint64_t)(grp * 32));
            tc::sf_copy(tmem + C::kSfbCol + grp * 4, dsfb + (uint64_t)(grp * 32));
          }
          const uint64_t da0 = tc::desc_sw128(tc::smem_u32(st)), db0 = tc::desc_sw128(tc::smem_u32(st + C::kA));
#pragma unroll
          for (int kk = 0; kk < F::kSteps; ++kk) {
            const uint64_t da = da0 + (uint64_t)(kk * 2), db = db0 + (uint64_t)(kk * 2);
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            if (FMT == MOE_FMT_NVFP4) {
              tc::mma_nvf4(d, da, db, idesc_nv, tmem + C::kSfaCol + 4 * kk, sfb0 + kk * 4, accum);
            } else {
              const uint32_t id2 = (uint32_t)(kk & 1) * 2;
              tc::mma_mxf4(d, da, db, tc::idesc_mxf4(n_mma, true, id2, id2), tmem + C::kSfaCol + 4 * (kk >> 1),
                           sfb0 + (kk >> 1) * 4, accum);
            }
          }
          tc::mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (tc::elect_one()) tc::mma_commit(&tfull[acc]);
      __syncwarp();
      if (++acc == C::kAccStages) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();
    pdl_trigger();
    const int ew = warp - 2;
    const int q = warp & 3;
    const int cw = ew / 4;
    const float gact1 = act_scale_of(FMT, g1.act_scale, g1.act_amax);
    const float gh = FMT == MOE_FMT_NVFP4 ? act_scale_of(FMT, g1.h_scale, nullptr) : 1.0f;
    const float gact2 = act_scale_of(FMT, g2.act_scale, g2.act_amax);
    if constexpr (FMT == MOE_FMT_NVFP4) {
      for (int c = ew * 32 + lane; c < 128; c += C::kEpiWarps * 32) r_tab[c] = nvfp4_multiplier((uint32_t)c, gh);
      asm volatile("bar.sync 15, %0;" ::"r"(C::kEpiWarps * 32) : "memory");
    }
    float hmax = 0.0f;
    int ypar = 0;   // down projection: the store-staging buffer in turn
    int acc = 0;
    uint32_t acc_phase = 0;
    const int pbar = 1 + (ew >> 1);   // this warp pair's named barrier
    for (int k = 0;; ++k) {
      const int j = k % kQ;
      // the two warps of a pair meet at named barriers in the SwiGLU
      // epilogue, so they go on, or give up, together
      if (!tc::pair_all(tc::mbar_wait(&q_full[j], (uint32_t)(k / kQ) & 1u, abort, wait_lim), pbar)) {
        if (lane == 0) raise_status(g1.status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
      const int id = q_id[j];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&q_free[j]);
      if (id < 0) break;
      bool up = false;
      int tt = 0, mt = 0;
      decode(id, up, tt, mt);
      const TileEntry te = plan.at(tt, BN);
      if (!tc::pair_all(tc::mbar_wait(&tfull[acc], acc_phase, abort, wait_lim), pbar)) {
        if (lane == 0) raise_status(g1.status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
      tc::fence_after_sync();
      const int ncol = min(BN, (te.nvalid + 15) & ~15);
      const int c_lo = cw * 64;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN) + (uint32_t)c_lo;
      uint32_t r0[16], r1[16], r2[16], r3[16];
      const int nch = c_lo < ncol ? min(4, (ncol - c_lo + 15) >> 4) : 0;
      if (nch > 0) {
        tc::tmem_ld16_async(tbase, r0);
        if (nch > 1) tc::tmem_ld16_async(tbase + 16, r1);
        if (nch > 2) tc::tmem_ld16_async(tbase + 32, r2);
        if (nch > 3) tc::tmem_ld16_async(tbase + 48, r3);
        tc::tmem_wait16(r0);
        if (nch > 1) tc::tmem_wait16(r1);
        if (nch > 2) tc::tmem_wait16(r2);
        if (nch > 3) tc::tmem_wait16(r3);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty[acc]);
      if (++acc == C::kAccStages) {
        acc = 0;
        acc_phase ^= 1u;
      }
      // the forward's combine in the down epilogue: lane r gets tile row r's
      // token and routing weight
      int ltok = -1;
      float lw = 0.0f;
      if (GATHER && !up && g2.out32 && f.slot_expert) {
        const int n = min(te.nvalid, kGatherMaxT);
        const int sl = lane < n && te.p0 + lane < f.S ? (int)s_slot[te.p0 + lane] : -1;
        ltok = sl >= 0 ? sl / f.k : -1;
        lw = sl >= 0 ? __ldg(f.topk_w + sl) : 0.0f;
      }
      if (up) {
        if (c_lo < ncol)
          epilogue_slice<FMT, kEpiUpQuant, BN>(g1, &tmap_y, te, mt, 0, nch, c_lo, ew, q, lane, gact1, gh, epi_tiles,
                                               r_tab, y_stage, 1, ypar, hmax, r0, r1, r2, r3);
        // this warp's slice of h is stored: count it for the down tiles
        tc::fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(f.tile_done + tt, 1);
      } else if (c_lo < ncol) {
        epilogue_slice<FMT, kEpiDown, BN>(g2, &tmap_y, te, mt, 0, nch, c_lo, ew, q, lane, gact2, 1.0f, epi_tiles,
                                          r_tab, y_stage, 1, ypar, hmax, r0, r1, r2, r3, ltok, lw);
      }
    }
    if (lane == 0) tc::bulk_wait_all();   // tensor stores done before the CTA exits
  }

  __syncwarp();
  __threadfence();   // this CTA's output reductions before the count below
  __syncthreads();
  if (*abort) {
    // let copies and MMAs already in flight land before the memory goes away
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000LL) {
    }
  }
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem, C::kTmemCols);
  if constexpr (GATHER) {
    if (f.out) {
      // the CTA that finishes last rounds the fp32 output rows to bf16
      __shared__ int last;
      if (threadIdx.x == 0) last = atomicAdd(f.done, 1) == (int)gridDim.x - 1;
      __syncthreads();
      if (last) {
        __threadfence();
        const int64_t n8 = f.T * (g2.R / 8);
        for (int64_t i = threadIdx.x; i < n8; i += blockDim.x) {
          const float4 a = __ldcg(reinterpret_cast<const float4*>(g2.out32) + 2 * i);
          const float4 b = __ldcg(reinterpret_cast<const float4*>(g2.out32) + 2 * i + 1);
          uint4 o;
          o.x = (uint32_t)f32_to_bf16_rn(a.x) | ((uint32_t)f32_to_bf16_rn(a.y) << 16);
          o.y = (uint32_t)f32_to_bf16_rn(a.z) | ((uint32_t)f32_to_bf16_rn(a.w) << 16);
          o.z = (uint32_t)f32_to_bf16_rn(b.x) | ((uint32_t)f32_to_bf16_rn(b.y) << 16);
          o.w = (uint32_t)f32_to_bf16_rn(b.z) | ((uint32_t)f32_to_bf16_rn(b.w) << 16);
          reinterpret_cast<uint4*>(f.out)[i] = o;
        }
      }
    }
  }
}

// ------------------------------------------------------------- tensor maps --
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

// Rows of `row_bytes` bytes, box = 128 bytes x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows) {
  EncodeTiled fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale-factor blocks as rows of a 2D map (128 x 32-bit = one 512-byte block
// per row), so a stage's groups arrive with one tensor copy.
bool make_sf_map(CUtensorMap* m, const void* base, int64_t nblocks, int box_blocks) {
  EncodeTiled fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {128u, (cuuint64_t)nblocks};
  cuuint64_t strides[1] = {512u};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_blocks};
  cuuint32_t es[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// y_perm rows for the down projection's tensor stores: box 32 outputs x 16 slots.
bool make_y_map(CUtensorMap* m, void* base, int64_t rows, int64_t ld) {
  EncodeTiled fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)ld, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {32u, 16u};
  cuuint32_t es[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// CTA pairs (MOE_OPT_GEMM_PAIR): 0 never, 1 wherever the tile allows, 2 where
// a tile's K loop has at least kPairMinStages stages -- shorter loops lose
// more to the pair's cross-CTA hand-offs than they gain from staging half of
// the token tile per CTA.
int g_gemm_pairs = 2;
constexpr int kPairMinStages = 12;

template <int FMT, int EPI, int BN, bool PAIR>
cudaError_t launch_cfg(const GemmArgs& g, const void* a_base, int64_t a_rows, const void* b_base, int64_t b_rows,
                       int num_sms, cudaStream_t s) {
  using C = Cfg<FMT, EPI, BN, PAIR>;
  using F = FmtTraits<FMT>;
  CUtensorMap ma, msfa, msfb, my;
  TokenMaps mb;
  memset(&msfa, 0, sizeof(msfa));
  memset(&msfb, 0, sizeof(msfb));
  memset(&my, 0, sizeof(my));
  if (EPI == kEpiDown && (g.y_rows < 1 || !make_y_map(&my, g.y, g.y_rows, g.ldy))) return cudaErrorInvalidValue;
  const int64_t rb = FMT == kFmtBF16 ? 2 * (int64_t)g.K : (FMT == MOE_FMT_FP8 ? g.K : g.K / 2);
  if (!make_map(&ma, a_base, a_rows, rb, 128)) return cudaErrorInvalidValue;
  // token boxes of 16, 32, 64, 128 and 256 rows, capped at the rows one CTA stages
  constexpr int kBRows = PAIR ? BN / 2 : BN;
  for (int i = 0; i < 5; ++i)
    if (!make_map(&mb.m[i], b_base, b_rows, rb, (16 << i) < kBRows ? (16 << i) : kBRows)) return cudaErrorInvalidValue;
  if (PAIR && F::kBs) {
    const int64_t groups = g.K / F::kBs / 4;  // 512-byte blocks per 128 rows
    if (!make_sf_map(&msfa, g.w_sf, a_rows / 128 * groups, F::kGroups)) return cudaErrorInvalidValue;
    if (!make_sf_map(&msfb, g.b_sf, b_rows / 128 * groups, F::kGroups)) return cudaErrorInvalidValue;
  }
  auto kern = grouped_gemm_kernel<FMT, EPI, BN, PAIR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  if constexpr (PAIR) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many pairs as can be resident at once
    static int max_pairs[16];
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 16) return cudaErrorInvalidDevice;
    if (max_pairs[dev] == 0) {
      cfg.gridDim = dim3((unsigned)(num_sms & ~1));
      cfg.numAttrs = 1;  // the cluster shape alone
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
      if (e != cudaSuccess) return e;
      if (n < 1) return cudaErrorInvalidConfiguration;
      max_pairs[dev] = n;
    }
    const int pairs = max_pairs[dev] < num_sms / 2 ? max_pairs[dev] : num_sms / 2;
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, ma, mb, msfa, msfb, my, g);
    if (e != cudaSuccess) return e;
  } else {
    e = launch_pdl(kern, dim3(num_sms), dim3(C::kThreads), C::kSmem, s, ma, mb, msfa, msfb, my, g);
    if (e != cudaSuccess) return e;
  }
  count_launches(1);
  return cudaGetLastError();
}

template <int FMT, int EPI>
cudaError_t launch_bn(const GemmArgs& g, int bn, const void* a, int64_t ar, const void* b, int64_t br, int sms,
                      cudaStream_t s) {
  if constexpr (FMT != kFmtBF16) {   // (no pair form of the bf16 MMA here)
    const bool pairs = EPI != kEpiLogits && g.R % 256 == 0 && sms >= 2 &&
                       (g_gemm_pairs == 1 || (g_gemm_pairs == 2 && g.K / FmtTraits<FMT>::kBK >= kPairMinStages));
    if (bn == 256 && pairs) return launch_cfg<FMT, EPI, 256, true>(g, a, ar, b, br, sms, s);
    if (bn == 192 && pairs) return launch_cfg<FMT, EPI, 192, true>(g, a, ar, b, br, sms, s);
  }
  if (bn == 256) return launch_cfg<FMT, EPI, 256, false>(g, a, ar, b, br, sms, s);
  if (bn == 192) return launch_cfg<FMT, EPI, 192, false>(g, a, ar, b, br, sms, s);
  if (bn == 64) return launch_cfg<FMT, EPI, 64, false>(g, a, ar, b, br, sms, s);
  return launch_cfg<FMT, EPI, 128, false>(g, a, ar, b, br, sms, s);
}

template <int FMT>
cudaError_t launch_epi(const GemmArgs& g, int epi, int bn, const void* a, int64_t ar, const void* b, int64_t br,
                       int sms, cudaStream_t s) {
  if (epi == kEpiDown) return launch_bn<FMT, kEpiDown>(g, bn, a, ar, b, br, sms, s);
  if (epi == kEpiUpF32) return launch_bn<FMT, kEpiUpF32>(g, bn, a, ar, b, br, sms, s);
  if (FMT == MOE_FMT_FP8) return cudaErrorInvalidValue;
  return launch_bn<FMT, kEpiUpQuant>(g, bn, a, ar, b, br, sms, s);
}

template <int FMT, int BN, bool GATHER>
cudaError_t launch_fused_cfg(const GemmArgs& g1, const GemmArgs& g2, const FusedArgs& f, const void* w13,
                             int64_t w13_rows, const void* w2, int64_t w2_rows, const void* xq, const void* hq,
                             int num_sms, cudaStream_t s) {
  using C = Cfg<FMT, kEpiUpQuant, BN, false>;
  CUtensorMap m13, m2, my;
  TokenMaps mx, mh;
  if (g2.y_rows < 1 || !make_y_map(&my, g2.y, g2.y_rows, g2.ldy)) return cudaErrorInvalidValue;
  if (!make_map(&m13, w13, w13_rows, g1.K / 2, 128)) return cudaErrorInvalidValue;
  if (!make_map(&m2, w2, w2_rows, g2.K / 2, 128)) return cudaErrorInvalidValue;
  for (int i = 0; i < 5; ++i) {
    const int rows = (16 << i) < BN ? (16 << i) : BN;
    if (!make_map(&mx.m[i], xq, f.P, g1.K / 2, rows)) return cudaErrorInvalidValue;
    if (!make_map(&mh.m[i], hq, f.P, g2.K / 2, rows)) return cudaErrorInvalidValue;
  }
  auto kern = fused_ffn_kernel<FMT, BN, GATHER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FusedCfg<FMT, BN>::kSmem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(num_sms), dim3(C::kThreads), FusedCfg<FMT, BN>::kSmem, s, m13, mx, m2, mh, my, g1, g2, f);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------ router with top-k --
// Router logits and the top-k of every token in one kernel for batches large
// enough that the 128-token tiles fill the SMs: 128 tokens of x on the MMA's
// M side, all E experts of Wr on its N side (bf16 kind::f16, fp32
// accumulation over all of H, E a multiple of 16 up to 256), so each
// accumulator lane holds one token's E logits.  The epilogue thread of lane
// t reads its row from tensor memory 16 columns at a time, adds the bias and
// keeps the k largest (descending, ties to the lower expert) in registers,
// while the other accumulator buffer takes the next tile's MMAs; the weights
// are exp(L_j - L_0) / sum over the k picks.  Smaller batches take the
// router GEMM split along H and the top-k kernel: with fewer tiles than SMs
// one CTA per tile streams its operands too slowly, and a cluster sharing
// each tile (partials exchanged through distributed shared memory) measured
// slower than the two kernels.
constexpr int kRouteTopkMaxK = 16;   // k beyond this takes the router GEMM and topk_kernel
constexpr int kRouteStages = 4;

template <int NE>
struct RouteTopkCfg {
  static constexpr int kA = 128 * 128;   // 128 token rows x 64 bf16
  static constexpr int kB = NE * 128;    // NE expert rows x 64 bf16
  static constexpr int kStage = (kA + kB + 1023) / 1024 * 1024;
  static constexpr int kSmem = kRouteStages * kStage + 1024 /*align*/ + 1024 /*barriers*/;
  static constexpr int kThreads = 6 * 32;   // producer, MMA, 4 epilogue warps
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(2 * NE <= 512, "two accumulators in tensor memory");
};

// Keeps tv/te (descending, an empty slot holding index -1) as the KMAX
// largest of the logits seen, offered in increasing expert order: only a
// strictly larger logit moves ahead, so an equal one stays behind the lower
// expert index; an empty slot takes anything.
template <int KMAX>
__device__ __forceinline__ void topk_insert(float (&tv)[KMAX], int (&te)[KMAX], float l, int e) {
  if (l > tv[KMAX - 1] || te[KMAX - 1] < 0) {
    float cv = l;
    int ce = e;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (cv > tv[j] || te[j] < 0) {
        const float sv = tv[j];
        const int se = te[j];
        tv[j] = cv;
        te[j] = ce;
        cv = sv;
        ce = se;
      }
    }
  }
}

// KMAX: k rounded up to a power of two; the epilogue thread keeps the KMAX
// largest logits sorted and reports the first k.
template <int NE, int KMAX>
__global__ void __launch_bounds__(RouteTopkCfg<NE>::kThreads, 1)
    router_topk_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_wr,
                       const float* __restrict__ bias, int64_t T, int H, int E, int k,
                       float* __restrict__ logits_out, int32_t* __restrict__ idx, float* __restrict__ wout,
                       int32_t* status, long long wait_lim) {
  using C = RouteTopkCfg<NE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ctrl = smem + kRouteStages * C::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + kRouteStages;
  uint64_t* tfull = empty + kRouteStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRouteStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&tfull[a], 1);
      tc::mbar_init(&tempty[a], 4);
    }
    *abort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&tmap_x);
    tc::prefetch_tmap(&tmap_wr);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 2 * NE);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // x comes from the caller's earlier work
  pdl_trigger();
  const int ntiles = (int)((T + 127) / 128);
  const int nkb = H / 64;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    for (int t = blockIdx.x; t < ntiles && !tc::aborted(abort); t += gridDim.x) {
      for (int kb = 0; kb < nkb; ++kb) {
        if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort, wait_lim)) {
          if (lane == 0) raise_status(status, MOE_ERR_TIMEOUT);
          *abort = 1;
          break;
        }
        if (tc::elect_one()) {
          uint8_t* st = smem + stage * C::kStage;
          tc::mbar_expect_tx(&full[stage], (uint32_t)(C::kA + E * 128));
          tc::tma_load_2d(st, &tmap_x, &full[stage], kb * 128, t * 128);
          tc::tma_load_2d(st + C::kA, &tmap_wr, &full[stage], kb * 128, 0);
        }
        __syncwarp();
        if (++stage == kRouteStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint32_t idesc = tc::idesc_bf16((uint32_t)E);
    for (int t = blockIdx.x; t < ntiles && !tc::aborted(abort); t += gridDim.x) {
      if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1u, abort, wait_lim)) {
        if (lane == 0) raise_status(status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
      tc::fence_after_sync();
      const uint32_t d = tmem + (uint32_t)(acc * NE);
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!tc::mbar_wait(&full[stage], phase, abort, wait_lim)) {
          if (lane == 0) raise_status(status, MOE_ERR_TIMEOUT);
          *abort = 1;
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (tc::elect_one()) {
          uint8_t* st = smem + stage * C::kStage;
          const uint64_t da0 = tc::desc_sw128(tc::smem_u32(st)), db0 = tc::desc_sw128(tc::smem_u32(st + C::kA));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(d, da0 + (uint64_t)(kk * 2), db0 + (uint64_t)(kk * 2), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          tc::mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kRouteStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (tc::elect_one()) tc::mma_commit(&tfull[acc]);
      __syncwarp();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;   // tensor-memory lane quarter: tokens 32q .. 32q + 31 of the tile
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      if (!tc::mbar_wait(&tfull[acc], acc_phase, abort, wait_lim)) {
        if (lane == 0) raise_status(status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
      tc::fence_after_sync();
      const int64_t tok = (int64_t)t * 128 + q * 32 + lane;
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * NE);
      // the KMAX largest so far, descending; an empty slot holds index -1
      float tv[KMAX];
      int te[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        tv[j] = -INFINITY;
        te[j] = -1;
      }
      bool bad = false;
      for (int c0 = 0; c0 < E; c0 += 16) {
        float v[16];
        tc::tmem_ld16(base + (uint32_t)c0, v);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int e = c0 + c;
          const float l = v[c] + (bias ? __ldg(bias + e) : 0.0f);
          if (logits_out && tok < T) logits_out[tok * E + e] = l;
          if (isnan(l)) bad = true;
          topk_insert<KMAX>(tv, te, l, e);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
      if (tok >= T) continue;
      if (!(tv[0] > -INFINITY)) bad = true;
      if (bad) {
        raise_status(status, MOE_ERR_DEVICE_FAULT);
        for (int j = 0; j < k; ++j) {
          idx[tok * k + j] = j;
          wout[tok * k + j] = 0.0f;
        }
        continue;
      }
      float ex[KMAX], sum = 0.0f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k) {
          ex[j] = expf(tv[j] - tv[0]);
          sum += ex[j];
        }
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k) {
          idx[tok * k + j] = te[j];
          wout[tok * k + j] = __fdiv_rn(ex[j], sum);
        }
    }
  }
  __syncwarp();
  __syncthreads();
  if (*abort) {
    const long long w0 = clock64();
    while (clock64() - w0 < 2000000LL) {
    }
  }
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem, 2 * NE);
}

}  // namespace

cudaError_t launch_grouped_gemm(const GemmArgs& g, int epi, int bn, const void* a_base, int64_t a_rows,
                                const void* b_base, int64_t b_rows, int num_sms, cudaStream_t s) {
  switch (g.fmt) {
    case MOE_FMT_NVFP4: return launch_epi<MOE_FMT_NVFP4>(g, epi, bn, a_base, a_rows, b_base, b_rows, num_sms, s);
    case MOE_FMT_MXFP4: return launch_epi<MOE_FMT_MXFP4>(g, epi, bn, a_base, a_rows, b_base, b_rows, num_sms, s);
    case MOE_FMT_FP8: return launch_epi<MOE_FMT_FP8>(g, epi, bn, a_base, a_rows, b_base, b_rows, num_sms, s);
    case kFmtBF16: return launch_epi<kFmtBF16>(g, epi, bn, a_base, a_rows, b_base, b_rows, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fused_ffn(const GemmArgs& g1, const GemmArgs& g2, const FusedArgs& f, const void* w13,
                             int64_t w13_rows, const void* w2, int64_t w2_rows, const void* xq, const void* hq,
                             int num_sms, cudaStream_t s) {
  if (g1.E > kFusedMaxE || g1.fmt != g2.fmt) return cudaErrorInvalidValue;
  // gather mode: a tile holds at most kGatherMaxT rows (T <= kGatherMaxT),
  // and its tokens come from perm_token or from the slots' experts
  if (f.xg && (f.T > kGatherMaxT || f.S > kGatherMaxS || !f.xsl || (!f.perm_token && !f.slot_expert) || f.k < 1))
    return cudaErrorInvalidValue;
  if (f.out && (!f.xg || !f.slot_expert || !g2.out32 || !f.done || !f.topk_w)) return cudaErrorInvalidValue;
  const FusedArgs& fa = f;
  switch (g1.fmt) {
    case MOE_FMT_NVFP4:
      return fa.xg ? launch_fused_cfg<MOE_FMT_NVFP4, 64, true>(g1, g2, fa, w13, w13_rows, w2, w2_rows, xq, hq, num_sms, s)
                   : launch_fused_cfg<MOE_FMT_NVFP4, 64, false>(g1, g2, fa, w13, w13_rows, w2, w2_rows, xq, hq,
                                                                num_sms, s);
    case MOE_FMT_MXFP4:
      return fa.xg ? launch_fused_cfg<MOE_FMT_MXFP4, 64, true>(g1, g2, fa, w13, w13_rows, w2, w2_rows, xq, hq, num_sms, s)
                   : launch_fused_cfg<MOE_FMT_MXFP4, 64, false>(g1, g2, fa, w13, w13_rows, w2, w2_rows, xq, hq,
                                                                num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

bool tensor_maps_available() { return encode_fn() != nullptr; }

long long tc_default_wait_cycles() { return tc::kDefaultWaitCycles; }

void set_gemm_pairs(int mode) { g_gemm_pairs = mode; }

static int g_early_weights = 1;  // MOE_OPT_EARLY_WEIGHTS
void set_early_weights(int mode) { g_early_weights = mode; }
int early_weights() { return g_early_weights; }


int router_ksplit(int64_t T, int E, int H, int num_sms) {
  const int64_t items = (T + kRouterBN - 1) / kRouterBN * (E / 128);
  int ks = items > 0 ? (int)(num_sms / items) : 1;
  ks = ks < 1 ? 1 : (ks > kRouterMaxSplit ? kRouterMaxSplit : ks);
  while (ks > 1 && (H / 64) / ks < 4) --ks;  // at least four 64-wide K blocks per split
  return ks;
}

cudaError_t launch_router_gemm(const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias, int E,
                               float* logits_parts, int64_t part_stride, int ksplit, int32_t* status, int num_sms,
                               cudaStream_t s) {
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.fmt = kFmtBF16;
  g.E = 1;
  g.K = H;
  g.R = E;
  g.dense_rows = T;
  g.logits = logits_parts;
  g.bias = bias;
  g.ksplit = ksplit;
  g.split_stride = part_stride;
  g.ldy = E;
  g.status = status;
  g.wait_cycles = wait_cycles();
  const int64_t items = (T + kRouterBN - 1) / kRouterBN * (E / 128) * ksplit;
  const int grid = (int)(items < num_sms ? items : num_sms);
  return launch_cfg<kFmtBF16, kEpiLogits, kRouterBN, false>(g, wr, E, x, T, grid, s);
}

bool router_topk_fits(int64_t T, int E, int H, int k, int num_sms) {
  return T >= 128 && (T + 127) / 128 >= num_sms / 2 && E >= 16 && E <= 256 && E % 16 == 0 && H % 64 == 0 && k >= 1 &&
         k <= kRouteTopkMaxK && tensor_maps_available();
}

cudaError_t launch_router_topk(const uint16_t* x, int64_t T, int H, const uint16_t* wr, const float* bias, int E,
                               int k, float* logits_out, int32_t* idx, float* w, int32_t* status, int num_sms,
                               cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (!router_topk_fits(T, E, H, k, num_sms)) return cudaErrorInvalidValue;
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, T, 2 * (int64_t)H, 128)) return cudaErrorInvalidValue;
  if (!make_map(&mw, wr, E, 2 * (int64_t)H, E)) return cudaErrorInvalidValue;
  const int64_t ntiles = (T + 127) / 128;
  const int grid = (int)(ntiles < num_sms ? ntiles : num_sms);
  const long long lim = wait_cycles();
  cudaError_t e = cudaErrorInvalidValue;
#define MOE_RT(NE, KM)                                                                                      \
  {                                                                                                         \
    auto kern = router_topk_kernel<NE, KM>;                                                                 \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, RouteTopkCfg<NE>::kSmem);    \
    if (e == cudaSuccess)                                                                                   \
      e = launch_pdl(kern, dim3(grid), dim3(RouteTopkCfg<NE>::kThreads), RouteTopkCfg<NE>::kSmem, s, mx, mw, \
                     bias, T, H, E, k, logits_out, idx, w, status, lim);                                    \
  }
#define MOE_RT_K(NE)                 \
  if (k <= 1) MOE_RT(NE, 1)          \
  else if (k <= 2) MOE_RT(NE, 2)     \
  else if (k <= 4) MOE_RT(NE, 4)     \
  else if (k <= 8) MOE_RT(NE, 8)     \
  else MOE_RT(NE, 16)
  if (E <= 128) {
    MOE_RT_K(128)
  } else {
    MOE_RT_K(256)
  }
#undef MOE_RT_K
#undef MOE_RT
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- planning --
// One block: padded offsets (every expert segment starts on a multiple of 128
// rows) and the tile list (expert, first padded row, valid rows, first slot).
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ offsets, int E, int64_t S, int bn,
                                                    int32_t* __restrict__ poff, TileEntry* __restrict__ tiles,
                                                    int32_t* __restrict__ num_tiles, int max_tiles,
                                                    int32_t* status) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();

  __shared__ int32_t s_pad[1024], s_til[1024];
  __shared__ int bad;
  const int e = threadIdx.x;
  if (e == 0) bad = (offsets[0] != 0 || offsets[E] != S) ? 1 : 0;
  __syncthreads();
  int32_t n = 0, pad = 0, til = 0, o0 = 0;
  if (e < E) {
    o0 = offsets[e];
    n = offsets[e + 1] - o0;
    if (n < 0) {
      bad = 1;
      n = 0;
    }
    pad = (n + 127) / 128 * 128;
    til = (n + bn - 1) / bn;
  }
  s_pad[e] = pad;
  s_til[e] = til;
  __syncthreads();
  // inclusive Hillis-Steele scans (E <= 1024)
  for (int d = 1; d < 1024; d <<= 1) {
    const int32_t a = e >= d ? s_pad[e - d] : 0, b = e >= d ? s_til[e - d] : 0;
    __syncthreads();
    s_pad[e] += a;
    s_til[e] += b;
    __syncthreads();
  }
  const int32_t pbase = s_pad[e] - pad, tbase = s_til[e] - til;
  if (e < E) {
    poff[e] = pbase;
    for (int j = 0; j < til && tbase + j < max_tiles; ++j) {
      TileEntry te;
      te.e = e;
      te.row0 = pbase + j * bn;
      te.nvalid = min(bn, n - j * bn);
      te.p0 = o0 + j * bn;
      tiles[tbase + j] = te;
    }
  }
  __syncthreads();
  if (e == E - 1) {
    poff[E] = s_pad[e];
    *num_tiles = bad ? 0 : min(s_til[e], max_tiles);
    if (bad) raise_status(status, MOE_ERR_DEVICE_FAULT);
  }
}

cudaError_t launch_plan(const int32_t* offsets, int E, int64_t S, int bn, int32_t* poff, TileEntry* tiles,
                        int32_t* num_tiles, int max_tiles, int32_t* status, cudaStream_t s) {
  cudaError_t e = launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, s, offsets, E, S, bn, poff, tiles, num_tiles,
                             max_tiles, status);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ---------------------------------------------------- padded quantisation --
// The tile plan inside one block of 256 threads: padded offsets into s_poff
// [E+1] (shared memory) and, when `write`, into plan.poff together with the
// tile list -- what plan_kernel computes.  Every thread calls it.
__device__ void plan_in_block(const int32_t* __restrict__ offsets, int E, int64_t S, const PlanOut& plan, bool write,
                              int32_t* s_poff, int32_t* status) {
  __shared__ int32_t warp_tot[8];
  const int per = (E + 255) / 256;
  const int e0 = threadIdx.x * per;
  // every offset is read once, all reads in flight together; the checks
  // (offsets[0] == 0, non-decreasing, offsets[E] == S) are or-reduced at the
  // first barrier of the scans
  int mybad = 0;
  int32_t pad_mine = 0, til_mine = 0;
  if (e0 < E) {
    int32_t prev = __ldg(offsets + e0);
    if (e0 == 0 && prev != 0) mybad = 1;
    for (int e = e0; e < e0 + per && e < E; ++e) {
      const int32_t hi = __ldg(offsets + e + 1);
      int32_t n = hi - prev;
      prev = hi;
      if (n < 0) {
        mybad = 1;
        n = 0;
      }
      if (e + 1 == E && hi != S) mybad = 1;
      pad_mine += (n + 127) / 128 * 128;
      til_mine += (n + plan.bn - 1) / plan.bn;
    }
  }
  // two exclusive scans over the 256 threads
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t res[2], tot[2];
  const int32_t val[2] = {pad_mine, til_mine};
  int bad = 0;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    int32_t incl = val[q];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (q == 0) bad = __syncthreads_or(mybad);
    else __syncthreads();
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int32_t base = 0, sum = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      base += w < warp ? warp_tot[w] : 0;
      sum += warp_tot[w];
    }
    res[q] = incl - val[q] + base;
    tot[q] = sum;
  }
  int32_t pbase = res[0], tbase = res[1];
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int32_t o = __ldg(offsets + e);
    const int32_t n = max(0, __ldg(offsets + e + 1) - o);
    s_poff[e] = pbase;
    const int til = (n + plan.bn - 1) / plan.bn;
    if (write) {
      plan.poff[e] = pbase;
      for (int j = 0; j < til && tbase + j < plan.max_tiles; ++j) {
        TileEntry te;
        te.e = e;
        te.row0 = pbase + j * plan.bn;
        te.nvalid = min(plan.bn, n - j * plan.bn);
        te.p0 = o + j * plan.bn;
        plan.tiles[tbase + j] = te;
      }
    }
    pbase += (n + 127) / 128 * 128;
    tbase += til;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    s_poff[E] = tot[0];
    if (write) {
      plan.poff[E] = tot[0];
      *plan.ntiles = bad ? 0 : min(tot[1], plan.max_tiles);
      if (bad) raise_status(status, MOE_ERR_DEVICE_FAULT);
    }
  }
  __syncthreads();
}

// Quantises activation rows into the padded, blocked layout the GEMM reads.
// One warp per slot p: its source row is x[perm_token[p]] (bf16, SRC_X) or
// h32[padded row] (fp32), its destination the padded row poff[e] + (p -
// offsets[e]); lane l quantises scale blocks l, l + 32, ... of the row.
template <int FMT, bool SRC_X>
__global__ void __launch_bounds__(256) quant_padded_kernel(QuantPaddedArgs a) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();
  if (a.zero && blockIdx.x == 0)
    for (int i = threadIdx.x; i < a.nzero; i += blockDim.x) a.zero[i] = 0;

  constexpr int bs = FMT == MOE_FMT_MXFP4 ? 32 : 16;
  const int nb = a.K / bs;
  const int lane = threadIdx.x & 31;
  const float scale = act_scale_of(FMT, a.scale, a.amax);
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  // With a.plan.bn > 0 every block derives the padded offsets from the
  // offsets itself (and block 0 also writes them and the tile list), so the
  // tile plan needs no launch of its own.
  __shared__ int32_t s_poff[1025];
  const int32_t* poff = a.poff;
  const int64_t p_first = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  // the first slot's token is read before the plan, in flight with its offsets
  int t_first = -1;
  if (SRC_X && lane == 0 && p_first < a.S) t_first = __ldg(a.perm_token + p_first);
  if (SRC_X && a.plan.bn > 0) {
    plan_in_block(a.offsets, a.E, a.S, a.plan, blockIdx.x == 0, s_poff, a.status);
    poff = s_poff;
  }
  for (int64_t p = p_first; p < a.S; p += warps) {
    int64_t row = -1;
    int t = -1;
    if (lane == 0) {
      const int e = segment_of(a.offsets, a.E, (int)p);
      const int32_t o = __ldg(a.offsets + e);
      row = (int64_t)poff[e] + (p - o);
      if (row < 0 || row >= a.P || p < o) row = -1;
      if (SRC_X) {
        t = p == p_first ? t_first : __ldg(a.perm_token + p);
        if (t < 0 || t >= a.T) row = -1;
      }
    }
    row = __shfl_sync(0xffffffffu, row, 0);
    t = __shfl_sync(0xffffffffu, t, 0);
    if (row < 0) {
      if (lane == 0) raise_status(a.status, MOE_ERR_DEVICE_FAULT);
      continue;
    }
    for (int b = lane; b < nb; b += 32) {
      float v[bs];
      if (SRC_X) {
        load_bf16_block<bs>(a.x + (int64_t)t * a.K + b * bs, v);
      } else {
        const float* src = a.h32 + row * a.K + b * bs;
#pragma unroll
        for (int i = 0; i < bs; i += 4) {
          const float4 w = *reinterpret_cast<const float4*>(src + i);
          v[i] = w.x;
          v[i + 1] = w.y;
          v[i + 2] = w.z;
          v[i + 3] = w.w;
        }
      }
      quant_block_store<FMT>(v, scale, a.codes, a.sf, row, b, nb, a.K);
    }
  }
}

// x rows by token: with a per-tensor (or per-block) activation scale a
// token's quantised row is the same in each of its k slots, so one warp
// quantises token t once -- lane l owns 64 consecutive elements of each
// 2048-element stretch -- and writes the codes and scales to the padded rows
// of the slots inv_perm[t * k + j].
template <int FMT>
__global__ void __launch_bounds__(256) quant_tokens_kernel(QuantPaddedArgs a) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();
  if (a.zero && blockIdx.x == 0)
    for (int i = threadIdx.x; i < a.nzero; i += blockDim.x) a.zero[i] = 0;

  __shared__ uint4 tbuf[8][TokenQuant<FMT>::kWarpBuf];  // per warp: the stretch's codes, for the reorder
  const float scale = act_scale_of(FMT, a.scale, a.amax);
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  // NVFP4: the multiplier r = 1 / (dec(sc) g) of every non-negative scale code
  __shared__ float r_tab[128];
  if (FMT == MOE_FMT_NVFP4) {
    for (int i = threadIdx.x; i < 128; i += blockDim.x) r_tab[i] = nvfp4_multiplier((uint32_t)i, scale);
    __syncthreads();
  }
  // padded row of the slot of (token t, pick j): -1 for a dropped slot, -2 if
  // the permutation is inconsistent
  auto resolve = [&](int64_t t, int j) -> int64_t {
    const int32_t p = __ldg(a.inv_perm + t * a.k + j);
    if (p >= a.S) return -2;
    if (p < 0) return -1;
    int e;
    if (a.slot_expert) {
      e = __ldg(a.slot_expert + t * a.k + j);
      if (e < 0 || e >= a.E) return -2;
    } else {
      e = segment_of(a.offsets, a.E, p);
    }
    const int32_t o = __ldg(a.offsets + e), o1 = __ldg(a.offsets + e + 1);
    const int64_t row = (int64_t)__ldg(a.poff + e) + (p - o);
    const bool ok = row >= 0 && row < a.P && p >= o && p < o1;
    if (ok && a.w_perm) a.w_perm[p] = __ldg(a.topk_w + t * a.k + j);   // the slot's routing weight
    return ok ? row : -2;
  };
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < a.T; t += warps)
    quant_token_slots<FMT>(a.x + t * a.K, a.K, a.k, scale, r_tab, tbuf[threadIdx.x >> 5],
                           [&](int j) { return resolve(t, j); }, a.codes, a.sf, a.status);
}

// x of a small batch into the gather layout (quant_token_gather): a warp per
// token, whatever the routing.
template <int FMT>
__global__ void __launch_bounds__(256) quant_gather_kernel(const uint16_t* __restrict__ x, int64_t T, int K,
                                                           GatherQuant q) {
  pdl_wait();  // inputs come from the previous kernels
  pdl_trigger();
  constexpr int bs = FMT == MOE_FMT_MXFP4 ? 32 : 16;
  __shared__ float r_tab[128];
  const float scale = act_scale_of(FMT, q.scale, q.amax);
  if (FMT == MOE_FMT_NVFP4 && threadIdx.x < 128) r_tab[threadIdx.x] = nvfp4_multiplier(threadIdx.x, scale);
  __syncthreads();
  if (q.zero && blockIdx.x == 0)
    for (int i = threadIdx.x; i < q.nzero; i += blockDim.x) q.zero[i] = 0;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t < T)
    quant_token_gather<FMT>(x + t * K, K, scale, r_tab, q.xg + t * 8 * (K / 2), q.xsl + t * (K / (4 * bs)) * 16);
}

cudaError_t launch_quant_gather(int fmt, const uint16_t* x, int64_t T, int K, const GatherQuant& q, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (T > kGatherMaxT || K % 256 != 0) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)((T + 7) / 8));
  cudaError_t e;
  if (fmt == MOE_FMT_NVFP4)
    e = launch_pdl(quant_gather_kernel<MOE_FMT_NVFP4>, grid, dim3(256), 0, s, x, T, K, q);
  else if (fmt == MOE_FMT_MXFP4)
    e = launch_pdl(quant_gather_kernel<MOE_FMT_MXFP4>, grid, dim3(256), 0, s, x, T, K, q);
  else
    return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_quant_padded(const QuantPaddedArgs& a, bool src_x, int fmt, int num_sms, cudaStream_t s) {
  if (a.S == 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  if (src_x && a.inv_perm && a.K % 64 == 0 && fmt != kFmtBF16) {
    const int64_t blocks = (a.T + 7) / 8;
    const int grid = (int)(blocks < (int64_t)num_sms * 8 ? blocks : (int64_t)num_sms * 8);
    switch (fmt) {
      case MOE_FMT_NVFP4: e = launch_pdl(quant_tokens_kernel<MOE_FMT_NVFP4>, dim3(grid), dim3(256), 0, s, a); break;
      case MOE_FMT_MXFP4: e = launch_pdl(quant_tokens_kernel<MOE_FMT_MXFP4>, dim3(grid), dim3(256), 0, s, a); break;
      case MOE_FMT_FP8: e = launch_pdl(quant_tokens_kernel<MOE_FMT_FP8>, dim3(grid), dim3(256), 0, s, a); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
  }
  const int64_t blocks = (a.S + 7) / 8;
  const int grid = (int)(blocks < (int64_t)num_sms * 8 ? blocks : (int64_t)num_sms * 8);
#define MOE_QP(F)                                                                  \
  e = src_x ? launch_pdl(quant_padded_kernel<F, true>, dim3(grid), dim3(256), 0, s, a) \
            : launch_pdl(quant_padded_kernel<F, false>, dim3(grid), dim3(256), 0, s, a);
  switch (fmt) {
    case MOE_FMT_NVFP4: MOE_QP(MOE_FMT_NVFP4) break;
    case MOE_FMT_MXFP4: MOE_QP(MOE_FMT_MXFP4) break;
    case MOE_FMT_FP8: MOE_QP(MOE_FMT_FP8) break;
    case kFmtBF16: MOE_QP(kFmtBF16) break;
    default: return cudaErrorInvalidValue;
  }
#undef MOE_QP
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace moe
