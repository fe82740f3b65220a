// Small-batch grouped expert FFN: every active expert's weights are streamed
// once from HBM, dequantised in registers and multiplied with the expert's
// (at most 8 per pass) token rows.
//
// This is the decode half of the prefill/decode kernel split that the
// atomicmilkshake/FreeToken fork README describes ("Quant types": MMQ for
// prefill, MMVQ for decode; "Known limits": a W4A8 decode kernel over the
// per-expert slot pool).  Here the "vector" side is up to eight token columns,
// so the multiply runs on mma.sync m16n8k16 with fp32 accumulation: the
// weights stream through 16-byte loads per lane, each byte of two e2m1 codes
// becomes an f16x2 (bf16x2 for MXFP4) multiplied by its block scale -- a
// product that is exact in 16 bits -- and lands directly in the A fragment.
// The token rows are converted once per CTA into B fragments in shared memory.
//
// K order.  A dot product does not depend on the order of its terms, so
// within each 128-element chunk lane q (= lane % 4) of a row quad owns the
// physical elements [32q, 32q + 32): MMA j (0..7) takes elements 32q + 4j
// + {0,1} as its k-pair 2q and 32q + 4j + {2,3} as its k-pair 2q + 8.  The B
// fragments in shared memory use the same map.  A lane's 16 bytes of NVFP4
// codes then hold exactly its fragment elements and their two scale blocks.
//
// Streaming: the kernel is persistent (one CTA per SM).  Work items are 64
// rows of one expert's weights for one group of at most 8 of its tokens; a
// CTA takes a contiguous, balanced range of items.  A producer warp moves
// each item's weights into a deep shared-memory ring with TMA (128-byte
// swizzled boxes of 64 rows x 128 bytes) plus bulk copies of the scale
// blocks, so each SM keeps on the order of 150 KB of weight traffic in
// flight; four consumer warps (16 rows each) read their fragments from the
// ring, dequantise and multiply.  Activations become B fragments once per
// token group and are reused across that group's row items.
//
// Rows: W13 rows are PREPARED (row 2i gate i, row 2i+1 up i), so a gate/up
// pair sits in lanes l and l ^ 4 and the SwiGLU epilogue needs one shuffle.
#include <cuda.h>

#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace moe {

constexpr int kNT = kGemvTokens;
constexpr int kGemvConsumers = 4;   // consumer warps, 16 rows each
constexpr int kItemRows = 64;

__device__ __forceinline__ int bfrag_index(int n, int k) {
  const int c = k >> 7, kk = k & 127;
  const int q = kk >> 5, r = kk & 31;
  const int j = r >> 2, p = (r >> 1) & 1, t = r & 1;
  const int lane = n * 4 + q;
  return ((((c * 8 + j) * 32) + lane) << 2) + p * 2 + t;
}

__device__ __forceinline__ uint16_t f32_to_f16_rn(float f) {
  uint16_t h;
  asm("cvt.rn.f16.f32 %0, %1;" : "=h"(h) : "f"(f));
  return h;
}

template <bool BF16>
__device__ __forceinline__ uint16_t to_mma_elem(float f) {
  return BF16 ? f32_to_bf16_rn(f) : f32_to_f16_rn(f);
}

__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t h2;
  asm("{ .reg .b8 b; cvt.u8.u32 b, %1; cvt.rn.f16x2.e2m1x2 %0, b; }" : "=r"(h2) : "r"(byte & 0xFFu));
  return h2;
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t h2;
  const uint16_t c = (uint16_t)(two & 0xFFFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return h2;
}

__device__ __forceinline__ uint32_t hmul2_f16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// f16x2 -> bf16x2 (exact for e2m1 values).
__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t h2) {
  float lo, hi;
  const uint16_t l = (uint16_t)(h2 & 0xFFFFu), h = (uint16_t)(h2 >> 16);
  asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"(l));
  asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"(h));
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <bool BF16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}


// A fragment registers of MMA j (0..7) for rows g (wa) and g + 8 (wb) from
// the lane's 16 bytes of FP4 codes (wa4/wb4) or 32 bytes of FP8 codes, and
// the rows' scale words.
template <int FMT>
__device__ __forceinline__ void a_frag(uint32_t (&a)[4], const uint4& ra0, const uint4& ra1, const uint4& rb0,
                                       const uint4& rb1, uint32_t sfa, uint32_t sfb, int j, int q) {
  if (FMT == MOE_FMT_FP8) {
    const uint32_t* wa = (j < 4) ? &ra0.x : &ra1.x;
    const uint32_t* wb = (j < 4) ? &rb0.x : &rb1.x;
    const uint32_t va = wa[j & 3], vb = wb[j & 3];
    a[0] = e4m3x2_to_f16x2(va & 0xFFFFu);
    a[2] = e4m3x2_to_f16x2(va >> 16);
    a[1] = e4m3x2_to_f16x2(vb & 0xFFFFu);
    a[3] = e4m3x2_to_f16x2(vb >> 16);
    return;
  }
  const uint32_t wa = (&ra0.x)[j >> 1] >> ((j & 1) * 16);
  const uint32_t wb = (&rb0.x)[j >> 1] >> ((j & 1) * 16);
  if (FMT == MOE_FMT_NVFP4) {
    const int sh = 8 * (2 * (q & 1) + (j >> 2));
    const uint32_t sa = e4m3x2_to_f16x2((sfa >> sh) & 0xFFu) & 0xFFFFu;
    const uint32_t sb = e4m3x2_to_f16x2((sfb >> sh) & 0xFFu) & 0xFFFFu;
    const uint32_t sa2 = sa | (sa << 16), sb2 = sb | (sb << 16);
    a[0] = hmul2_f16(e2m1x2_to_f16x2(wa), sa2);
    a[2] = hmul2_f16(e2m1x2_to_f16x2(wa >> 8), sa2);
    a[1] = hmul2_f16(e2m1x2_to_f16x2(wb), sb2);
    a[3] = hmul2_f16(e2m1x2_to_f16x2(wb >> 8), sb2);
  } else {  // MXFP4: bf16 operands, scale 2^(c-127) (bf16 exponent bias is 127)
    const uint32_t ca = (sfa >> (8 * q)) & 0xFFu, cb = (sfb >> (8 * q)) & 0xFFu;
    const uint32_t sa = ca ? (ca << 7) : 0x0040u, sb = cb ? (cb << 7) : 0x0040u;
    const uint32_t sa2 = sa | (sa << 16), sb2 = sb | (sb << 16);
    a[0] = hmul2_bf16(f16x2_to_bf16x2(e2m1x2_to_f16x2(wa)), sa2);
    a[2] = hmul2_bf16(f16x2_to_bf16x2(e2m1x2_to_f16x2(wa >> 8)), sa2);
    a[1] = hmul2_bf16(f16x2_to_bf16x2(e2m1x2_to_f16x2(wb)), sb2);
    a[3] = hmul2_bf16(f16x2_to_bf16x2(e2m1x2_to_f16x2(wb >> 8)), sb2);
  }
}

// Activation block of bs values -> dequantised values (without the tensor
// scale, which the epilogue applies) or the plain values in BF16 mode.
template <int FMT>
__device__ __forceinline__ void activate_block(float* v, int bs, bool match, float g) {
  if (!match) return;
  float bmax = 0.0f;
  for (int i = 0; i < bs; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
  if (FMT == MOE_FMT_NVFP4) {
    uint32_t sc;
    float r;
    nvfp4_block_scale(bmax, g, sc, r);
    const float dec = e4m3_decode(sc);
    for (int i = 0; i < bs; i += 2) {
      const float2 d = r != 0.0f ? e2m1x2_decode(e2m1x2_encode(__fmul_rn(v[i], r), __fmul_rn(v[i + 1], r)))
                                 : make_float2(0.0f, 0.0f);
      v[i] = d.x * dec;
      v[i + 1] = d.y * dec;
    }
  } else if (FMT == MOE_FMT_MXFP4) {
    uint32_t c;
    float inv;
    mxfp4_block_scale(bmax, c, inv);
    const float sc = e8m0_decode(c);
    for (int i = 0; i < bs; i += 2) {
      const float2 d = e2m1x2_decode(e2m1x2_encode(__fmul_rn(v[i], inv), __fmul_rn(v[i + 1], inv)));
      v[i] = d.x * sc;
      v[i + 1] = d.y * sc;
    }
  } else {
    const float inv = __frcp_rn(g);
    for (int i = 0; i < bs; i += 2) {
      const uint32_t two = e4m3x2_encode(__fmul_rn(v[i], inv), __fmul_rn(v[i + 1], inv));
      v[i] = e4m3_decode(two & 0xFFu);
      v[i + 1] = e4m3_decode(two >> 8);
    }
  }
}

template <int FMT>
struct GemvCfg {
  static constexpr int kSfBytes = FMT == MOE_FMT_NVFP4 ? 2048 : (FMT == MOE_FMT_MXFP4 ? 1024 : 0);
  static constexpr int kA = kItemRows * 128;                         // one 128-byte K chunk of 64 rows
  static constexpr int kStage = kA + kSfBytes;
  static constexpr int kChunkK = FMT == MOE_FMT_FP8 ? 128 : 256;     // K elements per stage
};

template <int FMT, int STAGE>
__global__ void __launch_bounds__((1 + kGemvConsumers) * 32, 1)
    gemv_ffn_kernel(const __grid_constant__ CUtensorMap tmap_w, GemvArgs a, int stages) {
  using C = GemvCfg<FMT>;
  constexpr bool BF16 = FMT == MOE_FMT_MXFP4;
  const int K = STAGE == 1 ? a.H : a.I;
  const int R = STAGE == 1 ? 2 * a.I : a.H;
  const int MT = R / kItemRows;
  const int bs = FMT == MOE_FMT_MXFP4 ? 32 : 16;
  const int ncols = FMT == MOE_FMT_FP8 ? 0 : K / bs;
  const int nkc = (K + C::kChunkK - 1) / C::kChunkK;  // an FP4 K of 128 mod 256 ends on a half chunk
  const bool match = a.act == MOE_ACT_MATCH;
  const uint8_t* SF = STAGE == 1 ? a.w13_sf : a.w2_sf;
  const float* WGS = STAGE == 1 ? a.w13_gs : a.w2_gs;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint16_t* bsm = reinterpret_cast<uint16_t*>(base);                         // B fragments, K * 8
  uint8_t* ring = base + (((size_t)K * kNT * 2 + 1023) & ~size_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)stages * C::kStage);
  uint64_t* empty = full + stages;
  uint64_t* bbar = empty + stages;  // consumer-group barrier around B fragment rebuilds
  volatile int* abort = reinterpret_cast<volatile int*>(bbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      tc::mbar_init(&full[i], 1);
      tc::mbar_init(&empty[i], kGemvConsumers);
    }
    tc::mbar_init(bbar, kGemvConsumers * 32);
    *abort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&tmap_w);
  }
  __syncthreads();
  pdl_wait();  // the setup above overlaps the previous kernel's tail
  pdl_trigger();

  const int n_items = __ldg(a.num_tiles) * MT;
  const int i0 = (int)((int64_t)blockIdx.x * n_items / gridDim.x);
  const int i1 = (int)((int64_t)(blockIdx.x + 1) * n_items / gridDim.x);

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    int stage = 0;
    uint32_t phase = 0;
    for (int it = i0; it < i1 && !tc::aborted(abort); ++it) {
      const TileEntry te = a.tiles[it / MT];
      const int rb = it % MT;
      const uint8_t* sf_blk = SF ? SF + (size_t)te.e * R * ncols + (size_t)(rb >> 1) * (ncols / 4) * 512 : nullptr;
      for (int kc = 0; kc < nkc; ++kc) {
        if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort, a.wait_cycles)) {
          if (lane == 0) raise_status(a.status, MOE_ERR_TIMEOUT);
          *abort = 1;
          break;
        }
        if (tc::elect_one()) {
          uint8_t* st = ring + (size_t)stage * C::kStage;
          const int half = (kc + 1) * C::kChunkK > K;  // codes past K arrive as TMA zero fill
          const uint32_t sfb = half ? C::kSfBytes / 2 : C::kSfBytes;
          tc::mbar_expect_tx(&full[stage], C::kA + sfb);
          tc::tma_load_2d(st, &tmap_w, &full[stage], kc * 128, te.e * R + rb * kItemRows);
          if (C::kSfBytes)  // the 128-row scale blocks of this chunk (both 64-row halves)
            tc::bulk_load(st + C::kA, sf_blk + (size_t)kc * C::kSfBytes, sfb, &full[stage]);
        }
        __syncwarp();
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else {
    // --------------------------------------------------------- consumers
    const int cw = warp - 1;
    const int ctid = threadIdx.x - 32;
    const int g = lane >> 2, q = lane & 3;
    float gact = 1.0f;
    if (match && FMT != MOE_FMT_MXFP4) {
      const float* st = STAGE == 1 ? a.x_scale : a.h_scale;
      const float* am = STAGE == 1 ? a.x_amax : a.h_amax;
      gact = st ? __ldg(st) : (FMT == MOE_FMT_NVFP4 ? nvfp4_tensor_scale(*am) : fp8_tensor_scale(*am));
    }
    int stage = 0;
    uint32_t phase = 0;
    int prev_entry = -1;
    uint32_t bphase = 0;
    float hmax = 0.0f;
    // Bounded barrier of the consumer warps (the producer keeps streaming).
    auto consumer_sync = [&]() -> bool {
      tc::mbar_arrive(bbar);
      const bool ok = tc::mbar_wait(bbar, bphase, abort, a.wait_cycles);
      bphase ^= 1u;
      if (!ok) {
        if (lane == 0) raise_status(a.status, MOE_ERR_TIMEOUT);
        *abort = 1;
      }
      return ok;
    };
    for (int it = i0; it < i1 && !tc::aborted(abort); ++it) {
      const int entry = it / MT;
      const TileEntry te = a.tiles[entry];
      const int rb = it % MT;
      if (entry != prev_entry) {
        // activations of this token group -> B fragments
        if (!consumer_sync()) break;
        const int nb = K / bs;
        for (int item = ctid; item < kNT * nb; item += kGemvConsumers * 32) {
          const int n = item / nb, b = item % nb;
          float v[32];
          if (n < te.nvalid) {
            const int p = te.p0 + n;
            if (STAGE == 1) {
              const int t = __ldg(a.perm_token + p);
              if (t >= 0 && t < a.T) {
                const uint16_t* src = a.x + (int64_t)t * K + b * bs;
                for (int i = 0; i < bs; ++i) v[i] = bf16_to_f32(__ldg(src + i));
              } else {
                if (b == 0) raise_status(a.status, MOE_ERR_DEVICE_FAULT);
                for (int i = 0; i < bs; ++i) v[i] = 0.0f;
              }
            } else {
              const float* src = a.h + (int64_t)p * K + b * bs;
              for (int i = 0; i < bs; ++i) v[i] = src[i];
            }
            activate_block<FMT>(v, bs, match, gact);
          } else {
            for (int i = 0; i < bs; ++i) v[i] = 0.0f;
          }
          for (int i = 0; i < bs; ++i) bsm[bfrag_index(n, b * bs + i)] = to_mma_elem<BF16>(v[i]);
        }
        if (!consumer_sync()) break;
        prev_entry = entry;
      }
      // rows of this warp: r0 = rb * 64 + cw * 16 + g and r0 + 8 (within the expert)
      const int rl = cw * 16 + g;                 // row within the 64-row box
      const int64_t r0 = (int64_t)rb * kItemRows + rl;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int kc = 0; kc < nkc; ++kc) {
        if (!tc::mbar_wait(&full[stage], phase, abort, a.wait_cycles)) {
          if (lane == 0) raise_status(a.status, MOE_ERR_TIMEOUT);
          *abort = 1;
          break;
        }
        const uint8_t* st = ring + (size_t)stage * C::kStage;
        const uint2* bf = reinterpret_cast<const uint2*>(bsm);
        if (FMT == MOE_FMT_FP8) {
          // one 128-element chunk: lane q owns bytes [32q, 32q + 32) of each row
          const int c = kc;
          uint4 ra[2], rb2[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j = 2 * q + h;
            ra[h] = *reinterpret_cast<const uint4*>(st + rl * 128 + ((j ^ (rl & 7)) << 4));
            rb2[h] = *reinterpret_cast<const uint4*>(st + (rl + 8) * 128 + ((j ^ ((rl + 8) & 7)) << 4));
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t af[4];
            a_frag<FMT>(af, ra[0], ra[1], rb2[0], rb2[1], 0u, 0u, j, q);
            const uint2 b = bf[(c * 8 + j) * 32 + lane];
            mma16816<BF16>(acc, af, b.x, b.y);
          }
        } else {
          const uint8_t* sfs = st + C::kA;
          const int rs = (int)(r0 & 127);          // row within its 128-row scale block
          const int nsub = (kc + 1) * C::kChunkK > K ? 1 : 2;
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            if (sub >= nsub) break;
            const int c = kc * 2 + sub;
            const int j = sub * 4 + q;
            const uint4 ra = *reinterpret_cast<const uint4*>(st + rl * 128 + ((j ^ (rl & 7)) << 4));
            const uint4 rbb = *reinterpret_cast<const uint4*>(st + (rl + 8) * 128 + ((j ^ ((rl + 8) & 7)) << 4));
            const int grp = FMT == MOE_FMT_NVFP4 ? 2 * sub + (q >> 1) : sub;
            const uint32_t sfa = *reinterpret_cast<const uint32_t*>(sfs + grp * 512 + (rs & 31) * 16 + (rs >> 5) * 4);
            const uint32_t sfb =
                *reinterpret_cast<const uint32_t*>(sfs + grp * 512 + ((rs + 8) & 31) * 16 + ((rs + 8) >> 5) * 4);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              uint32_t af[4];
              a_frag<FMT>(af, ra, ra, rbb, rbb, sfa, sfb, jj, q);
              const uint2 b = bf[(c * 8 + jj) * 32 + lane];
              mma16816<BF16>(acc, af, b.x, b.y);
            }
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&empty[stage]);
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // ---- epilogue: acc[0..1] = row r0, tokens 2q, 2q+1; acc[2..3] = row r0 + 8
      const int nt = te.nvalid;
      if (STAGE == 1) {
        const int part = (int)(r0 & 1);  // prepared rows: even gate, odd up
        const float ws = (FMT == MOE_FMT_MXFP4) ? 1.0f : __ldg(WGS + te.e * 2 + part);
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = acc[i] * ws * gact;
        float u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) u[i] = __shfl_xor_sync(0xffffffffu, v[i], 4);
        if (part == 0) {
          const int f0 = (int)(r0 >> 1);  // feature of row r0; row r0 + 8 is feature f0 + 4
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int tok = 2 * q + (i & 1);
            const int f = f0 + (i >> 1) * 4;
            if (tok < nt) {
              const float gg = v[i];
              const float hv = gg / (1.0f + __expf(-gg)) * u[i];
              a.h[(int64_t)(te.p0 + tok) * a.I + f] = hv;
              hmax = fmaxf(hmax, fabsf(hv));
            }
          }
        }
      } else {
        const float ws = (FMT == MOE_FMT_MXFP4) ? 1.0f : __ldg(WGS + te.e);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tok = 2 * q + (i & 1);
          const int64_t o = r0 + (i >> 1) * 8;
          if (tok < nt) a.y_perm[(int64_t)(te.p0 + tok) * a.H + o] = f32_to_bf16_rn(acc[i] * ws * gact);
        }
      }
    }
    if (STAGE == 1 && match && a.h_amax) {
      hmax = warp_max(hmax);
      if (lane == 0) atomic_max_nonneg(a.h_amax, hmax);
    }
  }
  __syncthreads();
  if (*abort) {
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000LL) {
    }
  }
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

template <int FMT, int STAGE>
static cudaError_t launch_stage(const GemvArgs& a, int num_sms, cudaStream_t s) {
  using C = GemvCfg<FMT>;
  const int K = STAGE == 1 ? a.H : a.I;
  const int R = STAGE == 1 ? 2 * a.I : a.H;
  const int64_t rowb = FMT == MOE_FMT_FP8 ? K : K / 2;
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)rowb, (cuuint64_t)a.E * R};
  cuuint64_t strides[1] = {(cuuint64_t)rowb};
  cuuint32_t box[2] = {128u, (cuuint32_t)kItemRows};
  cuuint32_t es[2] = {1u, 1u};
  if (fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(STAGE == 1 ? a.w13 : a.w2), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t bfrag = ((size_t)K * kNT * 2 + 1023) & ~size_t(1023);
  const size_t budget = 220 * 1024;
  int stages = (int)((budget - 1024 - bfrag - 1024) / C::kStage);
  stages = stages > 32 ? 32 : stages;
  if (stages < 2) return cudaErrorInvalidValue;
  const size_t smem = 1024 + bfrag + (size_t)stages * C::kStage + 1024;
  cudaError_t err =
      cudaFuncSetAttribute(gemv_ffn_kernel<FMT, STAGE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  err = launch_pdl(gemv_ffn_kernel<FMT, STAGE>, dim3(num_sms), dim3((1 + kGemvConsumers) * 32), smem, s, m, a, stages);
  if (err != cudaSuccess) return err;
  count_launches(1);
  return cudaGetLastError();
}

template <int STAGE>
static cudaError_t launch_any(const GemvArgs& a, int num_sms, cudaStream_t s) {
  switch (a.fmt) {
    case MOE_FMT_NVFP4: return launch_stage<MOE_FMT_NVFP4, STAGE>(a, num_sms, s);
    case MOE_FMT_MXFP4: return launch_stage<MOE_FMT_MXFP4, STAGE>(a, num_sms, s);
    case MOE_FMT_FP8: return launch_stage<MOE_FMT_FP8, STAGE>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

// GEMV1: W13 + SwiGLU -> h (fp32).  With a dynamic activation scale the
// caller has put amax(x) in a.x_amax; a.h_amax is cleared here and filled.
cudaError_t launch_gemv_up(const GemvArgs& a, int num_sms, cudaStream_t s) {
  if (a.h_amax) {
    cudaError_t e = cudaMemsetAsync(a.h_amax, 0, sizeof(float), s);
    if (e != cudaSuccess) return e;
  }
  return launch_any<1>(a, num_sms, s);
}

// GEMV2: W2 -> y_perm (bf16).
cudaError_t launch_gemv_down(const GemvArgs& a, int num_sms, cudaStream_t s) { return launch_any<2>(a, num_sms, s); }

}  // namespace moe
