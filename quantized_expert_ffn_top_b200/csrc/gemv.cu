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
// Rows: a CTA owns 128 rows of one expert (8 warps x 16 rows).  W13 rows are
// PREPARED (row 2i gate i, row 2i+1 up i), so a gate/up pair sits in lanes
// l and l ^ 4 and the SwiGLU epilogue needs one shuffle.
#include "kernels.cuh"

namespace moe {

constexpr int kNT = 8;          // token columns per pass (MMA n)
constexpr int kGemvWarps = 8;   // 16 rows each

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

// Weight bytes of one 128-element chunk for one row and lane quad position.
struct ChunkRegs {
  uint4 c0, c1;       // FP4: c0 = 16 bytes (32 codes); FP8: c0, c1 = 32 bytes
  uint32_t sf;        // scale word (blocked layout)
};

template <int FMT>
__device__ __forceinline__ void load_chunk(ChunkRegs& r, const uint8_t* row, const uint8_t* sf_e, int64_t row_idx,
                                           int ncols, int c, int q) {
  if (FMT == MOE_FMT_FP8) {
    const uint4* p = reinterpret_cast<const uint4*>(row + c * 128 + q * 32);
    r.c0 = __ldg(p);
    r.c1 = __ldg(p + 1);
    r.sf = 0u;
  } else {
    r.c0 = __ldg(reinterpret_cast<const uint4*>(row + c * 64 + q * 16));
    const int col = FMT == MOE_FMT_NVFP4 ? 8 * c + 2 * q : 4 * c + q;
    r.sf = __ldg(reinterpret_cast<const uint32_t*>(sf_e + sf_blocked_offset(row_idx, col & ~3, ncols)));
  }
}

// A fragment registers of MMA j for the rows held in ra (row g) and rb (g+8).
template <int FMT>
__device__ __forceinline__ void a_frag(uint32_t (&a)[4], const ChunkRegs& ra, const ChunkRegs& rb, int j, int q) {
  if (FMT == MOE_FMT_FP8) {
    const uint32_t* wa = (j < 4) ? &ra.c0.x : &ra.c1.x;
    const uint32_t* wb = (j < 4) ? &rb.c0.x : &rb.c1.x;
    const uint32_t va = wa[j & 3], vb = wb[j & 3];
    a[0] = e4m3x2_to_f16x2(va & 0xFFFFu);
    a[2] = e4m3x2_to_f16x2(va >> 16);
    a[1] = e4m3x2_to_f16x2(vb & 0xFFFFu);
    a[3] = e4m3x2_to_f16x2(vb >> 16);
    return;
  }
  const uint32_t wa = (&ra.c0.x)[j >> 1] >> ((j & 1) * 16);
  const uint32_t wb = (&rb.c0.x)[j >> 1] >> ((j & 1) * 16);
  if (FMT == MOE_FMT_NVFP4) {
    const int sh = 8 * (2 * (q & 1) + (j >> 2));
    const uint32_t sa = e4m3x2_to_f16x2((ra.sf >> sh) & 0xFFu) & 0xFFFFu;
    const uint32_t sb = e4m3x2_to_f16x2((rb.sf >> sh) & 0xFFu) & 0xFFFFu;
    const uint32_t sa2 = sa | (sa << 16), sb2 = sb | (sb << 16);
    a[0] = hmul2_f16(e2m1x2_to_f16x2(wa), sa2);
    a[2] = hmul2_f16(e2m1x2_to_f16x2(wa >> 8), sa2);
    a[1] = hmul2_f16(e2m1x2_to_f16x2(wb), sb2);
    a[3] = hmul2_f16(e2m1x2_to_f16x2(wb >> 8), sb2);
  } else {  // MXFP4: bf16 operands, scale 2^(c-127) (bf16 exponent bias is 127)
    const uint32_t ca = (ra.sf >> (8 * q)) & 0xFFu, cb = (rb.sf >> (8 * q)) & 0xFFu;
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

template <int FMT, int STAGE>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_ffn_kernel(GemvArgs a) {
  constexpr bool BF16 = FMT == MOE_FMT_MXFP4;
  const int e = blockIdx.y;
  const int off0 = __ldg(a.offsets + e);
  const int off1 = __ldg(a.offsets + e + 1);
  if (off0 < 0 || off1 < off0 || off1 > a.S) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(a.status, MOE_ERR_DEVICE_FAULT);
    return;
  }
  const int n_e = off1 - off0;
  if (n_e == 0) return;
  const int K = STAGE == 1 ? a.H : a.I;
  const int R = STAGE == 1 ? 2 * a.I : a.H;
  const int rowb = FMT == MOE_FMT_FP8 ? K : K / 2;
  const int bs = FMT == MOE_FMT_MXFP4 ? 32 : 16;
  const int ncols = FMT == MOE_FMT_FP8 ? 0 : K / bs;
  const bool match = a.act == MOE_ACT_MATCH;
  const uint8_t* W = STAGE == 1 ? a.w13 : a.w2;
  const uint8_t* SF = STAGE == 1 ? a.w13_sf : a.w2_sf;
  const float* WGS = STAGE == 1 ? a.w13_gs : a.w2_gs;
  extern __shared__ __align__(16) uint16_t bsm[];  // B fragments, K * kNT elements

  // Tensor scale of the activations (MATCH, NVFP4 / FP8).
  float gact = 1.0f;
  if (match && FMT != MOE_FMT_MXFP4) {
    const float* st = STAGE == 1 ? a.x_scale : a.h_scale;
    const float* am = STAGE == 1 ? a.x_amax : a.h_amax;
    gact = st ? __ldg(st) : (FMT == MOE_FMT_NVFP4 ? nvfp4_tensor_scale(*am) : fp8_tensor_scale(*am));
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int64_t r0 = (int64_t)blockIdx.x * 128 + warp * 16 + g;  // rows r0 and r0 + 8 of this expert
  const uint8_t* rowA = W + ((int64_t)e * R + r0) * rowb;
  const uint8_t* rowB = rowA + (int64_t)8 * rowb;
  const uint8_t* sf_e = SF ? SF + (int64_t)e * R * ncols : nullptr;
  const int nchunk = K / 128;
  float hmax = 0.0f;

  for (int c0 = 0; c0 < n_e; c0 += kNT) {
    const int nt = min(kNT, n_e - c0);
    __syncthreads();
    // ---- activations -> B fragments (shared memory)
    const int nb = K / bs;
    for (int item = threadIdx.x; item < kNT * nb; item += blockDim.x) {
      const int n = item / nb, b = item % nb;
      float v[32];
      if (n < nt) {
        if (STAGE == 1) {
          const int t = __ldg(a.perm_token + off0 + c0 + n);
          if (t >= 0 && t < a.T) {
            const uint16_t* src = a.x + (int64_t)t * K + b * bs;
            for (int i = 0; i < bs; ++i) v[i] = bf16_to_f32(__ldg(src + i));
          } else {
            if (b == 0) raise_status(a.status, MOE_ERR_DEVICE_FAULT);
            for (int i = 0; i < bs; ++i) v[i] = 0.0f;
          }
        } else {
          const float* src = a.h + (int64_t)(off0 + c0 + n) * K + b * bs;
          for (int i = 0; i < bs; ++i) v[i] = src[i];
        }
        activate_block<FMT>(v, bs, match, gact);
      } else {
        for (int i = 0; i < bs; ++i) v[i] = 0.0f;
      }
      for (int i = 0; i < bs; ++i) bsm[bfrag_index(n, b * bs + i)] = to_mma_elem<BF16>(v[i]);
    }
    __syncthreads();

    // ---- stream the weights
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    ChunkRegs ca, cb, na, nb2;
    load_chunk<FMT>(ca, rowA, sf_e, r0, ncols, 0, q);
    load_chunk<FMT>(cb, rowB, sf_e, r0 + 8, ncols, 0, q);
    for (int c = 0; c < nchunk; ++c) {
      if (c + 1 < nchunk) {
        load_chunk<FMT>(na, rowA, sf_e, r0, ncols, c + 1, q);
        load_chunk<FMT>(nb2, rowB, sf_e, r0 + 8, ncols, c + 1, q);
      }
      const uint2* bf = reinterpret_cast<const uint2*>(bsm) + (c * 8) * 32 + lane;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t af[4];
        a_frag<FMT>(af, ca, cb, j, q);
        const uint2 b = bf[j * 32];
        mma16816<BF16>(acc, af, b.x, b.y);
      }
      ca = na;
      cb = nb2;
    }

    // ---- epilogue: acc[0..1] = row r0, tokens 2q, 2q+1; acc[2..3] = row r0+8
    if (STAGE == 1) {
      const int part = (int)(r0 & 1);  // prepared rows: even gate, odd up
      const float ws = (FMT == MOE_FMT_MXFP4) ? 1.0f : __ldg(WGS + e * 2 + part);
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
            a.h[(int64_t)(off0 + c0 + tok) * a.I + f] = hv;
            hmax = fmaxf(hmax, fabsf(hv));
          }
        }
      }
    } else {
      const float ws = (FMT == MOE_FMT_MXFP4) ? 1.0f : __ldg(WGS + e);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tok = 2 * q + (i & 1);
        const int64_t o = r0 + (i >> 1) * 8;
        if (tok < nt) a.y_perm[(int64_t)(off0 + c0 + tok) * a.H + o] = f32_to_bf16_rn(acc[i] * ws * gact);
      }
    }
  }
  if (STAGE == 1 && match && a.h_amax) {
    hmax = warp_max(hmax);
    if (lane == 0) atomic_max_nonneg(a.h_amax, hmax);
  }
}

template <int FMT, int STAGE>
static cudaError_t launch_stage(const GemvArgs& a, cudaStream_t s) {
  const int K = STAGE == 1 ? a.H : a.I;
  const int R = STAGE == 1 ? 2 * a.I : a.H;
  const size_t smem = (size_t)K * kNT * sizeof(uint16_t);
  cudaError_t err =
      cudaFuncSetAttribute(gemv_ffn_kernel<FMT, STAGE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  gemv_ffn_kernel<FMT, STAGE><<<dim3(R / 128, a.E), kGemvWarps * 32, smem, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

template <int STAGE>
static cudaError_t launch_any(const GemvArgs& a, cudaStream_t s) {
  switch (a.fmt) {
    case MOE_FMT_NVFP4: return launch_stage<MOE_FMT_NVFP4, STAGE>(a, s);
    case MOE_FMT_MXFP4: return launch_stage<MOE_FMT_MXFP4, STAGE>(a, s);
    case MOE_FMT_FP8: return launch_stage<MOE_FMT_FP8, STAGE>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

// GEMV1: W13 + SwiGLU -> h (fp32).  With a dynamic activation scale the
// caller has put amax(x) in a.x_amax; a.h_amax is cleared here and filled.
cudaError_t launch_gemv_up(const GemvArgs& a, cudaStream_t s) {
  if (a.h_amax) {
    cudaError_t e = cudaMemsetAsync(a.h_amax, 0, sizeof(float), s);
    if (e != cudaSuccess) return e;
  }
  return launch_any<1>(a, s);
}

// GEMV2: W2 -> y_perm (bf16).
cudaError_t launch_gemv_down(const GemvArgs& a, cudaStream_t s) { return launch_any<2>(a, s); }

}  // namespace moe
