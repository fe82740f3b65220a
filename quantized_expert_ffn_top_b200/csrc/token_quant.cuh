// Activation quantisation of one token row into the padded rows of its slots
// (MATCH mode, a5): the token's K bf16 values are quantised once (NVFP4: e2m1
// codes with an e4m3 scale per 16 values and a per-tensor scale; MXFP4: e2m1
// with an e8m0 scale per 32; FP8: e4m3 with a per-tensor scale) and the codes
// and block scales are stored in the rows of every slot the token was routed
// to.  Used by the per-token x quantiser and by the small-batch permutation
// kernel, which quantises right after it has placed the slots.
#pragma once

#include <cstdint>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

// Per-tensor scale of a quantised activation: none for MXFP4 (its scales are
// per block only), otherwise the static scale when one is given, else the
// one derived from the tensor's amax.
__device__ __forceinline__ float act_scale_of(int fmt, const float* st, const float* amax) {
  if (fmt == MOE_FMT_MXFP4) return 1.0f;
  if (st) return __ldg(st);
  if (!amax) return 1.0f;
  return fmt == MOE_FMT_NVFP4 ? nvfp4_tensor_scale(*amax) : fp8_tensor_scale(*amax);
}

template <int FMT>
struct TokenQuant {
  static constexpr int kBs = FMT == MOE_FMT_MXFP4 ? 32 : 16;   // values per block scale
  static constexpr int kPer = 64;                              // values per lane per stretch
  static constexpr int kWords = FMT == MOE_FMT_FP8 ? 16 : 8;   // 32-bit code words per lane
  static constexpr int kLaneBytes = kWords * 4;
  static constexpr int kVec = kLaneBytes / 16;
  static constexpr int kWarpBuf = 32 * kVec;                   // uint4 of reorder buffer per warp
};

// One warp quantises the token row xt (K bf16 values, K % 64 == 0) and stores
// the codes and the block scales (blocked layout) in the padded rows of the
// token's k slots.  row_of(j), evaluated by lane j for j < k, gives slot j's
// padded row: -1 for a dropped slot, -2 when the permutation is inconsistent
// (the slot is skipped and the status word raised).  tb: the warp's reorder
// buffer (TokenQuant<FMT>::kWarpBuf uint4 of shared memory); r_tab: the NVFP4
// multipliers of the 128 non-negative scale codes for this scale.
template <int FMT, class RowOf>
__device__ __forceinline__ void quant_token_slots(const uint16_t* __restrict__ xt, int K, int k, float scale,
                                                  const float* r_tab, uint4* tb, RowOf&& row_of,
                                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                  int32_t* status) {
  using Q = TokenQuant<FMT>;
  constexpr int bs = Q::kBs, kPer = Q::kPer, kWords = Q::kWords, kLaneBytes = Q::kLaneBytes, kVec = Q::kVec;
  const int nb = K / bs;
  const int lane = threadIdx.x & 31;
  const int64_t row_first = lane < k ? row_of(lane) : -1;  // issued before the x loads
  for (int c0 = 0; c0 < K; c0 += 32 * kPer) {
    const int c = c0 + lane * kPer;
    const bool active = c < K;
    uint32_t w[kWords];
    uint32_t sfw = 0;
    if (active) {
      // the lane's 64 bf16 values stay packed (32 registers); each scale
      // block is unpacked when it is quantised
      uint32_t raw[kPer / 2];
      const uint4* src = reinterpret_cast<const uint4*>(xt + c);
#pragma unroll
      for (int i = 0; i < kPer / 8; ++i) {
        const uint4 u = __ldg(src + i);
        raw[4 * i] = u.x;
        raw[4 * i + 1] = u.y;
        raw[4 * i + 2] = u.z;
        raw[4 * i + 3] = u.w;
      }
      auto unpack = [&](float* v, int first, int n) {
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
          v[2 * i] = __uint_as_float(raw[first / 2 + i] << 16);
          v[2 * i + 1] = __uint_as_float(raw[first / 2 + i] & 0xFFFF0000u);
        }
      };
      if constexpr (FMT == MOE_FMT_NVFP4) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          float v[16];
          unpack(v, 16 * b, 16);
          float bmax = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
          const uint32_t sc = nvfp4_scale_code(bmax, scale);
          const uint2 cw = nvfp4_encode16(v, r_tab[sc]);
          w[2 * b] = cw.x;
          w[2 * b + 1] = cw.y;
          sfw |= sc << (8 * b);
        }
      } else if constexpr (FMT == MOE_FMT_MXFP4) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          float v[32];
          unpack(v, 32 * b, 32);
          float bmax = 0.0f;
#pragma unroll
          for (int i = 0; i < 32; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
          uint32_t sc;
          float inv;
          mxfp4_block_scale(bmax, sc, inv);
#pragma unroll
          for (int q = 0; q < 4; ++q) w[4 * b + q] = e2m1_encode8(v + 8 * q, inv);
          sfw |= sc << (8 * b);
        }
      } else {
        const float inv = __frcp_rn(scale);
#pragma unroll
        for (int i = 0; i < kWords; ++i) {
          float v[4];
          unpack(v, 4 * i, 4);
          w[i] = e4m3x2_encode(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)) |
                 (e4m3x2_encode(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)) << 16);
        }
      }
    }
    // Codes in store order: lane l's 16-byte pieces v are bytes 512 v + 16 l
    // of the stretch, so every store instruction covers 512 contiguous bytes.
    if (active) {
#pragma unroll
      for (int v = 0; v < kVec; ++v) tb[lane * kVec + v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }
    __syncwarp();
    const int seg = min(K - c0, 32 * kPer) * kLaneBytes / kPer;  // code bytes in this stretch
    uint4 wc[kVec];
#pragma unroll
    for (int v = 0; v < kVec; ++v) {
      const int off = 512 * v + 16 * lane;
      wc[v] = off < seg ? tb[off / 16] : make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
    for (int j0 = 0; j0 < k; j0 += 32) {
      // lane j holds the padded row of slot j0 + j
      const int64_t myrow = (j0 == 0) ? row_first : (j0 + lane < k ? row_of(j0 + lane) : -1);
      const int nj = min(32, k - j0);
      for (int jj = 0; jj < nj; ++jj) {
        const int64_t row = __shfl_sync(0xffffffffu, myrow, jj);
        if (row < 0) {
          if (row == -2 && lane == 0 && c0 == 0) raise_status(status, MOE_ERR_DEVICE_FAULT);
          continue;
        }
        uint4* dst = reinterpret_cast<uint4*>(codes + row * ((int64_t)K * kLaneBytes / kPer) +
                                              (int64_t)c0 * kLaneBytes / kPer);
#pragma unroll
        for (int v = 0; v < kVec; ++v)
          if (512 * v + 16 * lane < seg) dst[(512 * v) / 16 + lane] = wc[v];
        if (!active) continue;
        if constexpr (FMT == MOE_FMT_NVFP4)
          *reinterpret_cast<uint32_t*>(sf + sf_blocked_offset(row, c / bs, nb)) = sfw;
        else if constexpr (FMT == MOE_FMT_MXFP4)
          *reinterpret_cast<uint16_t*>(sf + sf_blocked_offset(row, c / bs, nb)) = (uint16_t)sfw;
      }
    }
  }
}

}  // namespace moe

namespace moe {

// Small batches: the quantised x rows in a layout the expert FFN can gather
// from with plain bulk copies, whatever the routing.  For token t and
// variant v (0..7) the codes of K-stage kb (256 values, 128 bytes) sit at
// xg[((t * 8 + v) * K / 2) + kb * 128] with their 16-byte pieces in the
// order of the tensor cores' 128-byte swizzle for a row r with r % 8 == v
// (piece p at position p ^ v): a row copied into tile row r of a stage is
// then already where the MMA reads it.  The block scales go to 16-byte
// lines, one per group of 4 scales (xsl[(t * K / (4 bs) + g) * 16]: the
// group's 4 scale bytes, then 12 zero bytes): copied to line r of the
// group's 512-byte block they are tile row r's scales for rows below 32.

template <int FMT>
__device__ __forceinline__ void quant_token_gather(const uint16_t* __restrict__ xt, int K, float scale,
                                                   const float* r_tab, uint8_t* __restrict__ xg_t,
                                                   uint8_t* __restrict__ xsl_t) {
  static_assert(FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_MXFP4, "block-scaled FP4 formats");
  using Q = TokenQuant<FMT>;
  constexpr int bs = Q::kBs, kPer = Q::kPer;
  const int lane = threadIdx.x & 31;
  for (int c0 = 0; c0 < K; c0 += 32 * kPer) {
    const int c = c0 + lane * kPer;
    const bool active = c < K;
    uint32_t w[8];
    uint32_t sfw = 0;
    if (active) {
      uint32_t raw[kPer / 2];
      const uint4* src = reinterpret_cast<const uint4*>(xt + c);
#pragma unroll
      for (int i = 0; i < kPer / 8; ++i) {
        const uint4 u = __ldg(src + i);
        raw[4 * i] = u.x;
        raw[4 * i + 1] = u.y;
        raw[4 * i + 2] = u.z;
        raw[4 * i + 3] = u.w;
      }
      auto unpack = [&](float* v, int first, int n) {
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
          v[2 * i] = __uint_as_float(raw[first / 2 + i] << 16);
          v[2 * i + 1] = __uint_as_float(raw[first / 2 + i] & 0xFFFF0000u);
        }
      };
      if constexpr (FMT == MOE_FMT_NVFP4) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          float v[16];
          unpack(v, 16 * b, 16);
          float bmax = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
          const uint32_t sc = nvfp4_scale_code(bmax, scale);
          const uint2 cw = nvfp4_encode16(v, r_tab[sc]);
          w[2 * b] = cw.x;
          w[2 * b + 1] = cw.y;
          sfw |= sc << (8 * b);
        }
      } else {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          float v[32];
          unpack(v, 32 * b, 32);
          float bmax = 0.0f;
#pragma unroll
          for (int i = 0; i < 32; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
          uint32_t sc;
          float inv;
          mxfp4_block_scale(bmax, sc, inv);
#pragma unroll
          for (int q = 0; q < 4; ++q) w[4 * b + q] = e2m1_encode8(v + 8 * q, inv);
          sfw |= sc << (8 * b);
        }
      }
    }
    // the lane's 32 code bytes are pieces 2 (lane % 4) and 2 (lane % 4) + 1
    // of K-stage (c / 256); one copy per variant
    if (active) {
      const int64_t kb_off = (int64_t)(c / 256) * 128;
      const int p0 = 2 * (lane & 3);
      const uint4 a = make_uint4(w[0], w[1], w[2], w[3]), b = make_uint4(w[4], w[5], w[6], w[7]);
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        uint8_t* row = xg_t + (int64_t)v * (K / 2) + kb_off;
        *reinterpret_cast<uint4*>(row + ((p0 ^ v) << 4)) = a;
        *reinterpret_cast<uint4*>(row + (((p0 + 1) ^ v) << 4)) = b;
      }
    }
    // scale lines: NVFP4 holds one group of 4 scales per lane, MXFP4 two
    // scales (half a group): the even lane of a pair writes the line
    if constexpr (FMT == MOE_FMT_NVFP4) {
      if (active) *reinterpret_cast<uint4*>(xsl_t + (int64_t)(c / 64) * 16) = make_uint4(sfw, 0u, 0u, 0u);
    } else {
      const uint32_t hi = __shfl_down_sync(0xffffffffu, sfw, 1);
      if (active && (lane & 1) == 0)
        *reinterpret_cast<uint4*>(xsl_t + (int64_t)(c / 128) * 16) = make_uint4(sfw | (hi << 16), 0u, 0u, 0u);
    }
  }
}

}  // namespace moe
