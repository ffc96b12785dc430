// Tile loaders shared by the forward and backward kernels: one warpgroup
// (128 threads) moves a [128 rows][D] tile of a [B][T][H][D] tensor from
// global memory into swizzled bf16 operand tiles in shared memory, applying
// the rotary embedding on the way for queries and keys.
//
// Rotary embedding (RoPE on queries and keys: "NanoEuler" write-up, aimsg.uk,
// section 2 "Model components"; "Tiny Hackable CUDA LM", section 1): the
// interleaved pair (x[2i], x[2i+1]) of position t turns by the angle
// t * base^(-2i/D); cos/sin come from a float table [T][D/2] of (cos, sin)
// pairs computed in double precision on the host.
//
// For float32 storage every element is written twice: its bf16 rounding to
// the "hi" tile and the bf16 rounding of the residual to the "lo" tile.
#pragma once

#include "nea_device.cuh"

namespace nea {

constexpr int kTileRows = 128;

template <int D>
struct TileGeom {
  static constexpr uint32_t kRowBytes = 2 * D;              // bf16 row of the operand tile
  static constexpr uint32_t kTileBytes = kTileRows * kRowBytes;
};

__device__ __forceinline__ void rot2(float& x0, float& x1, float c, float s) {
  const float y0 = x0 * c - x1 * s;
  const float y1 = x0 * s + x1 * c;
  x0 = y0;
  x1 = y1;
}

// Loads rows [row0, row0 + 128) of head `head` (batch b) of a [B][T][H][D]
// float32 tensor.  Rows at or beyond T are zero.  `pt` is the thread's index
// in the warpgroup.  ROPE selects the rotation; `hi`/`lo` are the operand
// tiles (`lo` unused when SPLIT is false).
template <int D, bool ROPE, bool SPLIT>
__device__ __forceinline__ void load_tile_f32(uint8_t* hi, uint8_t* lo, const float* __restrict__ src, int b,
                                              int row0, int head, int T, int H,
                                              const float2* __restrict__ rope, int pt) {
  constexpr int kChunksPerRow = D / 4;  // 16-byte chunks of four floats
  constexpr int kPerThread = kTileRows * kChunksPerRow / 128;
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  float4 x[kPerThread];
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int q = pt + 128 * k;
    const int r = q / kChunksPerRow, c = q % kChunksPerRow;
    const int t = row0 + r;
    if (t < T) {
      const float4* p = reinterpret_cast<const float4*>(src + ((size_t(b) * T + t) * H + head) * D) + c;
      x[k] = __ldg(p);
    } else {
      x[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int q = pt + 128 * k;
    const int r = q / kChunksPerRow, c = q % kChunksPerRow;
    const int t = row0 + r;
    float4 v = x[k];
    if (ROPE && rope != nullptr && t < T) {
      const float4 cs = __ldg(reinterpret_cast<const float4*>(rope + size_t(t) * (D / 2) + 2 * c));
      rot2(v.x, v.y, cs.x, cs.y);
      rot2(v.z, v.w, cs.z, cs.w);
    }
    const uint32_t off = swizzle(uint32_t(r) * RB + uint32_t(c) * 8, RB);
    uint2 h2, l2;
    if (SPLIT) {
      split_bf16(v.x, v.y, h2.x, l2.x);
      split_bf16(v.z, v.w, h2.y, l2.y);
      *reinterpret_cast<uint2*>(lo + off) = l2;
    } else {
      h2.x = pack_bf16(v.x, v.y);
      h2.y = pack_bf16(v.z, v.w);
    }
    *reinterpret_cast<uint2*>(hi + off) = h2;
  }
}

// Same for a bfloat16 tensor: 16-byte chunks of eight elements, rotated in
// float and rounded back to bf16.
template <int D, bool ROPE>
__device__ __forceinline__ void load_tile_bf16(uint8_t* dst, const __nv_bfloat16* __restrict__ src, int b,
                                               int row0, int head, int T, int H,
                                               const float2* __restrict__ rope, int pt) {
  constexpr int kChunksPerRow = D / 8;
  constexpr int kPerThread = kTileRows * kChunksPerRow / 128;
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  uint4 x[kPerThread];
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int q = pt + 128 * k;
    const int r = q / kChunksPerRow, c = q % kChunksPerRow;
    const int t = row0 + r;
    if (t < T) {
      const uint4* p = reinterpret_cast<const uint4*>(src + ((size_t(b) * T + t) * H + head) * D) + c;
      x[k] = __ldg(p);
    } else {
      x[k] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int q = pt + 128 * k;
    const int r = q / kChunksPerRow, c = q % kChunksPerRow;
    const int t = row0 + r;
    uint4 v = x[k];
    if (ROPE && rope != nullptr && t < T) {
      const float4* tp = reinterpret_cast<const float4*>(rope + size_t(t) * (D / 2) + 4 * c);
      const float4 cs0 = __ldg(tp), cs1 = __ldg(tp + 1);
      float a0 = bf16_lo_f(v.x), a1 = bf16_hi_f(v.x), a2 = bf16_lo_f(v.y), a3 = bf16_hi_f(v.y);
      float a4 = bf16_lo_f(v.z), a5 = bf16_hi_f(v.z), a6 = bf16_lo_f(v.w), a7 = bf16_hi_f(v.w);
      rot2(a0, a1, cs0.x, cs0.y);
      rot2(a2, a3, cs0.z, cs0.w);
      rot2(a4, a5, cs1.x, cs1.y);
      rot2(a6, a7, cs1.z, cs1.w);
      v.x = pack_bf16(a0, a1);
      v.y = pack_bf16(a2, a3);
      v.z = pack_bf16(a4, a5);
      v.w = pack_bf16(a6, a7);
    }
    const uint32_t off = swizzle(uint32_t(r) * RB + uint32_t(c) * 16, RB);
    *reinterpret_cast<uint4*>(dst + off) = v;
  }
}

// Dispatch on storage type: `parts` points at NSPLIT consecutive operand
// tiles (hi, then lo for float32 storage).
template <int D, bool F32IO, bool ROPE>
__device__ __forceinline__ void load_tile(uint8_t* parts, const void* src, int b, int row0, int head, int T,
                                          int H, const float2* rope, int pt) {
  if constexpr (F32IO) {
    load_tile_f32<D, ROPE, true>(parts, parts + TileGeom<D>::kTileBytes, static_cast<const float*>(src), b,
                                 row0, head, T, H, rope, pt);
  } else {
    load_tile_bf16<D, ROPE>(parts, static_cast<const __nv_bfloat16*>(src), b, row0, head, T, H, rope, pt);
  }
}

// Writes one D-wide output row held in registers (float) to a [B][T][H][D]
// tensor in the storage type.
template <int D, bool F32IO>
__device__ __forceinline__ void store_row(void* dst, int b, int t, int head, int T, int H, const float* v) {
  if constexpr (F32IO) {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(dst) + ((size_t(b) * T + t) * H + head) * D);
#pragma unroll
    for (int i = 0; i < D / 4; ++i) p[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else {
    uint4* p = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst) + ((size_t(b) * T + t) * H + head) * D);
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
      p[i] = make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                        pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
  }
}

}  // namespace nea
