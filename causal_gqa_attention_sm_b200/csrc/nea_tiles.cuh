// Tile geometry shared by the forward and backward kernels.
//
// A [128 rows][D] tile of one head of a [B][T][H][D] tensor arrives in shared
// memory by TMA (rows at or beyond T read as zero), already in the bf16
// operand layout the tcgen05 MMAs read: rows of 2*D bytes with the hardware
// swizzle whose atom equals the row.  Rows longer than the widest swizzle
// (D = 128: 256 bytes) are cut into column blocks of 64 elements, each a
// [128][64] tile of its own, kBlockBytes apart (two TMA boxes per tile).
// Float32 storage stages two such tiles per tensor tile (the hi and lo planes
// of the operand prologue).
#pragma once

#include "nea_device.cuh"

namespace nea {

constexpr int kTileRows = 128;

template <int D>
struct TileGeom {
  static constexpr uint32_t kRowBytes = 2 * D <= 128 ? 2 * D : 128;  // swizzle atom row of a column block
  static constexpr uint32_t kBlocks = 2 * D / kRowBytes;             // column blocks of a row
  static constexpr uint32_t kBlockBytes = kTileRows * kRowBytes;     // one column block of a tile
  static constexpr uint32_t kOpBytes = kTileRows * 2 * D;            // one bf16 operand tile
  // byte offset of the 16-column K slice kk of a K-major tile
  __host__ __device__ static constexpr uint32_t kslice(int kk) {
    return (kk * 32) % kRowBytes + (kk * 32) / kRowBytes * kBlockBytes;
  }
};

// Bytes a TMA tile occupies, and the operand tiles it becomes: fp32 storage
// gives two bf16 tiles (hi, lo) in the same bytes; bf16 storage one.
template <int D, bool F32IO>
struct Stage {
  static constexpr uint32_t kBytes = kTileRows * D * (F32IO ? 4 : 2);
  static constexpr uint32_t kLo = TileGeom<D>::kOpBytes;  // offset of the lo tile (fp32 storage)
};

// Turns the pair (x0, x1) by the angle with cosine c and sine s (rotary
// embedding on queries and keys: "NanoEuler" write-up, aimsg.uk, section 2
// "Model components"; with s negated, the inverse rotation).
__device__ __forceinline__ void rot2(float& x0, float& x1, float c, float s) {
  const float y0 = x0 * c - x1 * s;
  const float y1 = x0 * s + x1 * c;
  x0 = y0;
  x1 = y1;
}

// Writes N consecutive elements of a row held in registers (float) at
// element offset `off` of a tensor in the storage type (16-byte aligned).
template <int N, bool F32IO>
__device__ __forceinline__ void store_span(void* dst, size_t off, const float* v) {
  if constexpr (F32IO) {
    float4* q = reinterpret_cast<float4*>(static_cast<float*>(dst) + off);
#pragma unroll
    for (int i = 0; i < N / 4; ++i) q[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else {
    uint4* q = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst) + off);
#pragma unroll
    for (int i = 0; i < N / 8; ++i)
      q[i] = make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                        pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
  }
}

}  // namespace nea
