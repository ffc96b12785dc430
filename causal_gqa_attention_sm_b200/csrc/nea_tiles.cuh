// Tile staging for the forward and backward kernels.
//
// A [128 rows][D] tile of one head of a [B][T][H][D] tensor arrives in shared
// memory by TMA (rows at or beyond T read as zero).  One warpgroup (128
// threads) then turns it, in place, into the bf16 operand layout the tcgen05
// MMAs read (rows of 2*D bytes, hardware swizzle whose atom equals the row),
// applying the rotary embedding to queries and keys on the way:
//   - float32 storage: the TMA lands a dense fp32 tile; every thread reads
//     its chunks, the warpgroup meets at an mbarrier, and every element is
//     written back as its bf16 rounding ("hi" tile, first half of the buffer)
//     and the bf16 rounding of the remainder ("lo" tile, second half);
//   - bfloat16 storage: the TMA lands the tile already swizzled; only queries
//     and keys are touched, each 16-byte chunk rotated where it lies.
//
// Rotary embedding (RoPE on queries and keys: "NanoEuler" write-up, aimsg.uk,
// section 2 "Model components"; "Tiny Hackable CUDA LM", section 1): the
// interleaved pair (x[2i], x[2i+1]) at position t turns by t * base^(-2i/D).
// The (cos, sin) of that angle is composed from two rows of a table of
// (cos, sin) computed in double precision on the host: the row of the
// 64-row block start t0 (global table) and the row of the offset t - t0
// (first 64 rows of the same table, resident in shared memory).
#pragma once

#include "nea_device.cuh"

namespace nea {

constexpr int kTileRows = 128;
constexpr int kRopeRows = 64;  // resident offset rows of the rotary table

template <int D>
struct TileGeom {
  static constexpr uint32_t kRowBytes = 2 * D;                      // bf16 operand row
  static constexpr uint32_t kOpBytes = kTileRows * kRowBytes;       // one bf16 operand tile
  static constexpr uint32_t kRopeBytes = kRopeRows * (D / 2) * 8;   // resident offset table
};

// Bytes a TMA tile occupies, and the operand tiles it becomes: fp32 storage
// gives two bf16 tiles (hi, lo) in the same bytes; bf16 storage one.
template <int D, bool F32IO>
struct Stage {
  static constexpr uint32_t kBytes = kTileRows * D * (F32IO ? 4 : 2);
  static constexpr uint32_t kLo = TileGeom<D>::kOpBytes;  // offset of the lo tile (fp32 storage)
};

__device__ __forceinline__ void rot2(float& x0, float& x1, float c, float s) {
  const float y0 = x0 * c - x1 * s;
  const float y1 = x0 * s + x1 * c;
  x0 = y0;
  x1 = y1;
}

// (cos, sin) of a + b from (cos, sin) of a and of b.
__device__ __forceinline__ float2 compose(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.y * b.x + a.x * b.y);
}

// Per-thread rotary bases of one tile: the (cos, sin) rows of the two 64-row
// block starts row0 and row0 + 64, restricted to the pairs this thread owns
// (NP pairs starting at pair p0).  `base_rows` points at those two rows, in
// shared memory, bulk-copied next to the tile.
template <int NP>
struct RopeBase {
  float2 b[2][NP];
};

template <int NP>
__device__ __forceinline__ void load_rope_base(RopeBase<NP>& rb, const float2* base_rows, int D, int p0) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int i = 0; i < NP; ++i) rb.b[h][i] = base_rows[h * (D / 2) + p0 + i];
}

// Bytes of the two base rows of a tile in the table that follows the T rows
// of the rotary table (tile j: rows T + 2j and T + 2j + 1).
template <int D>
struct RopeBaseRows {
  static constexpr uint32_t kBytes = 2 * (D / 2) * 8;
};

// ----------------------------------------------------------------- float32
// In-place conversion of a dense fp32 tile into swizzled bf16 hi/lo tiles.
// Thread pt owns 16-byte chunk column c = pt % (D/4) (two rotary pairs) of
// rows pt / (D/4) + k * (128 / (D/4)).  `conv_bar` (count 128) separates the
// read and write phases; returns false if that rendezvous was abandoned.
template <int D, bool ROPE>
__device__ __forceinline__ bool convert_f32_tile(uint8_t* tile, const float2* rope_off, const float2* base_rows,
                                                 int row0, int T, uint64_t* conv_bar, uint32_t conv_parity,
                                                 const WaitCtl& wc, int pt) {
  const float2* rope = base_rows;  // nullptr: no rotation
  constexpr int kCpr = D / 4;             // chunks per row
  constexpr int kRowStep = 128 / kCpr;    // rows between a thread's chunks
  constexpr int kPer = kCpr;              // chunks per thread (128 rows * kCpr / 128)
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  const int c = pt % kCpr, r0 = pt / kCpr;
  float4 x[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k)
    x[k] = *reinterpret_cast<const float4*>(tile + (size_t(r0 + k * kRowStep) * D + 4 * c) * 4);
  RopeBase<2> rb;
  if (ROPE && rope != nullptr) load_rope_base<2>(rb, base_rows, D, 2 * c);
  mbar_arrive(conv_bar);
  if (!wait_warp(conv_bar, conv_parity, wc, kErrWaitProducer)) return false;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int r = r0 + k * kRowStep;
    float4 v = x[k];
    if (ROPE && rope != nullptr && row0 + r < T) {
      const int h = r / kRopeRows;
      const float4 off = *reinterpret_cast<const float4*>(rope_off + (r % kRopeRows) * (D / 2) + 2 * c);
      const float2 cs0 = compose(rb.b[h][0], make_float2(off.x, off.y));
      const float2 cs1 = compose(rb.b[h][1], make_float2(off.z, off.w));
      rot2(v.x, v.y, cs0.x, cs0.y);
      rot2(v.z, v.w, cs1.x, cs1.y);
    }
    uint2 hi, lo;
    split_bf16(v.x, v.y, hi.x, lo.x);
    split_bf16(v.z, v.w, hi.y, lo.y);
    const uint32_t off = swizzle(uint32_t(r) * RB + uint32_t(c) * 8, RB);
    *reinterpret_cast<uint2*>(tile + off) = hi;
    *reinterpret_cast<uint2*>(tile + Stage<D, true>::kLo + off) = lo;
  }
  return true;
}

// ----------------------------------------------------------------- bfloat16
// In-place rotation of a swizzled bf16 tile (TMA-landed).  Thread pt owns
// chunk column c = pt % (D/8) (four rotary pairs); each chunk is rewritten
// where it lies, so no rendezvous is needed.
template <int D>
__device__ __forceinline__ void rotate_bf16_tile(uint8_t* tile, const float2* rope_off, const float2* base_rows,
                                                 int row0, int T, int pt) {
  if (base_rows == nullptr) return;
  constexpr int kCpr = D / 8;
  constexpr int kRowStep = 128 / kCpr;
  constexpr int kPer = kCpr;
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  const int c = pt % kCpr, r0 = pt / kCpr;
  RopeBase<4> rb;
  load_rope_base<4>(rb, base_rows, D, 4 * c);
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int r = r0 + k * kRowStep;
    if (row0 + r >= T) continue;
    const uint32_t off = swizzle(uint32_t(r) * RB + uint32_t(c) * 16, RB);
    uint4 v = *reinterpret_cast<const uint4*>(tile + off);
    const int h = r / kRopeRows;
    const float4* op = reinterpret_cast<const float4*>(rope_off + (r % kRopeRows) * (D / 2) + 4 * c);
    const float4 o0 = op[0], o1 = op[1];
    const float2 cs0 = compose(rb.b[h][0], make_float2(o0.x, o0.y));
    const float2 cs1 = compose(rb.b[h][1], make_float2(o0.z, o0.w));
    const float2 cs2 = compose(rb.b[h][2], make_float2(o1.x, o1.y));
    const float2 cs3 = compose(rb.b[h][3], make_float2(o1.z, o1.w));
    float a0 = bf16_lo_f(v.x), a1 = bf16_hi_f(v.x), a2 = bf16_lo_f(v.y), a3 = bf16_hi_f(v.y);
    float a4 = bf16_lo_f(v.z), a5 = bf16_hi_f(v.z), a6 = bf16_lo_f(v.w), a7 = bf16_hi_f(v.w);
    rot2(a0, a1, cs0.x, cs0.y);
    rot2(a2, a3, cs1.x, cs1.y);
    rot2(a4, a5, cs2.x, cs2.y);
    rot2(a6, a7, cs3.x, cs3.y);
    v = make_uint4(pack_bf16(a0, a1), pack_bf16(a2, a3), pack_bf16(a4, a5), pack_bf16(a6, a7));
    *reinterpret_cast<uint4*>(tile + off) = v;
  }
}

// Converts one TMA-landed tile for the MMAs: rotated (queries, keys: pass the
// tile's two base rows, or nullptr when the rotation is off) or not (values,
// output gradients).  bf16 tiles without rotation need no work.
// `conv_count` counts this warpgroup's rendezvous (one per fp32 tile).
template <int D, bool F32IO, bool ROPE>
__device__ __forceinline__ bool prepare_tile(uint8_t* tile, const float2* rope_off, const float2* base_rows,
                                             int row0, int T, uint64_t* conv_bar, uint32_t& conv_count,
                                             const WaitCtl& wc, int pt) {
  if constexpr (F32IO) {
    const bool ok =
        convert_f32_tile<D, ROPE>(tile, rope_off, base_rows, row0, T, conv_bar, conv_count & 1, wc, pt);
    ++conv_count;
    return ok;
  } else {
    if (ROPE) rotate_bf16_tile<D>(tile, rope_off, base_rows, row0, T, pt);
    return true;
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
