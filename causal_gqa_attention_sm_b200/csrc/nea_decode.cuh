// Decode attention over a key/value cache: one new query per sequence attends
// to the cached positions 0 .. len_b - 1, the last of which is its own (the
// generation path of the same causal attention: "NanoEuler" write-up,
// aimsg.uk, section 1, head-0 generation; scores, softmax and GQA head map
// as in the training path; RoPE on the query at its position, section 2
// "Model components").  The cache holds keys already rotated at their
// positions, so only the query is rotated here.
//
// The work is one pass over the cache, so it is bound by HBM bandwidth: it is
// split over the cache (128 positions per CTA) so that every SM streams its
// share, then the splits are merged with their log-sum-exp weights.
//   attn_decode_split_kernel   grid (ceil(Tc/128), Hkv, B), 128 threads: two
//     TMA loads bring the 128 key and value rows of one kv head into shared
//     memory at once (no registers held while they fly); the G query heads
//     of the group are scored against them, and each split writes its
//     unnormalised o (fp32), max m and sum l (base 2).  The last split of a
//     (sequence, kv head) to finish, found by an atomic count, merges the
//     splits into O and LSE.
// The group's G queries share every cache row read (G = Hq / Hkv <= 8).
#pragma once

#include <cuda.h>

#include "nea_tiles.cuh"

namespace nea {

constexpr int kDecChunk = 128;  // cached positions per split
constexpr int kDecMaxG = 8;     // query heads per kv head

struct DecodeParams {
  CUtensorMap tm_k;    // Kc [B][Tc][Hkv][D], box {D, 1, 128, 1}, no swizzle
  CUtensorMap tm_v;    // Vc, same
  const void* Q;       // [B][Hq][D] un-rotated queries
  const int* lens;     // [B]
  void* O;             // [B][Hq][D]
  float* LSE;          // [B][Hq]
  float* part;         // [B*Hq][n_split][D + 2]: o, then m and l (base 2)
  int* count;          // [B*Hkv] finished splits, zero at launch
  const float2* rope;  // [Tc][D/2] (cos, sin), nullptr: no rotation
  int B, Tc, Hq, Hkv, G, n_split;
  float scale_log2;    // log2(e) / sqrt(D)
  int* err;
  unsigned long long wait_limit;
};

// Clamps a cache length read from device memory; an out-of-range value is
// recorded in the status word (the call's inputs were invalid).
__device__ __forceinline__ int decode_len(const DecodeParams& p, int b) {
  int len = __ldg(p.lens + b);
  if (len < 0 || len > p.Tc) {
    if (threadIdx.x == 0) atomicCAS(p.err, 0, kErrBadLength);
    len = len < 0 ? 0 : p.Tc;
  }
  return len;
}

// One 16-byte chunk of a row in shared memory as floats (4 fp32 or 8 bf16).
template <bool F32IO>
__device__ __forceinline__ void smem_chunk(const uint8_t* row, int c, float* x) {
  const uint4 u = reinterpret_cast<const uint4*>(row)[c];
  if constexpr (F32IO) {
    x[0] = __uint_as_float(u.x), x[1] = __uint_as_float(u.y), x[2] = __uint_as_float(u.z), x[3] = __uint_as_float(u.w);
  } else {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) x[2 * k] = bf16_lo_f(w[k]), x[2 * k + 1] = bf16_hi_f(w[k]);
  }
}

// The same chunk as packed float pairs (elements 2k, 2k + 1 in pair k).
template <bool F32IO>
__device__ __forceinline__ void smem_chunk2(const uint8_t* row, int c, uint64_t* x) {
  const uint4 u = reinterpret_cast<const uint4*>(row)[c];
  if constexpr (F32IO) {
    x[0] = f2_pack(__uint_as_float(u.x), __uint_as_float(u.y));
    x[1] = f2_pack(__uint_as_float(u.z), __uint_as_float(u.w));
  } else {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = f2_pack(bf16_lo_f(w[k]), bf16_hi_f(w[k]));
  }
}

template <bool F32IO>
__device__ __forceinline__ float load_elem(const void* base, size_t elem_off) {
  if constexpr (F32IO) return __ldg(static_cast<const float*>(base) + elem_off);
  else return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[elem_off]);
}

template <int D, bool F32IO>
struct DecSmem {
  static constexpr uint32_t kRow = D * (F32IO ? 4 : 2);
  static constexpr uint32_t kK = 0;                               // [128][D] keys
  static constexpr uint32_t kV = kK + kDecChunk * kRow;           // [128][D] values
  static constexpr uint32_t kQ = kV + kDecChunk * kRow;           // [8][D] f32 queries
  static constexpr uint32_t kS = kQ + kDecMaxG * D * 4;           // [8][128] f32 scores, then P
  static constexpr uint32_t kRed = kK;                            // [4 warps][8][D] f32 partial P V (over the keys)
  static constexpr uint32_t kMl = kS + kDecMaxG * kDecChunk * 4;  // [8][2] f32
  static constexpr uint32_t kBar = kMl + kDecMaxG * 8;            // mbarrier
  static constexpr uint32_t kBytes = kBar + 16;
};

// Each cached row is read from shared memory by a group of L = D*elem/16
// lanes, one 16-byte chunk each; 128 / L rows at a time.
template <int D, bool F32IO, int G>
__global__ void __launch_bounds__(128) attn_decode_split_kernel(const __grid_constant__ DecodeParams p) {
  using S = DecSmem<D, F32IO>;
  constexpr int EPC = F32IO ? 4 : 8;  // elements per chunk
  constexpr int L = D / EPC;          // lanes per row: 4, 8 or 16
  constexpr int R = 128 / L;          // rows in flight
  constexpr int NR = kDecChunk / R;   // rows per row slot
  extern __shared__ __align__(128) uint8_t sm[];
  float (*qs)[D] = reinterpret_cast<float (*)[D]>(sm + S::kQ);
  float (*sc)[kDecChunk] = reinterpret_cast<float (*)[kDecChunk]>(sm + S::kS);
  float* red = reinterpret_cast<float*>(sm + S::kRed);
  float (*ml)[2] = reinterpret_cast<float (*)[2]>(sm + S::kMl);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S::kBar);

  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int len = decode_len(p, b);
  const int j0 = s * kDecChunk;
  if (len == 0 && s == 0) {  // empty cache: O = 0, LSE = -inf
    for (int e = tid; e < G * D; e += blockDim.x) {
      const size_t bh = size_t(b) * p.Hq + g * G + e / D;
      if constexpr (F32IO) static_cast<float*>(p.O)[bh * D + e % D] = 0.f;
      else static_cast<__nv_bfloat16*>(p.O)[bh * D + e % D] = __float2bfloat16_rn(0.f);
      if (e % D == 0) p.LSE[bh] = -INFINITY;
    }
  }
  if (j0 >= len) return;  // no cached position of this split
  const int n = min(kDecChunk, len - j0);
  const int r = tid / L, c = tid % L;  // row slot, chunk of the row
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + S::kBar + 8);
  const WaitCtl wc{p.err, p.wait_limit, abort_flag};

  // ---- both 128-row chunks in flight at once
  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar, 1);
    mbar_init_fence();
    mbar_arrive_expect_tx(bar, 2 * kDecChunk * S::kRow);
    tma_load_4d(sm + S::kK, &p.tm_k, 0, g, j0, b, bar);
    tma_load_4d(sm + S::kV, &p.tm_v, 0, g, j0, b, bar);
  }

  // ---- queries of the group, rotated at position len - 1 and pre-scaled
  for (int e = tid; e < G * (D / 2); e += blockDim.x) {
    const int gi = e / (D / 2), i = e % (D / 2);
    const size_t qo = (size_t(b) * p.Hq + g * G + gi) * D + 2 * i;
    float x0 = load_elem<F32IO>(p.Q, qo), x1 = load_elem<F32IO>(p.Q, qo + 1);
    if (p.rope) {
      const float2 cs = __ldg(p.rope + size_t(len - 1) * (D / 2) + i);
      rot2(x0, x1, cs.x, cs.y);
    }
    qs[gi][2 * i] = x0 * p.scale_log2;
    qs[gi][2 * i + 1] = x1 * p.scale_log2;
  }
  __syncthreads();  // also publishes the barrier's initialisation
  const bool ok = wait_warp(bar, 0, wc, kErrWaitProducer);

  // ---- scores: lane (r, c) forms the partial dot products of its chunk c
  // with every head for the rows r, r + R, ... of its slot (NR == L rows; the
  // rows past n hold cache data or the copy's zero fill and are masked by the
  // softmax), then the L lanes of the slot trade halves of their partials,
  // log2 L times, so that lane c ends with the complete scores of row r + c R:
  // G (L - 1) shuffles per lane instead of G L log2 L.
  static_assert(NR == L, "one complete row per lane after the exchange");
  if (ok) {
    uint64_t q2[G][EPC / 2];  // this lane's chunk of every query, in pairs
#pragma unroll
    for (int gi = 0; gi < G; ++gi)
#pragma unroll
      for (int e = 0; e < EPC / 2; ++e) q2[gi][e] = f2_pack(qs[gi][c * EPC + 2 * e], qs[gi][c * EPC + 2 * e + 1]);
    float part[NR][G];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      uint64_t k2[EPC / 2];
      smem_chunk2<F32IO>(sm + S::kK + (r + i * R) * S::kRow, c, k2);
#pragma unroll
      for (int gi = 0; gi < G; ++gi) {
        uint64_t acc = f2_mul(q2[gi][0], k2[0]);
#pragma unroll
        for (int e = 1; e < EPC / 2; ++e) acc = f2_fma(q2[gi][e], k2[e], acc);
        float a0, a1;
        f2_unpack(acc, a0, a1);
        part[i][gi] = a0 + a1;
      }
    }
#pragma unroll
    for (int h = L / 2; h >= 1; h /= 2) {
      const bool up = (c & h) != 0;
#pragma unroll
      for (int j = 0; j < h; ++j)
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
          const float keep = up ? part[j + h][gi] : part[j][gi];
          const float send = up ? part[j][gi] : part[j + h][gi];
          part[j][gi] = keep + __shfl_xor_sync(kFullMask, send, h);
        }
    }
#pragma unroll
    for (int gi = 0; gi < G; ++gi) sc[gi][r + c * R] = part[0][gi];
  }
  __syncthreads();

  // ---- per query head: split max, P = exp2(s - m), split sum (one warp per head)
  for (int gi = warp; ok && gi < G; gi += 4) {
    float v[kDecChunk / 32];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kDecChunk / 32; ++i) {
      const int t = lane + 32 * i;
      v[i] = t < n ? sc[gi][t] : -INFINITY;
      m = fmaxf(m, v[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
    float l = 0.f;
#pragma unroll
    for (int i = 0; i < kDecChunk / 32; ++i) {
      const float e = ex2(v[i] - m);  // 0 past n
      sc[gi][lane + 32 * i] = e;
      l += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(kFullMask, l, off);
    if (lane == 0) {
      ml[gi][0] = m;
      ml[gi][1] = l;
    }
  }
  __syncthreads();

  // ---- o = P V: lane (r, c) sums rows r, r + R, ... of its chunk's columns,
  // then the row slots of a warp are folded by shuffles, the warps in smem
  uint64_t o2[G][EPC / 2];  // packed pairs of this lane's chunk columns
#pragma unroll
  for (int gi = 0; gi < G; ++gi)
#pragma unroll
    for (int e = 0; e < EPC / 2; ++e) o2[gi][e] = 0;  // the bit pattern of (+0, +0)
  if (ok) {
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int t = r + i * R;
      if (t >= n) break;  // never touch values past the cache length
      uint64_t v2[EPC / 2];
      smem_chunk2<F32IO>(sm + S::kV + t * S::kRow, c, v2);
#pragma unroll
      for (int gi = 0; gi < G; ++gi) {
        const float pw = sc[gi][t];
        const uint64_t pw2 = f2_pack(pw, pw);
#pragma unroll
        for (int e = 0; e < EPC / 2; ++e) o2[gi][e] = f2_fma(pw2, v2[e], o2[gi][e]);
      }
    }
  }
#pragma unroll
  for (int off = L; off < 32; off <<= 1)
#pragma unroll
    for (int gi = 0; gi < G; ++gi)
#pragma unroll
      for (int e = 0; e < EPC / 2; ++e) {
        float lo, hi;
        f2_unpack(o2[gi][e], lo, hi);
        o2[gi][e] = f2_add(o2[gi][e], f2_pack(__shfl_xor_sync(kFullMask, lo, off), __shfl_xor_sync(kFullMask, hi, off)));
      }
  if (lane < L)
#pragma unroll
    for (int gi = 0; gi < G; ++gi)
#pragma unroll
      for (int e = 0; e < EPC / 2; ++e) {
        float lo, hi;
        f2_unpack(o2[gi][e], lo, hi);
        *reinterpret_cast<float2*>(&red[(warp * kDecMaxG + gi) * D + c * EPC + 2 * e]) = make_float2(lo, hi);
      }
  __syncthreads();
  for (int e = tid; ok && e < G * D; e += blockDim.x) {
    const int gi = e / D, d = e % D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) acc += red[(w * kDecMaxG + gi) * D + d];
    float* dst = p.part + ((size_t(b) * p.Hq + g * G + gi) * p.n_split + s) * (D + 2);
    dst[d] = acc;
    if (d == 0) {
      dst[D] = ml[gi][0];
      dst[D + 1] = ml[gi][1];
    }
  }
  if (!ok) {
    if (tid == 0) drain_wait(bar, 0, wc);  // never exit with the copies in flight
    return;
  }

  // ---- the last split to finish merges: M = max m_s, w_s = 2^(m_s - M),
  // O = sum w_s o_s / sum w_s l_s, LSE = ln(2^M sum w_s l_s)
  __shared__ int last;
  __threadfence();  // this split's partials before its count
  __syncthreads();
  const int ns = (len + kDecChunk - 1) / kDecChunk;
  if (tid == 0) last = atomicAdd(p.count + b * p.Hkv + g, 1) == ns - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  // split weights of every head of the group staged in shared memory (the
  // score buffer is free now), then one independent load per split and column
  float* wsh = reinterpret_cast<float*>(sm + S::kS);  // [G][ns_max], ns <= 128 per pass
  for (int q0 = 0; q0 < ns; q0 += kDecChunk) {
    const int nq = min(kDecChunk, ns - q0);
    // pass 1: per head, the max over all splits (first chunk of splits only
    // needs it once; later chunks reuse it through ml)
    if (q0 == 0) {
      for (int gi = warp; gi < G; gi += 4) {
        const float* src = p.part + (size_t(b) * p.Hq + g * G + gi) * p.n_split * (D + 2);
        float m = -INFINITY;
        for (int q = lane; q < ns; q += 32) m = fmaxf(m, __ldcg(src + q * (D + 2) + D));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
        float l = 0.f;
        for (int q = lane; q < ns; q += 32) l += ex2(__ldcg(src + q * (D + 2) + D) - m) * __ldcg(src + q * (D + 2) + D + 1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(kFullMask, l, off);
        if (lane == 0) {
          ml[gi][0] = m;
          ml[gi][1] = l;
        }
      }
      __syncthreads();
    }
    for (int e = tid; e < G * nq; e += blockDim.x) {
      const int gi = e / nq, q = q0 + e % nq;
      const float* src = p.part + (size_t(b) * p.Hq + g * G + gi) * p.n_split * (D + 2);
      wsh[gi * kDecChunk + (q - q0)] = ex2(__ldcg(src + q * (D + 2) + D) - ml[gi][0]);
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += blockDim.x) {
      const int gi = e / D, d = e % D;
      const size_t bh = size_t(b) * p.Hq + g * G + gi;
      const float* src = p.part + bh * p.n_split * (D + 2);
      float o = q0 == 0 ? 0.f : red[gi * D + d];  // running sum over earlier split chunks
#pragma unroll 8
      for (int q = 0; q < nq; ++q) o = fmaf(wsh[gi * kDecChunk + q], __ldcg(src + (q0 + q) * (D + 2) + d), o);
      red[gi * D + d] = o;
    }
    __syncthreads();
  }
  for (int e = tid; e < G * D; e += blockDim.x) {
    const int gi = e / D, d = e % D;
    const size_t bh = size_t(b) * p.Hq + g * G + gi;
    const float out = red[gi * D + d] / ml[gi][1];
    if constexpr (F32IO) static_cast<float*>(p.O)[bh * D + d] = out;
    else static_cast<__nv_bfloat16*>(p.O)[bh * D + d] = __float2bfloat16_rn(out);
    // LSE = ln(2^m * l): m, l are in base-2 units of the scaled scores
    if (d == 0) p.LSE[bh] = (ml[gi][0] + log2f(ml[gi][1])) * 0.69314718055994531f;
  }
}

}  // namespace nea
