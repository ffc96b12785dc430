// Operand prologue: one pass over the inputs that applies the rotary
// embedding to queries and keys ("NanoEuler" write-up, aimsg.uk, section 2
// "Model components": RoPE on queries and keys) before the attention kernels
// stage them with TMA directly in the tensor-core operand layout.
//   - float32 storage: every element of Q, K, V (and dO in the backward) is
//     written as two bf16 planes, hi = bf16(x) and lo = bf16(x - hi), in the
//     same [B][T][H][D] layout; the kernels form each product from three bf16
//     products (hi*hi + hi*lo + lo*hi).  Reads 4 bytes and writes 4 per element.
//   - bfloat16 storage: Q and K are rotated into bf16 copies (V and dO are
//     read in place).  Reads 2 bytes and writes 2 per element.
// In the backward the same launch also writes the per-row terms of every
// query row (below); for float32 storage the threads that read dO for them
// also write its hi/lo planes, so dO is read once.  Everything here is bound
// by HBM bandwidth.
#pragma once

#include "nea_device.cuh"

namespace nea {

struct PrepJob {
  const void* src;        // [B][T][H][D], fp32 or bf16
  __nv_bfloat16* hi;      // same layout: bf16(x) (fp32), the rotated copy (bf16)
  __nv_bfloat16* lo;      // same layout: bf16(x - hi) (fp32 only)
  long long chunks;       // 16-byte chunks: B*T*H*D / 4 (fp32), / 8 (bf16)
  int rows;               // B*T*H head vectors
  int block0;             // first block of this job
  int H;                  // heads of this tensor
  int rope;               // 1: rotate (queries, keys)
  FastDiv divH;           // division by H
};

struct PrepParams {
  PrepJob job[4];
  int n_jobs;
  int T;
  const float2* rope;     // [T][D/2] (cos, sin) or nullptr
  long long total;        // sum of chunks
  int prep_blocks;        // blocks [0, prep_blocks) rotate/split, kPrepUnroll rows' chunks per thread
  // backward row terms (rt_rows == 0: none), blocks from prep_blocks on
  const void* O;
  const void* dO;
  const float* LSE;
  float* ws;
  __nv_bfloat16* do_hi;   // float32 storage: dO's bf16 planes, written with the row terms
  __nv_bfloat16* do_lo;
  int B, Tp, Hq;
  long long rt_rows;      // B * Tp * Hq
  FastDiv divT, divTp, divHq;
};

constexpr int kPrepUnroll = 4;  // 16-byte chunks in flight per thread

// ---------------------------------------------------------------- row term
// Per-row terms of the backward, in a workspace ws[B*Hq][2][Tp] (Tp = T
// rounded up to whole 128-row tiles, so a tile of it is one TMA box):
//   ws[bh][0][t] = -LSE[b][h][t] * log2(e)          (-inf for t >= T)
//   ws[bh][1][t] = Dv = sum_d dO[b][t][h][d] O[b][t][h][d]   (0 for t >= T)
// The padding makes P = exp2(s*c + ws0) vanish for queries past T.  A group
// of D/ELEMS consecutive lanes takes one (b, t, h) row, t over [0, Tp), one
// 16-byte chunk of O and dO per lane; each thread takes kPrepUnroll rows of
// the block (kSlots rows apart) with all their loads in flight at once.
template <int D, bool F32IO>
__device__ __forceinline__ void rowterm_block(const PrepParams& p, long long rb) {
  constexpr int kElems = F32IO ? 4 : 8;    // elements per 16-byte chunk
  constexpr int kLanes = D / kElems;       // lanes per row: 4, 8 or 16
  constexpr int kSlots = 256 / kLanes;     // rows per block step
  constexpr int kRowBytes = D * (F32IO ? 4 : 2);
  const int c = int(threadIdx.x) % kLanes, slot = int(threadIdx.x) / kLanes;
  uint4 a[kPrepUnroll], z[kPrepUnroll];
  long long row[kPrepUnroll];  // (b, t, h) row of O and dO; -1: padding row (t >= T); -2: past the end
  float* out[kPrepUnroll];
  int bh_t[kPrepUnroll];
#pragma unroll
  for (int u = 0; u < kPrepUnroll; ++u) {
    const long long prow = (rb * kPrepUnroll + u) * kSlots + slot;  // (b, t, h) over t in [0, Tp)
    row[u] = -2;
    if (prow >= p.rt_rows) continue;
    const uint32_t bt = fdiv(uint32_t(prow), p.divHq);
    const int h = int(uint32_t(prow) - bt * uint32_t(p.Hq));
    const uint32_t bq = fdiv(bt, p.divTp);
    const int t = int(bt - bq * uint32_t(p.Tp));
    const long long b = bq;
    out[u] = p.ws + (b * p.Hq + h) * 2 * (long long)p.Tp + t;
    bh_t[u] = int((b * p.Hq + h) * (long long)p.T + t);
    row[u] = -1;
    if (t >= p.T) continue;
    row[u] = (b * p.T + t) * p.Hq + h;
    a[u] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.O) + row[u] * kRowBytes) + c);
    z[u] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.dO) + row[u] * kRowBytes) + c);
  }
  // the kLanes lanes of a row are consecutive and share its row index
  const unsigned group = (kLanes == 32 ? kFullMask : ((1u << kLanes) - 1u) << (threadIdx.x & 31 & ~(kLanes - 1)));
#pragma unroll
  for (int u = 0; u < kPrepUnroll; ++u) {
    if (row[u] == -2) continue;
    if (row[u] == -1) {
      if (c == 0) {
        out[u][0] = -INFINITY;
        out[u][p.Tp] = 0.f;
      }
      continue;
    }
    float acc;
    if constexpr (F32IO) {
      const float4 x = make_float4(__uint_as_float(a[u].x), __uint_as_float(a[u].y), __uint_as_float(a[u].z),
                                   __uint_as_float(a[u].w));
      const float4 y = make_float4(__uint_as_float(z[u].x), __uint_as_float(z[u].y), __uint_as_float(z[u].z),
                                   __uint_as_float(z[u].w));
      acc = x.x * y.x + x.y * y.y + x.z * y.z + x.w * y.w;
      if (p.do_hi) {  // dO's planes for the gradient kernel
        uint2 hi, lo;
        split_bf16(y.x, y.y, hi.x, lo.x);
        split_bf16(y.z, y.w, hi.y, lo.y);
        const size_t ci = size_t(row[u]) * kLanes + c;
        reinterpret_cast<uint2*>(p.do_hi)[ci] = hi;
        reinterpret_cast<uint2*>(p.do_lo)[ci] = lo;
      }
    } else {
      acc = bf16_lo_f(a[u].x) * bf16_lo_f(z[u].x) + bf16_hi_f(a[u].x) * bf16_hi_f(z[u].x) +
            bf16_lo_f(a[u].y) * bf16_lo_f(z[u].y) + bf16_hi_f(a[u].y) * bf16_hi_f(z[u].y) +
            bf16_lo_f(a[u].z) * bf16_lo_f(z[u].z) + bf16_hi_f(a[u].z) * bf16_hi_f(z[u].z) +
            bf16_lo_f(a[u].w) * bf16_lo_f(z[u].w) + bf16_hi_f(a[u].w) * bf16_hi_f(z[u].w);
    }
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(group, acc, off);
    if (c == 0) {
      out[u][0] = __ldg(p.LSE + bh_t[u]) * -1.4426950408889634f;
      out[u][p.Tp] = acc;
    }
  }
}

// Blocks of the row-term pass for `rows` (b, t, h) rows.
template <int D, bool F32IO>
__host__ __device__ constexpr long long rowterm_blocks(long long rows) {
  return (rows + (256 / (D / (F32IO ? 4 : 8))) * kPrepUnroll - 1) / ((256 / (D / (F32IO ? 4 : 8))) * kPrepUnroll);
}

// One 16-byte chunk (chunk c of a head vector at position t) of job tensor
// data: rotate (queries, keys) and convert.
template <int D, bool F32IO>
__device__ __forceinline__ void prep_chunk(const PrepParams& p, const PrepJob& job, size_t ci, int c, int t,
                                           uint4 raw) {
  constexpr int kPerChunk = F32IO ? 4 : 8;  // elements per 16-byte chunk
  float x[kPerChunk];
  if constexpr (F32IO) {
    x[0] = __uint_as_float(raw.x), x[1] = __uint_as_float(raw.y);
    x[2] = __uint_as_float(raw.z), x[3] = __uint_as_float(raw.w);
  } else {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) x[2 * k] = bf16_lo_f(w[k]), x[2 * k + 1] = bf16_hi_f(w[k]);
  }
  if (job.rope) {
    const float4* cs = reinterpret_cast<const float4*>(p.rope + size_t(t) * (D / 2) + (kPerChunk / 2) * c);
#pragma unroll
    for (int k = 0; k < kPerChunk / 4; ++k) {
      const float4 r = __ldg(cs + k);  // (cos, sin) of two pairs
      float* y = x + 4 * k;
      const float y0 = y[0] * r.x - y[1] * r.y, y1 = y[0] * r.y + y[1] * r.x;
      const float y2 = y[2] * r.z - y[3] * r.w, y3 = y[2] * r.w + y[3] * r.z;
      y[0] = y0, y[1] = y1, y[2] = y2, y[3] = y3;
    }
  }
  if constexpr (F32IO) {
    uint2 hi, lo;
    split_bf16(x[0], x[1], hi.x, lo.x);
    split_bf16(x[2], x[3], hi.y, lo.y);
    reinterpret_cast<uint2*>(job.hi)[ci] = hi;
    reinterpret_cast<uint2*>(job.lo)[ci] = lo;
  } else {
    reinterpret_cast<uint4*>(job.hi)[ci] =
        make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
  }
}

// Work blocks [0, prep_blocks) cover the jobs' head vectors in memory order,
// the job chosen once per block: thread t takes chunk t % CPR of kPrepUnroll
// rows (CPR chunks per row), so a warp reads and writes contiguous 512-byte
// runs and the position of each row is found once per row, not per element.
// The remaining work blocks write the row terms.
template <int D, bool F32IO>
__device__ __forceinline__ void prep_block(const PrepParams& p, int vb) {
  constexpr int CPR = D * (F32IO ? 4 : 2) / 16;   // 16-byte chunks per head vector
  constexpr int kSlots = 256 / CPR;               // rows per block step
  int j = 0;
  while (j + 1 < p.n_jobs && vb >= p.job[j + 1].block0) ++j;
  const PrepJob& job = p.job[j];
  const int c = threadIdx.x % CPR;
  const int row0 = (vb - job.block0) * kSlots * kPrepUnroll + threadIdx.x / CPR;
  uint4 raw[kPrepUnroll];
#pragma unroll
  for (int u = 0; u < kPrepUnroll; ++u) {
    const int ri = row0 + u * kSlots;
    if (ri < job.rows) raw[u] = __ldg(reinterpret_cast<const uint4*>(job.src) + size_t(ri) * CPR + c);
  }
#pragma unroll
  for (int u = 0; u < kPrepUnroll; ++u) {
    const int ri = row0 + u * kSlots;
    if (ri >= job.rows) break;
    const uint32_t bt = fdiv(uint32_t(ri), job.divH);  // (b, t) of the row
    const int t = int(bt - fdiv(bt, p.divT) * uint32_t(p.T));
    prep_chunk<D, F32IO>(p, job, size_t(ri) * CPR + c, c, t, raw[u]);
  }
}

// One CTA per work block.
template <int D, bool F32IO>
__global__ void __launch_bounds__(256) attn_prep_kernel(const __grid_constant__ PrepParams p) {
  grid_dep_wait();
  grid_dep_launch();
  if (int(blockIdx.x) >= p.prep_blocks) rowterm_block<D, F32IO>(p, (long long)(blockIdx.x - p.prep_blocks));
  else prep_block<D, F32IO>(p, int(blockIdx.x));
}

}  // namespace nea
