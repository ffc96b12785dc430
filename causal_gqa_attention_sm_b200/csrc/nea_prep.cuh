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
// Both are bound by HBM bandwidth.
#pragma once

#include "nea_device.cuh"

namespace nea {

struct PrepJob {
  const void* src;        // [B][T][H][D], fp32 or bf16
  __nv_bfloat16* hi;      // same layout: bf16(x) (fp32), the rotated copy (bf16)
  __nv_bfloat16* lo;      // same layout: bf16(x - hi) (fp32 only)
  long long chunks;       // 16-byte chunks: B*T*H*D / 4 (fp32), / 8 (bf16)
  int H;                  // heads of this tensor
  int rope;               // 1: rotate (queries, keys)
};

struct PrepParams {
  PrepJob job[4];
  int n_jobs;
  int T;
  const float2* rope;     // [T][D/2] (cos, sin) or nullptr
  long long total;        // sum of chunks
};

template <int D, bool F32IO>
__global__ void __launch_bounds__(256) attn_prep_kernel(const __grid_constant__ PrepParams p) {
  constexpr int kPerChunk = F32IO ? 4 : 8;  // elements per 16-byte chunk
  constexpr int kCpr = D / kPerChunk;       // chunks per head vector
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < p.total; i += stride) {
    int j = 0;
    long long ci = i;
    while (j + 1 < p.n_jobs && ci >= p.job[j].chunks) {
      ci -= p.job[j].chunks;
      ++j;
    }
    const PrepJob& job = p.job[j];
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(job.src) + ci);
    float x[kPerChunk];
    if constexpr (F32IO) {
      x[0] = __uint_as_float(raw.x), x[1] = __uint_as_float(raw.y);
      x[2] = __uint_as_float(raw.z), x[3] = __uint_as_float(raw.w);
    } else {
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) x[2 * k] = bf16_lo_f(w[k]), x[2 * k + 1] = bf16_hi_f(w[k]);
    }
    if (job.rope && p.rope != nullptr) {
      const long long row = ci / kCpr;      // (b, t, h) row index
      const int c = int(ci % kCpr);         // pairs kPerChunk/2 * c ...
      const int t = int((row / job.H) % p.T);
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
}

}  // namespace nea
