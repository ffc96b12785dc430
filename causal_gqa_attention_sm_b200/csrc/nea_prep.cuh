// Operand prologue of the float32-storage path: one pass over Q, K, V (and
// dO in the backward) that applies the rotary embedding to queries and keys
// ("NanoEuler" write-up, aimsg.uk, section 2 "Model components": RoPE on
// queries and keys) and writes every element as two bf16 planes, hi = bf16(x)
// and lo = bf16(x - hi), in the same [B][T][H][D] layout.  The attention
// kernels then stage those planes with TMA directly in the tensor-core
// operand layout and form each product from three bf16 products
// (hi*hi + hi*lo + lo*hi).  The pass reads each fp32 element once and writes
// 4 bytes for it, so it is bound by HBM bandwidth.
#pragma once

#include "nea_device.cuh"

namespace nea {

struct PrepJob {
  const float* src;       // [B][T][H][D] fp32
  __nv_bfloat16* hi;      // same layout, bf16(x)
  __nv_bfloat16* lo;      // same layout, bf16(x - hi)
  long long chunks;       // B*T*H*D / 4 (16-byte chunks of four floats)
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

template <int D>
__global__ void __launch_bounds__(256) attn_prep_split_kernel(const __grid_constant__ PrepParams p) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < p.total; i += stride) {
    int j = 0;
    long long ci = i;
    while (j + 1 < p.n_jobs && ci >= p.job[j].chunks) {
      ci -= p.job[j].chunks;
      ++j;
    }
    const PrepJob& job = p.job[j];
    float4 x = __ldg(reinterpret_cast<const float4*>(job.src) + ci);
    if (job.rope && p.rope != nullptr) {
      constexpr int kCpr = D / 4;           // chunks per head vector
      const long long row = ci / kCpr;      // (b, t, h) row index
      const int c = int(ci % kCpr);         // pairs 2c, 2c+1
      const int t = int((row / job.H) % p.T);
      const float4 cs = __ldg(reinterpret_cast<const float4*>(p.rope + size_t(t) * (D / 2) + 2 * c));
      const float y0 = x.x * cs.x - x.y * cs.y, y1 = x.x * cs.y + x.y * cs.x;
      const float y2 = x.z * cs.z - x.w * cs.w, y3 = x.z * cs.w + x.w * cs.z;
      x = make_float4(y0, y1, y2, y3);
    }
    uint2 hi, lo;
    split_bf16(x.x, x.y, hi.x, lo.x);
    split_bf16(x.z, x.w, hi.y, lo.y);
    reinterpret_cast<uint2*>(job.hi)[ci] = hi;
    reinterpret_cast<uint2*>(job.lo)[ci] = lo;
  }
}

}  // namespace nea
