// The steps on either side of the attention in a pre-norm decoder block
// ("NanoEuler" write-up, aimsg.uk, section 1 "Architecture design" and
// section 2 "Model components": RMSNorm pre-norm, bias-free projections,
// residual update x <- x + f(x)):
//   forward   y = x rstd g (rstd = (mean_j x_j^2 + eps)^-1/2 per token),
//             q = y Wq, k = y Wk, v = y Wv;   h = x + o Wo
//   backward  dWo = o^T dh, do = dh Wo^T;  dW* = y^T d*, dy = sum d* W*^T,
//             dx = rstd g dy - x rstd^3 / C sum_j (g dy)_j x_j (+ dh), dg = sum_tokens dy x rstd
// and the block's feed-forward half, a pre-norm SwiGLU ("NanoEuler" write-up,
// section 2, "SwiGLU feed-forward": down(silu(gate(x)) * up(x)), silu(z) =
// z sigmoid(z)), F its inner width:
//   forward   a = y Wg, b = y Wu, act = silu(a) b, h = x + act Wd
//   backward  dact = dh Wd^T, da = dact b silu'(a), db = dact silu(a),
//             dWd = act^T dh, dWg = y^T da, dWu = y^T db, dy = da Wg^T + db Wu^T,
//             silu'(a) = s (1 + a (1 - s)) with s = sigmoid(a)
// The products run on one tcgen05 GEMM kernel, C = A B with A [M x K] and B
// [K x N] stored row-major in either orientation (an operand whose reduction
// index is the contiguous one is "K-major", else "MN-major"); operands are
// bf16 (bfloat16 storage) or bf16 hi/lo planes (float32 storage: every
// product hi*hi + hi*lo + lo*hi, fp32 accumulation, as in the attention).
// RMSNorm's reductions are row kernels that write the GEMM operands.
#pragma once

#include "nea_device.cuh"

namespace nea {

// Tiles are 128 rows (M) by BN = 128 or 256 columns (N); a k-step covers 64
// of K.  A 256-wide tile halves the A traffic per FLOP, which matters because
// the operands stream from L2 for every tile: the host takes it where the
// tile count still fills the SMs.
constexpr int kGemmBM = 128, kGemmBN = 128, kGemmBK = 64;
// warp 0: TMA, warp 1: MMA, warps 2-9: epilogue (two warps per 32-lane TMEM
// quarter, each taking half of the tile's columns)
constexpr int kGemmThreads = 320;
constexpr int kGemmEpiWarps = 8;

// Up to three operand segments.  Chained along K (kseg): out = sum_s A_s B_s,
// segment s owning k-steps [begin_s, begin_{s+1}).  Side by side along N:
// out_s = A B_s for the N tiles [begin_s, begin_{s+1}), A taken from
// segment 0.  Operands: hi planes (bf16 storage: the tensors themselves), lo
// planes (float32 storage); K-major maps have box {64, 128}, MN-major {64, 64}.
constexpr int kGemmMaxSeg = 3;
struct GemmSeg {
  CUtensorMap a_hi, a_lo, b_hi, b_lo;
  void* out;          // N segments: this segment's output [M][ldo]
  long long ldo;
  int begin;          // first k-step (K segments) or first N tile (N segments)
};
struct GemmParams {
  GemmSeg seg[kGemmMaxSeg];
  int n_seg;
  int kseg;           // 1: segments along K; 0: along N (one segment: either)
  void* out;          // K segments: [M][ldo] row-major, fp32 or bf16
  const void* res;    // residual added to the result (same layout as out), or nullptr
  long long ldo;
  int M, N, K;
  int out_f32;        // 1: fp32 output, 0: bf16
  int n_m, n_n, n_k, n_tiles;  // tiles of 128 x BN (mode 1: 128 output columns of each of a, b)
  // split K: work unit u is tile u % n_tiles over k-steps of chunk u /
  // n_tiles; with split > 1 each unit writes an fp32 partial tile to
  // part[u][128][bn] and gemm_reduce_kernel sums them into the output
  int split, k_per;   // chunks, k-steps per chunk
  int bn;             // the launch's tile width
  float* part;
  // epilogue mode: 0 the plain store above; 1 the SwiGLU forward: a 256-wide
  // tile whose B halves are the same 128 columns of seg[0].b (Wg) and
  // seg[1].b (Wu), so that one accumulator holds a = y Wg beside b = y Wu;
  // the tile writes a and b (seg[0].out, seg[1].out, each optional) and the
  // operand planes of act = silu(a) b (pl[0] hi, pl[1] lo); 2 the SwiGLU backward,
  // the product dact = dh Wd^T combined with the forward's a and b (ab[0],
  // ab[1]) into the planes of da (pl[0], pl[1]), db (pl[2], pl[3]) and act
  // (pl[4], pl[5]).  Lo planes (float32 storage) may be null; modes 1 and 2
  // write [M][ldo] tensors and run unsplit.
  int mode;
  void* pl[6];
  const void* ab[2];
  int* err;
  unsigned long long wait_limit;
};

// Segment holding index i (a k-step or an N tile).
__device__ __forceinline__ int gemm_seg_of(const GemmParams& p, int i) {
  int s = 0;
  while (s + 1 < p.n_seg && i >= p.seg[s + 1].begin) ++s;
  return s;
}

// Writes value v of output element (row, tile column c) of tile `ni`: the
// tile's N segment (or the one output), residual added, fp32 or bf16.
__device__ __forceinline__ void gemm_store(const GemmParams& p, int row, int ni, int c, float v) {
  const int ns = p.kseg ? 0 : gemm_seg_of(p, ni);
  void* const out = p.kseg ? p.out : p.seg[ns].out;
  const long long ldo = p.kseg ? p.ldo : p.seg[ns].ldo;
  const int col = (ni - (p.kseg ? 0 : p.seg[ns].begin)) * p.bn + c;
  if (row >= p.M || col >= (p.kseg ? p.N : int(ldo))) return;
  const size_t o = size_t(row) * ldo + col;
  if (p.out_f32) {
    static_cast<float*>(out)[o] = v + (p.res ? static_cast<const float*>(p.res)[o] : 0.f);
  } else {
    const float r = p.res ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.res)[o]) : 0.f;
    static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(v + r);
  }
}

// Sums the split partial tiles in chunk order (deterministic) and stores
// the output: bn / 8 CTAs per 128 x bn tile, four consecutive elements per
// thread.
__global__ void __launch_bounds__(256) gemm_reduce_kernel(const __grid_constant__ GemmParams p) {
  grid_dep_wait();
  grid_dep_launch();
  const int per = p.bn / 8;  // CTAs per tile
  const int t = int(blockIdx.x) / per, mi = t % p.n_m, ni = t / p.n_m;
  const int e = ((int(blockIdx.x) % per) * 256 + threadIdx.x) * 4;  // element of the 128 x bn tile
  const size_t tile = size_t(128) * p.bn;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < p.split; ++s) {
    const float4 u = *reinterpret_cast<const float4*>(p.part + (size_t(s) * p.n_tiles + t) * tile + e);
    v.x += u.x, v.y += u.y, v.z += u.z, v.w += u.w;
  }
  const int row = mi * 128 + e / p.bn, c = e % p.bn;
  gemm_store(p, row, ni, c, v.x);
  gemm_store(p, row, ni, c + 1, v.y);
  gemm_store(p, row, ni, c + 2, v.z);
  gemm_store(p, row, ni, c + 3, v.w);
}

// n (<= 8) consecutive values of a row, starting at element o of a tensor
// in the storage type (fp32, or bf16 when !f32).  Full runs of 8 move as
// 16-byte vectors (o is then a multiple of 8).
__device__ __forceinline__ void row_load8(const void* src, size_t o, bool f32, int n, float* v) {
  if (n >= 8) {
    if (f32) {
      const float4 u0 = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + o);
      const float4 u1 = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + o + 4);
      v[0] = u0.x, v[1] = u0.y, v[2] = u0.z, v[3] = u0.w, v[4] = u1.x, v[5] = u1.y, v[6] = u1.z, v[7] = u1.w;
    } else {
      const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src) + o);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) v[2 * i] = bf16_lo_f(w[i]), v[2 * i + 1] = bf16_hi_f(w[i]);
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j)  // a ragged run: static indices keep v in registers
    v[j] = j >= n ? 0.f
                  : f32 ? static_cast<const float*>(src)[o + j]
                        : __bfloat162float(static_cast<const __nv_bfloat16*>(src)[o + j]);
}

__device__ __forceinline__ void row_store8(void* dst, size_t o, bool f32, int n, const float* v) {
  if (n >= 8) {
    if (f32) {
      *reinterpret_cast<float4*>(static_cast<float*>(dst) + o) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(static_cast<float*>(dst) + o + 4) = make_float4(v[4], v[5], v[6], v[7]);
    } else {
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst) + o) =
          make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= n) break;
    if (f32) static_cast<float*>(dst)[o + j] = v[j];
    else static_cast<__nv_bfloat16*>(dst)[o + j] = __float2bfloat16_rn(v[j]);
  }
}

// The same values as GEMM operand planes: bf16 hi, and when `lo` is given
// the bf16 rounding remainder.
__device__ __forceinline__ void row_planes8(void* hi, void* lo, size_t o, int n, const float* v) {
  auto* h = static_cast<__nv_bfloat16*>(hi) + o;
  auto* l = static_cast<__nv_bfloat16*>(lo) + o;
  if (n >= 8) {
    uint32_t hh[4], ll[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split_bf16(v[2 * i], v[2 * i + 1], hh[i], ll[i]);
    *reinterpret_cast<uint4*>(h) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
    if (lo) *reinterpret_cast<uint4*>(l) = make_uint4(ll[0], ll[1], ll[2], ll[3]);
    return;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= n) break;
    const __nv_bfloat16 b = __float2bfloat16_rn(v[j]);
    h[j] = b;
    if (lo) l[j] = __float2bfloat16_rn(v[j] - __bfloat162float(b));
  }
}

// Single elements of a tensor in the storage type (fp32, or bf16 when
// !f32), and of a GEMM operand's bf16 planes (hi, and when `lo` is given the
// rounding remainder), for the transposed SwiGLU epilogues, whose lanes hold
// consecutive columns of one row.
__device__ __forceinline__ float elem_load(const void* src, size_t o, bool f32) {
  if (f32) return __ldg(static_cast<const float*>(src) + o);
  return __uint_as_float(uint32_t(__ldg(static_cast<const unsigned short*>(src) + o)) << 16);
}

__device__ __forceinline__ void elem_store(void* dst, size_t o, bool f32, float v) {
  if (f32) static_cast<float*>(dst)[o] = v;
  else static_cast<__nv_bfloat16*>(dst)[o] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ void elem_planes(void* hi, void* lo, size_t o, float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  static_cast<__nv_bfloat16*>(hi)[o] = h;
  if (lo) static_cast<__nv_bfloat16*>(lo)[o] = __float2bfloat16_rn(v - __bfloat162float(h));
}

// 1 / (1 + e^-z) with the fast exponential and division intrinsics; z is
// clamped at -80 so that e^-z stays below 2^126 (the divide's range), which
// changes the result only where it is below 2e-35.
__device__ __forceinline__ float sigmoid_f(float z) { return __fdividef(1.f, 1.f + __expf(-fmaxf(z, -80.f))); }

template <bool SPLIT, int BN>
struct GemmSmem {
  static constexpr uint32_t kOp = 128 * 128;             // one 128 x 64 bf16 operand tile (16 KB)
  static constexpr uint32_t kOpB = BN * 128;             // the B tile: BN x 64
  static constexpr int kPlanes = SPLIT ? 2 : 1;
  static constexpr uint32_t kStage = kPlanes * (kOp + kOpB);  // A planes, then B planes
  static constexpr int ST = (200 * 1024) / kStage;       // 6, 4 (bf16); 3, 2 (split): 192 KB
  static constexpr uint32_t kEpi = ST * kStage;          // each epilogue warp's 32 x 33 fp32 staging rows
  static constexpr uint32_t kBars = kEpi + kGemmEpiWarps * 32 * 33 * 4;  // full[ST], empty[ST], acc_full[2], acc_empty[2]
  static constexpr uint32_t kMisc = kBars + (2 * ST + 4) * 8;  // TMEM base, abort flag
  static constexpr uint32_t kBytes = kMisc + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory");
};

__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// One 128 x 64 operand tile (rows of the M or N extent, 64 of K) into
// shared memory: K-major, one box of 128 rows x 128 bytes; MN-major, two
// boxes of 64 K-rows x 64 MN-elements (the two MN halves 8 KB apart).
template <bool MN>
__device__ __forceinline__ void gemm_load_tile(uint8_t* dst, const CUtensorMap* map, int mn0, int k0, uint64_t* bar) {
  if constexpr (MN) {
    tma_load_2d(dst, map, mn0, k0, bar);
    tma_load_2d(dst + 8192, map, mn0 + 64, k0, bar);
  } else {
    tma_load_2d(dst, map, k0, mn0, bar);
  }
}

// Descriptor of the 16-wide K slice kk of a tile.  K-major: rows of 128
// bytes, the slice 32 bytes on.  MN-major: K rows of 128 bytes (64 MN
// elements), the slice 16 rows on, the second MN half 8 KB on.
template <bool MN>
__device__ __forceinline__ uint64_t gemm_desc(uint32_t tile, int kk) {
  return MN ? smem_desc(tile + kk * 2048, 128, 8192) : smem_desc(tile + kk * 32, 128, 16);
}

template <bool AMN, bool BMN, bool SPLIT, int BN>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  using L = GemmSmem<SPLIT, BN>;
  static_assert(BN == 128 || BN == 256, "tile width");
  extern __shared__ uint8_t raw[];
  uint8_t* sm = raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* empty = full + L::ST;
  uint64_t* acc_full = empty + L::ST;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMisc + 4);
  const WaitCtl wc{p.err, p.wait_limit, abort_flag};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < L::ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kGemmEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init_fence();
  }
  // two accumulators of BN fp32 columns
  constexpr uint32_t tcols = 2 * BN, acc_cols = BN;
  if (warp == 1) tmem_alloc(tmem_holder, tcols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_tiles * p.split && ok; u += gridDim.x) {
        const int t = u % p.n_tiles, kb = (u / p.n_tiles) * p.k_per, ke = min(p.n_k, kb + p.k_per);
        const int mi = t % p.n_m, ni = t / p.n_m;
        const int ns = (p.kseg || p.mode == 1) ? 0 : gemm_seg_of(p, ni);  // N segment of the tile
        const GemmSeg& sa = p.seg[0];
        const int n0 = p.mode == 1 ? ni * 128 : (ni - (p.kseg ? 0 : p.seg[ns].begin)) * BN;
        for (int ks = kb; ks < ke; ++ks, ++it) {
          const int s = it % L::ST;
          if (it >= uint32_t(L::ST) && !(ok = wait_thread(&empty[s], ((it / L::ST) - 1) & 1, wc, kErrWaitEmpty)))
            break;
          const int kq = p.kseg ? gemm_seg_of(p, ks) : 0;  // K segment of the step
          const GemmSeg& g = p.kseg ? p.seg[kq] : p.seg[ns];
          const GemmSeg& ga = p.kseg ? p.seg[kq] : sa;
          const int k0 = (ks - (p.kseg ? p.seg[kq].begin : 0)) * kGemmBK;
          uint8_t* st = sm + s * L::kStage;
          mbar_arrive_expect_tx(&full[s], L::kStage);
          gemm_load_tile<AMN>(st, &ga.a_hi, mi * kGemmBM, k0, &full[s]);
          if constexpr (SPLIT) gemm_load_tile<AMN>(st + L::kOp, &ga.a_lo, mi * kGemmBM, k0, &full[s]);
          uint8_t* const sb = st + L::kPlanes * L::kOp;  // B planes: hi, then lo
#pragma unroll
          for (int h = 0; h < BN / 128; ++h) {  // 128-column halves (mode 1: Wg, then Wu)
            const GemmSeg& gb = p.mode == 1 ? p.seg[h] : g;
            const int nb = p.mode == 1 ? n0 : n0 + h * 128;
            gemm_load_tile<BMN>(sb + h * L::kOp, &gb.b_hi, nb, k0, &full[s]);
            if constexpr (SPLIT) gemm_load_tile<BMN>(sb + L::kOpB + h * L::kOp, &gb.b_lo, nb, k0, &full[s]);
          }
        }
      }
      // never exit with copies in flight
      for (uint32_t i = it > uint32_t(L::ST) ? it - L::ST : 0; i < it; ++i)
        drain_wait(&full[i % L::ST], (i / L::ST) & 1, wc);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    constexpr uint32_t idesc = idesc_bf16(kGemmBM, BN, AMN, BMN);
    uint32_t it = 0, last = 0xffffffffu;  // the last stage use committed
    int lt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.n_tiles * p.split && ok; u += gridDim.x, ++lt) {
      const int kb = (u / p.n_tiles) * p.k_per, ke = min(p.n_k, kb + p.k_per);
      const int ab = lt & 1;
      if (lt >= 2) ok = wait_warp(&acc_empty[ab], ((lt >> 1) - 1) & 1, wc, kErrWaitSoftmax);
      tc_fence_after();
      for (int ks = kb; ks < ke && ok; ++ks, ++it) {
        const int s = it % L::ST;
        if (!(ok = wait_warp(&full[s], (it / L::ST) & 1, wc, kErrWaitProducer))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a = smem_u32(sm + s * L::kStage);
          const uint32_t b = a + L::kPlanes * L::kOp;
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk) {
#pragma unroll
            for (int term = 0; term < (SPLIT ? 3 : 1); ++term) {
              // hi*hi, hi*lo, lo*hi
              const uint32_t ap = a + (term == 2 ? L::kOp : 0), bp = b + (term == 1 ? L::kOpB : 0);
              mma_ss(tbase + ab * acc_cols, gemm_desc<AMN>(ap, kk), gemm_desc<BMN>(bp, kk), idesc,
                     ((ks - kb) | kk | term) != 0);
            }
          }
          tc_commit(&empty[s]);
          if (ks == ke - 1) tc_commit(&acc_full[ab]);
          last = it;
        }
        __syncwarp();
      }
    }
    // commits complete in order: once the last has, no product is in flight
    if (lane == 0 && last != 0xffffffffu) drain_wait(&empty[last % L::ST], (last / L::ST) & 1, wc);
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q4 = warp & 3;         // TMEM lanes 32 q4 .. 32 q4 + 31
    const int ch = (warp - 2) >> 2;  // column half of the tile
    // float32 storage, SwiGLU epilogues: a 32-column chunk of the warp's 32
    // TMEM lanes goes through the warp's staging rows in shared memory
    // (padded to 33 words: no bank conflicts either way), so that lane l then
    // holds column l of the 32 rows and every global access is one row's 32
    // consecutive elements.  The per-row 16-byte accesses these epilogues
    // would otherwise make (fp32 a and b, hi/lo planes: 12 to 20 bytes per
    // element in 16-byte pieces of 32 rows per warp instruction) cost more
    // than the staging; for the plain stores and for bf16 storage the
    // staging's shared-memory traffic, which competes with the MMAs' operand
    // reads, costs more than it saves.
    float* const stage_rows = reinterpret_cast<float*>(sm + L::kEpi) + (warp - 2) * (32 * 33);
    // the chunk at TMEM column `col`: v[r] = row r of this lane's column
    auto load_chunk = [&](uint32_t col, float* v) {
      uint32_t r[32];
      tmem_ld32(tmem_addr(tbase, q4 * 32, col), r);
#pragma unroll
      for (int j = 0; j < 32; ++j) stage_rows[lane * 33 + j] = __uint_as_float(r[j]);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = stage_rows[i * 33 + lane];
      __syncwarp();
    };
    int lt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.n_tiles * p.split && ok; u += gridDim.x, ++lt) {
      const int t = u % p.n_tiles;
      const int ab = lt & 1;
      if (!(ok = wait_warp(&acc_full[ab], (lt >> 1) & 1, wc, kErrWaitMma))) break;
      tc_fence_after();
      if (p.split > 1) {  // this chunk's partial tile, row-major 128 x BN fp32
        float* dst = p.part + size_t(u) * 128 * BN + size_t(q4 * 32 + lane) * BN;
#pragma unroll 1
        for (int c = ch * (BN / 64); c < (ch + 1) * (BN / 64); ++c) {
          uint32_t r[32];
          tmem_ld32(tmem_addr(tbase, q4 * 32, ab * acc_cols + c * 32), r);
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + c * 32 + j) = make_float4(
                __uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        continue;
      }
      const int mi = t % p.n_m, ni = t / p.n_m;
      const int row0 = mi * kGemmBM + q4 * 32;  // the warp's first row
      const int nrow = min(32, p.M - row0);     // its rows inside the product (warp-uniform)
      if constexpr (SPLIT) {  // float32 storage: the SwiGLU epilogues through the staging rows
        if (p.mode != 0) {
          if (p.mode == 1) {
            // SwiGLU forward: b 128 columns beside a; writes a, b and act's planes
#pragma unroll 1
            for (int c = ch * 2; c < ch * 2 + 2; ++c) {
              float a[32], b[32];
              load_chunk(ab * acc_cols + c * 32, a);
              load_chunk(ab * acc_cols + 128 + c * 32, b);
              const int col = ni * 128 + c * 32 + lane;
              if (col < p.N) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {  // full unroll: static indices keep the arrays in registers
                  if (i >= nrow) break;
                  const size_t o = size_t(row0 + i) * p.ldo + col;
                  if (p.seg[0].out) elem_store(p.seg[0].out, o, p.out_f32, a[i]);
                  if (p.seg[1].out) elem_store(p.seg[1].out, o, p.out_f32, b[i]);
                  elem_planes(p.pl[0], p.pl[1], o, a[i] * sigmoid_f(a[i]) * b[i]);
                }
              }
            }
          } else {
            // SwiGLU backward: dact with the forward's a and b -> planes of da, db, act
#pragma unroll 1
            for (int c = ch * (BN / 64); c < (ch + 1) * (BN / 64); ++c) {
              float d[32], a[32], b[32];
              load_chunk(ab * acc_cols + c * 32, d);
              const int col = ni * BN + c * 32 + lane;
              if (col < p.N) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {  // all of the chunk's loads in flight together
                  const size_t o = size_t(row0 + min(i, nrow - 1)) * p.ldo + col;
                  a[i] = elem_load(p.ab[0], o, p.out_f32);
                  b[i] = elem_load(p.ab[1], o, p.out_f32);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {  // full unroll: static indices keep the arrays in registers
                  if (i >= nrow) break;
                  const size_t o = size_t(row0 + i) * p.ldo + col;
                  const float sg = sigmoid_f(a[i]), si = a[i] * sg;
                  elem_planes(p.pl[0], p.pl[1], o, d[i] * b[i] * sg * (1.f + a[i] * (1.f - sg)));  // da
                  elem_planes(p.pl[2], p.pl[3], o, d[i] * si);                                     // db
                  elem_planes(p.pl[4], p.pl[5], o, si * b[i]);                                     // act
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          continue;
        }
      }
      const int row = row0 + lane;
      if (!SPLIT && p.mode != 0) {  // bfloat16 storage: the SwiGLU epilogues, 32 columns of a row per pass, 8 at a time
        const int nc = p.mode == 1 ? 2 : BN / 64;  // 32-column chunks per warp
#pragma unroll 1
        for (int c = ch * nc; c < ch * nc + nc; ++c) {
          uint32_t r0[32], r1[32];
          const uint32_t tc = ab * acc_cols + c * 32;
          tmem_ld32(tmem_addr(tbase, q4 * 32, tc), r0);
          if (p.mode == 1) tmem_ld32(tmem_addr(tbase, q4 * 32, tc + 128), r1);  // b beside a
          const int col0 = (p.mode == 1 ? ni * 128 : ni * BN) + c * 32;
          if (row >= p.M || col0 >= p.N) continue;
          const size_t o0 = size_t(row) * p.ldo + col0;
          if (p.mode == 1) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              const int n = min(8, p.N - col0 - j);
              if (n <= 0) break;
              float a[8], b[8], x[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                a[i] = __uint_as_float(r0[j + i]), b[i] = __uint_as_float(r1[j + i]);
                x[i] = a[i] * sigmoid_f(a[i]) * b[i];  // act
              }
              if (p.seg[0].out) row_store8(p.seg[0].out, o0 + j, p.out_f32, n, a);
              if (p.seg[1].out) row_store8(p.seg[1].out, o0 + j, p.out_f32, n, b);
              row_planes8(p.pl[0], p.pl[1], o0 + j, n, x);
            }
          } else {
            float a[32], b[32];  // the chunk's a and b, all loads in flight together
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              row_load8(p.ab[0], o0 + j, p.out_f32, p.N - col0 - j, a + j);
              row_load8(p.ab[1], o0 + j, p.out_f32, p.N - col0 - j, b + j);
            }
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              const int n = min(8, p.N - col0 - j);
              if (n <= 0) break;
              float x[8], y[8], z[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float d = __uint_as_float(r0[j + i]), aa = a[j + i], bb = b[j + i];
                const float sg = sigmoid_f(aa), si = aa * sg;
                x[i] = d * bb * sg * (1.f + aa * (1.f - sg));  // da
                y[i] = d * si;                                 // db
                z[i] = si * bb;                                // act
              }
              row_planes8(p.pl[0], p.pl[1], o0 + j, n, x);
              row_planes8(p.pl[2], p.pl[3], o0 + j, n, y);
              row_planes8(p.pl[4], p.pl[5], o0 + j, n, z);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        continue;
      }
      // the tile's output: its N segment's tensor, or the one output
      const int ns = p.kseg ? 0 : gemm_seg_of(p, ni);
      void* const out_base = p.kseg ? p.out : p.seg[ns].out;
      const long long ldo = p.kseg ? p.ldo : p.seg[ns].ldo;
      const int ncol0 = (ni - (p.kseg ? 0 : p.seg[ns].begin)) * BN;  // first column in that tensor
      const int nlim = p.kseg ? p.N : int(ldo);                           // its column count
#pragma unroll 1
      for (int c = ch * (BN / 64); c < (ch + 1) * (BN / 64); ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tbase, q4 * 32, ab * acc_cols + c * 32), r);
        const int col0 = ncol0 + c * 32;
        if (row >= p.M || col0 >= nlim) continue;
        const bool whole = col0 + 32 <= nlim;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        const size_t o0 = size_t(row) * ldo + col0;
        if (p.out_f32) {
          float* out = static_cast<float*>(out_base) + o0;
          const float* res = p.res ? static_cast<const float*>(p.res) + o0 : nullptr;
          if (whole) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              float4 w = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
              if (res) {
                const float4 u = *reinterpret_cast<const float4*>(res + j);
                w.x += u.x, w.y += u.y, w.z += u.z, w.w += u.w;
              }
              *reinterpret_cast<float4*>(out + j) = w;
            }
          } else {
            for (int j = 0; j < 32 && col0 + j < nlim; ++j) out[j] = v[j] + (res ? res[j] : 0.f);
          }
        } else {
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(out_base) + o0;
          const __nv_bfloat16* res = p.res ? static_cast<const __nv_bfloat16*>(p.res) + o0 : nullptr;
          if (whole) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              float w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) w[i] = v[j + i];
              if (res) {
                const uint4 u = *reinterpret_cast<const uint4*>(res + j);
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) w[2 * i] += bf16_lo_f(uw[i]), w[2 * i + 1] += bf16_hi_f(uw[i]);
              }
              *reinterpret_cast<uint4*>(out + j) =
                  make_uint4(pack_bf16(w[0], w[1]), pack_bf16(w[2], w[3]), pack_bf16(w[4], w[5]), pack_bf16(w[6], w[7]));
            }
          } else {
            for (int j = 0; j < 32 && col0 + j < nlim; ++j)
              out[j] = __float2bfloat16_rn(v[j] + (res ? __bfloat162float(res[j]) : 0.f));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, tcols);
  }
}

// ------------------------------------------------------------------ RMSNorm rows
// Elements of a row handled as 16-byte chunks: 4 fp32 or 8 bf16 values.
template <bool F32IO>
struct RowChunk {
  static constexpr int N = F32IO ? 4 : 8;
  float v[N];
  __device__ __forceinline__ void load(const void* base, size_t elem) {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(base) + elem * (F32IO ? 4 : 2));
    if constexpr (F32IO) {
      v[0] = __uint_as_float(u.x), v[1] = __uint_as_float(u.y), v[2] = __uint_as_float(u.z), v[3] = __uint_as_float(u.w);
    } else {
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) v[2 * k] = bf16_lo_f(w[k]), v[2 * k + 1] = bf16_hi_f(w[k]);
    }
  }
  __device__ __forceinline__ void store(void* base, size_t elem) const {
    uint4 u;
    if constexpr (F32IO) {
      u = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
    } else {
      u = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
    }
    *reinterpret_cast<uint4*>(static_cast<uint8_t*>(base) + elem * (F32IO ? 4 : 2)) = u;
  }
};

// One warp per token row of x [M][C] (C a multiple of 64): rstd = (mean x^2
// + eps)^-1/2, y = x rstd g written as the GEMM operand (bfloat16 storage:
// y in bf16; float32 storage: bf16 hi and lo planes of y).  Lanes take
// 16-byte chunks of the row.
template <bool F32IO>
__global__ void __launch_bounds__(256) rmsnorm_rows_kernel(const void* x, const void* g, __nv_bfloat16* y_hi,
                                                           __nv_bfloat16* y_lo, float* rstd, int M, int C,
                                                           float eps) {
  using RC = RowChunk<F32IO>;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  grid_dep_wait();
  grid_dep_launch();
  if (row >= M) return;
  const size_t r0 = size_t(row) * C;
  float ss = 0.f;
  for (int j = lane * RC::N; j < C; j += 32 * RC::N) {
    RC a;
    a.load(x, r0 + j);
#pragma unroll
    for (int k = 0; k < RC::N; ++k) ss = fmaf(a.v[k], a.v[k], ss);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(kFullMask, ss, off);
  const float rs = 1.f / sqrtf(ss / float(C) + eps);
  if (lane == 0) rstd[row] = rs;
  for (int j = lane * RC::N; j < C; j += 32 * RC::N) {
    RC a, gg;
    a.load(x, r0 + j);
    gg.load(g, j);
    float yv[RC::N];
#pragma unroll
    for (int k = 0; k < RC::N; ++k) yv[k] = a.v[k] * rs * gg.v[k];
    if constexpr (F32IO) {
      uint2 h, l;
      split_bf16(yv[0], yv[1], h.x, l.x);
      split_bf16(yv[2], yv[3], h.y, l.y);
      *reinterpret_cast<uint2*>(y_hi + r0 + j) = h;
      *reinterpret_cast<uint2*>(y_lo + r0 + j) = l;
    } else {
      *reinterpret_cast<uint4*>(y_hi + r0 + j) =
          make_uint4(pack_bf16(yv[0], yv[1]), pack_bf16(yv[2], yv[3]), pack_bf16(yv[4], yv[5]), pack_bf16(yv[6], yv[7]));
    }
  }
}

// fp32 tensors -> bf16 hi and lo planes, up to kSplitJobs tensors in one
// launch (the operands of one call), 16 bytes per thread per step.
constexpr int kSplitJobs = 6;
struct SplitJob {
  const float* src;
  __nv_bfloat16* hi;
  __nv_bfloat16* lo;
  long long start;  // first 4-element chunk of this tensor in the launch's range
};
struct SplitParams {
  SplitJob job[kSplitJobs];
  int n;
  long long total;  // 4-element chunks of all tensors
};

__global__ void __launch_bounds__(256) split_planes_kernel(const __grid_constant__ SplitParams p) {
  grid_dep_wait();
  grid_dep_launch();
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < p.total; i += 256ll * gridDim.x) {
    int j = 0;
    while (j + 1 < p.n && i >= p.job[j + 1].start) ++j;
    const SplitJob& q = p.job[j];
    const long long k = i - q.start;
    const float4 v = reinterpret_cast<const float4*>(q.src)[k];
    uint2 h, l;
    split_bf16(v.x, v.y, h.x, l.x);
    split_bf16(v.z, v.w, h.y, l.y);
    reinterpret_cast<uint2*>(q.hi)[k] = h;
    reinterpret_cast<uint2*>(q.lo)[k] = l;
  }
}

// RMSNorm backward, one warp per token row (rows grid-stride): from
// dy [M][C] (fp32) and the forward's x, g, rstd,
//   dx = rstd g dy - x rstd^3 / C sum_j (g dy)_j x_j  (+ dres),
// and this CTA's share of dg = sum_tokens dy x rstd, written to
// dg_part[blockIdx.x][C] (fp32).  Each warp sums its rows' dg terms in its
// own shared-memory row (every column owned by one lane), the CTA adds the
// eight rows at the end.
template <bool F32IO>
__global__ void __launch_bounds__(256) rmsnorm_bwd_rows_kernel(const void* x, const void* g, const float* rstd,
                                                               const float* dy, const void* dres, void* dx,
                                                               float* dg_part, int M, int C) {
  using RC = RowChunk<F32IO>;
  extern __shared__ float dg_s[];  // [8 warps][C]
  grid_dep_wait();
  grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* mine = dg_s + size_t(warp) * C;
  for (int j = lane; j < C; j += 32) mine[j] = 0.f;
  for (int row = blockIdx.x * 8 + warp; row < M; row += gridDim.x * 8) {
    const size_t r0 = size_t(row) * C;
    const float rs = rstd[row];
    float dot = 0.f;
    for (int j = lane * RC::N; j < C; j += 32 * RC::N) {
      RC a, gg;
      a.load(x, r0 + j);
      gg.load(g, j);
#pragma unroll
      for (int k = 0; k < RC::N; k += 4) {
        const float4 d = *reinterpret_cast<const float4*>(dy + r0 + j + k);
        dot = fmaf(gg.v[k] * d.x, a.v[k], dot);
        dot = fmaf(gg.v[k + 1] * d.y, a.v[k + 1], dot);
        dot = fmaf(gg.v[k + 2] * d.z, a.v[k + 2], dot);
        dot = fmaf(gg.v[k + 3] * d.w, a.v[k + 3], dot);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(kFullMask, dot, off);
    const float c2 = rs * rs * rs * dot / float(C);
    for (int j = lane * RC::N; j < C; j += 32 * RC::N) {
      RC a, gg, out;
      a.load(x, r0 + j);
      gg.load(g, j);
      RC rr;
      if (dres) rr.load(dres, r0 + j);
#pragma unroll
      for (int k = 0; k < RC::N; k += 4) {
        const float4 d = *reinterpret_cast<const float4*>(dy + r0 + j + k);
        const float dd[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          out.v[k + q] = rs * gg.v[k + q] * dd[q] - a.v[k + q] * c2 + (dres ? rr.v[k + q] : 0.f);
          mine[j + k + q] += dd[q] * a.v[k + q] * rs;
        }
      }
      out.store(dx, r0 + j);
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < C; j += 256) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += dg_s[size_t(w) * C + j];
    dg_part[size_t(blockIdx.x) * C + j] = acc;
  }
}

// dg[j] = sum over the parts of dg_part[.][j], in the storage type: a CTA
// per 32 columns, its eight warps summing every eighth part, then the warps'
// sums added in a fixed order.
template <bool F32IO>
__global__ void __launch_bounds__(256) colsum_kernel(const float* part, int n_part, int C, void* dg) {
  __shared__ float red[8][32];
  grid_dep_wait();
  grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (j < C)
    for (int i = warp; i < n_part; i += 8) s += part[size_t(i) * C + j];
  red[warp][lane] = s;
  __syncthreads();
  if (warp != 0 || j >= C) return;
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) t += red[w][lane];
  if (F32IO) static_cast<float*>(dg)[j] = t;
  else static_cast<__nv_bfloat16*>(dg)[j] = __float2bfloat16_rn(t);
}

}  // namespace nea
