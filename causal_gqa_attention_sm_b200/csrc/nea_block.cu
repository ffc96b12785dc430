// C ABI of the decoder-block steps beside the attention (include/nea_attn.h,
// "Decoder-block steps"): the RMSNorm pre-norm with the Q/K/V projections
// and the output projection with the residual add, and the pre-norm SwiGLU
// feed-forward with its residual add, forward and backward.
// Every product runs on nea::gemm_kernel (tcgen05, TMA, TMEM accumulators);
// the host side here chooses operand orientations, makes the operand planes
// and sequences the launches on the caller's stream.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "nea_attn.h"
#include "nea_block.cuh"
#include "nea_internal.h"

namespace {

std::mutex g_block_mu;

// Per-device workspace of the block steps (operand planes, the fp32 input
// gradient of the norm, the dg partial sums), grown when a call needs more.
struct BlockState {
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  uint32_t attr_done = 0;
};
BlockState g_block[64];

int fail(cudaError_t e) {
  (void)cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? NEA_ERR_NOMEM : NEA_ERR_CUDA;
}

size_t rup(size_t n) { return (n + 255) / 256 * 256; }
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// A bf16 row-major matrix [rows][cols] as a GEMM operand tile source.
// k_major: the reduction runs along `cols` (box 64 cols x 128 rows);
// otherwise along `rows` (box 64 cols x 64 rows, two per tile).
int mat_map(CUtensorMap* m, const void* base, long long rows, long long cols, bool k_major) {
  auto enc = encoder();
  if (!enc) return NEA_ERR_CUDA;
  const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
  const cuuint32_t box[2] = {64, k_major ? 128u : 64u};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NEA_OK : NEA_ERR_CUDA;
}

// An operand in the form the GEMM reads: bf16 hi (and, for float32 storage,
// lo) planes of a row-major matrix.
struct Operand {
  const void* hi = nullptr;
  const void* lo = nullptr;
  long long rows = 0, cols = 0;
};

struct Ctx {
  cudaStream_t stream;
  bool f32;
  int* err;
  int n_sm;
  BlockState* st;
  unsigned long long wait_limit;
  float* part = nullptr;  // split-K partial tiles (a piece of the workspace)
  size_t part_bytes = 0;
  nea::SplitParams planes{};  // operand-plane splits not launched yet
};

// Bytes set aside for split-K partial tiles: up to 4 chunks of every tile of
// a product with fewer tiles than SMs.
size_t part_reserve(int n_sm) { return size_t(n_sm) * 128 * 128 * 4 * 4; }

int setup(Ctx& c, int dtype, void* stream) {
  c.stream = static_cast<cudaStream_t>(stream);
  c.f32 = dtype == NEA_F32;
  int rc = nea_internal::device_status_word(&c.err, &c.n_sm);
  if (rc) return rc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(e);
  if (dev < 0 || dev >= 64) return NEA_ERR_UNSUPPORTED;
  c.st = &g_block[dev];
  c.wait_limit = static_cast<unsigned long long>(nea_internal::wait_limit_ns());
  return NEA_OK;
}

int ensure(Ctx& c, size_t bytes) {
  if (bytes <= c.st->ws_bytes) return NEA_OK;
  cudaError_t e = cudaDeviceSynchronize();  // in-flight kernels may still use the old buffer
  if (e != cudaSuccess) return fail(e);
  if (c.st->ws) cudaFree(c.st->ws);
  c.st->ws = nullptr;
  c.st->ws_bytes = 0;
  if ((e = cudaMalloc(&c.st->ws, bytes)) != cudaSuccess) return fail(e);
  c.st->ws_bytes = bytes;
  return NEA_OK;
}

// Bump allocator over the workspace (256-byte aligned pieces).
struct Carve {
  uint8_t* base;
  size_t off = 0;
  void* take(size_t bytes) {
    void* p = base + off;
    off += rup(bytes);
    return p;
  }
};

template <typename K, typename... A>
cudaError_t launch_pdl(K kern, unsigned grid, unsigned block, size_t smem, cudaStream_t stream, A... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Launches the pending operand-plane splits, if any, as one kernel.
int flush_planes(Ctx& c) {
  nea::SplitParams& sp = c.planes;
  if (sp.n == 0) return NEA_OK;
  const unsigned grid = unsigned(std::min<long long>((sp.total + 255) / 256, (long long)c.n_sm * 8));
  const cudaError_t e = launch_pdl(nea::split_planes_kernel, grid, 256u, size_t(0), c.stream, sp);
  sp = nea::SplitParams{};
  return e == cudaSuccess ? NEA_OK : fail(e);
}

// fp32 [rows][cols] -> hi/lo planes (float32 storage), queued: every product
// launch first flushes the queue, so one kernel splits all the operands a
// call needs.  bfloat16 storage reads the tensor itself.
int make_operand(Ctx& c, Carve& w, const void* src, long long rows, long long cols, Operand* op) {
  op->rows = rows;
  op->cols = cols;
  if (!c.f32) {
    op->hi = src;
    return NEA_OK;
  }
  const size_t n = size_t(rows) * cols;
  auto* hi = static_cast<__nv_bfloat16*>(w.take(n * 2));
  auto* lo = static_cast<__nv_bfloat16*>(w.take(n * 2));
  if (c.planes.n == nea::kSplitJobs) {
    const int rc = flush_planes(c);
    if (rc) return rc;
  }
  nea::SplitParams& sp = c.planes;
  sp.job[sp.n] = nea::SplitJob{static_cast<const float*>(src), hi, lo, sp.total};
  sp.n += 1;
  sp.total += static_cast<long long>(n / 4);
  op->hi = hi;
  op->lo = lo;
  return NEA_OK;
}

// Launches the kernel instance of an operand orientation (form = 2 a_mn +
// b_mn) for a plane count and tile width; `bit` indexes the instances whose
// shared-memory limit is already raised.
template <bool SPLIT, int BN, typename Run>
int launch_form(Run& run, int form) {
  constexpr uint32_t sm = nea::GemmSmem<SPLIT, BN>::kAlloc;
  constexpr int base = (SPLIT ? 0 : 4) + (BN == 256 ? 8 : 0);
  switch (form) {
    case 0: return run(nea::gemm_kernel<false, false, SPLIT, BN>, sm, base + 0);
    case 1: return run(nea::gemm_kernel<false, true, SPLIT, BN>, sm, base + 1);
    case 2: return run(nea::gemm_kernel<true, false, SPLIT, BN>, sm, base + 2);
    default: return run(nea::gemm_kernel<true, true, SPLIT, BN>, sm, base + 3);
  }
}

// One operand segment of a product: A and B operands (read K-major or
// MN-major as the product's flags say), and for N segments the output.
struct Seg {
  Operand A, B;
  void* out = nullptr;
  long long width = 0;  // K extent (K segments) or N extent = output columns (N segments)
};

// out = sum_s A_s B_s (kseg: segments along K, one output `out` [M][ldo]) or
// out_s = A_0 B_s (segments along N, output s [M][width_s]); A [M x K] is
// stored [M][K] (K-major) or [K][M] (MN-major), B [K x N] stored [N][K]
// (K-major) or [K][N] (MN-major).  `mode`, `pl` and `ab` select a SwiGLU
// epilogue (nea::GemmParams::mode); those products run unsplit.
int gemm_seg(Ctx& c, const Seg* segs, int n_seg, bool kseg, bool a_mn, bool b_mn, int M, void* out, long long ldo,
             bool out_f32, const void* res, int mode = 0, void* const* pl = nullptr, const void* const* ab = nullptr) {
  nea::GemmParams p{};
  int rc = flush_planes(c);  // the operands' planes first
  if (rc) return rc;
  const bool pair = mode == 1;  // segments 0 and 1 are the two halves of one 256-wide B tile
  for (int i = 0; i < n_seg; ++i) {
    const Seg& g = segs[i];
    nea::GemmSeg& q = p.seg[i];
    if ((rc = mat_map(&q.a_hi, g.A.hi, g.A.rows, g.A.cols, !a_mn)) ||
        (rc = mat_map(&q.b_hi, g.B.hi, g.B.rows, g.B.cols, !b_mn)))
      return rc;
    if (c.f32 && ((rc = mat_map(&q.a_lo, g.A.lo, g.A.rows, g.A.cols, !a_mn)) ||
                  (rc = mat_map(&q.b_lo, g.B.lo, g.B.rows, g.B.cols, !b_mn))))
      return rc;
    q.out = g.out;
    q.ldo = g.width;
  }
  // the N tiles of a tile width: N segments each start on a tile of their own
  auto n_tiles_n = [&](int bn) {
    if (kseg || pair) return int((ldo + bn - 1) / bn);
    int n = 0;
    for (int i = 0; i < n_seg; ++i) n += int((segs[i].width + bn - 1) / bn);
    return n;
  };
  const int n_m = (M + nea::kGemmBM - 1) / nea::kGemmBM;
  int n_k_all = 0;  // k-steps of the whole product
  for (int i = 0; i < n_seg; ++i)
    n_k_all += (kseg || (pair && i == 0)) ? int((segs[i].width + nea::kGemmBK - 1) / nea::kGemmBK) : 0;
  if (!kseg && !pair) n_k_all = int(((a_mn ? segs[0].A.rows : segs[0].A.cols) + nea::kGemmBK - 1) / nea::kGemmBK);
  // Tile width and split-K chunk count from a cost model in k-steps of a
  // 128-wide tile: waves of units x (k-steps per unit + 4 for a unit's ramp
  // and epilogue), a 256-wide unit counted as 1.4 such units with bf16
  // operands (they stream from L2, and the wider tile reads A once for twice
  // the columns) and 1.8 with hi/lo planes (whose 96 KB stages leave room
  // for two in flight, against three), plus 4 for the partial-tile reduce;
  // factors measured on the block's products.  A split writes fp32 partial
  // tiles (at most 4 chunks of two k-steps or more, within the reserve);
  // with hi/lo planes it pays on the feed-forward's down and dy products
  // (96 tiles of 256 columns, 48 and 96 k-steps: a 3-way split took the
  // forward from 250 to 238 us and the backward from 509 to 485 us).
  // The SwiGLU epilogues run unsplit; the forward pairs Wg and Wu in one
  // 256-wide tile.
  int bn = pair ? 256 : 128, split = 1;
  if (!pair && n_k_all > 0) {
    double best = 1e300;
    for (int w = 128; w <= 256; w += 128) {
      const long long tiles = static_cast<long long>(n_m) * n_tiles_n(w);
      for (int sp = 1; sp <= (mode == 0 && c.part ? 4 : 1); ++sp) {
        // bf16 products are fast enough that the partial tiles' traffic only
        // pays for 128-wide tiles that alone leave SMs idle (a 3-way split of
        // the feed-forward's down product, 96 tiles of 256 columns, took its
        // forward from 103 to 124 us)
        if (sp > 1 && (n_k_all < 2 * sp || size_t(tiles) * sp * 128 * w * 4 > c.part_bytes ||
                       (!c.f32 && (w == 256 || tiles >= c.n_sm))))
          break;
        const int k_per = (n_k_all + sp - 1) / sp;
        const long long waves = (tiles * sp + c.n_sm - 1) / c.n_sm;
        const double cost = double(waves) * (k_per + 4) * (w == 256 ? (c.f32 ? 1.8 : 1.4) : 1.0) + (sp > 1 ? 4 : 0);
        if (cost < best - 1e-9) best = cost, bn = w, split = sp;
      }
    }
  }
  int N = 0, K = 0, begin = 0;
  for (int i = 0; i < n_seg; ++i) {
    const Seg& g = segs[i];
    p.seg[i].begin = begin;
    if (pair) {
      K = int(g.width);
    } else if (kseg) {
      begin += int(g.width / nea::kGemmBK);
      K += int(g.width);
    } else {
      begin += int((g.width + bn - 1) / bn);
      N += int(g.width);
    }
  }
  if (kseg || pair) N = int(ldo);
  else K = int(a_mn ? segs[0].A.rows : segs[0].A.cols);
  p.n_seg = n_seg;
  p.kseg = kseg;
  p.out = out;
  p.res = res;
  p.ldo = ldo;
  p.M = M;
  p.N = N;
  p.K = K;
  p.out_f32 = out_f32;
  p.n_m = n_m;
  p.n_n = pair ? (N + 127) / 128 : (kseg ? (N + bn - 1) / bn : begin);
  p.n_k = (K + nea::kGemmBK - 1) / nea::kGemmBK;
  p.n_tiles = p.n_m * p.n_n;
  p.mode = mode;
  for (int i = 0; i < 6 && pl; ++i) p.pl[i] = pl[i];
  for (int i = 0; i < 2 && ab; ++i) p.ab[i] = ab[i];
  p.err = c.err;
  p.wait_limit = c.wait_limit;
  if (p.n_tiles == 0 || K == 0) return NEA_OK;
  p.split = split;
  p.bn = bn;
  p.k_per = (p.n_k + p.split - 1) / p.split;
  p.split = (p.n_k + p.k_per - 1) / p.k_per;
  p.part = p.split > 1 ? c.part : nullptr;
  const unsigned grid = unsigned(std::min(p.n_tiles * p.split, c.n_sm));
  auto run = [&](auto kern, uint32_t smem, int bit) -> int {
    if (!(c.st->attr_done & (1u << bit))) {
      const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      if (e != cudaSuccess) return fail(e);
      c.st->attr_done |= 1u << bit;
    }
    cudaError_t e = launch_pdl(kern, grid, unsigned(nea::kGemmThreads), size_t(smem), c.stream, p);
    if (e == cudaSuccess && p.split > 1)
      e = launch_pdl(nea::gemm_reduce_kernel, unsigned(p.n_tiles * (bn / 8)), 256u, size_t(0), c.stream, p);
    return e == cudaSuccess ? NEA_OK : fail(e);
  };
  const int form = (a_mn ? 2 : 0) + (b_mn ? 1 : 0);
  return c.f32 ? (bn == 256 ? launch_form<true, 256>(run, form) : launch_form<true, 128>(run, form))
               : (bn == 256 ? launch_form<false, 256>(run, form) : launch_form<false, 128>(run, form));
}

// out[M][N] = A B (+ res), one segment.
int gemm(Ctx& c, const Operand& A, bool a_mn, const Operand& B, bool b_mn, int M, int N, void* out, bool out_f32,
         const void* res) {
  Seg g;
  g.A = A;
  g.B = B;
  g.out = out;
  g.width = N;
  return gemm_seg(c, &g, 1, false, a_mn, b_mn, M, out, N, out_f32, res);
}

// y = x rstd g as an operand (planes), rstd into `rstd`.
int norm_rows(Ctx& c, Carve& w, const void* x, const void* g, int M, int C, float eps, Operand* y, float* rstd) {
  const size_t n = size_t(M) * C;
  auto* hi = static_cast<__nv_bfloat16*>(w.take(n * 2));
  auto* lo = c.f32 ? static_cast<__nv_bfloat16*>(w.take(n * 2)) : nullptr;
  const unsigned grid = unsigned((M + 7) / 8);
  const cudaError_t e = c.f32 ? launch_pdl(nea::rmsnorm_rows_kernel<true>, grid, 256u, size_t(0), c.stream, x, g, hi,
                                           lo, rstd, M, C, eps)
                              : launch_pdl(nea::rmsnorm_rows_kernel<false>, grid, 256u, size_t(0), c.stream, x, g, hi,
                                           lo, rstd, M, C, eps);
  if (e != cudaSuccess) return fail(e);
  y->hi = hi;
  y->lo = lo;
  y->rows = M;
  y->cols = C;
  return NEA_OK;
}

// Widths (C, Hkv D, hence Hq D) in whole 64-column operand boxes.
int check_dims(int M, int C, int Hq, int Hkv, int D, int dtype) {
  if (M < 0 || C < 64 || C > 4096 || C % 64 != 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return NEA_ERR_ARG;
  if (D < 8 || (Hkv * D) % 64 != 0 || (dtype != NEA_F32 && dtype != NEA_BF16)) return NEA_ERR_ARG;
  if (static_cast<long long>(M) * std::max(C, Hq * D) > (1LL << 31)) return NEA_ERR_ARG;
  return NEA_OK;
}

constexpr float kNormEps = 1e-5f;

// The feed-forward's widths: C and F in whole 64-column operand boxes.
int check_ffn(int M, int C, int F, int dtype) {
  if (M < 0 || C < 64 || C > 4096 || C % 64 != 0 || F < 64 || F % 64 != 0) return NEA_ERR_ARG;
  if (dtype != NEA_F32 && dtype != NEA_BF16) return NEA_ERR_ARG;
  if (static_cast<long long>(M) * std::max(C, F) > (1LL << 31) || static_cast<long long>(C) * F > (1LL << 31))
    return NEA_ERR_ARG;
  return NEA_OK;
}

// dx (with dres) and dg of the RMSNorm from dy: the rows kernel writes dx
// and per-CTA dg sums, the column kernel adds those.
int norm_bwd(Ctx& c, const void* x, const void* g, const float* rstd, const float* dy, const void* dres, void* dx,
             void* dg, float* dg_part, int n_part, int M, int C) {
  const size_t nb_smem = size_t(C) * 4 * 8;  // the eight warps' dg rows
  if (nb_smem > 48 * 1024) {
    const cudaError_t ea =
        c.f32 ? cudaFuncSetAttribute(nea::rmsnorm_bwd_rows_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(nb_smem))
              : cudaFuncSetAttribute(nea::rmsnorm_bwd_rows_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(nb_smem));
    if (ea != cudaSuccess) return fail(ea);
  }
  cudaError_t err = c.f32 ? launch_pdl(nea::rmsnorm_bwd_rows_kernel<true>, unsigned(n_part), 256u, nb_smem,
                                       c.stream, x, g, rstd, dy, dres, dx, dg_part, M, C)
                          : launch_pdl(nea::rmsnorm_bwd_rows_kernel<false>, unsigned(n_part), 256u, nb_smem,
                                       c.stream, x, g, rstd, dy, dres, dx, dg_part, M, C);
  if (err != cudaSuccess) return fail(err);
  const unsigned cg = unsigned((C + 31) / 32);
  err = c.f32 ? launch_pdl(nea::colsum_kernel<true>, cg, 256u, size_t(0), c.stream,
                           static_cast<const float*>(dg_part), n_part, C, dg)
              : launch_pdl(nea::colsum_kernel<false>, cg, 256u, size_t(0), c.stream,
                           static_cast<const float*>(dg_part), n_part, C, dg);
  return err == cudaSuccess ? NEA_OK : fail(err);
}

// bf16 planes of an [rows][cols] intermediate: hi, and lo for float32 storage.
Operand planes(Ctx& c, Carve& w, long long rows, long long cols) {
  Operand o;
  o.rows = rows;
  o.cols = cols;
  o.hi = w.take(size_t(rows) * cols * 2);
  o.lo = c.f32 ? w.take(size_t(rows) * cols * 2) : nullptr;
  return o;
}

}  // namespace

extern "C" {

int nea_block_qkv_fwd(const void* x, const void* g, const void* Wq, const void* Wk, const void* Wv, void* q, void* k,
                      void* v, int M, int C, int Hq, int Hkv, int D, int dtype, void* stream) {
  int rc = check_dims(M, C, Hq, Hkv, D, dtype);
  if (rc) return rc;
  if (M == 0) return NEA_OK;
  for (const void* ptr : {x, g, Wq, Wk, Wv, static_cast<const void*>(q), static_cast<const void*>(k),
                          static_cast<const void*>(v)})
    if (!ptr || !al16(ptr)) return NEA_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_block_mu);
  Ctx c;
  if ((rc = setup(c, dtype, stream))) return rc;
  const int Nq = Hq * D, Nk = Hkv * D;
  const int e = c.f32 ? 4 : 2;
  const size_t need = part_reserve(c.n_sm) + rup(size_t(M) * 4) + rup(size_t(M) * C * e) +
                      (c.f32 ? rup(size_t(C) * Nq * 4) + 2 * rup(size_t(C) * Nk * 4) : 0) + 4096;
  if ((rc = ensure(c, need))) return rc;
  Carve w{c.st->ws};
  c.part_bytes = part_reserve(c.n_sm);
  c.part = static_cast<float*>(w.take(c.part_bytes));
  auto* rstd = static_cast<float*>(w.take(size_t(M) * 4));
  Operand y, bq, bk, bv;
  if ((rc = norm_rows(c, w, x, g, M, C, kNormEps, &y, rstd))) return rc;
  if ((rc = make_operand(c, w, Wq, C, Nq, &bq)) || (rc = make_operand(c, w, Wk, C, Nk, &bk)) ||
      (rc = make_operand(c, w, Wv, C, Nk, &bv)))
    return rc;
  // q = y Wq: A = y [M][C] K-major; B = Wq [C][Nq], N contiguous: MN-major
  if (Nq % nea::kGemmBN == 0 && Nk % nea::kGemmBN == 0) {  // one launch, q | k | v side by side along N
    Seg g[3];
    g[0].A = y, g[0].B = bq, g[0].out = q, g[0].width = Nq;
    g[1].A = y, g[1].B = bk, g[1].out = k, g[1].width = Nk;
    g[2].A = y, g[2].B = bv, g[2].out = v, g[2].width = Nk;
    return gemm_seg(c, g, 3, false, false, true, M, nullptr, 0, c.f32, nullptr);
  }
  if ((rc = gemm(c, y, false, bq, true, M, Nq, q, c.f32, nullptr)) ||
      (rc = gemm(c, y, false, bk, true, M, Nk, k, c.f32, nullptr)) ||
      (rc = gemm(c, y, false, bv, true, M, Nk, v, c.f32, nullptr)))
    return rc;
  return NEA_OK;
}

int nea_block_qkv_bwd(const void* x, const void* g, const void* Wq, const void* Wk, const void* Wv, const void* dq,
                      const void* dk, const void* dv, const void* dres, void* dx, void* dg, void* dWq, void* dWk,
                      void* dWv, int M, int C, int Hq, int Hkv, int D, int dtype, void* stream) {
  int rc = check_dims(M, C, Hq, Hkv, D, dtype);
  if (rc) return rc;
  if (M == 0) return NEA_OK;
  for (const void* ptr : {x, g, Wq, Wk, Wv, dq, dk, dv, static_cast<const void*>(dx), static_cast<const void*>(dg),
                          static_cast<const void*>(dWq), static_cast<const void*>(dWk), static_cast<const void*>(dWv)})
    if (!ptr || !al16(ptr)) return NEA_ERR_ARG;
  if (dres && !al16(dres)) return NEA_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_block_mu);
  Ctx c;
  if ((rc = setup(c, dtype, stream))) return rc;
  const int Nq = Hq * D, Nk = Hkv * D;
  const int e = c.f32 ? 4 : 2;
  const int n_part = std::min((M + 7) / 8, c.n_sm * 4);
  const size_t need = part_reserve(c.n_sm) + rup(size_t(M) * 4) + rup(size_t(M) * C * e) + rup(size_t(M) * C * 4) +
                      rup(size_t(n_part) * C * 4) +
                      (c.f32 ? rup(size_t(C) * Nq * 4) + 2 * rup(size_t(C) * Nk * 4) + rup(size_t(M) * Nq * 4) +
                                   2 * rup(size_t(M) * Nk * 4)
                             : 0) +
                      4096;
  if ((rc = ensure(c, need))) return rc;
  Carve w{c.st->ws};
  c.part_bytes = part_reserve(c.n_sm);
  c.part = static_cast<float*>(w.take(c.part_bytes));
  auto* rstd = static_cast<float*>(w.take(size_t(M) * 4));
  auto* dy = static_cast<float*>(w.take(size_t(M) * C * 4));
  auto* dg_part = static_cast<float*>(w.take(size_t(n_part) * C * 4));
  Operand y, bq, bk, bv, gq, gk, gv;
  if ((rc = norm_rows(c, w, x, g, M, C, kNormEps, &y, rstd))) return rc;
  if ((rc = make_operand(c, w, Wq, C, Nq, &bq)) || (rc = make_operand(c, w, Wk, C, Nk, &bk)) ||
      (rc = make_operand(c, w, Wv, C, Nk, &bv)) || (rc = make_operand(c, w, dq, M, Nq, &gq)) ||
      (rc = make_operand(c, w, dk, M, Nk, &gk)) || (rc = make_operand(c, w, dv, M, Nk, &gv)))
    return rc;
  // dW* = y^T d*: A = y^T (y [M][C], C contiguous: MN-major); B = d* [M][N*], MN-major
  if (Nq % nea::kGemmBN == 0 && Nk % nea::kGemmBN == 0) {  // one launch, side by side along N
    Seg g[3];
    g[0].A = y, g[0].B = gq, g[0].out = dWq, g[0].width = Nq;
    g[1].A = y, g[1].B = gk, g[1].out = dWk, g[1].width = Nk;
    g[2].A = y, g[2].B = gv, g[2].out = dWv, g[2].width = Nk;
    if ((rc = gemm_seg(c, g, 3, false, true, true, C, nullptr, 0, c.f32, nullptr))) return rc;
  } else if ((rc = gemm(c, y, true, gq, true, C, Nq, dWq, c.f32, nullptr)) ||
             (rc = gemm(c, y, true, gk, true, C, Nk, dWk, c.f32, nullptr)) ||
             (rc = gemm(c, y, true, gv, true, C, Nk, dWv, c.f32, nullptr))) {
    return rc;
  }
  // dy = dq Wq^T + dk Wk^T + dv Wv^T (fp32), one product chained along K:
  // A = d* K-major; B = W*^T, i.e. W* [C][N*] read K-major
  {
    Seg g[3];
    g[0].A = gq, g[0].B = bq, g[0].width = Nq;
    g[1].A = gk, g[1].B = bk, g[1].width = Nk;
    g[2].A = gv, g[2].B = bv, g[2].width = Nk;
    if ((rc = gemm_seg(c, g, 3, true, false, false, M, dy, C, true, nullptr))) return rc;
  }
  return norm_bwd(c, x, g, rstd, dy, dres, dx, dg, dg_part, n_part, M, C);
}

int nea_block_out_fwd(const void* x, const void* o, const void* Wo, void* h, int M, int C, int Hq, int D, int dtype,
                      void* stream) {
  int rc = check_dims(M, C, Hq, Hq, D, dtype);
  if (rc) return rc;
  if (M == 0) return NEA_OK;
  for (const void* ptr : {x, o, Wo, static_cast<const void*>(h)})
    if (!ptr || !al16(ptr)) return NEA_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_block_mu);
  Ctx c;
  if ((rc = setup(c, dtype, stream))) return rc;
  const int Nq = Hq * D;
  const size_t need = part_reserve(c.n_sm) + (c.f32 ? rup(size_t(M) * Nq * 4) + rup(size_t(Nq) * C * 4) : 0) + 4096;
  if ((rc = ensure(c, need))) return rc;
  Carve w{c.st->ws};
  c.part_bytes = part_reserve(c.n_sm);
  c.part = static_cast<float*>(w.take(c.part_bytes));
  Operand a, b;
  if ((rc = make_operand(c, w, o, M, Nq, &a)) || (rc = make_operand(c, w, Wo, Nq, C, &b))) return rc;
  // h = x + o Wo: A = o [M][Nq] K-major; B = Wo [Nq][C], C contiguous: MN-major
  return gemm(c, a, false, b, true, M, C, h, c.f32, x);
}

int nea_block_out_bwd(const void* o, const void* Wo, const void* dh, void* do_, void* dWo, int M, int C, int Hq,
                      int D, int dtype, void* stream) {
  int rc = check_dims(M, C, Hq, Hq, D, dtype);
  if (rc) return rc;
  if (M == 0) return NEA_OK;
  for (const void* ptr : {o, Wo, dh, static_cast<const void*>(do_), static_cast<const void*>(dWo)})
    if (!ptr || !al16(ptr)) return NEA_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_block_mu);
  Ctx c;
  if ((rc = setup(c, dtype, stream))) return rc;
  const int Nq = Hq * D;
  const size_t need = part_reserve(c.n_sm) +
      (c.f32 ? rup(size_t(M) * Nq * 4) + rup(size_t(Nq) * C * 4) + rup(size_t(M) * C * 4) : 0) + 4096;
  if ((rc = ensure(c, need))) return rc;
  Carve w{c.st->ws};
  c.part_bytes = part_reserve(c.n_sm);
  c.part = static_cast<float*>(w.take(c.part_bytes));
  Operand a, b, d;
  if ((rc = make_operand(c, w, o, M, Nq, &a)) || (rc = make_operand(c, w, Wo, Nq, C, &b)) ||
      (rc = make_operand(c, w, dh, M, C, &d)))
    return rc;
  // do = dh Wo^T: A = dh [M][C] K-major; B = Wo^T, i.e. Wo [Nq][C] read K-major
  if ((rc = gemm(c, d, false, b, false, M, Nq, do_, c.f32, nullptr))) return rc;
  // dWo = o^T dh: A = o^T (o [M][Nq]: MN-major); B = dh [M][C], MN-major
  return gemm(c, a, true, d, true, Nq, C, dWo, c.f32, nullptr);
}

int nea_block_ffn_fwd(const void* x, const void* g, const void* Wg, const void* Wu, const void* Wd, void* h, void* a,
                      void* b, int M, int C, int F, int dtype, void* stream) {
  int rc = check_ffn(M, C, F, dtype);
  if (rc) return rc;
  if (M == 0) return NEA_OK;
  for (const void* ptr : {x, g, Wg, Wu, Wd, static_cast<const void*>(h)})
    if (!ptr || !al16(ptr)) return NEA_ERR_ARG;
  if ((a && !al16(a)) || (b && !al16(b))) return NEA_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_block_mu);
  Ctx c;
  if ((rc = setup(c, dtype, stream))) return rc;
  const int e = c.f32 ? 4 : 2;  // bytes of an operand element's planes
  const size_t need = part_reserve(c.n_sm) + rup(size_t(M) * 4) + rup(size_t(M) * C * e) + rup(size_t(M) * F * e) +
                      (c.f32 ? 3 * rup(size_t(C) * F * 4) : 0) + 4096;
  if ((rc = ensure(c, need))) return rc;
  Carve w{c.st->ws};
  c.part_bytes = part_reserve(c.n_sm);
  c.part = static_cast<float*>(w.take(c.part_bytes));
  auto* rstd = static_cast<float*>(w.take(size_t(M) * 4));
  Operand y, bg, bu, bd;
  if ((rc = norm_rows(c, w, x, g, M, C, kNormEps, &y, rstd))) return rc;
  if ((rc = make_operand(c, w, Wg, C, F, &bg)) || (rc = make_operand(c, w, Wu, C, F, &bu)) ||
      (rc = make_operand(c, w, Wd, F, C, &bd)))
    return rc;
  const Operand act = planes(c, w, M, F);
  // a = y Wg and b = y Wu side by side in one accumulator (the halves of a
  // 256-wide B tile), the epilogue writing a, b and act = silu(a) b: A = y
  // K-major; B = Wg, Wu [C][F], F contiguous: MN-major
  {
    Seg s[2];
    s[0].A = y, s[0].B = bg, s[0].out = a, s[0].width = C;
    s[1].A = y, s[1].B = bu, s[1].out = b, s[1].width = C;
    void* const pl[6] = {const_cast<void*>(act.hi), const_cast<void*>(act.lo), nullptr, nullptr, nullptr, nullptr};
    if ((rc = gemm_seg(c, s, 2, false, false, true, M, nullptr, F, c.f32, nullptr, 1, pl))) return rc;
  }
  // h = x + act Wd: A = act [M][F] K-major; B = Wd [F][C], C contiguous: MN-major
  return gemm(c, act, false, bd, true, M, C, h, c.f32, x);
}

int nea_block_ffn_bwd(const void* x, const void* g, const void* Wg, const void* Wu, const void* Wd, const void* a,
                      const void* b, const void* dh, void* dx, void* dg, void* dWg, void* dWu, void* dWd, int M, int C,
                      int F, int dtype, void* stream) {
  int rc = check_ffn(M, C, F, dtype);
  if (rc) return rc;
  if (M == 0) return NEA_OK;
  for (const void* ptr : {x, g, Wg, Wu, Wd, a, b, dh, static_cast<const void*>(dx), static_cast<const void*>(dg),
                          static_cast<const void*>(dWg), static_cast<const void*>(dWu), static_cast<const void*>(dWd)})
    if (!ptr || !al16(ptr)) return NEA_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_block_mu);
  Ctx c;
  if ((rc = setup(c, dtype, stream))) return rc;
  const int e = c.f32 ? 4 : 2;
  const int n_part = std::min((M + 7) / 8, c.n_sm * 4);
  const size_t need = part_reserve(c.n_sm) + rup(size_t(M) * 4) + rup(size_t(M) * C * e) + rup(size_t(M) * C * 4) +
                      rup(size_t(n_part) * C * 4) + 3 * rup(size_t(M) * F * e) +
                      (c.f32 ? 3 * rup(size_t(C) * F * 4) + rup(size_t(M) * C * 4) : 0) + 4096;
  if ((rc = ensure(c, need))) return rc;
  Carve w{c.st->ws};
  c.part_bytes = part_reserve(c.n_sm);
  c.part = static_cast<float*>(w.take(c.part_bytes));
  auto* rstd = static_cast<float*>(w.take(size_t(M) * 4));
  auto* dy = static_cast<float*>(w.take(size_t(M) * C * 4));
  auto* dg_part = static_cast<float*>(w.take(size_t(n_part) * C * 4));
  Operand y, bg, bu, bd, gh;
  if ((rc = norm_rows(c, w, x, g, M, C, kNormEps, &y, rstd))) return rc;
  if ((rc = make_operand(c, w, Wg, C, F, &bg)) || (rc = make_operand(c, w, Wu, C, F, &bu)) ||
      (rc = make_operand(c, w, Wd, F, C, &bd)) || (rc = make_operand(c, w, dh, M, C, &gh)))
    return rc;
  const Operand da = planes(c, w, M, F), db = planes(c, w, M, F), act = planes(c, w, M, F);
  // dact = dh Wd^T, combined in the epilogue with a and b into da, db and
  // act: A = dh [M][C] K-major; B = Wd^T, i.e. Wd [F][C] read K-major
  {
    Seg s;
    s.A = gh, s.B = bd, s.width = F;
    void* const pl[6] = {const_cast<void*>(da.hi), const_cast<void*>(da.lo), const_cast<void*>(db.hi),
                         const_cast<void*>(db.lo), const_cast<void*>(act.hi), const_cast<void*>(act.lo)};
    const void* const ab[2] = {a, b};
    if ((rc = gemm_seg(c, &s, 1, false, false, false, M, nullptr, F, c.f32, nullptr, 2, pl, ab))) return rc;
  }
  // dWd = act^T dh: A = act^T (act [M][F]: MN-major); B = dh [M][C], MN-major
  if ((rc = gemm(c, act, true, gh, true, F, C, dWd, c.f32, nullptr))) return rc;
  // dWg = y^T da, dWu = y^T db: A = y^T (MN-major); B = da, db [M][F], MN-major
  if (F % nea::kGemmBN == 0) {  // one launch, side by side along N
    Seg s[2];
    s[0].A = y, s[0].B = da, s[0].out = dWg, s[0].width = F;
    s[1].A = y, s[1].B = db, s[1].out = dWu, s[1].width = F;
    if ((rc = gemm_seg(c, s, 2, false, true, true, C, nullptr, 0, c.f32, nullptr))) return rc;
  } else if ((rc = gemm(c, y, true, da, true, C, F, dWg, c.f32, nullptr)) ||
             (rc = gemm(c, y, true, db, true, C, F, dWu, c.f32, nullptr))) {
    return rc;
  }
  // dy = da Wg^T + db Wu^T (fp32), chained along K: A = da, db K-major;
  // B = Wg^T, Wu^T, i.e. Wg, Wu [C][F] read K-major
  {
    Seg s[2];
    s[0].A = da, s[0].B = bg, s[0].width = F;
    s[1].A = db, s[1].B = bu, s[1].width = F;
    if ((rc = gemm_seg(c, s, 2, true, false, false, M, dy, C, true, nullptr))) return rc;
  }
  return norm_bwd(c, x, g, rstd, dy, dh, dx, dg, dg_part, n_part, M, C);
}

}  // extern "C"
