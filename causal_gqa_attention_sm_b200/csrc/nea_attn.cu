// C ABI of the attention library: argument checks, the per-device workspace
// (rotary table, backward row terms, fp32 operand planes, device error word),
// TMA descriptors and kernel launches.  Declarations and contracts:
// include/nea_attn.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>
#include <utility>
#include <vector>

#include "nea_attn.h"
#include "nea_internal.h"
#include "nea_bwd.cuh"
#include "nea_bwd_f32.cuh"
#include "nea_decode.cuh"
#include "nea_fwd.cuh"
#include "nea_prep.cuh"

namespace {

constexpr int kVersion = 300;  // 0.3.0

thread_local long long t_wait_limit_ns = 2000000000LL;
thread_local int t_debug_flags = 0;
thread_local void* const* t_prof_events = nullptr;
thread_local int t_prof_n = 0;

#ifdef NEA_TRACE
// Performance-analysis builds only: destination of the forward kernel's phase
// stamps (80 per CTA), set through nea_debug_set_trace.
thread_local unsigned long long* t_trace = nullptr;
thread_local unsigned long long* t_trace_bwd = nullptr;
#endif

void prof_record(int i, cudaStream_t stream) {
  if (t_prof_events && i < t_prof_n && t_prof_events[i])
    cudaEventRecord(static_cast<cudaEvent_t>(t_prof_events[i]), stream);
}

struct DeviceState {
  bool probed = false;
  bool sm100 = false;
  int* err = nullptr;          // device error word
  uint8_t* ws = nullptr;       // row terms and fp32 operand planes of the current call
  size_t ws_bytes = 0;
  // rotary tables keyed by (T, D, base bits); never freed while the process
  // runs, so in-flight kernels on any stream keep valid pointers
  std::map<std::tuple<int, int, uint32_t>, float2*> rope;
  uint32_t attr_done = 0;      // bitmask of kernels whose smem attribute is set
  uint64_t attr_dec = 0;       // the same for the decode kernels
  int n_sm = 148;              // streaming multiprocessors
};

std::mutex g_mu;
std::map<int, DeviceState> g_dev;

int cuda_fail(cudaError_t e) {
  (void)cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? NEA_ERR_NOMEM : NEA_ERR_CUDA;
}

size_t round_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

// ----------------------------------------------------------------- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    (void)cudaGetLastError();
  });
  return fn;
}

// Descriptor of a [B][T][H][D] tensor read as 128-row tiles of one head:
// dimensions (innermost first) {D, H, T, B}, box {min(D, 64), 1, 128, 1};
// rows past T read as zero.  bf16 tiles land in the operand swizzle (row =
// atom); D = 128 takes two boxes per tile, one per 64-column block.
int make_tile_map(CUtensorMap* m, const void* base, int B, int T, int H, int D) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return NEA_ERR_CUDA;
  const cuuint64_t e = 2;
  const cuuint32_t bx = D < 64 ? cuuint32_t(D) : 64u;
  const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(T), cuuint64_t(B)};
  const cuuint64_t strides[3] = {D * e, cuuint64_t(H) * D * e, cuuint64_t(T) * H * D * e};
  const cuuint32_t box[4] = {bx, 1, cuuint32_t(nea::kTileRows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapSwizzle sw = bx == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NEA_OK : NEA_ERR_CUDA;
}

// Descriptor of a decode cache [B][Tc][Hkv][D] (fp32 or bf16), described
// with its dimensions in the order (D, position, kv head, sequence), box
// {min(D, 128 bytes), rows, heads, 1}: `rows` consecutive positions of
// `heads` neighbouring kv heads, landing in shared memory head-major (fp32
// with D = 64 takes two boxes per piece, one per column half), each
// (head, position) line 128 bytes with the 128-byte swizzle or 64 bytes with
// the 64-byte swizzle; positions past Tc read as zero.
int make_cache_map(CUtensorMap* m, const void* base, int B, int Tc, int Hkv, int D, bool f32, int heads, int rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return NEA_ERR_CUDA;
  const cuuint64_t e = f32 ? 4 : 2;
  const cuuint32_t row_bytes = D * e < 128 ? cuuint32_t(D * e) : 128u;  // one swizzle atom row
  const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(Tc), cuuint64_t(Hkv), cuuint64_t(B)};
  const cuuint64_t strides[3] = {cuuint64_t(Hkv) * D * e, D * e, cuuint64_t(Tc) * Hkv * D * e};
  const cuuint32_t box[4] = {cuuint32_t(row_bytes / e), cuuint32_t(rows), cuuint32_t(heads), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NEA_OK : NEA_ERR_CUDA;
}

// Descriptor of the backward row terms ws[B*Hq][2][Tp], box {128, 2, 1}:
// one box is a column tile's LSE*log2e followed by its Dv.
int make_rowterm_map(CUtensorMap* m, const float* base, int BH, int Tp) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return NEA_ERR_CUDA;
  const cuuint64_t dims[3] = {cuuint64_t(Tp), 2, cuuint64_t(BH)};
  const cuuint64_t strides[2] = {cuuint64_t(Tp) * 4, cuuint64_t(Tp) * 8};
  const cuuint32_t box[3] = {cuuint32_t(nea::kTileRows), 2, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NEA_OK : NEA_ERR_CUDA;
}

// Returns the state of the current device, probing it once.
int device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  DeviceState& st = g_dev[dev];
  if (!st.probed) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e);
    st.sm100 = (major == 10 && minor == 0);
    if ((e = cudaDeviceGetAttribute(&st.n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e);
    if (st.sm100) {
      if ((e = cudaMalloc(&st.err, sizeof(int))) != cudaSuccess) return cuda_fail(e);
      if ((e = cudaMemset(st.err, 0, sizeof(int))) != cudaSuccess) return cuda_fail(e);
    }
    st.probed = true;
  }
  if (!st.sm100) return NEA_ERR_UNSUPPORTED;
  *out = &st;
  return NEA_OK;
}

// Rotary table [T][D/2] of (cos, sin) of t * base^(-2i/D): angle, cosine and
// sine in double precision, each rounded to float once.  Both the cached
// tables of the regular entry points and the allocation-free backward's table
// come from this kernel, so the two are bit-identical.
__global__ void rope_table_kernel(float2* out, int T, int D, double base) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int half = D / 2;
  if (idx >= (long long)T * half) return;
  const int t = int(idx / half), i = int(idx % half);
  const double a = double(t) * pow(base, -2.0 * double(i) / double(D));
  double sn, cs;
  sincos(a, &sn, &cs);
  out[idx] = make_float2(float(cs), float(sn));
}

cudaError_t launch_rope_table(float2* out, int T, int D, float base, cudaStream_t stream) {
  const long long n = (long long)T * (D / 2);
  rope_table_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(out, T, D, double(base));
  return cudaGetLastError();
}

// The cached table for (T, D, base), built on first use.
int rope_table(DeviceState& st, int T, int D, float base, cudaStream_t stream, const float2** out) {
  if (!(base > 0.f)) {
    *out = nullptr;
    return NEA_OK;
  }
  uint32_t bits;
  std::memcpy(&bits, &base, sizeof bits);
  auto key = std::make_tuple(T, D, bits);
  auto it = st.rope.find(key);
  if (it != st.rope.end()) {
    *out = it->second;
    return NEA_OK;
  }
  float2* d = nullptr;
  cudaError_t e = cudaMalloc(&d, size_t(T) * (D / 2) * sizeof(float2));
  if (e != cudaSuccess) return cuda_fail(e);
  e = launch_rope_table(d, T, D, base, stream);
  // later calls may use the table from another stream: finish it now
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    cudaFree(d);
    return cuda_fail(e);
  }
  st.rope.emplace(key, d);
  *out = d;
  return NEA_OK;
}

int ensure_ws(DeviceState& st, size_t bytes) {
  if (bytes <= st.ws_bytes) return NEA_OK;
  cudaError_t e;
  if (st.ws) {
    // kernels on any stream may still read the old buffer
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e);
    cudaFree(st.ws);
    st.ws = nullptr;
    st.ws_bytes = 0;
  }
  if ((e = cudaMalloc(&st.ws, bytes)) != cudaSuccess) return cuda_fail(e);
  st.ws_bytes = bytes;
  return NEA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape/dtype checks shared by the entry points.  `empty` is set when
// B*T == 0 (nothing to do, pointers may be null).  D = 128 only where
// `d128` is set (bfloat16 storage; not the allocation-free backward).
int check_shape(int B, int T, int Hq, int Hkv, int D, int dtype, int causal, bool* empty, bool d128 = false) {
  if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return NEA_ERR_ARG;
  if (D != 32 && D != 64 && !(D == 128 && d128 && dtype == NEA_BF16)) return NEA_ERR_ARG;
  if (dtype != NEA_F32 && dtype != NEA_BF16) return NEA_ERR_ARG;
  if (causal != 0 && causal != 1) return NEA_ERR_ARG;
  // 32-bit grid and tile indices: keep every launch well inside them
  const long long tiles = (static_cast<long long>(T) + 127) / 128;
  if (tiles * B * Hq > (1LL << 30) || static_cast<long long>(T) > (1LL << 24)) return NEA_ERR_ARG;
  if (static_cast<long long>(B) * (tiles * 128) * Hq > (1LL << 30)) return NEA_ERR_ARG;
  *empty = (static_cast<long long>(B) * T == 0);
  return NEA_OK;
}

// Launches a kernel with programmatic stream serialization: its blocks may
// start (barrier set-up, TMEM allocation) while the previous kernel in the
// stream drains; each kernel launched this way calls grid_dep_wait() before
// its first global access, so stream order still holds for memory.
template <typename... P, typename... A>
cudaError_t launch_dependent(void (*kern)(P...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                             A&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

template <typename Kern>
int set_smem(uint32_t& attr_done, int bit, Kern kern, uint32_t bytes) {
  if (attr_done & (1u << bit)) return NEA_OK;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  if (e != cudaSuccess) return cuda_fail(e);
  attr_done |= 1u << bit;
  return NEA_OK;
}

// Calls f(std::integral_constant<int, D>, std::bool_constant<F32IO>).
template <typename F>
int dispatch(int D, int dtype, F&& f) {
  const bool f32 = dtype == NEA_F32;
  if (D == 64)
    return f32 ? f(std::integral_constant<int, 64>{}, std::true_type{})
               : f(std::integral_constant<int, 64>{}, std::false_type{});
  return f32 ? f(std::integral_constant<int, 32>{}, std::true_type{})
             : f(std::integral_constant<int, 32>{}, std::false_type{});
}

// The decode kernels' dispatch: D = 32, 64 or 128, either storage type.
template <typename F>
int dispatch_dec(int D, int dtype, F&& f) {
  if (D == 128)
    return dtype == NEA_F32 ? f(std::integral_constant<int, 128>{}, std::true_type{})
                            : f(std::integral_constant<int, 128>{}, std::false_type{});
  return dispatch(D, dtype, f);
}

// ----------------------------------------------------------------- operand prologue
// Workspace bytes the prologue writes for `n` tensors of `elems[i]` elements:
// float32 storage, hi and lo planes of every tensor; bfloat16 storage, a
// rotated copy of each tensor with rot[i] set (none when the rotation is off).
// Every plane starts 256-byte aligned.
size_t prep_bytes(const size_t* elems, const int* rot, int n, bool f32, bool rope_on) {
  size_t b = 0;
  for (int i = 0; i < n; ++i) {
    if (f32) b += 2 * round_up(elems[i] * 2, 256);
    else if (rot[i] && rope_on) b += round_up(elems[i] * 2, 256);
  }
  return b;
}

// Carves the prologue's outputs for `n` tensors out of `base` (prep_bytes()
// bytes, same order).  jobs[i].hi (and .lo for float32 storage) are the
// operand tensors the attention kernels read: for bfloat16 storage the
// rotated copy or, for tensors left as they are, the input itself.
void carve_planes(uint8_t* base, const void* const* src, const size_t* elems, const int* H, const int* rot, int n,
                  int D, bool f32, const float2* table, nea::PrepJob* jobs) {
  size_t off = 0;
  for (int i = 0; i < n; ++i) {
    nea::PrepJob j{};
    j.src = src[i];
    j.H = H[i];
    j.divH = nea::make_fastdiv(uint32_t(H[i]));
    j.rope = rot[i] && table != nullptr;
    if (!f32 && !j.rope) {  // read in place
      j.hi = static_cast<__nv_bfloat16*>(const_cast<void*>(src[i]));
      jobs[i] = j;
      continue;
    }
    j.hi = reinterpret_cast<__nv_bfloat16*>(base + off);
    off += round_up(elems[i] * 2, 256);
    if (f32) {
      j.lo = reinterpret_cast<__nv_bfloat16*>(base + off);
      off += round_up(elems[i] * 2, 256);
    }
    j.chunks = static_cast<long long>(elems[i] / (f32 ? 4 : 8));
    j.rows = static_cast<int>(elems[i] / D);
    jobs[i] = j;
  }
}

// Runs the prologue over the jobs with run[i] set that have planes to write
// (and, with `rowterm`, the backward row terms in the same launch).
int launch_prep(const nea::PrepJob* jobs, const bool* run, int n, int T, int D, bool f32, const float2* table,
                cudaStream_t stream, const nea::PrepParams* rowterm = nullptr) {
  nea::PrepParams pp{};
  if (rowterm) pp = *rowterm;  // row-term fields of the backward
  pp.n_jobs = 0;
  pp.total = 0;
  pp.prep_blocks = 0;
  pp.T = T;
  pp.rope = table;
  pp.divT = nea::make_fastdiv(uint32_t(T));
  if (pp.rt_rows) {
    pp.divTp = nea::make_fastdiv(uint32_t(pp.Tp));
    pp.divHq = nea::make_fastdiv(uint32_t(pp.Hq));
  }
  const int rows_per_block = 256 / (D * (f32 ? 4 : 2) / 16) * nea::kPrepUnroll;
  for (int i = 0; i < n; ++i) {
    if (!run[i] || jobs[i].rows == 0) continue;  // nothing to write (in place, or planes made elsewhere)
    nea::PrepJob j = jobs[i];
    j.block0 = pp.prep_blocks;
    pp.prep_blocks += (j.rows + rows_per_block - 1) / rows_per_block;
    pp.job[pp.n_jobs++] = j;
    pp.total += j.chunks;
  }
  const long long rt_blocks = D == 128  ? nea::rowterm_blocks<128, false>(pp.rt_rows)  // bfloat16 only
                              : D == 64 ? (f32 ? nea::rowterm_blocks<64, true>(pp.rt_rows)
                                               : nea::rowterm_blocks<64, false>(pp.rt_rows))
                                        : (f32 ? nea::rowterm_blocks<32, true>(pp.rt_rows)
                                               : nea::rowterm_blocks<32, false>(pp.rt_rows));
  const long long blocks = pp.prep_blocks + rt_blocks;
  if (blocks == 0) return NEA_OK;
  const unsigned g = unsigned(blocks);
  auto kern = D == 128  ? nea::attn_prep_kernel<128, false>
              : D == 64 ? (f32 ? nea::attn_prep_kernel<64, true> : nea::attn_prep_kernel<64, false>)
                        : (f32 ? nea::attn_prep_kernel<32, true> : nea::attn_prep_kernel<32, false>);
  const cudaError_t e = launch_dependent(kern, g, 256, 0, stream, pp);
  return e == cudaSuccess ? NEA_OK : cuda_fail(e);
}

// Carves and runs the prologue for all `n` tensors.
int run_prep(uint8_t* base, const void* const* src, const size_t* elems, const int* H, const int* rot, int n,
             int T, int D, bool f32, const float2* table, nea::PrepJob* jobs_out, cudaStream_t stream,
             const nea::PrepParams* rowterm = nullptr) {
  carve_planes(base, src, elems, H, rot, n, D, f32, table, jobs_out);
  const bool run[4] = {true, true, true, true};
  return launch_prep(jobs_out, run, n, T, D, f32, table, stream, rowterm);
}

// ----------------------------------------------------------------- forward
template <int D, bool F32IO>
int launch_fwd(uint32_t& attr_done, const nea::FwdParams& p, cudaStream_t stream) {
  using L = nea::FwdSmem<D, F32IO>;
  auto kern = nea::attn_fwd_kernel<D, F32IO>;
  int rc = set_smem(attr_done, D == 128 ? 8 : (D == 64) * 2 + F32IO, kern, L::kAlloc);
  if (rc) return rc;
  const cudaError_t e = launch_dependent(kern, unsigned(p.B * p.Hq * p.n_pairs), L::kThreads, L::kAlloc, stream, p);
  return e == cudaSuccess ? NEA_OK : cuda_fail(e);
}

// ----------------------------------------------------------------- backward
// The gradient kernel (dK/dV and dQ units in one launch).  `ev` selects profiling events (the
// regular backward records them, the allocation-free one does not).
// Float32 storage runs the split-bf16 gradient kernel (nea_bwd_f32.cuh),
// bfloat16 storage the bf16 one (nea_bwd.cuh).
template <int D, bool F32IO>
int launch_bwd(uint32_t& attr_done, const nea::BwdParams& p, cudaStream_t stream, bool ev) {
  cudaError_t e;
  using L = std::conditional_t<F32IO, nea::Bwd32Smem<D>, nea::BwdSmem<D>>;
  auto kern = [] {
    if constexpr (F32IO) return nea::attn_bwd_f32_kernel<D>;
    else return nea::attn_bwd_kernel<D>;
  }();
  int rc = set_smem(attr_done, D == 128 ? 9 : 4 + (D == 64) * 2 + F32IO, kern, L::kAlloc);
  if (rc) return rc;
  e = launch_dependent(kern, unsigned(p.n_dkdv + p.B * p.Hq * p.n_tiles), L::kThreads, L::kAlloc, stream, p);
  if (e != cudaSuccess) return cuda_fail(e);
  if (ev) prof_record(4, stream);
  if (ev) prof_record(5, stream);
  return NEA_OK;
}

int check_bwd_args(const void* Q, const void* K, const void* V, const void* O, const float* LSE, const void* dO,
                   void* dQ, void* dK, void* dV, int B, int T, int Hq, int Hkv, int D, int dtype, float rope_base,
                   int causal, bool* empty, bool d128 = false) {
  int rc = check_shape(B, T, Hq, Hkv, D, dtype, causal, empty, d128);
  if (rc || *empty) return rc;
  if (!Q || !K || !V || !O || !LSE || !dO || !dQ || !dK || !dV) return NEA_ERR_ARG;
  for (const void* ptr : {Q, K, V, O, static_cast<const void*>(LSE), dO, static_cast<const void*>(dQ),
                          static_cast<const void*>(dK), static_cast<const void*>(dV)})
    if (!aligned16(ptr)) return NEA_ERR_ARG;
  if (!std::isfinite(rope_base)) return NEA_ERR_ARG;
  return NEA_OK;
}

// Bytes of backward workspace: the padded row terms, then the operand
// prologue's output (fp32: planes of Q, K, V, dO; bf16 with the rotation on:
// rotated Q and K).
// With `saved` planes only dO's share of the prologue output is needed.
size_t bwd_ws_bytes(int B, int T, int Hq, int Hkv, int D, bool f32, bool rope_on, size_t* rowterm_bytes,
                    bool saved = false) {
  const size_t Tp = round_up(size_t(T), nea::kTileRows);
  *rowterm_bytes = round_up(size_t(B) * Hq * 2 * Tp * sizeof(float), 256);
  const size_t nq = size_t(B) * T * Hq * D, nk = size_t(B) * T * Hkv * D;
  const size_t elems[4] = {nq, nk, nk, nq};
  const int rot[4] = {1, 1, 0, 0};
  if (saved) return *rowterm_bytes + prep_bytes(elems + 3, rot + 3, 1, f32, rope_on);
  return *rowterm_bytes + prep_bytes(elems, rot, 4, f32, rope_on);
}

// The backward after argument checks, given a workspace of bwd_ws_bytes()
// bytes, a rotary table (or nullptr) and a status word.
// With `saved` (the planes nea_attn_fwd_save wrote), the prologue converts
// only dO and writes the row terms; Q, K, V operands come from `saved`.
int run_bwd(uint32_t& attr_done, uint8_t* ws, const float2* rope, int* status, const void* Q, const void* K,
            const void* V, const void* O, const float* LSE, const void* dO, void* dQ, void* dK, void* dV, int B,
            int T, int Hq, int Hkv, int D, int dtype, int causal, cudaStream_t stream, bool ev,
            const uint8_t* saved = nullptr) {
  const bool f32 = dtype == NEA_F32;
  size_t rowterm_bytes = 0;
  (void)bwd_ws_bytes(B, T, Hq, Hkv, D, f32, rope != nullptr, &rowterm_bytes);
  nea::BwdParams p{};
  p.Tp = int(round_up(size_t(T), nea::kTileRows));
  p.ws = reinterpret_cast<const float*>(ws);
  int rc;
  if (ev) prof_record(2, stream);
  {
    // operand prologue: rotated Q and K (float32 storage: hi/lo planes of
    // rotated Q, K and of V, dO)
    const size_t nq = size_t(B) * T * Hq * D, nk = size_t(B) * T * Hkv * D;
    const void* src[4] = {Q, K, V, dO};
    const size_t elems[4] = {nq, nk, nk, nq};
    const int H[4] = {Hq, Hkv, Hkv, Hq}, rot[4] = {1, 1, 0, 0};
    nea::PrepJob jobs[4];
    nea::PrepParams rt{};  // the row terms ride in the same launch
    rt.O = O;
    rt.dO = dO;
    rt.LSE = LSE;
    rt.ws = reinterpret_cast<float*>(ws);
    rt.B = B;
    rt.Tp = p.Tp;
    rt.Hq = Hq;
    rt.rt_rows = static_cast<long long>(B) * p.Tp * Hq;
    // Q, K, V planes from the forward (`saved`) or made here; dO's planes
    // (float32 storage) are written by the row-term threads, which read dO
    if (saved) carve_planes(const_cast<uint8_t*>(saved), src, elems, H, rot, 3, D, f32, rope, jobs);
    else carve_planes(ws + rowterm_bytes, src, elems, H, rot, 3, D, f32, rope, jobs);
    const size_t q_planes = saved ? 0 : prep_bytes(elems, rot, 3, f32, rope != nullptr);
    carve_planes(ws + rowterm_bytes + q_planes, src + 3, elems + 3, H + 3, rot + 3, 1, D, f32, rope, jobs + 3);
    rt.do_hi = f32 ? jobs[3].hi : nullptr;
    rt.do_lo = f32 ? jobs[3].lo : nullptr;
    const bool run[4] = {!saved, !saved, !saved, false};
    if ((rc = launch_prep(jobs, run, 4, T, D, f32, rope, stream, &rt))) return rc;
    if (ev) prof_record(3, stream);
    if ((rc = make_tile_map(&p.tm_q, jobs[0].hi, B, T, Hq, D)) ||
        (rc = make_tile_map(&p.tm_k, jobs[1].hi, B, T, Hkv, D)) ||
        (rc = make_tile_map(&p.tm_v, jobs[2].hi, B, T, Hkv, D)) ||
        (rc = make_tile_map(&p.tm_do, jobs[3].hi, B, T, Hq, D)))
      return rc;
    if (f32 && ((rc = make_tile_map(&p.tm_q_lo, jobs[0].lo, B, T, Hq, D)) ||
                (rc = make_tile_map(&p.tm_k_lo, jobs[1].lo, B, T, Hkv, D)) ||
                (rc = make_tile_map(&p.tm_v_lo, jobs[2].lo, B, T, Hkv, D)) ||
                (rc = make_tile_map(&p.tm_do_lo, jobs[3].lo, B, T, Hq, D))))
      return rc;
  }
  if ((rc = make_rowterm_map(&p.tm_ws, p.ws, B * Hq, p.Tp))) return rc;
  p.dQ = dQ;
  p.dK = dK;
  p.dV = dV;
  p.rope = rope;
  p.B = B;
  p.T = T;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_tiles = (T + 127) / 128;
  p.n_dkdv = B * Hkv * p.n_tiles;
  p.causal = causal;
  p.scale = float(1.0 / std::sqrt(double(D)));
  p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
  p.err = status;
  p.wait_limit = static_cast<unsigned long long>(t_wait_limit_ns);
  p.debug = t_debug_flags & 2;  // bit 1 arms the next backward launch
  t_debug_flags &= ~2;
#ifdef NEA_TRACE
  p.trace = t_trace_bwd;
#endif
  if (D == 128) return launch_bwd<128, false>(attr_done, p, stream, ev);  // bfloat16 storage only
  return dispatch(D, dtype, [&](auto d, auto f) {
    return launch_bwd<decltype(d)::value, decltype(f)::value>(attr_done, p, stream, ev);
  });
}

// Bytes of the forward's operand planes: float32 storage, hi/lo planes of
// the rotated Q, K and of V; bfloat16 storage with the rotation on, rotated
// Q and K; otherwise none.
size_t fwd_plane_bytes(int B, int T, int Hq, int Hkv, int D, bool f32, bool rope_on) {
  const size_t nq = size_t(B) * T * Hq * D, nk = size_t(B) * T * Hkv * D;
  const size_t elems[3] = {nq, nk, nk};
  const int rot[3] = {1, 1, 0};
  return prep_bytes(elems, rot, 3, f32, rope_on);
}

int check_fwd_args(const void* Q, const void* K, const void* V, const void* O, const float* LSE, int B, int T,
                   int Hq, int Hkv, int D, int dtype, float rope_base, int causal, bool* empty, bool d128 = false) {
  int rc = check_shape(B, T, Hq, Hkv, D, dtype, causal, empty, d128);
  if (rc || *empty) return rc;
  if (!Q || !K || !V || !O || !LSE) return NEA_ERR_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return NEA_ERR_ARG;
  if (!std::isfinite(rope_base)) return NEA_ERR_ARG;
  return NEA_OK;
}

// The forward after argument checks; its operand planes go to `saved` when
// given, else to the device workspace.
int run_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int T, int Hq, int Hkv, int D,
            int dtype, float rope_base, int causal, cudaStream_t stream, uint8_t* saved) {
  const bool f32 = dtype == NEA_F32;
  int rc;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  nea::FwdParams p{};
  const float2* rope = nullptr;
  if ((rc = rope_table(*st, T, D, rope_base, stream, &rope))) return rc;
  prof_record(0, stream);
  {
    // operand prologue: rotated Q and K (float32 storage: hi/lo planes of
    // rotated Q, K and of V)
    const size_t nq = size_t(B) * T * Hq * D, nk = size_t(B) * T * Hkv * D;
    const void* src[3] = {Q, K, V};
    const size_t elems[3] = {nq, nk, nk};
    const int H[3] = {Hq, Hkv, Hkv}, rot[3] = {1, 1, 0};
    uint8_t* planes = saved;
    if (!planes) {
      if ((rc = ensure_ws(*st, fwd_plane_bytes(B, T, Hq, Hkv, D, f32, rope != nullptr)))) return rc;
      planes = st->ws;
    }
    nea::PrepJob jobs[3];
    if ((rc = run_prep(planes, src, elems, H, rot, 3, T, D, f32, rope, jobs, stream))) return rc;
    prof_record(6, stream);
    if ((rc = make_tile_map(&p.tm_q, jobs[0].hi, B, T, Hq, D)) ||
        (rc = make_tile_map(&p.tm_k, jobs[1].hi, B, T, Hkv, D)) ||
        (rc = make_tile_map(&p.tm_v, jobs[2].hi, B, T, Hkv, D)))
      return rc;
    if (f32 && ((rc = make_tile_map(&p.tm_q_lo, jobs[0].lo, B, T, Hq, D)) ||
                (rc = make_tile_map(&p.tm_k_lo, jobs[1].lo, B, T, Hkv, D)) ||
                (rc = make_tile_map(&p.tm_v_lo, jobs[2].lo, B, T, Hkv, D))))
      return rc;
  }
  p.O = O;
  p.LSE = LSE;
  p.B = B;
  p.T = T;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_tiles = (T + 127) / 128;
  p.n_pairs = (p.n_tiles + 1) / 2;
  p.causal = causal;
  p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
  p.err = st->err;
  p.wait_limit = static_cast<unsigned long long>(t_wait_limit_ns);
  p.debug = t_debug_flags & 1;  // bit 0 arms the next forward launch
  t_debug_flags &= ~1;
#ifdef NEA_TRACE
  p.trace = t_trace;
#endif
  rc = D == 128 ? launch_fwd<128, false>(st->attr_done, p, stream)  // bfloat16 storage only
                : dispatch(D, dtype, [&](auto d, auto f) {
                    return launch_fwd<decltype(d)::value, decltype(f)::value>(st->attr_done, p, stream);
                  });
  prof_record(1, stream);
  return rc;
}

}  // namespace

namespace nea_internal {

int device_status_word(int** err, int* n_sm) {
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  const int rc = device_state(&st);
  if (rc) return rc;
  *err = st->err;
  *n_sm = st->n_sm;
  return NEA_OK;
}

long long wait_limit_ns() { return t_wait_limit_ns; }

}  // namespace nea_internal

extern "C" {

int nea_attn_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int T, int Hq, int Hkv,
                 int D, int dtype, float rope_base, int causal, void* stream) {
  bool empty = false;
  int rc = check_fwd_args(Q, K, V, O, LSE, B, T, Hq, Hkv, D, dtype, rope_base, causal, &empty, true);
  if (rc || empty) return rc;
  return run_fwd(Q, K, V, O, LSE, B, T, Hq, Hkv, D, dtype, rope_base, causal, static_cast<cudaStream_t>(stream),
                 nullptr);
}

long long nea_attn_saved_bytes(int B, int T, int Hq, int Hkv, int D, int dtype, float rope_base) {
  bool empty = false;
  if (check_shape(B, T, Hq, Hkv, D, dtype, 1, &empty, true) || !std::isfinite(rope_base)) return -1;
  if (empty) return 0;
  return static_cast<long long>(fwd_plane_bytes(B, T, Hq, Hkv, D, dtype == NEA_F32, rope_base > 0.f));
}

int nea_attn_fwd_save(const void* Q, const void* K, const void* V, void* O, float* LSE, void* saved, int B, int T,
                      int Hq, int Hkv, int D, int dtype, float rope_base, int causal, void* stream) {
  bool empty = false;
  int rc = check_fwd_args(Q, K, V, O, LSE, B, T, Hq, Hkv, D, dtype, rope_base, causal, &empty, true);
  if (rc || empty) return rc;
  const bool need = fwd_plane_bytes(B, T, Hq, Hkv, D, dtype == NEA_F32, rope_base > 0.f) > 0;
  if (need && (!saved || !aligned16(saved))) return NEA_ERR_ARG;
  return run_fwd(Q, K, V, O, LSE, B, T, Hq, Hkv, D, dtype, rope_base, causal, static_cast<cudaStream_t>(stream),
                 need ? static_cast<uint8_t*>(saved) : nullptr);
}

int nea_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const float* LSE, const void* dO,
                 void* dQ, void* dK, void* dV, int B, int T, int Hq, int Hkv, int D, int dtype, float rope_base,
                 int causal, void* stream_) {
  bool empty = false;
  int rc = check_bwd_args(Q, K, V, O, LSE, dO, dQ, dK, dV, B, T, Hq, Hkv, D, dtype, rope_base, causal, &empty,
                          true);
  if (rc || empty) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  const float2* rope = nullptr;
  if ((rc = rope_table(*st, T, D, rope_base, stream, &rope))) return rc;
  size_t rowterm_bytes = 0;
  if ((rc = ensure_ws(*st, bwd_ws_bytes(B, T, Hq, Hkv, D, dtype == NEA_F32, rope != nullptr, &rowterm_bytes))))
    return rc;
  return run_bwd(st->attr_done, st->ws, rope, st->err, Q, K, V, O, LSE, dO, dQ, dK, dV, B, T, Hq, Hkv, D, dtype,
                 causal, stream, true);
}

int nea_attn_bwd_saved(const void* Q, const void* K, const void* V, const void* O, const float* LSE, const void* dO,
                       const void* saved, void* dQ, void* dK, void* dV, int B, int T, int Hq, int Hkv, int D,
                       int dtype, float rope_base, int causal, void* stream_) {
  bool empty = false;
  int rc = check_bwd_args(Q, K, V, O, LSE, dO, dQ, dK, dV, B, T, Hq, Hkv, D, dtype, rope_base, causal, &empty,
                          true);
  if (rc || empty) return rc;
  const bool f32 = dtype == NEA_F32, rope_on = rope_base > 0.f;
  if (fwd_plane_bytes(B, T, Hq, Hkv, D, f32, rope_on) == 0)  // nothing was saved: the regular backward
    return nea_attn_bwd(Q, K, V, O, LSE, dO, dQ, dK, dV, B, T, Hq, Hkv, D, dtype, rope_base, causal, stream_);
  if (!saved || !aligned16(saved)) return NEA_ERR_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  const float2* rope = nullptr;
  if ((rc = rope_table(*st, T, D, rope_base, stream, &rope))) return rc;
  size_t rowterm_bytes = 0;
  if ((rc = ensure_ws(*st, bwd_ws_bytes(B, T, Hq, Hkv, D, f32, rope_on, &rowterm_bytes, true)))) return rc;
  return run_bwd(st->attr_done, st->ws, rope, st->err, Q, K, V, O, LSE, dO, dQ, dK, dV, B, T, Hq, Hkv, D, dtype,
                 causal, stream, true, static_cast<const uint8_t*>(saved));
}

int nea_attn_decode(const void* Q, const void* Kc, const void* Vc, const int* lens, void* O, float* LSE, int B,
                    int Tc, int Hq, int Hkv, int D, int dtype, float rope_base, void* stream_) {
  if (B < 0 || Tc < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return NEA_ERR_ARG;
  if (D != 32 && D != 64 && D != 128) return NEA_ERR_ARG;
  if (dtype != NEA_F32 && dtype != NEA_BF16) return NEA_ERR_ARG;
  if (Hq / Hkv > nea::kDecMaxG || Hkv > 65535 || B > 65535) return NEA_ERR_ARG;
  if (!std::isfinite(rope_base)) return NEA_ERR_ARG;
  if (B == 0) return NEA_OK;
  if (Tc < 1 || Tc > (1 << 24)) return NEA_ERR_ARG;
  if (!Q || !Kc || !Vc || !lens || !O || !LSE) return NEA_ERR_ARG;
  if (!aligned16(Q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(O) || !aligned16(LSE) ||
      (reinterpret_cast<uintptr_t>(lens) & 3u))
    return NEA_ERR_ARG;
  const int G = Hq / Hkv;
  const int HP = nea::dec_heads_per_piece(Hkv, G, D, dtype == NEA_F32);
  const int R = nea::dec_lines(G, D, dtype == NEA_F32) / HP;
  const int NP = (Tc + R - 1) / R;
  const unsigned long long n_pieces = static_cast<unsigned long long>(B) * (Hkv / HP) * NP;
  const size_t part_bytes = round_up(size_t(n_pieces) * nea::kDecWarps * G * (D + 2) * sizeof(float), 256);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  nea::DecodeParams p{};
  if ((rc = rope_table(*st, Tc, D, rope_base, stream, &p.rope))) return rc;
  if ((rc = ensure_ws(*st, part_bytes))) return rc;
  p.Q = Q;
  p.lens = lens;
  p.O = O;
  p.LSE = LSE;
  p.part = reinterpret_cast<float*>(st->ws);
  p.B = B;
  p.Tc = Tc;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.HP = HP;
  p.NHG = Hkv / HP;
  p.WPH = nea::kDecWarps / HP;
  p.R = R;
  p.NP = NP;
  p.n_pieces = n_pieces;
  p.n_cta = static_cast<int>(std::min<unsigned long long>(
      n_pieces, static_cast<unsigned long long>(std::min(st->n_sm, nea::kDecMaxSeg - 1))));
  p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
  p.err = st->err;
  p.wait_limit = static_cast<unsigned long long>(t_wait_limit_ns);
  if ((rc = make_cache_map(&p.tm_k, Kc, B, Tc, Hkv, D, dtype == NEA_F32, HP, R)) ||
      (rc = make_cache_map(&p.tm_v, Vc, B, Tc, Hkv, D, dtype == NEA_F32, HP, R)))
    return rc;
  rc = dispatch_dec(D, dtype, [&](auto d, auto f) {
    constexpr int DD = decltype(d)::value;
    constexpr bool FF = decltype(f)::value;
    auto launch = [&](auto gtag) -> int {
      constexpr int GG = decltype(gtag)::value;
      using L = nea::DecLayout<DD, FF, GG>;
      auto kern = nea::attn_decode_kernel<DD, FF, GG>;
      const int bit = ((DD == 128 ? 2 : DD == 64 ? 1 : 0) * 2 + FF) * 8 + (GG - 1);
      if (!(st->attr_dec >> bit & 1)) {
        // both kernels ask for the largest shared-memory carveout, so that
        // the SMs keep one configuration from the stream to the merge
        cudaError_t ea = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(L::kAlloc));
        if (ea == cudaSuccess)
          ea = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, int(cudaSharedmemCarveoutMaxShared));
        if (ea == cudaSuccess)
          ea = cudaFuncSetAttribute(nea::attn_decode_merge_kernel<DD, FF, GG>,
                                    cudaFuncAttributePreferredSharedMemoryCarveout, int(cudaSharedmemCarveoutMaxShared));
        if (ea != cudaSuccess) return cuda_fail(ea);
        st->attr_dec |= uint64_t(1) << bit;
      }
      kern<<<unsigned(p.n_cta), nea::kDecThreads, L::kAlloc, stream>>>(p);
      const cudaError_t ek = cudaGetLastError();
      if (ek != cudaSuccess) return cuda_fail(ek);
      // the merge, one CTA per (sequence, kv head), resident while the stream drains
      const cudaError_t em = launch_dependent(nea::attn_decode_merge_kernel<DD, FF, GG>, unsigned(B * Hkv),
                                              unsigned(nea::dec_merge_groups(GG, DD) * GG * DD), 0, stream, p);
      return em == cudaSuccess ? NEA_OK : cuda_fail(em);
    };
    switch (p.G) {
      case 1: return launch(std::integral_constant<int, 1>{});
      case 2: return launch(std::integral_constant<int, 2>{});
      case 3: return launch(std::integral_constant<int, 3>{});
      case 4: return launch(std::integral_constant<int, 4>{});
      case 5: return launch(std::integral_constant<int, 5>{});
      case 6: return launch(std::integral_constant<int, 6>{});
      case 7: return launch(std::integral_constant<int, 7>{});
      default: return launch(std::integral_constant<int, 8>{});
    }
  });
  if (rc) return rc;
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? NEA_OK : cuda_fail(e);
}

long long nea_set_wait_limit_ns(long long ns) {
  const long long prev = t_wait_limit_ns;
  t_wait_limit_ns = ns < 1000000LL ? 1000000LL : ns;
  return prev;
}

void nea_debug_inject(int flags) { t_debug_flags = flags; }

#ifdef NEA_TRACE
void nea_debug_set_trace(void* buffer) { t_trace = static_cast<unsigned long long*>(buffer); }
void nea_debug_set_trace_bwd(void* buffer) { t_trace_bwd = static_cast<unsigned long long*>(buffer); }
#endif

void nea_set_profile_events(void* const* events, int n) {
  t_prof_events = (events && n > 0) ? events : nullptr;
  t_prof_n = t_prof_events ? n : 0;
}

const char* nea_status_string(int status) {
  switch (status) {
    case NEA_OK: return "NEA_OK";
    case NEA_ERR_ARG: return "NEA_ERR_ARG: invalid pointer, shape, alignment or dtype";
    case NEA_ERR_CUDA: return "NEA_ERR_CUDA: CUDA runtime call or kernel launch failed";
    case NEA_ERR_TIMEOUT: return "NEA_ERR_TIMEOUT: a kernel abandoned a bounded device-side wait";
    case NEA_ERR_UNSUPPORTED: return "NEA_ERR_UNSUPPORTED: current device is not sm_100";
    case NEA_ERR_NOMEM: return "NEA_ERR_NOMEM: workspace allocation failed";
    case NEA_ERR_SCRATCH_LIMIT:
      return "NEA_ERR_SCRATCH_LIMIT: problem exceeds the fixed scratch of nea_attn_bwd_noalloc";
    default: return "unknown status";
  }
}

int nea_version(void) { return kVersion; }

}  // extern "C"

// ===================================================================== no-allocation backward
// A second way into the same backward kernels for callers that may not
// allocate device memory.  Its scratch is this fixed array instead of the
// per-device workspace above; nothing here calls cudaMalloc/cudaFree.
namespace {

constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;  // 4 MiB
constexpr size_t kNoAllocStatusBytes = 256;                 // status word, padded
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// Host-side state per device: the array's device address (the host-side name
// `g_noalloc_scratch` is only a stand-in and must never reach a kernel) and
// which kernel attributes are set.  Fixed-size, so no host allocation either.
struct NoAllocDevice {
  bool ready = false;
  bool sm100 = false;
  uint8_t* scratch = nullptr;
  uint32_t attr_done = 0;
};
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];
std::mutex g_noalloc_mu;

}  // namespace

extern "C" int nea_attn_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const float* LSE,
                                    const void* dO, void* dQ, void* dK, void* dV, int B, int T, int Hq, int Hkv,
                                    int D, int dtype, float rope_base, int causal, void* stream_) {
  bool empty = false;
  int rc = check_bwd_args(Q, K, V, O, LSE, dO, dQ, dK, dV, B, T, Hq, Hkv, D, dtype, rope_base, causal, &empty);
  if (rc || empty) return rc;
  size_t rowterm_bytes = 0;
  const bool rope_on = rope_base > 0.f;
  const size_t ws_bytes = bwd_ws_bytes(B, T, Hq, Hkv, D, dtype == NEA_F32, rope_on, &rowterm_bytes);
  const size_t rope_bytes = rope_on ? round_up(size_t(T) * D * sizeof(float), 256) : 0;
  if (kNoAllocStatusBytes + ws_bytes + rope_bytes > kNoAllocScratchFloats * sizeof(float))
    return NEA_ERR_SCRATCH_LIMIT;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kNoAllocMaxDevices) return NEA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice& st = g_noalloc_dev[dev];
  if (!st.ready) {
    // one-time set-up on this device (it is current): resolve the array's
    // device address; the symbol itself is only a host-side placeholder
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e);
    st.sm100 = (major == 10 && minor == 0);
    if (st.sm100) {
      void* ptr = nullptr;
      if ((e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch)) != cudaSuccess) return cuda_fail(e);
      st.scratch = static_cast<uint8_t*>(ptr);
    }
    st.ready = true;
  }
  if (!st.sm100) return NEA_ERR_UNSUPPORTED;

  // scratch: status word | row terms (+ fp32 operand planes) | rotary table.
  // The status word starts at zero (static storage) and is read and cleared
  // by nea_device_status; the row terms, planes and table are rewritten in
  // full by their kernels, so nothing else needs clearing.
  int* status = reinterpret_cast<int*>(st.scratch);
  uint8_t* ws = st.scratch + kNoAllocStatusBytes;
  float2* rope = rope_bytes ? reinterpret_cast<float2*>(ws + ws_bytes) : nullptr;
  if (rope && (e = launch_rope_table(rope, T, D, rope_base, stream)) != cudaSuccess) return cuda_fail(e);
  return run_bwd(st.attr_done, ws, rope, status, Q, K, V, O, LSE, dO, dQ, dK, dV, B, T, Hq, Hkv, D, dtype, causal,
                 stream, false);
}

// ===================================================================== device status
namespace {

// Reads and clears one device status word (a synchronous copy and a memset;
// neither allocates).  Returns the CUDA error, or success with *v set.
cudaError_t take_status(int* word, int* v) {
  int x = 0;
  cudaError_t e = cudaMemcpy(&x, word, sizeof x, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && x != 0) e = cudaMemset(word, 0, sizeof(int));
  *v = x;
  return e;
}

}  // namespace

// Reads the status words of the current device -- the regular entry points'
// and the allocation-free backward's -- without setting either up, so that a
// caller of nea_attn_bwd_noalloc alone never causes an allocation here.
extern "C" int nea_device_status(void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e);
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e);
  int v = 0;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_dev.find(dev);
    if (it != g_dev.end() && it->second.probed && it->second.err) {
      if ((e = take_status(it->second.err, &v)) != cudaSuccess) return cuda_fail(e);
    }
  }
  if (dev >= 0 && dev < kNoAllocMaxDevices) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    const NoAllocDevice& na = g_noalloc_dev[dev];
    int w = 0;
    if (na.ready && na.scratch) {
      if ((e = take_status(reinterpret_cast<int*>(na.scratch), &w)) != cudaSuccess) return cuda_fail(e);
    }
    if (v == 0) v = w;
  }
  if (v == nea::kErrBadLength) return NEA_ERR_ARG;
  return v ? NEA_ERR_TIMEOUT : NEA_OK;
}
