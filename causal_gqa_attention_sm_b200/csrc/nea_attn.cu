// C ABI of the attention library: argument checks, the per-device workspace
// (rotary table, backward row term, device error word) and kernel launches.
// Declarations and contracts: include/nea_attn.h.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "nea_attn.h"
#include "nea_bwd.cuh"
#include "nea_fwd.cuh"

namespace {

constexpr int kVersion = 100;  // 0.1.0

thread_local long long t_wait_limit_ns = 2000000000LL;
thread_local int t_debug_flags = 0;
thread_local void* const* t_prof_events = nullptr;
thread_local int t_prof_n = 0;

void prof_record(int i, cudaStream_t stream) {
  if (t_prof_events && i < t_prof_n && t_prof_events[i])
    cudaEventRecord(static_cast<cudaEvent_t>(t_prof_events[i]), stream);
}

struct DeviceState {
  bool probed = false;
  bool sm100 = false;
  int* err = nullptr;          // device error word
  float* dvec = nullptr;       // backward row term [B][Hq][T]
  size_t dvec_elems = 0;
  // rotary tables keyed by (T, D, base bits); never freed while the process
  // runs, so in-flight kernels on any stream keep valid pointers
  std::map<std::tuple<int, int, uint32_t>, float2*> rope;
  uint32_t attr_done = 0;      // bitmask of kernels whose smem attribute is set
};

std::mutex g_mu;
std::map<int, DeviceState> g_dev;

int cuda_fail(cudaError_t e) {
  (void)cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? NEA_ERR_NOMEM : NEA_ERR_CUDA;
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

// Rotary table [T][D/2] of (cos, sin) of t * base^(-2i/D), computed in double.
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
  std::vector<float2> h(size_t(T) * (D / 2));
  for (int t = 0; t < T; ++t)
    for (int i = 0; i < D / 2; ++i) {
      const double a = double(t) * std::pow(double(base), -2.0 * i / double(D));
      h[size_t(t) * (D / 2) + i] = make_float2(float(std::cos(a)), float(std::sin(a)));
    }
  float2* d = nullptr;
  cudaError_t e = cudaMalloc(&d, h.size() * sizeof(float2));
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemcpyAsync(d, h.data(), h.size() * sizeof(float2), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);  // host buffer dies below
  if (e != cudaSuccess) {
    cudaFree(d);
    return cuda_fail(e);
  }
  st.rope.emplace(key, d);
  *out = d;
  return NEA_OK;
}

int ensure_dvec(DeviceState& st, size_t elems, cudaStream_t stream) {
  if (elems <= st.dvec_elems) return NEA_OK;
  cudaError_t e;
  if (st.dvec) {
    // kernels on any stream may still read the old buffer
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e);
    cudaFree(st.dvec);
    st.dvec = nullptr;
    st.dvec_elems = 0;
  }
  (void)stream;
  if ((e = cudaMalloc(&st.dvec, elems * sizeof(float))) != cudaSuccess) return cuda_fail(e);
  st.dvec_elems = elems;
  return NEA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape/dtype checks shared by both entry points.  `empty` is set when
// B*T == 0 (nothing to do, pointers may be null).
int check_shape(int B, int T, int Hq, int Hkv, int D, int dtype, int causal, bool* empty) {
  if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return NEA_ERR_ARG;
  if (D != 32 && D != 64) return NEA_ERR_ARG;
  if (dtype != NEA_F32 && dtype != NEA_BF16) return NEA_ERR_ARG;
  if (causal != 0 && causal != 1) return NEA_ERR_ARG;
  // 32-bit grid and tile indices: keep every launch well inside them
  const long long tiles = (static_cast<long long>(T) + 127) / 128;
  if (tiles * B * Hq > (1LL << 30) || static_cast<long long>(T) > (1LL << 24)) return NEA_ERR_ARG;
  if (static_cast<long long>(B) * T * Hq > (1LL << 30)) return NEA_ERR_ARG;
  *empty = (static_cast<long long>(B) * T == 0);
  return NEA_OK;
}

template <typename Kern>
int set_smem(DeviceState& st, int bit, Kern kern, uint32_t bytes) {
  if (st.attr_done & (1u << bit)) return NEA_OK;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  if (e != cudaSuccess) return cuda_fail(e);
  st.attr_done |= 1u << bit;
  return NEA_OK;
}

template <int D, bool F32IO>
int launch_fwd(DeviceState& st, const nea::FwdParams& p, cudaStream_t stream) {
  using L = nea::FwdSmem<D, F32IO>;
  auto kern = nea::attn_fwd_kernel<D, F32IO>;
  int rc = set_smem(st, (D == 64) * 2 + F32IO, kern, L::kAlloc);
  if (rc) return rc;
  prof_record(0, stream);
  kern<<<p.B * p.Hq * p.n_tiles, 288, L::kAlloc, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  prof_record(1, stream);
  return e == cudaSuccess ? NEA_OK : cuda_fail(e);
}

template <int D, bool F32IO>
int launch_bwd(DeviceState& st, const nea::BwdParams& p, const void* O, cudaStream_t stream) {
  const int rows = p.B * p.T * p.Hq;
  constexpr int kLanes = D / (F32IO ? 4 : 8);
  const long long threads = static_cast<long long>(rows) * kLanes;
  prof_record(2, stream);
  nea::attn_bwd_rowterm_kernel<D, F32IO>
      <<<unsigned((threads + 255) / 256), 256, 0, stream>>>(O, p.dO, const_cast<float*>(p.Dv), rows, p.T, p.Hq);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  prof_record(3, stream);

  using LK = nea::BwdSmem<D, F32IO, true>;
  auto kk = nea::attn_bwd_kernel<D, F32IO, true>;
  int rc = set_smem(st, 4 + (D == 64) * 2 + F32IO, kk, LK::kAlloc);
  if (rc) return rc;
  kk<<<p.B * p.Hkv * p.n_tiles, 288, LK::kAlloc, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
  prof_record(4, stream);

  using LQ = nea::BwdSmem<D, F32IO, false>;
  auto kq = nea::attn_bwd_kernel<D, F32IO, false>;
  rc = set_smem(st, 8 + (D == 64) * 2 + F32IO, kq, LQ::kAlloc);
  if (rc) return rc;
  kq<<<p.B * p.Hq * p.n_tiles, 288, LQ::kAlloc, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
  prof_record(5, stream);
  return NEA_OK;
}

}  // namespace

extern "C" {

int nea_attn_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int T, int Hq, int Hkv,
                 int D, int dtype, float rope_base, int causal, void* stream_) {
  bool empty = false;
  int rc = check_shape(B, T, Hq, Hkv, D, dtype, causal, &empty);
  if (rc) return rc;
  if (empty) return NEA_OK;
  if (!Q || !K || !V || !O || !LSE) return NEA_ERR_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return NEA_ERR_ARG;
  if (!std::isfinite(rope_base)) return NEA_ERR_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  nea::FwdParams p{};
  if ((rc = rope_table(*st, T, D, rope_base, stream, &p.rope))) return rc;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.O = O;
  p.LSE = LSE;
  p.B = B;
  p.T = T;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_tiles = (T + 127) / 128;
  p.causal = causal;
  p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
  p.err = st->err;
  p.wait_limit = static_cast<unsigned long long>(t_wait_limit_ns);
  p.debug = t_debug_flags;
  t_debug_flags = 0;
  const bool f32 = dtype == NEA_F32;
  if (D == 64) return f32 ? launch_fwd<64, true>(*st, p, stream) : launch_fwd<64, false>(*st, p, stream);
  return f32 ? launch_fwd<32, true>(*st, p, stream) : launch_fwd<32, false>(*st, p, stream);
}

int nea_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const float* LSE, const void* dO,
                 void* dQ, void* dK, void* dV, int B, int T, int Hq, int Hkv, int D, int dtype, float rope_base,
                 int causal, void* stream_) {
  bool empty = false;
  int rc = check_shape(B, T, Hq, Hkv, D, dtype, causal, &empty);
  if (rc) return rc;
  if (empty) return NEA_OK;
  if (!Q || !K || !V || !O || !LSE || !dO || !dQ || !dK || !dV) return NEA_ERR_ARG;
  for (const void* ptr : {Q, K, V, O, static_cast<const void*>(LSE), dO, static_cast<const void*>(dQ),
                          static_cast<const void*>(dK), static_cast<const void*>(dV)})
    if (!aligned16(ptr)) return NEA_ERR_ARG;
  if (!std::isfinite(rope_base)) return NEA_ERR_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  nea::BwdParams p{};
  if ((rc = rope_table(*st, T, D, rope_base, stream, &p.rope))) return rc;
  if ((rc = ensure_dvec(*st, size_t(B) * Hq * T, stream))) return rc;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.dO = dO;
  p.LSE = LSE;
  p.Dv = st->dvec;
  p.dQ = dQ;
  p.dK = dK;
  p.dV = dV;
  p.B = B;
  p.T = T;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_tiles = (T + 127) / 128;
  p.causal = causal;
  p.scale = float(1.0 / std::sqrt(double(D)));
  p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
  p.err = st->err;
  p.wait_limit = static_cast<unsigned long long>(t_wait_limit_ns);
  const bool f32 = dtype == NEA_F32;
  if (D == 64) return f32 ? launch_bwd<64, true>(*st, p, O, stream) : launch_bwd<64, false>(*st, p, O, stream);
  return f32 ? launch_bwd<32, true>(*st, p, O, stream) : launch_bwd<32, false>(*st, p, O, stream);
}

int nea_device_status(void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  int v = 0;
  if ((e = cudaMemcpy(&v, st->err, sizeof v, cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(e);
  if (v != 0 && (e = cudaMemset(st->err, 0, sizeof(int))) != cudaSuccess) return cuda_fail(e);
  return v ? NEA_ERR_TIMEOUT : NEA_OK;
}

long long nea_set_wait_limit_ns(long long ns) {
  const long long prev = t_wait_limit_ns;
  t_wait_limit_ns = ns < 1000000LL ? 1000000LL : ns;
  return prev;
}

void nea_debug_inject(int flags) { t_debug_flags = flags; }

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
constexpr size_t kNoAllocStatusFloats = 64;                 // status word, padded to 256 bytes
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// Host-side state per device: the array's device address (the host-side name
// `g_noalloc_scratch` is only a stand-in and must never reach a kernel) and
// which kernel attributes are set.  Fixed-size, so no host allocation either.
struct NoAllocDevice {
  bool ready = false;
  bool sm100 = false;
  float* scratch = nullptr;
  uint32_t attr_done = 0;
};
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];
std::mutex g_noalloc_mu;

// Rotary table [T][D/2] of (cos, sin) of t * base^(-2i/D), angles in double.
__global__ void noalloc_rope_table_kernel(float2* out, int T, int D, double base) {
  const long idx = long(blockIdx.x) * blockDim.x + threadIdx.x;
  const int half = D / 2;
  if (idx >= long(T) * half) return;
  const int t = int(idx / half), i = int(idx % half);
  const double a = double(t) * pow(base, -2.0 * double(i) / double(D));
  double sn, cs;
  sincos(a, &sn, &cs);
  out[idx] = make_float2(float(cs), float(sn));
}

size_t round4(size_t n) { return (n + 3) & ~size_t(3); }

template <typename Kern>
int noalloc_smem(NoAllocDevice& st, int bit, Kern kern, uint32_t bytes) {
  if (st.attr_done & (1u << bit)) return NEA_OK;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  if (e != cudaSuccess) return cuda_fail(e);
  st.attr_done |= 1u << bit;
  return NEA_OK;
}

template <int D, bool F32IO>
int noalloc_launch(NoAllocDevice& st, const nea::BwdParams& p, const void* O, cudaStream_t stream) {
  const int rows = p.B * p.T * p.Hq;
  constexpr int kLanes = D / (F32IO ? 4 : 8);
  const long long threads = static_cast<long long>(rows) * kLanes;
  nea::attn_bwd_rowterm_kernel<D, F32IO>
      <<<unsigned((threads + 255) / 256), 256, 0, stream>>>(O, p.dO, const_cast<float*>(p.Dv), rows, p.T, p.Hq);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  using LK = nea::BwdSmem<D, F32IO, true>;
  auto kk = nea::attn_bwd_kernel<D, F32IO, true>;
  int rc = noalloc_smem(st, (D == 64) * 2 + F32IO, kk, LK::kAlloc);
  if (rc) return rc;
  kk<<<p.B * p.Hkv * p.n_tiles, 288, LK::kAlloc, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
  using LQ = nea::BwdSmem<D, F32IO, false>;
  auto kq = nea::attn_bwd_kernel<D, F32IO, false>;
  rc = noalloc_smem(st, 4 + (D == 64) * 2 + F32IO, kq, LQ::kAlloc);
  if (rc) return rc;
  kq<<<p.B * p.Hq * p.n_tiles, 288, LQ::kAlloc, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
  return NEA_OK;
}

}  // namespace

extern "C" int nea_attn_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const float* LSE,
                                    const void* dO, void* dQ, void* dK, void* dV, int B, int T, int Hq, int Hkv,
                                    int D, int dtype, float rope_base, int causal, void* stream_) {
  bool empty = false;
  int rc = check_shape(B, T, Hq, Hkv, D, dtype, causal, &empty);
  if (rc) return rc;
  if (empty) return NEA_OK;
  if (!Q || !K || !V || !O || !LSE || !dO || !dQ || !dK || !dV) return NEA_ERR_ARG;
  for (const void* ptr : {Q, K, V, O, static_cast<const void*>(LSE), dO, static_cast<const void*>(dQ),
                          static_cast<const void*>(dK), static_cast<const void*>(dV)})
    if (!aligned16(ptr)) return NEA_ERR_ARG;
  if (!std::isfinite(rope_base)) return NEA_ERR_ARG;
  const size_t dv_floats = round4(size_t(B) * Hq * T);
  const size_t rope_floats = (rope_base > 0.f) ? round4(size_t(T) * D) : 0;
  if (kNoAllocStatusFloats + dv_floats + rope_floats > kNoAllocScratchFloats) return NEA_ERR_SCRATCH_LIMIT;
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
      st.scratch = static_cast<float*>(ptr);
    }
    st.ready = true;
  }
  if (!st.sm100) return NEA_ERR_UNSUPPORTED;

  int* status = reinterpret_cast<int*>(st.scratch);
  float* dv = st.scratch + kNoAllocStatusFloats;
  float2* rope = rope_floats ? reinterpret_cast<float2*>(dv + dv_floats) : nullptr;
  // the status word must start at zero; Dv is fully rewritten by the row-term
  // kernel and the table by its own kernel, so neither needs clearing
  if ((e = cudaMemsetAsync(status, 0, sizeof(int), stream)) != cudaSuccess) return cuda_fail(e);
  if (rope) {
    const long n = long(T) * (D / 2);
    noalloc_rope_table_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(rope, T, D, double(rope_base));
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
  }
  nea::BwdParams p{};
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.dO = dO;
  p.LSE = LSE;
  p.Dv = dv;
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
  p.causal = causal;
  p.scale = float(1.0 / std::sqrt(double(D)));
  p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
  p.err = status;
  p.wait_limit = static_cast<unsigned long long>(t_wait_limit_ns);
  const bool f32 = dtype == NEA_F32;
  if (D == 64) return f32 ? noalloc_launch<64, true>(st, p, O, stream) : noalloc_launch<64, false>(st, p, O, stream);
  return f32 ? noalloc_launch<32, true>(st, p, O, stream) : noalloc_launch<32, false>(st, p, O, stream);
}
