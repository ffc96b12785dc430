// Device-side building blocks for the sm_100a attention kernels: mbarriers
// with bounded waits, tensor-memory (TMEM) allocation and access, tcgen05 MMA
// issue, UMMA shared-memory / instruction descriptors, and the swizzled
// shared-memory operand layout those descriptors describe.
//
// Everything here is written against the public PTX ISA for sm_100a
// (tcgen05.*, mbarrier.*).  Operand tiles are bf16, one row of a [rows][D]
// tile per 2*D bytes, stored with the hardware swizzle whose atom width equals
// the row (128 B for D = 64, 64 B for D = 32); the same bytes serve as a
// K-major operand (contraction over D) and as an MN-major operand
// (contraction over rows).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

// Phase stamps for performance analysis: compiled only with -DNEA_TRACE, when
// `p.trace` receives per CTA 80 %globaltimer values (slot 79: SM id).
#ifdef NEA_TRACE
#define NEA_TRACE_STAMP(p, slot, cond)                                                  \
  do {                                                                                  \
    if ((p).trace && (cond)) {                                                          \
      (p).trace[size_t(blockIdx.x) * 80 + (slot)] = nea::global_timer_ns();             \
      if ((slot) == 0) {                                                                \
        unsigned smid_;                                                                 \
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid_));                              \
        (p).trace[size_t(blockIdx.x) * 80 + 79] = smid_;                                \
      }                                                                                 \
    }                                                                                   \
  } while (0)
#else
#define NEA_TRACE_STAMP(p, slot, cond) \
  do {                                 \
  } while (0)
#endif

namespace nea {

constexpr uint32_t kFullMask = 0xffffffffu;

// ------------------------------------------------------------------ status
// Device error codes written (first writer wins) into the library's error
// word; the host maps any nonzero value to NEA_ERR_TIMEOUT.
enum : int {
  kErrNone = 0,
  kErrWaitProducer = 0x100,  // a consumer gave up waiting for loaded tiles
  kErrWaitMma = 0x200,       // a consumer gave up waiting for an MMA commit
  kErrWaitSoftmax = 0x300,   // the MMA issuer gave up waiting for P / dS
  kErrWaitEmpty = 0x400,     // the producer gave up waiting for a free stage
  kErrBadLength = 0x800,     // a decode cache length outside [0, Tc] (clamped)
};

struct WaitCtl {
  int* err;                  // global error word
  unsigned long long limit;  // per-wait limit, nanoseconds of %globaltimer
  volatile int* abort;       // shared-memory abort flag of this CTA
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async proxy (tcgen05.commit).
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void raise_error(const WaitCtl& c, int code) {
  atomicCAS(c.err, 0, code);
  *c.abort = 1;
}

// Wait of a single thread for the phase of `bar` with the given parity to
// complete.  Returns false, after recording `code`, once the CTA aborted or
// the wait exceeded its limit.
static __device__ __noinline__ bool wait_thread_slow(uint64_t* bar, uint32_t parity, const WaitCtl& c, int code) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*c.abort) return false;
    if (global_timer_ns() - t0 > c.limit) {
      raise_error(c, code);
      return false;
    }
  }
}

// Same wait, taken by all 32 lanes of a warp with a warp-uniform outcome, so
// that warp-collective tcgen05 loads/stores after it stay converged.  Every
// lane performs its own successful try_wait (acquire) before proceeding.
static __device__ __noinline__ bool wait_warp_slow(uint64_t* bar, uint32_t parity, const WaitCtl& c, int code) {
  bool done = false;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    done = done || mbar_try_wait(bar, parity);
    if (__all_sync(kFullMask, done)) return true;
    const bool quit = (*c.abort != 0) || (global_timer_ns() - t0 > c.limit);
    if (__any_sync(kFullMask, quit)) {
      if ((threadIdx.x & 31) == 0 && *c.abort == 0) raise_error(c, code);
      __syncwarp();
      return false;
    }
  }
}

// The waits proper: a first test inline (no call, so nothing is saved around
// it when the phase is already complete), the bounded loop out of line.
__device__ __forceinline__ bool wait_thread(uint64_t* bar, uint32_t parity, const WaitCtl& c, int code) {
  return mbar_try_wait(bar, parity) || wait_thread_slow(bar, parity, c, code);
}
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, const WaitCtl& c, int code) {
  return __all_sync(kFullMask, mbar_try_wait(bar, parity)) || wait_warp_slow(bar, parity, c, code);
}

// Wait that ignores the CTA's abort flag (still bounded by the limit, records
// nothing): used before exit so that no copy or MMA is left in flight.
static __device__ __noinline__ bool drain_wait(uint64_t* bar, uint32_t parity, const WaitCtl& c) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_timer_ns() - t0 > c.limit) return false;
  return true;
}

// Barrier `id` (1..15; 0 is __syncthreads) over `count` threads, a multiple of 32.
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Arms `bar` for `bytes` of asynchronous copies and arrives once.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// ------------------------------------------------------------------ TMA
// Tiled 4-D tensor copy global -> shared (coordinates innermost first); the
// bytes land with complete_tx on `bar`.  Out-of-range elements read as zero.
__device__ __forceinline__ void tma_load_4d(void* dst, const void* tmap, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// Contiguous bulk copy global -> shared; 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ------------------------------------------------------------------ programmatic dependent launch
// A grid launched with programmatic stream serialization may start while the
// previous grid in its stream still runs.  grid_dep_wait() returns once every
// grid it depends on has completed and its memory writes are visible (at once
// for an ordinary launch); every block calls it before its first global
// access.  grid_dep_launch() lets the next such grid start its launch once
// every block of this one has called it or exited.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ proxies
// Generic-proxy shared-memory writes -> visible to tcgen05.mma operand reads.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrives on `bar` once every tcgen05 operation this thread issued so far has
// completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// TMEM address of (lane, column).
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

#define NEA_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                  "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define NEA_W8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                  "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// Loads 32 consecutive 32-bit columns of this thread's lane (warp-collective,
// 32x32b shape: lane = warp's quarter base + lane id) and waits for them.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : NEA_R8(0), NEA_R8(8), NEA_R8(16), NEA_R8(24)
      : "r"(taddr)
      : "memory");
}

// 64 consecutive columns in one load (one wait instead of two).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : NEA_R8(0), NEA_R8(8), NEA_R8(16), NEA_R8(24), NEA_R8(32), NEA_R8(40), NEA_R8(48), NEA_R8(56)
      : "r"(taddr)
      : "memory");
}

// 128 consecutive columns (a whole 128-wide score row) in one load.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,"
      "%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,"
      "%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
      "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : NEA_R8(0), NEA_R8(8), NEA_R8(16), NEA_R8(24), NEA_R8(32), NEA_R8(40), NEA_R8(48), NEA_R8(56),
        NEA_R8(64), NEA_R8(72), NEA_R8(80), NEA_R8(88), NEA_R8(96), NEA_R8(104), NEA_R8(112), NEA_R8(120)
      : "r"(taddr)
      : "memory");
}

// Two runs of 64 columns (at taddr0 into r[0..63], at taddr1 into
// r[64..127]) with one wait.
__device__ __forceinline__ void tmem_ld64x2(uint32_t taddr0, uint32_t taddr1, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%128];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,"
      "%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
      "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%129];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : NEA_R8(0), NEA_R8(8), NEA_R8(16), NEA_R8(24), NEA_R8(32), NEA_R8(40), NEA_R8(48), NEA_R8(56),
        NEA_R8(64), NEA_R8(72), NEA_R8(80), NEA_R8(88), NEA_R8(96), NEA_R8(104), NEA_R8(112), NEA_R8(120)
      : "r"(taddr0), "r"(taddr1)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : NEA_R8(0), NEA_R8(8)
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : NEA_R8(0)
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
      ::"r"(taddr), NEA_W8(0), NEA_W8(8), NEA_W8(16), NEA_W8(24)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n"
      ::"r"(taddr), NEA_W8(0), NEA_W8(8)
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

#undef NEA_R8
#undef NEA_W8

// ------------------------------------------------------------------ UMMA
// Instruction descriptor, kind::f16 with bf16 A and B, fp32 accumulator.
// a_mn / b_mn select MN-major (1) instead of K-major (0) operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                        // D format: f32
         | (1u << 7)                      // A format: bf16
         | (1u << 10)                     // B format: bf16
         | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory descriptor of a swizzled operand whose rows are `row_bytes`
// (64 or 128) wide, i.e. exactly one swizzle atom: 8 rows form an atom of
// 8*row_bytes bytes.  For a K-major operand the leading offset is unused
// (encoded 16 B); for an MN-major operand it is the distance between
// consecutive atom columns along MN, which these tiles never have.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t row_bytes, uint32_t lbo_bytes) {
  const uint64_t layout = (row_bytes == 128) ? 2ull : 4ull;  // SWIZZLE_128B : SWIZZLE_64B
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFF);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= uint64_t(((8 * row_bytes) >> 4) & 0x3FFF) << 32;  // stride between 8-row groups
  d |= 1ull << 46;                                        // descriptor version (sm_100)
  d |= layout << 61;
  return d;
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Byte offset, inside a 1024-aligned tile, of logical offset `off` under the
// swizzle whose atom row is `row_bytes` wide (XOR of the 16-byte chunk index
// with the row index inside the atom, as the hardware addresses it).
__host__ __device__ __forceinline__ uint32_t swizzle(uint32_t off, uint32_t row_bytes) {
  return row_bytes == 128 ? (off ^ (((off >> 7) & 7u) << 4)) : (off ^ (((off >> 7) & 3u) << 4));
}

// ------------------------------------------------------------------ numerics
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------- integer division
// Division of 32-bit unsigned n by an invariant divisor d >= 1 with one
// multiply-high, an add and two shifts (Granlund and Montgomery, "Division by
// invariant integers using multiplication", PLDI 1994: with l = ceil(log2 d),
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (t + ((n - t) >> 1)) >> (l - 1)
// where t = mulhi(m, n), for every n < 2^32).
struct FastDiv {
  uint32_t d, m, l;
};
__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while (l < 32 && (uint64_t(1) << l) < d) ++l;
  const uint32_t m = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d + 1);
  return FastDiv{d, m, l};
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  if (f.l == 0) return n;  // d == 1
  const uint32_t t = __umulhi(f.m, n);
  return (t + ((n - t) >> 1)) >> (f.l - 1);
}

// ------------------------------------------------------- packed fp32 pairs
// sm_100 executes two fp32 lanes per instruction (add/mul/fma .f32x2, each
// lane rounded to nearest even like its scalar form); a pair travels in one
// 64-bit register.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^x for a pair of floats on the FMA pipe, leaving the exponential unit
// free: x = j + f with j the nearest integer (adding and subtracting
// 1.5 * 2^23 rounds to it), 2^f from the degree-3 polynomial that
// exp2_poly_fit.py derives (relative error below 7.5e-5 for f in
// [-1/2, 1/2]), and 2^j added to the exponent field.  Inputs below -125
// (-inf included) give 0, as the exponential unit's flush-to-zero form does;
// a NaN input gives NaN.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  const uint64_t xc = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t magic = f2_pack(12582912.f, 12582912.f);
  const uint64_t y = f2_add(xc, magic);
  const uint64_t f = f2_sub(xc, f2_sub(y, magic));
  uint64_t p = f2_fma(f, f2_pack(0.05517132207751274f, 0.05517132207751274f),
                      f2_pack(0.24261054396629333f, 0.24261054396629333f));
  p = f2_fma(p, f, f2_pack(0.6932609677314758f, 0.6932609677314758f));
  p = f2_fma(p, f, f2_pack(0.9999281167984009f, 0.9999281167984009f));
  float y0, y1, p0, p1;
  f2_unpack(y, y0, y1);
  f2_unpack(p, p0, p1);
  // the low bits of y hold j; shifted into the exponent field (the bits of
  // 1.5 * 2^23 shift out of the word)
  const float r0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(y0) << 23));
  const float r1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(y1) << 23));
  // below the clamp: 0; NaN (every comparison false): the input itself
  return f2_pack(x0 >= -125.f ? r0 : (x0 < -125.f ? 0.f : x0), x1 >= -125.f ? r1 : (x1 < -125.f ? 0.f : x1));
}

// Maximum of three floats in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of a 128-column score row held as raw bits: a three-input tree
// (depth 6) instead of a 128-long dependent chain.
__device__ __forceinline__ float row_max128(const uint32_t (&s)[128]) {
  float a[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    a[k] = fmax3(__uint_as_float(s[k]), __uint_as_float(s[k + 16]), __uint_as_float(s[k + 32]));
    a[k] = fmax3(a[k], __uint_as_float(s[k + 48]), __uint_as_float(s[k + 64]));
    a[k] = fmax3(a[k], __uint_as_float(s[k + 80]), __uint_as_float(s[k + 96]));
    a[k] = fmaxf(a[k], __uint_as_float(s[k + 112]));
  }
  const float b0 = fmax3(a[0], a[1], a[2]), b1 = fmax3(a[3], a[4], a[5]), b2 = fmax3(a[6], a[7], a[8]);
  const float b3 = fmax3(a[9], a[10], a[11]), b4 = fmax3(a[12], a[13], a[14]);
  return fmax3(fmax3(b0, b1, b2), fmax3(b3, b4, a[15]), -INFINITY);
}

// Packs two floats into bf16x2 (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo_f(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Splits (a, b) into bf16 high parts and bf16 residuals so that
// a ~= hi.lo + lo.lo and b ~= hi.hi + lo.hi to about 2^-17 relative.
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(a, b);
  lo = pack_bf16(a - bf16_lo_f(hi), b - bf16_hi_f(hi));
}

}  // namespace nea
