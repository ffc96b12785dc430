// Decode attention over a key/value cache: one new query per sequence attends
// to the cached positions 0 .. len_b - 1, the last of which is its own (the
// generation path of the same causal attention: "NanoEuler" write-up,
// aimsg.uk, section 1, head-0 generation; scores, softmax and GQA head map
// as in the training path; RoPE on the query at its position, section 2
// "Model components").  The cache holds keys already rotated at their
// positions, so only the query is rotated here.
//
// The work is one pass over the cache, so it is bound by HBM bandwidth.  The
// cache [B][Tc][Hkv][D] is cut into pieces: R consecutive positions of HP
// neighbouring kv heads (a head group), so that each copy reads whole runs of
// HP D elements and every DRAM page is read in one go.  All pieces of the
// call, in (sequence, head group, position) order, are split into one
// contiguous range per CTA (one CTA per SM, ranges differing by at most one
// piece).  A CTA streams its range through a ring of shared-memory stages
// that one producer warp keeps filled with TMA copies, so the copies of the
// next pieces are in flight while eight consumer warps score the current one.
// With the first piece of each (sequence, head group) in the range the
// producer also copies the group's query rows and the rotary row of position
// len - 1, so the consumers never wait on a global load.
//
// Consumer warp w serves kv head w / WPH of the group (WPH = 8 / HP warps per
// head) and its own rows of each piece, and keeps its own online softmax
// (running max m, sum l and unnormalised output o, per query head) over
// them.  Where its range leaves a (sequence, head group), each warp writes
// its state as a partial (o, m, l) and goes on; no consumer waits for
// another.  A second kernel, launched behind the first with programmatic
// dependent launch (so it is resident when the first ends), merges the
// partials of each (sequence, kv head) with their log-sum-exp weights into O
// and LSE.
//
// Scoring, by storage type:
//   bfloat16: the G query heads of a kv head are the 16 rows of a warp-level
//     bf16 MMA (m16n8k16, fp32 accumulation; rows G..15 zero), the warp's 16
//     cached rows its columns: S = q' K^T in 8 MMAs per 16 rows (D = 64),
//     then O += P V in 8 more, with P rounded to bf16 as in the training
//     forward.  The arithmetic is small next to the bytes, so the MMA shape
//     is chosen for instruction count, not tensor throughput.
//   float32: CUDA-core fp32 (packed f32x2 FMA); TPR lanes share one cached
//     row, each holding 1/TPR of its columns and of the rotated queries, and
//     add their partial scores with TPR - 1 shuffles.
#pragma once

#include <cuda.h>

#include "nea_tiles.cuh"

namespace nea {

constexpr int kDecMaxG = 8;     // query heads per kv head
constexpr int kDecWarps = 8;    // consumer warps; one producer warp follows them
constexpr int kDecThreads = 32 * (kDecWarps + 1);
constexpr int kDecRingBytes = 200 * 1024;
constexpr int kDecQAux = 4096;  // per stage: the head group's query rows, then the rotary row (<= 256 B)
constexpr int kDecAux = 5120;
constexpr int kDecMaxSeg = 512; // ranges meeting one (sequence, head group): at most the CTAs + 1

// float32 path: lanes per cached row, the smallest power of two >= 2 that
// keeps a lane's share of the queries and outputs (2 G D / TPR floats) at
// most 96 registers while a lane keeps at least 8 columns.
__host__ __device__ constexpr int dec_tpr(int G, int D) {
  int t = 2;
  while (G * D / t > 48 && D / (2 * t) >= 8) t *= 2;
  return t;
}
// (row, kv head) lines per piece: bfloat16, 16 per consumer warp; float32,
// one per TPR lanes of every consumer warp.
__host__ __device__ constexpr int dec_lines(int G, int D, bool f32) {
  return f32 ? kDecWarps * 32 / dec_tpr(G, D) : kDecWarps * 16;
}
// kv heads per piece: the largest power of two <= 8 that divides Hkv and
// keeps the group's query rows (HP G D elements) within the aux area.
__host__ __device__ constexpr int dec_heads_per_piece(int Hkv, int G, int D, bool f32) {
  int hp = 8;
  while (hp > 1 && (Hkv % hp != 0 || hp * G * D * (f32 ? 4 : 2) > kDecQAux)) hp /= 2;
  return hp;
}

struct DecodeParams {
  CUtensorMap tm_k;    // Kc [B][Tc][Hkv][D] as (D, position, head, sequence), box {min(D, 128 B), R, HP, 1},
                       // 128- or 64-byte swizzle: line h R + r of a piece is position r of its head h
  CUtensorMap tm_v;    // Vc, same
  const void* Q;       // [B][Hq][D] un-rotated queries
  const int* lens;     // [B]
  void* O;             // [B][Hq][D]
  float* LSE;          // [B][Hq]
  float* part;         // [B*NHG*NP][warps][G][D + 2]: o, then m and l (base 2), at a range's first piece
  const float2* rope;  // [Tc][D/2] (cos, sin), nullptr: no rotation
  int B, Tc, Hq, Hkv, G;
  int HP, NHG, WPH;    // kv heads per piece, head groups (Hkv / HP), consumer warps per kv head (8 / HP)
  int R;               // positions per piece
  int NP;              // pieces per (sequence, head group) = ceil(Tc / R)
  int n_cta;           // CTAs of the grid
  unsigned long long n_pieces;  // B * NHG * NP
  float scale_log2;    // log2(e) / sqrt(D)
  int* err;
  unsigned long long wait_limit;
};

// First piece of CTA c's range (ranges tile [0, n_pieces) in CTA order).
__host__ __device__ __forceinline__ unsigned long long dec_range_lo(unsigned long long c, unsigned long long n,
                                                                     unsigned long long n_cta) {
  return c * n / n_cta;
}
// First CTA whose range ends after piece a: the least c with
// floor((c + 1) n / n_cta) > a, i.e. (c + 1) n >= (a + 1) n_cta.
__host__ __device__ __forceinline__ unsigned long long dec_first_cta(unsigned long long a, unsigned long long n,
                                                                      unsigned long long n_cta) {
  return ((a + 1) * n_cta + n - 1) / n - 1;
}

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

template <int D, bool F32IO, int G>
struct DecLayout {
  static constexpr int LP = dec_lines(G, D, F32IO);  // (row, kv head) lines per piece
  static constexpr int E = F32IO ? 4 : 2;            // element bytes
  static constexpr int RB = D * E < 128 ? D * E : 128;  // bytes per line of one copied array
  static constexpr int NA = D * E / RB;              // arrays per tensor (column halves for fp32, D = 64)
  static constexpr int EPA = RB / E;                 // elements per array line
  static constexpr uint32_t kArray = uint32_t(LP) * RB;
  static constexpr uint32_t kAuxOff = 2u * NA * kArray;  // K arrays, V arrays, then the aux rows
  static constexpr uint32_t kStage = kAuxOff + kDecAux;
  static constexpr int ST = kDecRingBytes / kStage < 8 ? kDecRingBytes / kStage : 8;
  static constexpr uint32_t kRing = 0;
  static constexpr uint32_t kBar = ST * kStage;      // full[ST], empty[ST]
  static constexpr uint32_t kFlag = kBar + 2 * ST * 8;  // abort flag
  static constexpr uint32_t kBytes = kFlag + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  // float32 path
  static constexpr int TPR = dec_tpr(G, D);
  static constexpr int RPW = 32 / TPR;               // lines per warp
  static constexpr int EPC = 16 / E;                 // elements per 16-byte chunk
  static constexpr int EPL = D / TPR;                // elements per lane
  static constexpr int CPL = EPL / EPC;              // chunks per lane
  static_assert(F32IO || LP == kDecWarps * 16, "bf16: 16 lines per warp");
  static_assert(!F32IO || (EPL % EPC == 0 && EPA % EPL == 0), "a lane's columns are whole chunks of one array");
  static_assert(kArray % 1024 == 0 && kStage % 1024 == 0, "arrays stay aligned to the swizzle atom");
  static_assert(kDecQAux + D / 2 * 8 <= kDecAux, "aux rows fit");
  static_assert(ST >= 2, "at least two stages");
};

// ------------------------------------------------------------ warp-level bf16 MMA
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// d += A B for A 16x16 (rows 8..15 zero: only a0, a2 given), B 16x8, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// A 4-D tile copy like tma_load_4d, with an L2 eviction policy: the cache is
// read once, so its lines are marked evict-first and do not push out what
// the call reads again (partials, queries, lengths).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void tma_load_4d_hint(void* dst, const void* tmap, int c0, int c1, int c2, int c3,
                                                 uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Partial of consumer warp `warp`, query head gi of its kv head, for the
// range of (sequence, head group) bhg that starts at piece k0.
__device__ __forceinline__ float* dec_partial(const DecodeParams& p, int bhg, int k0, int warp, int gi, int D) {
  return p.part + ((size_t(bhg) * p.NP + k0) * kDecWarps * p.G + size_t(warp) * p.G + gi) * (D + 2);
}

// Merge kernel: one CTA per (sequence, kv head).  O = sum w o / sum w l,
// w = 2^(m - M), M the largest m over the partials of all ranges of its
// head group (a range without cached rows wrote m = -inf and weighs 0);
// LSE = ln(2^M sum w l); no cached row: O = 0, LSE = -inf.
// NG groups of G D threads (one per output element, up to 1024 threads) each
// take every NG-th partial, eight at a time, so that the loads of many
// partials are in flight at once; the groups' (M, L, O) are then combined the
// same way.  The merge sits on the critical path behind the streaming
// kernel, so its loads are spread as wide as the CTA allows.
__host__ __device__ constexpr int dec_merge_groups(int G, int D) { return 1024 / (G * D) < 4 ? 1024 / (G * D) : 4; }
template <int D, bool F32IO, int G>
__global__ void __launch_bounds__(dec_merge_groups(G, D) * G * D) attn_decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int GD = G * D, NG = dec_merge_groups(G, D);
  __shared__ float red[NG][3][GD];   // per group: m, l, o of each element
  __shared__ int seg_r0[kDecMaxSeg];  // first piece of each range of (b, head group), relative to its first
  __shared__ int n_seg_s;
  const int bg = blockIdx.x, b = bg / p.Hkv, g = bg % p.Hkv;
  const int hg = g / p.HP, h = g % p.HP, bhg = b * p.NHG + hg;
  const int grp = threadIdx.x / GD, e = threadIdx.x % GD;
  const int gi = e / D, d = e % D;
  {  // the ranges of (b, hg): CTAs c_first .. c_last, one thread each
    const unsigned long long a = (unsigned long long)bhg * p.NP;
    const unsigned long long c_first = dec_first_cta(a, p.n_pieces, p.n_cta);
    const int n = int(dec_first_cta(a + p.NP - 1, p.n_pieces, p.n_cta) - c_first) + 1;
    for (int i = threadIdx.x; i < n && i < kDecMaxSeg; i += blockDim.x)
      seg_r0[i] = int(max(dec_range_lo(c_first + i, p.n_pieces, p.n_cta), a) - a);
    if (threadIdx.x == 0) n_seg_s = min(n, kDecMaxSeg);
  }
  __syncthreads();
  grid_dep_wait();  // the partials of the streaming kernel
  float mx = -INFINITY, ls = 0.f, o = 0.f;
  auto add = [&](float pm, float pl, float po) {
    if (pm == -INFINITY) return;  // no cached row behind this partial
    if (pm > mx) {
      const float f = ex2(mx - pm);  // 0 for the first
      ls *= f;
      o *= f;
      mx = pm;
    }
    const float wt = ex2(pm - mx);
    ls = fmaf(wt, pl, ls);
    o = fmaf(wt, po, o);
  };
  const int n_part = n_seg_s * p.WPH;  // the warps of kv head h in each range
  for (int q0 = grp; q0 < n_part; q0 += 8 * NG) {
    float pm[8], pl[8], po[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int qi = q0 + u * NG;
      pm[u] = -INFINITY, pl[u] = 0.f, po[u] = 0.f;
      if (qi < n_part) {
        const float* src = dec_partial(p, bhg, seg_r0[qi / p.WPH], h * p.WPH + qi % p.WPH, gi, D);
        pm[u] = src[D];
        pl[u] = src[D + 1];
        po[u] = src[d];
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) add(pm[u], pl[u], po[u]);
  }
  red[grp][0][e] = mx;
  red[grp][1][e] = ls;
  red[grp][2][e] = o;
  __syncthreads();
  if (grp != 0) return;
  mx = -INFINITY, ls = 0.f, o = 0.f;
#pragma unroll
  for (int k = 0; k < NG; ++k) add(red[k][0][e], red[k][1][e], red[k][2][e]);
  const size_t bh = size_t(b) * p.Hq + size_t(g) * G + gi;
  const float out = mx == -INFINITY ? 0.f : o / ls;
  if constexpr (F32IO) static_cast<float*>(p.O)[bh * D + d] = out;
  else static_cast<__nv_bfloat16*>(p.O)[bh * D + d] = __float2bfloat16_rn(out);
  // m and l are in base-2 units of the scaled scores
  if (d == 0) p.LSE[bh] = mx == -INFINITY ? -INFINITY : (mx + log2f(ls)) * 0.69314718055994531f;
}

// One rotated, pre-scaled query pair (columns 2i, 2i + 1 of query row qr of
// the head group) from the aux rows of a stage.
template <int D, bool F32IO>
__device__ __forceinline__ void dec_query_pair(const uint8_t* aux, bool rope, int qr, int i, float scale, float& x0,
                                               float& x1) {
  if constexpr (F32IO) {
    const float2 v = reinterpret_cast<const float2*>(aux)[qr * (D / 2) + i];
    x0 = v.x, x1 = v.y;
  } else {
    const uint32_t w = reinterpret_cast<const uint32_t*>(aux)[qr * (D / 2) + i];
    x0 = bf16_lo_f(w), x1 = bf16_hi_f(w);
  }
  if (rope) {
    const float2 cs = reinterpret_cast<const float2*>(aux + kDecQAux)[i];
    rot2(x0, x1, cs.x, cs.y);
  }
  x0 *= scale;
  x1 *= scale;
}

template <int D, bool F32IO, int G>
__global__ void __launch_bounds__(kDecThreads, 1) attn_decode_kernel(const __grid_constant__ DecodeParams p) {
  using L = DecLayout<D, F32IO, G>;
  extern __shared__ uint8_t raw[];
  uint8_t* sm = raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* empty = full + L::ST;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kFlag);
  const WaitCtl wc{p.err, p.wait_limit, abort_flag};
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (warp == kDecWarps && lane == 0) {
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
  }

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < L::ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecWarps);
    }
    mbar_init_fence();
  }
  __syncthreads();

  const unsigned long long lo = dec_range_lo(blockIdx.x, p.n_pieces, p.n_cta);
  const unsigned long long hi = dec_range_lo(blockIdx.x + 1ull, p.n_pieces, p.n_cta);
  grid_dep_launch();  // the merge kernel may take its place now; it waits for this grid's end

  // ---------------------------------------------------------------- producer
  if (warp == kDecWarps) {
    if (lane != 0) return;
    const uint32_t q_bytes = uint32_t(p.HP) * G * D * L::E;
    const uint64_t stream_policy = l2_evict_first_policy();
    uint32_t it = 0;
    bool ok = true;
    for (unsigned long long q = lo; q < hi && ok;) {
      const int bhg = int(q / p.NP), k0 = int(q % p.NP);
      const int k1 = int(min((unsigned long long)p.NP, (unsigned long long)k0 + (hi - q)));
      q += k1 - k0;
      const int b = bhg / p.NHG, hg = bhg % p.NHG;
      const int len = decode_len(p, b);
      const int kv = min(k1, (len + p.R - 1) / p.R);  // pieces holding cached rows
      for (int k = k0; k < kv; ++k, ++it) {
        const int s = it % L::ST;
        if (it >= uint32_t(L::ST) && !(ok = wait_thread(&empty[s], ((it / L::ST) - 1) & 1, wc, kErrWaitEmpty)))
          break;
        uint8_t* st = sm + L::kRing + s * L::kStage;
        const bool first = k == k0;
        const uint32_t aux = first ? q_bytes + (p.rope ? D / 2 * 8 : 0) : 0;
        mbar_arrive_expect_tx(&full[s], L::kAuxOff + aux);
#pragma unroll
        for (int a = 0; a < L::NA; ++a) {
          tma_load_4d_hint(st + a * L::kArray, &p.tm_k, a * L::EPA, k * p.R, hg * p.HP, b, &full[s], stream_policy);
          tma_load_4d_hint(st + (L::NA + a) * L::kArray, &p.tm_v, a * L::EPA, k * p.R, hg * p.HP, b, &full[s],
                           stream_policy);
        }
        if (first) {  // the head group's query rows and the rotary row of position len - 1
          bulk_load(st + L::kAuxOff,
                    static_cast<const uint8_t*>(p.Q) + (size_t(b) * p.Hq + size_t(hg) * p.HP * G) * D * L::E, q_bytes,
                    &full[s]);
          if (p.rope) bulk_load(st + L::kAuxOff + kDecQAux, p.rope + size_t(len - 1) * (D / 2), D / 2 * 8, &full[s]);
        }
      }
    }
    // never exit with copies in flight: the last stages issued have landed
    for (uint32_t i = it > uint32_t(L::ST) ? it - L::ST : 0; i < it; ++i)
      drain_wait(&full[i % L::ST], (i / L::ST) & 1, wc);
    return;
  }

  // ---------------------------------------------------------------- consumers
  const bool rope = p.rope != nullptr;
  const int hh = warp / p.WPH, rb = warp % p.WPH;  // kv head of the group, row block of the piece
  uint32_t it = 0;
  bool ok = true;
  for (unsigned long long q = lo; q < hi;) {
    const int bhg = int(q / p.NP), k0 = int(q % p.NP);
    const int k1 = int(min((unsigned long long)p.NP, (unsigned long long)k0 + (hi - q)));
    q += k1 - k0;
    const int len = decode_len(p, bhg / p.NHG);
    const int kv = min(k1, (len + p.R - 1) / p.R);
    if (kv <= k0) {  // no cached row in this range: an empty partial (the merge reads every range's)
      if (lane < G) dec_partial(p, bhg, k0, warp, lane, D)[D] = -INFINITY;
    } else {  // this range holds cached rows of (b, hg)
      if constexpr (!F32IO) {
        // ---- bf16: rows 16 rb .. 16 rb + 15 of each piece, kv head hh;
        // lane (gr, t) holds query head gr (rows gr + 8 of the MMA are zero)
        // and cached rows 2t, 2t + 1 of each 8-row column block
        const int gr = lane >> 2, t = lane & 3;
        constexpr int KS = D / 16;  // k-steps over the head dimension
        uint32_t qa[KS][2];         // A fragments of q' (rows gr), columns 16 ks + 2t (+8)
        float o[D / 8][4];          // O fragments: rows gr (o[.][0..1]) and gr + 8 (zero)
        float m = -INFINITY, l = 0.f;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        // ldmatrix line addresses (line = kv head R + row, so the 8 rows of
        // a matrix take 8 different swizzle phases): K (non-transposed) per
        // 8-row block nt and 32-column block h; V (transposed) per pair of
        // 8-column blocks.  Columns past a line of one array (D = 128: 64
        // per array) sit in the next array, kArray on.
        const int line0 = hh * p.R + 16 * rb;
        constexpr int HPA = L::EPA / 32;  // 32-column blocks per array
        uint32_t koff[2][D / 32], voff[D / 16];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int h = 0; h < D / 32; ++h)
            koff[nt][h] = (h / HPA) * L::kArray +
                          swizzle(uint32_t(line0 + 8 * nt + (lane & 7)) * L::RB + (4 * (h % HPA) + (lane >> 3)) * 16,
                                  L::RB);
#pragma unroll
        for (int jj = 0; jj < D / 16; ++jj)
          voff[jj] = (jj / (2 * HPA)) * L::kArray +
                     swizzle(uint32_t(line0 + 8 * ((lane >> 3) & 1) + (lane & 7)) * L::RB +
                                 (2 * (jj % (2 * HPA)) + (lane >> 4)) * 16,
                             L::RB);
        for (int k = k0; k < kv; ++k, ++it) {
          const int s = it % L::ST;
          ok = ok && wait_warp(&full[s], (it / L::ST) & 1, wc, kErrWaitProducer);
          if (ok) {
            const uint8_t* st = sm + L::kRing + s * L::kStage;
            if (k == k0) {  // queries of kv head hh, from the aux rows of the range's first piece
#pragma unroll
              for (int ks = 0; ks < KS; ++ks)
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                  float x0 = 0.f, x1 = 0.f;
                  if (gr < G)
                    dec_query_pair<D, false>(st + L::kAuxOff, rope, hh * G + gr, 8 * ks + t + 4 * h2, p.scale_log2,
                                             x0, x1);
                  qa[ks][h2] = pack_bf16(x0, x1);
                }
            }
            const uint32_t kb = smem_u32(st), vb = smem_u32(st + L::NA * L::kArray);
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int h = 0; h < D / 32; ++h) {
                uint32_t r[4];
                ldsm_x4(kb + koff[nt][h], r);
                mma_bf16_16816(sc[nt], qa[2 * h][0], qa[2 * h][1], r[0], r[1]);
                mma_bf16_16816(sc[nt], qa[2 * h + 1][0], qa[2 * h + 1][1], r[2], r[3]);
              }
            // scores of head gr for cached rows j0 + {0, 1, 8, 9}; rows past
            // the cache length take no part
            const int j0 = k * p.R + 16 * rb + 2 * t;
            float v[4] = {sc[0][0], sc[0][1], sc[1][0], sc[1][1]};
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (j0 + 8 * (i >> 1) + (i & 1) >= len) v[i] = -INFINITY;
            float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
            mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 2));
            if (__any_sync(kFullMask, mx > m)) {  // a new running max: rescale (the first scales zeros)
              const float f = mx > m ? ex2(m - mx) : 1.f;
              l *= f;
#pragma unroll
              for (int j = 0; j < D / 8; ++j) o[j][0] *= f, o[j][1] *= f;
              m = fmaxf(m, mx);
            }
            const float mb = m == -INFINITY ? 0.f : m;
            float pw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) pw[i] = ex2(v[i] - mb);
            l += (pw[0] + pw[1]) + (pw[2] + pw[3]);
            const uint32_t pa0 = pack_bf16(pw[0], pw[1]), pa2 = pack_bf16(pw[2], pw[3]);
#pragma unroll
            for (int jj = 0; jj < D / 16; ++jj) {
              uint32_t r[4];
              ldsm_x4_trans(vb + voff[jj], r);
              mma_bf16_16816(o[2 * jj], pa0, pa2, r[0], r[1]);
              mma_bf16_16816(o[2 * jj + 1], pa0, pa2, r[2], r[3]);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
        }
        // ---- the warp's partial: l summed over the quad; O row gr is
        // spread over the quad's lanes, two columns per 8-column block
        l += __shfl_xor_sync(kFullMask, l, 1);
        l += __shfl_xor_sync(kFullMask, l, 2);
        if (gr < G) {
          float* dst = dec_partial(p, bhg, k0, warp, gr, D);
#pragma unroll
          for (int j = 0; j < D / 8; ++j) *reinterpret_cast<float2*>(dst + 8 * j + 2 * t) = make_float2(o[j][0], o[j][1]);
          if (t == 0) {
            dst[D] = m;
            dst[D + 1] = l;
          }
        }
      } else {
        // ---- fp32: lane (part, rw) holds columns [part EPL, part EPL + EPL)
        // of row RPW rb + rw of each piece, kv head hh
        constexpr int NP2 = L::EPL / 2;  // packed pairs per lane
        const int part = lane / L::RPW, rw = lane % L::RPW;
        const int row = rb * L::RPW + rw;
        const int col0 = part * L::EPL;
        const int arr = col0 / L::EPA, c0 = (col0 % L::EPA) / L::EPC;
        uint32_t coff[L::CPL];
#pragma unroll
        for (int c = 0; c < L::CPL; ++c)
          coff[c] = swizzle(uint32_t(hh * p.R + row) * L::RB + (c0 + c) * 16, L::RB);
        uint64_t q2[G][NP2], o2[G][NP2];
        float m[G], l[G];
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
#pragma unroll
          for (int e = 0; e < NP2; ++e) o2[gi][e] = 0;  // the bit pattern of (+0, +0)
          m[gi] = -INFINITY;
          l[gi] = 0.f;
        }
        for (int k = k0; k < kv; ++k, ++it) {
          const int s = it % L::ST;
          ok = ok && wait_warp(&full[s], (it / L::ST) & 1, wc, kErrWaitProducer);
          if (ok) {
            const uint8_t* st = sm + L::kRing + s * L::kStage;
            if (k == k0) {
#pragma unroll
              for (int gi = 0; gi < G; ++gi)
#pragma unroll
                for (int e = 0; e < NP2; ++e) {
                  float x0, x1;
                  dec_query_pair<D, true>(st + L::kAuxOff, rope, hh * G + gi, col0 / 2 + e, p.scale_log2, x0, x1);
                  q2[gi][e] = f2_pack(x0, x1);
                }
            }
            const uint8_t* ka = st + arr * L::kArray;
            uint64_t x[NP2];
#pragma unroll
            for (int c = 0; c < L::CPL; ++c) {
              const float4 u = *reinterpret_cast<const float4*>(ka + coff[c]);
              x[2 * c] = f2_pack(u.x, u.y);
              x[2 * c + 1] = f2_pack(u.z, u.w);
            }
            float sc[G];
#pragma unroll
            for (int gi = 0; gi < G; ++gi) {  // two accumulators per head halve the dependent chain
              uint64_t a0 = f2_mul(q2[gi][0], x[0]), a1 = f2_mul(q2[gi][1], x[1]);
#pragma unroll
              for (int e = 2; e < NP2; e += 2) {
                a0 = f2_fma(q2[gi][e], x[e], a0);
                a1 = f2_fma(q2[gi][e + 1], x[e + 1], a1);
              }
              float u0, u1;
              f2_unpack(f2_add(a0, a1), u0, u1);
              sc[gi] = u0 + u1;
            }
            // complete scores: the TPR lanes of the row add their shares (the
            // same sums in every lane: addition is commutative)
#pragma unroll
            for (int off = L::RPW; off < 32; off <<= 1)
#pragma unroll
              for (int gi = 0; gi < G; ++gi) sc[gi] += __shfl_xor_sync(kFullMask, sc[gi], off);
            if (k * p.R + row < len) {  // rows past the cache length take no part
              const uint8_t* va = st + (L::NA + arr) * L::kArray;
#pragma unroll
              for (int c = 0; c < L::CPL; ++c) {
                const float4 u = *reinterpret_cast<const float4*>(va + coff[c]);
                x[2 * c] = f2_pack(u.x, u.y);
                x[2 * c + 1] = f2_pack(u.z, u.w);
              }
#pragma unroll
              for (int gi = 0; gi < G; ++gi) {
                if (sc[gi] > m[gi]) {  // new running max: rescale (the first row scales zeros)
                  const float f = ex2(m[gi] - sc[gi]);
                  const uint64_t f2 = f2_pack(f, f);
                  l[gi] *= f;
#pragma unroll
                  for (int e = 0; e < NP2; ++e) o2[gi][e] = f2_mul(o2[gi][e], f2);
                  m[gi] = sc[gi];
                }
                const float pw = ex2(sc[gi] - m[gi]);
                l[gi] += pw;
                const uint64_t p2 = f2_pack(pw, pw);
#pragma unroll
                for (int e = 0; e < NP2; ++e) o2[gi][e] = f2_fma(p2, x[e], o2[gi][e]);
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
        }
        // ---- the warp's partial: its rows' states rescaled to the warp max
        // and summed; lanes of row 0 write their columns
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
          float mx = m[gi];
#pragma unroll
          for (int off = 1; off < L::RPW; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, off));
          const float f = m[gi] == -INFINITY ? 0.f : ex2(m[gi] - mx);
          const uint64_t f2 = f2_pack(f, f);
          l[gi] *= f;
#pragma unroll
          for (int e = 0; e < NP2; ++e) o2[gi][e] = f2_mul(o2[gi][e], f2);
#pragma unroll
          for (int off = 1; off < L::RPW; off <<= 1) {
            l[gi] += __shfl_xor_sync(kFullMask, l[gi], off);
#pragma unroll
            for (int e = 0; e < NP2; ++e) {
              float u0, u1;
              f2_unpack(o2[gi][e], u0, u1);
              o2[gi][e] = f2_add(o2[gi][e], f2_pack(__shfl_xor_sync(kFullMask, u0, off),
                                                    __shfl_xor_sync(kFullMask, u1, off)));
            }
          }
          if (rw == 0) {
            float* dst = dec_partial(p, bhg, k0, warp, gi, D);
#pragma unroll
            for (int e = 0; e < NP2; ++e) {
              float u0, u1;
              f2_unpack(o2[gi][e], u0, u1);
              *reinterpret_cast<float2*>(dst + col0 + 2 * e) = make_float2(u0, u1);
            }
            if (part == 0) {
              dst[D] = mx;
              dst[D + 1] = l[gi];
            }
          }
        }
      }
    }
  }
}

}  // namespace nea
