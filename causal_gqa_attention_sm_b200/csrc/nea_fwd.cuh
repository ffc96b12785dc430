// Forward kernel: tiled causal GQA attention with RoPE on the tcgen05 tensor
// cores ("NanoEuler" write-up, aimsg.uk, section 4 "GPU version": tiled
// FlashAttention with an online softmax, the T x T matrix never resident;
// the pages' own kernel stages K/V tiles in shared memory and loops over them
// per query block -- smartinfralog.com post, "Tiled FlashAttention" section).
//
// One CTA computes two adjacent 128-row query tiles (A = 2m, B = 2m + 1) of
// one (batch, query head); both read the same key/value tiles, so every K/V
// tile is loaded (and rotated) once per pair.
//
// Operands.  An operand prologue (nea_prep.cuh) applies the rotary embedding
// to Q and K once, before this kernel: bf16 storage gets rotated bf16 copies
// (V is read in place), float32 storage gets bf16 hi/lo planes of Q, K, V.
// TMA lands every tile already in the swizzled tensor-core layout; for
// float32 storage it lands the hi and lo halves of each tile and every product
// is formed from three bf16 products (hi*hi + hi*lo + lo*hi).
//
// Warps:
//   0-3, 4-7   softmax of tile A, of tile B: thread r owns row r (TMEM lane
//              r) and loads its whole 128-column score row with one TMEM
//              load; the row max comes from a three-input max tree, then
//              P = exp(s - m) is written as bf16, with paired fp32
//              arithmetic; the running max m moves only when it grows by more
//              than 2^8 (O rescaled in TMEM then); the epilogue writes O / l
//              and LSE.
//   8, 9       MMA issuers, one thread each: warp 8 for tile A, warp 9 for
//              tile B.  bfloat16 storage: S_X(j+1) as soon as the softmax
//              holds S_X(j) in registers, so it runs under the exponentials
//              of step j; then PV_X(j).  float32 storage (S_X(j+1) must wait
//              for PV_X(j), which reads P over S): PV_X(j), then S_X(j+1),
//              and tile B starts only once tile A has written its first P, so
//              B runs about half a step behind A and each tile's softmax
//              overlaps the other tile's products (started together, the two
//              tiles stay in step and share the exponential unit).
//   10         TMA: query tiles, then K and V tiles into two rings (K stages
//              free as soon as S is computed, V stages after PV).
// TMEM per tile X: S [256X, 256X+128), O [256X+128, +D), and
//   bf16 storage: P [256X+192, +64) in its own columns, so S_X(j+1) is issued
//     as soon as the softmax has loaded S_X(j) and runs under its exponentials;
//   float32 storage: P hi over S [256X, +64), P lo [256X+192, +64) (hi and lo
//     need the room), so S_X(j+1) waits until PV_X(j) has read P.
// Causal tiles above the diagonal are never visited; only the diagonal tile
// and a ragged last tile are masked.
#pragma once

#include <cuda.h>

#include "nea_tiles.cuh"

namespace nea {

struct FwdParams {
  // bf16 storage: rotated Q, K (or the inputs when the rotation is off) and
  // V.  float32 storage: the hi planes.
  CUtensorMap tm_q;  // [B][T][Hq][D], box {D, 1, 128, 1}
  CUtensorMap tm_k;  // [B][T][Hkv][D]
  CUtensorMap tm_v;
  // float32 storage: the lo planes
  CUtensorMap tm_q_lo;
  CUtensorMap tm_k_lo;
  CUtensorMap tm_v_lo;
  void* O;
  float* LSE;
  int B, T, Hq, Hkv, G;
  int n_tiles;         // ceil(T / 128)
  int n_pairs;         // ceil(n_tiles / 2)
  int causal;
  float scale_log2;    // log2(e) / sqrt(D)
  int* err;
  unsigned long long wait_limit;
  int debug;
  unsigned long long* trace;  // per-CTA phase stamps (NEA_TRACE builds only)
};

template <int D, bool F32IO>
struct FwdSmem {
  // K and V ring stages (D = 128, bf16 only: 32 KB tiles, two of each)
  static constexpr int kNK = F32IO ? 3 : (D == 128 ? 2 : 4);
  static constexpr int kNV = F32IO ? 2 : (D == 128 ? 2 : 3);
  static constexpr uint32_t kTile = Stage<D, F32IO>::kBytes;  // one tile: hi (+ lo)
  static constexpr uint32_t kQA = 0;
  static constexpr uint32_t kQB = kTile;
  static constexpr uint32_t kK0 = 2 * kTile;
  static constexpr uint32_t kKStage = kTile;
  static constexpr uint32_t kV0 = kK0 + kNK * kKStage;
  static constexpr uint32_t kVStage = kTile;
  static constexpr uint32_t kBars = kV0 + kNV * kVStage;
  // qtma, K tma/empty, V tma/empty, s[2], p[2], o[2], fin[2], sread[2]
  static constexpr int kNumBars = 1 + 2 * kNK + 2 * kNV + 10;
  static constexpr uint32_t kMisc = kBars + 8 * kNumBars;
  static constexpr uint32_t kUsed = kMisc + 16;
  // +1024 for manual alignment; at least 116 KB so two CTAs never share an SM
  // (each takes all 512 TMEM columns)
  static constexpr uint32_t kAlloc = kUsed + 1024 > 116u * 1024u ? kUsed + 1024 : 116u * 1024u;
  // 11 warps: up to 184 registers per thread, room for a whole score row
  static constexpr int kThreads = 352;
  static_assert(kK0 % 1024 == 0 && kKStage % 1024 == 0 && kV0 % 1024 == 0 && kVStage % 1024 == 0,
                "operand tiles need 1024-byte alignment");
  static_assert(kAlloc <= 232448, "shared memory");
};

template <int D, bool F32IO>
__global__ void __launch_bounds__(FwdSmem<D, F32IO>::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ FwdParams p) {
  using L = FwdSmem<D, F32IO>;
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  constexpr uint32_t OPB = TileGeom<D>::kOpBytes;
  constexpr int NK = L::kNK, NV = L::kNV;
  constexpr int kTerms = F32IO ? 3 : 1;
  // P in its own TMEM columns; float32 storage (P hi over S, lo apart) and
  // D = 128 (O takes the columns P would) write P over S
  constexpr bool kSepP = !F32IO && D <= 64;
  static_assert(D <= 64 || !F32IO, "D = 128 runs with bfloat16 storage");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_qtma = bars + 0;
  uint64_t* bar_ktma = bars + 1;                        // [NK]
  uint64_t* bar_kempty = bars + 1 + NK;                 // [NK]
  uint64_t* bar_vtma = bars + 1 + 2 * NK;               // [NV]
  uint64_t* bar_vempty = bars + 1 + 2 * NK + NV;        // [NV]
  uint64_t* bar_s = bars + 1 + 2 * NK + 2 * NV;         // [2] S_X landed
  uint64_t* bar_p = bar_s + 2;                          // [2] P_X written (count 128)
  uint64_t* bar_o = bar_s + 4;                          // [2] PV_X done
  uint64_t* bar_fin = bar_s + 6;                        // [2] each issuer's last products
  uint64_t* bar_sread = bar_s + 8;                      // [2] S_X loaded by the softmax (count 128)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int n_bh = p.B * p.Hq;
  const int m = p.n_pairs - 1 - int(blockIdx.x) / n_bh;  // longest causal rows first
  const int bh = int(blockIdx.x) % n_bh;
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / p.G;
  const int qt_a = 2 * m, qt_b = 2 * m + 1;
  const bool has_b = qt_b < p.n_tiles;
  const int nkv_a = p.causal ? qt_a + 1 : p.n_tiles, nkv_b = has_b ? (p.causal ? qt_b + 1 : p.n_tiles) : 0;
  const int n_kv = has_b ? nkv_b : nkv_a;
  const WaitCtl wc{p.err, p.wait_limit, abort_flag};
  NEA_TRACE_STAMP(p, 0, tid == 0);

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar_qtma, 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(&bar_ktma[s], 1);
      mbar_init(&bar_kempty[s], has_b ? 2 : 1);  // one commit per tile using the stage
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&bar_vtma[s], 1);
      mbar_init(&bar_vempty[s], has_b ? 2 : 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar_s[x], 1);
      mbar_init(&bar_p[x], 128);
      mbar_init(&bar_o[x], 1);
      mbar_init(&bar_sread[x], 128);
    }
    mbar_init(&bar_fin[0], 1);
    mbar_init(&bar_fin[1], 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  grid_dep_wait();  // the operand planes come from the prologue grid
  grid_dep_launch();
  NEA_TRACE_STAMP(p, 1, tid == 0);

  if (warp < 8) {
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int x = warp >> 2;   // query tile A or B
    const int r = tid & 127;   // row inside the tile, TMEM lane
    const int my_qt = x ? qt_b : qt_a, my_nkv = x ? nkv_b : nkv_a;
    const int q = my_qt * kTileRows + r;
    const uint32_t lane_base = tmem_addr(tbase, uint32_t(warp & 3) * 32, 0);
    // pcol: P (bf16 storage) or P lo (float32 storage)
    const uint32_t scol = lane_base + 256 * x, ocol = scol + 128, pcol = scol + 192;
    float m_run = -INFINITY;
    uint64_t l01 = 0, l23 = 0;  // partial row sums, two packed pairs
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = x == 0 || has_b;
    for (int j = 0; ok && j < my_nkv; ++j) {
      if (!wait_warp(&bar_s[x], j & 1, wc, kErrWaitMma)) { ok = false; break; }
      NEA_TRACE_STAMP(p, 4 + 16 * x + 2 * min(j, 7), r == 0);
      tc_fence_after();
      uint32_t sv[128];
      tmem_ld128(scol, sv);
      if (kSepP) {  // S_X(j) is in registers: the next S may overwrite it
        tc_fence_before();
        mbar_arrive(&bar_sread[x]);
      }
      const int kv0 = j * kTileRows;
      if ((p.causal && j == my_qt) || kv0 + kTileRows > p.T) {  // same for the whole tile
        const int lim = (p.causal ? min(q, p.T - 1) : p.T - 1) - kv0;  // last visible column
#pragma unroll
        for (int i = 0; i < 128; ++i) sv[i] = i > lim ? 0xff800000u : sv[i];  // -inf: P = 0
      }
      const float m_tile = row_max128(sv) * p.scale_log2;
      float alpha = 1.f;
      if (m_tile > m_run + 8.f) {  // keep a stale max unless it grew by > 2^8
        alpha = ex2(m_run - m_tile);
        m_run = m_tile;
      }
      const uint64_t a2 = f2_pack(alpha, alpha);
      l01 = f2_mul(l01, a2);
      l23 = f2_mul(l23, a2);
      const uint64_t nm2 = f2_pack(-m_run, -m_run);
      // O rescale by alpha: O holds the sum over key tiles < j once PV_X(j-1)
      // has completed
      auto rescale_o = [&]() {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(ocol + 32 * c, rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
          tmem_st32(ocol + 32 * c, rr);
        }
      };
      if constexpr (!F32IO) {
        // P = exp2(s * scale_log2 - m) -> bf16, all 128 columns in registers;
        // one pair in four on the FMA pipe, the rest on the exponential unit
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const uint64_t t2 = f2_fma(f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sc2, nm2);
          float p0, p1;
          if ((i & 3) == 3) {
            f2_unpack(exp2_poly2(t2), p0, p1);
          } else {
            float t0, t1;
            f2_unpack(t2, t0, t1);
            p0 = ex2(t0);
            p1 = ex2(t1);
          }
          if (i & 1) l23 = f2_add(l23, f2_pack(p0, p1)); else l01 = f2_add(l01, f2_pack(p0, p1));
          pk[i] = pack_bf16(p0, p1);
        }
        // PV_X(j-1) has read P_X(j-1) and updated O before both are touched
        // (P over S: S_X(j) was issued after PV_X(j-1) completed)
        if (j > 0 && !wait_warp(&bar_o[x], (j - 1) & 1, wc, kErrWaitMma)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(kFullMask, alpha != 1.f && j > 0)) rescale_o();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t part[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) part[i] = pk[16 * c + i];
          tmem_st16((kSepP ? pcol : scol) + 16 * c, part);
        }
      } else {
        // P = exp2(s * scale_log2 - m) -> bf16 hi over S, lo apart
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = 32 * c + 2 * i;
            float t0, t1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, nm2), t0, t1);
            const float p0 = ex2(t0), p1 = ex2(t1);
            const uint64_t pp = f2_pack(p0, p1);
            if (i & 1) l23 = f2_add(l23, pp); else l01 = f2_add(l01, pp);
            hi[i] = pack_bf16(p0, p1);
            float r0, r1;
            f2_unpack(f2_sub(pp, f2_pack(bf16_lo_f(hi[i]), bf16_hi_f(hi[i]))), r0, r1);
            lo[i] = pack_bf16(r0, r1);
          }
          // every column of S is in registers already
          tmem_st16(scol + 16 * c, hi);
          tmem_st16(pcol + 16 * c, lo);
        }
        if (__any_sync(kFullMask, alpha != 1.f && j > 0)) {
          // PV_X(j-1) has landed (S_X(j) was issued after it)
          if (!wait_warp(&bar_o[x], (j - 1) & 1, wc, kErrWaitMma)) { ok = false; break; }
          tc_fence_after();
          rescale_o();
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar_p[x]);
      NEA_TRACE_STAMP(p, 5 + 16 * x + 2 * min(j, 7), r == 0);
    }
    if (ok && (x == 0 || has_b) && wait_warp(&bar_o[x], (my_nkv - 1) & 1, wc, kErrWaitMma)) {
      tc_fence_after();
      float o[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(ocol + 32 * c, rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[32 * c + i] = __uint_as_float(rr[i]);
      }
      if (q < p.T) {
        float la, lb, lc, ld;
        f2_unpack(l01, la, lb);
        f2_unpack(l23, lc, ld);
        const float l_run = (la + lb) + (lc + ld);
        const float inv = 1.f / l_run;
#pragma unroll
        for (int i = 0; i < D; ++i) o[i] *= inv;
        store_span<D, F32IO>(p.O, ((size_t(b) * p.T + q) * p.Hq + h) * D, o);
        // LSE = ln(2^m * l) with m in log2 units of the scaled scores
        p.LSE[(size_t(b) * p.Hq + h) * p.T + q] = (m_run + log2f(l_run)) * 0.69314718055994531f;
      }
      NEA_TRACE_STAMP(p, 76 + x, r == 0);
    }
  } else {
    if (warp == 10) {
      // ------------------------------------------------------------ TMA
      if ((tid & 31) == 0) {
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_k);
        prefetch_tmap(&p.tm_v);
        const int nq = has_b ? 2 : 1;
        // a load of `row0` of tensor X: the tile (bf16) or its hi and lo planes
        auto load_tile = [&](uint8_t* dst, const CUtensorMap* hi, const CUtensorMap* lo, int head, int row0,
                             uint64_t* bar) {
#pragma unroll
          for (uint32_t cb = 0; cb < TileGeom<D>::kBlocks; ++cb)  // column blocks of 64 elements (D = 128)
            tma_load_4d(dst + cb * TileGeom<D>::kBlockBytes, hi, int(cb) * 64, head, row0, b, bar);
          if (F32IO) tma_load_4d(dst + OPB, lo, 0, head, row0, b, bar);
        };
        // fault-injection hook: withhold the query tiles so every wait on them
        // runs into its limit
        const bool q_armed = !(p.debug & 1);
        if (q_armed) {
          mbar_arrive_expect_tx(bar_qtma, nq * L::kTile);
          load_tile(smem + L::kQA, &p.tm_q, &p.tm_q_lo, h, qt_a * kTileRows, bar_qtma);
          if (has_b) load_tile(smem + L::kQB, &p.tm_q, &p.tm_q_lo, h, qt_b * kTileRows, bar_qtma);
        }
        int armed_k = 0, armed_v = 0;
        for (int j = 0; j < n_kv; ++j) {
          const int sk = j % NK, sv = j % NV;
          if (j >= NK && !wait_thread(&bar_kempty[sk], ((j / NK) - 1) & 1, wc, kErrWaitEmpty)) break;
          uint8_t* kst = smem + L::kK0 + sk * L::kKStage;
          mbar_arrive_expect_tx(&bar_ktma[sk], L::kTile);
          load_tile(kst, &p.tm_k, &p.tm_k_lo, g, j * kTileRows, &bar_ktma[sk]);
          NEA_TRACE_STAMP(p, 52 + min(j, 7), true);
          armed_k = j + 1;
          if (j >= NV && !wait_thread(&bar_vempty[sv], ((j / NV) - 1) & 1, wc, kErrWaitEmpty)) break;
          mbar_arrive_expect_tx(&bar_vtma[sv], L::kTile);
          load_tile(smem + L::kV0 + sv * L::kVStage, &p.tm_v, &p.tm_v_lo, g, j * kTileRows, &bar_vtma[sv]);
          NEA_TRACE_STAMP(p, 60 + min(j, 7), true);
          armed_v = j + 1;
        }
        // never leave copies in flight: on an abort, wait (bounded) for every
        // load still outstanding before the CTA exits
        if (*abort_flag) {
          for (int j = max(0, armed_k - NK); j < armed_k; ++j) drain_wait(&bar_ktma[j % NK], (j / NK) & 1, wc);
          for (int j = max(0, armed_v - NV); j < armed_v; ++j) drain_wait(&bar_vtma[j % NV], (j / NV) & 1, wc);
          if (q_armed) drain_wait(bar_qtma, 0, wc);
        }
      }
      __syncwarp();
    } else if (warp < 10) {
      // ------------------------------------------------------------ MMA issuers (warps 8, 9)
      // S_X(j+1) may overwrite S_X(j) once the softmax holds S_X(j) in
      // registers (bf16 storage: P in its own columns) or once PV_X(j) has
      // read P_X(j) (float32 storage: P hi over S).  Stage releases count one
      // commit per tile; the last key tile of a causal pair is used by B
      // alone, but its stages are never refilled, so no one waits for that
      // release.
      const int xw = warp - 8;  // this warp's tile
      if ((tid & 31) == 0 && (xw == 0 || has_b)) {
        constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);
        const int n_x[2] = {nkv_a, nkv_b};
        auto issue_s = [&](int x, int j) {
          const uint32_t sQ = smem_u32(smem + (x ? L::kQB : L::kQA));
          const uint32_t sK = smem_u32(smem + L::kK0 + (j % NK) * L::kKStage);
          const uint32_t dS = tbase + 256 * x;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int term = 0; term < kTerms; ++term) {
              // float32 storage: hi*hi + hi*lo + lo*hi
              const uint32_t qa = sQ + (term == 2 ? OPB : 0) + TileGeom<D>::kslice(kk);
              const uint32_t kb = sK + (term == 1 ? OPB : 0) + TileGeom<D>::kslice(kk);
              mma_ss(dS, smem_desc(qa, RB, 16), smem_desc(kb, RB, 16), idS, (kk | term) != 0);
            }
          }
          tc_commit(&bar_s[x]);
          tc_commit(&bar_kempty[j % NK]);
        };
        auto issue_pv = [&](int x, int j) {
          const int sv = j % NV;
          const uint32_t sV = smem_u32(smem + L::kV0 + sv * L::kVStage);
          const uint32_t phi = tbase + 256 * x, plo = tbase + 256 * x + 192, dO = tbase + 256 * x + 128;
#pragma unroll
          for (int kk = 0; kk < kTileRows / 16; ++kk) {
#pragma unroll
            for (int term = 0; term < kTerms; ++term) {
              // float32 storage: Phi*Vhi + Phi*Vlo + Plo*Vhi
              const uint32_t pa = (kSepP ? plo : (term == 2 ? plo : phi)) + kk * 8;
              const uint32_t vb = sV + (term == 1 ? OPB : 0) + kk * 16 * RB;
              mma_ts(dO, pa, smem_desc(vb, RB, kTileRows * RB), idO, (j | kk | term) != 0);
            }
          }
          tc_commit(&bar_o[x]);
          tc_commit(&bar_vempty[sv]);
        };
        // S_X(j+1): key tile landed, and S_X(j) no longer needed
        auto next_s = [&](int x, int j) {
          const bool free = kSepP ? wait_thread(&bar_sread[x], j & 1, wc, kErrWaitSoftmax)
                                  : wait_thread(&bar_o[x], j & 1, wc, kErrWaitMma);
          if (!free || !wait_thread(&bar_ktma[(j + 1) % NK], ((j + 1) / NK) & 1, wc, kErrWaitProducer))
            return false;
          NEA_TRACE_STAMP(p, 44 + min(j, 7), x == 0);
          tc_fence_after();
          issue_s(x, j + 1);
          return true;
        };
        // PV_X(j): P_X(j) written and value tile landed
        auto next_pv = [&](int x, int j) {
          if (!wait_thread(&bar_p[x], j & 1, wc, kErrWaitSoftmax) ||
              !wait_thread(&bar_vtma[j % NV], (j / NV) & 1, wc, kErrWaitProducer))
            return false;
          NEA_TRACE_STAMP(p, 36 + min(j, 7), x == 0);
          tc_fence_after();
          issue_pv(x, j);
          return true;
        };
        bool ok = wait_thread(bar_qtma, 0, wc, kErrWaitProducer) &&
                  wait_thread(&bar_ktma[0], 0, wc, kErrWaitProducer);
        // float32 storage: tile B waits for tile A's first P (half a step)
        if (!kSepP && xw == 1) ok = ok && wait_thread(&bar_p[0], 0, wc, kErrWaitSoftmax);
        if (ok) {
          tc_fence_after();
          issue_s(xw, 0);
        }
        for (int j = 0; ok && j < n_x[xw]; ++j) {
          if (kSepP && j + 1 < n_x[xw] && !(ok = next_s(xw, j))) break;
          if (!(ok = next_pv(xw, j))) break;
          if (!kSepP && j + 1 < n_x[xw] && !(ok = next_s(xw, j))) break;
        }
        tc_commit(&bar_fin[xw]);
        drain_wait(&bar_fin[xw], 0, wc);
      }
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
  NEA_TRACE_STAMP(p, 78, tid == 0);
}

}  // namespace nea
