// Backward kernels.  The pages say only that every operator's backward is
// hand-written and gradient-checked ("NanoEuler" write-up, aimsg.uk, sections
// 3-4; agentlenshq.com summary, "Validation and stability"); the design here
// is the recompute-from-LSE backward of tiled attention:
//
//   row term     Dv_i = sum_d dO_id O_id                 (operand prologue, nea_prep.cuh)
//   per tile     S = Q' K'^T, P = exp(scale S - LSE), dP = dO V^T,
//                dS = P o (dP - Dv),
//                dV += P^T dO, dK' += dS^T Q', dQ' += dS K'  (x scale)
//   epilogue     dQ = R^T dQ', dK = R^T dK'   (inverse rotation per position)
//
// One kernel serves both gradient passes in one launch (the dK/dV units
// first, the longest first; the dQ units after them, longest first, so they
// fill the SMs the dK/dV units leave free), the "row" tile being resident in
// shared memory and the "column" tiles streamed past it:
//   DKDV  row = key tile j of kv head g (K'_j, V_j), columns = query tiles
//         i >= j of every query head of the group (Q'_i, dO_i, LSE, Dv); the
//         group's dK/dV sums stay in TMEM for the whole CTA, so the reduction
//         over the GQA group needs no extra pass or atomics.
//   DQ    row = query tile i of head h (Q'_i, dO_i), columns = key tiles
//         j <= i (K'_j, V_j).
// This kernel serves bfloat16 storage (float32 storage: nea_bwd_f32.cuh).
// Operands arrive by TMA in the swizzled operand layout: rotated copies of Q
// and K from the operand prologue (nea_prep.cuh) and the inputs V, dO.
// Warps: 0-7 elementwise work, warp w on TMEM lanes 32 (w % 4) .. + 31 (its
// rows) and columns 64 (w / 4) .. + 63 of the tile; 8 issues the MMAs; 9
// issues TMA (resident tiles, then column tiles and, for DKDV, the LSE/Dv
// slices into a ring).
//   S_rc  = R1 C1^T      (R1 = K' or Q', C1 = Q' or K')   -> TMEM [0,128)
//   dP_rc = R2 C2^T      (R2 = V or dO,  C2 = dO or V)    -> TMEM [128,256)
//   P is kept in fp32 registers for dS and, for DKDV, as bf16 in TMEM
//   [384,448) for the dV product; bf16 dS goes to TMEM [448,512)
//   DKDV: acc1 += P  C2   (dV), acc2 += dS C1 (dK)   (C1, C2 as MN-major B)
//   DQ:   acc1 += dS C1   (dQ)
// Issue order per item k: dP(k); S(k+1) as soon as the rows hold S(k) in
// registers; dV(k) once P(k) is written; dK/dQ(k) once dS(k) is written.  The
// rows overwrite P and dS of item k-1 only after the commit that follows
// dK/dQ(k-1) (which covers every earlier MMA).
// D = 128: the two accumulators take TMEM [256,512), so P goes over S and dS
// over dP, each warp half writing its 64 columns' bf16 pairs into the first
// 32 of its own 64 columns (no half overwrites scores the other still
// reads); S(k+1) is issued right after dV(k) (dK/dV units) and dP(k+1) right
// after dK/dQ(k): the tensor core runs one thread's MMAs in issue order, so
// each reads P or dS before the next product overwrites it.  The rings hold
// two stages (32 KB tiles).
#pragma once

#include <cuda.h>

#include "nea_prep.cuh"
#include "nea_tiles.cuh"

namespace nea {

// ---------------------------------------------------------------- main kernel
// Parameters of both gradient kernels (bfloat16 storage here, float32 storage
// in nea_bwd_f32.cuh).
struct BwdParams {
  // bf16 storage: rotated Q, K (the inputs when the rotation is off), V, dO.
  // float32 storage: the hi planes.
  CUtensorMap tm_q;    // [B][T][Hq][D]
  CUtensorMap tm_k;    // [B][T][Hkv][D]
  CUtensorMap tm_v;
  CUtensorMap tm_do;   // [B][T][Hq][D]
  // float32 storage: the lo planes
  CUtensorMap tm_q_lo;
  CUtensorMap tm_k_lo;
  CUtensorMap tm_v_lo;
  CUtensorMap tm_do_lo;
  CUtensorMap tm_ws;   // row terms ws[B*Hq][2][Tp] fp32, box {128, 2, 1}
  const float* ws;     // row terms, see nea_prep.cuh
  int Tp;              // T rounded up to a multiple of 128
  void* dQ;
  void* dK;
  void* dV;
  const float2* rope;  // rotary table [T][D/2] for the inverse rotation of dQ, dK; nullptr: off
  int B, T, Hq, Hkv, G;
  int n_tiles;
  int causal;
  float scale_log2;   // log2(e) / sqrt(D)
  float scale;        // 1 / sqrt(D)
  int* err;
  unsigned long long wait_limit;
  int n_dkdv;                 // units [0, n_dkdv) are dK/dV units, the rest dQ units
  int unit0;                  // unit of blockIdx.x == 0
  int debug;                  // bit 1: withhold the resident tiles (fault-injection hook)
  unsigned long long* trace;  // per-CTA phase stamps (NEA_TRACE builds only)
};

template <int D>
struct BwdSmem {
  static constexpr int kStages = D == 128 ? 2 : 3;
  static constexpr uint32_t kTile = TileGeom<D>::kOpBytes;
  static constexpr uint32_t kR1 = 0;
  static constexpr uint32_t kR2 = kR1 + kTile;
  static constexpr uint32_t kStage0 = kR2 + kTile;
  static constexpr uint32_t kColVec = 2 * kTile;             // per-column -LSE*log2e and Dv (DKDV)
  static constexpr uint32_t kStageBytes = kColVec + 1024;
  static constexpr uint32_t kBars = kStage0 + kStages * kStageBytes;
  // rtma, tma[S], empty[S], s, dp, p, ds, dk, fin, sread
  static constexpr int kNumBars = 1 + 2 * kStages + 7;
  static constexpr uint32_t kMisc = kBars + 8 * kNumBars;
  static constexpr uint32_t kUsed = kMisc + 16;
  static constexpr uint32_t kAlloc = kUsed + 1024 > 116u * 1024u ? kUsed + 1024 : 116u * 1024u;
  static constexpr int kThreads = 320;
  static_assert(kStage0 % 1024 == 0 && kStageBytes % 1024 == 0, "operand tiles need 1024-byte alignment");
  static_assert(kAlloc <= 232448, "shared memory");
};

// N consecutive TMEM columns of this thread's lane (N = 8, 16, 32 or 64).
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, float* v) {
  if constexpr (N == 64) {
    uint32_t r[64];
    tmem_ld64(taddr, r);
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
  } else if constexpr (N == 32) {
    uint32_t r[32];
    tmem_ld32(taddr, r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  } else if constexpr (N == 16) {
    uint32_t r[16];
    tmem_ld16(taddr, r);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  } else {
    static_assert(N == 8, "8, 16, 32 or 64 columns");
    uint32_t r[8];
    tmem_ld8(taddr, r);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
  }
}

// One unit (a dK/dV unit when DKDV, else a dQ unit; `bid` its index among
// units of its kind), specialised per pass so that neither pays for the
// other's branches.
template <int D, bool DKDV>
__device__ __forceinline__ void attn_bwd_unit(const BwdParams& p, int bid) {
  using L = BwdSmem<D>;
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  constexpr int NS = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_rtma = bars + 0;             // resident tiles landed
  uint64_t* bar_tma = bars + 1;              // [NS] column tiles landed
  uint64_t* bar_empty = bars + 1 + NS;       // [NS] MMAs done with the stage
  uint64_t* bar_s = bars + 1 + 2 * NS;       // S landed
  uint64_t* bar_dp = bar_s + 1;              // dP landed
  uint64_t* bar_p = bar_s + 2;               // rows read S, wrote P (count 256)
  uint64_t* bar_ds = bar_s + 3;              // rows wrote dS (count 256)
  uint64_t* bar_dk = bar_s + 4;              // dS MMA of an item done
  uint64_t* bar_fin = bar_s + 5;
  uint64_t* bar_sread = bar_s + 6;           // rows hold S in registers (count 256)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const WaitCtl wc{p.err, p.wait_limit, abort_flag};
  NEA_TRACE_STAMP(p, 0, tid == 0);

  // ---- work decomposition
  // DKDV: blockIdx -> (key tile ascending = most causal work first, b, g)
  // DQ:   blockIdx -> (query tile descending, b, h)
  int b, rt, head_r, n_items, c0;
  if (DKDV) {
    const int n_bg = p.B * p.Hkv;
    rt = bid / n_bg;
    const int bg = bid % n_bg;
    b = bg / p.Hkv;
    head_r = bg % p.Hkv;
    c0 = p.causal ? rt : 0;                       // first query tile
    n_items = p.G * (p.n_tiles - c0);
  } else {
    const int n_bh = p.B * p.Hq;
    rt = p.n_tiles - 1 - bid / n_bh;
    const int bh = bid % n_bh;
    b = bh / p.Hq;
    head_r = bh % p.Hq;
    c0 = 0;
    n_items = p.causal ? rt + 1 : p.n_tiles;      // key tiles 0 .. rt
  }
  const int n_ct = p.n_tiles - c0;  // column tiles per query head (DKDV)
  // item k -> (column head, column tile)
  auto item_head = [&](int k) { return DKDV ? head_r * p.G + k / n_ct : head_r / p.G; };
  auto item_tile = [&](int k) { return DKDV ? c0 + k % n_ct : k; };

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar_rtma, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_tma[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 256);
    mbar_init(bar_ds, 256);
    mbar_init(bar_dk, 1);
    mbar_init(bar_fin, 1);
    mbar_init(bar_sread, 256);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  grid_dep_wait();  // operand planes and row terms come from the prologue grid
  grid_dep_launch();
  constexpr uint32_t kColS = 0, kColDP = 128, kColAcc1 = 256, kColAcc2 = 256 + D, kColP = 384, kColDS = 448;
  constexpr bool kOver = D == 128;  // P over S, dS over dP (see the header)
  // TMEM column of the 16-column slice kk of P or dS (bf16 pairs)
  auto p_col = [](int kk) -> uint32_t { return kOver ? kColS + 64 * (kk / 4) + 8 * (kk % 4) : kColP + 8 * kk; };
  auto ds_col = [](int kk) -> uint32_t { return kOver ? kColDP + 64 * (kk / 4) + 8 * (kk % 4) : kColDS + 8 * kk; };

  if (warp == 9) {
    // ------------------------------------------------------------ TMA
    if ((tid & 31) == 0) {
      const CUtensorMap* m_r1 = DKDV ? &p.tm_k : &p.tm_q;
      const CUtensorMap* m_r2 = DKDV ? &p.tm_v : &p.tm_do;
      const CUtensorMap* m_c1 = DKDV ? &p.tm_q : &p.tm_k;
      const CUtensorMap* m_c2 = DKDV ? &p.tm_do : &p.tm_v;
      prefetch_tmap(m_r1);
      prefetch_tmap(m_r2);
      prefetch_tmap(m_c1);
      prefetch_tmap(m_c2);
      auto load_tile = [&](uint8_t* dst, const CUtensorMap* m, int head, int row0, uint64_t* bar) {
#pragma unroll
        for (uint32_t cb = 0; cb < TileGeom<D>::kBlocks; ++cb)  // column blocks of 64 elements (D = 128)
          tma_load_4d(dst + cb * TileGeom<D>::kBlockBytes, m, int(cb) * 64, head, row0, b, bar);
      };
      // fault-injection hook: withhold the resident tiles so every wait on
      // them runs into its limit
      const bool r_armed = !(p.debug & 2);
      if (r_armed) {
        mbar_arrive_expect_tx(bar_rtma, 2 * L::kTile);
        load_tile(smem + L::kR1, m_r1, head_r, rt * kTileRows, bar_rtma);
        load_tile(smem + L::kR2, m_r2, head_r, rt * kTileRows, bar_rtma);
      }
      int armed = 0;
      for (int k = 0; k < n_items; ++k) {
        const int s = k % NS;
        if (k >= NS && !wait_thread(&bar_empty[s], ((k / NS) - 1) & 1, wc, kErrWaitEmpty)) break;
        uint8_t* st = smem + L::kStage0 + s * L::kStageBytes;
        const int ch = item_head(k), ct = item_tile(k);
        mbar_arrive_expect_tx(&bar_tma[s], 2 * L::kTile + (DKDV ? 1024 : 0));
        load_tile(st, m_c1, ch, ct * kTileRows, &bar_tma[s]);
        load_tile(st + L::kTile, m_c2, ch, ct * kTileRows, &bar_tma[s]);
        if (DKDV)  // -LSE*log2e then Dv of the 128 queries of this column tile
          tma_load_3d(st + L::kColVec, &p.tm_ws, ct * kTileRows, 0, b * p.Hq + ch, &bar_tma[s]);
        armed = k + 1;
      }
      if (*abort_flag) {
        for (int k = max(0, armed - NS); k < armed; ++k) drain_wait(&bar_tma[k % NS], (k / NS) & 1, wc);
        if (r_armed) drain_wait(bar_rtma, 0, wc);
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if ((tid & 31) == 0) {
      constexpr uint32_t idSS = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idAcc = idesc_bf16(128, D, 0, 1);
      const uint32_t sR1 = smem_u32(smem + L::kR1), sR2 = smem_u32(smem + L::kR2);
      constexpr uint32_t accG = DKDV ? kColAcc2 : kColAcc1;  // accumulator of dS C1
      auto stage_c1 = [&](int k) { return smem_u32(smem + L::kStage0 + (k % NS) * L::kStageBytes); };
      auto issue_s = [&](int k) {
        const uint32_t sC1 = stage_c1(k);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tbase + kColS, smem_desc(sR1 + TileGeom<D>::kslice(kk), RB, 16),
                 smem_desc(sC1 + TileGeom<D>::kslice(kk), RB, 16), idSS, kk != 0);
        tc_commit(bar_s);
      };
      bool ok = wait_thread(bar_rtma, 0, wc, kErrWaitProducer) &&
                (n_items == 0 || wait_thread(&bar_tma[0], 0, wc, kErrWaitProducer));
      if (ok && n_items > 0) {
        tc_fence_after();
        issue_s(0);
      }
      for (int k = 0; ok && k < n_items; ++k) {
        const uint32_t sC1 = stage_c1(k), sC2 = sC1 + L::kTile;
        // dP(k) overwrites dP(k-1), which the rows read before dS(k-1)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tbase + kColDP, smem_desc(sR2 + TileGeom<D>::kslice(kk), RB, 16),
                 smem_desc(sC2 + TileGeom<D>::kslice(kk), RB, 16), idSS, kk != 0);
        tc_commit(bar_dp);
        NEA_TRACE_STAMP(p, 36 + min(k, 7), true);
        if ((!kOver || !DKDV) && k + 1 < n_items) {
          // S(k+1) overwrites S(k): the rows must hold it in registers
          if (!wait_thread(bar_sread, k & 1, wc, kErrWaitSoftmax) ||
              !wait_thread(&bar_tma[(k + 1) % NS], ((k + 1) / NS) & 1, wc, kErrWaitProducer)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(k + 1);
          NEA_TRACE_STAMP(p, 44 + min(k, 7), true);
        }
        if (DKDV) {
          if (!wait_thread(bar_p, k & 1, wc, kErrWaitSoftmax)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTileRows / 16; ++kk)
            mma_ts(tbase + kColAcc1, tbase + p_col(kk), smem_desc(sC2 + kk * 16 * RB, RB, kTileRows * RB),
                   idAcc, (k | kk) != 0);
          NEA_TRACE_STAMP(p, 52 + min(k, 7), true);
          if (kOver && k + 1 < n_items) {
            // S(k+1) overwrites P(k): issued after dV(k), which reads it first
            // (the tensor core runs this thread's MMAs in issue order)
            if (!wait_thread(&bar_tma[(k + 1) % NS], ((k + 1) / NS) & 1, wc, kErrWaitProducer)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(k + 1);
          }
        }
        // acc += dS(k) C1(k), then release the stage of item k
        if (!wait_thread(bar_ds, k & 1, wc, kErrWaitSoftmax)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk)
          mma_ts(tbase + accG, tbase + ds_col(kk), smem_desc(sC1 + kk * 16 * RB, RB, kTileRows * RB), idAcc,
                 (k | kk) != 0);
        tc_commit(&bar_empty[k % NS]);
        tc_commit(bar_dk);
        NEA_TRACE_STAMP(p, 60 + min(k, 7), true);
        // (D = 128: dP(k+1), next, overwrites dS(k) after dK/dQ(k) has read it,
        // in issue order)
      }
      tc_commit(bar_fin);
      drain_wait(bar_fin, 0, wc);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise (warps 0-7)
    const int hf = warp >> 2;            // column half
    const int r = (warp & 3) * 32 + (tid & 31);
    const int row = rt * kTileRows + r;  // key position (DKDV) or query position (DQ)
    const int cb = 64 * hf;              // first column of this warp
    const uint32_t lane_base = tmem_addr(tbase, uint32_t(warp & 3) * 32, 0);
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    uint64_t nl2_row = 0, dv_row = 0;
    if (!DKDV) {  // padded rows read -inf / 0, so their P and dS vanish
      const float* w = p.ws + (size_t(b) * p.Hq + head_r) * 2 * p.Tp + row;
      const float nl2 = __ldg(w), dv = __ldg(w + p.Tp);
      nl2_row = f2_pack(nl2, nl2);
      dv_row = f2_pack(dv, dv);
    }
    bool ok = true;
    for (int k = 0; k < n_items; ++k) {
      const int s = k % NS;
      const float4* colvec =
          reinterpret_cast<const float4*>(smem + L::kStage0 + s * L::kStageBytes + L::kColVec) + cb / 4;
      const int ct = item_tile(k);
      // DKDV reads the per-column -LSE*log2e / Dv the TMA landed in the stage
      if (DKDV && !wait_warp(&bar_tma[s], (k / NS) & 1, wc, kErrWaitProducer)) { ok = false; break; }
      if (!wait_warp(bar_s, k & 1, wc, kErrWaitMma)) { ok = false; break; }
      NEA_TRACE_STAMP(p, 4 + min(k, 7), tid == 0);
      tc_fence_after();
      const int col0 = ct * kTileRows + cb;  // position of this warp's first column
      // ---- P phase: P = exp2(s * scale_log2 - LSE*log2e), masked
      uint32_t sv[64];
      tmem_ld64(lane_base + kColS + cb, sv);
      tc_fence_before();
      mbar_arrive(bar_sread);  // S(k+1) may overwrite S(k) now
      if ((p.causal && ct == rt) || ct * kTileRows + kTileRows > p.T) {  // same for the whole tile
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          // DKDV: key (row) after query (column); DQ: key (column) after query
          // (row) or past T.  Queries past T have -inf row terms already.
          const bool masked = DKDV ? (p.causal && row > col0 + i) : ((p.causal && col0 + i > row) || col0 + i >= p.T);
          sv[i] = masked ? 0xff800000u : sv[i];
        }
      }
      float pv[64];
#pragma unroll
      for (int i = 0; i < 16; ++i) {  // four columns per step
        uint64_t nl2a = nl2_row, nl2b = nl2_row;
        if (DKDV) {
          const float4 c = colvec[i];
          nl2a = f2_pack(c.x, c.y);
          nl2b = f2_pack(c.z, c.w);
        }
        float t0, t1, t2, t3;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * i]), __uint_as_float(sv[4 * i + 1])), sc2, nl2a), t0, t1);
        f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * i + 2]), __uint_as_float(sv[4 * i + 3])), sc2, nl2b), t2, t3);
        pv[4 * i] = ex2(t0);
        pv[4 * i + 1] = ex2(t1);
        pv[4 * i + 2] = ex2(t2);
        pv[4 * i + 3] = ex2(t3);
      }
      // P(k-1) and dS(k-1) stay in TMEM until dV/dK/dQ(k-1) have read them
      // (D = 128: they lie under S(k) and dP(k), whose commits cover those
      // products)
      if (!kOver && k > 0 && !wait_warp(bar_dk, (k - 1) & 1, wc, kErrWaitMma)) { ok = false; break; }
      if (DKDV) {  // bf16 P for the dV product
        tc_fence_after();
        uint32_t ph[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) ph[i] = pack_bf16(pv[2 * i], pv[2 * i + 1]);
        tmem_st32(lane_base + (kOver ? kColS + 64 * hf : kColP + 32 * hf), ph);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p);
      }
      NEA_TRACE_STAMP(p, 12 + min(k, 7), tid == 0);
      // ---- dS phase: dS = P (dP - Dv), bf16, into its own TMEM columns
      if (!wait_warp(bar_dp, k & 1, wc, kErrWaitMma)) { ok = false; break; }
      NEA_TRACE_STAMP(p, 20 + min(k, 7), tid == 0);
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t rr[32], pk[16];
        tmem_ld32(lane_base + kColDP + cb + 32 * c, rr);
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // four columns per step
          const int e = 32 * c + 4 * i;
          uint64_t dva = dv_row, dvb = dv_row;
          if (DKDV) {
            const float4 d = colvec[32 + e / 4];
            dva = f2_pack(d.x, d.y);
            dvb = f2_pack(d.z, d.w);
          }
          float a0, a1, a2, a3;
          f2_unpack(f2_mul(f2_pack(pv[e], pv[e + 1]),
                           f2_sub(f2_pack(__uint_as_float(rr[4 * i]), __uint_as_float(rr[4 * i + 1])), dva)),
                    a0, a1);
          f2_unpack(f2_mul(f2_pack(pv[e + 2], pv[e + 3]),
                           f2_sub(f2_pack(__uint_as_float(rr[4 * i + 2]), __uint_as_float(rr[4 * i + 3])), dvb)),
                    a2, a3);
          pk[2 * i] = pack_bf16(a0, a1);
          pk[2 * i + 1] = pack_bf16(a2, a3);
        }
        tmem_st16(lane_base + (kOver ? kColDP + 64 * hf : kColDS + 32 * hf) + 16 * c, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_ds);
      NEA_TRACE_STAMP(p, 28 + min(k, 7), tid == 0);
    }
    if (ok && wait_warp(bar_fin, 0, wc, kErrWaitMma)) {
      tc_fence_after();
      // TMEM loads are warp-collective: every lane loads, only valid rows store
      constexpr int DH = D / 2;
      if (DKDV) {
        // half 0 writes the row of dV, half 1 the row of dK
        float acc[D];
        constexpr int NL = D < 64 ? D : 64;  // columns per TMEM load
#pragma unroll
        for (int c = 0; c < D / NL; ++c) tmem_ld_n<NL>(lane_base + (hf ? kColAcc2 : kColAcc1) + NL * c, acc + NL * c);
        if (hf) {
#pragma unroll
          for (int i = 0; i < D; ++i) acc[i] *= p.scale;
        }
        if (row < p.T) {
          if (hf && p.rope) {
            // gradient w.r.t. the un-rotated input: apply R_t^T
            const float4* tp = reinterpret_cast<const float4*>(p.rope + size_t(row) * (D / 2));
#pragma unroll
            for (int i = 0; i < D / 4; ++i) {
              const float4 cs = __ldg(tp + i);
              rot2(acc[4 * i], acc[4 * i + 1], cs.x, -cs.y);
              rot2(acc[4 * i + 2], acc[4 * i + 3], cs.z, -cs.w);
            }
          }
          const size_t off = ((size_t(b) * p.T + row) * p.Hkv + head_r) * D;
          store_span<D, false>(hf ? p.dK : p.dV, off, acc);
        }
      } else {
        // half h writes columns [h D/2, h D/2 + D/2) of the row of dQ
        float acc[DH];
        tmem_ld_n<DH>(lane_base + kColAcc1 + DH * hf, acc);
#pragma unroll
        for (int i = 0; i < DH; ++i) acc[i] *= p.scale;
        if (row < p.T) {
          if (p.rope) {
            const float4* tp = reinterpret_cast<const float4*>(p.rope + size_t(row) * (D / 2) + DH / 2 * hf);
#pragma unroll
            for (int i = 0; i < DH / 4; ++i) {
              const float4 cs = __ldg(tp + i);
              rot2(acc[4 * i], acc[4 * i + 1], cs.x, -cs.y);
              rot2(acc[4 * i + 2], acc[4 * i + 3], cs.z, -cs.w);
            }
          }
          const size_t off = ((size_t(b) * p.T + row) * p.Hq + head_r) * D + DH * hf;
          store_span<DH, false>(p.dQ, off, acc);
        }
      }
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

template <int D>
__global__ void __launch_bounds__(BwdSmem<D>::kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ BwdParams p) {
  const int unit = p.unit0 + int(blockIdx.x);
  if (unit < p.n_dkdv)
    attn_bwd_unit<D, true>(p, unit);
  else
    attn_bwd_unit<D, false>(p, unit - p.n_dkdv);
}

}  // namespace nea
