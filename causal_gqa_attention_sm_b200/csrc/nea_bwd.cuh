// Backward kernels.  The pages say only that every operator's backward is
// hand-written and gradient-checked ("NanoEuler" write-up, aimsg.uk, sections
// 3-4; agentlenshq.com summary, "Validation and stability"); the design here
// is the recompute-from-LSE backward of tiled attention:
//
//   row term     Dv_i = sum_d dO_id O_id                 (attn_bwd_rowterm)
//   per tile     S = Q' K'^T, P = exp(scale S - LSE), dP = dO V^T,
//                dS = P o (dP - Dv),
//                dV += P^T dO, dK' += dS^T Q', dQ' += dS K'  (x scale)
//   epilogue     dQ = R^T dQ', dK = R^T dK'   (inverse rotation per position)
//
// One kernel template serves both gradient passes, the "row" tile being
// resident in shared memory and the "column" tiles streamed past it:
//   DKDV  row = key tile j of kv head g (K'_j, V_j), columns = query tiles
//         i >= j of every query head of the group (Q'_i, dO_i, LSE, Dv); the
//         group's dK/dV sums stay in TMEM for the whole CTA, so the reduction
//         over the GQA group needs no extra pass or atomics.
//   DQ    row = query tile i of head h (Q'_i, dO_i), columns = key tiles
//         j <= i (K'_j, V_j).
// Operands arrive by TMA: bf16 storage lands tiles in the swizzled operand
// layout and the converter warps rotate queries/keys in place (RoPE fused into
// the tile load); float32 storage reads the pre-rotated bf16 hi/lo planes of
// the operand prologue (nea_prep.cuh) and forms S and dP from three bf16
// products, the gradient products from the hi parts.
// Warps: 0-3 own the 128 rows (TMEM lanes), 4 issues the MMAs, 5 issues TMA
// (resident tiles, then column tiles and, for DKDV, the LSE/Dv slices into a
// ring), 6-9 (bf16 only) rotate tiles.
//   S_rc  = R1 C1^T      (R1 = K' or Q', C1 = Q' or K')   -> TMEM [0,128)
//   dP_rc = R2 C2^T      (R2 = V or dO,  C2 = dO or V)    -> TMEM [128,256)
//   P (bf16 hi, lo) is kept in TMEM [384,512); dS overwrites dP in place
//   DKDV: acc1 += P  C2   (dV), acc2 += dS C1 (dK)   (C1, C2 as MN-major B)
//   DQ:   acc1 += dS C1   (dQ)
// S of item k+1 is issued as soon as the rows have read S of item k, so it
// overlaps the dS phase; dP of item k+1 waits for the dS MMA of item k.
#pragma once

#include <cuda.h>

#include "nea_tiles.cuh"

namespace nea {

// ---------------------------------------------------------------- row term
// Per-row terms of the backward, in a workspace ws[B*Hq][2][Tp] (Tp = T
// rounded up to whole 128-row tiles, so a tile of it is one TMA box):
//   ws[bh][0][t] = LSE[b][h][t] * log2(e)          (+inf for t >= T)
//   ws[bh][1][t] = Dv = sum_d dO[b][t][h][d] O[b][t][h][d]   (0 for t >= T)
// The padding makes P = exp2(s*c - lse2) vanish for queries past T.  One group
// of D/ELEMS lanes per (b, t, h) row, t over [0, Tp).
template <int D, bool F32IO>
__global__ void __launch_bounds__(256) attn_bwd_rowterm_kernel(const void* __restrict__ O,
                                                               const void* __restrict__ dO,
                                                               const float* __restrict__ LSE,
                                                               float* __restrict__ ws, int B, int T, int Tp,
                                                               int Hq) {
  constexpr int kElems = F32IO ? 4 : 8;    // elements per 16-byte chunk
  constexpr int kLanes = D / kElems;       // lanes per row: 4, 8 or 16
  const long gtid = long(blockIdx.x) * blockDim.x + threadIdx.x;
  const long prow = gtid / kLanes;         // (b, t, h) over t in [0, Tp)
  const int c = int(gtid % kLanes);
  const int h = int(prow % Hq);
  const long bt = prow / Hq;
  const int t = int(bt % Tp);
  const long b = bt / Tp;
  if (b >= B) return;  // whole groups of lanes leave together
  float* out = ws + (b * Hq + h) * 2 * long(Tp) + t;
  if (t >= T) {
    if (c == 0) {
      out[0] = INFINITY;
      out[Tp] = 0.f;
    }
    return;
  }
  const long row = (b * T + t) * Hq + h;
  float acc = 0.f;
  {
    if constexpr (F32IO) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(O) + row * D) + c);
      const float4 z = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(dO) + row * D) + c);
      acc = a.x * z.x + a.y * z.y + a.z * z.z + a.w * z.w;
    } else {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(O) + row * D) + c);
      const uint4 z = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(dO) + row * D) + c);
      acc = bf16_lo_f(a.x) * bf16_lo_f(z.x) + bf16_hi_f(a.x) * bf16_hi_f(z.x) + bf16_lo_f(a.y) * bf16_lo_f(z.y) +
            bf16_hi_f(a.y) * bf16_hi_f(z.y) + bf16_lo_f(a.z) * bf16_lo_f(z.z) + bf16_hi_f(a.z) * bf16_hi_f(z.z) +
            bf16_lo_f(a.w) * bf16_lo_f(z.w) + bf16_hi_f(a.w) * bf16_hi_f(z.w);
    }
  }
  // the kLanes lanes of a row are consecutive and leave or stay together
  const unsigned group = (kLanes == 32 ? kFullMask : ((1u << kLanes) - 1u) << (threadIdx.x & 31 & ~(kLanes - 1)));
#pragma unroll
  for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(group, acc, off);
  if (c == 0) {
    out[0] = __ldg(LSE + (b * Hq + h) * long(T) + t) * 1.4426950408889634f;
    out[Tp] = acc;
  }
}

// ---------------------------------------------------------------- main kernel
struct BwdParams {
  // bf16 storage: the inputs.  float32 storage: the hi planes.
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
  const float* ws;     // see attn_bwd_rowterm_kernel
  int Tp;              // T rounded up to a multiple of 128
  void* dQ;
  void* dK;
  void* dV;
  // rotary table [T][D/2] (+ block-start rows): in-place rotation of bf16
  // tiles and the inverse rotation of dQ, dK
  const float2* rope;
  int B, T, Hq, Hkv, G;
  int n_tiles;
  int causal;
  float scale_log2;   // log2(e) / sqrt(D)
  float scale;        // 1 / sqrt(D)
  int* err;
  unsigned long long wait_limit;
};

template <int D, bool F32IO, bool DKDV>
struct BwdSmem {
  static constexpr bool kConv = !F32IO;  // converter warps (in-place RoPE)
  static constexpr int kStages = F32IO ? 2 : 3;
  static constexpr uint32_t kTile = Stage<D, F32IO>::kBytes;
  static constexpr uint32_t kBase = RopeBaseRows<D>::kBytes;
  static constexpr uint32_t kSide = kConv ? 1024 : 0;
  static constexpr uint32_t kR1 = 0;
  static constexpr uint32_t kR2 = kR1 + kTile;
  static constexpr uint32_t kR1Base = kR2 + kTile;  // rotary base rows of the row tile
  static constexpr uint32_t kRope = kR1Base + kSide;
  static constexpr uint32_t kStage0 = kRope + (kConv ? TileGeom<D>::kRopeBytes : 0);
  static constexpr uint32_t kCBase = 2 * kTile;              // rotary base rows of C1
  static constexpr uint32_t kColVec = kCBase + kSide;        // per-column LSE and Dv (DKDV)
  static constexpr uint32_t kStageBytes = kColVec + (DKDV ? 1024 : 0);
  static constexpr uint32_t kBars = kStage0 + kStages * kStageBytes;
  // res_tma, res, tma[S], full[S], empty[S], s, dp, p, ds, dk, fin
  static constexpr int kNumBars = 2 + 3 * kStages + 6;
  static constexpr uint32_t kMisc = kBars + 8 * kNumBars;
  static constexpr uint32_t kUsed = kMisc + 16;
  static constexpr uint32_t kAlloc = kUsed + 1024 > 116u * 1024u ? kUsed + 1024 : 116u * 1024u;
  static constexpr int kThreads = kConv ? 320 : 192;
  static_assert(kStage0 % 1024 == 0 && kStageBytes % 1024 == 0, "operand tiles need 1024-byte alignment");
  static_assert(kAlloc <= 232448, "shared memory");
};

template <int D, bool F32IO, bool DKDV>
__global__ void __launch_bounds__(BwdSmem<D, F32IO, DKDV>::kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ BwdParams p) {
  using L = BwdSmem<D, F32IO, DKDV>;
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  constexpr uint32_t OPB = TileGeom<D>::kOpBytes;
  constexpr int NS = L::kStages;
  constexpr int kTerms = F32IO ? 3 : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_rtma = bars + 0;             // resident tiles (+ rotary rows) landed
  uint64_t* bar_rconv = bars + 1;            // resident tiles rotated (count 128)
  uint64_t* bar_tma = bars + 2;              // [NS] column tiles landed
  uint64_t* bar_conv = bars + 2 + NS;        // [NS] column tiles rotated (count 128)
  uint64_t* bar_empty = bars + 2 + 2 * NS;   // [NS] MMAs done with the stage
  uint64_t* bar_s = bars + 2 + 3 * NS;       // S landed
  uint64_t* bar_dp = bar_s + 1;              // dP landed
  uint64_t* bar_p = bar_s + 2;               // rows read S, wrote P (count 128)
  uint64_t* bar_ds = bar_s + 3;              // rows wrote dS (count 128)
  uint64_t* bar_dk = bar_s + 4;              // dS MMA of an item done
  uint64_t* bar_fin = bar_s + 5;
  uint64_t* bar_res = L::kConv ? bar_rconv : bar_rtma;  // resident operands ready
  uint64_t* bar_full = L::kConv ? bar_conv : bar_tma;   // column operands ready
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const float2* rope_off = reinterpret_cast<const float2*>(smem + L::kRope);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const WaitCtl wc{p.err, p.wait_limit, abort_flag};

  // ---- work decomposition
  // DKDV: blockIdx -> (key tile ascending = most causal work first, b, g)
  // DQ:   blockIdx -> (query tile descending, b, h)
  int b, rt, head_r, n_items, c0;
  if (DKDV) {
    const int n_bg = p.B * p.Hkv;
    rt = int(blockIdx.x) / n_bg;
    const int bg = int(blockIdx.x) % n_bg;
    b = bg / p.Hkv;
    head_r = bg % p.Hkv;
    c0 = p.causal ? rt : 0;                       // first query tile
    n_items = p.G * (p.n_tiles - c0);
  } else {
    const int n_bh = p.B * p.Hq;
    rt = p.n_tiles - 1 - int(blockIdx.x) / n_bh;
    const int bh = int(blockIdx.x) % n_bh;
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
    mbar_init(bar_rconv, 128);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_tma[s], 1);
      mbar_init(&bar_conv[s], 128);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 128);
    mbar_init(bar_ds, 128);
    mbar_init(bar_dk, 1);
    mbar_init(bar_fin, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  constexpr uint32_t kColS = 0, kColDP = 128, kColAcc1 = 256, kColAcc2 = 256 + D, kColP = 384, kColPlo = 448;

  if (warp == 5) {
    // ------------------------------------------------------------ TMA
    if ((tid & 31) == 0) {
      const CUtensorMap* m_r1 = DKDV ? &p.tm_k : &p.tm_q;
      const CUtensorMap* m_r2 = DKDV ? &p.tm_v : &p.tm_do;
      const CUtensorMap* m_c1 = DKDV ? &p.tm_q : &p.tm_k;
      const CUtensorMap* m_c2 = DKDV ? &p.tm_do : &p.tm_v;
      const CUtensorMap* m_r1l = DKDV ? &p.tm_k_lo : &p.tm_q_lo;
      const CUtensorMap* m_r2l = DKDV ? &p.tm_v_lo : &p.tm_do_lo;
      const CUtensorMap* m_c1l = DKDV ? &p.tm_q_lo : &p.tm_k_lo;
      const CUtensorMap* m_c2l = DKDV ? &p.tm_do_lo : &p.tm_v_lo;
      prefetch_tmap(m_r1);
      prefetch_tmap(m_r2);
      prefetch_tmap(m_c1);
      prefetch_tmap(m_c2);
      const bool rot = L::kConv && p.rope != nullptr;
      const uint32_t rope_bytes = rot ? uint32_t(min(p.T, kRopeRows)) * (D / 2) * 8 : 0;
      const uint32_t base_bytes = rot ? L::kBase : 0;
      const float2* base_table = rot ? p.rope + size_t(p.T) * (D / 2) : nullptr;
      auto load_tile = [&](uint8_t* dst, const CUtensorMap* hi, const CUtensorMap* lo, int head, int row0,
                           uint64_t* bar) {
        tma_load_4d(dst, hi, 0, head, row0, b, bar);
        if (F32IO) tma_load_4d(dst + OPB, lo, 0, head, row0, b, bar);
      };
      mbar_arrive_expect_tx(bar_rtma, 2 * L::kTile + rope_bytes + base_bytes);
      load_tile(smem + L::kR1, m_r1, m_r1l, head_r, rt * kTileRows, bar_rtma);
      load_tile(smem + L::kR2, m_r2, m_r2l, head_r, rt * kTileRows, bar_rtma);
      if (rot) {
        bulk_load(smem + L::kRope, p.rope, rope_bytes, bar_rtma);
        bulk_load(smem + L::kR1Base, base_table + size_t(2 * rt) * (D / 2), base_bytes, bar_rtma);
      }
      int armed = 0;
      for (int k = 0; k < n_items; ++k) {
        const int s = k % NS;
        if (k >= NS && !wait_thread(&bar_empty[s], ((k / NS) - 1) & 1, wc, kErrWaitEmpty)) break;
        uint8_t* st = smem + L::kStage0 + s * L::kStageBytes;
        const int ch = item_head(k), ct = item_tile(k);
        mbar_arrive_expect_tx(&bar_tma[s], 2 * L::kTile + base_bytes + (DKDV ? 1024 : 0));
        load_tile(st, m_c1, m_c1l, ch, ct * kTileRows, &bar_tma[s]);
        load_tile(st + L::kTile, m_c2, m_c2l, ch, ct * kTileRows, &bar_tma[s]);
        if (rot) bulk_load(st + L::kCBase, base_table + size_t(2 * ct) * (D / 2), base_bytes, &bar_tma[s]);
        if (DKDV)  // LSE*log2e then Dv of the 128 queries of this column tile
          tma_load_3d(st + L::kColVec, &p.tm_ws, ct * kTileRows, 0, b * p.Hq + ch, &bar_tma[s]);
        armed = k + 1;
      }
      if (*abort_flag) {
        for (int k = max(0, armed - NS); k < armed; ++k) drain_wait(&bar_tma[k % NS], (k / NS) & 1, wc);
        drain_wait(bar_rtma, 0, wc);
      }
    }
    __syncwarp();
  } else if (L::kConv && warp >= 6) {
    // ------------------------------------------------------------ converter (bf16: in-place RoPE)
    const int pt = tid - 192;
    uint32_t conv_count = 0;  // unused: bf16 tiles need no rendezvous
    const float2* r1base = p.rope ? reinterpret_cast<const float2*>(smem + L::kR1Base) : nullptr;
    bool ok = wait_warp(bar_rtma, 0, wc, kErrWaitProducer);
    if (ok) {
      prepare_tile<D, false, true>(smem + L::kR1, rope_off, r1base, rt * kTileRows, p.T, nullptr, conv_count, wc,
                                   pt);
      fence_async_smem();
      mbar_arrive(bar_rconv);
    }
    for (int k = 0; ok && k < n_items; ++k) {
      const int s = k % NS;
      if (!wait_warp(&bar_tma[s], (k / NS) & 1, wc, kErrWaitProducer)) break;
      uint8_t* st = smem + L::kStage0 + s * L::kStageBytes;
      const float2* cbase = p.rope ? reinterpret_cast<const float2*>(st + L::kCBase) : nullptr;
      prepare_tile<D, false, true>(st, rope_off, cbase, item_tile(k) * kTileRows, p.T, nullptr, conv_count, wc,
                                   pt);
      fence_async_smem();
      mbar_arrive(&bar_conv[s]);
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if ((tid & 31) == 0) {
      constexpr uint32_t idSS = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idAcc = idesc_bf16(128, D, 0, 1);
      const uint32_t sR1 = smem_u32(smem + L::kR1), sR2 = smem_u32(smem + L::kR2);
      constexpr uint32_t accG = DKDV ? kColAcc2 : kColAcc1;  // accumulator of dS C1
      auto stage_c1 = [&](int k) { return smem_u32(smem + L::kStage0 + (k % NS) * L::kStageBytes); };
      // acc += dS_k C1_k, then release the stage of item k
      auto issue_ds = [&](int k) -> bool {
        if (!wait_thread(bar_ds, k & 1, wc, kErrWaitSoftmax)) return false;
        tc_fence_after();
        const uint32_t sC1 = stage_c1(k);
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk)
          mma_ts(tbase + accG, tbase + kColDP + kk * 8, smem_desc(sC1 + kk * 16 * RB, RB, kTileRows * RB), idAcc,
                 (k | kk) != 0);
        tc_commit(&bar_empty[k % NS]);
        tc_commit(bar_dk);
        return true;
      };
      bool ok = wait_thread(bar_res, 0, wc, kErrWaitProducer);
      for (int k = 0; ok && k < n_items; ++k) {
        const int s = k % NS;
        if (!wait_thread(&bar_full[s], (k / NS) & 1, wc, kErrWaitProducer)) { ok = false; break; }
        // S_k overwrites S_{k-1}: the rows must have read it
        if (k > 0 && !wait_thread(bar_p, (k - 1) & 1, wc, kErrWaitSoftmax)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sC1 = stage_c1(k), sC2 = sC1 + L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int term = 0; term < kTerms; ++term)
            mma_ss(tbase + kColS, smem_desc(sR1 + (term == 2 ? OPB : 0) + kk * 32, RB, 16),
                   smem_desc(sC1 + (term == 1 ? OPB : 0) + kk * 32, RB, 16), idSS, (kk | term) != 0);
        tc_commit(bar_s);
        if (k > 0) {
          // dP_k overwrites dS_{k-1}: issue its MMA and wait until it has run
          if (!issue_ds(k - 1) || !wait_thread(bar_dk, (k - 1) & 1, wc, kErrWaitMma)) { ok = false; break; }
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int term = 0; term < kTerms; ++term)
            mma_ss(tbase + kColDP, smem_desc(sR2 + (term == 2 ? OPB : 0) + kk * 32, RB, 16),
                   smem_desc(sC2 + (term == 1 ? OPB : 0) + kk * 32, RB, 16), idSS, (kk | term) != 0);
        tc_commit(bar_dp);
        if (DKDV) {
          if (!wait_thread(bar_p, k & 1, wc, kErrWaitSoftmax)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTileRows / 16; ++kk)
            mma_ts(tbase + kColAcc1, tbase + kColP + kk * 8, smem_desc(sC2 + kk * 16 * RB, RB, kTileRows * RB),
                   idAcc, (k | kk) != 0);
        }
      }
      if (ok && n_items > 0) issue_ds(n_items - 1);
      tc_commit(bar_fin);
      drain_wait(bar_fin, 0, wc);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ rows
    const int r = tid;
    const int row = rt * kTileRows + r;  // key position (DKDV) or query position (DQ)
    const uint32_t lane_base = tmem_addr(tbase, uint32_t(warp) * 32, 0);
    float row_lse2 = 0.f, row_dv = 0.f;
    if (!DKDV) {  // padded rows read +inf / 0, so their P and dS vanish
      const float* w = p.ws + (size_t(b) * p.Hq + head_r) * 2 * p.Tp + row;
      row_lse2 = __ldg(w);
      row_dv = __ldg(w + p.Tp);
    }
    bool ok = true;
    for (int k = 0; k < n_items; ++k) {
      const int s = k % NS;
      const float* colvec = reinterpret_cast<const float*>(smem + L::kStage0 + s * L::kStageBytes + L::kColVec);
      const int ct = item_tile(k);
      // DKDV reads the per-column LSE/Dv the TMA landed in the stage
      if (DKDV && !wait_warp(&bar_tma[s], (k / NS) & 1, wc, kErrWaitProducer)) { ok = false; break; }
      if (!wait_warp(bar_s, k & 1, wc, kErrWaitMma)) { ok = false; break; }
      tc_fence_after();
      const int col0 = ct * kTileRows;
      const bool diag = p.causal && ct == rt;
      const bool tail = col0 + kTileRows > p.T;
      // ---- P phase: P = exp2(s * scale_log2 - LSE*log2e), masked, kept in TMEM
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + kColS + 32 * c, rr);
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float pv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int cc = 32 * c + 2 * i + e;
            const float l2 = DKDV ? colvec[cc] : row_lse2;  // +inf past T: P = 0
            float v = ex2(fmaf(__uint_as_float(rr[2 * i + e]), p.scale_log2, -l2));
            if (DKDV) {
              if (diag && row > col0 + cc) v = 0.f;  // key after query
            } else {
              if ((diag && col0 + cc > row) || (tail && col0 + cc >= p.T)) v = 0.f;
            }
            pv[e] = v;
          }
          if (F32IO) {
            split_bf16(pv[0], pv[1], hi[i], lo[i]);
          } else {
            hi[i] = pack_bf16(pv[0], pv[1]);
          }
        }
        tmem_st16(lane_base + kColP + 16 * c, hi);
        if (F32IO) tmem_st16(lane_base + kColPlo + 16 * c, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p);
      // ---- dS phase: dS = P (dP - Dv), bf16, over dP in TMEM
      if (!wait_warp(bar_dp, k & 1, wc, kErrWaitMma)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32], ph[16], pl[16];
        tmem_ld32(lane_base + kColDP + 32 * c, rr);
        tmem_ld16(lane_base + kColP + 16 * c, ph);
        if (F32IO) tmem_ld16(lane_base + kColPlo + 16 * c, pl);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int cc = 32 * c + 2 * i;
          float p0 = bf16_lo_f(ph[i]), p1 = bf16_hi_f(ph[i]);
          if (F32IO) {
            p0 += bf16_lo_f(pl[i]);
            p1 += bf16_hi_f(pl[i]);
          }
          const float d0 = DKDV ? colvec[128 + cc] : row_dv;
          const float d1 = DKDV ? colvec[128 + cc + 1] : row_dv;
          pk[i] = pack_bf16(p0 * (__uint_as_float(rr[2 * i]) - d0), p1 * (__uint_as_float(rr[2 * i + 1]) - d1));
        }
        // columns [16c, 16c+16) of dP were read in chunk c/2 <= c already
        tmem_st16(lane_base + kColDP + 16 * c, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_ds);
    }
    if (ok && wait_warp(bar_fin, 0, wc, kErrWaitMma)) {
      tc_fence_after();
      // TMEM loads are warp-collective: every lane loads, only valid rows store
      float acc[D];
      if (DKDV) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(lane_base + kColAcc1 + 32 * c, rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[32 * c + i] = __uint_as_float(rr[i]);
        }
        if (row < p.T) store_row<D, F32IO>(p.dV, b, row, head_r, p.T, p.Hkv, acc);
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + (DKDV ? kColAcc2 : kColAcc1) + 32 * c, rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[32 * c + i] = __uint_as_float(rr[i]) * p.scale;
      }
      if (row < p.T) {
        if (p.rope) {
          // gradient w.r.t. the un-rotated input: apply R_t^T
          const float4* tp = reinterpret_cast<const float4*>(p.rope + size_t(row) * (D / 2));
#pragma unroll
          for (int i = 0; i < D / 4; ++i) {
            const float4 cs = __ldg(tp + i);
            rot2(acc[4 * i], acc[4 * i + 1], cs.x, -cs.y);
            rot2(acc[4 * i + 2], acc[4 * i + 3], cs.z, -cs.w);
          }
        }
        if (DKDV)
          store_row<D, F32IO>(p.dK, b, row, head_r, p.T, p.Hkv, acc);
        else
          store_row<D, F32IO>(p.dQ, b, row, head_r, p.T, p.Hq, acc);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace nea
