// Gradient kernel for float32 storage: the recompute-from-LSE backward of
// tiled attention with every product formed from bf16 high and low parts (the
// pages state only that each operator's backward is hand-written and
// gradient-checked: "NanoEuler" write-up, aimsg.uk, sections 3-4;
// agentlenshq.com summary, "Validation and stability"):
//
//   S = Q' K'^T,  P = exp(scale S - LSE),  dP = dO V^T,  dS = P o (dP - Dv),
//   dV += P^T dO,  dK' += scale dS^T Q',  dQ' += scale dS K',
//   dQ = R^T dQ',  dK = R^T dK'.
//
// Precision.  Every operand x is x_hi + x_lo with x_hi = bf16(x) and
// x_lo = bf16(x - x_hi) (about 16 significant bits together), and every
// product a b is formed as a_hi b_hi + a_hi b_lo + a_lo b_hi with fp32
// accumulation: finer than TF32 (11 bits) in every product.  The operand
// prologue (nea_prep.cuh) writes the hi and lo planes of Q' = RoPE(Q),
// K' = RoPE(K), V and dO and the row terms -LSE log2(e) and
// Dv = rowsum(dO o O); P and dS are split by the elementwise warps.
//
// Units (as in the bf16 kernel, nea_bwd.cuh): a dK/dV unit keeps key tile j of
// kv head g resident (K'_j, V_j) and streams the query tiles i >= j of every
// query head of the group, so the GQA reduction of dK and dV stays in TMEM; a
// dQ unit keeps query tile i of head h resident (Q'_i, dO_i) and streams the
// key tiles j <= i.
//
// Gradient products: three bf16 products of N = D per 16-row step
// (A_hi C_hi, A_hi C_lo, A_lo C_hi) into one accumulator of D columns.
//
// TMEM (D = 64): S in two buffers [0,128) and [128,256) (item k uses buffer
// k % 2; P_hi / P_lo are written over it); dP [256,384) (dS_hi / dS_lo
// over it); accumulator A [384, 384+D) (dV or dQ), accumulator B
// [384+D, 384+2D) (dK).  Column quarter q of the elementwise warps rewrites
// only its own columns [32q, 32q+32) of S and dP: hi parts in the first 16,
// lo parts in the next 16 (two bf16 per column), so no warp overwrites
// scores another still has to read.
// Issue order of the MMA thread, per item k (the streamed tiles one stage
// ahead):
//   dK/dV units:  dV(k) | S(k+1) | dK(k) | dP(k+1) | dV(k+1) | S(k+2) | ...
//   dQ units:     S(k+1) | dQ(k) | dP(k+1) | S(k+2) | ...
// S(k+1) goes to the other S buffer as soon as its tiles have landed, so the
// rows form P(k+1) while dK/dQ(k) and dP(k+1) run; dV(k) waits for P(k),
// dK/dQ(k) for dS(k) (formed while dV(k) and S(k+1) run), dP(k+1) for
// dK/dQ(k) to have read dS(k) (the wait overlaps S(k+1) or dK(k)).
// Warps: 0-15 elementwise (warp w: TMEM lanes 32 (w % 4) .. + 31, columns
// 32 (w / 4) .. + 31 of each 128-column tile; four warps per SM
// sub-partition, so that one warp's TMEM loads overlap the others' work),
// 16 MMA issue, 17 TMA.
#pragma once

#include <cuda.h>

#include "nea_bwd.cuh"

namespace nea {

template <int D>
struct Bwd32Smem {
  static constexpr uint32_t kOp = TileGeom<D>::kOpBytes;  // one bf16 plane of a tile
  static constexpr uint32_t kTile = 2 * kOp;              // hi plane, then lo plane
  static constexpr int kStages = 2;
  static constexpr uint32_t kR1 = 0;
  static constexpr uint32_t kR2 = kTile;
  static constexpr uint32_t kStage0 = 2 * kTile;
  static constexpr uint32_t kColVec = 2 * kTile;  // per-column -LSE*log2e and Dv (dK/dV units)
  static constexpr uint32_t kStageBytes = kColVec + 1024;
  static constexpr uint32_t kBars = kStage0 + kStages * kStageBytes;
  // rtma, tma[S], empty[S], s[2], dp, p, ds, dk, fin
  static constexpr int kNumBars = 1 + 2 * kStages + 7;
  static constexpr uint32_t kMisc = kBars + 8 * kNumBars;
  static constexpr uint32_t kUsed = kMisc + 16;
  static constexpr uint32_t kAlloc = kUsed + 1024 > 116u * 1024u ? kUsed + 1024 : 116u * 1024u;
  static constexpr int kRowWarps = 16;  // elementwise warps
  static constexpr int kRowThreads = 32 * kRowWarps;
  static constexpr int kThreads = kRowThreads + 64;
  static_assert(kStage0 % 1024 == 0 && kStageBytes % 1024 == 0, "operand tiles need 1024-byte alignment");
  static_assert(kAlloc <= 232448, "shared memory");
};

template <int D, bool DKDV>
__device__ __forceinline__ void attn_bwd_f32_unit(const BwdParams& p, int bid) {
  using L = Bwd32Smem<D>;
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  constexpr uint32_t OPB = L::kOp;
  constexpr int NS = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_rtma = bars + 0;        // resident tiles landed
  uint64_t* bar_tma = bars + 1;         // [NS] streamed tiles landed
  uint64_t* bar_empty = bars + 1 + NS;  // [NS] products done with the stage
  uint64_t* bar_s = bars + 1 + 2 * NS;  // [2] S landed in buffer 0 / 1
  uint64_t* bar_dp = bar_s + 2;         // dP landed
  uint64_t* bar_p = bar_s + 3;          // rows wrote P over S (all row threads; dK/dV units)
  uint64_t* bar_ds = bar_s + 4;         // rows wrote dS over dP (all row threads)
  uint64_t* bar_dk = bar_s + 5;         // all products of an item done
  uint64_t* bar_fin = bar_s + 6;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const WaitCtl wc{p.err, p.wait_limit, abort_flag};
  NEA_TRACE_STAMP(p, 0, tid == 0);

  // ---- work decomposition (as in the bf16 kernel)
  int b, rt, head_r, n_items, c0;
  if (DKDV) {
    const int n_bg = p.B * p.Hkv;
    rt = bid / n_bg;
    const int bg = bid % n_bg;
    b = bg / p.Hkv;
    head_r = bg % p.Hkv;
    c0 = p.causal ? rt : 0;
    n_items = p.G * (p.n_tiles - c0);
  } else {
    const int n_bh = p.B * p.Hq;
    rt = p.n_tiles - 1 - bid / n_bh;
    const int bh = bid % n_bh;
    b = bh / p.Hq;
    head_r = bh % p.Hq;
    c0 = 0;
    n_items = p.causal ? rt + 1 : p.n_tiles;
  }
  const int n_ct = p.n_tiles - c0;
  auto item_head = [&](int k) { return DKDV ? head_r * p.G + k / n_ct : head_r / p.G; };
  auto item_tile = [&](int k) { return DKDV ? c0 + k % n_ct : k; };

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar_rtma, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_tma[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(&bar_s[0], 1);
    mbar_init(&bar_s[1], 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, L::kRowThreads);
    mbar_init(bar_ds, L::kRowThreads);
    mbar_init(bar_dk, 1);
    mbar_init(bar_fin, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  grid_dep_wait();  // operand planes and row terms come from the prologue grid
  grid_dep_launch();
  NEA_TRACE_STAMP(p, 1, tid == 0);
  constexpr uint32_t kColS = 0, kColDP = 256, kColAccA = 384, kColAccB = 384 + D;

  constexpr int kWarpMma = L::kRowWarps, kWarpTma = L::kRowWarps + 1;
  if (warp == kWarpTma) {
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
      auto load_tile = [&](uint8_t* dst, const CUtensorMap* hi, const CUtensorMap* lo, int head, int row0,
                           uint64_t* bar) {
        tma_load_4d(dst, hi, 0, head, row0, b, bar);
        tma_load_4d(dst + OPB, lo, 0, head, row0, b, bar);
      };
      // fault-injection hook: withhold the resident tiles so every wait on
      // them runs into its limit
      const bool r_armed = !(p.debug & 2);
      if (r_armed) {
        mbar_arrive_expect_tx(bar_rtma, 2 * L::kTile);
        load_tile(smem + L::kR1, m_r1, m_r1l, head_r, rt * kTileRows, bar_rtma);
        load_tile(smem + L::kR2, m_r2, m_r2l, head_r, rt * kTileRows, bar_rtma);
      }
      NEA_TRACE_STAMP(p, 73, true);
      int armed = 0;
      for (int k = 0; k < n_items; ++k) {
        const int s = k % NS;
        if (k >= NS && !wait_thread(&bar_empty[s], ((k / NS) - 1) & 1, wc, kErrWaitEmpty)) break;
        uint8_t* st = smem + L::kStage0 + s * L::kStageBytes;
        const int ch = item_head(k), ct = item_tile(k);
        mbar_arrive_expect_tx(&bar_tma[s], 2 * L::kTile + (DKDV ? 1024 : 0));
        load_tile(st, m_c1, m_c1l, ch, ct * kTileRows, &bar_tma[s]);
        load_tile(st + L::kTile, m_c2, m_c2l, ch, ct * kTileRows, &bar_tma[s]);
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
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if ((tid & 31) == 0) {
      constexpr uint32_t idSS = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idG = idesc_bf16(128, D, 0, 1);
      const uint32_t sR1 = smem_u32(smem + L::kR1), sR2 = smem_u32(smem + L::kR2);
      auto stage_c1 = [&](int k) { return smem_u32(smem + L::kStage0 + (k % NS) * L::kStageBytes); };
      // dst (+)= R C^T from the three split products, contraction over D
      auto issue_sc = [&](uint32_t dst, uint32_t sR, uint32_t sC) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int term = 0; term < 3; ++term)  // hi*hi, hi*lo, lo*hi
            mma_ss(tbase + dst, smem_desc(sR + (term == 2 ? OPB : 0) + kk * 32, RB, 16),
                   smem_desc(sC + (term == 1 ? OPB : 0) + kk * 32, RB, 16), idSS, (kk | term) != 0);
      };
      auto issue_s = [&](int k) {
        issue_sc(kColS + 128 * (k & 1), sR1, stage_c1(k));
        tc_commit(&bar_s[k & 1]);
      };
      auto issue_dp = [&](int k) {
        issue_sc(kColDP, sR2, stage_c1(k) + L::kTile);
        tc_commit(bar_dp);
      };
      // acc (+)= A C, contraction over the 128 rows of the streamed tile, as
      // A_hi C_hi + A_hi C_lo + A_lo C_hi.  A (P or dS) sits at a_col: column
      // quarter q wrote its 32 columns' hi parts at a_col + 32 q and lo parts
      // 16 after; K-step kk (16 columns) is half kk % 2 of quarter kk / 2.
      auto issue_grad = [&](uint32_t acc, uint32_t a_col, uint32_t sC, bool first) {
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk) {
          const uint32_t a_hi = tbase + a_col + 32 * (kk >> 1) + 8 * (kk & 1);
          const uint32_t c = sC + kk * 16 * RB;
          mma_ts(tbase + acc, a_hi, smem_desc(c, RB, OPB), idG, (first && kk == 0) ? 0u : 1u);
          mma_ts(tbase + acc, a_hi, smem_desc(c + OPB, RB, OPB), idG, 1u);
          mma_ts(tbase + acc, a_hi + 16, smem_desc(c, RB, OPB), idG, 1u);
        }
      };
      bool ok = wait_thread(bar_rtma, 0, wc, kErrWaitProducer) &&
                (n_items == 0 || wait_thread(&bar_tma[0], 0, wc, kErrWaitProducer));
      if (ok && n_items > 0) {
        NEA_TRACE_STAMP(p, 72, true);
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int k = 0; ok && k < n_items; ++k) {
        const uint32_t sC1 = stage_c1(k), sC2 = sC1 + L::kTile;
        if (DKDV) {  // dV += P(k) C2(k), once the rows have written P(k) over S(k)
          if (!wait_thread(bar_p, k & 1, wc, kErrWaitSoftmax)) { ok = false; break; }
          NEA_TRACE_STAMP(p, 8 + min(k, 7), true);
          tc_fence_after();
          issue_grad(kColAccA, kColS + 128 * (k & 1), sC2, k == 0);
        }
        if (k + 1 < n_items) {
          // S(k+1) into the other buffer: its P(k-1) (or, in dQ units, S(k-1))
          // was consumed before item k-1's products completed, waited for
          // before dP(k)
          if (!wait_thread(&bar_tma[(k + 1) % NS], ((k + 1) / NS) & 1, wc, kErrWaitProducer)) { ok = false; break; }
          NEA_TRACE_STAMP(p, 24 + min(k, 7), true);
          tc_fence_after();
          issue_s(k + 1);
        }
        // dK (dK/dV units) or dQ (dQ units) += dS(k) C1(k), then release the stage
        if (!wait_thread(bar_ds, k & 1, wc, kErrWaitSoftmax)) { ok = false; break; }
        NEA_TRACE_STAMP(p, 16 + min(k, 7), true);
        tc_fence_after();
        issue_grad(DKDV ? kColAccB : kColAccA, kColDP, sC1, k == 0);
        tc_commit(&bar_empty[k % NS]);
        tc_commit(bar_dk);
        if (k + 1 < n_items) {
          // dP(k+1) overwrites dS(k): wait for item k's products
          if (!wait_thread(bar_dk, k & 1, wc, kErrWaitMma)) { ok = false; break; }
          NEA_TRACE_STAMP(p, 32 + min(k, 7), true);
          tc_fence_after();
          issue_dp(k + 1);
        }
      }
      tc_commit(bar_fin);
      drain_wait(bar_fin, 0, wc);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise (warps 0-15)
    const int q = warp >> 2;             // column quarter
    const int r = (warp & 3) * 32 + (tid & 31);
    const int row = rt * kTileRows + r;  // key position (dK/dV) or query position (dQ)
    const int cb = 32 * q;               // first column of this warp
    const uint32_t lane_base = tmem_addr(tbase, uint32_t(warp & 3) * 32, 0);
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    uint64_t nl2_row = 0, dv_row = 0;
    if (!DKDV) {  // padded rows read -inf / 0, so their P and dS vanish
      const float* w = p.ws + (size_t(b) * p.Hq + head_r) * 2 * p.Tp + row;
      const float nl2 = __ldg(w), dv = __ldg(w + p.Tp);
      nl2_row = f2_pack(nl2, nl2);
      dv_row = f2_pack(dv, dv);
    }
    // writes 32 values as bf16 hi parts at col, lo parts at col + 16
    auto store_split = [&](uint32_t col, const float* v) {
      uint32_t hi[16], lo[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) split_bf16(v[2 * i], v[2 * i + 1], hi[i], lo[i]);
      tmem_st16(col, hi);
      tmem_st16(col + 16, lo);
    };
    bool ok = true;
    for (int k = 0; k < n_items; ++k) {
      const int s = k % NS;
      const float4* colvec =
          reinterpret_cast<const float4*>(smem + L::kStage0 + s * L::kStageBytes + L::kColVec) + cb / 4;
      const int ct = item_tile(k);
      if (DKDV && !wait_warp(&bar_tma[s], (k / NS) & 1, wc, kErrWaitProducer)) { ok = false; break; }
      if (!wait_warp(&bar_s[k & 1], (k >> 1) & 1, wc, kErrWaitMma)) { ok = false; break; }
      NEA_TRACE_STAMP(p, 40 + min(k, 7), tid == 0);
      tc_fence_after();
      const int col0 = ct * kTileRows + cb;  // position of this warp's first column
      // ---- P = exp2(s * scale_log2 - LSE*log2e), masked
      uint32_t sv[32];
      const uint32_t scol = lane_base + kColS + 128 * (k & 1) + cb;
      tmem_ld32(scol, sv);
      if ((p.causal && ct == rt) || ct * kTileRows + kTileRows > p.T) {  // same for the whole tile
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const bool masked = DKDV ? (p.causal && row > col0 + i) : ((p.causal && col0 + i > row) || col0 + i >= p.T);
          sv[i] = masked ? 0xff800000u : sv[i];
        }
      }
      float pv[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {  // four columns per step
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
      if (DKDV) {  // P hi / lo over this warp's S columns: the A operand of dV(k)
        store_split(scol, pv);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p);
        NEA_TRACE_STAMP(p, 48 + min(k, 7), tid == 0);
      }
      // ---- dS = P (dP - Dv), hi / lo over this warp's dP columns
      if (!wait_warp(bar_dp, k & 1, wc, kErrWaitMma)) { ok = false; break; }
      NEA_TRACE_STAMP(p, 56 + min(k, 7), tid == 0);
      tc_fence_after();
      float ds[32];
      {
        uint32_t rr[32];
        tmem_ld32(lane_base + kColDP + cb, rr);
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // four columns per step
          const int e = 4 * i;
          uint64_t dva = dv_row, dvb = dv_row;
          if (DKDV) {
            const float4 d = colvec[32 + i];
            dva = f2_pack(d.x, d.y);
            dvb = f2_pack(d.z, d.w);
          }
          f2_unpack(f2_mul(f2_pack(pv[e], pv[e + 1]),
                           f2_sub(f2_pack(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1])), dva)),
                    ds[e], ds[e + 1]);
          f2_unpack(f2_mul(f2_pack(pv[e + 2], pv[e + 3]),
                           f2_sub(f2_pack(__uint_as_float(rr[e + 2]), __uint_as_float(rr[e + 3])), dvb)),
                    ds[e + 2], ds[e + 3]);
        }
      }
      store_split(lane_base + kColDP + cb, ds);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_ds);
      NEA_TRACE_STAMP(p, 64 + min(k, 7), tid == 0);
    }
    // warp-uniform: every lane of a warp saw the same waits
    const bool epi = ok && wait_warp(bar_fin, 0, wc, kErrWaitMma);
    NEA_TRACE_STAMP(p, 76, tid == 0);
    if (epi) tc_fence_after();
    if (DKDV) {
      // quarter q: tensor q / 2 (dV, dK), columns [(q % 2) D/2, +D/2)
      constexpr int DH = D / 2;
      const int tensor = q >> 1, c0h = (q & 1) * DH;
      float acc[DH];
      if (epi) tmem_ld_n<DH>(lane_base + (tensor ? kColAccB : kColAccA) + c0h, acc);
      if (epi && row < p.T) {
        if (tensor) {
#pragma unroll
          for (int i = 0; i < DH; ++i) acc[i] *= p.scale;
          if (p.rope) {  // gradient w.r.t. the un-rotated input: apply R_t^T
            const float4* tp = reinterpret_cast<const float4*>(p.rope + size_t(row) * (D / 2) + c0h / 2);
#pragma unroll
            for (int i = 0; i < DH / 4; ++i) {
              const float4 cs = __ldg(tp + i);
              rot2(acc[4 * i], acc[4 * i + 1], cs.x, -cs.y);
              rot2(acc[4 * i + 2], acc[4 * i + 3], cs.z, -cs.w);
            }
          }
        }
        const size_t off = ((size_t(b) * p.T + row) * p.Hkv + head_r) * D + c0h;
        store_span<DH, true>(tensor ? p.dK : p.dV, off, acc);
      }
    } else if (epi) {
      // quarter q writes columns [q D/4, q D/4 + D/4) of the row of dQ
      constexpr int DQQ = D / 4;
      const int c0q = q * DQQ;
      float acc[DQQ];
      tmem_ld_n<DQQ>(lane_base + kColAccA + c0q, acc);
#pragma unroll
      for (int i = 0; i < DQQ; ++i) acc[i] *= p.scale;
      if (row < p.T) {
        if (p.rope) {
          const float4* tp = reinterpret_cast<const float4*>(p.rope + size_t(row) * (D / 2) + c0q / 2);
#pragma unroll
          for (int i = 0; i < DQQ / 4; ++i) {
            const float4 cs = __ldg(tp + i);
            rot2(acc[4 * i], acc[4 * i + 1], cs.x, -cs.y);
            rot2(acc[4 * i + 2], acc[4 * i + 3], cs.z, -cs.w);
          }
        }
        const size_t off = ((size_t(b) * p.T + row) * p.Hq + head_r) * D + c0q;
        store_span<DQQ, true>(p.dQ, off, acc);
      }
    }
  }
  NEA_TRACE_STAMP(p, 77, tid == 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
  NEA_TRACE_STAMP(p, 78, tid == 0);
}

template <int D>
__global__ void __launch_bounds__(Bwd32Smem<D>::kThreads, 1)
    attn_bwd_f32_kernel(const __grid_constant__ BwdParams p) {
  const int unit = p.unit0 + int(blockIdx.x);
  if (unit < p.n_dkdv)
    attn_bwd_f32_unit<D, true>(p, unit);
  else
    attn_bwd_f32_unit<D, false>(p, unit - p.n_dkdv);
}

}  // namespace nea
