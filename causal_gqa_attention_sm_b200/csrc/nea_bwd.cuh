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
// Warp roles as in the forward: warps 0-3 own the 128 rows (TMEM lanes),
// warps 4-7 load tiles (RoPE fused), warp 8 issues the MMAs:
//   S_rc  = R1 C1^T      (R1 = K' or Q', C1 = Q' or K')   -> TMEM cols [0,128)
//   dP_rc = R2 C2^T      (R2 = V or dO,  C2 = dO or V)    -> TMEM cols [128,256)
//   DKDV: acc_v += P  C2   (P from TMEM, C2 = dO as MN-major B)
//         acc_k += dS C1   (dS from TMEM, C1 = Q' as MN-major B)
//   DQ:   acc   += dS C1   (C1 = K')
// With float32 storage S and dP use the three-term split-bf16 product; the
// gradient products use the bf16 high parts.
#pragma once

#include "nea_tiles.cuh"

namespace nea {

// ---------------------------------------------------------------- row term
// Dv[b][h][t] = sum_d dO[b][t][h][d] * O[b][t][h][d], one group of D/ELEMS
// lanes per row.
template <int D, bool F32IO>
__global__ void __launch_bounds__(256) attn_bwd_rowterm_kernel(const void* __restrict__ O,
                                                               const void* __restrict__ dO,
                                                               float* __restrict__ Dv, int rows, int T, int Hq) {
  constexpr int kElems = F32IO ? 4 : 8;    // elements per 16-byte chunk
  constexpr int kLanes = D / kElems;       // lanes per row: 4, 8 or 16
  const long gtid = long(blockIdx.x) * blockDim.x + threadIdx.x;
  const long row = gtid / kLanes;
  const int c = int(gtid % kLanes);
  float acc = 0.f;
  if (row < rows) {
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
#pragma unroll
  for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(kFullMask, acc, off);
  if (row < rows && c == 0) {
    // row = (b * T + t) * Hq + h  ->  Dv[(b * Hq + h) * T + t]
    const long bt = row / Hq;
    const int h = int(row % Hq);
    const long b = bt / T;
    const int t = int(bt % T);
    Dv[(b * Hq + h) * T + t] = acc;
  }
}

// ---------------------------------------------------------------- main kernel
struct BwdParams {
  const void* Q;
  const void* K;
  const void* V;
  const void* dO;
  const float* LSE;   // [B][Hq][T]
  const float* Dv;    // [B][Hq][T]
  void* dQ;
  void* dK;
  void* dV;
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
  static constexpr int kParts = F32IO ? 2 : 1;
  static constexpr int kStages = 2;
  static constexpr uint32_t kTile = TileGeom<D>::kTileBytes;
  static constexpr uint32_t kR1 = 0;
  static constexpr uint32_t kR2 = kR1 + kParts * kTile;
  static constexpr uint32_t kStage0 = kR2 + kParts * kTile;
  static constexpr uint32_t kColVec = 2 * kParts * kTile;            // offset of per-column LSE/Dv
  static constexpr uint32_t kStageBytes = kColVec + (DKDV ? 2 * 128 * 4 : 0);
  static constexpr uint32_t kBars = kStage0 + kStages * kStageBytes;
  static constexpr int kNumBars = 1 + 2 * kStages + 4 + 1 + 1;
  static constexpr uint32_t kMisc = kBars + 8 * kNumBars;
  static constexpr uint32_t kUsed = kMisc + 16;
  static constexpr uint32_t kAlloc = (kUsed + 1024 > 120u * 1024u) ? kUsed + 1024 : 120u * 1024u;
};

template <int D, bool F32IO, bool DKDV>
__global__ void __launch_bounds__(288, 1) attn_bwd_kernel(const __grid_constant__ BwdParams p) {
  using L = BwdSmem<D, F32IO, DKDV>;
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  constexpr int NS = L::kStages;
  constexpr int kTerms = F32IO ? 3 : 1;
  constexpr float kLog2e = 1.4426950408889634f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_res = bars + 0;
  uint64_t* bar_full = bars + 1;            // [NS]
  uint64_t* bar_empty = bars + 1 + NS;      // [NS]
  uint64_t* bar_s = bars + 1 + 2 * NS;      // S landed
  uint64_t* bar_dp = bars + 2 + 2 * NS;     // dP landed
  uint64_t* bar_p = bars + 3 + 2 * NS;      // P written (DKDV)
  uint64_t* bar_ds = bars + 4 + 2 * NS;     // dS written
  uint64_t* bar_item = bars + 5 + 2 * NS;   // all MMAs of an item done
  uint64_t* bar_fin = bars + 6 + 2 * NS;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const WaitCtl wc{p.err, p.wait_limit, abort_flag};

  // ---- work decomposition
  // DKDV: blockIdx -> (key tile jt ascending = most causal work first, b, g)
  // DQ:   blockIdx -> (query tile it descending, b, h)
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

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar_res, 128);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_full[s], 128);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 128);
    mbar_init(bar_ds, 128);
    mbar_init(bar_item, 1);
    mbar_init(bar_fin, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  constexpr uint32_t kColS = 0, kColDP = 128, kColAcc1 = 256, kColAcc2 = 256 + D;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ producer
    const int pt = tid - 128;
    if (DKDV) {
      load_tile<D, F32IO, true>(smem + L::kR1, p.K, b, rt * kTileRows, head_r, p.T, p.Hkv, p.rope, pt);
      load_tile<D, F32IO, false>(smem + L::kR2, p.V, b, rt * kTileRows, head_r, p.T, p.Hkv, nullptr, pt);
    } else {
      load_tile<D, F32IO, true>(smem + L::kR1, p.Q, b, rt * kTileRows, head_r, p.T, p.Hq, p.rope, pt);
      load_tile<D, F32IO, false>(smem + L::kR2, p.dO, b, rt * kTileRows, head_r, p.T, p.Hq, nullptr, pt);
    }
    fence_async_smem();
    mbar_arrive(bar_res);
    for (int k = 0; k < n_items; ++k) {
      const int s = k % NS;
      if (k >= NS && !wait_warp(&bar_empty[s], ((k / NS) - 1) & 1, wc, kErrWaitEmpty)) break;
      uint8_t* st = smem + L::kStage0 + s * L::kStageBytes;
      if (DKDV) {
        const int h = head_r * p.G + k / n_ct;
        const int it = c0 + k % n_ct;
        load_tile<D, F32IO, true>(st, p.Q, b, it * kTileRows, h, p.T, p.Hq, p.rope, pt);
        load_tile<D, F32IO, false>(st + L::kParts * L::kTile, p.dO, b, it * kTileRows, h, p.T, p.Hq, nullptr, pt);
        float* colvec = reinterpret_cast<float*>(st + L::kColVec);
        const int q = it * kTileRows + pt;
        const size_t idx = (size_t(b) * p.Hq + h) * p.T + q;
        colvec[pt] = (q < p.T) ? __ldg(p.LSE + idx) * kLog2e : INFINITY;  // P = 0 for padding queries
        colvec[128 + pt] = (q < p.T) ? __ldg(p.Dv + idx) : 0.f;
      } else {
        const int jt = k;
        load_tile<D, F32IO, true>(st, p.K, b, jt * kTileRows, head_r / p.G, p.T, p.Hkv, p.rope, pt);
        load_tile<D, F32IO, false>(st + L::kParts * L::kTile, p.V, b, jt * kTileRows, head_r / p.G, p.T, p.Hkv,
                                   nullptr, pt);
      }
      fence_async_smem();
      mbar_arrive(&bar_full[s]);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if ((tid & 31) == 0) {
      constexpr uint32_t idSS = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idAcc = idesc_bf16(128, D, 0, 1);
      const uint32_t sR1 = smem_u32(smem + L::kR1), sR2 = smem_u32(smem + L::kR2);
      bool ok = wait_thread(bar_res, 0, wc, kErrWaitProducer);
      for (int k = 0; ok && k < n_items; ++k) {
        const int s = k % NS;
        if (!wait_thread(&bar_full[s], (k / NS) & 1, wc, kErrWaitProducer)) break;
        // S and dP overwrite the P / dS columns the previous item's MMAs read
        if (k > 0 && !wait_thread(bar_item, (k - 1) & 1, wc, kErrWaitMma)) break;
        tc_fence_after();
        const uint32_t sC1 = smem_u32(smem + L::kStage0 + s * L::kStageBytes);
        const uint32_t sC2 = sC1 + L::kParts * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int term = 0; term < kTerms; ++term)
            mma_ss(tbase + kColS, smem_desc(sR1 + (term == 2 ? L::kTile : 0) + kk * 32, RB, 16),
                   smem_desc(sC1 + (term == 1 ? L::kTile : 0) + kk * 32, RB, 16), idSS, (kk | term) != 0);
        tc_commit(bar_s);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int term = 0; term < kTerms; ++term)
            mma_ss(tbase + kColDP, smem_desc(sR2 + (term == 2 ? L::kTile : 0) + kk * 32, RB, 16),
                   smem_desc(sC2 + (term == 1 ? L::kTile : 0) + kk * 32, RB, 16), idSS, (kk | term) != 0);
        tc_commit(bar_dp);
        if (DKDV) {
          if (!wait_thread(bar_p, k & 1, wc, kErrWaitSoftmax)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTileRows / 16; ++kk)
            mma_ts(tbase + kColAcc1, tbase + kColS + kk * 8, smem_desc(sC2 + kk * 16 * RB, RB, kTileRows * RB),
                   idAcc, (k | kk) != 0);
        }
        if (!wait_thread(bar_ds, k & 1, wc, kErrWaitSoftmax)) break;
        tc_fence_after();
        const uint32_t acc = DKDV ? kColAcc2 : kColAcc1;
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk)
          mma_ts(tbase + acc, tbase + kColDP + kk * 8, smem_desc(sC1 + kk * 16 * RB, RB, kTileRows * RB), idAcc,
                 (k | kk) != 0);
        tc_commit(&bar_empty[s]);
        tc_commit(bar_item);
      }
      tc_commit(bar_fin);
      wait_thread(bar_fin, 0, wc, kErrWaitMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ rows
    const int r = tid;
    const int row = rt * kTileRows + r;  // key position (DKDV) or query position (DQ)
    const uint32_t lane_base = tmem_addr(tbase, uint32_t(warp) * 32, 0);
    float row_lse2 = 0.f, row_dv = 0.f;
    if (!DKDV) {
      const size_t idx = (size_t(b) * p.Hq + head_r) * p.T + row;
      row_lse2 = (row < p.T) ? __ldg(p.LSE + idx) * kLog2e : INFINITY;
      row_dv = (row < p.T) ? __ldg(p.Dv + idx) : 0.f;
    }
    bool ok = true;
    for (int k = 0; k < n_items; ++k) {
      const int s = k % NS;
      const float* colvec = reinterpret_cast<const float*>(smem + L::kStage0 + s * L::kStageBytes + L::kColVec);
      const int ct = DKDV ? c0 + k % n_ct : k;   // column tile index
      // DKDV reads the stage's per-column LSE/Dv written by the producer
      if (DKDV && !wait_warp(&bar_full[s], (k / NS) & 1, wc, kErrWaitProducer)) { ok = false; break; }
      if (!wait_warp(bar_s, k & 1, wc, kErrWaitMma)) { ok = false; break; }
      tc_fence_after();
      float pr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + kColS + 32 * c, rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) pr[32 * c + i] = __uint_as_float(rr[i]);
      }
      // P = exp(scale * s - LSE); causal mask: key position > query position
      const int col0 = ct * kTileRows;
      const bool diag = p.causal && ct == rt;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float l2 = DKDV ? colvec[c] : row_lse2;
        float v = ex2(fmaf(pr[c], p.scale_log2, -l2));
        if (DKDV) {
          if (diag && row > col0 + c) v = 0.f;
        } else {
          if ((diag && col0 + c > row) || col0 + c >= p.T) v = 0.f;
        }
        pr[c] = v;
      }
      if (DKDV) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(pr[32 * c + 2 * i], pr[32 * c + 2 * i + 1]);
          tmem_st16(lane_base + kColS + 16 * c, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p);
      }
      if (!wait_warp(bar_dp, k & 1, wc, kErrWaitMma)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + kColDP + 32 * c, rr);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c0i = 32 * c + 2 * i;
          const float d0 = DKDV ? colvec[128 + c0i] : row_dv;
          const float d1 = DKDV ? colvec[128 + c0i + 1] : row_dv;
          const float ds0 = pr[c0i] * (__uint_as_float(rr[2 * i]) - d0);
          const float ds1 = pr[c0i + 1] * (__uint_as_float(rr[2 * i + 1]) - d1);
          pk[i] = pack_bf16(ds0, ds1);
        }
        // columns [16c, 16c+16) were read by chunk c/2 <= c already
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
  // The epilogue reads TMEM only after all waits ended; abandoned waits may
  // leave barrier phases mismatched but nothing remains in flight: the issuer
  // drained its MMAs on bar_fin.
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace nea
