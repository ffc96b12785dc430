// Forward kernel: tiled causal GQA attention with RoPE on the tcgen05 tensor
// cores ("NanoEuler" write-up, aimsg.uk, section 4 "GPU version": tiled
// FlashAttention with an online softmax, the T x T matrix never resident;
// the pages' own kernel stages K/V tiles in shared memory and loops over them
// per query block -- smartinfralog.com post, "Tiled FlashAttention" section).
//
// One CTA computes a 128-row query tile of one (batch, query head):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r; reads S from
//              TMEM, masks, keeps the running max m and sum l, writes
//              P = exp(s - m) back into the same TMEM columns as bf16 (hi and
//              lo parts for float32 storage), rescales O in TMEM when m grows
//              by more than 2^8, and writes O / l and LSE at the end.
//   warps 4-7  producer: loads the query tile once, then key/value tiles into
//              a two-stage ring, applying RoPE to Q and K on the way.
//   warp 8     MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM
//              score buffers, then O += P_j V_j with P_j read from TMEM.
// Causal tiles above the diagonal are never visited; only the diagonal tile
// and a ragged last tile are masked.  Key/value tiles are visited in order, so
// the issue of S_{j+1} overlaps the softmax of tile j.
#pragma once

#include "nea_tiles.cuh"

namespace nea {

struct FwdParams {
  const void* Q;
  const void* K;
  const void* V;
  void* O;
  float* LSE;
  const float2* rope;  // [T][D/2] (cos, sin) or nullptr when the rotation is off
  int B, T, Hq, Hkv, G;
  int n_tiles;         // ceil(T / 128)
  int causal;
  float scale_log2;    // log2(e) / sqrt(D)
  int* err;
  unsigned long long wait_limit;
  int debug;
};

template <int D, bool F32IO>
struct FwdSmem {
  static constexpr int kParts = F32IO ? 2 : 1;
  static constexpr int kStages = 2;
  static constexpr uint32_t kTile = TileGeom<D>::kTileBytes;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kStage0 = kQ + kParts * kTile;
  static constexpr uint32_t kStageBytes = 2 * kParts * kTile;  // K parts, then V parts
  static constexpr uint32_t kBars = kStage0 + kStages * kStageBytes;
  static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 1 + 1;
  static constexpr uint32_t kMisc = kBars + 8 * kNumBars;
  static constexpr uint32_t kUsed = kMisc + 16;
  // +1024 for manual alignment; at least 120 KB so two CTAs never share an SM
  // (each allocates all 512 TMEM columns).
  static constexpr uint32_t kAlloc = (kUsed + 1024 > 120u * 1024u) ? kUsed + 1024 : 120u * 1024u;
};

template <int D, bool F32IO>
__global__ void __launch_bounds__(288, 1) attn_fwd_kernel(const __grid_constant__ FwdParams p) {
  using L = FwdSmem<D, F32IO>;
  constexpr uint32_t RB = TileGeom<D>::kRowBytes;
  constexpr int NS = L::kStages;
  constexpr int kTerms = F32IO ? 3 : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_full = bars + 1;             // [NS]
  uint64_t* bar_empty = bars + 1 + NS;       // [NS]
  uint64_t* bar_s = bars + 1 + 2 * NS;       // [2]
  uint64_t* bar_p = bars + 3 + 2 * NS;       // [2]
  uint64_t* bar_o = bars + 5 + 2 * NS;
  uint64_t* bar_fin = bars + 6 + 2 * NS;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int n_bh = p.B * p.Hq;
  const int qt = p.n_tiles - 1 - int(blockIdx.x) / n_bh;  // longest causal rows first
  const int bh = int(blockIdx.x) % n_bh;
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / p.G;
  const int n_kv = p.causal ? qt + 1 : p.n_tiles;
  const WaitCtl wc{p.err, p.wait_limit, abort_flag};

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar_q, 128);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_full[s], 128);
      mbar_init(&bar_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_s[s], 1);
      mbar_init(&bar_p[s], 128);
    }
    mbar_init(bar_o, 1);
    mbar_init(bar_fin, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  constexpr uint32_t kColO = 256;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ producer
    const int pt = tid - 128;
    load_tile<D, F32IO, true>(smem + L::kQ, p.Q, b, qt * kTileRows, h, p.T, p.Hq, p.rope, pt);
    fence_async_smem();
    if (!(p.debug & 1)) mbar_arrive(bar_q);
    for (int j = 0; j < n_kv; ++j) {
      const int s = j % NS;
      if (j >= NS && !wait_warp(&bar_empty[s], ((j / NS) - 1) & 1, wc, kErrWaitEmpty)) break;
      uint8_t* st = smem + L::kStage0 + s * L::kStageBytes;
      load_tile<D, F32IO, true>(st, p.K, b, j * kTileRows, g, p.T, p.Hkv, p.rope, pt);
      load_tile<D, F32IO, false>(st + L::kParts * L::kTile, p.V, b, j * kTileRows, g, p.T, p.Hkv, nullptr, pt);
      fence_async_smem();
      mbar_arrive(&bar_full[s]);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if ((tid & 31) == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);
      const uint32_t sQ = smem_u32(smem + L::kQ);
      auto issue_s = [&](int j) -> bool {
        const int s = j % NS;
        if (!wait_thread(&bar_full[s], (j / NS) & 1, wc, kErrWaitProducer)) return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + L::kStage0 + s * L::kStageBytes);
        const uint32_t dS = tbase + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
          for (int term = 0; term < kTerms; ++term) {
            // float32 storage: hi*hi + hi*lo + lo*hi
            const uint32_t qa = sQ + (term == 2 ? L::kTile : 0) + kk * 32;
            const uint32_t kb = sK + (term == 1 ? L::kTile : 0) + kk * 32;
            mma_ss(dS, smem_desc(qa, RB, 16), smem_desc(kb, RB, 16), idS, (kk | term) != 0);
          }
        }
        tc_commit(&bar_s[j & 1]);
        return true;
      };
      bool ok = wait_thread(bar_q, 0, wc, kErrWaitProducer) && issue_s(0);
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv) {
          // the score buffer of tile j+1 still holds P_{j-1}: wait for PV_{j-1}
          if (j >= 1 && !wait_thread(bar_o, (j - 1) & 1, wc, kErrWaitMma)) break;
          if (!issue_s(j + 1)) break;
        }
        if (!wait_thread(&bar_p[j & 1], (j >> 1) & 1, wc, kErrWaitSoftmax)) break;
        tc_fence_after();
        const int s = j % NS;
        const uint32_t sV = smem_u32(smem + L::kStage0 + s * L::kStageBytes + L::kParts * L::kTile);
        const uint32_t pcol = tbase + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk) {
#pragma unroll
          for (int term = 0; term < kTerms; ++term) {
            // float32 storage: Phi*Vhi + Phi*Vlo + Plo*Vhi
            const uint32_t pa = pcol + (term == 2 ? 64 : 0) + kk * 8;
            const uint32_t vb = sV + (term == 1 ? L::kTile : 0) + kk * 16 * RB;
            mma_ts(tbase + kColO, pa, smem_desc(vb, RB, kTileRows * RB), idO, (j | kk | term) != 0);
          }
        }
        tc_commit(bar_o);
        tc_commit(&bar_empty[s]);
      }
      tc_commit(bar_fin);
      wait_thread(bar_fin, 0, wc, kErrWaitMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int r = tid;  // query row inside the tile, TMEM lane
    const int q = qt * kTileRows + r;
    const uint32_t lane_base = tmem_addr(tbase, uint32_t(warp) * 32, 0);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!wait_warp(&bar_s[j & 1], (j >> 1) & 1, wc, kErrWaitMma)) { ok = false; break; }
      tc_fence_after();
      const uint32_t scol = lane_base + (j & 1) * 128;
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tmem_ld32(scol + 32 * c, rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(rr[i]);
      }
      const int kv0 = j * kTileRows;
      if ((p.causal && j == qt) || kv0 + kTileRows > p.T) {
        const int lim = p.causal ? min(q, p.T - 1) : p.T - 1;  // last visible key
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (kv0 + c > lim) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
      const float m_tile = mx * p.scale_log2;
      float alpha = 1.f;
      if (m_tile > m_run + 8.f) {  // keep a stale max unless it grew by > 2^8
        alpha = ex2(m_run - m_tile);
        m_run = m_tile;
      }
      l_run *= alpha;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2(fmaf(s[32 * c + 2 * i], p.scale_log2, -m_run));
          const float p1 = ex2(fmaf(s[32 * c + 2 * i + 1], p.scale_log2, -m_run));
          l_run += p0 + p1;
          if (F32IO) {
            split_bf16(p0, p1, hi[i], lo[i]);
          } else {
            hi[i] = pack_bf16(p0, p1);
          }
        }
        tmem_st16(scol + 16 * c, hi);
        if (F32IO) tmem_st16(scol + 64 + 16 * c, lo);
      }
      if (__any_sync(kFullMask, alpha != 1.f && j > 0)) {
        // O holds sum over tiles < j: wait until PV_{j-1} has landed, rescale
        if (!wait_warp(bar_o, (j - 1) & 1, wc, kErrWaitMma)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(lane_base + kColO + 32 * c, rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
          tmem_st32(lane_base + kColO + 32 * c, rr);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar_p[j & 1]);
    }
    // bar_o can trail by two phases here; the issuer's final commit cannot.
    if (ok && wait_warp(bar_fin, 0, wc, kErrWaitMma)) {
      tc_fence_after();
      float o[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + kColO + 32 * c, rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[32 * c + i] = __uint_as_float(rr[i]);
      }
      if (q < p.T) {
        const float inv = 1.f / l_run;
#pragma unroll
        for (int i = 0; i < D; ++i) o[i] *= inv;
        store_row<D, F32IO>(p.O, b, q, h, p.T, p.Hq, o);
        // LSE = ln(2^m * l) with m in log2 units of the scaled scores
        p.LSE[(size_t(b) * p.Hq + h) * p.T + q] = (m_run + log2f(l_run)) * 0.69314718055994531f;
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
