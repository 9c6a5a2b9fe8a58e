// dQ of the deterministic backward, for sm_100a: one work item per (b, h, 128-row Q tile),
// dQ accumulated in TMEM over the visible KV tiles in a fixed order (no atomics), so the result
// is bitwise reproducible. The pages' call carries a `deterministic` flag
// ("FlashAttention技术解析：加速GPT训练的核心优化" §2.2).
//
// Per KV tile j (P and dS as in the main backward, transposed: here a thread owns a query row):
//   S  = Q_i K_j^T          (TMEM, 128 columns)
//   dP = dO_i V_j^T         (TMEM, 128 columns)
//   P  = exp2(S * scale * log2(e) - LSE_row * log2(e)),  dS = P * (dP - D_row)   (bf16)
//   dQ += dS K_j            (A = dS read from TMEM, written over the dP columns already read)
// dQ * scale -> bf16 -> TMA store at the end of the item.
//
// Work items come from the second counter of the workspace's counter block.
// Roles (256 threads): warp 0 TMA producer (Q_i, dO_i per item; K_j / V_j ring), warp 1 MMA
// issuer and TMEM owner, warps 4-7 P and dS (one thread per query row) and the epilogue.
// MMA order per j: S(j), dP(j), then after dS(j): S(j+1), dQ(j), dP(j+1) — S(j+1) goes into the
// S columns (free once P(j) was formed), so the next tile's exponentials overlap dQ(j).
#pragma once

#include "fa_bwd.cuh"
#include "fa_fwd.cuh"

namespace fa {

template <int D>
struct BwdDqCfg {
  static constexpr int kThreads = 256;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kSlots = (D == 128) ? 4 : 8;
  static constexpr int kOffQ = 0;  // Q_i (also dQ staging)
  static constexpr int kOffDO = kTileBytes;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kSlots * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256;
  static constexpr uint32_t kTmemCols = 512;
};

constexpr int kBwdDqMaxSlots = 8;

struct BwdDqBars {
  uint64_t q_full, q_empty;  // Q_i and dO_i; released by the epilogue once the dQ staging is read
  uint64_t kv_full[kBwdDqMaxSlots], kv_empty[kBwdDqMaxSlots];
  uint64_t s_full, dp_full, ds_full, dq_full, dq_empty;
  uint64_t mma_done;
  uint64_t item_full[2], item_empty[2];
  int item_w[2];
  uint32_t tmem_base;
  int abort_flag;
};

// Consumers of a fetched item: the MMA thread and the 4 compute warps.
constexpr uint32_t kBwdDqItemConsumers = 5;

// Heads per scheduling group of the dQ kernel: the K/V rows of the few heads in flight stay in L2.
constexpr int kBwdHeadGroup = 4;

// Item w -> (b, h, i): groups of kBwdHeadGroup heads; inside a group, Q tiles longest first
// under causal masking (descending i), across the group's heads.
__device__ __forceinline__ void bwd_dq_decode(const BwdParams& p, int w, int& b, int& h, int& i) {
  const int per_group = kBwdHeadGroup * p.num_kv_tiles;
  const int g = w / per_group;
  const int pos = w - g * per_group;
  const int gs = min(kBwdHeadGroup, p.B * p.H - g * kBwdHeadGroup);
  const int r = pos / gs;
  i = p.causal ? (p.num_kv_tiles - 1 - r) : r;
  const int bh = g * kBwdHeadGroup + (pos - r * gs);
  b = bh / p.H;
  h = bh - b * p.H;
}

__device__ __forceinline__ int bwd_dq_take_item(BwdDqBars* bars, uint32_t n, bool arrive, Abort ab) {
  const uint32_t slot = n & 1;
  const bool ok = mbar_wait_ring(smem_u32(&bars->item_full[slot]), (n >> 1) & 1, ab);
  const int w = *reinterpret_cast<volatile int*>(&bars->item_w[slot]);
  __syncwarp(__activemask());
  if (arrive) mbar_arrive(smem_u32(&bars->item_empty[slot]));
  return ok ? w : 0x7fffffff;
}

// The ranges and masks of the forward apply: Q tile rows [i*128, i*128+127] see the KV tiles of
// fwd_kv_range, and fwd_tile_unmasked says when a KV tile needs no per-element mask.
__device__ __forceinline__ FwdParams bwd_dq_as_fwd(const BwdParams& p) {
  FwdParams f{};
  f.B = p.B;
  f.N = p.N;
  f.H = p.H;
  f.win_l = p.win_l;
  f.win_r = p.win_r;
  f.causal = p.causal;
  f.cu_seqlens = p.cu_seqlens;
  f.nseg = p.nseg;
  return f;
}

template <int D, bool kAlibi = false, bool kVarlen = false>
__global__ void __launch_bounds__(256, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const __grid_constant__ CUtensorMap tmdQ, const BwdParams p) {
  using Cfg = BwdDqCfg<D>;
  using Bars = BwdDqBars;
  static_assert(Cfg::kSlots <= kBwdDqMaxSlots, "barrier block too small");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_u32(smem_raw));
  Bars* bars = reinterpret_cast<Bars*>(smem_gen + Cfg::kOffBar);
  auto bar = [&](uint64_t& x) { return smem_u32(&x); };
  const int warp = threadIdx.x >> 5;
  const Abort ab{&bars->abort_flag};
  const FwdParams fp = bwd_dq_as_fwd(p);

  if (threadIdx.x == 0) {
    bars->abort_flag = 0;
    mbar_init(bar(bars->q_full), 1);
    mbar_init(bar(bars->q_empty), 1);
    for (int s = 0; s < Cfg::kSlots; ++s) {
      mbar_init(bar(bars->kv_full[s]), 1);
      mbar_init(bar(bars->kv_empty[s]), 1);
    }
    mbar_init(bar(bars->s_full), 1);
    mbar_init(bar(bars->dp_full), 1);
    mbar_init(bar(bars->ds_full), 128);
    mbar_init(bar(bars->dq_full), 1);
    mbar_init(bar(bars->dq_empty), 128);
    mbar_init(bar(bars->mma_done), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(bars->item_full[s]), 1);
      mbar_init(bar(bars->item_empty[s]), kBwdDqItemConsumers);
    }
    fence_barrier_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
    prefetch_tmap(&tmdQ);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), Cfg::kTmemCols);
    tmem_relinquish();
    tc_fence_before_sync();
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sQ = smem_base + Cfg::kOffQ, sDO = smem_base + Cfg::kOffDO, sKV = smem_base + Cfg::kOffKV;
  const uint32_t smem_end = smem_u32(smem_raw) + Cfg::kSmemBytes;  // for the FA_DEBUG bounds checks
  auto tile_ok = [&](uint32_t dst, int row, int b, int h) {  // FA_DEBUG: the tile's d/64 boxes
    bool ok = true;
#pragma unroll
    for (int bx = 0; bx < Cfg::kBoxes; ++bx)
      ok = ok && dbg_tma(ab, bx * 64, row, h, b, D, p.N, p.H, p.B, 2, dst + bx * 16384, 16384, smem_base, smem_end);
    return ok;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- work fetch + TMA producer
    if (lane_id() == 0) {
      uint32_t slot = 0, phase = 0, qn = 0;
      int last_slot_parity[Cfg::kSlots];
      for (int s = 0; s < Cfg::kSlots; ++s) last_slot_parity[s] = -1;
      for (uint32_t n = 0;; ++n) {
        const uint32_t islot = n & 1;
        mbar_wait_ring(bar(bars->item_empty[islot]), ((n >> 1) & 1) ^ 1, ab);  // slot read by every consumer
        const int w = ab.raised() ? p.num_items : atomicAdd(p.next_item + 1, 1);
        bars->item_w[islot] = w;
        mbar_arrive(bar(bars->item_full[islot]));
        if (w >= p.num_items) break;
        int b, h, i;
        bwd_dq_decode(p, w, b, h, i);
        int lo, hi;
        fwd_kv_range<kVarlen>(fp, i * 128, lo, hi);
        mbar_wait(bar(bars->q_empty), (qn & 1) ^ 1, ab);
        if (!tile_ok(sQ, i * 128, b, h) || !tile_ok(sDO, i * 128, b, h)) break;
        mbar_arrive_expect_tx(bar(bars->q_full), 2 * Cfg::kTileBytes);
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
          tma_load_4d(sQ + bx * 16384, &tmQ, bar(bars->q_full), bx * 64, i * 128, h, b);
          tma_load_4d(sDO + bx * 16384, &tmdO, bar(bars->q_full), bx * 64, i * 128, h, b);
        }
        ++qn;
        for (int j = lo; j <= hi && !(FA_DEBUG && ab.raised()); ++j) {
          for (int kv = 0; kv < 2; ++kv) {
            mbar_wait(bar(bars->kv_empty[slot]), phase ^ 1, ab);
            const uint32_t dst = sKV + slot * Cfg::kTileBytes;
            if (!tile_ok(dst, j * 128, b, h)) break;
            mbar_arrive_expect_tx(bar(bars->kv_full[slot]), Cfg::kTileBytes);
#pragma unroll
            for (int bx = 0; bx < Cfg::kBoxes; ++bx)
              tma_load_4d(dst + bx * 16384, kv ? &tmV : &tmK, bar(bars->kv_full[slot]), bx * 64, j * 128, h, b);
            last_slot_parity[slot] = phase;
            if (++slot == Cfg::kSlots) { slot = 0; phase ^= 1; }
          }
        }
      }
      for (int s = 0; s < Cfg::kSlots; ++s)
        if (last_slot_parity[s] >= 0) mbar_drain(bar(bars->kv_full[s]), last_slot_parity[s]);
      if (qn > 0) mbar_drain(bar(bars->q_full), (qn - 1) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);  // S, dP: both operands K-major
      constexpr uint32_t idQ = idesc_bf16_f32(128, D, false, true);     // dQ: dS from TMEM, K MN-major
      const uint32_t tS = tmem + Cfg::kColS, tDP = tmem + Cfg::kColDP, tDQ = tmem + Cfg::kColDQ;
      uint32_t slot = 0, phase = 0, qn = 0, n = 0;
      auto take_kv = [&](uint32_t& s_out) {
        s_out = slot;
        mbar_wait(bar(bars->kv_full[slot]), phase, ab);
        if (++slot == Cfg::kSlots) { slot = 0; phase ^= 1; }
        tc_fence_after_sync();
      };
      auto issue_qk = [&](uint32_t dtm, uint32_t a_smem, uint32_t b_smem) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(dtm, sdesc_kmajor(a_smem + off), sdesc_kmajor(b_smem + off), idS, kk > 0);
        }
      };
      for (uint32_t it = 0;; ++it) {
        const int w = bwd_dq_take_item(bars, it, true, ab);
        if (w >= p.num_items) break;
        int b, h, i;
        bwd_dq_decode(p, w, b, h, i);
        int lo, hi;
        fwd_kv_range<kVarlen>(fp, i * 128, lo, hi);
        mbar_wait(bar(bars->q_full), qn & 1, ab);
        tc_fence_after_sync();
        uint32_t k_slot, v_slot;
        take_kv(k_slot);
        issue_qk(tS, sQ, sKV + k_slot * Cfg::kTileBytes);  // S(lo)
        mma_commit(bar(bars->s_full));
        take_kv(v_slot);
        issue_qk(tDP, sDO, sKV + v_slot * Cfg::kTileBytes);  // dP(lo)
        mma_commit(bar(bars->dp_full));
        mma_commit(bar(bars->kv_empty[v_slot]));
        for (int j = lo; j <= hi; ++j, ++n) {
          mbar_wait(bar(bars->ds_full), n & 1, ab);
          if (j == lo) mbar_wait(bar(bars->dq_empty), (qn & 1) ^ 1, ab);
          tc_fence_after_sync();
          uint32_t nk_slot = 0, nv_slot = 0;
          if (j < hi) {  // S(j+1) into the S columns, which P(j) no longer needs
            take_kv(nk_slot);
            issue_qk(tS, sQ, sKV + nk_slot * Cfg::kTileBytes);
            mma_commit(bar(bars->s_full));
          }
          // dQ += dS K_j, dS packed in TMEM over dP columns [0, 64)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tDQ, tDP + kk * 8, sdesc_mnmajor(sKV + k_slot * Cfg::kTileBytes + kk * 2048, 16384), idQ,
                   j > lo || kk > 0);
          mma_commit(bar(bars->kv_empty[k_slot]));
          if (j < hi) {  // dP(j+1) after dQ(j) has read dS(j)
            take_kv(nv_slot);
            issue_qk(tDP, sDO, sKV + nv_slot * Cfg::kTileBytes);
            mma_commit(bar(bars->dp_full));
            mma_commit(bar(bars->kv_empty[nv_slot]));
          }
          k_slot = nk_slot;
        }
        mma_commit(bar(bars->dq_full));
        ++qn;
      }
      mma_commit(bar(bars->mma_done));
      mbar_drain(bar(bars->mma_done), 0);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- P, dS, epilogue
    const int row = threadIdx.x - 128;  // query row within the tile == TMEM lane
    const uint32_t lane_field = (uint32_t)((row & ~31) << 16);
    const uint32_t tS = tmem + lane_field + Cfg::kColS, tDP = tmem + lane_field + Cfg::kColDP;
    const uint32_t tDQ = tmem + lane_field + Cfg::kColDQ;
    const float c = p.scale_log2;
    uint32_t n = 0, qn = 0;
    for (uint32_t it = 0;; ++it) {
      const int w = bwd_dq_take_item(bars, it, lane_id() == 0, ab);
      if (w >= p.num_items) break;
      int b, h, i;
      bwd_dq_decode(p, w, b, h, i);
      int lo, hi;
      fwd_kv_range<kVarlen>(fp, i * 128, lo, hi);
      const int q = i * 128 + row;
      const size_t stat = ((size_t)b * p.H + h) * (size_t)p.N_pad + q;  // padded rows hold 0
      const float nlse2 = p.lse2[stat];                                 // -LSE * log2(e)
      const float nd = p.dvec[stat];                                     // -D
      const float nslope2 = kAlibi ? -p.alibi_slopes[b * p.H + h] * kLog2e : 0.0f;  // ALiBi: -m log2(e)
      int kmin, kmax;
      if constexpr (kVarlen) {
        fwd_row_keys<true>(fp, q, kmin, kmax);
      } else {
        kmin = p.win_l >= 0 ? q - p.win_l : 0;
        kmax = (q >= p.N) ? -1 : (p.win_r >= 0 ? min(p.N - 1, q + p.win_r) : p.N - 1);
      }
      int seg_first = 0, seg_last = 0;  // sequence of the tile's first row (packed batches)
      if (kVarlen) seg_bounds(p.cu_seqlens, p.nseg, p.N, i * 128, seg_first, seg_last);
      for (int j = lo; j <= hi; ++j, ++n) {
        const bool masked = !fwd_tile_unmasked<kVarlen>(fp, i * 128, j, seg_first, seg_last) || (i * 128 + 127 >= p.N);
        // key j * 128 + c is visible iff 0 <= j * 128 + c - kmin <= kmax - kmin (one unsigned
        // compare per score; an empty range masks every key)
        const unsigned span = kmax >= kmin ? (unsigned)(kmax - kmin) : 0u;
        const int off = kmax >= kmin ? j * 128 - kmin : -(1 << 30);
        mbar_wait(bar(bars->s_full), n & 1, ab);
        tc_fence_after_sync();
        uint32_t pk[64];  // P(q, keys) as bf16 pairs
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t sv[32];
          tmem_ld32(tS + q4 * 32, sv);
          tmem_wait_ld(sv);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float2 xv = fma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])),
                             make_float2(c, c), make_float2(nlse2, nlse2));
            if (kAlibi) {  // bias -m |q - key| with key = j * 128 + q4 * 32 + e
              const float d0 = (float)(q - j * 128 - q4 * 32);
              xv.x = fmaf(fabsf(d0 - (float)e), nslope2, xv.x);
              xv.y = fmaf(fabsf(d0 - (float)(e + 1)), nslope2, xv.y);
            }
            float2 pv = make_float2(ex2_approx(xv.x), ex2_approx(xv.y));
            if (masked) {
              pv.x = ((unsigned)(off + q4 * 32 + e) <= span) ? pv.x : 0.0f;
              pv.y = ((unsigned)(off + q4 * 32 + e + 1) <= span) ? pv.y : 0.0f;
            }
            pk[q4 * 16 + (e >> 1)] = pack_bf16x2(pv.x, pv.y);
          }
        }
        mbar_wait(bar(bars->dp_full), n & 1, ab);
        tc_fence_after_sync();
        // dS = P * (dP - D), chunk by chunk; chunk k is written to dP columns [16k, 16k+16),
        // which this thread has already read.
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t dv[32];
          tmem_ld32(tDP + q4 * 32, dv);
          tmem_wait_ld(dv);
          uint32_t ds[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint32_t pp = pk[q4 * 16 + (e >> 1)];
            const float2 diff = add2(make_float2(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])),
                                     make_float2(nd, nd));
            const float2 v = mul2(make_float2(bf16lo_to_f32(pp), bf16hi_to_f32(pp)), diff);
            ds[e >> 1] = pack_bf16x2(v.x, v.y);
          }
          tmem_st16(tDP + q4 * 16, ds);
        }
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(bar(bars->ds_full));
      }
      // Epilogue: dQ * scale -> bf16 -> staging (the Q buffer: every S of the item is done) -> TMA store.
      mbar_wait(bar(bars->dq_full), qn & 1, ab);
      tc_fence_after_sync();
#pragma unroll 1
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t o[32];
        tmem_ld32(tDQ + cc, o);
        tmem_wait_ld(o);
        const uint32_t box = sQ + (cc >> 6) * 16384;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w4[e] = pack_bf16x2(__uint_as_float(o[ch * 8 + 2 * e]) * p.scale,
                                __uint_as_float(o[ch * 8 + 2 * e + 1]) * p.scale);
          st_shared_v4(box + sw128_offset(row, ((cc & 63) >> 3) + ch), w4[0], w4[1], w4[2], w4[3]);
        }
      }
      tc_fence_before_sync();
      mbar_arrive(bar(bars->dq_empty));
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (row == 0) {
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx)
          if (dbg_tma(ab, bx * 64, i * 128, h, b, D, p.N, p.H, p.B, 2, sQ + bx * 16384, 16384, smem_base, smem_end))
            tma_store_4d(&tmdQ, sQ + bx * 16384, bx * 64, i * 128, h, b);
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(bar(bars->q_empty));
      }
      ++qn;
    }
    if (row == 0) bulk_wait_group0();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace fa
