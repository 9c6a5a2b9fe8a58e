// Backward kernels of exact attention for sm_100a (recompute-based).
//
// The forward saves only O and LSE ("Flash Attention V2核心网络算子解析" §二.1 step 3: the
// backward reuses what the forward kept); scores and probabilities are recomputed tile by
// tile. With P = exp(scale * Q K^T - LSE) (masked entries 0):
//   dV = P^T dO,  dP = dO V^T,  D_i = rowsum(dO * O)_i,  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three launches on the caller's stream:
//   fa_bwd_pre_kernel   D (fp32), LSE * log2(e) (fp32), zero the fp32 dQ accumulator
//   fa_bwd_kernel       one work item per (b, h, 128-key tile j): K_j, V_j stay in shared
//                       memory, dK_j and dV_j accumulate in TMEM over the visible Q tiles i;
//                       dQ_i partial products are added into the fp32 accumulator in global memory
//   fa_dq_convert_kernel  dQ = bf16(accumulator)
//
// fa_bwd_kernel roles (512 threads):
//   warp 0       TMA producer: K_j, V_j per item; Q_i, dO_i, LSE2_i, D_i in a 2-stage ring
//   warp 1       MMA issuer, TMEM owner
//   warps 4-7    dQ: TMEM -> registers -> red.global.add.v4.f32 into the accumulator
//   warps 8-11   P/dS for query columns [0, 64) of each tile; dK epilogue
//   warps 12-15  P/dS for query columns [64, 128); dV epilogue
// TMEM: dK [0,D), dV [D,2D), dP^T / dQ [2D, 2D+128), S^T / P^T [2D+128, 2D+256).
// Per Q tile i the MMA warp issues S^T = K Q_i^T, dP^T = V dO_i^T, dV += P^T dO_i (P^T from
// TMEM), dK += dS^T Q_i and dQ_i = dS K_j (dS^T in shared memory, read K-major for dK and
// MN-major for dQ).
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

constexpr float kLog2e = 1.4426950408889634074f;

struct BwdParams {
  int B, N, H, N_pad;  // N_pad = N rounded up to 128 (row stride of LSE2 and D)
  float scale;
  float scale_log2;    // scale * log2(e)
  int win_l;           // -1 = unbounded
  int win_r;           // effective right bound (0 under causal), -1 = unbounded
  int causal;
  int num_kv_tiles;    // ceil(N / 128)
  int num_items;       // B * H * num_kv_tiles
  float* dq_acc;       // (B, N, H, d) fp32
  const float* lse2;   // (B, H, N_pad) fp32: LSE * log2(e)
  const float* dvec;   // (B, H, N_pad) fp32: rowsum(dO * O)
};

// ------------------------------------------------------------------ preprocess

// One warp per (b, n, h) row with n < N_pad: D = sum_c dO*O in fp32 and LSE2 = LSE*log2(e)
// (0 for padding rows), and the row of the dQ accumulator set to zero.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dout,
                                                         const float* __restrict__ lse, float* __restrict__ lse2,
                                                         float* __restrict__ dvec, float* __restrict__ dq_acc,
                                                         int B, int N, int H, int N_pad) {
  const long long warp_g = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long total = (long long)B * N_pad * H;
  if (warp_g >= total) return;
  const int h = (int)(warp_g % H);
  const long long bn = warp_g / H;
  const int n = (int)(bn % N_pad);
  const int b = (int)(bn / N_pad);
  const size_t stat = ((size_t)b * H + h) * (size_t)N_pad + n;
  if (n >= N) {
    if (lane == 0) { lse2[stat] = 0.0f; dvec[stat] = 0.0f; }
    return;
  }
  const size_t row = (((size_t)b * N + n) * H + h) * (size_t)D;
  constexpr int kPer = D / 32;  // bf16 elements per lane: 2 (D=64) or 4 (D=128)
  float acc = 0.0f;
  if (kPer == 4) {
    const uint2 ov = *reinterpret_cast<const uint2*>(o + row + lane * 4);
    const uint2 gv = *reinterpret_cast<const uint2*>(dout + row + lane * 4);
    acc = bf16lo_to_f32(ov.x) * bf16lo_to_f32(gv.x) + bf16hi_to_f32(ov.x) * bf16hi_to_f32(gv.x) +
          bf16lo_to_f32(ov.y) * bf16lo_to_f32(gv.y) + bf16hi_to_f32(ov.y) * bf16hi_to_f32(gv.y);
    *reinterpret_cast<float4*>(dq_acc + row + lane * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
    const uint32_t ov = *reinterpret_cast<const uint32_t*>(o + row + lane * 2);
    const uint32_t gv = *reinterpret_cast<const uint32_t*>(dout + row + lane * 2);
    acc = bf16lo_to_f32(ov) * bf16lo_to_f32(gv) + bf16hi_to_f32(ov) * bf16hi_to_f32(gv);
    *reinterpret_cast<float2*>(dq_acc + row + lane * 2) = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    dvec[stat] = acc;
    lse2[stat] = lse[((size_t)b * H + h) * (size_t)N + n] * kLog2e;
  }
}

// ------------------------------------------------------------------ dQ conversion

__global__ void __launch_bounds__(256) fa_dq_convert_kernel(const float* __restrict__ acc,
                                                            __nv_bfloat16* __restrict__ dq, long long n8) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * idx];
  const float4 c = reinterpret_cast<const float4*>(acc)[2 * idx + 1];
  uint4 out;
  out.x = pack_bf16x2(a.x, a.y);
  out.y = pack_bf16x2(a.z, a.w);
  out.z = pack_bf16x2(c.x, c.y);
  out.w = pack_bf16x2(c.z, c.w);
  reinterpret_cast<uint4*>(dq)[idx] = out;
}

// ------------------------------------------------------------------ main backward kernel

template <int D>
struct BwdCfg {
  static constexpr int kThreads = 512;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kStages = 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;                      // + stage * 2 tiles
  static constexpr int kOffDS = kOffQ + kStages * 2 * kTileBytes;   // 128 x 128 bf16
  static constexpr int kOffStat = kOffDS + 32768;                   // + stage * 1024: LSE2[128], D[128]
  static constexpr int kOffBar = kOffStat + kStages * 1024;
  static constexpr int kSmemBytes = kOffBar + 256;
  static constexpr uint32_t kColDK = 0, kColDV = D, kColDP = 2 * D, kColS = 2 * D + 128;
  static constexpr uint32_t kTmemCols = 512;
};

struct BwdBars {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full, dp_full, p_full, ds_full, ds_empty, dq_full, dq_empty, dkv_full, dkv_empty;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// Item w -> (b, h, j). Under causal masking low key tiles (more Q tiles to visit) come first.
__device__ __forceinline__ void bwd_decode(const BwdParams& p, int w, int& b, int& h, int& j) {
  const int bh_count = p.B * p.H;
  const int r = w / bh_count, bh = w - r * bh_count;
  j = r;
  b = bh / p.H;
  h = bh - b * p.H;
}

// Q tiles whose rows see any key of KV tile j.
__device__ __forceinline__ void bwd_q_range(const BwdParams& p, int j, int& lo, int& hi) {
  const int k0 = j * 128;
  const int k1 = min(k0 + 127, p.N - 1);
  const int qlo = p.win_r >= 0 ? max(0, k0 - p.win_r) : 0;
  const int qhi = p.win_l >= 0 ? min(p.N - 1, k1 + p.win_l) : p.N - 1;
  lo = qlo >> 7;
  hi = qhi >> 7;
}

__device__ __forceinline__ bool bwd_tile_unmasked(const BwdParams& p, int j, int i) {
  const int k0 = j * 128, k1 = k0 + 127, q0 = i * 128, q1 = q0 + 127;
  if (k1 >= p.N || q1 >= p.N) return false;
  if (p.win_l >= 0 && k0 < q1 - p.win_l) return false;
  if (p.win_r >= 0 && k1 > q0 + p.win_r) return false;
  return true;
}

template <int D>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                  const BwdParams p) {
  using Cfg = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = smem_u32(smem_raw);
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem_raw + Cfg::kOffBar);
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };
  // 128-byte swizzled tiles need 1024-byte alignment; the kernel reports instead of faulting.
  if (smem_base & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_fa_error, 2);
    return;
  }

  const int warp = threadIdx.x >> 5;
  const Abort ab{&bars->abort_flag};

  if (threadIdx.x == 0) {
    bars->abort_flag = 0;
    mbar_init(bar(bars->kv_full), 1);
    mbar_init(bar(bars->kv_empty), 2);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(bars->q_full[s]), 1);
      mbar_init(bar(bars->q_empty[s]), 1);
    }
    mbar_init(bar(bars->s_full), 1);
    mbar_init(bar(bars->dp_full), 1);
    mbar_init(bar(bars->p_full), 256);
    mbar_init(bar(bars->ds_full), 256);
    mbar_init(bar(bars->ds_empty), 1);
    mbar_init(bar(bars->dq_full), 1);
    mbar_init(bar(bars->dq_empty), 128);
    mbar_init(bar(bars->dkv_full), 1);
    mbar_init(bar(bars->dkv_empty), 256);
    mbar_init(bar(bars->mma_done), 1);
    fence_barrier_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
    prefetch_tmap(&tmdK);
    prefetch_tmap(&tmdV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), Cfg::kTmemCols);
    tmem_relinquish();
    tc_fence_before_sync();
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  const uint32_t sK = smem_base + Cfg::kOffK, sV = smem_base + Cfg::kOffV;
  const uint32_t sDS = smem_base + Cfg::kOffDS;
  auto sQ = [&](int s) { return smem_base + Cfg::kOffQ + s * 2 * Cfg::kTileBytes; };
  auto sdO = [&](int s) { return smem_base + Cfg::kOffQ + s * 2 * Cfg::kTileBytes + Cfg::kTileBytes; };
  auto sStat = [&](int s) { return smem_base + Cfg::kOffStat + s * 1024; };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane_id() == 0) {
      uint32_t items = 0, stage = 0, sphase = 0;
      int last_stage_parity[2] = {-1, -1};
      for (int round = 0;; ++round) {
        const int w = sched_item(round, blockIdx.x, gridDim.x);
        if (w >= p.num_items || ab.raised()) break;
        int b, h, j;
        bwd_decode(p, w, b, h, j);
        int lo, hi;
        bwd_q_range(p, j, lo, hi);
        mbar_wait(bar(bars->kv_empty), (items & 1) ^ 1, ab);
        mbar_arrive_expect_tx(bar(bars->kv_full), 2 * Cfg::kTileBytes);
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
          tma_load_4d(sK + bx * 16384, &tmK, bar(bars->kv_full), bx * 64, j * 128, h, b);
          tma_load_4d(sV + bx * 16384, &tmV, bar(bars->kv_full), bx * 64, j * 128, h, b);
        }
        ++items;
        const size_t stat_row = ((size_t)b * p.H + h) * (size_t)p.N_pad;
        for (int i = lo; i <= hi; ++i) {
          mbar_wait(bar(bars->q_empty[stage]), sphase ^ 1, ab);
          const uint32_t fb = bar(bars->q_full[stage]);
          mbar_arrive_expect_tx(fb, 2 * Cfg::kTileBytes + 1024);
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
            tma_load_4d(sQ(stage) + bx * 16384, &tmQ, fb, bx * 64, i * 128, h, b);
            tma_load_4d(sdO(stage) + bx * 16384, &tmdO, fb, bx * 64, i * 128, h, b);
          }
          bulk_load(sStat(stage), p.lse2 + stat_row + i * 128, 512, fb);
          bulk_load(sStat(stage) + 512, p.dvec + stat_row + i * 128, 512, fb);
          last_stage_parity[stage] = sphase;
          if (++stage == 2) { stage = 0; sphase ^= 1; }
        }
      }
      for (int s = 0; s < 2; ++s)
        if (last_stage_parity[s] >= 0) mbar_drain(bar(bars->q_full[s]), last_stage_parity[s]);
      if (items > 0) mbar_drain(bar(bars->kv_full), (items - 1) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      constexpr uint32_t idSP = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T: K-major A and B
      constexpr uint32_t idKV = idesc_bf16_f32(128, D, false, true);     // dV, dK: B (dO, Q) MN-major
      constexpr uint32_t idQ = idesc_bf16_f32(128, D, true, true);       // dQ: A (dS) and B (K) MN-major
      const uint32_t tDK = tmem + Cfg::kColDK, tDV = tmem + Cfg::kColDV;
      const uint32_t tDP = tmem + Cfg::kColDP, tS = tmem + Cfg::kColS;
      uint32_t items = 0, n = 0, stage = 0, sphase = 0;
      for (int round = 0;; ++round) {
        const int w = sched_item(round, blockIdx.x, gridDim.x);
        if (w >= p.num_items || ab.raised()) break;
        int b, h, j;
        bwd_decode(p, w, b, h, j);
        int lo, hi;
        bwd_q_range(p, j, lo, hi);
        mbar_wait(bar(bars->kv_full), items & 1, ab);
        tc_fence_after_sync();
        bool first = true;
        for (int i = lo; i <= hi; ++i, ++n) {
          mbar_wait(bar(bars->q_full[stage]), sphase, ab);
          tc_fence_after_sync();
          const uint32_t q = sQ(stage), g = sdO(stage);
          // S^T = K_j Q_i^T
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_ss(tS, sdesc_kmajor(sK + off), sdesc_kmajor(q + off), idSP, kk > 0);
          }
          mma_commit(bar(bars->s_full));
          // dP^T = V_j dO_i^T, into the columns dQ_{i-1} occupied
          mbar_wait(bar(bars->dq_empty), (n & 1) ^ 1, ab);
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_ss(tDP, sdesc_kmajor(sV + off), sdesc_kmajor(g + off), idSP, kk > 0);
          }
          mma_commit(bar(bars->dp_full));
          // dV += P^T dO_i (P^T packed in TMEM: queries [0,64) in S columns [0,32), [64,128) in [64,96))
          mbar_wait(bar(bars->p_full), n & 1, ab);
          if (first) mbar_wait(bar(bars->dkv_empty), (items & 1) ^ 1, ab);
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t acol = (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8;
            mma_ts(tDV, tS + acol, sdesc_mnmajor(g + kk * 2048, 16384), idKV, !first || kk > 0);
          }
          // dK += dS^T Q_i ; dQ_i = dS K_j
          mbar_wait(bar(bars->ds_full), n & 1, ab);
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_ss(tDK, sdesc_kmajor(sDS + off), sdesc_mnmajor(q + kk * 2048, 16384), idKV, !first || kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tDP, sdesc_mnmajor(sDS + kk * 2048, 16384), sdesc_mnmajor(sK + kk * 2048, 16384), idQ, kk > 0);
          mma_commit(bar(bars->dq_full));
          mma_commit(bar(bars->ds_empty));
          mma_commit(bar(bars->q_empty[stage]));
          first = false;
          if (++stage == 2) { stage = 0; sphase ^= 1; }
        }
        mma_commit(bar(bars->dkv_full));
        ++items;
      }
      mma_commit(bar(bars->mma_done));
      mbar_drain(bar(bars->mma_done), 0);
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------------------------------------------- dQ accumulation
    const int row = threadIdx.x - 128;
    const uint32_t tDQ = tmem + ((uint32_t)(row & ~31) << 16) + Cfg::kColDP;
    uint32_t n = 0;
    for (int round = 0;; ++round) {
      const int w = sched_item(round, blockIdx.x, gridDim.x);
      if (w >= p.num_items) break;
      int b, h, j;
      bwd_decode(p, w, b, h, j);
      int lo, hi;
      bwd_q_range(p, j, lo, hi);
      for (int i = lo; i <= hi; ++i, ++n) {
        mbar_wait(bar(bars->dq_full), n & 1, ab);
        tc_fence_after_sync();
        const int qrow = i * 128 + row;
        float* dst = p.dq_acc + (((size_t)b * p.N + qrow) * p.H + h) * (size_t)D;
#pragma unroll 1
        for (int cc = 0; cc < D; cc += 32) {
          uint32_t v[32];
          tmem_ld32(tDQ + cc, v);
          tmem_wait_ld(v);
          if (cc + 32 >= D) {
            tc_fence_before_sync();
            mbar_arrive(bar(bars->dq_empty));
          }
          if (qrow < p.N) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              red_add_v4_f32(dst + cc + e, __uint_as_float(v[e]) * p.scale, __uint_as_float(v[e + 1]) * p.scale,
                             __uint_as_float(v[e + 2]) * p.scale, __uint_as_float(v[e + 3]) * p.scale);
          }
        }
      }
    }
  } else if (warp >= 8) {
    // ---------------------------------------------------------------- P, dS and the dK / dV epilogue
    const int grp = (warp - 8) >> 2;              // 0: query columns [0,64) and dK; 1: [64,128) and dV
    const int row = threadIdx.x - 256 - 128 * grp;  // key row within the tile == TMEM lane
    const uint32_t lane_field = (uint32_t)((row & ~31) << 16);
    const uint32_t tS = tmem + lane_field + Cfg::kColS + 64 * grp;
    const uint32_t tDP = tmem + lane_field + Cfg::kColDP + 64 * grp;
    const float c = p.scale_log2;
    uint32_t items = 0, n = 0, stage = 0, sphase = 0;
    for (int round = 0;; ++round) {
      const int w = sched_item(round, blockIdx.x, gridDim.x);
      if (w >= p.num_items) break;
      int b, h, j;
      bwd_decode(p, w, b, h, j);
      int lo, hi;
      bwd_q_range(p, j, lo, hi);
      const int k = j * 128 + row;
      const int qlo = p.win_r >= 0 ? k - p.win_r : 0;
      const int qhi = (k >= p.N) ? -1 : (p.win_l >= 0 ? min(p.N - 1, k + p.win_l) : p.N - 1);
      for (int i = lo; i <= hi; ++i, ++n) {
        // wait for the stage's Q_i / dO_i / LSE2_i / D_i (the statistics are read here)
        mbar_wait(bar(bars->q_full[stage]), sphase, ab);
        const float* lse2 = reinterpret_cast<const float*>(smem_raw + Cfg::kOffStat + stage * 1024);
        const float* dv = lse2 + 128;
        const bool masked = !bwd_tile_unmasked(p, j, i);
        const int qbase = i * 128 + 64 * grp;

        mbar_wait(bar(bars->s_full), n & 1, ab);
        tc_fence_after_sync();
        uint32_t s0[32], s1[32];
        tmem_ld32(tS, s0);
        tmem_ld32(tS + 32, s1);
        tmem_wait_ld(s0);
        tmem_wait_ld(s1);
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float a0 = __uint_as_float(e < 32 ? s0[e] : s1[e - 32]);
          const float a1 = __uint_as_float(e < 32 ? s0[e + 1] : s1[e - 31]);
          const int qc = 64 * grp + e;
          float p0 = ex2_approx(fmaf(a0, c, -lse2[qc]));
          float p1 = ex2_approx(fmaf(a1, c, -lse2[qc + 1]));
          if (masked) {
            const int q0 = qbase + e;
            p0 = (q0 >= qlo && q0 <= qhi) ? p0 : 0.0f;
            p1 = (q0 + 1 >= qlo && q0 + 1 <= qhi) ? p1 : 0.0f;
          }
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
        {
          uint32_t lo16[16], hi16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) { lo16[e] = pk[e]; hi16[e] = pk[16 + e]; }
          tmem_st16(tS, lo16);
          tmem_st16(tS + 16, hi16);
        }
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(bar(bars->p_full));

        mbar_wait(bar(bars->dp_full), n & 1, ab);
        tc_fence_after_sync();
        uint32_t d0[32], d1[32];
        tmem_ld32(tDP, d0);
        tmem_ld32(tDP + 32, d1);
        tmem_wait_ld(d0);
        tmem_wait_ld(d1);
        // dS^T(row, q) = P^T(row, q) * (dP^T(row, q) - D_q) -> bf16 -> shared, 128B-swizzled rows of keys
        mbar_wait(bar(bars->ds_empty), (n & 1) ^ 1, ab);
        const uint32_t box = sDS + grp * 16384;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = ch * 8 + 2 * e;  // 0..63 within the group
            const float g0 = __uint_as_float(col < 32 ? d0[col] : d1[col - 32]);
            const float g1 = __uint_as_float(col < 32 ? d0[col + 1] : d1[col - 31]);
            const uint32_t pp = pk[col >> 1];
            const float ds0 = bf16lo_to_f32(pp) * (g0 - dv[64 * grp + col]);
            const float ds1 = bf16hi_to_f32(pp) * (g1 - dv[64 * grp + col + 1]);
            w4[e] = pack_bf16x2(ds0, ds1);
          }
          st_shared_v4(box + sw128_offset(row, ch), w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        mbar_arrive(bar(bars->ds_full));
        if (++stage == 2) { stage = 0; sphase ^= 1; }
      }

      // Epilogue: dK (group 0, times scale) or dV (group 1) -> bf16 -> the K_j / V_j buffer -> TMA store.
      mbar_wait(bar(bars->dkv_full), items & 1, ab);
      tc_fence_after_sync();
      const uint32_t src = tmem + lane_field + (grp ? Cfg::kColDV : Cfg::kColDK);
      const uint32_t stage_buf = grp ? sV : sK;
      const float mult = grp ? 1.0f : p.scale;
#pragma unroll 1
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t v[32];
        tmem_ld32(src + cc, v);
        tmem_wait_ld(v);
        const uint32_t bx = stage_buf + (cc >> 6) * 16384;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w4[e] = pack_bf16x2(__uint_as_float(v[ch * 8 + 2 * e]) * mult, __uint_as_float(v[ch * 8 + 2 * e + 1]) * mult);
          st_shared_v4(bx + sw128_offset(row, ((cc & 63) >> 3) + ch), w4[0], w4[1], w4[2], w4[3]);
        }
      }
      tc_fence_before_sync();
      mbar_arrive(bar(bars->dkv_empty));
      fence_proxy_async_smem();
      named_bar_sync(1 + grp, 128);
      if (row == 0) {
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx)
          tma_store_4d(grp ? &tmdV : &tmdK, stage_buf + bx * 16384, bx * 64, j * 128, h, b);
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(bar(bars->kv_empty));
      }
      ++items;
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
