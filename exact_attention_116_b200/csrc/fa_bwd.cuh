// Backward kernels of exact attention for sm_100a (recompute-based).
//
// The forward saves only O and LSE ("Flash Attention V2核心网络算子解析" §二.1 step 3: the
// backward reuses what the forward kept); scores and probabilities are recomputed tile by
// tile. With P = exp(scale * Q K^T - LSE) (masked entries 0):
//   dV = P^T dO,  dP = dO V^T,  D_i = rowsum(dO * O)_i,  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three launches on the caller's stream:
//   fa_bwd_pre_kernel   -D (fp32), -LSE * log2(e) (fp32), zero the fp32 dQ accumulator
//   fa_bwd_kernel       one work item per (b, h, 128-key tile j): K_j, V_j stay in shared
//                       memory, dK_j and dV_j accumulate in TMEM over the visible Q tiles i;
//                       dQ_i partial products are added into the fp32 accumulator in global memory
//   fa_dq_convert_kernel  dQ = bf16(accumulator)
//
// fa_bwd_kernel roles (512 or 768 threads):
//   warp 0       work fetch (atomic counter, head-grouped order: bwd_decode) and TMA producer: K_j, V_j
//                per item; Q_i with LSE2_i, D_i in two slots; dO_i in one slot
//   warp 1       MMA issuer, TMEM owner
//   warps 4-7    dQ: TMEM -> registers -> shared staging -> TMA reduce-add into the accumulator;
//                at d = 64 also the dK and dV epilogue of each item (dK / dV have two TMEM buffers
//                there, so the P/dS warps go on to the next item meanwhile), staged in the
//                item's K/V buffers; at d = 128 the dV epilogue, staged in the dQ buffer
//   warps 8-      P/dS in groups of four warps, each for W query columns of every tile: four
//                groups (W = 32, 768 threads) at d = 64, two (W = 64, 512 threads) at d = 128; at
//                d = 128 each group also stores dK columns [W g, W g + W), staged in the dS buffer
// At d = 128 the epilogue thus leaves K_j and V_j alone: their single slot is released by the
// MMA warp's commit after the item's last product, and the next item's K/V load overlaps the
// epilogue.
// TMEM: dK [0,D), dV [D,2D), dP^T / dQ [2D, 2D+128), S^T / P^T [2D+128, 2D+256).
// Per Q tile i the MMA warp issues dP^T = V dO_i^T, dV += P^T dO_i (P^T from TMEM), then
// S^T for tile i+1 (= K Q_{i+1}^T), dQ_i = dS K_j and dK += dS^T Q_i (dS^T in shared memory,
// read MN-major for dQ and K-major for dK). At d = 64, S(i+1) goes before dQ(i): the P of tile
// i+1 is computed while dQ and dK of tile i run. At d = 128, dQ(i) goes before S(i+1): its
// columns, which dP(i+1) reuses, free up one matrix product earlier (measured faster at each
// head dim respectively). dQ always precedes dK.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {


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
  const float* lse2;   // (B, H, N_pad) fp32: -LSE * log2(e)
  const float* dvec;   // (B, H, N_pad) fp32: -rowsum(dO * O)
  int* next_item;      // work counters (zeroed by the preprocess kernel): [0] main kernel, [1] dQ kernel
  const float* alibi_slopes;  // ALiBi only: (B, H) slopes m, bias -m |i - j| on the scaled scores
  const int* cu_seqlens;      // packed variable-length batch (B = 1, N = total): nseg + 1 offsets, or null
  int nseg;
  int head_group;             // heads per scheduling group of the main kernel (>= 1)
  int tail_tiles;             // the last (shortest under causal masking) KV tiles, dealt over all heads
};

// Share of the exponentials computed by exp2_poly on the FMA pipes (pair p of a thread's pairs
// uses the polynomial when p % kPolyDen < kPolyNum). None by default: with the P/dS work spread
// over four warps per SM sub-partition (d = 64) the MUFU unit has room, and the polynomial's
// instructions cost more issue slots than they save (window main kernel 0.1987 ms with 1/4,
// 0.1951 with none, 0.208 with 2/4; train 1.3075 / 1.3005 / 1.2995 ms).
#ifndef FA_BWD_POLY_NUM
#define FA_BWD_POLY_NUM 0
#endif
#ifndef FA_BWD_POLY_DEN
#define FA_BWD_POLY_DEN 4
#endif
constexpr int kBwdPolyNum = FA_BWD_POLY_NUM, kBwdPolyDen = FA_BWD_POLY_DEN;


// ------------------------------------------------------------------ preprocess

// Per (b, h) row n < N_pad: -D = -sum_c dO*O in fp32 and -LSE*log2(e) (0 for padding rows;
// stored negated so that the main kernel adds them), and the row of the dQ accumulator set to
// zero. A CTA takes kPreRows consecutive rows of one (b, h), D/8 threads per row with 16-byte
// loads of O and dO, so the row vectors are read and written contiguously. Also resets the
// main kernel's work counters.
template <int D>
struct PreCfg {
  static constexpr int kThreadsPerRow = D / 8;                // 8 bf16 (16 bytes) per thread
  static constexpr int kRows = 256 / kThreadsPerRow;           // rows per CTA: 16 (D=128), 32 (D=64)
};

template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dout,
                                                         const float* __restrict__ lse, float* __restrict__ lse2,
                                                         float* __restrict__ dvec, float* __restrict__ dq_acc,
                                                         int* __restrict__ next_item, int B, int N, int H,
                                                         int N_pad) {
  using Cfg = PreCfg<D>;
  if (blockIdx.x == 0 && threadIdx.x < 2) next_item[threadIdx.x] = 0;
  const int blocks_per_head = N_pad / Cfg::kRows;
  const long long bh = blockIdx.x / blocks_per_head;  // b * H + h
  const int n = (int)(blockIdx.x % blocks_per_head) * Cfg::kRows + (int)threadIdx.x / Cfg::kThreadsPerRow;
  const int part = (int)threadIdx.x % Cfg::kThreadsPerRow;
  if (bh >= (long long)B * H) return;
  const int b = (int)(bh / H), h = (int)(bh % H);
  const size_t stat = (size_t)bh * (size_t)N_pad + n;
  const Abort none{nullptr};
  // (FA_DEBUG: a failed check skips the accesses; every thread still takes part in the shuffle)
  const bool stat_ok = dbg_range(none, (long long)stat, 1, (long long)B * H * N_pad);
  float acc = 0.0f;
  const size_t row = (((size_t)b * N + n) * H + h) * (size_t)D + part * 8;
  if (n < N && dbg_range(none, (long long)row, 8, (long long)B * N * H * D)) {
    const uint4 ov = *reinterpret_cast<const uint4*>(o + row);
    const uint4 gv = *reinterpret_cast<const uint4*>(dout + row);
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      acc += bf16lo_to_f32(ow[e]) * bf16lo_to_f32(gw[e]) + bf16hi_to_f32(ow[e]) * bf16hi_to_f32(gw[e]);
    float4* z = reinterpret_cast<float4*>(dq_acc + row);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = Cfg::kThreadsPerRow / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (part == 0 && stat_ok) {
    dvec[stat] = n < N ? -acc : 0.0f;
    lse2[stat] = n < N ? -lse[(size_t)bh * (size_t)N + n] * kLog2e : 0.0f;
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
  // P/dS groups of four warps, kGroupCols query columns each: four at d = 64, where their
  // exponentials and dS bound the kernel, two at d = 128, where the dQ reduction does and the
  // smaller register budget of a 768-thread CTA measured slower
  static constexpr int kGroups = (D == 64) ? 4 : 2;
  static constexpr int kGroupCols = 128 / kGroups;
  static constexpr int kThreads = 256 + 128 * kGroups;
  static constexpr uint32_t kItemConsumers = 1 + 4 + 4 * kGroups;  // MMA thread, dQ and P/dS warps
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxes = D / 64;
  // d = 64: two K/V slots and two dK/dV TMEM buffers, alternating per work item, so that the
  // next item's K/V load and first MMAs overlap this item's tail and dK/dV epilogue.
  static constexpr int kKVSlots = (D == 64) ? 2 : 1;
  static constexpr int kOffK = 0;                     // slot s: K at 2 s tiles, V right after
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kKVSlots * kTileBytes;        // two Q slots
  static constexpr int kDOSlots = kKVSlots;                      // dO slots (two at d = 64)
  static constexpr int kOffDO = kOffQ + 2 * kTileBytes;
  static constexpr int kOffDS = kOffDO + kDOSlots * kTileBytes;  // dS^T, 128 x 128 bf16
  static constexpr int kOffDQ = kOffDS + 32768;       // dQ staging: 128 rows x 64 fp32 (two 32-column boxes)
  static constexpr int kOffStat = kOffDQ + 32768;     // per Q slot: LSE2[128], D[128]
  static constexpr int kOffBar = kOffStat + 2 * 1024;
  static constexpr int kSmemBytes = kOffBar + 256;
  static constexpr int kDqRounds = D / 64;            // staging rounds per dQ tile
  static constexpr uint32_t kColDK = 0, kColDV = D, kColDP = 2 * D, kColS = 2 * D + 128;
  static constexpr uint32_t kColDK1 = 2 * D + 256, kColDV1 = 3 * D + 256;  // second dK/dV buffer (d = 64)
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kKVSlots == 1 || kColDV1 + D <= kTmemCols, "TMEM budget");
};

struct BwdBars {
  uint64_t kv_full[2], kv_empty[2];      // per K/V slot
  uint64_t q_full[2], q_empty[2];  // Q_i and its LSE2 / D rows
  uint64_t do_full[2], do_empty[2];     // per dO slot
  uint64_t s_full, dp_full, p_full, ds_full, ds_empty, dq_full, dq_empty;
  uint64_t dkv_full[2], dkv_empty[2];    // per dK/dV buffer
  uint64_t mma_done;
  uint64_t item_full[2], item_empty[2];  // ring of fetched work items, producer -> other roles
  int item_w[2];
  uint32_t tmem_base;
  int abort_flag;
};

// Item w -> (b, h, j), in two phases:
//   1. KV tiles [0, num_kv_tiles - tail_tiles): groups of head_group heads in order, inside a
//      group the KV tile ascending (under causal masking the low tiles visit the most Q tiles)
//      and the heads fastest, so that the Q, dO and dQ-accumulator rows of the heads in flight
//      stay in L2;
//   2. the last tail_tiles KV tiles of every head, tile-major: the items dealt last are the
//      shortest, whatever group ran last, so the CTAs finish together.
__device__ __forceinline__ void bwd_decode(const BwdParams& p, int w, int& b, int& h, int& j) {
  const int bh_count = p.B * p.H;
  const int tiles1 = p.num_kv_tiles - p.tail_tiles;
  const int n1 = bh_count * tiles1;
  int bh;
  if (w < n1) {
    const int per_group = p.head_group * tiles1;
    const int g = w / per_group;
    const int pos = w - g * per_group;
    const int gs = min(p.head_group, bh_count - g * p.head_group);
    j = pos / gs;
    bh = g * p.head_group + (pos - j * gs);
  } else {
    const int w2 = w - n1;
    const int j2 = w2 / bh_count;
    j = tiles1 + j2;
    bh = w2 - j2 * bh_count;
  }
  b = bh / p.H;
  h = bh - b * p.H;
}

// Next work item of a consumer role (n counts the items this role has taken). Returns the
// item index; values >= num_items mean "no more work".
__device__ __forceinline__ int bwd_take_item(BwdBars* bars, uint32_t n, bool arrive, Abort ab) {
  const uint32_t slot = n & 1;
  const bool ok = mbar_wait_ring(smem_u32(&bars->item_full[slot]), (n >> 1) & 1, ab);
  const int w = *reinterpret_cast<volatile int*>(&bars->item_w[slot]);
  __syncwarp(__activemask());
  if (arrive) mbar_arrive(smem_u32(&bars->item_empty[slot]));
  return ok ? w : 0x7fffffff;
}

// Q tiles whose rows see any key of KV tile j.
template <bool kVarlen>
__device__ __forceinline__ void bwd_q_range(const BwdParams& p, int j, int& lo, int& hi) {
  const int k0 = j * 128;
  const int k1 = min(k0 + 127, p.N - 1);
  int first = 0, last = p.N - 1, dummy;
  if (kVarlen) {  // packed sequences: the first key's sequence start to the last key's end
    seg_bounds(p.cu_seqlens, p.nseg, p.N, k0, first, dummy);
    seg_bounds(p.cu_seqlens, p.nseg, p.N, k1, dummy, last);
  }
  const int qlo = p.win_r >= 0 ? max(first, k0 - p.win_r) : first;
  const int qhi = p.win_l >= 0 ? min(last, k1 + p.win_l) : last;
  lo = qlo >> 7;
  hi = qhi >> 7;
}

// Packed sequences (kVarlen): [seg_first, seg_last] are the rows of the sequence of key j * 128.
template <bool kVarlen>
__device__ __forceinline__ bool bwd_tile_unmasked(const BwdParams& p, int j, int i, int seg_first = 0,
                                                  int seg_last = 0) {
  const int k0 = j * 128, k1 = k0 + 127, q0 = i * 128, q1 = q0 + 127;
  if (k1 >= p.N || q1 >= p.N) return false;
  if (p.win_l >= 0 && k0 < q1 - p.win_l) return false;
  if (p.win_r >= 0 && k1 > q0 + p.win_r) return false;
  if (kVarlen && (k1 > seg_last || q0 < seg_first || q1 > seg_last)) return false;  // one sequence only
  return true;
}

// P^T for W query columns of this thread's key row: exp2(S^T * c - LSE_q * log2(e)), zero
// where masked (kMasked), packed to bf16 pairs (even column low). nlse2 holds -LSE * log2(e)
// of the same W queries.
template <int W, bool kMasked, bool kAlibi = false>
__device__ __forceinline__ void bwd_probs(const uint32_t (&s0)[W], float c, const float* nlse2, int qbase, int qlo,
                                          int qhi, uint32_t (&pk)[W / 2], float d0 = 0.0f, float nslope2 = 0.0f) {
  // ALiBi: d0 = qbase - key; the bias of column f is nslope2 * |d0 + f| (nslope2 = -m log2(e)).
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int e = 0; e < W; e += 4) {
    const float4 nl = *reinterpret_cast<const float4*>(nlse2 + e);
#pragma unroll
    for (int h2 = 0; h2 < 4; h2 += 2) {
      const int f = e + h2;
      const float2 sv = make_float2(__uint_as_float(s0[f]), __uint_as_float(s0[f + 1]));
      float2 xv = fma2(sv, c2, h2 ? make_float2(nl.z, nl.w) : make_float2(nl.x, nl.y));
      if (kAlibi) {
        xv.x = fmaf(fabsf(d0 + (float)f), nslope2, xv.x);
        xv.y = fmaf(fabsf(d0 + (float)(f + 1)), nslope2, xv.y);
      }
      float2 pv;
      if (((f >> 1) % kBwdPolyDen) < kBwdPolyNum) {
        pv = exp2_poly2(xv);
      } else {
        pv = make_float2(ex2_approx(xv.x), ex2_approx(xv.y));
      }
      if (kMasked) {  // query qbase + f is visible iff 0 <= qbase + f - qlo <= qhi - qlo
        const bool any = qhi >= qlo;
        const unsigned span = any ? (unsigned)(qhi - qlo) : 0u;
        const int off = any ? qbase - qlo : -(1 << 30);
        pv.x = ((unsigned)(off + f) <= span) ? pv.x : 0.0f;
        pv.y = ((unsigned)(off + f + 1) <= span) ? pv.y : 0.0f;
      }
      pk[f >> 1] = pack_bf16x2(pv.x, pv.y);
    }
  }
}

template <int D, bool kDQ, bool kAlibi = false, bool kVarlen = false>
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                  const __grid_constant__ CUtensorMap tmdQacc, const BwdParams p) {
  using Cfg = BwdCfg<D>;
  static_assert(sizeof(BwdBars) <= 256, "barrier block");
  constexpr bool kDqFirst = D == 128;  // MMA order per Q tile: see the issuer
  constexpr bool kEpiInDq = Cfg::kKVSlots == 2;  // d = 64: the dQ warps store dK and dV
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = smem_u32(smem_raw);
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem_raw + Cfg::kOffBar);
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };
  // 128-byte swizzled tiles need 1024-byte alignment; the kernel reports instead of faulting.
  if (smem_base & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_fa_error, kErrSmemAlign);
    return;
  }

  const int warp = threadIdx.x >> 5;
  const Abort ab{&bars->abort_flag};
  const uint32_t smem_end = smem_base + Cfg::kSmemBytes;  // for the FA_DEBUG bounds checks
  // FA_DEBUG: the d/64 boxes of the 128-row bf16 tile at `row` of (b, h)
  auto tile_ok = [&](uint32_t dst, int row, int b, int h) {
    bool ok = true;
#pragma unroll
    for (int bx = 0; bx < Cfg::kBoxes; ++bx)
      ok = ok && dbg_tma(ab, bx * 64, row, h, b, D, p.N, p.H, p.B, 2, dst + bx * 16384, 16384, smem_base, smem_end);
    return ok;
  };

  if (threadIdx.x == 0) {
    bars->abort_flag = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(bars->kv_full[s]), 1);
      mbar_init(bar(bars->kv_empty[s]), 1);
      mbar_init(bar(bars->dkv_full[s]), 1);
      mbar_init(bar(bars->dkv_empty[s]), kEpiInDq ? 128 : 128 + 128 * Cfg::kGroups);
      mbar_init(bar(bars->q_full[s]), 1);
      mbar_init(bar(bars->q_empty[s]), 1);
      mbar_init(bar(bars->item_full[s]), 1);
      mbar_init(bar(bars->item_empty[s]), Cfg::kItemConsumers);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(bars->do_full[s]), 1);
      mbar_init(bar(bars->do_empty[s]), 1);
    }
    mbar_init(bar(bars->s_full), 1);
    mbar_init(bar(bars->dp_full), 1);
    mbar_init(bar(bars->p_full), 128 * Cfg::kGroups);
    mbar_init(bar(bars->ds_full), 128 * Cfg::kGroups);
    mbar_init(bar(bars->ds_empty), 1);
    mbar_init(bar(bars->dq_full), 1);
    mbar_init(bar(bars->dq_empty), 128);
    mbar_init(bar(bars->mma_done), 1);
    fence_barrier_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
    prefetch_tmap(&tmdK);
    prefetch_tmap(&tmdV);
    prefetch_tmap(&tmdQacc);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), Cfg::kTmemCols);
    tmem_relinquish();
    tc_fence_before_sync();
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  // K/V slot of the items-th work item of a role (the items of a CTA alternate between slots)
  auto sKs = [&](uint32_t items) { return smem_base + Cfg::kOffK + (items % Cfg::kKVSlots) * 2 * Cfg::kTileBytes; };
  auto sVs = [&](uint32_t items) { return smem_base + Cfg::kOffV + (items % Cfg::kKVSlots) * 2 * Cfg::kTileBytes; };
  // dO slot of the n-th Q tile a role handles (Q tiles of a CTA alternate between the slots)
  auto sDOs = [&](uint32_t n) { return smem_base + Cfg::kOffDO + (n % Cfg::kDOSlots) * Cfg::kTileBytes; };
  const uint32_t sDS = smem_base + Cfg::kOffDS;
  const uint32_t sDQ = smem_base + Cfg::kOffDQ;
  auto sQ = [&](int s) { return smem_base + Cfg::kOffQ + s * Cfg::kTileBytes; };
  auto sStat = [&](int s) { return smem_base + Cfg::kOffStat + s * 1024; };

  if (warp == 0) {
    // ---------------------------------------------------------------- work fetch + TMA producer
    if (lane_id() == 0) {
      uint32_t items = 0, qs = 0, qphase = 0, dn = 0;
      int last_q_parity[2] = {-1, -1};
      for (uint32_t n = 0;; ++n) {
        const uint32_t slot = n & 1;
        mbar_wait_ring(bar(bars->item_empty[slot]), ((n >> 1) & 1) ^ 1, ab);  // slot read by every consumer
        const int w = ab.raised() ? p.num_items : atomicAdd(p.next_item, 1);
        bars->item_w[slot] = w;
        mbar_arrive(bar(bars->item_full[slot]));
        if (w >= p.num_items) break;
        int b, h, j;
        bwd_decode(p, w, b, h, j);
        int lo, hi;
        bwd_q_range<kVarlen>(p, j, lo, hi);
        const uint32_t kvs = items % Cfg::kKVSlots, kvphase = (items / Cfg::kKVSlots) & 1;
        mbar_wait(bar(bars->kv_empty[kvs]), kvphase ^ 1, ab);
        if (!tile_ok(sKs(items), j * 128, b, h) || !tile_ok(sVs(items), j * 128, b, h)) break;
        mbar_arrive_expect_tx(bar(bars->kv_full[kvs]), 2 * Cfg::kTileBytes);
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
          tma_load_4d(sKs(items) + bx * 16384, &tmK, bar(bars->kv_full[kvs]), bx * 64, j * 128, h, b);
          tma_load_4d(sVs(items) + bx * 16384, &tmV, bar(bars->kv_full[kvs]), bx * 64, j * 128, h, b);
        }
        ++items;
        const size_t stat_row = ((size_t)b * p.H + h) * (size_t)p.N_pad;
        for (int i = lo; i <= hi; ++i, ++dn) {
          // Q_i and its statistics into the next Q slot
          mbar_wait(bar(bars->q_empty[qs]), qphase ^ 1, ab);
          const uint32_t fb = bar(bars->q_full[qs]);
          const long long stat_size = (long long)p.B * p.H * p.N_pad;
          if (!tile_ok(sQ(qs), i * 128, b, h) || !dbg_range(ab, (long long)stat_row + i * 128, 128, stat_size) ||
              !dbg_range(ab, sStat(qs) - smem_base, 1024, smem_end - smem_base))
            break;
          mbar_arrive_expect_tx(fb, Cfg::kTileBytes + 1024);
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx) tma_load_4d(sQ(qs) + bx * 16384, &tmQ, fb, bx * 64, i * 128, h, b);
          bulk_load(sStat(qs), p.lse2 + stat_row + i * 128, 512, fb);
          bulk_load(sStat(qs) + 512, p.dvec + stat_row + i * 128, 512, fb);
          last_q_parity[qs] = qphase;
          if (++qs == 2) { qs = 0; qphase ^= 1; }
          // dO_i into the single dO slot (freed when dV_{i-1} is done)
          const uint32_t dos = dn % Cfg::kDOSlots, dophase = (dn / Cfg::kDOSlots) & 1;
          mbar_wait(bar(bars->do_empty[dos]), dophase ^ 1, ab);
          if (!tile_ok(sDOs(dn), i * 128, b, h)) break;  // (the next fetch then ends the loop)
          mbar_arrive_expect_tx(bar(bars->do_full[dos]), Cfg::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_4d(sDOs(dn) + bx * 16384, &tmdO, bar(bars->do_full[dos]), bx * 64, i * 128, h, b);
        }
      }
      for (int s = 0; s < 2; ++s)
        if (last_q_parity[s] >= 0) mbar_drain(bar(bars->q_full[s]), last_q_parity[s]);
      for (uint32_t t = (dn > Cfg::kDOSlots ? dn - Cfg::kDOSlots : 0); t < dn; ++t)
        mbar_drain(bar(bars->do_full[t % Cfg::kDOSlots]), (t / Cfg::kDOSlots) & 1);
      for (uint32_t t = (items > Cfg::kKVSlots ? items - Cfg::kKVSlots : 0); t < items; ++t)
        mbar_drain(bar(bars->kv_full[t % Cfg::kKVSlots]), (t / Cfg::kKVSlots) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // Per Q tile i: dP(i), dV(i), then S(i+1), dQ(i), dK(i) at d = 64 (the P of tile i+1 is
    // computed while the tensor core works on dQ and dK of tile i) or dQ(i), S(i+1), dK(i) at
    // d = 128 (dQ(i) and its drain from TMEM, which the next dP waits for, start earlier).
    if (elect_one()) {
      constexpr uint32_t idSP = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T: K-major A and B
      constexpr uint32_t idKV = idesc_bf16_f32(128, D, false, true);     // dV, dK: B (dO, Q) MN-major
      constexpr uint32_t idQ = idesc_bf16_f32(128, D, true, true);       // dQ: A (dS) and B (K) MN-major
      const uint32_t tDP = tmem + Cfg::kColDP, tS = tmem + Cfg::kColS;
      uint32_t items = 0, n = 0, qs = 0, qphase = 0;
      uint32_t sK = sKs(0), sV = sVs(0);
      auto issue_s = [&](uint32_t slot, uint32_t phase) {
        mbar_wait(bar(bars->q_full[slot]), phase, ab);
        tc_fence_after_sync();
        const uint32_t q = sQ(slot);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tS, sdesc_kmajor(sK + off), sdesc_kmajor(q + off), idSP, kk > 0);
        }
        mma_commit(bar(bars->s_full));
      };
      for (uint32_t it = 0;; ++it) {
        const int w = bwd_take_item(bars, it, true, ab);
        if (w >= p.num_items) break;
        int b, h, j;
        bwd_decode(p, w, b, h, j);
        int lo, hi;
        bwd_q_range<kVarlen>(p, j, lo, hi);
        const uint32_t kvs = items % Cfg::kKVSlots, kvphase = (items / Cfg::kKVSlots) & 1;
        sK = sKs(items);
        sV = sVs(items);
        const uint32_t tDK = tmem + (kvs ? Cfg::kColDK1 : Cfg::kColDK);
        const uint32_t tDV = tmem + (kvs ? Cfg::kColDV1 : Cfg::kColDV);
        mbar_wait(bar(bars->kv_full[kvs]), kvphase, ab);
        tc_fence_after_sync();
        issue_s(qs, qphase);  // S(lo)
        for (int i = lo; i <= hi; ++i, ++n) {
          const bool first = (i == lo);
          const uint32_t q = sQ(qs);
          // dP^T = V_j dO_i^T into the columns dQ_{i-1} occupied
          const uint32_t sDO = sDOs(n), dos = n % Cfg::kDOSlots;
          mbar_wait(bar(bars->do_full[dos]), (n / Cfg::kDOSlots) & 1, ab);
          if (kDQ) mbar_wait(bar(bars->dq_empty), (n & 1) ^ 1, ab);
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_ss(tDP, sdesc_kmajor(sV + off), sdesc_kmajor(sDO + off), idSP, kk > 0);
          }
          mma_commit(bar(bars->dp_full));
          // dV += P^T dO_i (P^T packed in TMEM: the W = kGroupCols queries [W g, W g + W) of P/dS
          // group g in S columns [W g, W g + W / 2))
          mbar_wait(bar(bars->p_full), n & 1, ab);
          if (first) mbar_wait(bar(bars->dkv_empty[kvs]), kvphase ^ 1, ab);
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            constexpr int W = Cfg::kGroupCols;
            const uint32_t acol = (16 * kk / W) * W + (16 * kk % W) / 2;
            mma_ts(tDV, tS + acol, sdesc_mnmajor(sDO + kk * 2048, 16384), idKV, !first || kk > 0);
          }
          mma_commit(bar(bars->do_empty[dos]));
          // S(i+1): overwrites P^T(i), which dV(i) (issued before) has read. d = 64 issues it
          // here, ahead of dQ(i), so that the P of tile i+1 is computed meanwhile; d = 128
          // issues dQ(i) first, which shortens the chain dS(i) -> dQ(i) -> dQ drained -> dP(i+1).
          const uint32_t nqs = qs ^ 1, nqphase = qs ? (qphase ^ 1) : qphase;
          if (!kDqFirst && i < hi) issue_s(nqs, nqphase);
          // dQ_i = dS K_j, then dK += dS^T Q_i
          mbar_wait(bar(bars->ds_full), n & 1, ab);
          tc_fence_after_sync();
          if (kDQ) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tDP, sdesc_mnmajor(sDS + kk * 2048, 16384), sdesc_mnmajor(sK + kk * 2048, 16384), idQ, kk > 0);
            mma_commit(bar(bars->dq_full));
          }
          if (kDqFirst && i < hi) issue_s(nqs, nqphase);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_ss(tDK, sdesc_kmajor(sDS + off), sdesc_mnmajor(q + kk * 2048, 16384), idKV, !first || kk > 0);
          }
          mma_commit(bar(bars->ds_empty));
          mma_commit(bar(bars->q_empty[qs]));
          qs = nqs;
          qphase = nqphase;
        }
        mma_commit(bar(bars->dkv_full[kvs]));
        // d = 128: the epilogue stages through the dS and dQ buffers, so K_j and V_j are free
        // once the item's products are done (d = 64 stages through them: the dQ warps release)
        if constexpr (!kEpiInDq) mma_commit(bar(bars->kv_empty[kvs]));
        ++items;
      }
      mma_commit(bar(bars->mma_done));
      mbar_drain(bar(bars->mma_done), 0);
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------------------------------------------- dQ accumulation
    // dQ_i (fp32, times scale) goes TMEM -> registers -> a 128B-swizzled staging tile in shared
    // memory, and the TMA unit adds it into the accumulator in global memory, 64 columns per round.
    const int row = threadIdx.x - 128;
    const uint32_t tDQ = tmem + ((uint32_t)(row & ~31) << 16) + Cfg::kColDP;
    uint32_t n = 0, items = 0;
    for (uint32_t it = 0;; ++it) {
      const int w = bwd_take_item(bars, it, lane_id() == 0, ab);
      if (w >= p.num_items) break;
      int b, h, j;
      bwd_decode(p, w, b, h, j);
      int lo, hi;
      bwd_q_range<kVarlen>(p, j, lo, hi);
      // Without kDQ, dQ comes from its own kernel: these warps only follow the items.
      for (int i = lo; kDQ && i <= hi; ++i, ++n) {
        mbar_wait(bar(bars->dq_full), n & 1, ab);
        tc_fence_after_sync();
#pragma unroll
        for (int r = 0; r < Cfg::kDqRounds; ++r) {
          uint32_t v0[32], v1[32];
          tmem_ld32(tDQ + r * 64, v0);
          tmem_ld32(tDQ + r * 64 + 32, v1);
          tmem_wait_ld(v0);
          tmem_wait_ld(v1);
          if (r == Cfg::kDqRounds - 1) {
            tc_fence_before_sync();
            mbar_arrive(bar(bars->dq_empty));
          }
          if (row == 0) bulk_wait_group_read0();  // the previous reduction has read the staging tile
          named_bar_sync(3, 128);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            st_shared_v4(sDQ + sw128_offset(row, ch), __float_as_uint(__uint_as_float(v0[4 * ch]) * p.scale),
                         __float_as_uint(__uint_as_float(v0[4 * ch + 1]) * p.scale),
                         __float_as_uint(__uint_as_float(v0[4 * ch + 2]) * p.scale),
                         __float_as_uint(__uint_as_float(v0[4 * ch + 3]) * p.scale));
            st_shared_v4(sDQ + 16384 + sw128_offset(row, ch), __float_as_uint(__uint_as_float(v1[4 * ch]) * p.scale),
                         __float_as_uint(__uint_as_float(v1[4 * ch + 1]) * p.scale),
                         __float_as_uint(__uint_as_float(v1[4 * ch + 2]) * p.scale),
                         __float_as_uint(__uint_as_float(v1[4 * ch + 3]) * p.scale));
          }
          fence_proxy_async_smem();
          named_bar_sync(3, 128);
          if (row == 0 &&
              dbg_tma(ab, r * 64, i * 128, h, b, D, p.N, p.H, p.B, 4, sDQ, 16384, smem_base, smem_end) &&
              dbg_tma(ab, r * 64 + 32, i * 128, h, b, D, p.N, p.H, p.B, 4, sDQ + 16384, 16384, smem_base, smem_end)) {
            tma_reduce_add_4d(&tmdQacc, sDQ, r * 64, i * 128, h, b);
            tma_reduce_add_4d(&tmdQacc, sDQ + 16384, r * 64 + 32, i * 128, h, b);
            bulk_commit_group();
          }
        }
      }
      if constexpr (kEpiInDq) {
        // dK (times scale) and dV -> bf16 -> this item's K_j / V_j buffers -> TMA store
        const uint32_t kvs = items % Cfg::kKVSlots, kvphase = (items / Cfg::kKVSlots) & 1;
        mbar_wait(bar(bars->dkv_full[kvs]), kvphase, ab);
        tc_fence_after_sync();
        const uint32_t lane_field = (uint32_t)((row & ~31) << 16);
#pragma unroll 1
        for (int g = 0; g < 2; ++g) {
          const uint32_t src =
              tmem + lane_field + (g ? (kvs ? Cfg::kColDV1 : Cfg::kColDV) : (kvs ? Cfg::kColDK1 : Cfg::kColDK));
          const uint32_t stage_buf = g ? sVs(items) : sKs(items);
          const float mult = g ? 1.0f : p.scale;
#pragma unroll
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
                w4[e] = pack_bf16x2(__uint_as_float(v[ch * 8 + 2 * e]) * mult,
                                    __uint_as_float(v[ch * 8 + 2 * e + 1]) * mult);
              st_shared_v4(bx + sw128_offset(row, ((cc & 63) >> 3) + ch), w4[0], w4[1], w4[2], w4[3]);
            }
          }
        }
        tc_fence_before_sync();
        mbar_arrive(bar(bars->dkv_empty[kvs]));
        fence_proxy_async_smem();
        named_bar_sync(3, 128);
        if (row == 0) {
#pragma unroll
          for (int g = 0; g < 2; ++g)
#pragma unroll
            for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
              const uint32_t sb = (g ? sVs(items) : sKs(items)) + bx * 16384;
              if (dbg_tma(ab, bx * 64, j * 128, h, b, D, p.N, p.H, p.B, 2, sb, 16384, smem_base, smem_end))
                tma_store_4d(g ? &tmdV : &tmdK, sb, bx * 64, j * 128, h, b);
            }
          bulk_commit_group();
          bulk_wait_group_read0();
          mbar_arrive(bar(bars->kv_empty[kvs]));
        }
      } else {
        // d = 128: dV -> bf16 -> the dQ staging buffer (two 64-column boxes) -> TMA store, once
        // the item's last dQ reduction has read that buffer; the next item's first staging
        // round waits for this store to read it in turn (the same bulk-group wait)
        const uint32_t kvs = items % Cfg::kKVSlots, kvphase = (items / Cfg::kKVSlots) & 1;
        mbar_wait(bar(bars->dkv_full[kvs]), kvphase, ab);
        tc_fence_after_sync();
        if (row == 0) bulk_wait_group_read0();
        named_bar_sync(3, 128);
        const uint32_t src = tmem + ((uint32_t)(row & ~31) << 16) + Cfg::kColDV;
#pragma unroll 1
        for (int cc = 0; cc < D; cc += 32) {
          uint32_t v[32];
          tmem_ld32(src + cc, v);
          tmem_wait_ld(v);
          const uint32_t bx = sDQ + (cc >> 6) * 16384;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w4[e] = pack_bf16x2(__uint_as_float(v[ch * 8 + 2 * e]), __uint_as_float(v[ch * 8 + 2 * e + 1]));
            st_shared_v4(bx + sw128_offset(row, ((cc & 63) >> 3) + ch), w4[0], w4[1], w4[2], w4[3]);
          }
        }
        tc_fence_before_sync();
        mbar_arrive(bar(bars->dkv_empty[kvs]));
        fence_proxy_async_smem();
        named_bar_sync(3, 128);
        if (row == 0) {
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            if (dbg_tma(ab, bx * 64, j * 128, h, b, D, p.N, p.H, p.B, 2, sDQ + bx * 16384, 16384, smem_base, smem_end))
              tma_store_4d(&tmdV, sDQ + bx * 16384, bx * 64, j * 128, h, b);
          bulk_commit_group();
        }
      }
      ++items;
    }
    if (row == 0) bulk_wait_group0();
  } else if (warp >= 8) {
    // ---------------------------------------------------------------- P, dS and the dK epilogue
    // kGroups groups of four warps; group g takes the W query columns [W g, W g + W) of every
    // tile (and, at d = 128, dK columns [W g, W g + W) of the epilogue).
    constexpr int W = Cfg::kGroupCols;
    const int grp = (warp - 8) >> 2;
    const int row = (threadIdx.x - 256) & 127;  // key row within the tile == TMEM lane
    const uint32_t lane_field = (uint32_t)((row & ~31) << 16);
    const uint32_t tS = tmem + lane_field + Cfg::kColS + W * grp;
    const uint32_t tDP = tmem + lane_field + Cfg::kColDP + W * grp;
    // this group's queries in the dS tile: box (W grp) / 64, 16-byte chunks from (W grp % 64) / 8
    const uint32_t ds_box = sDS + (W * grp / 64) * 16384;
    const int ds_chunk0 = (W * grp % 64) / 8;
    const float c = p.scale_log2;
    uint32_t items = 0, n = 0, qs = 0, qphase = 0;
    for (uint32_t it = 0;; ++it) {
      const int w = bwd_take_item(bars, it, lane_id() == 0, ab);
      if (w >= p.num_items) break;
      int b, h, j;
      bwd_decode(p, w, b, h, j);
      int lo, hi;
      bwd_q_range<kVarlen>(p, j, lo, hi);
      const int k = j * 128 + row;
      const float nslope2 = kAlibi ? -p.alibi_slopes[b * p.H + h] * kLog2e : 0.0f;
      int first = 0, last = p.N - 1;
      if (kVarlen && k < p.N) seg_bounds(p.cu_seqlens, p.nseg, p.N, k, first, last);
      int seg_first = 0, seg_last = 0;  // sequence of the tile's first key (packed batches)
      if (kVarlen) seg_bounds(p.cu_seqlens, p.nseg, p.N, j * 128, seg_first, seg_last);
      const int qlo = p.win_r >= 0 ? max(first, k - p.win_r) : first;
      const int qhi = (k >= p.N) ? -1 : (p.win_l >= 0 ? min(last, k + p.win_l) : last);
      for (int i = lo; i <= hi; ++i, ++n) {
        // the Q slot's LSE2_i / D_i rows are read here
        mbar_wait(bar(bars->q_full[qs]), qphase, ab);
        const float* nlse2 = reinterpret_cast<const float*>(smem_raw + Cfg::kOffStat + qs * 1024);  // -LSE*log2(e)
        const float* nd = nlse2 + 128;                                                              // -D
        const bool masked = !bwd_tile_unmasked<kVarlen>(p, j, i, seg_first, seg_last);
        const int qbase = i * 128 + W * grp;

        mbar_wait(bar(bars->s_full), n & 1, ab);
        tc_fence_after_sync();
        uint32_t s0[W];
#pragma unroll
        for (int q = 0; q < W / 32; ++q) tmem_ld32(tS + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&s0[32 * q]));
#pragma unroll
        for (int q = 0; q < W / 32; ++q) tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&s0[32 * q]));
        uint32_t pk[W / 2];  // packed P over the first W / 2 of this group's S columns, read above
        const float dist0 = (float)(qbase - k);
        if (masked)
          bwd_probs<W, true, kAlibi>(s0, c, nlse2 + W * grp, qbase, qlo, qhi, pk, dist0, nslope2);
        else
          bwd_probs<W, false, kAlibi>(s0, c, nlse2 + W * grp, qbase, qlo, qhi, pk, dist0, nslope2);
#pragma unroll
        for (int q = 0; q < W / 32; ++q) tmem_st16(tS + 16 * q, *reinterpret_cast<uint32_t(*)[16]>(&pk[16 * q]));
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(bar(bars->p_full));

        mbar_wait(bar(bars->dp_full), n & 1, ab);
        tc_fence_after_sync();
        uint32_t d0[W];
#pragma unroll
        for (int q = 0; q < W / 32; ++q) tmem_ld32(tDP + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&d0[32 * q]));
#pragma unroll
        for (int q = 0; q < W / 32; ++q) tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&d0[32 * q]));
        // dS^T(row, q) = P^T(row, q) * (dP^T(row, q) - D_q) -> bf16 -> shared, 128B-swizzled rows of
        // keys (the group's queries: chunks ds_chunk0 .. ds_chunk0 + W / 8 - 1 of box ds_box)
        mbar_wait(bar(bars->ds_empty), (n & 1) ^ 1, ab);
#pragma unroll
        for (int ch = 0; ch < W / 8; ++ch) {
          uint32_t w4[4];
          const float4 nda = *reinterpret_cast<const float4*>(nd + W * grp + ch * 8);
          const float4 ndb = *reinterpret_cast<const float4*>(nd + W * grp + ch * 8 + 4);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = ch * 8 + 2 * e;  // within the group
            const float2 g = make_float2(__uint_as_float(d0[col]), __uint_as_float(d0[col + 1]));
            const uint32_t pp = pk[col >> 1];
            const float2 ndv = e == 0 ? make_float2(nda.x, nda.y) : e == 1 ? make_float2(nda.z, nda.w)
                             : e == 2 ? make_float2(ndb.x, ndb.y) : make_float2(ndb.z, ndb.w);
            const float2 diff = add2(g, ndv);
            const float2 ds = mul2(make_float2(bf16lo_to_f32(pp), bf16hi_to_f32(pp)), diff);
            w4[e] = pack_bf16x2(ds.x, ds.y);
          }
          st_shared_v4(ds_box + sw128_offset(row, ds_chunk0 + ch), w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        mbar_arrive(bar(bars->ds_full));
        if (++qs == 2) { qs = 0; qphase ^= 1; }
      }

      // Epilogue (d = 128; at d = 64 the dQ warps do it): dK times scale, columns [W grp,
      // W grp + W) -> bf16 -> the group's chunks of the dS buffer (free: the item's last dQ and
      // dK have read it) -> TMA store of each 64-column box once the groups that fill it are
      // done. Their next dS waits for the store to read the box.
      if constexpr (!kEpiInDq) {
        constexpr int kBoxGroups = 64 / W;  // groups per 64-column box
        const uint32_t kvs = items % Cfg::kKVSlots, kvphase = (items / Cfg::kKVSlots) & 1;
        mbar_wait(bar(bars->dkv_full[kvs]), kvphase, ab);
        tc_fence_after_sync();
#pragma unroll 1
        for (int cc = 0; cc < W; cc += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_field + Cfg::kColDK + W * grp + cc, v);
          tmem_wait_ld(v);
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w4[e] = pack_bf16x2(__uint_as_float(v[ch * 8 + 2 * e]) * p.scale,
                                  __uint_as_float(v[ch * 8 + 2 * e + 1]) * p.scale);
            st_shared_v4(ds_box + sw128_offset(row, ds_chunk0 + cc / 8 + ch), w4[0], w4[1], w4[2], w4[3]);
          }
        }
        tc_fence_before_sync();
        mbar_arrive(bar(bars->dkv_empty[kvs]));
        fence_proxy_async_smem();
        const int box = W * grp / 64;
        named_bar_sync(1 + box, 128 * kBoxGroups);
        if (row == 0 && grp % kBoxGroups == 0) {
          if (dbg_tma(ab, 64 * box, j * 128, h, b, D, p.N, p.H, p.B, 2, ds_box, 16384, smem_base, smem_end))
            tma_store_4d(&tmdK, ds_box, 64 * box, j * 128, h, b);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
        named_bar_sync(1 + box, 128 * kBoxGroups);
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
