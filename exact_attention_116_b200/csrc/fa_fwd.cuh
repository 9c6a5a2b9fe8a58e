// Forward kernel of exact attention for sm_100a.
//
// What it computes ("Flash Attention V2核心网络算子解析" §二.1; "FlashAttention 剖析" §3):
// for every (b, h) and query row i, O_i = sum_j softmax_j(scale * q_i . k_j) v_j over the
// keys j visible to i (causal / (left, right) window), and LSE_i = ln sum_j exp(scale * q_i . k_j).
// Keys are visited in 128-key tiles with a running maximum and running sum per row
// ("FlashAttention技术解析：加速GPT训练的核心优化" §1 item 3), so the N x N score matrix
// never leaves the SM.
//
// Work decomposition (persistent, one CTA per SM):
//   work item = (b, h, pair of 128-row Q tiles); the two Q tiles share every K/V tile load.
//   Items are dealt dynamically: the producer takes the next item from an atomic counter (one
//   slot of a library-owned ring per call, zeroed by the kernel launched just before) and hands
//   it to the other roles through a two-entry ring in shared memory. Items are ordered in groups
//   of heads small enough that the K/V of the heads in flight stay in L2, longest first
//   inside a group under causal masking, and the shortest pair ranks of every head come last
//   (fwd_decode).
//   warp 0      : work fetch and TMA producer (Q tiles; a ring of K/V tile slots)
//   warp 1      : tcgen05 MMA issuer (one elected thread) and TMEM owner
//   warps 2-3   : no role
//   warps 4-7   : softmax + epilogue for Q tile 0 (one thread per query row / TMEM lane)
//   warps 8-11  : softmax + epilogue for Q tile 1
//   warps 12-19 : the second 64 scores of every row of tile 0 (warps 12-15) and tile 1
//                 (warps 16-19); warps 4-11 take the first 64 (640 threads). The two warps of
//                 a row exchange partial maxima and sums (see FwdCfg).
// TMEM (512 columns): O0 [256,256+D), O1 [256+D, 256+2D); S and P as below. P_t (bf16, two
// per column; E4M3, four) is the A operand of O_t += P_t V_j, read straight from TMEM.
//
// D = 128 (kShareS): the two tiles share one S buffer (columns [0,128)), P_t has its own
// columns (P0 from 128, P1 from 192: 64 columns of bf16 pairs or 32 of E4M3 quads), O0
// [256,384), O1 [384,512). The S buffer holds S0(j), S1(j), S0(j+1), ... in turn, each issued
// as soon as the softmax threads have read the previous one into registers ("S empty"), so a
// tile's next scores do not wait for its P·V. MMA issue order per KV tile j: S0(j+1), PV0(j),
// S1(j+1), PV1(j). A softmax thread writes P_t(j+1) and rescales O_t only after the commit of
// PV_t(j) ("PV done"). bf16: the O tile is staged for its TMA store in the Q_t buffer (free
// once the item's last PV_t is done); E4M3: O has staging buffers of its own and Q_t is
// released by the commit of the item's last S_t.
//
// D = 64: each tile has its own S (S0 [0,128), S1 [128,256)) and P (P0 [384,448), P1
// [448,512)) columns, so S_t(j+1) is issued as soon as the softmax threads have read S_t(j)
// into registers ("S empty"), one tile ahead of PV_t(j): the next scores are ready when a
// softmax thread finishes a tile. A softmax thread writes P_t(j+1) and rescales O_t only after
// the commit of PV_t(j) ("PV done"). O is staged in buffers of its own, so Q_t is released by
// the commit of the item's last S_t and the next item's Q and K/V loads overlap this item's
// last tiles and epilogue.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

struct FwdParams {
  int B, N, H;
  float scale_log2;  // softmax scale * log2(e)
  int win_l;         // -1 = unbounded
  int win_r;         // effective right bound (0 under causal), -1 = unbounded
  int causal;
  int num_pairs;     // ceil(N / 256)
  int num_items;     // B * H * num_pairs
  float* lse;        // (B, H, N) fp32
  int debug_drop_s_signal;  // test only: withhold the first "S ready" signal (a wait must time out)
  const float* q_descale;   // E4M3 inputs only: (B, H) factors, value = descale * code
  const float* k_descale;
  const float* v_descale;
  const float* alibi_slopes;  // ALiBi only: (B, H) slopes m, bias -m |i - j| on the scaled scores
  const int* cu_seqlens;      // packed variable-length batch (B = 1, N = total): nseg + 1 offsets, or null
  int nseg;
  int head_group;             // heads per scheduling group (>= 1)
  int tail_ranks;             // shortest pair ranks dealt last over all heads at once (<= num_pairs)
  int counter_slot;           // this call's work counter: g_fwd_next_item[counter_slot]
};

// Work counters of the forward, one per call in flight: the host hands out the slots in turn
// and zeroes a call's slot with fa_fwd_counter_reset_kernel just before the forward kernel.
constexpr int kFwdCounterSlots = 1024;
__device__ int g_fwd_next_item[kFwdCounterSlots];

__global__ void fa_fwd_counter_reset_kernel(int slot) {
  griddep_launch_dependents();  // the forward (its programmatic dependent) may start setting up
  if (threadIdx.x == 0) g_fwd_next_item[slot] = 0;
}

constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may grow to 2^8 before O is rescaled

// Packed batches: the cost of a pair of Q tiles (its visible KV tiles) does not fall with its
// index, so every CTA sorts the pairs by decreasing cost (ties: higher index first) before
// dealing them out; the same deterministic order in every CTA keeps each item dealt once.
// Up to kFwdSortMaxPairs pairs (524288 tokens); above that the index order is kept.
constexpr int kFwdSortMaxPairs = 2048;
constexpr int kFwdSortBytes = 4 * kFwdSortMaxPairs;  // uint16 cost and order per pair

// Share of the exponentials computed by exp2_poly on the FMA pipes instead of MUFU: pair p of
// a row's 64 pairs uses the polynomial when p % kPolyDen < kPolyNum.
#ifndef FA_FWD_POLY_NUM
#define FA_FWD_POLY_NUM 1
#endif
#ifndef FA_FWD_POLY_DEN
#define FA_FWD_POLY_DEN 8
#endif
constexpr int kFwdPolyNum = FA_FWD_POLY_NUM, kFwdPolyDen = FA_FWD_POLY_DEN;

constexpr float kLn2 = 0.69314718055994530942f;

// kF8: Q, K, V are E4M3 (one byte per element), S and P·V run as kind::f8f6f4 with P
// quantised to E4M3 in TMEM (four per column); O is bf16 as for bf16 inputs.
template <int D, bool kF8 = false>
struct FwdCfg {
  // Each row's 128 scores of a KV tile are split over two warps (64 each), which exchange their
  // partial row maxima through shared memory, so that four softmax warps share each SM
  // sub-partition (kept as a switch: kSplitRow = false is the one-warp-per-row layout).
  static constexpr bool kSplitRow = true;
  static constexpr int kHalves = kSplitRow ? 2 : 1;
  static constexpr int kCols = 128 / kHalves;              // scores per softmax thread and KV tile
  static constexpr int kThreads = 128 + 256 * kHalves;     // 384, or 640 with the row split
  static constexpr uint32_t kItemConsumers = 1 + 8 * kHalves;  // MMA thread and softmax warps
  static constexpr int kXBytes = kSplitRow ? 8192 : 0;     // row-split exchange: maxima, then sums
  static constexpr int kElem = kF8 ? 1 : 2;        // bytes per Q/K/V element
  static constexpr int kTileBytes = 128 * D * kElem;  // one 128-row tile of Q, K or V
  static constexpr int kOTileBytes = 128 * D * 2;     // one 128-row bf16 tile of O
  static constexpr int kBoxes = D * kElem / 128;      // 128-byte-wide TMA boxes per Q/K/V tile
  static constexpr int kBoxElems = 128 / kElem;       // elements per box row
  static constexpr int kOBoxes = D / 64;              // 64-column boxes per O tile
  static constexpr int kSlots = (kTileBytes == 32768) ? 4 : (kF8 && kSplitRow) ? 7 : 8;
  static constexpr bool kShareS = (D == 128);          // one S buffer for both tiles
  static_assert(D == 128 || !kF8, "E4M3 tiles are 128 bytes wide: d = 128");
  static constexpr bool kSepO = (D == 64) || kF8;     // O staging apart from Q; Q freed by the last S
  static constexpr int kKSteps = D * kElem / 32;      // MMA steps over d (32 bytes of K each)
  static constexpr int kPvSteps = kF8 ? 4 : 8;        // MMA steps over the 128 keys of P
  static constexpr int kOffQ = 0;                     // Q0, Q1 (also O staging unless kSepO)
  static constexpr int kOffO = 2 * kTileBytes;        // O staging 0, 1 (kSepO)
  static constexpr int kOffKV = kSepO ? kOffO + 2 * kOTileBytes : 2 * kTileBytes;
  static constexpr int kOffX = kOffKV + kSlots * kTileBytes;
  static constexpr int kOffBar = kOffX + kXBytes;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;  // barriers + alignment slack
  static constexpr int kOffSort = kOffBar + 512;            // packed batches: pair costs and order
  static constexpr uint32_t kColS0 = 0, kColS1 = kShareS ? 0 : 128, kColO0 = 256, kColO1 = 256 + D;
  static constexpr uint32_t kColP0 = kShareS ? 128 : 384, kColP1 = kShareS ? 192 : 448;  // P apart from S
  static constexpr uint32_t kTmemCols = 512;
};

// Barrier block at the end of shared memory.
template <class Cfg>
struct FwdBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[Cfg::kSlots], kv_empty[Cfg::kSlots];
  uint64_t s_full[2], p_full[2];
  uint64_t s_empty[2], pv_done[2];  // kShareS: s_empty[0] for the shared S
  uint64_t mma_done;
  uint64_t item_full[2], item_empty[2];  // ring of fetched work items, producer -> other roles
  int item_w[2];
  uint32_t tmem_base;
  int abort_flag;
};

// Next work item of a consumer role (n counts the items this role has taken); values >=
// num_items mean "no more work".
template <class Bars>
__device__ __forceinline__ int fwd_take_item(Bars* bars, uint32_t n, bool arrive, Abort ab) {
  const uint32_t slot = n & 1;
  const bool ok = mbar_wait_ring(smem_u32(&bars->item_full[slot]), (n >> 1) & 1, ab);
  const int w = *reinterpret_cast<volatile int*>(&bars->item_w[slot]);
  __syncwarp(__activemask());
  if (arrive) mbar_arrive(smem_u32(&bars->item_empty[slot]));
  return ok ? w : 0x7fffffff;
}

// Item w -> (b, h, pair). Pair rank r is pair num_pairs - 1 - r under causal masking (longest
// first), order[r] for a packed batch (pairs by decreasing cost), else r. Two phases:
//   1. ranks [0, num_pairs - tail_ranks): groups of head_group heads in order, inside a group
//      the rank slowest and the heads fastest, so that the K/V read by the items in flight
//      belong to few heads and stay in L2;
//   2. the tail_ranks shortest ranks over all heads, rank-major: the last items dealt are the
//      shortest, whatever group ran last, so the CTAs finish together (the items of this phase
//      read only the first few K/V tiles of each head).
__device__ __forceinline__ void fwd_decode(const FwdParams& p, int w, int& b, int& h, int& pair,
                                           const uint16_t* order = nullptr) {
  const int bh_count = p.B * p.H;
  const int ranks1 = p.num_pairs - p.tail_ranks;
  const int n1 = bh_count * ranks1;
  int r, bh;
  if (w < n1) {
    const int per_group = p.head_group * ranks1;
    const int g = w / per_group;
    const int pos = w - g * per_group;
    const int gs = min(p.head_group, bh_count - g * p.head_group);  // heads in this group
    r = pos / gs;
    bh = g * p.head_group + (pos - r * gs);
  } else {
    const int w2 = w - n1;
    const int r2 = w2 / bh_count;
    r = ranks1 + r2;
    bh = w2 - r2 * bh_count;
  }
  pair = order ? (int)order[r] : p.causal ? (p.num_pairs - 1 - r) : r;
  b = bh / p.H;
  h = bh - b * p.H;
}

// KV tiles visible from Q rows [r0, min(r0+127, N-1)]; empty (hi < lo) if r0 >= N.
// Packed sequences (kVarlen): the keys of the first row's sequence start to the last row's
// sequence end.
template <bool kVarlen>
__device__ __forceinline__ void fwd_kv_range(const FwdParams& p, int r0, int& lo, int& hi) {
  if (r0 >= p.N) { lo = 0; hi = -1; return; }
  const int r1 = min(r0 + 127, p.N - 1);
  int first = 0, last = p.N - 1, dummy;
  if (kVarlen) {
    seg_bounds(p.cu_seqlens, p.nseg, p.N, r0, first, dummy);
    seg_bounds(p.cu_seqlens, p.nseg, p.N, r1, dummy, last);
  }
  const int kmin = p.win_l >= 0 ? max(first, r0 - p.win_l) : first;
  const int kmax = p.win_r >= 0 ? min(last, r1 + p.win_r) : last;
  lo = kmin >> 7;
  hi = kmax >> 7;
}

// Visible keys [kmin, kmax] of query row i (its own sequence only when packed).
template <bool kVarlen>
__device__ __forceinline__ void fwd_row_keys(const FwdParams& p, int i, int& kmin, int& kmax) {
  int first = 0, last = p.N - 1;
  if (kVarlen && i < p.N) seg_bounds(p.cu_seqlens, p.nseg, p.N, i, first, last);
  kmin = p.win_l >= 0 ? max(first, i - p.win_l) : first;
  kmax = (i >= p.N) ? -1 : (p.win_r >= 0 ? min(last, i + p.win_r) : last);
}

// True when every valid row of the Q tile sees every key of KV tile j (no masking needed).
// Packed sequences (kVarlen): [seg_first, seg_last] are the rows of the sequence of row r0.
template <bool kVarlen>
__device__ __forceinline__ bool fwd_tile_unmasked(const FwdParams& p, int r0, int j, int seg_first = 0,
                                                  int seg_last = 0) {
  const int r1 = min(r0 + 127, p.N - 1);
  const int k0 = j * 128, k1 = k0 + 127;
  if (k1 >= p.N) return false;
  if (p.win_l >= 0 && k0 < r1 - p.win_l) return false;
  if (p.win_r >= 0 && k1 > r0 + p.win_r) return false;
  if (kVarlen && (r1 > seg_last || k0 < seg_first || k1 > seg_last)) return false;  // one sequence only
  return true;
}

// ------------------------------------------------------------------ softmax role

// Maximum of this thread's kC scores of a key tile (scaled, log2 units), x[0] being key kbase,
// with masking. x is scaled in place when the scale is not positive, and always with ALiBi,
// whose bias nslope2 * |d0 - cc| (nslope2 = -m log2(e), d0 = row - kbase) is added after the
// scaling.
template <bool kPosScale, bool kAlibi = false, int kC>
__device__ __forceinline__ float fwd_tile_max(float (&x)[kC], bool masked, int kbase, int kmin, int kmax, float c,
                                              float d0 = 0.0f, float nslope2 = 0.0f) {
  static_assert(!(kAlibi && kPosScale), "the ALiBi bias is added to scaled scores");
  if (kAlibi) {
#pragma unroll
    for (int cc = 0; cc < kC; ++cc) x[cc] = fmaf(fabsf(d0 - (float)cc), nslope2, x[cc] * c);
  } else if (!kPosScale) {  // then masking must follow the scaling
#pragma unroll
    for (int cc = 0; cc < kC; cc += 2) {
      const float2 v = mul2(make_float2(x[cc], x[cc + 1]), make_float2(c, c));
      x[cc] = v.x;
      x[cc + 1] = v.y;
    }
  }
  if (masked) {
    // key kbase + cc is visible iff 0 <= kbase + cc - kmin <= kmax - kmin: one unsigned compare
    // per score (an empty range masks every key)
    const bool any = kmax >= kmin;
    const unsigned span = any ? (unsigned)(kmax - kmin) : 0u;
    const int off = any ? kbase - kmin : -(1 << 30);
#pragma unroll
    for (int cc = 0; cc < kC; ++cc) x[cc] = ((unsigned)(off + cc) <= span) ? x[cc] : -INFINITY;
  }
  float mx[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
#pragma unroll
  for (int k = 0; k < kC / 2; ++k) mx[k & 7] = max3(mx[k & 7], x[2 * k], x[2 * k + 1]);
  float m_tile = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
  if (kPosScale) m_tile *= c;
  return m_tile;
}

// Lazy update of the reference maximum from a tile's row maximum: it moves only when the row
// maximum exceeds it by more than kRescaleThreshold, and alpha (the factor for O and the sums)
// is then 2^(old - new).
__device__ __forceinline__ void fwd_update_max(float m_tile, float& m_run, float& alpha, bool& updated) {
  const float m_new = fmaxf(m_run, m_tile);
  updated = m_new > m_run + kRescaleThreshold;
  alpha = 1.0f;
  if (updated) {
    alpha = ex2_approx(m_run - m_new);  // 0 when m_run was -inf
    m_run = m_new;
  }
}

// Exponentials of 32 columns (16 pairs starting at pair k0) against the reference maximum,
// packed to bf16 pairs (even column low) and summed twice: `sum` adds the fp32 values (the
// row sum of the log-sum-exp), `rsum` the bf16 values the tensor core multiplies with V (the
// divisor of O, so that O is a weighted mean of V rows under exactly the weights applied: a
// row dominated by one key then returns that key's value row, not the row times the
// relative rounding error of its weight).
template <bool kPosScale, int kC>
__device__ __forceinline__ void fwd_exp_chunk(const float (&x)[kC], int k0, float c, float m_use, uint32_t (&pk)[16],
                                              float2& sum, float2& rsum) {
  const float2 neg_m = make_float2(-m_use, -m_use);
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float2 xv = make_float2(x[2 * (k0 + k)], x[2 * (k0 + k) + 1]);
    const float2 a = kPosScale ? fma2(xv, c2, neg_m) : add2(xv, neg_m);
    float2 pv;
    if ((k % kFwdPolyDen) < kFwdPolyNum) {
      pv = exp2_poly2(a);
    } else {
      pv = make_float2(ex2_approx(a.x), ex2_approx(a.y));
    }
    sum = add2(sum, pv);
    pk[k] = pack_bf16x2(pv.x, pv.y);
    rsum = add_bf16x2_f32x2(pk[k], rsum);
  }
}

// Same for E4M3 P: 32 columns -> 8 words of four E4M3 values (column 4w + i in byte i). The
// row sum takes the exponentials before quantisation.
template <bool kPosScale, int kC>
__device__ __forceinline__ void fwd_exp_chunk_e4m3(const float (&x)[kC], int k0, float c, float m_use,
                                                   uint32_t (&pk)[8], float2& sum) {
  const float2 neg_m = make_float2(-m_use, -m_use);
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int k = 0; k < 16; k += 2) {
    float2 pv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float2 xv = make_float2(x[2 * (k0 + k + u)], x[2 * (k0 + k + u) + 1]);
      const float2 a = kPosScale ? fma2(xv, c2, neg_m) : add2(xv, neg_m);
      if (((k + u) % kFwdPolyDen) < kFwdPolyNum)
        pv[u] = exp2_poly2(a);
      else
        pv[u] = make_float2(ex2_approx(a.x), ex2_approx(a.y));
      sum = add2(sum, pv[u]);
    }
    pk[k >> 1] = pack_e4m3x4(pv[0].x, pv[0].y, pv[1].x, pv[1].y);
  }
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, bool kF8 = false, bool kAlibi = false, bool kVarlen = false>
__global__ void __launch_bounds__(FwdCfg<D, kF8>::kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  using Cfg = FwdCfg<D, kF8>;
  using Bars = FwdBars<Cfg>;
  static_assert(sizeof(Bars) <= 512, "barrier block");
  static_assert(!kF8 || D == 128, "E4M3 inputs: head dim 128 (one 128-byte row per TMA box)");
  static_assert(!(kF8 && kAlibi), "ALiBi is built for bf16 inputs");
  static_assert(!(kF8 && kVarlen), "packed batches are built for bf16 inputs");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_u32(smem_raw));
  // end of this launch's dynamic shared memory (for the FA_DEBUG bounds checks)
  const uint32_t smem_end = smem_u32(smem_raw) + Cfg::kSmemBytes + (kVarlen ? kFwdSortBytes : 0);
  Bars* bars = reinterpret_cast<Bars*>(smem_gen + Cfg::kOffBar);
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };

  const int warp = threadIdx.x >> 5;
  const Abort ab{&bars->abort_flag};

  if (threadIdx.x == 0) {
    bars->abort_flag = 0;
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(bars->q_full[t]), 1);
      mbar_init(bar(bars->q_empty[t]), 1);
      mbar_init(bar(bars->s_full[t]), 1);
      mbar_init(bar(bars->p_full[t]), 128 * Cfg::kHalves);
      mbar_init(bar(bars->s_empty[t]), 128 * Cfg::kHalves);
      mbar_init(bar(bars->pv_done[t]), 1);
    }
    for (int s = 0; s < Cfg::kSlots; ++s) {
      mbar_init(bar(bars->kv_full[s]), 1);
      mbar_init(bar(bars->kv_empty[s]), 1);
    }
    mbar_init(bar(bars->mma_done), 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(bars->item_full[t]), 1);
      mbar_init(bar(bars->item_empty[t]), Cfg::kItemConsumers);
    }
    fence_barrier_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), Cfg::kTmemCols);
    tmem_relinquish();
    tc_fence_before_sync();
  }
  // packed batch: pair order by decreasing cost, computed by the whole CTA
  const uint16_t* order = nullptr;
  if constexpr (kVarlen) {
    if (p.num_pairs <= kFwdSortMaxPairs) {
      uint16_t* sCost = reinterpret_cast<uint16_t*>(smem_gen + Cfg::kOffSort);
      uint16_t* sOrder = sCost + kFwdSortMaxPairs;
      for (int q = threadIdx.x; q < p.num_pairs; q += blockDim.x) {
        int lo0, hi0, lo1, hi1;
        fwd_kv_range<true>(p, q * 256, lo0, hi0);
        fwd_kv_range<true>(p, q * 256 + 128, lo1, hi1);
        sCost[q] = (uint16_t)(max(0, hi0 - lo0 + 1) + max(0, hi1 - lo1 + 1));
      }
      __syncthreads();
      for (int q = threadIdx.x; q < p.num_pairs; q += blockDim.x) {
        const int c = sCost[q];
        int rank = 0;
        for (int u = 0; u < p.num_pairs; ++u) {
          const int cu = sCost[u];
          rank += (cu > c) | ((cu == c) & (u > q));
        }
        sOrder[rank] = (uint16_t)q;
      }
      order = sOrder;
    }
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  const uint32_t sQ[2] = {smem_base + Cfg::kOffQ, smem_base + Cfg::kOffQ + Cfg::kTileBytes};
  const uint32_t sO[2] = {Cfg::kSepO ? smem_base + Cfg::kOffO : sQ[0],
                          Cfg::kSepO ? smem_base + Cfg::kOffO + Cfg::kOTileBytes : sQ[1]};
  const uint32_t sKV = smem_base + Cfg::kOffKV;

  // Registers: the launch gives every thread 168 (384 threads, no row split) or 96 (640); the
  // producer / MMA warpgroup (warps 0-3) needs few and hands some back, and the softmax
  // warpgroups take them: 128 x (96 + 2 x 200) = 63488 <= 384 x 168 = 64512, and
  // 128 x (80 + 4 x 96) = 59392 <= 640 x 96 = 61440 registers of the launch.
  if (warp < 4) {  // ---- producer / MMA warpgroup (warps 0-3)
  if constexpr (Cfg::kSplitRow)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;" ::: "memory");
  else
    asm volatile("setmaxnreg.dec.sync.aligned.u32 96;" ::: "memory");
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane_id() == 0) {
      uint32_t slot = 0, phase = 0;
      uint32_t qn[2] = {0, 0};
      int last_slot_parity[Cfg::kSlots];
      for (int s = 0; s < Cfg::kSlots; ++s) last_slot_parity[s] = -1;
      griddep_wait();  // this call's counter slot has been zeroed
      int* counter = &g_fwd_next_item[p.counter_slot];
      if (!dbg_range(ab, p.counter_slot, 1, kFwdCounterSlots)) counter = nullptr;
      for (uint32_t n = 0;; ++n) {
        const uint32_t islot = n & 1;
        mbar_wait_ring(bar(bars->item_empty[islot]), ((n >> 1) & 1) ^ 1, ab);  // slot read by every consumer
        const int w = (ab.raised() || !counter) ? p.num_items : atomicAdd(counter, 1);
        bars->item_w[islot] = w;
        mbar_arrive(bar(bars->item_full[islot]));
        if (w >= p.num_items) break;
        int b, h, pair;
        fwd_decode(p, w, b, h, pair, order);
        int lo_t[2], hi_t[2];
        fwd_kv_range<kVarlen>(p, pair * 256, lo_t[0], hi_t[0]);
        fwd_kv_range<kVarlen>(p, pair * 256 + 128, lo_t[1], hi_t[1]);
        const bool act1 = hi_t[1] >= lo_t[1];
        const int lo = act1 ? min(lo_t[0], lo_t[1]) : lo_t[0];
        const int hi = act1 ? max(hi_t[0], hi_t[1]) : hi_t[0];
        // FA_DEBUG: a tile whose boxes fail the bounds check is neither armed nor loaded
        auto tile_ok = [&](uint32_t dst, int row) {
          bool ok = true;
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            ok = ok && dbg_tma(ab, bx * Cfg::kBoxElems, row, h, b, D, p.N, p.H, p.B, Cfg::kElem, dst + bx * 16384,
                               16384, smem_base, smem_end);
          return ok;
        };
        for (int t = 0; t < 2; ++t) {
          if (hi_t[t] < lo_t[t]) continue;
          mbar_wait(bar(bars->q_empty[t]), (qn[t] & 1) ^ 1, ab);
          if (!tile_ok(sQ[t], pair * 256 + t * 128)) break;
          mbar_arrive_expect_tx(bar(bars->q_full[t]), Cfg::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_4d(sQ[t] + bx * 16384, &tmQ, bar(bars->q_full[t]), bx * Cfg::kBoxElems, pair * 256 + t * 128, h,
                        b);
          ++qn[t];
        }
        for (int j = lo; j <= hi && !(FA_DEBUG && ab.raised()); ++j) {
          for (int kv = 0; kv < 2; ++kv) {
            mbar_wait(bar(bars->kv_empty[slot]), phase ^ 1, ab);
            const uint32_t dst = sKV + slot * Cfg::kTileBytes;
            if (!tile_ok(dst, j * 128)) break;
            mbar_arrive_expect_tx(bar(bars->kv_full[slot]), Cfg::kTileBytes);
#pragma unroll
            for (int bx = 0; bx < Cfg::kBoxes; ++bx)
              tma_load_4d(dst + bx * 16384, kv ? &tmV : &tmK, bar(bars->kv_full[slot]), bx * Cfg::kBoxElems, j * 128,
                          h, b);
            last_slot_parity[slot] = phase;
            if (++slot == Cfg::kSlots) { slot = 0; phase ^= 1; }
          }
        }
        if (FA_DEBUG && ab.raised()) break;
      }
      // Drain: every load issued must have landed before the CTA can exit.
      for (int s = 0; s < Cfg::kSlots; ++s)
        if (last_slot_parity[s] >= 0) mbar_drain(bar(bars->kv_full[s]), last_slot_parity[s]);
      for (int t = 0; t < 2; ++t)
        if (qn[t] > 0) mbar_drain(bar(bars->q_full[t]), (qn[t] - 1) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      // S = Q K^T (both K-major), O += P V (V MN-major)
      constexpr uint32_t idS = kF8 ? idesc_e4m3_f32(128, 128, false, false) : idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idO = kF8 ? idesc_e4m3_f32(128, D, false, true) : idesc_bf16_f32(128, D, false, true);
      const uint32_t tS[2] = {tmem + Cfg::kColS0, tmem + Cfg::kColS1};
      const uint32_t tO[2] = {tmem + Cfg::kColO0, tmem + Cfg::kColO1};
      const uint32_t tP[2] = {tmem + Cfg::kColP0, tmem + Cfg::kColP1};
      uint32_t qn[2] = {0, 0}, pn[2] = {0, 0};
      uint32_t kvn = 0, sq[2] = {0, 0};  // K/V stream position, S issued (per tile, or shared)
      bool drop_s_signal = p.debug_drop_s_signal != 0;

      auto issue_s = [&](int t, uint32_t k_smem) {
#pragma unroll
        for (int kk = 0; kk < Cfg::kKSteps; ++kk) {  // 32 bytes of d per step, 4 steps per 128-byte box
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          if constexpr (kF8)
            mma_ss_f8(tS[t], sdesc_kmajor(sQ[t] + off), sdesc_kmajor(k_smem + off), idS, kk > 0);
          else
            mma_ss(tS[t], sdesc_kmajor(sQ[t] + off), sdesc_kmajor(k_smem + off), idS, kk > 0);
        }
      };
      auto issue_pv = [&](int t, uint32_t v_smem, bool accumulate) {
        // 16 (bf16) or 32 (E4M3) keys per step: 8 TMEM columns of P, as many 128-byte rows of V
#pragma unroll
        for (int kk = 0; kk < Cfg::kPvSteps; ++kk) {
          const uint64_t vd = sdesc_mnmajor(v_smem + kk * (kF8 ? 4096 : 2048), 16384);
          if constexpr (kF8)
            mma_ts_f8(tO[t], tP[t] + kk * 8, vd, idO, accumulate || kk > 0);
          else
            mma_ts(tO[t], tP[t] + kk * 8, vd, idO, accumulate || kk > 0);
        }
      };

      for (uint32_t it = 0;; ++it) {
        const int w = fwd_take_item(bars, it, true, ab);
        if (w >= p.num_items) break;
        int b, h, pair;
        fwd_decode(p, w, b, h, pair, order);
        int lo_t[2], hi_t[2];
        fwd_kv_range<kVarlen>(p, pair * 256, lo_t[0], hi_t[0]);
        fwd_kv_range<kVarlen>(p, pair * 256 + 128, lo_t[1], hi_t[1]);
        const bool act[2] = {true, hi_t[1] >= lo_t[1]};
        const int lo = act[1] ? min(lo_t[0], lo_t[1]) : lo_t[0];
        const int hi = act[1] ? max(hi_t[0], hi_t[1]) : hi_t[0];
        auto active = [&](int t, int j) { return act[t] && j >= lo_t[t] && j <= hi_t[t]; };
        bool first_pv[2] = {true, true};
        for (int t = 0; t < 2; ++t)
          if (act[t]) mbar_wait(bar(bars->q_full[t]), qn[t] & 1, ab);
        tc_fence_after_sync();

        if constexpr (Cfg::kShareS) {
          // K(j) is tile n0 + 2(j - lo) of the K/V stream and V(j) the next one; stream tile n
          // sits in slot n % kSlots, filled for the (n / kSlots)-th time.
          const uint32_t n0 = kvn;
          auto kv_wait = [&](uint32_t n) {
            const uint32_t s = n % Cfg::kSlots;
            mbar_wait(bar(bars->kv_full[s]), (n / Cfg::kSlots) & 1, ab);
            tc_fence_after_sync();
            return s;
          };
          auto s_shared = [&](int t, int j, uint32_t ks) {  // S_t(j) into the shared buffer once the last S is read
            mbar_wait(bar(bars->s_empty[0]), (sq[0] & 1) ^ 1, ab);
            ++sq[0];
            tc_fence_after_sync();
            issue_s(t, sKV + ks * Cfg::kTileBytes);
            if (drop_s_signal) drop_s_signal = false;
            else mma_commit(bar(bars->s_full[t]));
            if (Cfg::kSepO && j == hi_t[t]) mma_commit(bar(bars->q_empty[t]));  // last read of Q_t (O staged apart)
          };
          auto pv = [&](int t, uint32_t vs) {
            mbar_wait(bar(bars->p_full[t]), pn[t] & 1, ab);
            ++pn[t];
            tc_fence_after_sync();
            issue_pv(t, sKV + vs * Cfg::kTileBytes, !first_pv[t]);
            first_pv[t] = false;
            mma_commit(bar(bars->pv_done[t]));
          };
          {
            const uint32_t ks = kv_wait(n0);  // S0(lo), S1(lo)
            for (int t = 0; t < 2; ++t)
              if (active(t, lo)) s_shared(t, lo, ks);
            mma_commit(bar(bars->kv_empty[ks]));
          }
          for (int j = lo; j <= hi; ++j) {
            const bool more = j < hi;
            const uint32_t vs = kv_wait(n0 + 2 * (j - lo) + 1);
            const uint32_t ks = more ? kv_wait(n0 + 2 * (j + 1 - lo)) : 0;
            if (more && active(0, j + 1)) s_shared(0, j + 1, ks);
            if (active(0, j)) pv(0, vs);
            if (more && active(1, j + 1)) s_shared(1, j + 1, ks);
            if (more) mma_commit(bar(bars->kv_empty[ks]));
            if (active(1, j)) pv(1, vs);
            mma_commit(bar(bars->kv_empty[vs]));
          }
          kvn = n0 + 2 * (hi - lo + 1);
          for (int t = 0; t < 2; ++t)
            if (act[t]) ++qn[t];
        } else {
          // K(j) is tile n0 + 2(j - lo) of the K/V stream and V(j) the next one; stream tile n
          // sits in slot n % kSlots, filled for the (n / kSlots)-th time.
          const uint32_t n0 = kvn;
          auto kv_wait = [&](uint32_t n) {
            const uint32_t s = n % Cfg::kSlots;
            mbar_wait(bar(bars->kv_full[s]), (n / Cfg::kSlots) & 1, ab);
            tc_fence_after_sync();
            return s;
          };
          auto s_step = [&](int j) {  // S0(j), S1(j), each once the previous S_t has been read
            const uint32_t ks = kv_wait(n0 + 2 * (j - lo));
            for (int t = 0; t < 2; ++t) {
              if (!active(t, j)) continue;
              mbar_wait(bar(bars->s_empty[t]), (sq[t] & 1) ^ 1, ab);
              ++sq[t];
              tc_fence_after_sync();
              issue_s(t, sKV + ks * Cfg::kTileBytes);
              if (drop_s_signal) drop_s_signal = false;
              else mma_commit(bar(bars->s_full[t]));
              if (j == hi_t[t]) mma_commit(bar(bars->q_empty[t]));  // last read of Q_t in this item
            }
            mma_commit(bar(bars->kv_empty[ks]));
          };
          s_step(lo);
          for (int j = lo; j <= hi; ++j) {
            if (j < hi) s_step(j + 1);
            const uint32_t vs = kv_wait(n0 + 2 * (j - lo) + 1);
            for (int t = 0; t < 2; ++t) {
              if (!active(t, j)) continue;
              mbar_wait(bar(bars->p_full[t]), pn[t] & 1, ab);
              ++pn[t];
              tc_fence_after_sync();
              issue_pv(t, sKV + vs * Cfg::kTileBytes, !first_pv[t]);
              first_pv[t] = false;
              mma_commit(bar(bars->pv_done[t]));
            }
            mma_commit(bar(bars->kv_empty[vs]));
          }
          kvn = n0 + 2 * (hi - lo + 1);
          for (int t = 0; t < 2; ++t)
            if (act[t]) ++qn[t];
        }

      }
      mma_commit(bar(bars->mma_done));
      mbar_drain(bar(bars->mma_done), 0);
    }
  }
  } else {  // ---- softmax warpgroups (warps 4-11, or 4-19 with the row split)
  if constexpr (Cfg::kSplitRow)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 96;" ::: "memory");
  else
    asm volatile("setmaxnreg.inc.sync.aligned.u32 200;" ::: "memory");
  {
    // ---------------------------------------------------------------- softmax + epilogue
    constexpr int kC = Cfg::kCols;            // scores of a row per thread and KV tile
    const int t = ((warp - 4) >> 2) & 1;      // Q tile of the pair handled by this warpgroup
    const int half = (warp - 4) >> 3;         // row split: columns [kC half, kC half + kC)
    const int row = (threadIdx.x - 128) & 127;  // 0..127: TMEM lane and row within the tile
    const uint32_t lane_field = (uint32_t)((row & ~31) << 16);
    const uint32_t tS = tmem + lane_field + (t ? Cfg::kColS1 : Cfg::kColS0) + kC * half;
    const uint32_t tO = tmem + lane_field + (t ? Cfg::kColO1 : Cfg::kColO0);
    const uint32_t tP = tmem + lane_field + (t ? Cfg::kColP1 : Cfg::kColP0) + (kC / (kF8 ? 4 : 2)) * half;
    uint32_t sn = 0, pvn = 0;
    // Row split: the two warps holding the same 32 rows of tile t (same TMEM lanes, so the same
    // sub-partition) meet at named barrier 4 + 4 t + row / 32 and exchange their partial maxima
    // (two parity slots, so a fast partner never overwrites a value not yet read) and, at the
    // end of an item, their sums.
    float* xm = reinterpret_cast<float*>(smem_gen + Cfg::kOffX) + t * 512;         // [parity][half][row]
    float* xl = reinterpret_cast<float*>(smem_gen + Cfg::kOffX) + 1024 + t * 512;  // [sum][half][row]
    uint32_t xu = 0;
    auto pair_sync = [&]() { named_bar_sync(4 + 4 * t + (row >> 5), 64); };

    for (uint32_t it = 0;; ++it) {
      const int w = fwd_take_item(bars, it, lane_id() == 0, ab);
      if (w >= p.num_items) break;
      int b, h, pair;
      fwd_decode(p, w, b, h, pair, order);
      const int r0 = pair * 256 + t * 128;
      int lo, hi;
      fwd_kv_range<kVarlen>(p, r0, lo, hi);
      if (hi < lo) continue;
      float c = p.scale_log2, o_mul = 1.0f;  // log2-domain score factor; O factor
      float nslope2 = 0.0f;                  // ALiBi: -m log2(e)
      if (!dbg_range(ab, (long long)b * p.H + h, 1, (long long)p.B * p.H)) break;
      if constexpr (kAlibi) nslope2 = -p.alibi_slopes[b * p.H + h] * kLog2e;
      if constexpr (kF8) {
        const int bh = b * p.H + h;
        c *= p.q_descale[bh] * p.k_descale[bh];
        o_mul = p.v_descale[bh];
      }
      const int i = r0 + row;
      int kmin, kmax;
      if constexpr (kVarlen) {
        fwd_row_keys<true>(p, i, kmin, kmax);
      } else {
        kmin = p.win_l >= 0 ? i - p.win_l : 0;
        kmax = p.win_r >= 0 ? min(p.N - 1, i + p.win_r) : p.N - 1;
      }
      int seg_first = 0, seg_last = 0;  // sequence of the tile's first row (packed batches)
      if (kVarlen) seg_bounds(p.cu_seqlens, p.nseg, p.N, r0, seg_first, seg_last);
      float m_run = -INFINITY, l_run = 0.0f;
      float lr_run = 0.0f;  // sum of the bf16-rounded weights (bf16 P): the divisor of O

      for (int j = lo; j <= hi; ++j) {
        mbar_wait(bar(bars->s_full[t]), sn & 1, ab);
        ++sn;
        tc_fence_after_sync();
        uint32_t r[kC / 32][32];
#pragma unroll
        for (int q4 = 0; q4 < kC / 32; ++q4) tmem_ld32(tS + q4 * 32, r[q4]);
#pragma unroll
        for (int q4 = 0; q4 < kC / 32; ++q4) tmem_wait_ld(r[q4]);
        tc_fence_before_sync();  // the S buffer may now take the next scores
        mbar_arrive(bar(bars->s_empty[Cfg::kShareS ? 0 : t]));
        float x[kC];
#pragma unroll
        for (int cc = 0; cc < kC; ++cc) x[cc] = __uint_as_float(r[cc >> 5][cc & 31]);

        const bool masked = !fwd_tile_unmasked<kVarlen>(p, r0, j, seg_first, seg_last);
        const int kbase = j * 128 + kC * half;  // key of x[0]
        const bool pos_scale = !kAlibi && c > 0.0f;  // with ALiBi the scores are scaled before the max
        float m_tile;
        if constexpr (kAlibi)
          m_tile = fwd_tile_max<false, true>(x, masked, kbase, kmin, kmax, c, (float)(i - kbase), nslope2);
        else if (pos_scale)
          m_tile = fwd_tile_max<true>(x, masked, kbase, kmin, kmax, c);
        else
          m_tile = fwd_tile_max<false>(x, masked, kbase, kmin, kmax, c);
        if constexpr (Cfg::kSplitRow) {
          float* slot = xm + (xu & 1) * 256;
          slot[half * 128 + row] = m_tile;
          pair_sync();
          m_tile = fmaxf(m_tile, slot[(half ^ 1) * 128 + row]);
          ++xu;
        }
        float alpha;
        bool updated;
        fwd_update_max(m_tile, m_run, alpha, updated);
        const float m_use = (m_run == -INFINITY) ? 0.0f : m_run;
        if (j > lo) {  // PV_t(j-1) has read P_t and O_t is quiescent
          mbar_wait(bar(bars->pv_done[t]), pvn & 1, ab);
          ++pvn;
          tc_fence_after_sync();
        }
        // P in 32-column chunks straight into TMEM (E4M3: over S columns already read into registers)
        float2 sum0 = make_float2(0.0f, 0.0f), sum1 = make_float2(0.0f, 0.0f);
        float2 rs0 = make_float2(0.0f, 0.0f), rs1 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int q4 = 0; q4 < kC / 32; ++q4) {
          if constexpr (kF8) {
            uint32_t pk[8];
            if (pos_scale)
              fwd_exp_chunk_e4m3<true>(x, q4 * 16, c, m_use, pk, (q4 & 1) ? sum1 : sum0);
            else
              fwd_exp_chunk_e4m3<false>(x, q4 * 16, c, m_use, pk, (q4 & 1) ? sum1 : sum0);
            tmem_st8(tP + q4 * 8, pk);
          } else {
            uint32_t pk[16];
            if (pos_scale)
              fwd_exp_chunk<true>(x, q4 * 16, c, m_use, pk, (q4 & 1) ? sum1 : sum0, (q4 & 1) ? rs1 : rs0);
            else
              fwd_exp_chunk<false>(x, q4 * 16, c, m_use, pk, (q4 & 1) ? sum1 : sum0, (q4 & 1) ? rs1 : rs0);
            tmem_st16(tP + q4 * 16, pk);
          }
        }
        const float2 s01 = add2(sum0, sum1);
        l_run = l_run * alpha + (s01.x + s01.y);
        if constexpr (!kF8) {
          const float2 r01 = add2(rs0, rs1);
          lr_run = lr_run * alpha + (r01.x + r01.y);
        }

        // Rescale O_t in TMEM when this warp's reference maximum moved (not on the first tile:
        // the first PV of an item overwrites O_t).
        if (__any_sync(0xffffffffu, updated && j > lo)) {
#pragma unroll 1
          for (int cc = (D / Cfg::kHalves) * half; cc < (D / Cfg::kHalves) * (half + 1); cc += 32) {
            uint32_t o[32];
            tmem_ld32(tO + cc, o);
            tmem_wait_ld(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + cc, o);
          }
        }
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(bar(bars->p_full[t]));
      }

      // Epilogue: O_t / l -> bf16 -> staging (the Q_t buffer, free once the last PV_t is done) -> TMA store.
      mbar_wait(bar(bars->pv_done[t]), pvn & 1, ab);  // the item's last PV_t
      ++pvn;
      tc_fence_after_sync();
      if constexpr (Cfg::kSepO) {
        if (row == 0 && half == 0) bulk_wait_group_read0();  // the previous store has read the staging tile
        named_bar_sync(1 + t, 128 * Cfg::kHalves);
      }
      // bf16 P: O is divided by the sum of the weights it was accumulated with; E4M3 P keeps the
      // fp32 sum (its tolerance is derived for that divisor). Row split: each half summed its
      // own columns against the same reference maximum, so the row's sums add.
      float l_tot = l_run, l_o = kF8 ? l_run : lr_run;
      if constexpr (Cfg::kSplitRow) {
        xl[half * 128 + row] = l_run;
        xl[256 + half * 128 + row] = lr_run;
        pair_sync();
        l_tot = l_run + xl[(half ^ 1) * 128 + row];
        l_o = kF8 ? l_tot : lr_run + xl[256 + (half ^ 1) * 128 + row];
      }
      const float inv_l = l_o > 0.0f ? o_mul / l_o : 0.0f;
      const uint32_t stage = sO[t];
#pragma unroll 1
      for (int cc = (D / Cfg::kHalves) * half; cc < (D / Cfg::kHalves) * (half + 1); cc += 32) {
        uint32_t o[32];
        tmem_ld32(tO + cc, o);
        tmem_wait_ld(o);
        const uint32_t box = stage + (cc >> 6) * 16384;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w4[e] = pack_bf16x2(__uint_as_float(o[ch * 8 + 2 * e]) * inv_l, __uint_as_float(o[ch * 8 + 2 * e + 1]) * inv_l);
          st_shared_v4(box + sw128_offset(row, ((cc & 63) >> 3) + ch), w4[0], w4[1], w4[2], w4[3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + t, 128 * Cfg::kHalves);
      if (row == 0 && half == 0) {
#pragma unroll
        for (int bx = 0; bx < Cfg::kOBoxes; ++bx)
          if (dbg_tma(ab, bx * 64, r0, h, b, D, p.N, p.H, p.B, 2, stage + bx * 16384, 16384, smem_base, smem_end))
            tma_store_4d(&tmO, stage + bx * 16384, bx * 64, r0, h, b);
        bulk_commit_group();
        if constexpr (!Cfg::kSepO) {  // the Q_t buffer is free again once the store has read it
          bulk_wait_group_read0();
          mbar_arrive(bar(bars->q_empty[t]));
        }
      }
      if (i < p.N && half == 0) {
        const float lse = l_tot > 0.0f ? (m_run + lg2_approx(l_tot)) * kLn2 : -INFINITY;
        const long long li = ((long long)b * p.H + h) * (long long)p.N + i;
        if (dbg_range(ab, li, 1, (long long)p.B * p.H * p.N)) p.lse[li] = lse;
      }
    }
    if (row == 0 && half == 0) bulk_wait_group0();
  }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace fa
