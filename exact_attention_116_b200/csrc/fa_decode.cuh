// Attention of a few new query rows against a paged KV cache (decoding), for sm_100a.
//
// What it computes ("FlashAttention技术解析：加速GPT训练的核心优化" §5, FlashDecoding;
// "突破大模型训练瓶颈：Flash-Attention编译优化与内存占用解决方案", Paged KV Cache): for every
// sequence b, head h and new query row i (0 <= i < Sq, at position pos = seqlen_b - Sq + i),
// O = softmax(scale * q . k_j) V over the cached keys j < seqlen_b that the mask leaves visible,
// and LSE = ln sum_j exp(scale * q . k_j). Key j of sequence b is row j % page_size of page
// block_table[b][j / page_size] of the (num_pages, page_size, H, d) cache.
//
// The work is one pass over the cache: HBM-bound (each K/V element is used by Sq <= 8 rows).
// Both products still run on the tensor core (see the kernel below): on the CUDA cores the dot
// products and P V of even one to four rows kept the kernel from the cache read.
//
// Work split (split-KV, balanced over the whole batch): for each head, the 64-key units that
// the new rows can see are listed sequence after sequence, and that list is cut into P equal
// contiguous pieces, one CTA each (grid (H, P), P chosen so that the grid fills the GPU once).
// Every CTA therefore streams the same number of units (within one), whatever the mix of
// lengths, and no CTA waits in a second wave. A piece may cover the end of one sequence, some
// whole sequences and the start of another: the CTA keeps one running state per sequence
// part ("segment") and its TMA ring runs on across segment boundaries. A sequence that lies
// in one piece is finished by that CTA; otherwise each of its pieces writes a partial
// (O / l, log2 l + m) to slot b + piece (unique: a piece after another one on the list never
// holds an earlier sequence), counts itself on the (b, h) arrival counter, and the piece that
// arrives last merges the partials by their log-sum-exp, in piece order. The counters are
// zeroed by fa_decode_prep_kernel, launched just before on the same stream; the decode kernel
// is launched as its programmatic dependent and waits for it only before its first arrival.
//
// CTAs of the same piece for consecutive heads are launched next to each other (head is the
// fastest grid index) and walk the same units, so the 128-byte head slices of one cache row
// (H x d bf16, contiguous) are read at about the same time.
//
// With new K/V rows given (flash_attn_with_kvcache's in-place update of the cache), the CTA
// whose piece holds a new row's unit writes that row's d columns of its head into the cache
// before it loads any tile: every new row is visible to the newest query row, so exactly one
// piece of each head holds it, and no other CTA reads those bytes.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kDecMaxSq = 8;         // new query rows per call
constexpr int kDecTile = 64;         // keys per unit of the work split (one TMA box; a kernel tile is two)
constexpr int kDecThreads = 128;     // the four softmax warps, which also run the set-up and the merge
constexpr int kDecMmaThreads = 224;  // the decode kernel's CTA: softmax warps, a producer, two MMA issuers
constexpr float kDecLn2 = 0.69314718055994530942f;

// Warp-collective TMEM load of 8 consecutive 32-bit columns: thread t of the warp reads lane
// (lane field of taddr) + t; and the wait for it (the registers pass through so that no use is
// hoisted above the wait).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])::"memory");
}

// Maximum of x over the 32 lanes of the warp (all lanes active), one instruction on sm_100a.
__device__ __forceinline__ float warp_max_f32(float x) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
  return r;
}

// Generic-proxy writes to global memory by this thread are ordered before later async-proxy
// (TMA) accesses that a barrier orders after this fence.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

struct DecParams {
  int B, Sq, H, page_size, max_pages, num_pages;
  float scale_log2;  // scale * log2(e)
  int win_l, win_r;  // -1 = unbounded; causal already folded into win_r = 0
  int pieces;        // P: CTAs per head
  const int* block_table;  // (B, max_pages)
  const int* seqlens;      // (B)
  const __nv_bfloat16* q;  // (B, Sq, H, d)
  __nv_bfloat16* o;        // (B, Sq, H, d)
  float* lse;              // (B, H, Sq), natural log
  float* o_part;           // (B + P - 1, H, Sq, d) fp32 (P > 1)
  float* lse_part;         // (B + P - 1, H, Sq), log2 domain (P > 1)
  int* arrivals;           // (B, H) pieces finished (P > 1), zeroed by the prep kernel
  const __nv_bfloat16* k_new;  // (B, Sq, H, d) rows to write into the cache, or null
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_cache;  // (num_pages, page_size, H, d)
  __nv_bfloat16* v_cache;
};

// Length of sequence b; an out-of-range length counts as 0 (reported when `report`).
__device__ __forceinline__ int dec_len(const DecParams& p, int b, bool report) {
  const int n = p.seqlens[b];
  if (n < 0 || n > p.max_pages * p.page_size) {
    if (report) atomicOr(&g_fa_error, kErrBadInput);
    return 0;
  }
  return n;
}

// Number of 64-key units, from unit vt0 on, that the rows of a sequence of n keys can see
// (0 for an empty sequence; at least 1 otherwise: each row sees its own key).
__device__ __forceinline__ int dec_vis_units(const DecParams& p, int n, int& vt0) {
  vt0 = 0;
  if (n <= 0) return 0;
  const int pos0 = n - p.Sq, pos1 = n - 1;
  const int vis_lo = p.win_l >= 0 ? max(0, pos0 - p.win_l) : 0;
  const int vis_hi = p.win_r >= 0 ? min(n - 1, pos1 + p.win_r) : n - 1;
  vt0 = vis_lo / kDecTile;
  return vis_hi / kDecTile + 1 - vt0;
}

// The next sequence after b with a visible unit (p.B when there is none), its length, first
// visible unit and unit count.
__device__ __forceinline__ int dec_next_seq(const DecParams& p, int b, int& n, int& vt0, int& cnt) {
  for (++b; b < p.B; ++b) {
    n = dec_len(p, b, false);
    cnt = dec_vis_units(p, n, vt0);
    if (cnt > 0) return b;
  }
  return p.B;
}

// Pieces: piece r of P <= T covers units [T r / P, T (r + 1) / P) of a head's T units (at least
// one); the piece that holds unit u (0 <= u < T) is the largest r with T r / P <= u.
__device__ __forceinline__ long long dec_piece_lo(long long T, int P, int r) { return T * r / P; }
__device__ __forceinline__ int dec_piece_of(long long T, int P, long long u) {
  return (int)(((u + 1) * P - 1) / T);
}

// A walk over the 64-key units of one piece, segment by segment: sequence b (n keys), whose
// visible units start at position `start` of the list, contributes its units [t0, t1).
struct DecWalk {
  int b, n, vt0, cnt, t0, t1;
  long long start;
  __device__ __forceinline__ void clip(long long u0, long long u1) {
    t0 = vt0 + (int)max(0LL, u0 - start);
    t1 = vt0 + (int)min((long long)cnt, u1 - start);
  }
  // first segment: sequence b0 starting at unit s0 (b0 == p.B: the piece is empty)
  __device__ __forceinline__ void begin(const DecParams& p, int b0, long long s0, long long u0, long long u1) {
    b = b0;
    start = s0;
    n = vt0 = cnt = t0 = t1 = 0;
    if (b < p.B) {
      n = dec_len(p, b, false);
      cnt = dec_vis_units(p, n, vt0);
      clip(u0, u1);
    }
  }
  // move to the next segment; false when the piece has no more
  __device__ __forceinline__ bool next_seg(const DecParams& p, long long u0, long long u1) {
    start += cnt;
    b = dec_next_seq(p, b, n, vt0, cnt);
    if (b >= p.B || start >= u1) {
      b = p.B;
      return false;
    }
    clip(u0, u1);
    return true;
  }
  __device__ __forceinline__ bool valid(const DecParams& p) const { return b < p.B; }
};

// A CTA's piece of a head's unit list: the list's length T, the pieces in use Pe, this piece's
// units [u0, u1) and its first segment (sequence b_first, whose units start at position
// start_first).
struct DecPiece {
  long long T, u0, u1, start_first;
  int Pe, b_first;
};

// Set-up of the decode kernel (all threads of the CTA; threads 0 .. kDecThreads - 1 do the work,
// the others only meet the barriers): the piece from the lengths (a
// block-wide prefix sum of unit counts, each thread summing a contiguous run of sequences); O = 0,
// LSE = -inf for the sequences without a visible unit (written by piece b % P); with new K/V rows
// given, this piece's new rows of head h written into the cache before any tile load. sSum holds
// 5 and sInt 1 values of scratch in shared memory.
template <int D>
__device__ __forceinline__ DecPiece dec_prologue(const DecParams& p, int h, int piece, Abort ab, long long* sSum,
                                                 int* sInt) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Sq = p.Sq, P = p.pieces;
  const long long o_size = (long long)p.B * p.Sq * p.H * D, lse_size = (long long)p.B * p.H * p.Sq;
  const long long cache_size = (long long)p.num_pages * p.page_size * p.H * D;
  // ---- unit counts of all sequences, prefix sums (each thread a contiguous run of sequences)
  const int run = (p.B + kDecThreads - 1) / kDecThreads;
  const int rb0 = min(p.B, tid * run), rb1 = min(p.B, rb0 + run);
  const bool report = h == 0 && piece == 0;
  long long mine = 0;
  for (int b = rb0; b < rb1; ++b) {
    int vt0;
    mine += dec_vis_units(p, dec_len(p, b, report), vt0);
  }
  long long incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31 && warp < 4) sSum[warp] = incl;  // (threads past the first 128 hold no sequences)
  __syncthreads();
  long long T = 0, excl = incl - mine;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const long long sw = sSum[w];
    T += sw;
    if (w < warp) excl += sw;
  }
  // With fewer units than CTAs only the first T pieces get one each (every piece in use then
  // holds at least one unit, which the arrival count and the merge rely on).
  const int Pe = (int)min((long long)P, T);
  const long long u0 = piece < Pe ? dec_piece_lo(T, Pe, piece) : T;
  const long long u1 = piece < Pe ? dec_piece_lo(T, Pe, piece + 1) : T;
  if (u0 < u1 && excl <= u0 && u0 < excl + mine) {  // this thread's run holds the piece's first unit
    long long s = excl;
    for (int b = rb0; b < rb1; ++b) {
      int vt0;
      const int c = dec_vis_units(p, dec_len(p, b, false), vt0);
      if (u0 < s + c) {
        sInt[0] = b;
        sSum[4] = s;
        break;
      }
      s += c;
    }
  }
  __syncthreads();
  const int b_first = sInt[0];
  const long long start_first = b_first < p.B ? sSum[4] : 0;

  // ---- sequences without a visible unit (empty): O = 0, LSE = -inf, written by piece b % P
  for (int b = piece; b < p.B && tid < kDecThreads; b += P) {
    int vt0;
    if (dec_vis_units(p, dec_len(p, b, false), vt0) != 0) continue;
    for (int e = tid; e < Sq * D; e += kDecThreads) {
      const int i = e / D, col = e - i * D;
      const long long oi = (((long long)b * Sq + i) * p.H + h) * D + col;
      if (dbg_range(ab, oi, 1, o_size)) p.o[oi] = __float2bfloat16_rn(0.0f);
    }
    const long long li = ((long long)b * p.H + h) * Sq + tid;
    if (tid < Sq && dbg_range(ab, li, 1, lse_size)) p.lse[li] = -INFINITY;
  }

  // ---- new rows in this piece's units: head h's columns go into the cache before any tile load
  if (p.k_new != nullptr) {
    constexpr int kChunks = D / 8;  // 16-byte chunks of one head's row
    bool wrote = false;
    DecWalk w;
    w.begin(p, b_first, start_first, u0, u1);
    for (bool more = w.valid(p); more; more = w.next_seg(p, u0, u1)) {
      for (int i = 0; i < Sq; ++i) {
        const int pos = w.n - Sq + i;
        if (pos < 0 || pos / kDecTile < w.t0 || pos / kDecTile >= w.t1) continue;  // another piece's, or nobody's
        const int page = p.block_table[(size_t)w.b * p.max_pages + pos / p.page_size];
        if (page < 0 || page >= p.num_pages) continue;  // reported when the tile is loaded
        const size_t src = (((size_t)w.b * Sq + i) * p.H + h) * D;
        const size_t dst = (((size_t)page * p.page_size + pos % p.page_size) * p.H + h) * D;
        if (!dbg_range(ab, (long long)src, D, o_size) || !dbg_range(ab, (long long)dst, D, cache_size)) continue;
        if (tid < kChunks) {
          reinterpret_cast<uint4*>(p.k_cache + dst)[tid] = reinterpret_cast<const uint4*>(p.k_new + src)[tid];
        } else if (tid < 2 * kChunks) {
          reinterpret_cast<uint4*>(p.v_cache + dst)[tid - kChunks] =
              reinterpret_cast<const uint4*>(p.v_new + src)[tid - kChunks];
        }
        wrote = true;
      }
    }
    if (wrote) fence_proxy_async_global();  // ordered before the TMA loads by the barrier below
  }
  __syncthreads();

  DecPiece pc;
  pc.T = T;
  pc.Pe = Pe;
  pc.u0 = u0;
  pc.u1 = u1;
  pc.b_first = b_first;
  pc.start_first = start_first;
  return pc;
}

// Segment end of a sequence spread over pieces pf..pl (threads 0 .. kDecThreads - 1, which meet on
// named barrier 1, after this piece's partial is written): count this piece on the (b, h) arrival
// counter; the piece that arrives last merges the partials by their log-sum-exp, in piece order.
// sInt holds one flag.
template <int D>
__device__ __forceinline__ void dec_arrive_merge(const DecParams& p, int b, int h, int pf, int pl, Abort ab,
                                                 int* sInt) {
  const int tid = threadIdx.x, Sq = p.Sq;
  const long long o_size = (long long)p.B * p.Sq * p.H * D, lse_size = (long long)p.B * p.H * p.Sq;
  const long long part_rows = ((long long)p.B + p.pieces - 1) * p.H * p.Sq;
  {
    // arrival: the last piece of (b, h) merges all partials
    __threadfence();  // this thread's partials are visible device-wide before the arrival
    named_bar_sync(1, kDecThreads);
    if (tid == 0) {
      griddep_wait();  // the prep kernel has zeroed the counters
      const long long ai = (long long)b * p.H + h;
      const int before = dbg_range(ab, ai, 1, (long long)p.B * p.H) ? atomicAdd(&p.arrivals[ai], 1) : -1;
      sInt[1] = before == pl - pf;
    }
    named_bar_sync(1, kDecThreads);
    if (sInt[1]) {
      __threadfence();
      // O = sum_r 2^(L_r - L) O_r, L = log2 sum_r 2^L_r, in piece order (the same sum whichever
      // piece arrives last)
      for (int e = tid; e < Sq * D; e += kDecThreads) {
        const int i = e / D, col = e - i * D;
        float mx = -INFINITY;
        if (!dbg_range(ab, (((long long)b + pf) * p.H + h) * Sq + i, 1, part_rows) ||
            !dbg_range(ab, (((long long)b + pl) * p.H + h) * Sq + i, 1, part_rows))
          continue;
        for (int r = pf; r <= pl; ++r)
          mx = fmaxf(mx, __ldcg(p.lse_part + (((size_t)b + r) * p.H + h) * Sq + i));
        float wsum = 0.0f, v = 0.0f;
        if (mx != -INFINITY) {
          for (int r = pf; r <= pl; ++r) {
            const size_t row = (((size_t)b + r) * p.H + h) * Sq + i;
            const float wr = ex2_approx(__ldcg(p.lse_part + row) - mx);
            wsum += wr;
            v = fmaf(wr, __ldcg(p.o_part + row * D + col), v);
          }
        }
        const long long oi = (((long long)b * Sq + i) * p.H + h) * D + col, li = ((long long)b * p.H + h) * Sq + i;
        if (dbg_range(ab, oi, 1, o_size)) p.o[oi] = __float2bfloat16_rn(wsum > 0.0f ? v / wsum : 0.0f);
        if (col == 0 && dbg_range(ab, li, 1, lse_size))
          p.lse[li] = mx == -INFINITY ? -INFINITY : (mx + __log2f(wsum)) * kDecLn2;
      }
    }
    }
}

// ------------------------------------------------------------------ the decode kernel
//
// Both products run on the tensor core, transposed so that the keys, not the few new rows, fill
// the 128 rows of a tcgen05 tile. Per tile of 128 keys
// (two 64-key units of one sequence, each from its own page):
//   S^T = K Q^T    M = 128 keys, N = 16 (the Sq <= 8 new rows, zero-padded), K = d
//   O^T += V^T P^T M = d, N = 16, K = 128 keys          (d = 128)
//                  M = 128, N = 32, K = 64 keys         (d = 64: the two 64-key halves stacked in
//                  M, each half's weights in its own 16 columns of N; the two diagonal blocks are
//                  added up once per segment, the off-diagonal ones are never read)
// Thread i of the four softmax warps owns key i of the tile (TMEM lane i of S^T): its scores for
// every new row come in one TMEM load; the row maxima over the tile are exchanged between the
// warps through shared memory; P^T goes to shared memory as bf16, the B operand of the second
// product; O^T stays in TMEM (lane = column of O) across the tiles of a segment. Warp 4 loads the
// tiles (a ring of 3 stages at d = 128, 6 at d = 64: one CTA per SM), warp 5 issues the products,
// S(k + 1) ahead of P V(k). O is rescaled only when a row's maximum has grown by more than 2^8.
// P is rounded to bf16 for the product, so O is divided by the sum of the rounded weights and
// the log-sum-exp taken from the fp32 sum, as in the training forward. Pieces are counted in
// 64-key units (see the work split above).
constexpr float kDecRescale = 8.0f;  // log2 units

template <int D>
struct DecTcCfg {
  static constexpr int kTileKeys = 128;
  static constexpr int kBoxes = D / 64;                      // 64-column (128-byte) boxes per row
  static constexpr int kBoxBytes = kTileKeys * 128;          // one box of a 128-key tile (16 KB)
  static constexpr int kTileBytes = kBoxes * kBoxBytes;      // one K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;         // K, then V
  static constexpr int kStages = D == 64 ? 6 : 3;
  static constexpr int kOffKV = 0;
  static constexpr int kOffQ = kStages * kStageBytes;        // Q^T operand: 16 rows x d, K-major boxes of 2 KB
  static constexpr int kQBytes = 16 * D * 2;
  static constexpr int kNO = D == 64 ? 32 : 16;              // N of the second product
  static constexpr int kPBytes = 4096;                       // P^T operand: kNO rows x (2 x 64 or 64) keys
  static constexpr int kOffP = kOffQ + kQBytes;              // two P^T buffers, by tile parity
  static constexpr int kOffRed = kOffP + 2 * kPBytes;        // [2][4][8] row maxima of the warps, then [4][16] sums
  static constexpr int kOffEpi = kOffRed + 512;              // d = 64: [64][8] second-half columns of O
  static constexpr int kOffMisc = kOffEpi + (D == 64 ? 64 * 8 * 4 : 0);  // scan sums, first segment, flags
  static constexpr int kOffBar = kOffMisc + 128;  // full, empty [kStages]; s_bar, o_bar, p_full [2]; q_full, done
  static constexpr int kBarBytes = 256;                      // TMEM slot and abort flag in the last 64 bytes
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + alignment slack
  static constexpr uint32_t kColS = 0;                       // S^T buffers at columns 0 and 16
  static constexpr uint32_t kColO = 32;                      // O^T (kNO columns)
  static constexpr uint32_t kTmemCols = 64;
  static_assert((2 * kStages + 8) * 8 <= kBarBytes - 64, "barrier area");
  static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0, "swizzled operands sit on 1024-byte boundaries");
};

// A walk over the 128-key tiles of one piece: the units [t0, t1) of each segment, paired from t0
// (the last tile of a segment with an odd unit count has one unit).
struct DecTcWalk {
  DecWalk w;
  int ta;  // first unit of the current tile
  __device__ __forceinline__ void begin(const DecParams& p, int b0, long long s0, long long u0, long long u1) {
    w.begin(p, b0, s0, u0, u1);
    ta = w.t0;
  }
  __device__ __forceinline__ bool valid(const DecParams& p) const { return w.valid(p); }
  __device__ __forceinline__ int units() const { return min(2, w.t1 - ta); }
  // next tile; true when it starts a new segment (false at the end too: then valid() is false)
  __device__ __forceinline__ bool next(const DecParams& p, long long u0, long long u1) {
    ta += 2;
    if (ta < w.t1) return false;
    const bool more = w.next_seg(p, u0, u1);
    ta = w.t0;
    return more;
  }
};

// Pages and first rows of the (one or two) units of the walk's current tile. The loads are
// issued here and consumed by dec_tc_issue, so that their latency overlaps the producer's wait
// for a free slot.
struct DecTcPages {
  int page[2], row[2], units;
};
__device__ __forceinline__ DecTcPages dec_tc_pages(const DecParams& p, const DecTcWalk& tw, Abort ab) {
  DecTcPages pg;
  pg.units = tw.units();
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int key = (tw.ta + min(u, pg.units - 1)) * kDecTile;
    const long long ti = (long long)tw.w.b * p.max_pages + key / p.page_size;
    pg.page[u] = dbg_range(ab, ti, 1, (long long)p.B * p.max_pages) ? p.block_table[ti] : 0;
    pg.row[u] = key % p.page_size;
  }
  return pg;
}

// The producer's loads of one tile into its ring slot: one TMA box per 64-column box and unit,
// for K and for V; a missing second unit is left as it is (its keys are masked, its V rows
// zeroed by the softmax warps).
template <int D>
__device__ __forceinline__ bool dec_tc_issue(const DecParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                             uint32_t dst, uint64_t* full_bar, int h, DecTcPages pg, Abort ab,
                                             uint32_t smem_lo, uint32_t smem_end) {
  using Cfg = DecTcCfg<D>;
  const int nu = pg.units;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    if (u >= nu) break;
    if (pg.page[u] < 0 || pg.page[u] >= p.num_pages) {  // the TMA would read zeros there; report it
      atomicOr(&g_fa_error, kErrBadInput);
      pg.page[u] = 0;
    }
    for (int bx = 0; bx < Cfg::kBoxes; ++bx)
      if (!dbg_tma(ab, bx * 64, h, pg.row[u], pg.page[u], Cfg::kBoxes * 64, p.H, p.page_size, p.num_pages, 2,
                   dst + bx * Cfg::kBoxBytes + u * 8192, Cfg::kStageBytes - bx * Cfg::kBoxBytes - u * 8192, smem_lo,
                   smem_end))
        return false;
  }
  mbar_arrive_expect_tx(smem_u32(full_bar), (uint32_t)(nu * 2 * Cfg::kBoxes * 8192));
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int bx = 0; bx < Cfg::kBoxes && u < nu; ++bx) {
      const uint32_t off = bx * Cfg::kBoxBytes + u * 8192;
      tma_load_4d(dst + off, tmK, smem_u32(full_bar), bx * 64, h, pg.row[u], pg.page[u]);
      tma_load_4d(dst + Cfg::kTileBytes + off, tmV, smem_u32(full_bar), bx * 64, h, pg.row[u], pg.page[u]);
    }
  return true;
}

template <int D, int kRows>
__global__ void __launch_bounds__(kDecMmaThreads, 1)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const DecParams p) {
  using Cfg = DecTcCfg<D>;
  constexpr int kStages = Cfg::kStages;
  static_assert(kDecThreads == 128 && kDecMmaThreads == kDecThreads + 96, "softmax warps, producer, two issuers");
  static_assert(kRows == 4 || kRows == 8, "new rows a thread handles (padded to N = 16)");
  static_assert(kDecMaxSq <= 8, "at most 8 new rows");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (smem_base - smem_u32(smem_raw));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Cfg::kOffBar);
  uint64_t* empty = full + kStages;       // slot free again (P V of its tile completed)
  uint64_t* s_bar = full + 2 * kStages;   // [2] S(k) done, by k & 1
  uint64_t* o_bar = s_bar + 2;            // [2] P V(k) done, by k & 1
  uint64_t* p_full = s_bar + 4;           // [2] P^T(k) written, O rescaled, by k & 1 (one arrival per softmax warp)
  uint64_t* q_full = s_bar + 6;           // Q^T of a segment written (one arrival per softmax warp)
  uint64_t* done_bar = s_bar + 7;         // every product of both issuers has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::kOffBar + Cfg::kBarBytes - 64);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::kOffBar + Cfg::kBarBytes - 60);
  float* sRed = reinterpret_cast<float*>(sm + Cfg::kOffRed);
  float* sEpi = reinterpret_cast<float*>(sm + Cfg::kOffEpi);
  long long* sSum = reinterpret_cast<long long*>(sm + Cfg::kOffMisc);  // [0, 4) warp sums, [4] first start
  int* sInt = reinterpret_cast<int*>(sm + Cfg::kOffMisc + 48);          // [0] first sequence, [1] last flag
  const Abort ab{abort_flag};
  const uint32_t smem_end = smem_u32(smem_raw) + Cfg::kSmemBytes;  // for the FA_DEBUG bounds checks
  const long long o_size = (long long)p.B * p.Sq * p.H * D, lse_size = (long long)p.B * p.H * p.Sq;
  const long long part_rows = ((long long)p.B + p.pieces - 1) * p.H * p.Sq;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, piece = blockIdx.y;
  const int Sq = p.Sq;
  const uint32_t sQ = smem_base + Cfg::kOffQ;

  if (tid == 0) {
    *abort_flag = 0;
    sInt[0] = p.B;
    for (int i = 0; i < 2 * kStages + 4; ++i) mbar_init(smem_u32(&full[i]), 1);  // full, empty, s_bar, o_bar
    mbar_init(smem_u32(&p_full[0]), 4);
    mbar_init(smem_u32(&p_full[1]), 4);
    mbar_init(smem_u32(q_full), 4);
    mbar_init(smem_u32(done_bar), 2);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
    tc_fence_before_sync();
  }
  // P^T rows of no new row stay zero: both buffers cleared once
  for (int e = tid; e < 2 * Cfg::kPBytes / 16; e += kDecMmaThreads)
    st_shared_v4(smem_base + Cfg::kOffP + e * 16, 0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  const DecPiece pc = dec_prologue<D>(p, h, piece, ab, sSum, sInt);  // (its barriers publish the TMEM base)
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const long long T = pc.T, u0 = pc.u0, u1 = pc.u1, start_first = pc.start_first;
  const int Pe = pc.Pe, b_first = pc.b_first;
  auto kv_smem = [&](long long j) { return smem_base + Cfg::kOffKV + (uint32_t)(j % kStages) * Cfg::kStageBytes; };

  if (warp == 4) {
    // ---- producer: the piece's tiles in order (index j), each into its ring slot once the
    // P V of the tile before it in that slot has completed
    if (lane == 0 && u0 < u1) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      DecTcWalk tw;
      tw.begin(p, b_first, start_first, u0, u1);
      long long j = 0;
      DecTcPages pg = dec_tc_pages(p, tw, ab);
      for (bool more = tw.valid(p); more && !ab.raised(); ++j) {
        if (j >= kStages) mbar_wait(smem_u32(&empty[j % kStages]), (uint32_t)(((j / kStages) - 1) & 1), ab);
        if (ab.raised() || !dec_tc_issue<D>(p, &tmK, &tmV, kv_smem(j), &full[j % kStages], h, pg, ab, smem_base,
                                            smem_end))
          break;
        tw.next(p, u0, u1);
        more = tw.valid(p);
        if (more) pg = dec_tc_pages(p, tw, ab);  // the next tile's pages, read while this slot waits
      }
      if (ab.raised())  // loads issued past a wait that gave up land before the CTA exits
        for (long long i = max(0LL, j - kStages); i < j; ++i)
          mbar_drain(smem_u32(&full[i % kStages]), (uint32_t)((i / kStages) & 1));
    }
  } else if (warp == 5) {
    // ---- S issuer: S(k) into buffer k & 1 once the softmax of tile k - 2 has read it
    if (elect_one()) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 16, false, false);  // S^T: A (K) and B (Q) K-major
      long long k = 0;
      uint32_t seg = 0;
      DecTcWalk tw;
      tw.begin(p, b_first, start_first, u0, u1);
      for (bool more = tw.valid(p), seg_start = true; more; ++k) {
        if (seg_start) mbar_wait(smem_u32(q_full), (seg++) & 1, ab);  // this segment's Q^T
        if (k >= 2) mbar_wait(smem_u32(&p_full[k & 1]), (uint32_t)(((k - 2) >> 1) & 1), ab);
        mbar_wait(smem_u32(&full[k % kStages]), (uint32_t)((k / kStages) & 1), ab);
        tc_fence_after_sync();
        const uint32_t kt = kv_smem(k);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)  // 16 columns of d per step, 4 steps per box
          mma_ss(tmem + Cfg::kColS + (uint32_t)(k & 1) * 16,
                 sdesc_kmajor(kt + (kk >> 2) * Cfg::kBoxBytes + (kk & 3) * 32),
                 sdesc_kmajor(sQ + (kk >> 2) * 2048 + (kk & 3) * 32), idS, kk > 0);
        mma_commit(smem_u32(&s_bar[k & 1]));
        seg_start = tw.next(p, u0, u1);
        more = tw.valid(p);
      }
      mma_commit(smem_u32(done_bar));
    }
  } else if (warp == 6) {
    // ---- P V issuer: O^T += V^T P^T(k) once P^T(k) is written
    if (elect_one()) {
      constexpr uint32_t idO = idesc_bf16_f32(128, Cfg::kNO, true, false);  // O^T: A (V^T) MN-major, B (P^T) K-major
      long long k = 0;
      DecTcWalk tw;
      tw.begin(p, b_first, start_first, u0, u1);
      for (bool more = tw.valid(p), first = true; more; ++k) {
        mbar_wait(smem_u32(&p_full[k & 1]), (uint32_t)((k >> 1) & 1), ab);
        tc_fence_after_sync();
        const uint32_t vt = kv_smem(k) + Cfg::kTileBytes;
        const uint32_t pb = smem_base + Cfg::kOffP + (uint32_t)(k & 1) * Cfg::kPBytes;
        if constexpr (D == 128) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // 16 keys per step: 16 rows of V, 32 bytes of each P^T row
            mma_ss(tmem + Cfg::kColO, sdesc_mnmajor(vt + kk * 2048, Cfg::kBoxBytes),
                   sdesc_kmajor(pb + (kk >> 2) * 2048 + (kk & 3) * 32), idO, !first || kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // keys 16 kk.. of each half; the halves 8 KB apart in M
            mma_ss(tmem + Cfg::kColO, sdesc_mnmajor(vt + kk * 2048, 8192), sdesc_kmajor(pb + kk * 32), idO,
                   !first || kk > 0);
        }
        mma_commit(smem_u32(&o_bar[k & 1]));
        mma_commit(smem_u32(&empty[k % kStages]));  // (S(k) completed before P^T(k) was written)
        first = tw.next(p, u0, u1);
        more = tw.valid(p);
      }
      mma_commit(smem_u32(done_bar));
      mbar_drain(smem_u32(done_bar), 0);  // every product has completed before the TMEM is freed
    }
  } else {
    // ---- softmax warps 0-3: thread i owns key i of each tile (TMEM lane i of S^T)
    const uint32_t my_lanes = (uint32_t)(warp * 32) << 16;
    // O^T lanes: column d of O for d = 128; for d = 64, lanes 64..127 hold the second half's
    // sums of column d - 64 in O^T columns 16..23
    const uint32_t tO = tmem + Cfg::kColO + my_lanes + (D == 64 && warp >= 2 ? 16u : 0u);
    const float c = p.scale_log2;
    const int kk64 = tid & 63, half = tid >> 6;  // this thread's key within its 64-key unit, and the unit
    long long k = 0;
    DecTcWalk tw;
    tw.begin(p, b_first, start_first, u0, u1);
    bool more = tw.valid(p);
    while (more) {
      const int b = tw.w.b, n = tw.w.n, t_last = tw.w.t1;  // the segment ends at unit t_last
      const long long seg_start_unit = tw.w.start, seg_cnt = tw.w.cnt;
      // Q^T: row i holds new row i of (b, h) (zeros for rows past Sq); the previous segment's
      // products have all completed
      for (int e = tid; e < 16 * (D / 8); e += kDecThreads) {
        const int i = e / (D / 8), ch = e - i * (D / 8);
        const long long qi = (((long long)b * Sq + i) * p.H + h) * D + ch * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (i < Sq && dbg_range(ab, qi, 8, o_size)) v = *reinterpret_cast<const uint4*>(p.q + qi);
        st_shared_v4(sQ + (ch >> 3) * 2048 + sw128_offset(i, ch & 7), v.x, v.y, v.z, v.w);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(q_full));
      // per new row: the visible keys [kmin, khi] of this segment
      int kmin[kRows], khi[kRows];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int pos = n - Sq + i;
        kmin[i] = p.win_l >= 0 ? pos - p.win_l : 0;
        khi[i] = min(min(n - 1, t_last * kDecTile - 1), p.win_r >= 0 ? pos + p.win_r : n - 1);
        if (i >= Sq) khi[i] = -1;
      }
      float m_used[kRows], l_part[kRows], lr_part[kRows];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        m_used[i] = -INFINITY;
        l_part[i] = 0.0f;
        lr_part[i] = 0.0f;
      }
      bool seg_end = false;
      for (bool first = true; !seg_end; first = false, ++k) {
        const int key0 = tw.ta * kDecTile, nu = tw.units();
        // ---- scores of key key0 + tid for every new row; the row maxima over the tile
        mbar_wait(smem_u32(&s_bar[k & 1]), (uint32_t)((k >> 1) & 1), ab);
        tc_fence_after_sync();
        uint32_t sr[8];
        tmem_ld8(tmem + Cfg::kColS + (uint32_t)(k & 1) * 16 + my_lanes, sr);
        tmem_wait_ld(sr);
        const int key = key0 + tid;
        float x[kRows], wm[kRows];
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          x[i] = (key >= kmin[i] && key <= khi[i]) ? __uint_as_float(sr[i]) * c : -INFINITY;
          wm[i] = warp_max_f32(x[i]);
        }
        float4* red4 = reinterpret_cast<float4*>(sRed + ((k & 1) * 4 + warp) * 8);
        if (lane == 0) {
#pragma unroll
          for (int i = 0; i < kRows; i += 4) red4[i / 4] = make_float4(wm[i], wm[i + 1], wm[i + 2], wm[i + 3]);
        }
        named_bar_sync(2, kDecThreads);
        float m_tile[kRows];
#pragma unroll
        for (int i = 0; i < kRows; i += 4) {
          const float4* r4 = reinterpret_cast<const float4*>(sRed + (k & 1) * 32) + i / 4;
          const float4 a0 = r4[0], a1 = r4[2], a2 = r4[4], a3 = r4[6];
          m_tile[i] = fmaxf(fmaxf(a0.x, a1.x), fmaxf(a2.x, a3.x));
          m_tile[i + 1] = fmaxf(fmaxf(a0.y, a1.y), fmaxf(a2.y, a3.y));
          m_tile[i + 2] = fmaxf(fmaxf(a0.z, a1.z), fmaxf(a2.z, a3.z));
          m_tile[i + 3] = fmaxf(fmaxf(a0.w, a1.w), fmaxf(a2.w, a3.w));
        }
        // lazy rescale: a row's reference maximum moves only when the tile's exceeds it by more
        // than 2^8 (from -inf: at its first visible key); alpha = 2^(old - new), 0 from -inf
        float alpha[kRows];
        bool moved = false;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          const bool mv = m_tile[i] > m_used[i] + kDecRescale;
          alpha[i] = ex2_approx(mv ? m_used[i] - m_tile[i] : 0.0f);
          m_used[i] = mv ? m_tile[i] : m_used[i];
          moved = moved || mv;
        }
        // the P^T buffer of this parity is free once P V(k - 2) has completed
        if (k >= 2) mbar_wait(smem_u32(&o_bar[k & 1]), (uint32_t)(((k - 2) >> 1) & 1), ab);
        // P^T element (row i, key): d = 128: box key / 64 (2 KB each), row i; d = 64: row
        // 16 (key / 64) + i of one box; either way 2048 (key / 64) + 128 i bytes in
        const uint32_t pb = smem_base + Cfg::kOffP + (uint32_t)(k & 1) * Cfg::kPBytes + (uint32_t)half * 2048u;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          const float m_sub = m_used[i] == -INFINITY ? 0.0f : m_used[i];
          const float pv = ex2_approx(x[i] - m_sub);  // 2^-inf = 0
          const __nv_bfloat16 pr = __float2bfloat16_rn(pv);
          l_part[i] = fmaf(l_part[i], alpha[i], pv);
          lr_part[i] = fmaf(lr_part[i], alpha[i], __bfloat162float(pr));
          const uint32_t addr = pb + (uint32_t)i * 128u + ((((uint32_t)kk64 >> 3) ^ (uint32_t)(i & 7)) << 4) +
                                ((uint32_t)kk64 & 7u) * 2u;
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(__bfloat16_as_ushort(pr)) : "memory");
        }
        // O^T *= alpha (column i of O^T is new row i) for the rows whose maximum moved, once
        // P V(k - 1) has completed
        if (!first && moved) {
          mbar_wait(smem_u32(&o_bar[(k - 1) & 1]), (uint32_t)(((k - 1) >> 1) & 1), ab);
          tc_fence_after_sync();
          uint32_t o[8];
          tmem_ld8(tO, o);
          tmem_wait_ld(o);
#pragma unroll
          for (int i = 0; i < kRows; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[i]);
          tmem_st8(tO, o);
        }
        // V rows past the last valid key of the tile (the sequence's end, the piece's last unit,
        // a missing second unit) may hold anything, a NaN among it: zero them before the product
        const int v_end = min(n, t_last * kDecTile) - key0;
        if (v_end < nu * kDecTile || nu < 2) {
          mbar_wait(smem_u32(&full[k % kStages]), (uint32_t)((k / kStages) & 1), ab);
          const uint32_t vt = kv_smem(k) + Cfg::kTileBytes;
          const int from = max(0, v_end);
          for (int e = tid; e < (Cfg::kTileKeys - from) * Cfg::kBoxes * 8; e += kDecThreads) {
            const int row = from + e / (Cfg::kBoxes * 8), rest = e % (Cfg::kBoxes * 8);
            st_shared_v4(vt + (rest >> 3) * Cfg::kBoxBytes + row * 128 + (rest & 7) * 16, 0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&p_full[k & 1]));
        seg_end = tw.next(p, u0, u1);
        more = tw.valid(p);
        seg_end = seg_end || !more;
      }

      // ---- segment end: row sums over the CTA; O / (sum of the weights applied), log2-sum-exp
      // of the fp32 sum
      mbar_wait(smem_u32(&o_bar[(k - 1) & 1]), (uint32_t)(((k - 1) >> 1) & 1), ab);
      tc_fence_after_sync();
      float* sL = sRed + 64;  // [4][16]: per warp, fp32 and rounded sums of the rows
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        float a = l_part[i], r = lr_part[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          a += __shfl_xor_sync(0xffffffffu, a, off);
          r += __shfl_xor_sync(0xffffffffu, r, off);
        }
        if (lane == 0) {
          sL[warp * 16 + i] = a;
          sL[warp * 16 + 8 + i] = r;
        }
      }
      uint32_t o[8];
      tmem_ld8(tO, o);
      tmem_wait_ld(o);
      if (D == 64 && warp >= 2) {
#pragma unroll
        for (int i = 0; i < kRows; ++i) sEpi[(tid - 64) * 8 + i] = __uint_as_float(o[i]);
      }
      named_bar_sync(2, kDecThreads);
      const int pf = dec_piece_of(T, Pe, seg_start_unit), pl = dec_piece_of(T, Pe, seg_start_unit + seg_cnt - 1);
      const size_t slot = (size_t)b + piece;  // partial slot of (b, this piece)
      if (D == 128 || warp < 2) {
        const int col = tid;  // column of O
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          if (i >= Sq) break;
          const float lr = sL[i + 8] + sL[16 + i + 8] + sL[32 + i + 8] + sL[48 + i + 8];
          float v = __uint_as_float(o[i]);
          if (D == 64) v += sEpi[tid * 8 + i];
          v = lr > 0.0f ? v / lr : 0.0f;
          if (pf == pl) {
            const long long oi = (((long long)b * Sq + i) * p.H + h) * D + col;
            if (dbg_range(ab, oi, 1, o_size)) p.o[oi] = __float2bfloat16_rn(v);
          } else {
            const long long pi = (((long long)slot * p.H + h) * Sq + i) * D + col;
            if (dbg_range(ab, pi, 1, part_rows * D)) p.o_part[pi] = v;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kRows; ++i) {  // thread i writes row i's statistic
        if (i != tid || i >= Sq) continue;
        const float l = sL[i] + sL[16 + i] + sL[32 + i] + sL[48 + i];
        const float l2 = l > 0.0f ? m_used[i] + __log2f(l) : -INFINITY;
        if (pf == pl) {
          const long long li = ((long long)b * p.H + h) * Sq + i;
          if (dbg_range(ab, li, 1, lse_size)) p.lse[li] = l2 == -INFINITY ? -INFINITY : l2 * kDecLn2;
        } else {
          const long long pi = ((long long)slot * p.H + h) * Sq + i;
          if (dbg_range(ab, pi, 1, part_rows)) p.lse_part[pi] = l2;
        }
      }
      tc_fence_before_sync();
      if (pf != pl) dec_arrive_merge<D>(p, b, h, pf, pl, ab, sInt);
      named_bar_sync(1, kDecThreads);  // the next segment rewrites the sums, the exchange and the last flag
    }
  }

  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// Zero the (b, h) arrival counters of a call with several pieces per head. It lets the split
// kernel launch at once (that kernel waits for this one only before its first arrival).
__global__ void __launch_bounds__(256) fa_decode_prep_kernel(int* arrivals, int count) {
  griddep_launch_dependents();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += gridDim.x * blockDim.x) arrivals[i] = 0;
}

}  // namespace fa
