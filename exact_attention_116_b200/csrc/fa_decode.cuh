// Attention of a few new query rows against a paged KV cache (decoding), for sm_100a.
//
// What it computes ("FlashAttention技术解析：加速GPT训练的核心优化" §5, FlashDecoding;
// "突破大模型训练瓶颈：Flash-Attention编译优化与内存占用解决方案", Paged KV Cache): for every
// sequence b, head h and new query row i (0 <= i < Sq, at position pos = seqlen_b - Sq + i),
// O = softmax(scale * q . k_j) V over the cached keys j < seqlen_b that the mask leaves visible,
// and LSE = ln sum_j exp(scale * q . k_j). Key j of sequence b is row j % page_size of page
// block_table[b][j / page_size] of the (num_pages, page_size, H, d) cache.
//
// The work is one pass over the cache: HBM-bound (each K/V element is used by Sq <= 8 rows),
// so it runs on the CUDA cores, not the tensor cores. Split-KV: the keys of every (b, h) are
// cut into `splits` contiguous ranges, one CTA each; a CTA streams its 64-key K/V tiles by TMA
// into a 3-stage ring (a 64-key tile never straddles a page: page_size is a multiple of 64),
// keeps a running maximum and sum per row (log2 domain) and writes a partial (O / l, log2 l + m).
// The last CTA of a (b, h) to finish (an arrival counter per (b, h)) merges the partials by
// their log-sum-exp and writes O and LSE; with one split the CTA writes them itself. The
// counters are zeroed by fa_decode_prep_kernel, launched just before on the same stream; the
// split kernel is launched as its programmatic dependent, so it streams the cache while the
// prep kernel runs and waits for it only before its first arrival.
//
// CTA (128 threads), per tile of 64 keys:
//   A: thread (key t = tid % 64, half = tid / 64) forms half of q_i . k_t for every row i
//   B: warp w owns rows w and w + 4: mask, tile max, exponentials, running max / sum, rescale
//      factor alpha_i; P goes to shared memory
//   C: thread (column pair, key group) accumulates O_i += P_i,t v_t over its keys
// The kernel is compiled for kSq = 1, 2, 4, 8 rows (the call's Sq rounded up; the extra rows
// have q = 0 and are not written). CTAs of the same (b, split) for consecutive heads are
// launched next to each other (head is the fastest grid index), so the 128-byte rows of one
// cache row (H x d bf16, contiguous) are read by concurrent CTAs.
//
// With new K/V rows given (flash_attn_with_kvcache's in-place update of the cache), the CTA
// whose key range holds a new row writes that row's d columns of its head into the cache
// before it loads any tile: every new row is visible to the newest query row, so exactly one
// split of each head covers it, and no other CTA reads those bytes.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kDecMaxSq = 8;       // new query rows per call
constexpr int kDecTile = 64;       // keys per tile
constexpr int kStagesMax = 3;   // K/V ring depth for 8 new rows
constexpr int kDecThreads = 128;
constexpr float kDecLn2 = 0.69314718055994530942f;

// Generic-proxy writes to global memory by this thread are ordered before later async-proxy
// (TMA) accesses that a barrier orders after this fence.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Programmatic dependent launch: let the next kernel on the stream (launched with the
// programmatic-serialization attribute) start, and, in that kernel, wait until the grids it
// depends on have finished and their writes are visible. The wait returns at once in a
// kernel launched without the attribute.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

struct DecParams {
  int B, Sq, H, page_size, max_pages, num_pages;
  float scale_log2;      // scale * log2(e)
  int win_l, win_r;      // -1 = unbounded; causal already folded into win_r = 0
  int splits;
  const int* block_table;  // (B, max_pages)
  const int* seqlens;      // (B)
  const __nv_bfloat16* q;  // (B, Sq, H, d)
  __nv_bfloat16* o;        // (B, Sq, H, d)
  float* lse;              // (B, H, Sq), natural log
  float* o_part;           // (B, H, Sq, splits, d) fp32 (splits > 1)
  float* lse_part;         // (B, H, Sq, splits), log2 domain (splits > 1)
  int* arrivals;           // (B, H) split CTAs finished (splits > 1), zeroed by the prep kernel
  const __nv_bfloat16* k_new;  // (B, Sq, H, d) rows to write into the cache, or null
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_cache;  // (num_pages, page_size, H, d)
  __nv_bfloat16* v_cache;
};

// Shared memory of a CTA compiled for kSq rows: up to 4 rows a 2-stage ring (about 67 KB at
// d = 128, so that three CTAs share an SM and hide each other's per-tile latency), 8 rows a
// 3-stage ring (two CTAs per SM).
template <int D, int kSq>
struct DecCfg {
  static constexpr int kStages = (kSq <= 4) ? 2 : kStagesMax;
  static constexpr int kBoxes = D / 64;                       // 64-column (128-byte) boxes per row
  static constexpr int kTileBytes = kDecTile * D * 2;         // one K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;          // K and V
  static constexpr int kOffKV = 0;
  static constexpr int kOffQ = kStages * kStageBytes;          // q rows, fp32 (kSq x D)
  static constexpr int kOffS = kOffQ + kSq * D * 4;            // half-dot products (2 x kSq x 64)
  static constexpr int kOffP = kOffS + 2 * kSq * kDecTile * 4;  // P (kSq x 64)
  static constexpr int kOffAlpha = kOffP + kSq * kDecTile * 4;  // rescale factor per row
  static constexpr int kPairs = D / 2;                          // column pairs
  static constexpr int kKeyGroups = kDecThreads / kPairs;       // 2 (D=128) or 4 (D=64)
  static constexpr int kOffRed = kOffKV;  // final reduction (key groups x kSq x D), over the drained ring
  static_assert(kKeyGroups * kSq * D * 4 <= kStages * kStageBytes, "reduction buffer");
  static constexpr int kOffBar = (kOffAlpha + kSq * 4 + 63) & ~63;
  static constexpr int kSmemBytes = kOffBar + 128 + 1024;       // barriers + alignment slack
};

// Keys [t0 * 64, t1 * 64) of sequence b that split s covers, clipped to what rows
// [pos0, pos0 + Sq) can see. Returns false when the split has nothing to do.
__device__ __forceinline__ bool dec_tile_range(const DecParams& p, int n, int s, int& t0, int& t1) {
  const int tiles = (n + kDecTile - 1) / kDecTile;
  t0 = (int)((long long)s * tiles / p.splits);
  t1 = (int)((long long)(s + 1) * tiles / p.splits);
  const int pos0 = n - p.Sq, pos1 = n - 1;
  const int vis_lo = p.win_l >= 0 ? max(0, pos0 - p.win_l) : 0;
  const int vis_hi = p.win_r >= 0 ? min(n - 1, pos1 + p.win_r) : n - 1;
  t0 = max(t0, vis_lo / kDecTile);
  t1 = min(t1, vis_hi / kDecTile + 1);
  return n > 0 && t1 > t0;
}

template <int D, int kSq>
__global__ void __launch_bounds__(kDecThreads)
    fa_decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const DecParams p) {
  using Cfg = DecCfg<D, kSq>;
  constexpr int kStages = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (smem_base - smem_u32(smem_raw));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Cfg::kOffBar);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::kOffBar + 64);
  float* sQ = reinterpret_cast<float*>(sm + Cfg::kOffQ);
  float* sS = reinterpret_cast<float*>(sm + Cfg::kOffS);
  float* sP = reinterpret_cast<float*>(sm + Cfg::kOffP);
  float* sAlpha = reinterpret_cast<float*>(sm + Cfg::kOffAlpha);
  float* sRed = reinterpret_cast<float*>(sm + Cfg::kOffRed);
  const Abort ab{abort_flag};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  static_assert(kSq >= 1 && kSq <= kDecMaxSq, "rows per CTA");
  const int h = blockIdx.x, s = blockIdx.y, b = blockIdx.z;
  const int Sq = p.Sq;
  int n = p.seqlens[b];
  if (n < 0 || n > p.max_pages * p.page_size) {  // reported by fa_check; the sequence is treated as empty
    if (threadIdx.x == 0) atomicOr(&g_fa_error, kErrBadInput);
    n = 0;
  }

  int t0 = 0, t1 = 0;
  if (!dec_tile_range(p, n, s, t0, t1)) t1 = t0;

  // new rows in this CTA's key range: head h's columns go into the cache before any tile load
  if (p.k_new != nullptr && t1 > t0) {
    const int key_lo = t0 * kDecTile, key_hi = t1 * kDecTile;
    constexpr int kChunks = D / 8;  // 16-byte chunks of one head's row
    bool wrote = false;
    for (int i = 0; i < Sq; ++i) {
      const int pos = n - Sq + i;
      if (pos < key_lo || pos >= key_hi) continue;  // another split's (or, pos < 0, nobody's)
      const int page = p.block_table[(size_t)b * p.max_pages + pos / p.page_size];
      if (page < 0 || page >= p.num_pages) {  // reported below when the tile is loaded
        continue;
      }
      const size_t src = (((size_t)b * Sq + i) * p.H + h) * D;
      const size_t dst = (((size_t)page * p.page_size + pos % p.page_size) * p.H + h) * D;
      if (tid < kChunks) {
        reinterpret_cast<uint4*>(p.k_cache + dst)[tid] = reinterpret_cast<const uint4*>(p.k_new + src)[tid];
      } else if (tid < 2 * kChunks) {
        reinterpret_cast<uint4*>(p.v_cache + dst)[tid - kChunks] =
            reinterpret_cast<const uint4*>(p.v_new + src)[tid - kChunks];
      }
      wrote = true;
    }
    if (wrote) fence_proxy_async_global();  // ordered before the TMA loads by the barrier below
  }

  if (tid == 0) {
    *abort_flag = 0;
    for (int st = 0; st < kStages; ++st) mbar_init(smem_u32(&full[st]), 1);
    fence_barrier_init();
  }
  if (tid < kSq) sAlpha[tid] = 0.0f;  // rows past Sq keep alpha = 0 (their O stays 0)
  // q rows -> shared memory (fp32); rows >= Sq are zero
  for (int e = tid; e < kSq * D; e += kDecThreads) {
    const int i = e / D, c = e - i * D;
    sQ[e] = i < Sq ? __bfloat162float(p.q[(((size_t)b * Sq + i) * p.H + h) * D + c]) : 0.0f;
  }
  __syncthreads();

  // TMA: tile t of this sequence -> stage slot; keys [64 t, 64 t + 64) lie in one page.
  auto issue = [&](int t) {
    const int st = (t - t0) % kStages;
    const int key = t * kDecTile;
    int page = p.block_table[(size_t)b * p.max_pages + key / p.page_size];
    if (page < 0 || page >= p.num_pages) {  // the TMA would read zeros there; report it
      atomicOr(&g_fa_error, kErrBadInput);
      page = 0;
    }
    const int row = key % p.page_size;
    const uint32_t dst = smem_base + Cfg::kOffKV + st * Cfg::kStageBytes;
    mbar_arrive_expect_tx(smem_u32(&full[st]), Cfg::kStageBytes);
#pragma unroll
    for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
      tma_load_4d(dst + bx * (kDecTile * 128), &tmK, smem_u32(&full[st]), bx * 64, h, row, page);
      tma_load_4d(dst + Cfg::kTileBytes + bx * (kDecTile * 128), &tmV, smem_u32(&full[st]), bx * 64, h, row, page);
    }
  };
  if (tid == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    for (int t = t0; t < t1 && t < t0 + kStages; ++t) issue(t);
  }

  // running state: warp w owns rows w and w + 4 (warp-uniform values)
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
  // O accumulators of this thread: rows 0..Sq-1, columns 2 cp and 2 cp + 1, keys of group kg
  const int cp = tid % Cfg::kPairs, kg = tid / Cfg::kPairs;
  float acc[kSq][2];
#pragma unroll
  for (int i = 0; i < kSq; ++i) acc[i][0] = acc[i][1] = 0.0f;
  const float c = p.scale_log2;

  for (int t = t0; t < t1; ++t) {
    const int st = (t - t0) % kStages;
    mbar_wait(smem_u32(&full[st]), ((t - t0) / kStages) & 1, ab);
    const uint8_t* kgen = sm + Cfg::kOffKV + st * Cfg::kStageBytes;
    const uint8_t* vgen = kgen + Cfg::kTileBytes;
    // ---- A: half dot products, key kt = tid % 64, dims [half * D/2, half * D/2 + D/2)
    {
      const int kt = tid % kDecTile, half = tid / kDecTile;
      float part[kSq];
#pragma unroll
      for (int i = 0; i < kSq; ++i) part[i] = 0.0f;
#pragma unroll
      for (int ch = 0; ch < D / 16; ++ch) {  // 16-byte chunks of this thread's half row
        const int col0 = half * (D / 2) + ch * 8;
        const int bx = col0 / 64, chunk = (col0 % 64) / 8;
        const uint4 raw = *reinterpret_cast<const uint4*>(kgen + bx * (kDecTile * 128) + sw128_offset(kt, chunk));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        float kv[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kv[2 * e] = bf16lo_to_f32(w[e]);
          kv[2 * e + 1] = bf16hi_to_f32(w[e]);
        }
#pragma unroll
        for (int i = 0; i < kSq; ++i) {  // rows past Sq have q = 0
          const float4 qa = *reinterpret_cast<const float4*>(&sQ[i * D + col0]);
          const float4 qb = *reinterpret_cast<const float4*>(&sQ[i * D + col0 + 4]);
          part[i] = fmaf(qa.x, kv[0], part[i]);
          part[i] = fmaf(qa.y, kv[1], part[i]);
          part[i] = fmaf(qa.z, kv[2], part[i]);
          part[i] = fmaf(qa.w, kv[3], part[i]);
          part[i] = fmaf(qb.x, kv[4], part[i]);
          part[i] = fmaf(qb.y, kv[5], part[i]);
          part[i] = fmaf(qb.z, kv[6], part[i]);
          part[i] = fmaf(qb.w, kv[7], part[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < kSq; ++i) sS[(half * kSq + i) * kDecTile + kt] = part[i];
    }
    __syncthreads();
    // every thread has finished with the previous tile's slot: refill it (not after a wait gave
    // up: that slot's barrier may still be waiting for bytes, and must not be armed twice)
    if (tid == 0 && t > t0 && t - 1 + kStages < t1 && !ab.raised()) issue(t - 1 + kStages);
    // ---- B: softmax bookkeeping, warp w -> rows w, w + 4
#pragma unroll
    for (int r = 0; r < (kSq + 3) / 4; ++r) {
      const int i = warp + 4 * r;
      if (i < Sq) {
        const int pos = n - Sq + i;
        const int kmin = p.win_l >= 0 ? pos - p.win_l : 0;
        const int kmax = p.win_r >= 0 ? min(n - 1, pos + p.win_r) : n - 1;
        float x[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int kt = lane + 32 * u, key = t * kDecTile + kt;
          const float sc = (sS[i * kDecTile + kt] + sS[(kSq + i) * kDecTile + kt]) * c;
          x[u] = (key >= kmin && key <= kmax) ? sc : -INFINITY;
        }
        float tmax = fmaxf(x[0], x[1]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
        const float m_new = fmaxf(m_run[r], tmax);
        const float m_use = m_new == -INFINITY ? 0.0f : m_new;
        const float alpha = m_run[r] == -INFINITY ? 0.0f : ex2_approx(m_run[r] - m_use);
        float psum = 0.0f;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float pv = ex2_approx(x[u] - m_use);  // exp2(-inf) = 0
          sP[i * kDecTile + lane + 32 * u] = pv;
          psum += pv;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
        l_run[r] = l_run[r] * alpha + psum;
        m_run[r] = m_new;
        if (lane == 0) sAlpha[i] = alpha;
      }
    }
    __syncthreads();
    // ---- C: O_i = alpha_i O_i + sum_t P_i,t v_t over this thread's keys t = kg, kg + kKeyGroups, ...
    {
      const int col = 2 * cp, bx = col / 64, chunk = (col % 64) / 8, within = (col % 8) * 2;
#pragma unroll
      for (int i = 0; i < kSq; ++i) {  // rows past Sq stay 0
        const float a = sAlpha[i];
        acc[i][0] *= a;
        acc[i][1] *= a;
      }
#pragma unroll 4
      for (int kt = kg; kt < kDecTile; kt += Cfg::kKeyGroups) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(vgen + bx * (kDecTile * 128) + sw128_offset(kt, chunk) +
                                                              within);
        const float v0 = bf16lo_to_f32(w), v1 = bf16hi_to_f32(w);
#pragma unroll
        for (int i = 0; i < kSq; ++i) {
          const float pv = sP[i * kDecTile + kt];
          acc[i][0] = fmaf(pv, v0, acc[i][0]);
          acc[i][1] = fmaf(pv, v1, acc[i][1]);
        }
      }
    }
  }

  // drain: loads issued past a wait that gave up must land before the ring is reused
  if (tid == 0 && ab.raised()) {
    for (int t = max(t0, t1 - kStages); t < t1; ++t) {
      const int st = (t - t0) % kStages;
      mbar_drain(smem_u32(&full[st]), ((t - t0) / kStages) & 1);
    }
  }
  __syncthreads();  // the K/V ring is free: it holds the reduction below
  // ---- combine the key groups' partial sums, normalise, write
#pragma unroll
  for (int i = 0; i < kSq; ++i) {
    sRed[(kg * kSq + i) * D + 2 * cp] = acc[i][0];
    sRed[(kg * kSq + i) * D + 2 * cp + 1] = acc[i][1];
  }
  // row statistics of warp-owned rows -> shared (reuse the alpha slots as 1/l, S as log2 l + m)
  __syncthreads();
#pragma unroll
  for (int r = 0; r < (kSq + 3) / 4; ++r) {
    const int i = warp + 4 * r;
    if (i < Sq && lane == 0) {
      sAlpha[i] = l_run[r] > 0.0f ? 1.0f / l_run[r] : 0.0f;
      sS[i] = l_run[r] > 0.0f ? m_run[r] + __log2f(l_run[r]) : -INFINITY;
    }
  }
  __syncthreads();
  for (int e = tid; e < Sq * D; e += kDecThreads) {
    const int i = e / D, col = e - i * D;
    float v = 0.0f;
#pragma unroll
    for (int g = 0; g < Cfg::kKeyGroups; ++g) v += sRed[(g * kSq + i) * D + col];
    v *= sAlpha[i];
    if (p.splits == 1) {
      p.o[(((size_t)b * Sq + i) * p.H + h) * D + col] = __float2bfloat16_rn(v);
    } else {
      p.o_part[((((size_t)b * p.H + h) * Sq + i) * p.splits + s) * D + col] = v;
    }
  }
  if (tid < Sq) {
    const float l2 = sS[tid];
    if (p.splits == 1)
      p.lse[((size_t)b * p.H + h) * Sq + tid] = l2 == -INFINITY ? -INFINITY : l2 * kDecLn2;
    else
      p.lse_part[(((size_t)b * p.H + h) * Sq + tid) * p.splits + s] = l2;
  }
  if (p.splits == 1) return;

  // ---- arrival: the last split of (b, h) merges all partials
  __threadfence();  // this thread's partials are visible device-wide before the arrival
  __syncthreads();
  int* last = abort_flag + 1;
  if (tid == 0) {
    griddep_wait();  // the prep kernel has zeroed the counters
    const int before = atomicAdd(&p.arrivals[(size_t)b * p.H + h], 1);
    *last = before == p.splits - 1;
  }
  __syncthreads();
  if (!*last) return;
  __threadfence();
  // O = sum_s 2^(L_s - L) O_s, L = log2 sum_s 2^L_s, in split order (the same sum whichever
  // CTA arrives last)
  for (int e = tid; e < Sq * D; e += kDecThreads) {
    const int i = e / D, col = e - i * D;
    const size_t row = ((size_t)b * p.H + h) * Sq + i;
    const float* lp = p.lse_part + row * p.splits;
    float mx = -INFINITY;
    for (int u = 0; u < p.splits; ++u) mx = fmaxf(mx, __ldcg(lp + u));
    float wsum = 0.0f, v = 0.0f;
    if (mx != -INFINITY) {
      for (int u = 0; u < p.splits; ++u) {
        const float w = ex2_approx(__ldcg(lp + u) - mx);
        wsum += w;
        v = fmaf(w, __ldcg(p.o_part + (row * p.splits + u) * D + col), v);
      }
    }
    p.o[(((size_t)b * Sq + i) * p.H + h) * D + col] = __float2bfloat16_rn(wsum > 0.0f ? v / wsum : 0.0f);
    if (col == 0) p.lse[row] = mx == -INFINITY ? -INFINITY : (mx + __log2f(wsum)) * kDecLn2;
  }
}

// Zero the (b, h) arrival counters of a split call. It lets the split kernel launch at once
// (that kernel waits for this one only before its first arrival).
__global__ void __launch_bounds__(256) fa_decode_prep_kernel(int* arrivals, int count) {
  griddep_launch_dependents();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += gridDim.x * blockDim.x) arrivals[i] = 0;
}

}  // namespace fa
