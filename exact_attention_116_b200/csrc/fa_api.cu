// Host side of the fa_sm100 C ABI: argument validation, TMA tensor maps, per-device
// kernel attributes, launches on the caller's stream and device-side error reporting.
// The kernels live in fa_fwd.cuh / fa_bwd.cuh and are compiled into this one translation
// unit (they share the device error word).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "fa_sm100.h"
#include "fa_bwd.cuh"
#include "fa_bwd_dq.cuh"
#include "fa_decode.cuh"
#include "fa_fwd.cuh"

namespace {

constexpr int kMaxDevices = 64;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
int g_sm_count[kMaxDevices] = {0};
bool g_attr_done[kMaxDevices] = {false};
bool g_is_sm100[kMaxDevices] = {false};

EncodeTiledFn encode_fn() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}

bool log_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = std::getenv("FA_LOG");
    on = (e && e[0] == '1') ? 1 : 0;
  }
  return on == 1;
}

// Per-device set-up: SM count, sm_100 check, dynamic shared memory opt-in of every kernel.
// Shared-memory attributes of every (ALiBi, packed) variant of the bf16 kernels of head dim D.
template <int D, bool kAlibi, bool kVarlen>
bool variant_attributes() {
  const auto attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
  const int smem = fa::BwdCfg<D>::kSmemBytes, smem_dq = fa::BwdDqCfg<D>::kSmemBytes;
  const int smem_fwd = fa::FwdCfg<D>::kSmemBytes + (kVarlen ? fa::kFwdSortBytes : 0);
  return cudaFuncSetAttribute(fa::fa_fwd_kernel<D, false, kAlibi, kVarlen>, attr, smem_fwd) == cudaSuccess &&
         cudaFuncSetAttribute(fa::fa_bwd_kernel<D, true, kAlibi, kVarlen>, attr, smem) == cudaSuccess &&
         cudaFuncSetAttribute(fa::fa_bwd_kernel<D, false, kAlibi, kVarlen>, attr, smem) == cudaSuccess &&
         cudaFuncSetAttribute(fa::fa_bwd_dq_kernel<D, kAlibi, kVarlen>, attr, smem_dq) == cudaSuccess;
}

template <int D>
bool bwd_attributes() {
  return variant_attributes<D, false, false>() && variant_attributes<D, true, false>() &&
         variant_attributes<D, false, true>() && variant_attributes<D, true, true>();
}

// Dynamic shared memory size of the decode kernel, and the largest shared-memory carveout (one
// CTA takes nearly all of an SM's).
template <int D>
bool decode_attributes() {
  for (const void* k : {(const void*)fa::fa_decode_kernel<D, 4>, (const void*)fa::fa_decode_kernel<D, 8>})
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, fa::DecTcCfg<D>::kSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
            cudaSuccess)
      return false;
  return true;
}

int device_setup(int* dev_out, int* sm_count) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_attr_done[dev]) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    g_is_sm100[dev] = (major == 10 && minor == 0);
    g_sm_count[dev] = sms;
    if (g_is_sm100[dev]) {
      if (cudaFuncSetAttribute(fa::fa_fwd_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::FwdCfg<128, true>::kSmemBytes) != cudaSuccess ||
          !decode_attributes<64>() || !decode_attributes<128>() ||
          !bwd_attributes<64>() || !bwd_attributes<128>())
        return FA_ERR_CUDA;
    }
    g_attr_done[dev] = true;
  }
  if (!g_is_sm100[dev]) return FA_ERR_UNSUPPORTED;
  *dev_out = dev;
  *sm_count = g_sm_count[dev];
  return FA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Shape {
  int B, N, H, d;
  size_t elems() const { return (size_t)B * N * H * d; }
  size_t tensor_bytes() const { return elems() * 2; }
  size_t rowvec_bytes() const { return (size_t)B * H * N * 4; }
  int n_pad() const { return (N + 127) / 128 * 128; }
};

// Sizes, head dim, windows and scale. Windows are normalised: causal forces win_r = 0,
// and a bound that reaches the whole sequence becomes -1 (unbounded).
int check_problem(int B, int N, int H, int d, float scale, int causal, int* win_l, int* win_r) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return FA_ERR_INVALID_ARG;
  if (*win_l < -1 || *win_r < -1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  // TMA: strides < 2^40 bytes; item counts and coordinates stay in int.
  const double row_stride = (double)N * H * d * 2;
  if (row_stride >= 1099511627776.0) return FA_ERR_INVALID_ARG;
  if ((double)B * H * ((N + 127) / 128) >= 2147483647.0) return FA_ERR_INVALID_ARG;
  if (causal) *win_r = 0;
  if (*win_l >= N - 1) *win_l = -1;
  if (*win_r >= N - 1) *win_r = -1;
  return FA_OK;
}

// 4-D map over a (B, N, H, d) bf16 tensor: dims (d, N, H, B), box (64, 128, 1, 1), 128B swizzle.
int make_map(CUtensorMap* m, const void* base, const Shape& s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)s.d, (cuuint64_t)s.N, (cuuint64_t)s.H, (cuuint64_t)s.B};
  const cuuint64_t strides[3] = {(cuuint64_t)s.H * s.d * 2, (cuuint64_t)s.d * 2, (cuuint64_t)s.N * s.H * s.d * 2};
  const cuuint32_t box[4] = {64, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_INVALID_ARG;
}

// 4-D map over a (B, N, H, d) tensor of E4M3 codes: dims (d, N, H, B), box (128, 128, 1, 1)
// (128 bytes x 128 rows), 128B swizzle.
int make_map_u8(CUtensorMap* m, const void* base, const Shape& s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)s.d, (cuuint64_t)s.N, (cuuint64_t)s.H, (cuuint64_t)s.B};
  const cuuint64_t strides[3] = {(cuuint64_t)s.H * s.d, (cuuint64_t)s.d, (cuuint64_t)s.N * s.H * s.d};
  const cuuint32_t box[4] = {128, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_INVALID_ARG;
}

// 4-D map over a paged (num_pages, page_size, H, d) bf16 cache: dims (d, H, page_size, num_pages),
// box (64, 1, 64, 1) (128 bytes x 64 rows of one head and one page), 128B swizzle.
int make_map_cache(CUtensorMap* m, const void* base, int num_pages, int page_size, int H, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)page_size, (cuuint64_t)num_pages};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)page_size * H * d * 2};
  const cuuint32_t box[4] = {64, 1, 64, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_INVALID_ARG;
}

// 4-D map over the (B, N, H, d) fp32 dQ accumulator for TMA reduce-add: box (32, 128, 1, 1)
// (128 bytes x 128 rows), 128B swizzle.
int make_map_f32_acc(CUtensorMap* m, const void* base, const Shape& s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)s.d, (cuuint64_t)s.N, (cuuint64_t)s.H, (cuuint64_t)s.B};
  const cuuint64_t strides[3] = {(cuuint64_t)s.H * s.d * 4, (cuuint64_t)s.d * 4, (cuuint64_t)s.N * s.H * s.d * 4};
  const cuuint32_t box[4] = {32, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_INVALID_ARG;
}

struct Workspace {
  float* dq_acc;
  float* lse2;
  float* dvec;
  int* next_item;
};

size_t workspace_bytes(const Shape& s) {
  return align256(s.elems() * 4) + 2 * align256((size_t)s.B * s.H * s.n_pad() * 4) + 256;
}

// Layout: dQ accumulator | -LSE*log2(e) | -D | work counter, each 256-byte aligned.
Workspace carve(void* ws, const Shape& s) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  Workspace w;
  w.dq_acc = reinterpret_cast<float*>(p);
  p += align256(s.elems() * 4);
  w.lse2 = reinterpret_cast<float*>(p);
  p += align256((size_t)s.B * s.H * s.n_pad() * 4);
  w.dvec = reinterpret_cast<float*>(p);
  p += align256((size_t)s.B * s.H * s.n_pad() * 4);
  w.next_item = reinterpret_cast<int*>(p);
  return w;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

// ---------------------------------------------------------------- launches (arguments already checked)

// The forward's work counter: slots of fa::g_fwd_next_item are handed out in turn per device,
// so calls in flight at the same time (on different streams) count in different slots as long
// as fewer than kFwdCounterSlots of them overlap. Each launch zeroes its slot first.
std::atomic<unsigned> g_fwd_slot_seq[kMaxDevices];

// The counter-reset kernel, then the forward kernel as its programmatic dependent (it sets up
// while the reset runs and waits for it before taking its first item).
template <int D, bool kF8, bool kAlibi, bool kVarlen>
int fwd_launch(int grid, cudaStream_t stream, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const CUtensorMap& mo, const fa::FwdParams& p) {
  fa::fa_fwd_counter_reset_kernel<<<1, 32, 0, stream>>>(p.counter_slot);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(fa::FwdCfg<D, kF8>::kThreads);
  cfg.dynamicSmemBytes = fa::FwdCfg<D, kF8>::kSmemBytes + (kVarlen ? fa::kFwdSortBytes : 0);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fa::fa_fwd_kernel<D, kF8, kAlibi, kVarlen>, mq, mk, mv, mo, p) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

template <int D>
int fwd_variant(bool alibi, bool varlen, int grid, cudaStream_t stream, const CUtensorMap& mq, const CUtensorMap& mk,
                const CUtensorMap& mv, const CUtensorMap& mo, const fa::FwdParams& p) {
  if (alibi && varlen) return fwd_launch<D, false, true, true>(grid, stream, mq, mk, mv, mo, p);
  if (alibi) return fwd_launch<D, false, true, false>(grid, stream, mq, mk, mv, mo, p);
  if (varlen) return fwd_launch<D, false, false, true>(grid, stream, mq, mk, mv, mo, p);
  return fwd_launch<D, false, false, false>(grid, stream, mq, mk, mv, mo, p);
}

// Pair ranks of the forward's final phase (all heads, shortest last): enough for two items per
// CTA, so that the end of the run is made of short items; all of them when that is more.
int fwd_tail_ranks(const Shape& s, int num_pairs, int sm_count) {
  const int bh = s.B * s.H;
  const int k = (2 * sm_count + bh - 1) / bh;
  return k < num_pairs ? k : num_pairs;
}

// Heads per scheduling group of the forward: as many as keep the K/V of one group within
// 24 MiB (two groups in flight stay well inside L2), at least 1.
int fwd_head_group(const Shape& s, int elem_bytes) {
  const double kv_per_head = 2.0 * s.N * s.d * elem_bytes;
  const double g = (24.0 * 1024 * 1024) / kv_per_head;
  const int bh = s.B * s.H;
  return g < 1.0 ? 1 : (g >= bh ? bh : (int)g);
}

// Offsets of a packed batch: cu[0] = 0, non-decreasing, cu[nseg] = n; a violation is reported
// through fa_check (the kernels clamp every bound, so bad offsets cannot send work out of range).
__global__ void __launch_bounds__(256) fa_check_cu_kernel(const int* cu, int nseg, int n) {
  bool bad = false;
  if (threadIdx.x == 0) bad = cu[0] != 0 || cu[nseg] != n;
  for (int i = threadIdx.x; i < nseg; i += blockDim.x) bad |= cu[i + 1] < cu[i];
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&fa::g_fa_error, fa::kErrBadInput);
}

int launch_check_cu(const int* cu, int nseg, int n, cudaStream_t stream) {
  fa_check_cu_kernel<<<1, 256, 0, stream>>>(cu, nseg, n);
  return launch_status();
}

// alibi != nullptr: (B, H) ALiBi slopes (bf16 inputs).
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const Shape& s, float scale,
               int causal, int win_l, int win_r, int sm_count, cudaStream_t stream,
               int dev, const float* const* descales = nullptr, const float* alibi = nullptr, const int* cu = nullptr,
               int nseg = 0) {
  CUtensorMap mq, mk, mv, mo;
  int st;
  auto in_map = descales ? make_map_u8 : make_map;
  if ((st = in_map(&mq, q, s)) || (st = in_map(&mk, k, s)) || (st = in_map(&mv, v, s)) ||
      (st = make_map(&mo, o, s)))
    return st;
  fa::FwdParams p;
  p.cu_seqlens = cu;
  p.nseg = nseg;
  p.q_descale = descales ? descales[0] : nullptr;
  p.k_descale = descales ? descales[1] : nullptr;
  p.v_descale = descales ? descales[2] : nullptr;
  p.alibi_slopes = alibi;
  p.B = s.B;
  p.N = s.N;
  p.H = s.H;
  p.scale_log2 = scale * fa::kLog2e;
  p.win_l = win_l;
  p.win_r = win_r;
  p.causal = causal ? 1 : 0;
  p.num_pairs = (s.N + 255) / 256;
  p.num_items = s.B * s.H * p.num_pairs;
  p.lse = lse;
  if (cu) {  // packed batch: the cost-sorted pairs in one group (their order already ends short)
    p.head_group = s.B * s.H;
    p.tail_ranks = 0;
  } else {
    p.head_group = fwd_head_group(s, descales ? 1 : 2);
    p.tail_ranks = fwd_tail_ranks(s, p.num_pairs, sm_count);
  }
  p.counter_slot = (int)(g_fwd_slot_seq[dev].fetch_add(1, std::memory_order_relaxed) % fa::kFwdCounterSlots);
  // Test-only fault knob: the forward withholds one internal signal so that a bounded wait in
  // the kernel runs out (it must report FA_ERR_TIMEOUT through fa_check, not hang).
  const char* drop = std::getenv("FA_DEBUG_DROP_S_SIGNAL");
  p.debug_drop_s_signal = (drop && drop[0] == '1') ? 1 : 0;
  const int grid = p.num_items < sm_count ? p.num_items : sm_count;
  if (log_enabled())
    std::fprintf(stderr, "[fa] fwd B=%d N=%d H=%d d=%d causal=%d win=(%d,%d) items=%d grid=%d smem=%d\n", s.B, s.N,
                 s.H, s.d, p.causal, win_l, win_r, p.num_items, grid,
                 s.d == 64 ? fa::FwdCfg<64>::kSmemBytes : fa::FwdCfg<128>::kSmemBytes);
  if (descales)
    st = fwd_launch<128, true, false, false>(grid, stream, mq, mk, mv, mo, p);
  else if (s.d == 64)
    st = fwd_variant<64>(alibi != nullptr, cu != nullptr, grid, stream, mq, mk, mv, mo, p);
  else
    st = fwd_variant<128>(alibi != nullptr, cu != nullptr, grid, stream, mq, mk, mv, mo, p);
  return st ? st : launch_status();
}

int launch_pre(const void* o, const float* lse, const void* dO, const Shape& s, const Workspace& w,
               cudaStream_t stream) {
  const long long rows_per_cta = s.d == 64 ? fa::PreCfg<64>::kRows : fa::PreCfg<128>::kRows;
  const long long blocks = (long long)s.B * s.H * (s.n_pad() / rows_per_cta);
  if (s.d == 64)
    fa::fa_bwd_pre_kernel<64><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, w.lse2, w.dvec, w.dq_acc,
        w.next_item, s.B, s.N, s.H, s.n_pad());
  else
    fa::fa_bwd_pre_kernel<128><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, w.lse2, w.dvec, w.dq_acc,
        w.next_item, s.B, s.N, s.H, s.n_pad());
  return launch_status();
}

// Packed sequences travel with the backward's other options.
struct BwdOptions {
  const float* alibi = nullptr;
  const int* cu = nullptr;
  int nseg = 0;
};

fa::BwdParams bwd_params(const Shape& s, float scale, int causal, int win_l, int win_r, const Workspace& w,
                         const BwdOptions& opt, int sm_count_hint) {
  fa::BwdParams p;
  p.alibi_slopes = opt.alibi;
  p.cu_seqlens = opt.cu;
  p.nseg = opt.nseg;
  p.B = s.B;
  p.N = s.N;
  p.H = s.H;
  p.N_pad = s.n_pad();
  p.scale = scale;
  p.scale_log2 = scale * fa::kLog2e;
  p.win_l = win_l;
  p.win_r = win_r;
  p.causal = causal ? 1 : 0;
  p.num_kv_tiles = (s.N + 127) / 128;
  p.num_items = s.B * s.H * p.num_kv_tiles;
  // Head groups of the main kernel: the Q, dO (bf16) and dQ accumulator (fp32) rows of a group,
  // 8 N d bytes per head, within 32 MiB; the last KV tiles (the shortest under causal masking,
  // enough for four items per CTA) dealt over all heads at the end.
  const double per_head = 8.0 * s.N * s.d;
  const double g = (32.0 * 1024 * 1024) / per_head;
  const int bh = s.B * s.H;
  p.head_group = g < 1.0 ? 1 : (g >= bh ? bh : (int)g);
  const int sms = sm_count_hint > 0 ? sm_count_hint : 148;
  const int k = (4 * sms + bh - 1) / bh;
  p.tail_tiles = k < p.num_kv_tiles ? k : p.num_kv_tiles;
  p.dq_acc = w.dq_acc;
  p.lse2 = w.lse2;
  p.dvec = w.dvec;
  p.next_item = w.next_item;
  return p;
}

template <int D, bool kDQ, bool kAlibi, bool kVarlen>
void main_launch(int grid, cudaStream_t stream, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                 const CUtensorMap& mdo, const CUtensorMap& mdk, const CUtensorMap& mdv, const CUtensorMap& mdq,
                 const fa::BwdParams& p) {
  fa::fa_bwd_kernel<D, kDQ, kAlibi, kVarlen><<<grid, fa::BwdCfg<D>::kThreads, fa::BwdCfg<D>::kSmemBytes, stream>>>(
      mq, mk, mv, mdo, mdk, mdv, mdq, p);
}

template <int D, bool kDQ>
void main_kernel(bool alibi, bool varlen, int grid, cudaStream_t stream, const CUtensorMap& mq, const CUtensorMap& mk,
                 const CUtensorMap& mv, const CUtensorMap& mdo, const CUtensorMap& mdk, const CUtensorMap& mdv,
                 const CUtensorMap& mdq, const fa::BwdParams& p) {
  if (alibi && varlen) main_launch<D, kDQ, true, true>(grid, stream, mq, mk, mv, mdo, mdk, mdv, mdq, p);
  else if (alibi) main_launch<D, kDQ, true, false>(grid, stream, mq, mk, mv, mdo, mdk, mdv, mdq, p);
  else if (varlen) main_launch<D, kDQ, false, true>(grid, stream, mq, mk, mv, mdo, mdk, mdv, mdq, p);
  else main_launch<D, kDQ, false, false>(grid, stream, mq, mk, mv, mdo, mdk, mdv, mdq, p);
}

template <int D, bool kAlibi, bool kVarlen>
void dq_launch(int grid, cudaStream_t stream, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const CUtensorMap& mdo, const CUtensorMap& mdq, const fa::BwdParams& p) {
  fa::fa_bwd_dq_kernel<D, kAlibi, kVarlen><<<grid, fa::BwdDqCfg<D>::kThreads, fa::BwdDqCfg<D>::kSmemBytes, stream>>>(
      mq, mk, mv, mdo, mdq, p);
}

template <int D>
void dq_kernel(bool alibi, bool varlen, int grid, cudaStream_t stream, const CUtensorMap& mq, const CUtensorMap& mk,
               const CUtensorMap& mv, const CUtensorMap& mdo, const CUtensorMap& mdq, const fa::BwdParams& p) {
  if (alibi && varlen) dq_launch<D, true, true>(grid, stream, mq, mk, mv, mdo, mdq, p);
  else if (alibi) dq_launch<D, true, false>(grid, stream, mq, mk, mv, mdo, mdq, p);
  else if (varlen) dq_launch<D, false, true>(grid, stream, mq, mk, mv, mdo, mdq, p);
  else dq_launch<D, false, false>(grid, stream, mq, mk, mv, mdo, mdq, p);
}

// Main backward kernel; with_dq = false computes dK and dV only (the deterministic backward).
int launch_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, const Shape& s,
                float scale, int causal, int win_l, int win_r, const Workspace& w, int sm_count,
                cudaStream_t stream, bool with_dq = true, const BwdOptions& opt = BwdOptions()) {
  CUtensorMap mq, mk, mv, mdo, mdk, mdv, mdq;
  int st;
  if ((st = make_map(&mq, q, s)) || (st = make_map(&mk, k, s)) || (st = make_map(&mv, v, s)) ||
      (st = make_map(&mdo, dO, s)) || (st = make_map(&mdk, dk, s)) || (st = make_map(&mdv, dv, s)) ||
      (st = make_map_f32_acc(&mdq, w.dq_acc, s)))
    return st;
  const fa::BwdParams p = bwd_params(s, scale, causal, win_l, win_r, w, opt, sm_count);
  const int grid = p.num_items < sm_count ? p.num_items : sm_count;
  if (log_enabled())
    std::fprintf(stderr, "[fa] bwd B=%d N=%d H=%d d=%d causal=%d win=(%d,%d) items=%d grid=%d smem=%d\n", s.B, s.N,
                 s.H, s.d, p.causal, win_l, win_r, p.num_items, grid,
                 s.d == 64 ? fa::BwdCfg<64>::kSmemBytes : fa::BwdCfg<128>::kSmemBytes);
  const bool a = opt.alibi != nullptr, vl = opt.cu != nullptr;
  if (s.d == 64 && with_dq)
    main_kernel<64, true>(a, vl, grid, stream, mq, mk, mv, mdo, mdk, mdv, mdq, p);
  else if (s.d == 64)
    main_kernel<64, false>(a, vl, grid, stream, mq, mk, mv, mdo, mdk, mdv, mdq, p);
  else if (with_dq)
    main_kernel<128, true>(a, vl, grid, stream, mq, mk, mv, mdo, mdk, mdv, mdq, p);
  else
    main_kernel<128, false>(a, vl, grid, stream, mq, mk, mv, mdo, mdk, mdv, mdq, p);
  return launch_status();
}

// dQ of the deterministic backward: one item per (b, h, Q tile), dQ accumulated in TMEM.
int launch_dq(const void* q, const void* k, const void* v, const void* dO, void* dq, const Shape& s, float scale,
              int causal, int win_l, int win_r, const Workspace& w, int sm_count, cudaStream_t stream,
              const BwdOptions& opt = BwdOptions()) {
  CUtensorMap mq, mk, mv, mdo, mdq;
  int st;
  if ((st = make_map(&mq, q, s)) || (st = make_map(&mk, k, s)) || (st = make_map(&mv, v, s)) ||
      (st = make_map(&mdo, dO, s)) || (st = make_map(&mdq, dq, s)))
    return st;
  const fa::BwdParams p = bwd_params(s, scale, causal, win_l, win_r, w, opt, sm_count);
  const int grid = p.num_items < sm_count ? p.num_items : sm_count;
  if (s.d == 64)
    dq_kernel<64>(opt.alibi != nullptr, opt.cu != nullptr, grid, stream, mq, mk, mv, mdo, mdq, p);
  else
    dq_kernel<128>(opt.alibi != nullptr, opt.cu != nullptr, grid, stream, mq, mk, mv, mdo, mdq, p);
  return launch_status();
}

int launch_convert(void* dq, const Shape& s, const Workspace& w, cudaStream_t stream) {
  const long long n8 = (long long)(s.elems() / 8);
  const long long blocks = (n8 + 255) / 256;
  fa::fa_dq_convert_kernel<<<(unsigned)blocks, 256, 0, stream>>>(w.dq_acc, static_cast<__nv_bfloat16*>(dq), n8);
  return launch_status();
}

// Common checks of the backward calls: problem, pointers, workspace.
int check_workspace(void* workspace, size_t bytes, const Shape& s) {
  if (!workspace || !aligned(workspace, 256) || bytes < workspace_bytes(s)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

}  // namespace

// ---------------------------------------------------------------- backward without allocation
//
// Scratch for fa_bwd_static_workspace: a fixed array in the library's device image. Host code
// sees only a stand-in symbol; the device address is looked up once per device (with that
// device current) and cached. No cudaMalloc, cudaFree or allocating library call is made.
namespace {
constexpr size_t kStaticWorkspaceBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];
void* g_static_workspace_ptr[kMaxDevices] = {nullptr};

int static_workspace_address(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_static_workspace_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    g_static_workspace_ptr[dev] = p;
  }
  *out = g_static_workspace_ptr[dev];
  return FA_OK;
}
}  // namespace

extern "C" {

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: head dim or device not supported";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA runtime error";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a device-side wait timed out";
    case FA_ERR_NO_MEMORY: return "FA_ERR_NO_MEMORY: workspace allocation failed";
    case FA_ERR_DEVICE: return "FA_ERR_DEVICE: a device-side check failed";
    default: return "FA_ERR_UNKNOWN";
  }
}

size_t fa_bwd_workspace_bytes(int B, int N, int H, int d) {
  int wl = -1, wr = -1;
  if (check_problem(B, N, H, d, 1.0f, 0, &wl, &wr) != FA_OK) return 0;
  return workspace_bytes(Shape{B, N, H, d});
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N, int H, int d, float scale,
           int causal, int win_l, int win_r, fa_stream_t stream) {
  int st = check_problem(B, N, H, d, scale, causal, &win_l, &win_r);
  if (st) return st;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_INVALID_ARG;
  const Shape s{B, N, H, d};
  const size_t tb = s.tensor_bytes(), lb = s.rowvec_bytes();
  if (overlap(o, tb, q, tb) || overlap(o, tb, k, tb) || overlap(o, tb, v, tb) || overlap(lse, lb, q, tb) ||
      overlap(lse, lb, k, tb) || overlap(lse, lb, v, tb) || overlap(lse, lb, o, tb))
    return FA_ERR_INVALID_ARG;
  int dev, sms;
  if ((st = device_setup(&dev, &sms))) return st;
  return launch_fwd(q, k, v, o, lse, s, scale, causal, win_l, win_r, sms, reinterpret_cast<cudaStream_t>(stream),
                    dev);
}

int fa_fwd_ex(const void* q, const void* k, const void* v, const float* alibi_slopes, void* o, float* lse, int B,
              int N, int H, int d, float scale, int causal, int win_l, int win_r, fa_stream_t stream) {
  int st = check_problem(B, N, H, d, scale, causal, &win_l, &win_r);
  if (st) return st;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(alibi_slopes, 4))
    return FA_ERR_INVALID_ARG;
  const Shape s{B, N, H, d};
  const size_t tb = s.tensor_bytes(), lb = s.rowvec_bytes(), ab = (size_t)B * H * 4;
  if (overlap(o, tb, q, tb) || overlap(o, tb, k, tb) || overlap(o, tb, v, tb) || overlap(lse, lb, q, tb) ||
      overlap(lse, lb, k, tb) || overlap(lse, lb, v, tb) || overlap(lse, lb, o, tb))
    return FA_ERR_INVALID_ARG;
  if (alibi_slopes && (overlap(o, tb, alibi_slopes, ab) || overlap(lse, lb, alibi_slopes, ab)))
    return FA_ERR_INVALID_ARG;
  int dev, sms;
  if ((st = device_setup(&dev, &sms))) return st;
  return launch_fwd(q, k, v, o, lse, s, scale, causal, win_l, win_r, sms, reinterpret_cast<cudaStream_t>(stream),
                    dev, nullptr, alibi_slopes);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, const int* cu_seqlens, const float* alibi_slopes,
                  void* o, float* lse, int B, int total, int H, int d, float scale, int causal, int win_l,
                  int win_r, fa_stream_t stream) {
  if (B < 1 || !cu_seqlens || !aligned(cu_seqlens, 4)) return FA_ERR_INVALID_ARG;
  int st = check_problem(1, total, H, d, scale, causal, &win_l, &win_r);
  if (st) return st;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(alibi_slopes, 4))
    return FA_ERR_INVALID_ARG;
  const Shape s{1, total, H, d};
  const size_t tb = s.tensor_bytes(), lb = s.rowvec_bytes(), ab = (size_t)H * 4, cb = (size_t)(B + 1) * 4;
  const void* ins[5] = {q, k, v, cu_seqlens, alibi_slopes};
  const size_t in_bytes[5] = {tb, tb, tb, cb, alibi_slopes ? ab : 0};
  for (int i = 0; i < 5; ++i)
    if (overlap(o, tb, ins[i], in_bytes[i]) || overlap(lse, lb, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
  if (overlap(o, tb, lse, lb)) return FA_ERR_INVALID_ARG;
  int dev, sms;
  if ((st = device_setup(&dev, &sms))) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if ((st = launch_check_cu(cu_seqlens, B, total, cs))) return st;
  return launch_fwd(q, k, v, o, lse, s, scale, causal, win_l, win_r, sms, cs, dev, nullptr, alibi_slopes, cu_seqlens,
                    B);
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, const float* q_descale, const float* k_descale,
               const float* v_descale, void* o, float* lse, int B, int N, int H, int d, float scale, int causal,
               int win_l, int win_r, fa_stream_t stream) {
  int st = check_problem(B, N, H, d, scale, causal, &win_l, &win_r);
  if (st) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !q_descale || !k_descale || !v_descale || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(q_descale, 4) || !aligned(k_descale, 4) || !aligned(v_descale, 4))
    return FA_ERR_INVALID_ARG;
  const Shape s{B, N, H, d};
  const size_t ib = s.elems(), ob = s.tensor_bytes(), lb = s.rowvec_bytes(), db = (size_t)B * H * 4;
  const void* ins[6] = {q, k, v, q_descale, k_descale, v_descale};
  const size_t in_bytes[6] = {ib, ib, ib, db, db, db};
  for (int i = 0; i < 6; ++i)
    if (overlap(o, ob, ins[i], in_bytes[i]) || overlap(lse, lb, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
  if (overlap(o, ob, lse, lb)) return FA_ERR_INVALID_ARG;
  int dev, sms;
  if ((st = device_setup(&dev, &sms))) return st;
  const float* descales[3] = {q_descale, k_descale, v_descale};
  return launch_fwd(q, k, v, o, lse, s, scale, causal, win_l, win_r, sms, reinterpret_cast<cudaStream_t>(stream),
                    dev, descales);
}

}  // extern "C"

namespace {

// The decode kernel, compiled for up to 4 or up to 8 new rows, launched as the programmatic
// dependent of the kernel before it on the stream (the prep kernel, when there are splits).
template <int D>
int launch_decode(dim3 grid, const CUtensorMap& mk, const CUtensorMap& mv, const fa::DecParams& p,
                  cudaStream_t cs) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(fa::kDecMmaThreads);
  cfg.dynamicSmemBytes = fa::DecTcCfg<D>::kSmemBytes;
  cfg.stream = cs;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = p.Sq <= 4 ? cudaLaunchKernelEx(&cfg, fa::fa_decode_kernel<D, 4>, mk, mv, p)
                                  : cudaLaunchKernelEx(&cfg, fa::fa_decode_kernel<D, 8>, mk, mv, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  return launch_status();
}

// Workspace of a call with P > 1 pieces per head: partial O (fp32) and partial LSE for the
// B + P - 1 (sequence, piece) slots, one arrival counter per (b, h).
size_t decode_workspace_bytes(int B, int Sq, int H, int d, int pieces) {
  if (pieces <= 1) return 0;
  const size_t rows = ((size_t)B + pieces - 1) * H * Sq;
  return align256(rows * d * 4) + align256(rows * 4) + align256((size_t)B * H * 4);
}

// CTAs of the decode kernel that fit on one SM at a time (0 on error).
template <int D>
int decode_ctas_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fa::fa_decode_kernel<D, 8>, fa::kDecMmaThreads,
                                                    fa::DecTcCfg<D>::kSmemBytes) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Pieces per head when the caller passes 0: as many as fill every CTA slot of the GPU once
// (H x P <= resident CTAs), at least 1, no more than the batch can have tiles, at most 65535.
int decode_auto_pieces(int B, int Sq, int H, int d, int max_keys, int sm_count) {
  const int per_sm = d == 64 ? decode_ctas_per_sm<64>() : decode_ctas_per_sm<128>();
  long long pieces = (long long)std::max(per_sm, 1) * sm_count / H;
  const long long tiles = (long long)B * ((max_keys + fa::kDecTile - 1) / fa::kDecTile);
  pieces = std::min(pieces, std::min(tiles, 65535LL));
  return pieces < 1 ? 1 : (int)pieces;
}

}  // namespace

extern "C" {

int fa_decode_splits(int B, int Sq, int H, int d, int max_keys) {
  if (B < 1 || Sq < 1 || H < 1 || max_keys < 1 || d < 1) return -FA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || Sq > fa::kDecMaxSq) return -FA_ERR_UNSUPPORTED;
  int dev, sms, st;
  if ((st = device_setup(&dev, &sms))) return -st;
  return decode_auto_pieces(B, Sq, H, d, max_keys, sms);
}

size_t fa_decode_workspace_bytes(int B, int Sq, int H, int d, int splits) {
  if (B < 1 || Sq < 1 || H < 1 || (d != 64 && d != 128) || splits < 0) return 0;
  return decode_workspace_bytes(B, Sq, H, d, splits);
}

int fa_decode_paged(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                    const int* block_table, const int* seqlens, void* o, float* lse, int B, int Sq, int H, int d,
                    int num_pages,
                    int page_size, int max_pages, float scale, int causal, int win_l, int win_r, int splits,
                    void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  if (B < 1 || H < 1 || Sq < 1 || num_pages < 1 || max_pages < 1 || page_size < 1 || splits < 0)
    return FA_ERR_INVALID_ARG;
  if (win_l < -1 || win_r < -1 || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Sq > fa::kDecMaxSq || page_size % fa::kDecTile != 0) return FA_ERR_UNSUPPORTED;
  if ((double)num_pages * page_size * H * d * 2 >= 1099511627776.0 ||
      (double)max_pages * page_size >= 2147483647.0)
    return FA_ERR_INVALID_ARG;
  if (splits > 65535 || (long long)B * H >= 2147483647LL) return FA_ERR_INVALID_ARG;  // grid and counter limits
  if (!q || !k_cache || !v_cache || !block_table || !seqlens || !o || !lse) return FA_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(block_table, 4) || !aligned(seqlens, 4) || !aligned(k_new, 16) || !aligned(v_new, 16))
    return FA_ERR_INVALID_ARG;
  if (causal) win_r = 0;
  const size_t qb = (size_t)B * Sq * H * d * 2, cb = (size_t)num_pages * page_size * H * d * 2;
  const size_t lb = (size_t)B * H * Sq * 4, tb = (size_t)B * max_pages * 4, sb = (size_t)B * 4;
  const void* ins[7] = {q, k_cache, v_cache, block_table, seqlens, k_new, v_new};
  const size_t in_bytes[7] = {qb, cb, cb, tb, sb, k_new ? qb : 0, v_new ? qb : 0};
  for (int i = 0; i < 7; ++i)
    if (overlap(o, qb, ins[i], in_bytes[i]) || overlap(lse, lb, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
  if (overlap(o, qb, lse, lb) || overlap(k_cache, cb, v_cache, cb)) return FA_ERR_INVALID_ARG;
  for (int i = 0; i < 7; ++i)  // the caches are written when new rows are given: nothing may alias them
    if (k_new && i != 1 && i != 2 &&
        (overlap(k_cache, cb, ins[i], in_bytes[i]) || overlap(v_cache, cb, ins[i], in_bytes[i])))
      return FA_ERR_INVALID_ARG;
  int dev, sms, st;
  if ((st = device_setup(&dev, &sms))) return st;
  if (splits == 0) splits = decode_auto_pieces(B, Sq, H, d, max_pages * page_size, sms);
  const size_t wbytes = decode_workspace_bytes(B, Sq, H, d, splits);
  if (wbytes > 0 && workspace) {
    if (!aligned(workspace, 256) || workspace_bytes_ < wbytes) return FA_ERR_INVALID_ARG;
    for (int i = 0; i < 7; ++i)
      if (overlap(workspace, wbytes, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
    if (overlap(workspace, wbytes, o, qb) || overlap(workspace, wbytes, lse, lb)) return FA_ERR_INVALID_ARG;
  }
  CUtensorMap mk, mv;
  if ((st = make_map_cache(&mk, k_cache, num_pages, page_size, H, d)) ||
      (st = make_map_cache(&mv, v_cache, num_pages, page_size, H, d)))
    return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  void* ws = workspace;
  if (wbytes > 0 && !ws) {
    if (cudaMallocAsync(&ws, wbytes, cs) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_NO_MEMORY;
    }
  }
  fa::DecParams p;
  p.B = B;
  p.Sq = Sq;
  p.H = H;
  p.page_size = page_size;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.scale_log2 = scale * fa::kLog2e;
  p.win_l = win_l;
  p.win_r = win_r;
  p.pieces = splits;
  p.block_table = block_table;
  p.seqlens = seqlens;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.o_part = static_cast<float*>(ws);
  const size_t part_rows = ((size_t)B + splits - 1) * H * Sq;  // (sequence, piece) slots
  const size_t part_bytes = align256(part_rows * d * 4);
  const size_t lse_part_bytes = align256(part_rows * 4);
  p.lse_part = wbytes ? reinterpret_cast<float*>(static_cast<char*>(ws) + part_bytes) : nullptr;
  p.arrivals = wbytes ? reinterpret_cast<int*>(static_cast<char*>(ws) + part_bytes + lse_part_bytes) : nullptr;
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  st = FA_OK;
  if (splits > 1) {
    const int count = B * H;
    const int blocks = (int)std::min<long long>((count + 255) / 256, sms);
    fa::fa_decode_prep_kernel<<<blocks, 256, 0, cs>>>(p.arrivals, count);
    st = launch_status();
  }
  if (!st) {
    const dim3 grid(H, splits);  // heads fastest: concurrent CTAs share cache rows
    if (d == 64)
      st = launch_decode<64>(grid, mk, mv, p, cs);
    else
      st = launch_decode<128>(grid, mk, mv, p, cs);
  }
  if (wbytes > 0 && !workspace && cudaFreeAsync(ws, cs) != cudaSuccess && !st) st = FA_ERR_CUDA;
  return st;
}

int fa_bwd_preprocess(const void* o, const float* lse, const void* dO, int B, int N, int H, int d, void* workspace,
                      size_t workspace_bytes_, fa_stream_t stream) {
  int wl = -1, wr = -1;
  int st = check_problem(B, N, H, d, 1.0f, 0, &wl, &wr);
  if (st) return st;
  const Shape s{B, N, H, d};
  if (!o || !lse || !dO || !aligned(o, 16) || !aligned(dO, 16) || !aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  if ((st = check_workspace(workspace, workspace_bytes_, s))) return st;
  const size_t tb = s.tensor_bytes(), wb = workspace_bytes(s), lb = s.rowvec_bytes();
  if (overlap(workspace, wb, o, tb) || overlap(workspace, wb, dO, tb) || overlap(workspace, wb, lse, lb))
    return FA_ERR_INVALID_ARG;
  int dev, sms;
  if ((st = device_setup(&dev, &sms))) return st;
  return launch_pre(o, lse, dO, s, carve(workspace, s), reinterpret_cast<cudaStream_t>(stream));
}

int fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, int B, int N, int H,
                int d, float scale, int causal, int win_l, int win_r, void* workspace, size_t workspace_bytes_,
                fa_stream_t stream) {
  int st = check_problem(B, N, H, d, scale, causal, &win_l, &win_r);
  if (st) return st;
  const Shape s{B, N, H, d};
  if (!q || !k || !v || !dO || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dO, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16))
    return FA_ERR_INVALID_ARG;
  if ((st = check_workspace(workspace, workspace_bytes_, s))) return st;
  const size_t tb = s.tensor_bytes(), wb = workspace_bytes(s);
  const void* ins[4] = {q, k, v, dO};
  for (const void* in : ins)
    if (overlap(dk, tb, in, tb) || overlap(dv, tb, in, tb) || overlap(workspace, wb, in, tb)) return FA_ERR_INVALID_ARG;
  if (overlap(dk, tb, dv, tb) || overlap(workspace, wb, dk, tb) || overlap(workspace, wb, dv, tb))
    return FA_ERR_INVALID_ARG;
  int dev, sms;
  if ((st = device_setup(&dev, &sms))) return st;
  return launch_main(q, k, v, dO, dk, dv, s, scale, causal, win_l, win_r, carve(workspace, s), sms,
                     reinterpret_cast<cudaStream_t>(stream));
}

int fa_bwd_dq_convert(void* dq, int B, int N, int H, int d, void* workspace, size_t workspace_bytes_,
                      fa_stream_t stream) {
  int wl = -1, wr = -1;
  int st = check_problem(B, N, H, d, 1.0f, 0, &wl, &wr);
  if (st) return st;
  const Shape s{B, N, H, d};
  if (!dq || !aligned(dq, 16)) return FA_ERR_INVALID_ARG;
  if ((st = check_workspace(workspace, workspace_bytes_, s))) return st;
  if (overlap(workspace, workspace_bytes(s), dq, s.tensor_bytes())) return FA_ERR_INVALID_ARG;
  int dev, sms;
  if ((st = device_setup(&dev, &sms))) return st;
  return launch_convert(dq, s, carve(workspace, s), reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                    void* dq, void* dk, void* dv, int B, int N, int H, int d, float scale, int causal, int win_l,
                    int win_r, void* workspace, size_t workspace_bytes_, fa_stream_t stream, bool deterministic,
                    const float* alibi = nullptr, const int* cu = nullptr, int nseg = 0) {
  int st = check_problem(B, N, H, d, scale, causal, &win_l, &win_r);
  if (st) return st;
  const Shape s{B, N, H, d};
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  const void* ptrs[8] = {q, k, v, o, dO, dq, dk, dv};
  for (const void* x : ptrs)
    if (!aligned(x, 16)) return FA_ERR_INVALID_ARG;
  if (!aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  const size_t tb = s.tensor_bytes(), lb = s.rowvec_bytes();
  const void* ins[5] = {q, k, v, o, dO};
  void* outs[3] = {dq, dk, dv};
  for (void* out : outs) {
    for (const void* in : ins)
      if (overlap(out, tb, in, tb)) return FA_ERR_INVALID_ARG;
    if (overlap(out, tb, lse, lb)) return FA_ERR_INVALID_ARG;
  }
  if (overlap(dq, tb, dk, tb) || overlap(dq, tb, dv, tb) || overlap(dk, tb, dv, tb)) return FA_ERR_INVALID_ARG;
  if (alibi) {
    if (!aligned(alibi, 4)) return FA_ERR_INVALID_ARG;
    for (void* out : outs)
      if (overlap(out, tb, alibi, (size_t)B * H * 4)) return FA_ERR_INVALID_ARG;
  }
  if (workspace) {
    if ((st = check_workspace(workspace, workspace_bytes_, s))) return st;
    if (alibi && overlap(workspace, workspace_bytes(s), alibi, (size_t)B * H * 4)) return FA_ERR_INVALID_ARG;
    const size_t wb = workspace_bytes(s);
    for (const void* in : ins)
      if (overlap(workspace, wb, in, tb)) return FA_ERR_INVALID_ARG;
    for (void* out : outs)
      if (overlap(workspace, wb, out, tb)) return FA_ERR_INVALID_ARG;
    if (overlap(workspace, wb, lse, lb)) return FA_ERR_INVALID_ARG;
  }
  int dev, sms;
  if ((st = device_setup(&dev, &sms))) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  void* ws = workspace;
  const size_t wbytes = workspace_bytes(s);
  if (!ws) {
    if (cudaMallocAsync(&ws, wbytes, cs) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_NO_MEMORY;
    }
  }
  const Workspace w = carve(ws, s);
  st = launch_pre(o, lse, dO, s, w, cs);
  BwdOptions opt;
  opt.alibi = alibi;
  opt.cu = cu;
  opt.nseg = nseg;
  if (!st && cu) st = launch_check_cu(cu, nseg, N, cs);
  if (deterministic) {
    if (!st) st = launch_main(q, k, v, dO, dk, dv, s, scale, causal, win_l, win_r, w, sms, cs, false, opt);
    if (!st) st = launch_dq(q, k, v, dO, dq, s, scale, causal, win_l, win_r, w, sms, cs, opt);
  } else {
    if (!st) st = launch_main(q, k, v, dO, dk, dv, s, scale, causal, win_l, win_r, w, sms, cs, true, opt);
    if (!st) st = launch_convert(dq, s, w, cs);
  }
  if (!workspace && cudaFreeAsync(ws, cs) != cudaSuccess && !st) st = FA_ERR_CUDA;
  return st;
}

extern "C" {

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, void* dq,
           void* dk, void* dv, int B, int N, int H, int d, float scale, int causal, int win_l, int win_r,
           void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, N, H, d, scale, causal, win_l, win_r, workspace,
                  workspace_bytes_, stream, false);
}

int fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
              const float* alibi_slopes, void* dq, void* dk, void* dv, int B, int N, int H, int d, float scale,
              int causal, int win_l, int win_r, int deterministic, void* workspace, size_t workspace_bytes_,
              fa_stream_t stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, N, H, d, scale, causal, win_l, win_r, workspace,
                  workspace_bytes_, stream, deterministic != 0, alibi_slopes);
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                  const int* cu_seqlens, const float* alibi_slopes, void* dq, void* dk, void* dv, int B, int total,
                  int H, int d, float scale, int causal, int win_l, int win_r, int deterministic, void* workspace,
                  size_t workspace_bytes_, fa_stream_t stream) {
  if (B < 1 || !cu_seqlens || !aligned(cu_seqlens, 4)) return FA_ERR_INVALID_ARG;
  const size_t tb = (size_t)total * H * d * 2, cb = (size_t)(B + 1) * 4;
  void* outs[3] = {dq, dk, dv};
  for (void* out : outs)
    if (out && total > 0 && H > 0 && d > 0 && overlap(out, tb, cu_seqlens, cb)) return FA_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, 1, total, H, d, scale, causal, win_l, win_r, workspace,
                  workspace_bytes_, stream, deterministic != 0, alibi_slopes, cu_seqlens, B);
}

int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, int B, int N, int H, int d, float scale,
                         int causal, int win_l, int win_r, void* workspace, size_t workspace_bytes_,
                         fa_stream_t stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, N, H, d, scale, causal, win_l, win_r, workspace,
                  workspace_bytes_, stream, true);
}

int fa_bwd_static_workspace(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dO, void* dq, void* dk, void* dv, int B, int N, int H, int d, float scale,
                            int causal, int win_l, int win_r, fa_stream_t stream) {
  int st = check_problem(B, N, H, d, scale, causal, &win_l, &win_r);
  if (st) return st;
  const Shape s{B, N, H, d};
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  const void* ptrs[8] = {q, k, v, o, dO, dq, dk, dv};
  for (const void* x : ptrs)
    if (!aligned(x, 16)) return FA_ERR_INVALID_ARG;
  if (!aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  const size_t tb = s.tensor_bytes(), lb = s.rowvec_bytes();
  const void* ins[5] = {q, k, v, o, dO};
  void* outs[3] = {dq, dk, dv};
  for (void* out : outs) {
    for (const void* in : ins)
      if (overlap(out, tb, in, tb)) return FA_ERR_INVALID_ARG;
    if (overlap(out, tb, lse, lb)) return FA_ERR_INVALID_ARG;
  }
  if (overlap(dq, tb, dk, tb) || overlap(dq, tb, dv, tb) || overlap(dk, tb, dv, tb)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes(s) > kStaticWorkspaceBytes) return FA_ERR_UNSUPPORTED;
  int dev, sms;
  if ((st = device_setup(&dev, &sms))) return st;
  void* ws = nullptr;
  if ((st = static_workspace_address(dev, &ws))) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const Workspace w = carve(ws, s);  // the preprocess launch zeroes dQ and rewrites LSE2 / D
  st = launch_pre(o, lse, dO, s, w, cs);
  if (!st) st = launch_main(q, k, v, dO, dk, dv, s, scale, causal, win_l, win_r, w, sms, cs);
  if (!st) st = launch_convert(dq, s, w, cs);
  return st;
}

int fa_check(fa_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int err = 0;
  if (cudaMemcpyFromSymbol(&err, fa::g_fa_error, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (err == 0) return FA_OK;
  const int zero = 0;
  if (cudaMemcpyToSymbol(fa::g_fa_error, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  return (err & fa::kErrWaitTimeout) ? FA_ERR_TIMEOUT : FA_ERR_DEVICE;
}

}  // extern "C"
