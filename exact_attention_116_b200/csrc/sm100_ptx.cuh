// Device primitives for sm_100a written as inline PTX: mbarriers, TMA (tiled loads
// and stores, 1-D bulk copies; never the .multicast::cluster forms), tcgen05 MMA
// with TMEM accumulators, TMEM allocation and loads/stores, and the shared-memory
// matrix / instruction descriptors the MMA reads.
//
// Every wait is bounded: after FA_WAIT_TIMEOUT_NS of polling it records an error
// code in the device error word and returns false, so that no kernel can hang.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#ifndef FA_WAIT_TIMEOUT_NS
#define FA_WAIT_TIMEOUT_NS 2000000000ull  // 2 s
#endif

namespace fa {

// Device-side error word (one per loaded module, per device). Written with atomicOr; read and
// cleared by the host. The library is a single translation unit, so it is defined here.
__device__ int g_fa_error = 0;

constexpr float kLog2e = 1.4426950408889634074f;

// Packed variable-length batches: sequence b holds rows [cu[b], cu[b+1]) of the token axis.
// seg_of returns the sequence of `row` (the largest b < nseg with cu[b] <= row); seg_bounds
// gives its first and last row, clamped into [0, n - 1] so that malformed offsets (reported
// separately) can only shrink the work, never send it out of range.
__device__ __forceinline__ int seg_of(const int* cu, int nseg, int row) {
  int lo = 0, hi = nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= row) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void seg_bounds(const int* cu, int nseg, int n, int row, int& first, int& last) {
  const int s = seg_of(cu, nseg, row);
  first = min(max(__ldg(cu + s), 0), n - 1);
  last = min(max(__ldg(cu + s + 1) - 1, 0), n - 1);
}

enum DeviceError : int {
  kErrWaitTimeout = 1,  // a bounded mbarrier wait gave up
  kErrSmemAlign = 2,    // dynamic shared memory not at the alignment a kernel's layout needs
  kErrBadInput = 4,     // a device-resident argument (sequence length, page index) out of range
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared abort flag of a CTA: once any wait times out, every later wait returns at once.
struct Abort {
  volatile int* flag;  // in shared memory
  __device__ __forceinline__ bool raised() const { return *flag != 0; }
};

// ------------------------------------------------------------------ bounds checks (FA_DEBUG builds)
//
// Built with -DFA_DEBUG=1, the kernels check every computed TMA coordinate, bulk-copy range,
// shared-memory destination and global index before using it. A failed check records
// kErrBadInput in the device error word, raises the CTA's abort flag (so that its waits return
// at once and its roles run out their loops) and skips the access; it never traps. In other
// builds the checks are constant true and compile away. They stand in for a memory checker.
#ifndef FA_DEBUG
#define FA_DEBUG 0
#endif

__device__ __forceinline__ bool dbg_fail(Abort ab) {
  if (ab.flag) *ab.flag = 1;
  atomicOr(&g_fa_error, kErrBadInput);
  return false;
}

// The box of a tiled TMA copy starts inside the tensor (c0 on a 16-byte boundary of elements of
// `elem` bytes, 0 <= c_k < e_k) and its `bytes` in shared memory lie in [lo, hi).
__device__ __forceinline__ bool dbg_tma(Abort ab, int c0, int c1, int c2, int c3, int e0, int e1, int e2, int e3,
                                        int elem, uint32_t dst, uint32_t bytes, uint32_t lo, uint32_t hi) {
  if (!FA_DEBUG) return true;
  const bool ok = c0 >= 0 && c0 < e0 && (c0 * elem) % 16 == 0 && c1 >= 0 && c1 < e1 && c2 >= 0 && c2 < e2 &&
                  c3 >= 0 && c3 < e3 && dst >= lo && dst + bytes <= hi && (dst & 15u) == 0;
  return ok || dbg_fail(ab);
}

// A plain index or element range [first, first + count) inside [0, size).
__device__ __forceinline__ bool dbg_range(Abort ab, long long first, long long count, long long size) {
  if (!FA_DEBUG) return true;
  const bool ok = first >= 0 && count >= 0 && first + count <= size;
  return ok || dbg_fail(ab);
}

// Wait until the phase with the given parity has completed. Returns false on timeout
// or when another role of the CTA has already given up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, Abort ab) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (ab.raised()) return false;
      if (global_timer_ns() - t0 > FA_WAIT_TIMEOUT_NS) break;
    }
  }
  *ab.flag = 1;
  atomicOr(&g_fa_error, kErrWaitTimeout);
  return false;
}

// Wait on the work-item ring: it ignores the abort flag and allows twice the usual time. Every
// consumer of an item then decides from the same published value whether to stop, whatever the
// abort flag reads at the moment it looks, so warps that meet at named barriers (which cannot
// time out) take the same items; and the producer overwrites a slot only after every consumer
// has read it, abort or not (the consumers keep fetching, since their other waits return at
// once after an abort). Once the flag is raised the producer publishes stop items, well within
// this limit. Returns false (and raises the flag) if the phase did not complete in time: a
// role has stopped for good.
__device__ __forceinline__ bool mbar_wait_ring(uint32_t bar, uint32_t parity, Abort ab) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0 && global_timer_ns() - t0 > 2 * FA_WAIT_TIMEOUT_NS) break;
  }
  *ab.flag = 1;
  atomicOr(&g_fa_error, kErrWaitTimeout);
  return false;
}

// Bounded wait that ignores the abort flag: used to drain copies already in flight.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return;
    if ((it & 63u) == 0 && global_timer_ns() - t0 > FA_WAIT_TIMEOUT_NS) {
      atomicOr(&g_fa_error, kErrWaitTimeout);
      return;
    }
  }
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ TMA / bulk copies

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// Tiled 4-D load global -> shared, completion counted in bytes on `bar`.
// Coordinates are element indices, innermost first; c0 * elem_size must be a multiple of 16.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Tiled 4-D store shared -> global (rows outside the tensor are clipped by the TMA unit).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* m, uint32_t src, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// Tiled 4-D reduction shared -> global: the TMA unit adds the box into global memory (the
// element type and the add come from the tensor map; rows outside the tensor are clipped).
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* m, uint32_t src, int c0, int c1, int c2,
                                                  int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Untiled bulk copy global -> shared; both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the async proxy
// (TMA stores and tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05: TMEM

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM address: lane in bits [31:16], column in bits [15:0].
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

#define FA_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), \
                 "=r"(r[i + 6]), "=r"(r[i + 7])
#define FA_P8(i) "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]), \
                 "+r"(r[i + 6]), "+r"(r[i + 7])
#define FA_I8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), "r"(r[i + 5]), \
                 "r"(r[i + 6]), "r"(r[i + 7])

// Warp-collective load: thread t of the warp reads TMEM lane (lane field of taddr) + t,
// 32 consecutive 32-bit columns starting at the column field of taddr.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24)
      : "r"(taddr));
}

// Wait for this thread's TMEM loads; the registers pass through so no use is hoisted above it.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : FA_P8(0), FA_P8(8), FA_P8(16), FA_P8(24)::"memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Warp-collective store of 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      FA_I8(0), FA_I8(8)
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), FA_I8(0)
               : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      FA_I8(0), FA_I8(8), FA_I8(16), FA_I8(24)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#undef FA_R8
#undef FA_P8
#undef FA_I8

// ------------------------------------------------------------------ tcgen05: MMA

// Instruction descriptor for kind::f16 with bf16 A/B and an fp32 accumulator.
// Bits: [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format,
// 15 A major (0 = K, 1 = MN), 16 B major, [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Instruction descriptor, kind::f8f6f4 with E4M3 A and B, FP32 accumulate: [4,6) D format
// (1 = F32), [7,10) A format and [10,13) B format (0 = E4M3), the rest as for kind::f16.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(uint32_t M, uint32_t N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) | ((N >> 3) << 17) |
         ((M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 layout:
// [0,14) start >> 4, [16,30) leading byte offset >> 4, [32,46) stride byte offset >> 4,
// [46,48) version = 1, [61,64) layout = 2 (SWIZZLE_128B). Tiles are 1024-byte aligned.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// K-major operand: rows of 128 bytes (64 bf16 along K), 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_kmajor(uint32_t saddr) { return sdesc_sw128(saddr, 16, 1024); }

// MN-major operand: 64 bf16 along M/N per 128-byte row, K rows 128 bytes apart,
// 8-row K groups 1024 bytes apart, consecutive 64-wide M/N chunks `mn_chunk_bytes` apart.
__device__ __forceinline__ uint64_t sdesc_mnmajor(uint32_t saddr, uint32_t mn_chunk_bytes) {
  return sdesc_sw128(saddr, mn_chunk_bytes, 1024);
}

// D[tmem] (+)= A[smem] * B[smem]^T-style product (operand majors in idesc).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Same with A read from TMEM (K-major, two bf16 per 32-bit column).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// kind::f8f6f4 forms (8-bit operands, 32 K-elements per instruction; from TMEM, four per column).
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// ------------------------------------------------------------------ math helpers

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA and integer pipes, to take load off the MUFU unit that ex2.approx uses.
// Cody-Waite split x = j + f with j = round(x) and |f| <= 1/2 (adding 1.5 * 2^23 rounds x to
// an integer held in the low mantissa bits), a degree-3 minimax polynomial for 2^f on
// [-1/2, 1/2] (coefficients fitted by csrc/fit_exp2_poly.py, max relative error 7.5e-5), and
// j added to the exponent field of the polynomial's value. The reduction runs on x clamped at
// -125 (so that 2^j p(f) stays a normal float), and for x < -125, -inf included, the result is
// exactly 0: a masked score (-inf) must carry no weight, as 2^-inf = 0 does on MUFU.
constexpr float kExp2C0 = 9.999280572e-01f;
constexpr float kExp2C1 = 6.932608485e-01f;
constexpr float kExp2C2 = 2.426111549e-01f;
constexpr float kExp2C3 = 5.517221987e-02f;

__device__ __forceinline__ float exp2_poly(float x_in) {
  const float x = fmaxf(x_in, -125.0f);
  const float t = x + 12582912.0f;
  const float f = x - (t - 12582912.0f);
  float p = fmaf(kExp2C3, f, kExp2C2);
  p = fmaf(p, f, kExp2C1);
  p = fmaf(p, f, kExp2C0);
  const float r = __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
  return x_in >= -125.0f ? r : 0.0f;
}

// Packed fp32 pair arithmetic of sm_100 (one instruction for two lanes of a float2) and the
// three-input maximum.
__device__ __forceinline__ uint64_t f2_bits(float2 v) { return *reinterpret_cast<const uint64_t*>(&v); }
__device__ __forceinline__ float2 bits_f2(uint64_t v) { return *reinterpret_cast<const float2*>(&v); }

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return bits_f2(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// exp2_poly on a pair, with the same operations as the scalar version done as packed pairs.
__device__ __forceinline__ float2 exp2_poly2(float2 x_in) {
  const float2 x = make_float2(fmaxf(x_in.x, -125.0f), fmaxf(x_in.y, -125.0f));
  const float2 t = add2(x, make_float2(12582912.0f, 12582912.0f));
  const float2 jf = add2(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = fma2(jf, make_float2(-1.0f, -1.0f), x);
  float2 p = fma2(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  p = fma2(p, f, make_float2(kExp2C1, kExp2C1));
  p = fma2(p, f, make_float2(kExp2C0, kExp2C0));
  const float rx = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
  const float ry = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
  return make_float2(x_in.x >= -125.0f ? rx : 0.0f, x_in.y >= -125.0f ? ry : 0.0f);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Four floats -> E4M3 (round to nearest even, saturating to +-448), x0 in the lowest byte.
// cvt ...e4m3x2.f32 d, a, b puts a in the upper byte of d and b in the lower.
__device__ __forceinline__ uint32_t pack_e4m3x4(float x0, float x1, float x2, float x3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(x1), "f"(x0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(x3), "f"(x2));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

// acc.x += low bf16 of v, acc.y += high bf16 of v: sm_100's mixed-precision add (the bf16
// operand is widened exactly), so a packed pair is summed without unpacking it first.
__device__ __forceinline__ float2 add_bf16x2_f32x2(uint32_t v, float2 acc) {
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.bf16 %0, lo, %0;\n\t"
      "add.rn.f32.bf16 %1, hi, %1;\n\t}"
      : "+f"(acc.x), "+f"(acc.y)
      : "r"(v));
  return acc;
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a 128B-swizzled tile whose
// rows are 128 bytes: the chunk index is XORed with the row index modulo 8.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void red_add_v4_f32(float* gptr, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(gptr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// Programmatic dependent launch: let the next kernel on the stream (launched with the
// programmatic-serialization attribute) start, and, in that kernel, wait until the grids it
// depends on have finished and their writes are visible. The wait returns at once in a
// kernel launched without the attribute.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace fa
