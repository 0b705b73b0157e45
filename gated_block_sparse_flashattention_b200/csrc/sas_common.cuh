// Shared device helpers for the SAS sm_100a kernels: status word, bounded
// mbarrier waits, TMA tensor copies, tcgen05 (TMEM / UMMA) wrappers and the
// shared-memory matrix descriptors the tensor cores read.
//
// Every wait on an mbarrier is bounded in time. When a bound expires the
// waiting thread records SAS_DEV_ERR_TIMEOUT in the launch's status word and
// the kernel winds down instead of spinning forever.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sas {

constexpr int kBlock = 64;                       // tokens per KV block (SAS paper §5.1)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device status codes, written to the status word in the caller's workspace.
enum DeviceStatus : int32_t { SAS_DEV_OK = 0, SAS_DEV_ERR_TIMEOUT = 1, SAS_DEV_ERR_BOUNDS = 2 };

// Default wall-clock limit for one mbarrier wait (nanoseconds). Legitimate waits
// inside these kernels last microseconds; one second means something is broken.
// Kernels that take a limit as a parameter get it from sas_set_wait_limit_ns().
constexpr uint64_t kWaitLimitNs = 1000000000ull;
// Limit for waits while winding down: copies and MMAs already issued finish in
// microseconds, so a few milliseconds bound a kernel that is aborting.
constexpr uint64_t kDrainLimitNs = 20000000ull;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Raise the expected transaction bytes of the current phase without arriving.
__device__ __forceinline__ void mbar_add_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking check of a phase (never suspends the thread): for polling loops
// that watch several barriers at once.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed. Returns false (and
// records a timeout) when the wait exceeds limit_ns or another thread of the
// launch has already recorded an error.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* status,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (it == 1u || (it & 255u) == 0u) {   // the first check early: a tiny test limit trips at once
      if (*reinterpret_cast<volatile int32_t*>(status) != 0) return false;
      if (global_ns() - t0 > limit_ns) {
        set_status(status, SAS_DEV_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// mbar_wait taken by a whole warp: true only if every lane's wait succeeded,
// so warp-collective tcgen05 instructions that follow stay convergent.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int32_t* status,
                                          uint64_t limit_ns = kWaitLimitNs) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, status, limit_ns));
}

// Wait used only while winding down (copies or MMAs still in flight): ignores
// the status word, gives up after kDrainLimitNs.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kDrainLimitNs) return;
  }
}

// Named barrier over a subset of the CTA's warps (id 1..15; count = threads).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier that also ANDs a predicate over the participating threads:
// every thread returns the same value.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 4-byte global -> shared copy (cp.async through L1).
__device__ __forceinline__ void cp_async4(uint32_t dst_smem, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst_smem), "l"(src) : "memory");
}

// 16-byte global -> shared copy (cp.async, L2 only), and its group wait.
__device__ __forceinline__ void cp_async16(uint32_t dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst_smem), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// Wait until at most N of this thread's most recent cp.async groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]; kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]; A in TMEM is K-major: lane = row, 32-bit
// column c holds the bf16 pair (2c, 2c+1) of the K dimension.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

// Arrive once on the mbarrier when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// TMEM address of (lane, column): lane in bits [31:16], column in bits [15:0].
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

// ------------------------------------------------------------------ UMMA descriptors
// Shared-memory matrix descriptor (sm_100 format): start address >> 4 in bits
// [0,14), leading byte offset >> 4 in [16,30), stride byte offset >> 4 in
// [32,46), descriptor version 1 in [46,48), base offset 0, layout type in
// [61,64) with 2 = 128-byte swizzle.
//
// Tiles here use the 128-byte swizzle: rows of 128 bytes (64 bf16), eight rows
// per 1024-byte swizzle atom, the 16-byte chunk index XOR-ed with (row % 8).
//  * K-major operand (rows of the M/N dimension, K contiguous): SBO = 1024
//    (next group of 8 rows); LBO unused (set to 1).
//  * MN-major operand (M/N contiguous, rows of the K dimension): LBO = byte
//    distance between consecutive 64-element M/N chunks, SBO = 1024 (next group
//    of 8 K-rows).
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;   // version
  d |= (uint64_t)2u << 61;   // 128-byte swizzle
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulate.
// c_format (F32 = 1) in bits [4,6), a_format (BF16 = 1) [7,10), b_format [10,13),
// a_major [15], b_major [16] (0 = K-major, 1 = MN-major), N >> 3 in [17,23),
// M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Fire-and-forget fp32 vector reduction into global memory (no return value, no wait).
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void red_add_v2(float* addr, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(addr), "f"(a), "f"(b) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// ------------------------------------------------------------------ small math
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Order-preserving map of a float to uint32 (larger float -> larger key), with
// -0.0 mapped to the key of +0.0 so signed zeros tie.
__device__ __forceinline__ uint32_t float_key(float v) {
  uint32_t u = __float_as_uint(v);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// 128-byte swizzle: byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a tile of 128-byte rows.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// ---------------------------------------------------------------------------
// Top-K threshold of one row by a warp: the H-th largest value among row[0..c)
// (c > H > 0), equal values going to the lower index.
//
// Keys (order-preserving uint32 images of the values, -0.0 == +0.0) are held in
// registers, key of index m = lane + 32*i in keys[i] (rows up to 32*KREG values).
// Key 0 (the image of a negative NaN) marks an empty slot.
constexpr int kSelectReg = 32;   // rows of up to 1024 values are selected from registers

template <int KREG>
__device__ __forceinline__ void load_row_keys(const float* __restrict__ row, int c, uint32_t (&keys)[KREG]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < KREG; ++i) {
    const int m = lane + 32 * i;
    keys[i] = (m < c) ? float_key(__ldg(row + m)) : 0u;
  }
}

// Key of the H-th largest value; *take_equal = how many values equal to it are kept.
// MSB-first bisection, one bit per step: the candidate keeps bit b when at least
// `remaining` keys share the candidate's higher bits and have bit b set. Counts
// use a warp reduction (no shared-memory atomics, so skewed digit distributions
// cost nothing extra).
template <int KREG>
__device__ __forceinline__ uint32_t radix_select_keys(const uint32_t (&keys)[KREG], int c, int H, uint32_t* hist,
                                                      int* take_equal) {
  (void)hist;
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0u;
  int remaining = H;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = (prefix | (1u << bit)) >> bit;
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < KREG; ++i) cnt += (lane + 32 * i < c && (keys[i] >> bit) == cand) ? 1 : 0;
    cnt = (int)__reduce_add_sync(0xffffffffu, (unsigned)cnt);
    if (cnt >= remaining)
      prefix |= 1u << bit;
    else
      remaining -= cnt;
  }
  *take_equal = remaining;
  return prefix;
}

// Index of the take_equal-th (1-based) value equal to tkey, ascending.
template <int KREG>
__device__ __forceinline__ int tie_index_keys(const uint32_t (&keys)[KREG], int c, uint32_t tkey, int take_equal) {
  const int lane = threadIdx.x & 31;
  int run = 0;
#pragma unroll
  for (int i = 0; i < KREG; ++i) {
    const int m = lane + 32 * i;
    const uint32_t bal = __ballot_sync(0xffffffffu, m < c && keys[i] == tkey);
    const int cnt = __popc(bal);
    if (run + cnt >= take_equal) {
      uint32_t bb = bal;
      for (int k = 1; k < take_equal - run; ++k) bb &= bb - 1u;
      return 32 * i + __ffs(bb) - 1;
    }
    run += cnt;
  }
  return -1;
}

// Bitonic sort of one value per lane across the warp, descending by lane.
__device__ __forceinline__ uint32_t warp_sort_desc(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
      v = keep_max ? max(v, o) : min(v, o);
    }
  }
  return v;
}

__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
      v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
    }
  }
  return v;
}

// Threshold of the H largest keys (ties toward the lower index) for H <= 32,
// without bisection. The H-th largest of the 32 per-lane maxima is a lower bound
// of the threshold: H lanes each hold a key at least that large. Keys below it are
// never taken, so when at most 32 keys reach it, those candidates are sorted
// across the warp by (key descending, index ascending) and the H-th one is the
// threshold key *tkey with its index *tidx (the largest index taken at that key).
// *asc gets, on lane i < H, the i-th smallest selected index (when asc != null);
// *top gets, on lane i < H, the index of the i-th selected key in (key descending,
// index ascending) order (when top != null).
// Returns false, with nothing written, when more than 32 keys reach the bound.
// Requires c > H. `cand` is 32 uint2 of this warp's shared memory.
template <int KREG>
__device__ __forceinline__ bool pivot_select_keys(const uint32_t (&keys)[KREG], int c, int H, uint2* cand,
                                                  uint32_t* tkey, int* tidx, uint32_t* asc = nullptr,
                                                  uint32_t* top = nullptr) {
  const int lane = threadIdx.x & 31;
  uint32_t lmax = 0u;
#pragma unroll
  for (int i = 0; i < KREG; ++i) lmax = max(lmax, keys[i]);   // empty slots hold key 0
  const uint32_t bound = __shfl_sync(0xffffffffu, warp_sort_desc(lmax), H - 1);
  int n = 0;
#pragma unroll
  for (int i = 0; i < KREG; ++i) n += (lane + 32 * i < c && keys[i] >= bound) ? 1 : 0;
  int incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (total > 32) return false;
  int pos = incl - n;
#pragma unroll
  for (int i = 0; i < KREG; ++i)
    if (lane + 32 * i < c && keys[i] >= bound) cand[pos++] = make_uint2(keys[i], (uint32_t)(lane + 32 * i));
  __syncwarp();
  uint64_t v = 0ull;   // below every candidate
  if (lane < total) {
    const uint2 e = cand[lane];
    v = ((uint64_t)e.x << 32) | (uint64_t)(0xffffffffu - e.y);
  }
  __syncwarp();
  v = warp_sort_desc(v);
  const uint64_t th = __shfl_sync(0xffffffffu, v, H - 1);
  *tkey = (uint32_t)(th >> 32);
  *tidx = (int)(0xffffffffu - (uint32_t)th);
  if (top) *top = 0xffffffffu - (uint32_t)v;
  if (asc) {
    // Lanes 0..H-1 hold the selection; order it by index (complements sorted
    // descending), the unselected lanes last.
    const uint32_t comp = (lane < H) ? (uint32_t)v : 0u;
    *asc = 0xffffffffu - warp_sort_desc(comp);
  }
  return true;
}

// Bitonic sort of 64 values held two per lane (element e = lane + 32 r in v[r]),
// descending by element index.
template <typename T>
__device__ __forceinline__ void warp_sort64_desc(T (&v)[2]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 32) {   // partners in the same lane
        const bool keep_max = ((lane + 0) & k) == 0;   // element lane keeps the max when ascending block
        const T hi = v[0] > v[1] ? v[0] : v[1], lo = v[0] > v[1] ? v[1] : v[0];
        v[0] = keep_max ? hi : lo;
        v[1] = keep_max ? lo : hi;
      } else {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int e = lane + 32 * r;
          const T o = __shfl_xor_sync(0xffffffffu, v[r], j);
          const bool keep_max = ((e & j) == 0) == ((e & k) == 0);
          v[r] = keep_max ? (v[r] > o ? v[r] : o) : (v[r] < o ? v[r] : o);
        }
      }
    }
  }
}

// Threshold of the H largest keys for 16 < H <= 63 (ties toward the lower index),
// the pivot select of pivot_select_keys with a tighter bound: each lane's two
// largest keys give 64 values whose H-th largest is a lower bound of the
// threshold (H distinct keys reach it); with about H + a few keys at or above it,
// the candidates are sorted across the warp two per lane by (key descending,
// index ascending). Returns false, with nothing written, when more than 64 keys
// reach the bound. Requires c > H. `cand`
// is 64 uint2 of this warp's shared memory.
template <int KREG>
__device__ __forceinline__ bool pivot2_select_keys(const uint32_t (&keys)[KREG], int c, int H, uint2* cand,
                                                   uint32_t* tkey, int* tidx) {
  const int lane = threadIdx.x & 31;
  uint32_t top[2] = {0u, 0u};   // this lane's two largest keys (empty slots hold key 0)
#pragma unroll
  for (int i = 0; i < KREG; ++i) {
    const uint32_t k = keys[i];
    if (k > top[0]) {
      top[1] = top[0];
      top[0] = k;
    } else if (k > top[1]) {
      top[1] = k;
    }
  }
  warp_sort64_desc(top);
  const int hb = H - 1;
  const uint32_t bound = __shfl_sync(0xffffffffu, top[hb >> 5], hb & 31);
  int n = 0;
#pragma unroll
  for (int i = 0; i < KREG; ++i) n += (lane + 32 * i < c && keys[i] >= bound) ? 1 : 0;
  int incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (total > 64) return false;
  int pos = incl - n;
#pragma unroll
  for (int i = 0; i < KREG; ++i)
    if (lane + 32 * i < c && keys[i] >= bound) cand[pos++] = make_uint2(keys[i], (uint32_t)(lane + 32 * i));
  __syncwarp();
  uint64_t v[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int e = lane + 32 * r;
    v[r] = 0ull;   // below every candidate
    if (e < total) {
      const uint2 x = cand[e];
      v[r] = ((uint64_t)x.x << 32) | (uint64_t)(0xffffffffu - x.y);
    }
  }
  __syncwarp();
  warp_sort64_desc(v);
  const uint64_t th = __shfl_sync(0xffffffffu, v[hb >> 5], hb & 31);
  *tkey = (uint32_t)(th >> 32);
  *tidx = (int)(0xffffffffu - (uint32_t)th);
  return true;
}

// Threshold key and tie index of the H largest keys (c > H): the pivot path when
// it applies, else the bisection and the tie scan.
template <int KREG>
__device__ __forceinline__ void threshold_keys(const uint32_t (&keys)[KREG], int c, int H, uint2* cand,
                                               uint32_t* tkey, int* tidx) {
  if (H <= 16 && pivot_select_keys(keys, c, H, cand, tkey, tidx)) return;
  if (H > 16 && H <= 63 && pivot2_select_keys(keys, c, H, cand, tkey, tidx)) return;
  int take_eq = 0;
  *tkey = radix_select_keys(keys, c, H, nullptr, &take_eq);
  *tidx = tie_index_keys(keys, c, *tkey, take_eq);
}

// Generic path for rows longer than 32*kSelectReg: keys re-read from memory on every pass.
__device__ __forceinline__ uint32_t radix_select_global(const float* __restrict__ row, int c, int H, uint32_t* hist,
                                                        int* take_equal) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0u, pmask = 0u;
  int remaining = H;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int i = 0; i < 8; ++i) hist[lane * 8 + i] = 0u;
    __syncwarp();
    for (int m = lane; m < c; m += 32) {
      const uint32_t key = float_key(row[m]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    uint32_t cnt[8];
    uint32_t local = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cnt[i] = hist[255 - 8 * lane - i];
      local += cnt[i];
    }
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - local;
    const bool mine = (excl < (uint32_t)remaining) && ((uint32_t)remaining <= incl);
    const uint32_t who = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    uint32_t digit = 0u;
    int rem_next = 0;
    if (mine) {
      uint32_t run = excl;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (run + cnt[i] >= (uint32_t)remaining) {
          digit = 255u - 8u * lane - i;
          rem_next = remaining - (int)run;
          break;
        }
        run += cnt[i];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, who);
    remaining = __shfl_sync(0xffffffffu, rem_next, who);
    prefix |= digit << shift;
    pmask |= 255u << shift;
    __syncwarp();
  }
  *take_equal = remaining;
  return prefix;
}

__device__ __forceinline__ int tie_index_global(const float* __restrict__ row, int c, uint32_t tkey, int take_equal) {
  const int lane = threadIdx.x & 31;
  int run = 0;
  for (int base = 0; base < c; base += 32) {
    const int m = base + lane;
    const uint32_t bal = __ballot_sync(0xffffffffu, m < c && float_key(row[m]) == tkey);
    const int cnt = __popc(bal);
    if (run + cnt >= take_equal) {
      uint32_t bb = bal;
      for (int k = 1; k < take_equal - run; ++k) bb &= bb - 1u;
      return base + __ffs(bb) - 1;
    }
    run += cnt;
  }
  return -1;
}

}  // namespace sas
