// Shared device/host helpers of the jenga library (sm_100a only).
//
// Error plumbing: every exported call returns jenga_status; kernels that detect a
// fault (bounded wait expired, index out of range) record it in a module-global
// device error word that jenga_check_device_status() reads and clears.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <string>

#include "../../include/jenga.h"

namespace jenga {

typedef __nv_bfloat16 bf16;

// ------------------------------------------------------------------ host errors
void set_last_error(const std::string& msg);
jenga_status fail(jenga_status st, const char* fmt, ...);

#define JENGA_CUDA_TRY(expr)                                                        \
  do {                                                                              \
    cudaError_t _e = (expr);                                                        \
    if (_e != cudaSuccess)                                                          \
      return ::jenga::fail(JENGA_ECUDA, "%s failed: %s (%s:%d)", #expr,             \
                           cudaGetErrorString(_e), __FILE__, __LINE__);             \
  } while (0)

#define JENGA_CHECK_ARG(cond, ...)                                                  \
  do {                                                                              \
    if (!(cond)) return ::jenga::fail(JENGA_EINVAL, __VA_ARGS__);                   \
  } while (0)

#define JENGA_LAUNCH_CHECK()                                                        \
  do {                                                                              \
    cudaError_t _e = cudaGetLastError();                                            \
    if (_e != cudaSuccess)                                                          \
      return ::jenga::fail(JENGA_ECUDA, "kernel launch failed: %s (%s:%d)",         \
                           cudaGetErrorString(_e), __FILE__, __LINE__);             \
  } while (0)

// ------------------------------------------------------------------ device errors
// err[0] = first error code (JENGA_E*), err[1] = site id, err[2] = detail.
// Defined here: the library is one translation unit (csrc/jenga_all.cu).
__device__ unsigned int g_device_error[4];

enum ErrSite : unsigned int {
  SITE_GEMM_PRODUCER = 1,
  SITE_GEMM_MMA = 2,
  SITE_GEMM_EPILOGUE = 3,
  SITE_SCORE_TC = 4,
  SITE_INDEX_RANGE = 5,
  SITE_NKEPT_RANGE = 6,
  SITE_ATTN = 7,
  SITE_TEST_WAIT = 8,
  SITE_PACK_RANGE = 9,  // a weight outside fp16's range at pack time (detail: element index)
};

__device__ __forceinline__ void record_device_error(unsigned code, unsigned site, unsigned detail) {
  if (atomicCAS(&g_device_error[0], 0u, code) == 0u) {
    g_device_error[1] = site;
    g_device_error[2] = detail;
  }
}

// wait budget for mbarrier spins, in nanoseconds of %globaltimer (host-settable)
__device__ unsigned long long g_wait_budget_ns = 2000000000ull;

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}

// Bounded wait: returns false (and records a timeout) if the phase does not
// complete within the wait budget.  Never spins forever.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t phase, unsigned site) {
  if (mbar_try_wait(bar, phase)) return true;
  const unsigned long long t0 = global_timer_ns();
  const unsigned long long budget = g_wait_budget_ns;
  while (true) {
    if (mbar_try_wait(bar, phase)) return true;
    if (global_timer_ns() - t0 > budget) {
      record_device_error(JENGA_ETIMEOUT, site, phase);
      return false;
    }
  }
}

// Same, recording a caller-chosen detail word (e.g. tile index) on timeout.
__device__ __forceinline__ bool mbar_wait_at(uint64_t* bar, uint32_t phase, unsigned site, unsigned detail) {
  if (mbar_try_wait(bar, phase)) return true;
  const unsigned long long t0 = global_timer_ns();
  const unsigned long long budget = g_wait_budget_ns;
  while (true) {
    if (mbar_try_wait(bar, phase)) return true;
    if (global_timer_ns() - t0 > budget) {
      record_device_error(JENGA_ETIMEOUT, site, detail);
      return false;
    }
  }
}

// 2D TMA tile load into shared memory, completion counted on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Named barrier over `threads` threads (a multiple of 32) that also returns the AND of
// every participant's predicate: warps that must leave a loop together use it.
__device__ __forceinline__ bool bar_and(bool v, int bar_id, int threads) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(bar_id), "r"(threads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool pair_all(bool v, int bar_id) { return bar_and(v, bar_id, 64); }

// Element-wise add of a shared-memory tile into global memory through a tensor map (the L2
// performs the additions); the copy belongs to this thread's current bulk async-group.
// Coordinates must be non-negative, x a multiple of 4 (fp32, 16 bytes).
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* smem_src, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}
// Plain store of a shared-memory tile through a tensor map (rows past the map's extent are
// clipped); same bulk async-group rules as tma_reduce_add_2d.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk group of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until at most N of this thread's committed bulk groups are still reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// 1D bulk copy global -> shared (both addresses and the size multiples of 16 bytes),
// completion counted on an mbarrier.
__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tcgen05 (5th-generation tensor core, accumulators in tensor memory)
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_holder, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_holder)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
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

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate (kind::f16)
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, fp32 accumulate (kind::f16).  A sits in
// tensor memory with row i in lane i and element k of the row in column k / 2 (bf16 pairs,
// even k in the low half), so one K = 16 step spans 8 columns.  Reading A from tensor
// memory instead of shared memory halves the shared-memory traffic of an M 128 x N 128 MMA,
// which otherwise saturates shared-memory bandwidth before the tensor core.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Load 32 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes 32*(w%4)..).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Same load without the wait (issue several, then tmem_wait_ld once).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Load 16 consecutive 32-bit columns of this thread's TMEM lane, without the wait.
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Store 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Copy row r of a 128 x 128 bf16 tile held in shared memory as two 64-column boxes with the
// 128-byte swizzle (the TMA layout) into tensor-memory columns [col, col + 64) of lane r,
// in the A-operand layout of umma_bf16_ts.  Warp-collective (tcgen05.st).
__device__ __forceinline__ void tile_row_to_tmem(const uint8_t* tile, int r, uint32_t taddr_lane_col) {
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint32_t w[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 q = *reinterpret_cast<const uint4*>(tile + b * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
      w[4 * c] = q.x;
      w[4 * c + 1] = q.y;
      w[4 * c + 2] = q.z;
      w[4 * c + 3] = q.w;
    }
    tmem_st32(taddr_lane_col + b * 32, w);
  }
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy
// (tensor-core operand reads, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory descriptor for an MN-major operand tile stored as 64-element (128-byte)
// rows with the 128-byte swizzle: consecutive K rows 128 bytes apart in 8-row (1024-byte)
// groups (SBO), successive 64-element MN groups mn_group_bytes apart (LBO).
__device__ __forceinline__ uint64_t umma_desc_mn_sw128(uint32_t smem_addr, uint32_t mn_group_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  d |= (uint64_t)((mn_group_bytes >> 4) & 0x3FFF) << 16;  // leading byte offset: next 64-wide MN group
  d |= (uint64_t)(1024 >> 4) << 32;                         // stride byte offset: next 8 K rows
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16 bf16 -> fp32, A K-major, B MN-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_bmn(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction for two lanes' worth)
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x on the FMA / integer pipes, for kernels whose exponentials would otherwise queue on
// the multi-function unit (16 results per clock per SM).  Binary split x = j + f with j the
// integer nearest x (the 1.5 * 2^23 shifter rounds x into the low mantissa bits) and
// |f| <= 1/2; 2^f is a cubic whose relative error is equal-ripple on [-1/2, 1/2]
// (coefficients: a Lawson IRLS minimax fit, refitted and checked by tests/test_exp2_fit.py;
// max relative error 7.5e-5);
// 2^j is added into the exponent field.  Inputs are clamped to [-125, HI], so the result
// is >= 2^-125.5 for very negative x and finite for large x.
template <int HI = 64>
__device__ __forceinline__ float exp2_fma(float x) {
  x = fminf(fmaxf(x, -125.f), (float)HI);
  const float t = __fadd_rn(x, 12582912.f);
  const float f = __fsub_rn(x, __fsub_rn(t, 12582912.f));
  float p = fmaf(0x1.c3f760p-5f, f, 0x1.f0de1ap-3f);
  p = fmaf(p, f, 0x1.62f31ap-1f);
  p = fmaf(p, f, 0x1.fff692p-1f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Pair form of exp2_fma (same arithmetic, f32x2 instructions for the split and the cubic);
// HI < 0 skips the upper clamp (callers whose inputs are known to be <= 0).
template <int HI = 64>
__device__ __forceinline__ uint64_t exp2_fma_x2(uint64_t x2) {
  float x0, x1;
  f2unpack(x2, x0, x1);
  x0 = fmaxf(x0, -125.f);
  x1 = fmaxf(x1, -125.f);
  if constexpr (HI >= 0) {
    x0 = fminf(x0, (float)HI);
    x1 = fminf(x1, (float)HI);
  }
  const uint64_t x = f2pack(x0, x1);
  const uint64_t t = fadd2(x, f2pack(12582912.f, 12582912.f));
  const uint64_t j = fadd2(t, f2pack(-12582912.f, -12582912.f));
  const uint64_t f = ffma2(j, f2pack(-1.f, -1.f), x);
  uint64_t p = ffma2(f2pack(0x1.c3f760p-5f, 0x1.c3f760p-5f), f, f2pack(0x1.f0de1ap-3f, 0x1.f0de1ap-3f));
  p = ffma2(p, f, f2pack(0x1.62f31ap-1f, 0x1.62f31ap-1f));
  p = ffma2(p, f, f2pack(0x1.fff692p-1f, 0x1.fff692p-1f));
  float p0, p1, t0, t1;
  f2unpack(p, p0, p1);
  f2unpack(t, t0, t1);
  return f2pack(__int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23)),
                __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23)));
}

// 2^x for both halves of a pair on the multi-function unit
__device__ __forceinline__ uint64_t exp2_mufu_x2(uint64_t x2) {
  float x0, x1;
  f2unpack(x2, x0, x1);
  return f2pack(fast_exp2(x0), fast_exp2(x1));
}

// Shared-memory matrix descriptor for a K-major tile whose rows are 128 bytes
// (64 bf16), stored with the 128-byte swizzle in 1024-byte groups of 8 rows.
__device__ __forceinline__ uint64_t umma_desc_k_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);          // start address (16-byte units)
  d |= (uint64_t)1 << 16;                               // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024 >> 4) << 32;                     // stride byte offset: 8-row group pitch
  d |= (uint64_t)1 << 46;                               // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                               // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16, A/B bf16 K-major, D fp32, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ float bf16_to_f(bf16 v) { return __bfloat162float(v); }

// two floats -> packed bf16 pair (round to nearest even), a in the low half
__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ------------------------------------------------------------------ host helpers
// Encode a 2D row-major bf16 tensor map (rows x cols, row pitch ld elements) with a
// box of box_rows x 64 columns and the 128-byte swizzle.
jenga_status make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                            uint32_t box_rows);
// Same for an fp16 tensor (box of box_rows x 64 columns).
jenga_status make_tmap_f16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                           uint32_t box_rows);
// Same for an fp32 tensor: box of box_rows x 32 columns (128-byte rows), 128-byte swizzle.
jenga_status make_tmap_f32(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                           uint32_t box_rows);

int sm_count();
unsigned long long host_wait_budget_ns();

// Per-launch timing (off by default): when enabled with jenga_profile_enable, every
// kernel launch is bracketed by two CUDA events recorded on its own stream, and
// jenga_profile_report aggregates launches and milliseconds per kernel name.
int prof_begin(const char* name, cudaStream_t st);
void prof_end(int slot, cudaStream_t st);

}  // namespace jenga
