// Device helpers shared by the bifocal kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bf {

// ---------------------------------------------------------------------------------
// Device status word: the first event of a launch sequence that the kernels cannot
// turn into a correct result records a code here and the kernel carries on or leaves:
//   kDevTimeout | site << 8   a bounded wait gave up (site numbers the wait in the source)
//   kDevRange   | site << 8   an operand of the fp16 QK^T product was not finite after
//                             rounding to fp16 (|x| >= 65520, inf or NaN)
//   kDevIndex   | site << 8   an index read from device memory (a sequence length or a
//                             block-table entry) was out of range; the reads and writes it
//                             would have addressed were skipped
// Read and cleared by bifocal_last_device_error().
// ---------------------------------------------------------------------------------
enum : int { kDevOk = 0, kDevTimeout = 1, kDevRange = 2, kDevIndex = 3 };
__device__ int g_device_status = 0;

// Wall-clock limit of every bounded wait, in ns (2 s; a test may shorten it through
// bifocal_test_set_fault so that an expiry costs milliseconds). A wait reads it only once it
// has already waited kWaitFloorNs (20 ms, far beyond any wait of a healthy launch), so the
// polling loops of normal operation compare against a constant and never touch global memory.
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;
constexpr unsigned long long kWaitFloorNs = 20000000ull;

__device__ __forceinline__ void report_status(int code, int where) {
  if (*reinterpret_cast<volatile int*>(&g_device_status) == kDevOk) atomicCAS(&g_device_status, kDevOk, code | (where << 8));
}
__device__ __forceinline__ void report_timeout(int where) { report_status(kDevTimeout, where); }

// fp16 operand range guard: true when rounding x to fp16 gives a finite value (|x| < 65520;
// from 65520 on round-to-nearest gives inf); false for larger magnitudes, inf and NaN.
__device__ __forceinline__ bool f16_ok(float x) { return fabsf(x) < 65520.f; }

// ---------------------------------------------------------------------------------
// RoPE angles. The angle p * omega reaches ~1.3e5 rad at 128K tokens, where an fp32
// angle would be off by up to 4e-3 rad. The product and the reduction to [-pi, pi]
// run in fp64; only the reduced angle goes through the fast fp32 sine/cosine, whose
// absolute error on [-pi, pi] is a few 1e-7.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void angle_cos_sin(double angle, float& c, float& s) {
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  double r = fma(-two_pi, rint(angle * inv_two_pi), angle);
  __sincosf(static_cast<float>(r), &s, &c);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// bf16 pair -> fp16 pair (exact for values inside the fp16 normal range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  float2 f = __bfloat1622float2(v);
  return pack_f16x2(f.x, f.y);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 lanes in one 64-bit register pair, for the packed f32x2 arithmetic of sm_100
// (one issue slot for two FMAs or two adds).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// bf16x2 -> packed fp32 pair (a bf16 is the upper half of its fp32); packed pair -> fp16x2 (RN)
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t f2_to_f16x2(uint64_t v) {
  float lo, hi;
  f2_unpack(v, lo, hi);
  return pack_f16x2(lo, hi);
}

// ---------------------------------------------------------------------------------
// Legacy warp-level tensor core path (used where tensor throughput is not the limit).
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// m16n8k8, bf16: a0 = A[g][2t..2t+1], a1 = A[g+8][2t..2t+1]; b0 = B[2t..2t+1][g]
__device__ __forceinline__ void mma_bf16_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t smem_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t smem_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async_16(uint32_t smem_addr, const void* gptr, bool pred) {
  int src_size = pred ? 16 : 0;  // zero-fill when the row is out of range
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr), "l"(gptr), "r"(src_size));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// ---------------------------------------------------------------------------------
// mbarrier + TMA (bulk tensor copies, no multicast)
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::);
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::);
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)));
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase));
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: polls the barrier; after g_wait_limit_ns of wall time it records a timeout and
// returns false so that the caller can leave instead of hanging the GPU.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t phase, int where) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, phase)) return true;
    if ((it & 63) == 0) {
      const uint64_t el = global_ns() - t0;
      if (el > kWaitFloorNs && el > *reinterpret_cast<volatile unsigned long long*>(&g_wait_limit_ns)) break;
    }
  }
  report_timeout(where);
  return false;
}

// Bounded wait for a thread that has nothing else to do until the phase completes (a
// producer waiting for its last copies before the CTA exits): sleeps between polls, so it
// takes no issue slots from the warps still working on the same SM sub-partition.
__device__ __forceinline__ bool mbar_wait_sleepy(uint64_t* bar, uint32_t phase, int where) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, phase)) {
    __nanosleep(500);
    const uint64_t el = global_ns() - t0;
    if (el > kWaitFloorNs && el > *reinterpret_cast<volatile unsigned long long*>(&g_wait_limit_ns)) {
      report_timeout(where);
      return false;
    }
  }
  return true;
}

// Same, but also gives up as soon as *abort is set (by any warp of the CTA), and sets it
// on its own timeout, so that one expired wait makes every later wait of the CTA return.
__device__ __forceinline__ bool mbar_wait_abortable(uint64_t* bar, uint32_t phase, int where, volatile int* abort) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, phase)) return true;
    if ((it & 63) == 0) {
      if (*abort) return false;
      const uint64_t el = global_ns() - t0;
      if (el > kWaitFloorNs && el > *reinterpret_cast<volatile unsigned long long*>(&g_wait_limit_ns)) break;
    }
  }
  *abort = 1;
  report_timeout(where);
  return false;
}

// Warp-level wait: lane 0 polls (bounded, abortable), then every lane takes its own
// acquire with one try_wait on the (now completed) phase. Returns a warp-uniform result.
// The caller guarantees the barrier cannot advance past this phase before the warp acts.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t phase, int where, volatile int* abort) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait_abortable(bar, phase, where, abort);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) ok = mbar_try_wait(bar, phase) ? 1 : 0;
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];\n" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];\n" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// Programmatic dependent launch: let the next kernel on the stream start its prologue now /
// wait until the previous kernel has completed and its writes are visible.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];\n" ::"l"(map) : "memory");
}

}  // namespace bf
