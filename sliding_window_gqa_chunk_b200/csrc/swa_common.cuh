// swa_common.cuh - small device helpers shared by the libswa kernels
// (bf16 packing, exp2, warp-level matrix ops, mbarrier waits with a bound).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "swa.h"

namespace swa {

// Programmatic dependent launch: the library's kernels are launched with
// programmatic stream serialization, so they may be scheduled while the
// previous kernel in the stream is still running; this wait (before a kernel
// reads or writes any global memory) returns once that kernel has completed
// and its memory writes are visible, which keeps ordinary stream order for
// everything they read or write.  Only the launch latency and the kernel's
// own set-up are overlapped.
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the next kernel in the stream (launched with programmatic stream
// serialization) be scheduled onto free SMs now instead of at this kernel's
// end; it still waits in wait_prior_grid for this kernel to complete.  Issued
// right after this kernel's own wait, so at most one kernel runs ahead.
__device__ __forceinline__ void allow_next_grid() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Status word codes written by kernels (first error wins).
__device__ __forceinline__ void raise_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Two fp32 -> packed bf16x2, round to nearest even; `lo` goes to bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 2^x on the SFU (MUFU.EX2); flushes denormal results to zero, exact 0 for -inf.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte permute: picks bytes of {b, a} by the nibbles of `sel`.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Transpose of an 8x8 b16 matrix held one row-pair per lane (m8n8 fragment).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D += A * B for one 16x8x16 bf16 tile, fp32 accumulators (warp-wide).
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte global load that bypasses L1 allocation (streamed once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ldg_stream8(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ldg_stream4(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

}  // namespace swa
