// Device helpers shared by the sm_100a kernels of the block step.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dflash2.h"

#define DEVI __device__ __forceinline__

namespace dfl {

constexpr int kUnit = 256;            // K granularity of the streaming GEMV (one Q4_K super-block)
constexpr int kQ4Bytes = 2304;        // prepared Q4_K tile x super-block: 2048 B codes + 256 B scales
constexpr int kTopK = 16;
constexpr int kHeadDim = 128;
constexpr int kPage = 16;
constexpr int kAttnKeys = 64;         // cache keys per attention chunk (4 pages)
constexpr int kAttnStride = 136;      // bf16 elements per staged K/V/Q row (272 B, conflict-free ldmatrix)
constexpr int kHeadTiles = 16;  // tiles (of 16 rows) per prepared output-head record
constexpr long long kWaitLimit = 1ll << 26;  // bounded spin on an mbarrier

DEVI float bf2f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
DEVI uint16_t f2bf(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }
DEVI uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 16-byte streaming load: read once, do not keep in L1.
DEVI uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// 16-byte load of a ring slot that the slot's release hands back to the copy engine: a volatile
// shared load, so the compiler neither repeats it after the release (rematerialising the value
// from memory that may by then hold the next copy) nor moves it past the release.
DEVI uint4 lds_slot(const void* p) {
  uint4 r;
  asm volatile("ld.volatile.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"((uint32_t)__cvta_generic_to_shared(p))
               : "memory");
  return r;
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
// a[0]: (row g, k 2t..2t+1), a[1]: (row g+8, k 2t..), a[2]: (row g, k 2t+8..), a[3]: (row g+8, k 2t+8..)
// b0: (k 2t..2t+1, n g), b1: (k 2t+8.., n g); d: (g, 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1)
DEVI void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Packed fp32 pair FMA (sm_100): d = a * b + c on two lanes of a 64-bit register pair.
DEVI float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ra, rb, rc, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}

DEVI uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

DEVI void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
DEVI void ldmatrix_x2(uint32_t& r0, uint32_t& r1, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(smem_u32(p)));
}
DEVI void ldmatrix_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
DEVI void ldmatrix_x2_trans(uint32_t& r0, uint32_t& r1, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(smem_u32(p)));
}

// ---- mbarrier + bulk async copy (TMA engine, 1-D form) ----
DEVI void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
DEVI void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
DEVI void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
DEVI bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; returns false when the limit expired.
DEVI bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  for (long long i = 0; i < kWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
// Same, but the waiting thread is suspended (up to a few microseconds per try) instead of
// spinning, leaving issue slots to the warps that do work (the producer in particular).
DEVI bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(4000u)
      : "memory");
  return ok != 0;
}
DEVI bool mbar_wait_sleep_bounded(uint64_t* bar, uint32_t parity) {
  for (long long i = 0; i < (kWaitLimit >> 6); ++i)
    if (mbar_try_wait_sleep(bar, parity)) return true;
  return false;
}
// global -> shared bulk copy; dst/src 16-byte aligned, bytes a multiple of 16.
DEVI void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

DEVI float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Ordering of candidates: larger logit first, smaller token id on equal logits.
DEVI bool better(float a, int ia, float b, int ib) { return a > b || (a == b && ia < ib); }

// Programmatic dependent launch: let the next kernel on the stream start its prologue, and
// wait until every earlier kernel has finished and its writes are visible.
DEVI void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
DEVI void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Named barrier 1 over the first NTHR threads of the CTA.
template <int NTHR>
DEVI void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NTHR) : "memory"); }
// Order this thread's view of global memory before its later bulk (async-proxy) copies.
DEVI void fence_proxy_async() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

DEVI void set_err(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace dfl
