// kvq_device.cuh -- device-side building blocks shared by the kvq kernels:
// layout constants, mbarrier / bulk-copy wrappers with bounded waits, warp
// MMA wrappers, packed fp32x2 arithmetic, the hardware 2^x, the warp
// Walsh-Hadamard rotation and the device error word.
#pragma once

#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kPage = 16;
// slack factor on the certified bound and on Delta (absorbs the fp32 rounding
// of the quantizer, of the dequantization and of the rotation)
constexpr float kKappa = 1.0f + 1.0f / 1024.0f;
// relative size of the fp32 rotation error allowance (see the bound's Delta)
constexpr float kRotSlack = 1.0f / 65536.0f;
constexpr float kLog2e = 1.4426950408889634f;
// iteration limit of every spin on an mbarrier (each try_wait already
// suspends for a hardware-defined time, so this is on the order of seconds)
constexpr uint32_t kSpinLimit = 1u << 22;

// Outlier section of a block (outlier extraction): chunk indices of K and V,
// then the chunks' fp16 values, [16][4] each.
constexpr int kOutBytes = 2 * kPage + 2 * kPage * 4 * 2;
constexpr uint8_t kNoOutlier = 0xFF;

// Byte layout of one (page, kv head) block of the quantized pool.
struct BlockLayout {
  int d, kbits, kgroup;
  int out = 0;  // 1: the block ends in the outlier section
  __host__ __device__ int ngk() const { return d / kgroup; }
  __host__ __device__ int nb() const { return d / 32; }
  __host__ __device__ int k_row() const { return d * kbits / 8; }
  __host__ __device__ int v_row() const { return d / 2; }
  __host__ __device__ int k_bytes() const { return kPage * k_row(); }
  __host__ __device__ int v_bytes() const { return kPage * v_row(); }
  __host__ __device__ int ks_bytes() const { return kPage * ngk() * 2; }
  __host__ __device__ int vm_bytes() const { return kPage * nb() * 4; }
  __host__ __device__ int v_off() const { return k_bytes(); }
  __host__ __device__ int ks_off() const { return k_bytes() + v_bytes(); }
  __host__ __device__ int vm_off() const { return ks_off() + ks_bytes(); }
  __host__ __device__ int out_off() const { return vm_off() + vm_bytes(); }
  __host__ __device__ int bytes() const { return out_off() + (out ? kOutBytes : 0); }
};

__device__ __forceinline__ void set_error(int32_t* word, int code) {
  if (word) atomicCAS(word, 0, code);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier --------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for phase `parity` of `bar`; false if the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// ---- bulk copies (global -> shared, completion on an mbarrier) -------------
// L2 policy for data read once: its lines are the first evicted, so a stream of
// them leaves the small inputs every launch re-reads (context lengths, page
// table, queries, eta, split records) resident in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// One bulk copy of `bytes` (16-byte aligned addresses and size) into this
// CTA's shared memory; its bytes complete the transaction count of `bar`.
// `policy` is an L2 cache policy (l2_evict_first_policy for streamed data).
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Programmatic dependent launch.  A grid launched with programmatic stream
// serialization may start while the grid before it in the stream is still
// finishing; griddepcontrol.wait holds the thread until that grid has
// completed and its writes are visible (a no-op for an ordinary launch).
// launch_dependents lets the next such grid begin launching; it starts once
// every CTA of this grid has run (or passed) that point, so its CTAs take only
// SM slots this grid has left.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Bring [src, src + bytes) into L2 (16-byte aligned address and size); no
// destination, no completion, no effect on memory contents.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---- 2^x by the hardware approximation (PTX ex2.approx.ftz.f32) -------------
// Relative error about 2^-22; results below the normal range flush to +0 and
// 2^-inf = +0.  Softmax weights and the bound's exponentials need no more.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- compile-time loop: f(std::integral_constant<int, I>) for I in [B, E) -----
template <int B, int E, class F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (B < E) {
    f(std::integral_constant<int, B>{});
    static_for<B + 1, E>(f);
  }
}

// ---- warp-level MMA (fragment layouts of the PTX m16n8k32 / m16n8k16 shapes) --
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Ticket of a split-K merge: atomic add with acquire-release semantics at GPU
// scope, so one thread publishes the records its CTA wrote before a barrier and,
// when it draws the last ticket, sees every other CTA's records.
__device__ __forceinline__ int atomic_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
__device__ __forceinline__ uint32_t lop_and_or(uint32_t x, uint32_t m, uint32_t o) {
  return (x & m) | o;
}
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}

// ---- packed fp32x2 arithmetic (one instruction for two IEEE fp32 lanes) ------
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 pa, pb, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
      "mul.rn.f32x2 pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 pa, pb, pc, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
      "mov.b64 pc, {%6, %7};\n\tfma.rn.f32x2 pd, pa, pb, pc;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

// ---- randomized Walsh-Hadamard rotation of one vector held by a warp ------
// Lane l holds elements [l*E, l*E + E) of a d = 32*E vector.  Computes
// y = c * H_d * (sigma o x) with butterflies in the fixed order stride 1, 2,
// ..., d/2 (pair (a, b) at (j, j+stride) -> (a+b, a-b)), then the product by
// c = fp32(1/sqrt(d)); every operation is a single fp32 add, sub or mul, so
// the result does not depend on how the butterflies are distributed.
template <int E>
__device__ __forceinline__ void warp_hadamard(float (&x)[E], int lane, float c);
template <int E>
__device__ __forceinline__ void warp_rotate(float (&x)[E], const int8_t* sigma, int lane,
                                            float c) {
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (sigma[lane * E + e] < 0) x[e] = -x[e];
  warp_hadamard<E>(x, lane, c);
}
// The butterflies and the product by c of warp_rotate, without the signs:
// y = c * H_d * x (its own inverse, since (c H_d)^2 = I).
template <int E>
__device__ __forceinline__ void warp_hadamard(float (&x)[E], int lane, float c) {
#pragma unroll
  for (int h = 1; h < E; h *= 2) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if ((e & h) == 0) {
        float a = x[e], b = x[e + h];
        x[e] = __fadd_rn(a, b);
        x[e + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int hl = 1; hl < 32; hl *= 2) {
    const bool upper = (lane & hl) != 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float other = __shfl_xor_sync(0xffffffffu, x[e], hl);
      // lower element a (index j), upper element b (index j + stride)
      x[e] = upper ? __fsub_rn(other, x[e]) : __fadd_rn(x[e], other);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = __fmul_rn(x[e], c);
}

__device__ __forceinline__ float load_elem(const void* p, int is_bf16, int64_t i) {
  if (is_bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}

}  // namespace kvq
