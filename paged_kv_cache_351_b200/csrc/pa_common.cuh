// Device helpers shared by the paged-KV kernels (sm_100a).
//
// Everything here is a thin wrapper over documented PTX: mbarrier
// init/arrive/try_wait, the non-multicast bulk copy global -> shared that
// completes on an mbarrier, proxy fences, the global nanosecond timer, and
// programmatic-dependent-launch controls.  No multicast form is used
// anywhere in this library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pa.h"

namespace pa {

// Per-device status word: bits PA_DEV_* set by kernels, read and cleared by
// pa_get_device_status.  One translation unit holds every kernel, so this
// needs no relocatable device code.
__device__ unsigned int g_status;

__device__ __forceinline__ void flag(unsigned int bits) { atomicOr(&g_status, bits); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- mbarrier --------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make initialised barriers visible to the async proxy (bulk copies).
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns
// false (and sets PA_DEV_TIMEOUT) if it has not completed after timeout_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int k = 0; k < 32; ++k)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > timeout_ns) {
      flag(PA_DEV_TIMEOUT);
      return false;
    }
  }
}

// ---- bulk copy (TMA engine, 1-D, no tensor map, no multicast) --------------
// dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst_smem, const void* src, uint32_t bytes, uint32_t bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          dst_smem),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Starts moving the cache line holding p into L1 (no register, no wait).
__device__ __forceinline__ void prefetch_l1(const void* p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

// ---- programmatic dependent launch -----------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// ---- numeric helpers ---------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// d = a * b + d on two fp32 lanes at once (packed FMA, sm_100).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rd, {%0, %1};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rd;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// d = a + b on two fp32 lanes at once (packed add, sm_100), round to nearest.
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// 2^x for two values on the FMA pipe (a stand-in for the special-function
// unit when that unit is the bottleneck).  Range reduction x = n + f with n
// the nearest integer (adding 1.5 * 2^23 rounds to it) and |f| <= 1/2; 2^f
// from a cubic whose coefficients were fitted here by iteratively reweighted
// least squares on [-1/2, 1/2] for the smallest maximum relative error
// (1.0e-4, below a bf16 rounding step of 3.9e-3); 2^n is added to the
// exponent field.  Inputs are clamped to >= -126 (results below 2^-126 come
// out as about 2^-126 instead of 0); inputs must be <= 127.
__device__ __forceinline__ void ex2_poly2(float& a, float& b) {
  constexpr float kRound = 12582912.0f;
  constexpr float kC1 = 0.6932829022407532f, kC2 = 0.24221085011959076f, kC3 = 0.05500883609056473f;
  a = fmaxf(a, -126.f);
  b = fmaxf(b, -126.f);
  float ta, tb, ra, rb;
  fadd2(ta, tb, a, b, kRound, kRound);
  fadd2(ra, rb, ta, tb, -kRound, -kRound);
  float fa = a, fb = b;
  ffma2(fa, fb, ra, rb, -1.f, -1.f);  // f = x - n
  float pa = kC2, pb = kC2;
  ffma2(pa, pb, fa, fb, kC3, kC3);
  float qa = kC1, qb = kC1;
  ffma2(qa, qb, fa, fb, pa, pb);
  float ua = 1.f, ub = 1.f;
  ffma2(ua, ub, fa, fb, qa, qb);
  a = __int_as_float(__float_as_int(ua) + (__float_as_int(ta) << 23));
  b = __int_as_float(__float_as_int(ub) + (__float_as_int(tb) << 23));
}

// The two e4m3 codes in the low (lo) or high (hi) half of w, low byte
// first -> two f16 in one register (exact): one cvt.rn.f16x2.e4m3x2, the
// half selected by register pairing.
__device__ __forceinline__ uint32_t e4m3x2_lo_to_f16x2(uint32_t w) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(r) : "r"(w));
  return r;
}
__device__ __forceinline__ uint32_t e4m3x2_hi_to_f16x2(uint32_t w) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, hi;\n\t}" : "=r"(r) : "r"(w));
  return r;
}

// Two f16 in one register -> two fp32 (exact).
__device__ __forceinline__ void f16x2_to_f32(uint32_t h, float& lo, float& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h));
}

// Storage-type traits: a 16-byte vector holds EPV elements.
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int EPV = 4;
  __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static uint4 pack(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int EPV = 8;
  // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits.
  __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
  __device__ __forceinline__ static uint4 pack(const float* f) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * k], f[2 * k + 1]);
      w[k] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// FP8 e4m3 codes (a quantized KV cache): a 16-byte vector holds 16 codes.
// Decoding goes e4m3x2 -> f16x2 -> 2 x f32, all exact; the per-head scale is
// applied by the caller.  Only decoding exists here: codes are produced by the
// cache write (quantize_e4m3x2).
template <>
struct Elem<__nv_fp8_e4m3> {
  static constexpr int EPV = 16;
  __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f16x2_to_f32(e4m3x2_lo_to_f16x2(w[k]), f[4 * k + 0], f[4 * k + 1]);
      f16x2_to_f32(e4m3x2_hi_to_f16x2(w[k]), f[4 * k + 2], f[4 * k + 3]);
    }
  }
};

// Two floats -> two e4m3 codes (round to nearest even, saturating to +-448;
// NaN stays NaN), first value in the low byte.
__device__ __forceinline__ uint32_t quantize_e4m3x2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// d += a * b on the tensor cores: m16n8k16, f16 inputs, fp32 accumulate.
// Fragment layout (lane = 4 * gr + tig): a = {(row gr, k 2tig..+1),
// (row gr + 8, k 2tig..+1), (row gr, k 2tig+8..+9), (row gr + 8, k 2tig+8..+9)},
// b = {(k 2tig..+1, col gr), (k 2tig+8..+9, col gr)}, d = {(gr, 2tig),
// (gr, 2tig+1), (gr + 8, 2tig), (gr + 8, 2tig+1)}.
__device__ __forceinline__ void mma_16816_f16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two floats -> two bf16 (round to nearest even) in one register, first in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint4 ld_nc_v4(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

}  // namespace pa
