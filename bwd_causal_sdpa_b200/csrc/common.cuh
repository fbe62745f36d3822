// common.cuh -- small device helpers shared by every kernel of libattn.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "attn.h"

// Device status word (one per device context). Kernels record the first
// device-detected problem here instead of trapping; attn_get_status() reads
// and clears it.
__device__ int g_attn_status;

// Internal status: a kernel found its shared-memory window misaligned for the
// 128-byte swizzle and did nothing (reported to callers as ATTN_ECUDA).
#define ATTN_ECUDA_LAYOUT ATTN_ECUDA

__device__ __forceinline__ void report_status(int code) {
  atomicCAS(&g_attn_status, 0, code);
}

// Executed tile products of the tensor-core kernels since the last read by
// attn_tile_counts(): [0] forward (128-query x 128-key tiles a forward CTA
// computes), [1] backward key-tile kernel, [2] backward query-tile (dQ) pass,
// in the same unit. One atomic add per CTA.
__device__ unsigned long long g_attn_tiles[3];

#ifdef ATTN_DEBUG_HOOKS
// Watchdog test build only: a load the forward's TMA warp withholds (0 = none,
// 1 = the first V tile), so that a consumer's bounded wait runs out.
__device__ int g_attn_withhold;
#endif

// Programmatic dependent launch. Every kernel of this library runs this first:
// wait until the kernel before it in the stream has completed and its memory
// operations are visible (a no-op when launched without the attribute), so no
// global access of this kernel, read or write, can overlap its predecessor;
// then let the next kernel be scheduled (it will wait the same way), which
// hides launch latency behind this kernel's tail.
__device__ __forceinline__ void pdl_wait_and_trigger() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- storage type conversions ---------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Load / store NC consecutive elements (NC = 2 or 4) as fp32.
template <int NC>
__device__ __forceinline__ void load_vec(const float* p, float* out) {
  if constexpr (NC == 4) {
    float4 t = *reinterpret_cast<const float4*>(p);
    out[0] = t.x; out[1] = t.y; out[2] = t.z; out[3] = t.w;
  } else {
    float2 t = *reinterpret_cast<const float2*>(p);
    out[0] = t.x; out[1] = t.y;
  }
}
template <int NC>
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float* out) {
  if constexpr (NC == 4) {
    uint2 t = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&t.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&t.y);
    out[0] = __low2float(a); out[1] = __high2float(a);
    out[2] = __low2float(b); out[3] = __high2float(b);
  } else {
    __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(p);
    out[0] = __low2float(a); out[1] = __high2float(a);
  }
}
template <int NC>
__device__ __forceinline__ void store_vec(float* p, const float* v) {
  if constexpr (NC == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  }
}
template <int NC>
__device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float* v) {
  if constexpr (NC == 4) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 t;
    t.x = *reinterpret_cast<uint32_t*>(&a);
    t.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = t;
  } else {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// fp16 storage of rotated q / k tiles: fp16 keeps 3 more mantissa bits than
// bf16 (which the lse bound needs) but has a narrow range (overflow above
// 65504, subnormals below 2^-14). A 128-row tile is therefore stored times
// the power of two that brings its largest magnitude amax into [2^14, 2^15):
// large tiles cannot overflow and small ones keep all 11 bits down to 2^-28
// of their maximum. The exponent is clamped so
// that the factor and its inverse stay normal floats; an all-zero tile keeps
// factor 1.
__device__ __forceinline__ float fp16_tile_factor(float amax) {
  if (!(amax > 0.f && amax <= 3.0e38f)) return 1.f;
  return ldexpf(1.f, max(-100, min(100, 14 - ilogbf(amax))));
}
// RoPE table entries for eight consecutive dimensions d0.. (d0 a multiple of
// 8) at position pos: four pairs' cos and sin, one 16-byte load each (the
// tables must be 16-byte aligned); rotate8 applies them with the same
// roundings as rope_pairs.
struct Rope8 {
  float4 c, s;
};
template <int D>
__device__ __forceinline__ Rope8 rope8_load(const float* rc, const float* rs, int pos, int d0) {
  Rope8 t;
  t.c = *reinterpret_cast<const float4*>(rc + (size_t)pos * (D / 2) + (d0 >> 1));
  t.s = *reinterpret_cast<const float4*>(rs + (size_t)pos * (D / 2) + (d0 >> 1));
  return t;
}
__device__ __forceinline__ void rotate8(float* x, const Rope8& t) {
  const float cs[4] = {t.c.x, t.c.y, t.c.z, t.c.w}, sn[4] = {t.s.x, t.s.y, t.s.z, t.s.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float x0 = x[2 * e], x1 = x[2 * e + 1];
    x[2 * e] = fmaf(x0, cs[e], -__fmul_rn(x1, sn[e]));
    x[2 * e + 1] = fmaf(x0, sn[e], __fmul_rn(x1, cs[e]));
  }
}

// Eight floats times f as eight fp16 values (round to nearest even).
__device__ __forceinline__ uint4 pack8_half(const float* v, float f) {
  uint4 out;
  uint32_t* w = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __half2 hv = __floats2half2_rn(v[2 * e] * f, v[2 * e + 1] * f);
    w[e] = *reinterpret_cast<uint32_t*>(&hv);
  }
  return out;
}

// Rotate (in place) NC consecutive elements starting at an even dimension d0
// by the RoPE angles of position pos: pairs (x[2i], x[2i+1]) -> (x0 c - x1 s,
// x0 s + x1 c). inverse = true applies the transpose rotation. For NC a
// multiple of 8, d0 must be a multiple of 8 and the tables 16-byte aligned:
// four pairs' cos and sin then come in one 16-byte load each. The rounding is
// spelled out (one product, then one fused multiply-add), so every kernel
// that rotates the same value gets the same bits: the backward recomputes
// the forward's scores from its own rotated copies.
template <int NC, int D>
__device__ __forceinline__ void rope_pairs(float* x, const float* rc, const float* rs,
                                           int pos, int d0, bool inverse) {
  if constexpr (NC % 8 == 0) {
    const float4* c4 = reinterpret_cast<const float4*>(rc + (size_t)pos * (D / 2) + (d0 >> 1));
    const float4* s4 = reinterpret_cast<const float4*>(rs + (size_t)pos * (D / 2) + (d0 >> 1));
#pragma unroll
    for (int q = 0; q < NC / 8; ++q) {
      const float4 cq = c4[q], sq0 = s4[q];
      const float cs[4] = {cq.x, cq.y, cq.z, cq.w};
      const float sn[4] = {inverse ? -sq0.x : sq0.x, inverse ? -sq0.y : sq0.y,
                           inverse ? -sq0.z : sq0.z, inverse ? -sq0.w : sq0.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = x[8 * q + 2 * e], x1 = x[8 * q + 2 * e + 1];
        x[8 * q + 2 * e] = fmaf(x0, cs[e], -__fmul_rn(x1, sn[e]));
        x[8 * q + 2 * e + 1] = fmaf(x0, sn[e], __fmul_rn(x1, cs[e]));
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < NC; c += 2) {
      const int pi = (d0 + c) >> 1;
      const float cs = rc[(size_t)pos * (D / 2) + pi];
      const float sn = inverse ? -rs[(size_t)pos * (D / 2) + pi] : rs[(size_t)pos * (D / 2) + pi];
      const float x0 = x[c], x1 = x[c + 1];
      x[c] = fmaf(x0, cs, -__fmul_rn(x1, sn));
      x[c + 1] = fmaf(x0, sn, __fmul_rn(x1, cs));
    }
  }
}
