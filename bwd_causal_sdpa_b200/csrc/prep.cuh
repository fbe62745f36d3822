// prep.cuh -- small preprocessing kernels: packed-document ranges and the
// backward's row term Delta_i = sum_d dO[i][d] * o[i][d].
#pragma once

#include <type_traits>

#include "common.cuh"

// From cu_seqlens (over the flattened B*T token axis, end marker B*T) build,
// for every token, the flattened index where its document starts and where it
// ends (exclusive). One block: thread 0 walks the array up to the end marker
// (never past it) and validates it; then all threads fill the per-token
// arrays by binary search. A malformed array sets ATTN_EDEVICE_INPUT and the
// arrays fall back to "each row is one document", so later kernels stay in
// bounds. (Cort33x, "Preserving context in the data": documents packed into
// one window; attention stays within a document.)
__global__ void __launch_bounds__(1024) doc_ranges_kernel(const int32_t* __restrict__ cu, int B, int T,
                                                          int32_t* __restrict__ doc_start,
                                                          int32_t* __restrict__ doc_end) {
  pdl_wait_and_trigger();
  __shared__ int s_ok, s_n;
  const int BT = B * T;
  if (threadIdx.x == 0) {
    int ok = 1, n = 0;
    int prev = cu[0];
    if (prev != 0) ok = 0;
    // Strictly rising values bounded by BT: at most BT steps.
    while (ok && prev < BT) {
      const int nxt = cu[n + 1];  // exists: prev < BT is not the end marker
      if (nxt <= prev || nxt > BT || (prev / T) != ((nxt - 1) / T)) {
        ok = 0;
        break;
      }
      prev = nxt;
      ++n;
    }
    s_ok = ok;
    s_n = n;
  }
  __syncthreads();
  if (s_ok) {
    const int n = s_n;
    for (int t = threadIdx.x; t < BT; t += blockDim.x) {
      int lo = 0, hi = n;  // cu[lo] <= t < cu[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid;
      }
      doc_start[t] = cu[lo];
      doc_end[t] = cu[hi];
    }
  } else {
    if (threadIdx.x == 0) report_status(ATTN_EDEVICE_INPUT);
    for (int t = threadIdx.x; t < BT; t += blockDim.x) {
      doc_start[t] = (t / T) * T;
      doc_end[t] = (t / T) * T + T;
    }
  }
}

// Delta_i = sum_d dO[i][d] * o[i][d] in fp32, one warp per row of the
// flattened [B*H*T, D] view.
template <typename TIO, int D>
__global__ void __launch_bounds__(256) delta_kernel(const TIO* __restrict__ o, const TIO* __restrict__ dO,
                                                   float* __restrict__ delta, long rows) {
  pdl_wait_and_trigger();
  constexpr int NC = D / 32;
  const long row = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float a[NC], g[NC];
  load_vec<NC>(o + row * D + lane * NC, a);
  load_vec<NC>(dO + row * D + lane * NC, g);
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < NC; ++c) s = fmaf(a[c], g[c], s);
  s = warp_sum(s);
  if (lane == 0) delta[row] = s;
}

// RoPE pre-pass for the tensor-core kernels: rotate q and k once (fp32
// arithmetic, interleaved pairs at the token's document position) and store
// the rotated tiles in the 16-bit type the MMAs read. blockIdx = (128-row
// tile, head, 0 for q / 1 for k); the head is b*H + h for q and b*Hkv + h
// for k (blocks past B*Hkv return at once).
//
// kTileScale (forward, fp16 output): fp16 keeps 3 more mantissa bits than
// bf16, which the lse bound needs, but has a narrow range; a tile whose
// largest magnitude reaches 2^14 is multiplied by a power of two that brings
// it into [2^14, 2^15), and fac[] receives the inverse factor (exact), which
// the forward folds into its score scale. Without kTileScale (bf16 output)
// values are stored as they are.
constexpr int kRopePrepThreads = 512;

template <typename OutT, int D, bool kTileScale>
__global__ void __launch_bounds__(kRopePrepThreads) rope_prep_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const float* __restrict__ rc, const float* __restrict__ rs,
    const int32_t* __restrict__ doc_start, OutT* __restrict__ qo, OutT* __restrict__ ko,
    float* __restrict__ qfac, float* __restrict__ kfac, int H, int Hkv, int T, int ntiles) {
  pdl_wait_and_trigger();
  constexpr int CH = D / 8;              // 16-byte chunks per row
  constexpr int NT = kRopePrepThreads;
  constexpr int PER = 128 * CH / NT;     // chunks per thread
  // grid (ntiles, B*H, 2): z = 0 rotates q heads, z = 1 the B*Hkv k heads
  const int tile = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const int heads = which ? Hkv : H;
  const int b = bh / heads, row0 = b * T, t0 = tile * 128;
  if (b >= (int)gridDim.y / H) return;  // k has fewer heads than q
  const __nv_bfloat16* src = which ? k : q;
  OutT* dst = which ? ko : qo;
  float v[PER][8];
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int idx = threadIdx.x + u * NT, r = idx / CH, c8 = idx % CH, t = t0 + r;
#pragma unroll
    for (int e = 0; e < 8; ++e) v[u][e] = 0.f;
    if (t < T) {
      const uint4 raw = *reinterpret_cast<const uint4*>(src + ((size_t)bh * T + t) * D + c8 * 8);
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[u][e] = __bfloat162float(h[e]);
      const int pos = t - (doc_start ? doc_start[row0 + t] - row0 : 0);
      rope_pairs<8, D>(v[u], rc, rs, pos, c8 * 8, false);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[u][e]));
    }
  }
  float f = 1.f;
  if constexpr (kTileScale) {
    __shared__ float red[NT / 32];
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) amax = fmaxf(amax, red[w]);
    if (amax >= 16384.f && amax <= 3.0e38f) f = ldexpf(1.f, 14 - ilogbf(amax));
    if (threadIdx.x == 0) (which ? kfac : qfac)[bh * ntiles + tile] = 1.f / f;
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int idx = threadIdx.x + u * NT, r = idx / CH, c8 = idx % CH, t = t0 + r;
    if (t >= T) continue;
    uint4 out;
    uint32_t* w = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if constexpr (sizeof(OutT) == 2 && std::is_same<OutT, __half>::value) {
        __half2 hv = __floats2half2_rn(v[u][2 * e] * f, v[u][2 * e + 1] * f);
        w[e] = *reinterpret_cast<uint32_t*>(&hv);
      } else {
        __nv_bfloat162 hv = __floats2bfloat162_rn(v[u][2 * e] * f, v[u][2 * e + 1] * f);
        w[e] = *reinterpret_cast<uint32_t*>(&hv);
      }
    }
    *reinterpret_cast<uint4*>(dst + ((size_t)bh * T + t) * D + c8 * 8) = out;
  }
}

// Eight bf16 values (16 bytes) as fp32, and back.
__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* p, float* v) {
  const uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = __low2float(h[e]);
    v[2 * e + 1] = __high2float(h[e]);
  }
}
__device__ __forceinline__ void store8_bf16(__nv_bfloat16* p, const float* v) {
  uint4 raw;
  uint32_t* w = reinterpret_cast<uint32_t*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    w[e] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = raw;
}

// Backward preprocessing for the tensor-core path over the tile-padded
// [B*H][ntiles*128] row view, D/8 threads per row (16 bytes of each bf16 row
// per thread, so a warp covers 32*8/D whole rows): stores -Delta_i (Delta_i =
// sum_d dO[i][d] * o[i][d]) and -lse_i * log2(e), negated so the main kernel
// folds them in with one fused multiply-add (both 0 for padding rows t >= T,
// so its per-tile loads never leave the arrays), zeroes the fp32 dq
// accumulator row and, with RoPE tables, writes the rotated q and k rows
// (bf16) the main kernel reads; when the grouped-query backward splits its
// groups, it also zeroes the fp32 dk, dv accumulator rows. The grid covers
// rows_pad * D/8 threads exactly (rows_pad is a multiple of 128), so every
// warp is full.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ lse, float* __restrict__ delta_pad, float* __restrict__ lse2_pad,
    float* __restrict__ dq_acc, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k, const float* __restrict__ rc,
    const float* __restrict__ rs, const int32_t* __restrict__ doc_start,
    __nv_bfloat16* __restrict__ qr, __nv_bfloat16* __restrict__ kr, float* __restrict__ dk_acc,
    float* __restrict__ dv_acc, int H, int Hkv, int T, int Tpad, long rows_pad) {
  pdl_wait_and_trigger();
  constexpr int TPR = D / 8;  // threads per row
  const long gt = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long row = gt / TPR;
  const int c8 = (int)(gt - row * TPR) * 8;
  const long bh = row / Tpad;
  const int t = (int)(row - bh * Tpad);
  float s = 0.f;
  if (row < rows_pad && t < T) {
    const long r = bh * T + t;
    float a[8], g[8];
    load8_bf16(o + r * D + c8, a);
    load8_bf16(dO + r * D + c8, g);
#pragma unroll
    for (int e = 0; e < 8; ++e) s = fmaf(a[e], g[e], s);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float4*>(dq_acc + r * D + c8)[0] = z;
    reinterpret_cast<float4*>(dq_acc + r * D + c8)[1] = z;
    if (dk_acc && bh < (rows_pad / Tpad) / H * Hkv) {  // a row of the [B*Hkv][T] view
      reinterpret_cast<float4*>(dk_acc + r * D + c8)[0] = z;
      reinterpret_cast<float4*>(dk_acc + r * D + c8)[1] = z;
      reinterpret_cast<float4*>(dv_acc + r * D + c8)[0] = z;
      reinterpret_cast<float4*>(dv_acc + r * D + c8)[1] = z;
    }
    if (rc) {
      const int b = (int)(bh / H);
      const int pos = t - (doc_start ? doc_start[b * T + t] - b * T : 0);
      float x[8];
      load8_bf16(q + r * D + c8, x);
      rope_pairs<8, D>(x, rc, rs, pos, c8, false);
      store8_bf16(qr + r * D + c8, x);
      // row r of the [B*Hkv][T] k view exists for the first B*Hkv heads; its
      // batch (hence document layout) is bh / Hkv
      if (bh < (rows_pad / Tpad) / H * Hkv) {
        const int bk = (int)(bh / Hkv);
        const int posk = t - (doc_start ? doc_start[bk * T + t] - bk * T : 0);
        load8_bf16(k + r * D + c8, x);
        rope_pairs<8, D>(x, rc, rs, posk, c8, false);
        store8_bf16(kr + r * D + c8, x);
      }
    }
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (c8 == 0 && row < rows_pad) {
    delta_pad[row] = -s;
    lse2_pad[row] = t < T ? -lse[bh * T + t] * 1.4426950408889634f : 0.f;
  }
}

// dq = R(pos)^T (scale * dq_acc), stored as bf16; one thread per 8 values.
template <int D>
__global__ void __launch_bounds__(256) dq_finalize_kernel(
    const float* __restrict__ dq_acc, const float* __restrict__ rc, const float* __restrict__ rs,
    const int32_t* __restrict__ doc_start, __nv_bfloat16* __restrict__ dq, int H, int T,
    float scale, long n8) {
  pdl_wait_and_trigger();
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n8) return;
  const long e0 = idx * 8;
  const long row = e0 / D;  // bh*T + t
  const int d0 = (int)(e0 - row * D);
  const int t = (int)(row % T);
  const int b = (int)((row / T) / H);
  float v[8];
  load_vec<4>(dq_acc + e0, v);
  load_vec<4>(dq_acc + e0 + 4, v + 4);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] *= scale;
  if (rc) {
    const int pos = t - (doc_start ? doc_start[b * T + t] - b * T : 0);
    rope_pairs<8, D>(v, rc, rs, pos, d0, true);
  }
  store_vec<4>(dq + e0, v);
  store_vec<4>(dq + e0 + 4, v + 4);
}
