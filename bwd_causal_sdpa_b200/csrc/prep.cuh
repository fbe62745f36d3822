// prep.cuh -- small preprocessing kernels: packed-document ranges and the
// backward's row term Delta_i = sum_d dO[i][d] * o[i][d].
#pragma once

#include "common.cuh"

// From cu_seqlens (over the flattened B*T token axis, end marker B*T) build,
// for every token, the flattened index where its document starts and where it
// ends (exclusive). One block: thread 0 walks the array up to the end marker
// (never past it), validates it and copies up to kDocRangesSmem + 1
// boundaries into shared memory; then all threads fill the per-token arrays
// by binary search over that copy (over the global array when it has more
// documents). A malformed array sets ATTN_EDEVICE_INPUT and the arrays fall
// back to "each row is one document", so later kernels stay in bounds.
// (Cort33x, "Preserving context in the data": documents packed into one
// window; attention stays within a document.)
constexpr int kDocRangesSmem = 4096;

__global__ void __launch_bounds__(1024) doc_ranges_kernel(const int32_t* __restrict__ cu, int B, int T,
                                                          int32_t* __restrict__ doc_start,
                                                          int32_t* __restrict__ doc_end) {
  pdl_wait_and_trigger();
  __shared__ int s_cu[kDocRangesSmem + 1];
  __shared__ int s_ok, s_n;
  const int BT = B * T;
  if (threadIdx.x == 0) {
    int ok = 1, n = 0;
    int prev = cu[0];
    if (prev != 0) ok = 0;
    s_cu[0] = prev;
    // Strictly rising values bounded by BT: at most BT steps.
    while (ok && prev < BT) {
      const int nxt = cu[n + 1];  // exists: prev < BT is not the end marker
      if (nxt <= prev || nxt > BT || (prev / T) != ((nxt - 1) / T)) {
        ok = 0;
        break;
      }
      prev = nxt;
      ++n;
      if (n <= kDocRangesSmem) s_cu[n] = nxt;
    }
    s_ok = ok;
    s_n = n;
  }
  __syncthreads();
  if (s_ok) {
    const int n = s_n;
    const int32_t* bounds = n <= kDocRangesSmem ? s_cu : cu;
    for (int t = threadIdx.x; t < BT; t += blockDim.x) {
      int lo = 0, hi = n;  // bounds[lo] <= t < bounds[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (bounds[mid] <= t) lo = mid; else hi = mid;
      }
      doc_start[t] = bounds[lo];
      doc_end[t] = bounds[hi];
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

// RoPE pre-pass for the forward: rotate q and k once (fp32 arithmetic,
// interleaved pairs at the token's document position) and store every
// 128-row tile as fp16 times its power-of-two factor (fp16_tile_factor of the
// tile's largest pair norm); fac[] receives the inverse factor (exact), which
// the forward folds into its score scale. blockIdx = (128-row tile, head,
// 0 for q / 1 for k); the head is b*H + h for q and b*Hkv + h for k (blocks
// past B*Hkv return at once).
constexpr int kRopePrepThreads = 512;

template <int D>
__global__ void __launch_bounds__(kRopePrepThreads) rope_prep_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const float* __restrict__ rc, const float* __restrict__ rs,
    const int32_t* __restrict__ doc_start, __half* __restrict__ qo, __half* __restrict__ ko,
    float* __restrict__ qfac, float* __restrict__ kfac, int B, int H, int Hkv, int T,
    int ntiles) {
  pdl_wait_and_trigger();
  constexpr int CH = D / 8;              // 16-byte chunks per row
  constexpr int NT = kRopePrepThreads;
  constexpr int PER = 128 * CH / NT;     // chunks per thread
  const int tile = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const int heads = which ? Hkv : H;
  if (bh >= B * heads) return;  // k has fewer heads than q
  const int b = bh / heads, row0 = b * T, t0 = tile * 128;
  const __nv_bfloat16* src = which ? k : q;
  __half* dst = which ? ko : qo;
  float v[PER][8];
  float n2 = 0.f;
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
      n2 = fmaxf(n2, pair_norm2_max8(v[u]));
    }
  }
  __shared__ float red[NT / 32];
  n2 = warp_max(n2);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = n2;
  __syncthreads();
  n2 = red[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) n2 = fmaxf(n2, red[w]);
  const float f = fp16_tile_factor(sqrtf(n2));
  if (threadIdx.x == 0) (which ? kfac : qfac)[(size_t)bh * ntiles + tile] = 1.f / f;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int idx = threadIdx.x + u * NT, r = idx / CH, c8 = idx % CH, t = t0 + r;
    if (t >= T) continue;
    rope_pairs<8, D>(v[u], rc, rs, t - (doc_start ? doc_start[row0 + t] - row0 : 0), c8 * 8, false);
    *reinterpret_cast<uint4*>(dst + ((size_t)bh * T + t) * D + c8 * 8) = pack8_half(v[u], f);
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

// Backward preprocessing for the tensor-core path, one block per (128-row
// tile, query head bh). Per row it stores -Delta_i (Delta_i = sum_d dO[i][d]
// * o[i][d]) and -lse_i * log2(e) in the tile-padded [B*H][Tpad] arrays,
// negated so the main kernel folds them in with one fused multiply-add (both
// 0 for rows t >= T, so its per-tile loads never leave the arrays), and
// zeroes the row of the fp32 dq accumulator (when the grouped-query backward
// splits its groups, also of the dk, dv accumulators: blocks with bh below
// B*Hkv take those rows of key/value head bh). Per tile it records the
// largest |dO_i| (Euclidean norm) and |Delta_i|, which bound dS for the main
// kernel's fp16 scaling.
//
// kRope: the tile's q rows (and, for bh below B*Hkv, the same rows of key/value
// head bh's k) are rotated and stored as fp16 times the tile's power-of-two
// factor (fp16_tile_factor of the largest pair norm, found in the first read
// of the rows), with the inverse factors in qinv (a 16-byte record per tile,
// value first, so the main kernel can bulk-load it) and kinv: the same values the
// forward's scores were computed from, so the main kernel recomputes exactly
// those scores. The rows are read again (from cache) to be rotated.
constexpr int kBwdPrepThreads = 256;

template <int D, bool kRope>
__global__ void __launch_bounds__(kBwdPrepThreads) bwd_prep_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ lse, float* __restrict__ delta_pad, float* __restrict__ lse2_pad,
    float* __restrict__ dq_acc, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k, const float* __restrict__ rc,
    const float* __restrict__ rs, const int32_t* __restrict__ doc_start,
    __half* __restrict__ q16, __half* __restrict__ k16, float* __restrict__ qinv,
    float* __restrict__ kinv, float* __restrict__ dmax, float* __restrict__ deltamax,
    float* __restrict__ dk_acc, float* __restrict__ dv_acc, int B, int H, int Hkv, int T,
    int Tpad, int ntiles) {
  pdl_wait_and_trigger();
  constexpr int CPR = D / 8;                    // 16-byte chunks per row
  constexpr int RPP = kBwdPrepThreads / CPR;    // rows per pass
  constexpr int NP = 128 / RPP;                 // passes over the tile
  const int tile = blockIdx.x, bh = blockIdx.y;
  const int b = bh / H;
  const bool kv = bh < B * Hkv;  // also a key/value head index
  const int bk = kv ? bh / Hkv : 0;
  const int c = threadIdx.x % CPR, rsub = threadIdx.x / CPR;
  float dmx = 0.f, dlx = 0.f, aq = 0.f, ak = 0.f;
  for (int u = 0; u < NP; ++u) {
    const int t = tile * 128 + u * RPP + rsub;
    const bool valid = t < T;
    const size_t off = ((size_t)bh * T + (valid ? t : 0)) * D + 8 * c;
    float s = 0.f, n2 = 0.f;
    if (valid) {
      float a[8], g[8];
      load8_bf16(o + off, a);
      load8_bf16(dO + off, g);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        s = fmaf(a[e], g[e], s);
        n2 = fmaf(g[e], g[e], n2);
      }
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      reinterpret_cast<float4*>(dq_acc + off)[0] = z;
      reinterpret_cast<float4*>(dq_acc + off)[1] = z;
      if (dk_acc && kv) {
        reinterpret_cast<float4*>(dk_acc + off)[0] = z;
        reinterpret_cast<float4*>(dk_acc + off)[1] = z;
        reinterpret_cast<float4*>(dv_acc + off)[0] = z;
        reinterpret_cast<float4*>(dv_acc + off)[1] = z;
      }
      if constexpr (kRope) {  // the tiles' largest pair norms (squared), before rotating
        float x[8];
        load8_bf16(q + off, x);
        aq = fmaxf(aq, pair_norm2_max8(x));
        if (kv) {
          load8_bf16(k + off, x);
          ak = fmaxf(ak, pair_norm2_max8(x));
        }
      }
    }
    // a row's CPR chunks sit in consecutive lanes of one warp
#pragma unroll
    for (int sh = CPR / 2; sh > 0; sh >>= 1) {
      s += __shfl_xor_sync(0xffffffffu, s, sh);
      n2 += __shfl_xor_sync(0xffffffffu, n2, sh);
    }
    if (c == 0) {
      delta_pad[(size_t)bh * Tpad + t] = valid ? -s : 0.f;
      lse2_pad[(size_t)bh * Tpad + t] = valid ? -lse[(size_t)bh * T + t] * 1.4426950408889634f : 0.f;
    }
    if (valid) {
      dmx = fmaxf(dmx, sqrtf(n2));
      dlx = fmaxf(dlx, fabsf(s));
    }
  }
  __shared__ float red[4][kBwdPrepThreads / 32];
  dmx = warp_max(dmx);
  dlx = warp_max(dlx);
  aq = warp_max(aq);
  ak = warp_max(ak);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = dmx;
    red[1][w] = dlx;
    red[2][w] = aq;
    red[3][w] = ak;
  }
  __syncthreads();
  float m[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    m[j] = red[j][0];
#pragma unroll
    for (int i = 1; i < kBwdPrepThreads / 32; ++i) m[j] = fmaxf(m[j], red[j][i]);
  }
  const float fq = fp16_tile_factor(sqrtf(m[2])), fk = fp16_tile_factor(sqrtf(m[3]));
  if (threadIdx.x == 0) {
    dmax[(size_t)bh * ntiles + tile] = m[0];
    deltamax[(size_t)bh * ntiles + tile] = m[1];
    if (kRope) {
      reinterpret_cast<float4*>(qinv)[(size_t)bh * ntiles + tile] = make_float4(1.f / fq, 0.f, 0.f, 0.f);
      if (kv) kinv[(size_t)bh * ntiles + tile] = 1.f / fk;
    }
  }
  if constexpr (kRope) {
    for (int u = 0; u < NP; ++u) {
      const int t = tile * 128 + u * RPP + rsub;
      if (t >= T) continue;
      const size_t off = ((size_t)bh * T + t) * D + 8 * c;
      float x[8];
      load8_bf16(q + off, x);
      rope_pairs<8, D>(x, rc, rs, t - (doc_start ? doc_start[b * T + t] - b * T : 0), 8 * c, false);
      *reinterpret_cast<uint4*>(q16 + off) = pack8_half(x, fq);
      if (kv) {
        load8_bf16(k + off, x);
        rope_pairs<8, D>(x, rc, rs, t - (doc_start ? doc_start[bk * T + t] - bk * T : 0), 8 * c,
                         false);
        *reinterpret_cast<uint4*>(k16 + off) = pack8_half(x, fk);
      }
    }
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
