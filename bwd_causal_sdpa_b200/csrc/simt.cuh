// simt.cuh -- fp32-arithmetic (CUDA cores) attention kernels.
//
// These carry the float32 storage path (whose error bound, 1e-5 relative,
// is out of reach of any reduced-precision tensor-core format) and serve as
// an independent-in-structure second implementation of the bf16 path. Every
// product and sum is fp32 FMA; exponentials use expf.
//
// Index conventions: bh = b*H + h; a row of one (b, h) slice is t in [0, T);
// doc_start / doc_end (when non-null) hold flattened token indices b*T + t.
// Grouped-query attention: k, v (and dk, dv) have Hkv heads; query head h
// reads key/value head h / (H / Hkv).
#pragma once

#include "common.cuh"

struct DocView {
  const int32_t* start;  // nullable
  const int32_t* end;    // nullable
  int row0;              // b*T
  int T;
  __device__ __forceinline__ int dstart(int t) const { return start ? start[row0 + t] - row0 : 0; }
  __device__ __forceinline__ int dend(int t) const { return end ? end[row0 + t] - row0 : T; }
};

// ---------------------------------------------------------------------------
// Forward: 16 query rows per block (4 per warp), keys streamed through shared
// memory 32 at a time; lane j scores key j, then the warp folds the chunk into
// each row's running max / sum and its output accumulator.
// ---------------------------------------------------------------------------
template <typename TIO, int D>
__global__ void __launch_bounds__(128) simt_fwd_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k, const TIO* __restrict__ v,
    const float* __restrict__ rc, const float* __restrict__ rs,
    const int32_t* __restrict__ doc_start, TIO* __restrict__ o, float* __restrict__ lse,
    int H, int Hkv, int T, float scale) {
  pdl_wait_and_trigger();
  constexpr int ROWS = 16, KC = 32, NC = D / 32, KP = D + 4;
  __shared__ __align__(16) float sQ[ROWS][D];
  __shared__ __align__(16) float sK[KC][KP];
  __shared__ __align__(16) float sV[KC][D];

  const int bh = blockIdx.x, b = bh / H;
  const int i0 = (gridDim.y - 1 - blockIdx.y) * ROWS;  // longest rows first
  const size_t base = (size_t)bh * T * D;
  const size_t kvbase = ((size_t)b * Hkv + (bh % H) / (H / Hkv)) * T * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const DocView doc{doc_start, nullptr, b * T, T};

  for (int idx = tid; idx < ROWS * (D / 2); idx += 128) {
    const int r = idx / (D / 2), pi = idx % (D / 2), t = i0 + r;
    float x[2] = {0.f, 0.f};
    if (t < T) {
      load_vec<2>(q + base + (size_t)t * D + 2 * pi, x);
      if (rc) rope_pairs<2, D>(x, rc, rs, t - doc.dstart(t), 2 * pi, false);
    }
    sQ[r][2 * pi] = x[0] * scale;
    sQ[r][2 * pi + 1] = x[1] * scale;
  }
  const int iend = min(i0 + ROWS, T);
  const int kv_lo = doc.dstart(i0);

  float m[4], l[4], acc[4][NC];
  int dsi[4];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[rr][c] = 0.f;
    const int i = i0 + warp * 4 + rr;
    dsi[rr] = i < T ? doc.dstart(i) : 0;
  }

  for (int kb = kv_lo; kb < iend; kb += KC) {
    __syncthreads();
    for (int idx = tid; idx < KC * (D / 2); idx += 128) {
      const int r = idx / (D / 2), pi = idx % (D / 2), t = kb + r;
      float x[2] = {0.f, 0.f}, y[2] = {0.f, 0.f};
      if (t < iend) {
        load_vec<2>(k + kvbase + (size_t)t * D + 2 * pi, x);
        if (rc) rope_pairs<2, D>(x, rc, rs, t - doc.dstart(t), 2 * pi, false);
        load_vec<2>(v + kvbase + (size_t)t * D + 2 * pi, y);
      }
      sK[r][2 * pi] = x[0];
      sK[r][2 * pi + 1] = x[1];
      sV[r][2 * pi] = y[0];
      sV[r][2 * pi + 1] = y[1];
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = warp * 4 + rr, i = i0 + r;
      if (i >= T) break;
      const int j = kb + lane;
      float s = -INFINITY;
      if (j <= i && j >= dsi[rr]) {
        float a = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; d += 4) {
          const float4 kk = *reinterpret_cast<const float4*>(&sK[lane][d]);
          const float4 qq = *reinterpret_cast<const float4*>(&sQ[r][d]);
          a = fmaf(qq.x, kk.x, a);
          a = fmaf(qq.y, kk.y, a);
          a = fmaf(qq.z, kk.z, a);
          a = fmaf(qq.w, kk.w, a);
        }
        s = a;
      }
      const float cm = warp_max(s);
      if (cm == -INFINITY) continue;
      const float mn = fmaxf(m[rr], cm);
      const float corr = expf(m[rr] - mn);
      const float p = (s == -INFINITY) ? 0.f : expf(s - mn);
      l[rr] = l[rr] * corr + warp_sum(p);
#pragma unroll
      for (int c = 0; c < NC; ++c) acc[rr][c] *= corr;
#pragma unroll 4
      for (int jj = 0; jj < KC; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, p, jj);
        float vv[NC];
        load_vec<NC>(&sV[jj][lane * NC], vv);
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[rr][c] = fmaf(pj, vv[c], acc[rr][c]);
      }
      m[rr] = mn;
    }
  }
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int i = i0 + warp * 4 + rr;
    if (i >= T) break;
    const float inv = 1.f / l[rr];
    float out[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) out[c] = acc[rr][c] * inv;
    store_vec<NC>(o + base + (size_t)i * D + lane * NC, out);
    if (lane == 0) lse[(size_t)bh * T + i] = m[rr] + logf(l[rr]);
  }
}

// ---------------------------------------------------------------------------
// Backward, key-parallel part: 32 keys per block (8 per warp, lanes over D);
// query rows from the block's first key to the end of its last key's document
// are streamed through shared memory. Accumulates dv = P^T dO and
// dk = scale * dS^T q_r, then rotates dk back (R^T) and stores dk, dv.
// ---------------------------------------------------------------------------
template <typename TIO, int D>
__global__ void __launch_bounds__(128) simt_dkdv_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k, const TIO* __restrict__ v,
    const TIO* __restrict__ dO, const float* __restrict__ lse, const float* __restrict__ delta,
    const float* __restrict__ rc, const float* __restrict__ rs,
    const int32_t* __restrict__ doc_start, const int32_t* __restrict__ doc_end,
    TIO* __restrict__ dk, TIO* __restrict__ dv, int H, int Hkv, int T, float scale) {
  pdl_wait_and_trigger();
  constexpr int KC = 32, QC = 32, NC = D / 32, KW = 8;
  __shared__ __align__(16) float sQ[QC][D];
  __shared__ __align__(16) float sG[QC][D];
  __shared__ float sL[QC], sDl[QC];

  const int bhk = blockIdx.x, b = bhk / Hkv;  // key/value head of this block
  const int G = H / Hkv;                       // query heads reading it
  const int j0 = (gridDim.y - 1 - blockIdx.y) * KC;
  const size_t base = (size_t)bhk * T * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const DocView doc{doc_start, doc_end, b * T, T};

  float kr[KW][NC], vv[KW][NC], dka[KW][NC], dva[KW][NC];
  int de[KW];
#pragma unroll
  for (int kk = 0; kk < KW; ++kk) {
    const int j = j0 + warp * KW + kk;
#pragma unroll
    for (int c = 0; c < NC; ++c) { kr[kk][c] = vv[kk][c] = dka[kk][c] = dva[kk][c] = 0.f; }
    de[kk] = -1;
    if (j < T) {
      load_vec<NC>(k + base + (size_t)j * D + lane * NC, kr[kk]);
      if (rc) rope_pairs<NC, D>(kr[kk], rc, rs, j - doc.dstart(j), lane * NC, false);
      load_vec<NC>(v + base + (size_t)j * D + lane * NC, vv[kk]);
      de[kk] = doc.dend(j);
    }
  }
  const int jlast = min(j0 + KC, T) - 1;
  const int qhi = doc.dend(jlast);

  for (int gi = 0; gi < G; ++gi) {
  const int bhq = b * H + (bhk % Hkv) * G + gi;  // a query head of the group
  const size_t qbase = (size_t)bhq * T * D;
  for (int ib = j0; ib < qhi; ib += QC) {
    __syncthreads();
    for (int idx = tid; idx < QC * (D / 2); idx += 128) {
      const int r = idx / (D / 2), pi = idx % (D / 2), t = ib + r;
      float x[2] = {0.f, 0.f}, g[2] = {0.f, 0.f};
      if (t < qhi) {
        load_vec<2>(q + qbase + (size_t)t * D + 2 * pi, x);
        if (rc) rope_pairs<2, D>(x, rc, rs, t - doc.dstart(t), 2 * pi, false);
        load_vec<2>(dO + qbase + (size_t)t * D + 2 * pi, g);
      }
      sQ[r][2 * pi] = x[0];
      sQ[r][2 * pi + 1] = x[1];
      sG[r][2 * pi] = g[0];
      sG[r][2 * pi + 1] = g[1];
    }
    if (tid < QC) {
      const int t = ib + tid;
      sL[tid] = t < qhi ? lse[(size_t)bhq * T + t] : 0.f;
      sDl[tid] = t < qhi ? delta[(size_t)bhq * T + t] : 0.f;
    }
    __syncthreads();
    const int iend = min(ib + QC, qhi);
    for (int i = ib; i < iend; ++i) {
      const int ii = i - ib;
      float qi[NC], gi[NC];
      load_vec<NC>(&sQ[ii][lane * NC], qi);
      load_vec<NC>(&sG[ii][lane * NC], gi);
      const float Li = sL[ii], Di = sDl[ii];
#pragma unroll
      for (int kk = 0; kk < KW; ++kk) {
        const int j = j0 + warp * KW + kk;
        if (j > i || i >= de[kk]) continue;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          s = fmaf(qi[c], kr[kk][c], s);
          dp = fmaf(gi[c], vv[kk][c], dp);
        }
        s = warp_sum(s);
        dp = warp_sum(dp);
        const float p = expf(s * scale - Li);
        const float dsv = p * (dp - Di);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          dva[kk][c] = fmaf(p, gi[c], dva[kk][c]);
          dka[kk][c] = fmaf(dsv, qi[c], dka[kk][c]);
        }
      }
    }
  }
  __syncthreads();  // the next query head restages the shared tiles
  }
#pragma unroll
  for (int kk = 0; kk < KW; ++kk) {
    const int j = j0 + warp * KW + kk;
    if (j >= T) break;
#pragma unroll
    for (int c = 0; c < NC; ++c) dka[kk][c] *= scale;
    if (rc) rope_pairs<NC, D>(dka[kk], rc, rs, j - doc.dstart(j), lane * NC, true);
    store_vec<NC>(dk + base + (size_t)j * D + lane * NC, dka[kk]);
    store_vec<NC>(dv + base + (size_t)j * D + lane * NC, dva[kk]);
  }
}

// ---------------------------------------------------------------------------
// Backward, query-parallel dq pass: 32 query rows per block (8 per warp,
// lanes over D), keys of the rows' documents streamed through shared memory.
// dq = R^T (scale * dS k_r).
// ---------------------------------------------------------------------------
template <typename TIO, int D>
__global__ void __launch_bounds__(128) simt_dq_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k, const TIO* __restrict__ v,
    const TIO* __restrict__ dO, const float* __restrict__ lse, const float* __restrict__ delta,
    const float* __restrict__ rc, const float* __restrict__ rs,
    const int32_t* __restrict__ doc_start, TIO* __restrict__ dq, int H, int Hkv, int T,
    float scale) {
  pdl_wait_and_trigger();
  constexpr int QC = 32, KC = 32, NC = D / 32, QW = 8;
  __shared__ __align__(16) float sK[KC][D];
  __shared__ __align__(16) float sV[KC][D];

  const int bh = blockIdx.x, b = bh / H;
  const int i0 = (gridDim.y - 1 - blockIdx.y) * QC;
  const size_t base = (size_t)bh * T * D;
  const size_t kvbase = ((size_t)b * Hkv + (bh % H) / (H / Hkv)) * T * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const DocView doc{doc_start, nullptr, b * T, T};

  float qr[QW][NC], gi[QW][NC], dqa[QW][NC], L[QW], Dl[QW];
  int dsi[QW];
#pragma unroll
  for (int rr = 0; rr < QW; ++rr) {
    const int i = i0 + warp * QW + rr;
#pragma unroll
    for (int c = 0; c < NC; ++c) { qr[rr][c] = gi[rr][c] = dqa[rr][c] = 0.f; }
    L[rr] = Dl[rr] = 0.f;
    dsi[rr] = T + 1;  // no key passes for rows beyond T
    if (i < T) {
      load_vec<NC>(q + base + (size_t)i * D + lane * NC, qr[rr]);
      const int ds = doc.dstart(i);
      if (rc) rope_pairs<NC, D>(qr[rr], rc, rs, i - ds, lane * NC, false);
#pragma unroll
      for (int c = 0; c < NC; ++c) qr[rr][c] *= scale;
      load_vec<NC>(dO + base + (size_t)i * D + lane * NC, gi[rr]);
      L[rr] = lse[(size_t)bh * T + i];
      Dl[rr] = delta[(size_t)bh * T + i];
      dsi[rr] = ds;
    }
  }
  const int kv_lo = doc.dstart(i0);
  const int kv_hi = min(i0 + QC, T);
  for (int jb = kv_lo; jb < kv_hi; jb += KC) {
    __syncthreads();
    for (int idx = tid; idx < KC * (D / 2); idx += 128) {
      const int r = idx / (D / 2), pi = idx % (D / 2), t = jb + r;
      float x[2] = {0.f, 0.f}, y[2] = {0.f, 0.f};
      if (t < kv_hi) {
        load_vec<2>(k + kvbase + (size_t)t * D + 2 * pi, x);
        if (rc) rope_pairs<2, D>(x, rc, rs, t - doc.dstart(t), 2 * pi, false);
        load_vec<2>(v + kvbase + (size_t)t * D + 2 * pi, y);
      }
      sK[r][2 * pi] = x[0];
      sK[r][2 * pi + 1] = x[1];
      sV[r][2 * pi] = y[0];
      sV[r][2 * pi + 1] = y[1];
    }
    __syncthreads();
    const int jend = min(jb + KC, kv_hi);
    for (int j = jb; j < jend; ++j) {
      float kj[NC], vj[NC];
      load_vec<NC>(&sK[j - jb][lane * NC], kj);
      load_vec<NC>(&sV[j - jb][lane * NC], vj);
#pragma unroll
      for (int rr = 0; rr < QW; ++rr) {
        const int i = i0 + warp * QW + rr;
        if (j > i || j < dsi[rr]) continue;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          s = fmaf(qr[rr][c], kj[c], s);
          dp = fmaf(gi[rr][c], vj[c], dp);
        }
        s = warp_sum(s);
        dp = warp_sum(dp);
        const float p = expf(s - L[rr]);
        const float dsv = p * (dp - Dl[rr]);
#pragma unroll
        for (int c = 0; c < NC; ++c) dqa[rr][c] = fmaf(dsv, kj[c], dqa[rr][c]);
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < QW; ++rr) {
    const int i = i0 + warp * QW + rr;
    if (i >= T) break;
#pragma unroll
    for (int c = 0; c < NC; ++c) dqa[rr][c] *= scale;
    if (rc) rope_pairs<NC, D>(dqa[rr], rc, rs, i - dsi[rr], lane * NC, true);
    store_vec<NC>(dq + base + (size_t)i * D + lane * NC, dqa[rr]);
  }
}
