// prep.cuh -- small preprocessing kernels: packed-document ranges and the
// backward's row term Delta_i = sum_d dO[i][d] * o[i][d].
#pragma once

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
