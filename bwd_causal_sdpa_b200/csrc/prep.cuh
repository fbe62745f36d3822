// prep.cuh -- small preprocessing kernels: packed-document ranges and the
// backward's row term Delta_i = sum_d dO[i][d] * o[i][d].
#pragma once

#include "common.cuh"

// From cu_seqlens (over the flattened B*T token axis, end marker B*T) build,
// for every token, the flattened index where its document starts and where it
// ends (exclusive). In every block thread 0 walks the array up to the end
// marker (never past it), validates it and copies up to kDocRangesSmem + 1
// boundaries into shared memory (the blocks reach the same verdict); then
// the block's threads fill their grid-stride share of the per-token arrays by
// binary search over that copy (over the global array when it has more
// documents). A malformed array sets ATTN_EDEVICE_INPUT (block 0) and the
// arrays fall back to "each row is one document", so later kernels stay in
// bounds. Any grid size is correct; doc_ranges_blocks gives the one used.
// (Cort33x, "Preserving context in the data": documents packed into one
// window; attention stays within a document.)
constexpr int kDocRangesSmem = 4096;
// one block per 2048 tokens, at most 64 (the walk is repeated per block)
inline unsigned doc_ranges_blocks(int B, int T) {
  const long bt = (long)B * T;
  const long g = (bt + 2047) / 2048;
  return (unsigned)(g < 1 ? 1 : (g > 64 ? 64 : g));
}

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
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < BT; t += gridDim.x * blockDim.x) {
      int lo = 0, hi = n;  // bounds[lo] <= t < bounds[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (bounds[mid] <= t) lo = mid; else hi = mid;
      }
      doc_start[t] = bounds[lo];
      doc_end[t] = bounds[hi];
    }
  } else {
    if (threadIdx.x == 0 && blockIdx.x == 0) report_status(ATTN_EDEVICE_INPUT);
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < BT; t += gridDim.x * blockDim.x) {
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

// RoPE pre-pass: rotate q and k once (fp32 arithmetic, interleaved pairs at
// the token's document position) and store every 128-row tile as fp16 times
// a power-of-two factor, fp16_tile_factor of the largest pair norm
// sqrt(x_2m^2 + x_2m+1^2) in the tile: a rotation keeps each pair's norm, so
// that bounds every rotated value (and is at most sqrt(2) times the largest
// of them), and it needs no table, so the factor is known before any
// rotation. qfac receives the inverse factor of each q tile as a 16-byte
// record (value first, so the backward's main kernel can bulk-load it with
// the tile), kfac that of each k tile; the forward folds them into its score
// scale and the backward's main kernel into its own, which therefore
// recomputes the forward's scores exactly (same values). hstat (backward
// only, else null): zeroed here (all B*H*4 slots, by the first block) for the
// row pass that follows, which fills it with atomic maxima.
//
// One block per (128-row tile, batch, head), heads numbered q heads first
// (0 .. H-1), then k heads (H .. H+Hkv-1): each thread loads its chunks of
// the tile, the block reduces the largest pair norm, and each thread rotates
// its chunks (table rows from L2) and stores them scaled. Small blocks with
// few registers and no shared tables keep many tiles in flight per SM.
constexpr int kRopePrepThreads = 256;

template <int D>
__global__ void __launch_bounds__(kRopePrepThreads) rope_prep_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const float* __restrict__ rc, const float* __restrict__ rs,
    const int32_t* __restrict__ doc_start, __half* __restrict__ qo, __half* __restrict__ ko,
    float* __restrict__ qfac, float* __restrict__ kfac, float* __restrict__ hstat, int B, int H,
    int Hkv, int T, int ntiles) {
  pdl_wait_and_trigger();
  constexpr int CH = D / 8;                        // 16-byte chunks per row
  constexpr int NT = kRopePrepThreads;
  constexpr int PER = 128 * CH / NT;               // chunks per thread
  __shared__ float red[NT / 32];
  const int tile = blockIdx.x, b = blockIdx.y, hh = blockIdx.z;
  const int row0 = b * T, t0 = tile * 128;
  if (hstat && tile == 0 && b == 0 && hh == 0)
    for (int e = threadIdx.x; e < 4 * B * H; e += NT) hstat[e] = 0.f;
  const bool is_k = hh >= H;
  const int bh = is_k ? b * Hkv + (hh - H) : b * H + hh;
  const __nv_bfloat16* src = (is_k ? k : q) + (size_t)bh * T * D;
  __half* dst = (is_k ? ko : qo) + (size_t)bh * T * D;
  const int c8 = threadIdx.x % CH;  // this thread's chunk column, rows threadIdx.x / CH + u * NT / CH
  // At D = 64 the tile waits for its factor in shared memory, not in
  // registers: more blocks per SM (rope_prep 0.0224 -> 0.0214 ms on the 237M
  // layer, same box); at D = 128 the register version measured faster.
  constexpr bool kStage = D == 64;
  __shared__ uint4 tile_s[kStage ? 128 * CH : 1];
  uint4 raw[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int t = t0 + (threadIdx.x + u * NT) / CH;
    raw[u] = t < T ? *reinterpret_cast<const uint4*>(src + (size_t)t * D + c8 * 8)
                   : make_uint4(0u, 0u, 0u, 0u);  // rows past T are zeros and stay zero
  }
  float n2 = 0.f;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    if constexpr (kStage) tile_s[threadIdx.x + u * NT] = raw[u];
    const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = __low2float(hv[e]), x1 = __high2float(hv[e]);
      n2 = fmaxf(n2, fmaf(x0, x0, x1 * x1));
    }
  }
  n2 = warp_max(n2);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = n2;
  __syncthreads();
  n2 = red[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) n2 = fmaxf(n2, red[w]);
  const float f = fp16_tile_factor(sqrtf(n2));
  if (threadIdx.x == 0) {
    const size_t ti = (size_t)bh * ntiles + tile;
    if (is_k) kfac[ti] = 1.f / f;
    else reinterpret_cast<float4*>(qfac)[ti] = make_float4(1.f / f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int t = t0 + (threadIdx.x + u * NT) / CH;
    if (t >= T) continue;
    const int pos = t - (doc_start ? doc_start[row0 + t] - row0 : 0);
    float v[8];
    const uint4 rw = kStage ? tile_s[threadIdx.x + u * NT] : raw[u];  // this thread's own chunk
    const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&rw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = __low2float(hv[e]);
      v[2 * e + 1] = __high2float(hv[e]);
    }
    rotate8(v, rope8_load<D>(rc, rs, pos, c8 * 8));
    *reinterpret_cast<uint4*>(dst + (size_t)t * D + c8 * 8) = pack8_half(v, f);
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

// Backward row pass for the tensor-core path over the tile-padded
// [B*H][Tpad] row view, D/8 threads per row (16 bytes of each bf16 row per
// thread, so a warp covers 32*8/D whole rows of one head): stores -Delta_i
// (Delta_i = sum_d dO[i][d] * o[i][d]) and -lse_i * log2(e), negated so the
// main kernel folds them in with one fused multiply-add (both 0 for padding
// rows t >= T, so its per-tile loads never leave the arrays), and zeroes the
// fp32 dq accumulator row; when the grouped-query backward splits its groups
// it also zeroes the fp32 dk, dv accumulator rows (rows of the first B*Hkv
// heads of the view). dq_acc null: dQ comes from the query-tile pass and no
// accumulator is used. hstat (fp16 operands, else null; [B*H][4]): per query
// head the largest |dO_i| (Euclidean norm) and |Delta_i|, per key/value head
// the largest |v_j| (slots zeroed by rope_prep, filled here by atomic maxima
// of non-negative floats), which bound dS for the main kernels' fp16 scaling.
// The grid covers rows_pad * D/8 threads exactly (rows_pad is a multiple of
// 128), so every warp is full.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ lse, float* __restrict__ delta_pad, float* __restrict__ lse2_pad,
    float* __restrict__ dq_acc, float* __restrict__ dk_acc, float* __restrict__ dv_acc,
    const __nv_bfloat16* __restrict__ v, float* __restrict__ hstat, int H, int Hkv, int T,
    int Tpad, long rows_pad) {
  pdl_wait_and_trigger();
  constexpr int TPR = D / 8;  // threads per row
  const long gt = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long row = gt / TPR;
  const int c8 = (int)(gt - row * TPR) * 8;
  const long bh = row / Tpad;
  const int t = (int)(row - bh * Tpad);
  float s = 0.f, g2 = 0.f, v2 = 0.f;
  const bool kv_row = bh < (rows_pad / Tpad) / H * Hkv;  // a row of the [B*Hkv][T] view
  if (row < rows_pad && t < T) {
    const long r = bh * T + t;
    float a[8], g[8];
    load8_bf16(o + r * D + c8, a);
    load8_bf16(dO + r * D + c8, g);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      s = fmaf(a[e], g[e], s);
      g2 = fmaf(g[e], g[e], g2);
    }
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    if (dq_acc) {
      reinterpret_cast<float4*>(dq_acc + r * D + c8)[0] = z;
      reinterpret_cast<float4*>(dq_acc + r * D + c8)[1] = z;
    }
    if (hstat && kv_row) {
      float x[8];
      load8_bf16(v + r * D + c8, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) v2 = fmaf(x[e], x[e], v2);
    }
    if (dk_acc && kv_row) {
      reinterpret_cast<float4*>(dk_acc + r * D + c8)[0] = z;
      reinterpret_cast<float4*>(dk_acc + r * D + c8)[1] = z;
      reinterpret_cast<float4*>(dv_acc + r * D + c8)[0] = z;
      reinterpret_cast<float4*>(dv_acc + r * D + c8)[1] = z;
    }
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, off);
    g2 += __shfl_xor_sync(0xffffffffu, g2, off);
    v2 += __shfl_xor_sync(0xffffffffu, v2, off);
  }
  if (c8 == 0 && row < rows_pad) {
    delta_pad[row] = -s;
    lse2_pad[row] = t < T ? -lse[bh * T + t] * 1.4426950408889634f : 0.f;
  }
  if (hstat) {
    // The block's rows share one head (a block covers 256 * 8 / D rows and
    // Tpad is a multiple of 128); padding rows contribute zeros. One atomic
    // maximum per block and quantity: many same-address atomics from every
    // warp would serialise in L2.
    __shared__ float red[3][8];
    const float dn = warp_max(sqrtf(g2)), dl = warp_max(fabsf(s)), vn = warp_max(sqrtf(v2));
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
      red[0][w] = dn;
      red[1][w] = dl;
      red[2][w] = vn;
    }
    __syncthreads();
    if (threadIdx.x < 3) {
      float m = red[threadIdx.x][0];
#pragma unroll
      for (int i = 1; i < 8; ++i) m = fmaxf(m, red[threadIdx.x][i]);
      const long row_b = (long)blockIdx.x * (256 / TPR);  // the block's first row
      const long bh_b = row_b / Tpad;
      const bool kv_b = bh_b < (rows_pad / Tpad) / H * Hkv;
      if (row_b < rows_pad && (threadIdx.x < 2 || kv_b))
        atomicMax(reinterpret_cast<int*>(hstat) + 4 * bh_b + threadIdx.x, __float_as_int(m));
    }
  }
}

// dq = R(pos)^T (scale * dq_acc), stored as bf16; one thread per two groups
// of 8 values, half the array apart (both loads in flight at once; the grid
// covers ceil(n8 / 2) threads).
// With fp16 operands (qinv non-null) the accumulator holds Cg qinv_i dS K for
// query tile i (Cg per key/value head, in the fourth statistics slot of its
// index), which is divided out here. The same pass finishes split dk, dv
// accumulators (H the key/value heads, qinv null).
template <int D>
__global__ void __launch_bounds__(256) dq_finalize_kernel(
    const float* __restrict__ dq_acc, const float* __restrict__ rc, const float* __restrict__ rs,
    const int32_t* __restrict__ doc_start, __nv_bfloat16* __restrict__ dq, int H, int T,
    float scale, long n8, const float* __restrict__ qinv, const float* __restrict__ hstat,
    int Hkv, int ntiles) {
  pdl_wait_and_trigger();
  const long half = (n8 + 1) >> 1;
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= half) return;
  const bool two = idx + half < n8;
  float v[2][8];
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    if (g == 1 && !two) break;
    const long e0 = (idx + g * half) * 8;
    load_vec<4>(dq_acc + e0, v[g]);
    load_vec<4>(dq_acc + e0 + 4, v[g] + 4);
  }
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    if (g == 1 && !two) break;
    const long e0 = (idx + g * half) * 8;
    const long row = e0 / D;  // bh*T + t
    const int d0 = (int)(e0 - row * D);
    const int t = (int)(row % T);
    const int bh = (int)(row / T);
    const int b = bh / H;
    float f = scale;
    if (qinv) {
      const int bhk = b * Hkv + (bh - b * H) / (H / Hkv);
      f /= hstat[4 * bhk + 3] * qinv[((size_t)bh * ntiles + (t >> 7)) * 4];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) v[g][e] *= f;
    if (rc) {
      // clamped into the row (the ranges may come from the caller's saved buffer)
      const int pos = t - (doc_start ? min(max(doc_start[b * T + t] - b * T, 0), t) : 0);
      rope_pairs<8, D>(v[g], rc, rs, pos, d0, true);
    }
    store_vec<4>(dq + e0, v[g]);
    store_vec<4>(dq + e0 + 4, v[g] + 4);
  }
}
