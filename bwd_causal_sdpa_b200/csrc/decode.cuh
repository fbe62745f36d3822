// decode.cuh -- decode attention: one new token per sequence against a
// key/value cache (split over key chunks, then combined).
//
// Sources (page, section): Forge README, "Roadmap" (a KV cache for
// generation on the training attention module, "Architecture": attention
// with GQA + RoPE) and ARK README, "Inference architecture (EKO)" (RoPE from
// precomputed tables). The cache holds cache_lens[b] tokens at positions
// 0 .. cache_lens[b]-1 with keys already rotated; the new query sits at
// position cache_lens[b]-1 and sees every cached token.
//
// The work is a read of the cache: per cached token 2*D values and ~4*G*D
// flops for the G query heads sharing it, so the CUDA cores keep up with HBM
// for the group sizes in use and no tensor-core tile would be full (M = G).
// One CTA takes one chunk of kDecodeChunk cached tokens of one key/value
// head: it copies the chunk's K and V rows into shared memory (cp.async,
// rows padded by 16 bytes so that one row per lane is conflict-free), scores
// them against the G queries (rotated and scaled once), takes the chunk's
// max and exponentials (base 2) and its partial weighted sum, and stores
// (m, l, sum) per query head; decode_combine_kernel merges the chunks.
#pragma once

#include "common.cuh"

constexpr int kDecodeChunk = 128;   // cached tokens per CTA
constexpr int kDecodeThreads = 256;
constexpr int kDecodeMaxGroup = 64;  // query heads per key/value head

template <typename TIO, int D>
struct DecodeLayout {
  static constexpr int kRowBytes = D * (int)sizeof(TIO) + 16;  // padded cache row
  static constexpr int kK = 0;
  static constexpr int kV = kK + kDecodeChunk * kRowBytes;
  static constexpr int kQ = kV + kDecodeChunk * kRowBytes;       // [G][D] f32
  __host__ __device__ static constexpr int s_off(int G) { return kQ + G * D * 4; }   // [G][C] f32
  __host__ __device__ static constexpr int red_off(int G) { return s_off(G) + G * kDecodeChunk * 4; }
  // [8 warps][D] f32 partial sums when a head is split over warps, then m, l
  __host__ __device__ static constexpr int ml_off(int G) { return red_off(G) + 8 * D * 4; }
  __host__ __device__ static constexpr int bytes(int G) { return ml_off(G) + 2 * G * 4; }
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Grid (chunks of the longest cache, B*Hkv). Partials for query head bh and
// chunk c: o_part[(bh * n_chunks + c) * D + d] (unnormalised), m_part and
// l_part[bh * n_chunks + c] (max in log2 units and the sum of exponentials).
template <typename TIO, int D>
__global__ void __launch_bounds__(kDecodeThreads) decode_chunk_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k_cache, const TIO* __restrict__ v_cache,
    const int32_t* __restrict__ cache_lens, const float* __restrict__ rc,
    const float* __restrict__ rs, float* __restrict__ o_part, float* __restrict__ m_part,
    float* __restrict__ l_part, int H, int Hkv, int T_max, int n_chunks, float scale_log2) {
  using L = DecodeLayout<TIO, D>;
  constexpr int C = kDecodeChunk;
  constexpr int VEC = 16 / (int)sizeof(TIO);  // elements per 16-byte piece
  extern __shared__ __align__(16) uint8_t sm[];
  const int G = H / Hkv;
  const int bhk = blockIdx.y, b = bhk / Hkv, hk = bhk - b * Hkv;
  const int c = blockIdx.x;
  int len = cache_lens[b];
  if (len < 1 || len > T_max) {
    if (threadIdx.x == 0 && c == 0 && hk == 0) report_status(ATTN_EDEVICE_INPUT);
    len = len < 1 ? 1 : T_max;
  }
  const int j0 = c * C;
  if (j0 >= len) return;  // uniform: this chunk is past the cache
  const int nk = min(C, len - j0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // 1. K and V rows of the chunk into shared memory (rows past the cache zero-filled)
  const TIO* kb = k_cache + ((size_t)bhk * T_max + j0) * D;
  const TIO* vb = v_cache + ((size_t)bhk * T_max + j0) * D;
  constexpr int PIECES = C * D / VEC;
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(sm);
  for (int i = tid; i < PIECES; i += kDecodeThreads) {
    const int r = i / (D / VEC), p = i - r * (D / VEC);
    const uint32_t nb = r < nk ? 16u : 0u;
    const int rr = r < nk ? r : 0;  // in-bounds source even when nothing is read
    cp_async16(sbase + L::kK + r * L::kRowBytes + p * 16, kb + (size_t)rr * D + p * VEC, nb);
    cp_async16(sbase + L::kV + r * L::kRowBytes + p * 16, vb + (size_t)rr * D + p * VEC, nb);
  }
  // 2. the G queries, rotated to position len-1 and scaled by scale*log2(e)
  float* qs = reinterpret_cast<float*>(sm + L::kQ);
  for (int i = tid; i < G * (D / 2); i += kDecodeThreads) {
    const int g = i / (D / 2), pi = i - g * (D / 2);
    float x[2];
    load_vec<2>(q + ((size_t)b * H + hk * G + g) * D + 2 * pi, x);
    if (rc) rope_pairs<2, D>(x, rc, rs, len - 1, 2 * pi, false);
    qs[g * D + 2 * pi] = x[0] * scale_log2;
    qs[g * D + 2 * pi + 1] = x[1] * scale_log2;
  }
  cp_async_wait_all();
  __syncthreads();

  // 3. scores: thread -> (key j, every second head); K row j read in 16-byte
  // pieces (the query values are the same across a warp: broadcast reads)
  float* ss = reinterpret_cast<float*>(sm + L::s_off(G));
  {
    const int j = tid % C, h0 = tid / C;  // h0 uniform per warp
    const uint8_t* krow = sm + L::kK + j * L::kRowBytes;
    for (int g = h0; g < G; g += kDecodeThreads / C) {
      const float* qg = qs + g * D;
      float acc = 0.f;
#pragma unroll 4
      for (int p = 0; p < D / VEC; ++p) {
        float kv[VEC];
        if constexpr (VEC == 8) {
          load_vec<4>(reinterpret_cast<const TIO*>(krow + p * 16), kv);
          load_vec<4>(reinterpret_cast<const TIO*>(krow + p * 16) + 4, kv + 4);
        } else {
          load_vec<4>(reinterpret_cast<const TIO*>(krow + p * 16), kv);
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc = fmaf(qg[p * VEC + e], kv[e], acc);
      }
      ss[g * C + j] = j < nk ? acc : -INFINITY;
    }
  }
  __syncthreads();

  // 4. per head: chunk max, exponentials (base 2) in place, their sum
  float* ml = reinterpret_cast<float*>(sm + L::ml_off(G));
  for (int g = warp; g < G; g += kDecodeThreads / 32) {
    float m = -INFINITY;
    for (int j = lane; j < C; j += 32) m = fmaxf(m, ss[g * C + j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j < C; j += 32) {
      const float p = exp2f(ss[g * C + j] - m);  // masked keys: exp2(-inf) = 0
      ss[g * C + j] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) {
      ml[g] = m;
      ml[G + g] = l;
    }
  }
  __syncthreads();

  // 5. partial sums o_g = sum_j p_gj v_j, lanes over D (D/32 values each)
  constexpr int NC = D / 32;
  constexpr int NW = kDecodeThreads / 32;
  auto store_part = [&](int g, const float* acc) {
    const size_t slot = ((size_t)b * H + hk * G + g) * n_chunks + c;
    store_vec<NC>(o_part + slot * D + lane * NC, acc);
    if (lane == 0) {
      m_part[slot] = ml[g];
      l_part[slot] = ml[G + g];
    }
  };
  if (G >= NW) {
    // every warp takes whole heads
    for (int g = warp; g < G; g += NW) {
      float acc[NC];
#pragma unroll
      for (int e = 0; e < NC; ++e) acc[e] = 0.f;
      for (int j = 0; j < nk; ++j) {
        const float p = ss[g * C + j];
        float vv[NC];
        load_vec<NC>(reinterpret_cast<const TIO*>(sm + L::kV + j * L::kRowBytes) + lane * NC, vv);
#pragma unroll
        for (int e = 0; e < NC; ++e) acc[e] = fmaf(p, vv[e], acc[e]);
      }
      store_part(g, acc);
    }
  } else {
    // fewer heads than warps: head g's keys are split over wph warps
    const int wph = NW / G;
    const int g = warp / wph, part = warp - g * wph;
    const bool active = g < G;
    float* red = reinterpret_cast<float*>(sm + L::red_off(G));
    float acc[NC];
#pragma unroll
    for (int e = 0; e < NC; ++e) acc[e] = 0.f;
    if (active) {
      for (int j = part; j < nk; j += wph) {
        const float p = ss[g * C + j];
        float vv[NC];
        load_vec<NC>(reinterpret_cast<const TIO*>(sm + L::kV + j * L::kRowBytes) + lane * NC, vv);
#pragma unroll
        for (int e = 0; e < NC; ++e) acc[e] = fmaf(p, vv[e], acc[e]);
      }
#pragma unroll
      for (int e = 0; e < NC; ++e) red[warp * D + lane * NC + e] = acc[e];
    }
    __syncthreads();
    if (active && part == 0) {
      for (int w = 1; w < wph; ++w)
#pragma unroll
        for (int e = 0; e < NC; ++e) acc[e] += red[(warp + w) * D + lane * NC + e];
      store_part(g, acc);
    }
  }
}

// Merge the chunk partials of one (b, h): M = max m_c, l = sum l_c 2^(m_c-M),
// o = sum o_c 2^(m_c-M) / l, lse = (M + log2 l) ln 2. One warp per query head.
template <typename TIO, int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(
    const float* __restrict__ o_part, const float* __restrict__ m_part,
    const float* __restrict__ l_part, const int32_t* __restrict__ cache_lens, TIO* __restrict__ o,
    float* __restrict__ lse, int H, int T_max, int n_chunks, int BH) {
  constexpr int NC = D / 32;
  const int bh = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (bh >= BH) return;
  int len = cache_lens[bh / H];
  len = len < 1 ? 1 : (len > T_max ? T_max : len);
  const int nch = (len + kDecodeChunk - 1) / kDecodeChunk;
  const size_t base = (size_t)bh * n_chunks;
  float M = -INFINITY;
  for (int c = 0; c < nch; ++c) M = fmaxf(M, m_part[base + c]);
  float l = 0.f, acc[NC];
#pragma unroll
  for (int e = 0; e < NC; ++e) acc[e] = 0.f;
  for (int c = 0; c < nch; ++c) {
    const float w = exp2f(m_part[base + c] - M);
    l = fmaf(l_part[base + c], w, l);
    float v[NC];
    load_vec<NC>(o_part + (base + c) * D + lane * NC, v);
#pragma unroll
    for (int e = 0; e < NC; ++e) acc[e] = fmaf(v[e], w, acc[e]);
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < NC; ++e) acc[e] *= inv;
  store_vec<NC>(o + (size_t)bh * D + lane * NC, acc);
  if (lane == 0) lse[bh] = (M + log2f(l)) * 0.69314718055994531f;
}
