// decode.cuh -- decode attention: one new token per sequence against a
// key/value cache (split over key ranges, then combined).
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
// head (small CTAs, several resident per SM, so that some load while others
// compute): it copies the chunk's K and V rows into shared memory (cp.async,
// rows padded by 16 bytes against bank conflicts), scores them against the G
// queries (rotated and scaled once; four threads per key, each K row read
// once), takes the chunk's max and exponentials (base 2) and its partial
// weighted sum (each V row read once when G <= 8), and stores (m, l, sum)
// per query head; decode_combine_kernel merges the chunks.
#pragma once

#include "common.cuh"

constexpr int kDecodeChunk = 64;     // cached tokens per CTA
constexpr int kDecodeThreads = 256;
constexpr int kDecodeMaxGroup = 64;  // query heads per key/value head

template <typename TIO, int D>
struct DecodeLayout {
  // every region starts on a 16-byte boundary (vector accesses)
  __host__ __device__ static constexpr int a16(int x) { return (x + 15) & ~15; }
  static constexpr int kRowBytes = D * (int)sizeof(TIO) + 16;  // padded cache row
  static constexpr int kK = 0;
  static constexpr int kV = kDecodeChunk * kRowBytes;
  // queries f32 [G][4 quarters][D/4 + 4]: the four threads scoring one key
  // read different quarters, padded apart onto different banks
  static constexpr int kQuarter = D / 4 + 4;
  static constexpr int kQ = 2 * kDecodeChunk * kRowBytes;
  __host__ __device__ static constexpr int s_off(int G) { return a16(kQ + G * 4 * kQuarter * 4); }  // [G][C] f32
  __host__ __device__ static constexpr int ml_off(int G) { return a16(s_off(G) + G * kDecodeChunk * 4); }
  // [8 warps][G <= 8][D] f32 partial sums of the key slices
  __host__ __device__ static constexpr int red_off(int G) { return a16(ml_off(G) + 2 * G * 4); }
  __host__ __device__ static constexpr int bytes(int G) {
    return red_off(G) + (G <= 8 ? 8 * G * D * 4 : 0);
  }
};
static_assert(DecodeLayout<__nv_bfloat16, 128>::kRowBytes % 16 == 0, "padded rows stay 16-byte aligned");
static_assert(DecodeLayout<float, 64>::kQuarter * 4 % 16 == 0, "query quarters stay 16-byte aligned");
static_assert(DecodeLayout<__nv_bfloat16, 128>::red_off(1) % 16 == 0, "partial sums 16-byte aligned");

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Grid (n_split, B*Hkv): CTA s takes cache tokens [s*C, min((s+1)*C, len))
// of key/value head bhk. Partials for query head bh and chunk s:
// o_part[(bh * n_split + s) * D + d] (unnormalised), m_part and
// l_part[bh * n_split + s] (max in log2 units, sum of exponentials).
template <typename TIO, int D>
__global__ void __launch_bounds__(kDecodeThreads) decode_split_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k_cache, const TIO* __restrict__ v_cache,
    const int32_t* __restrict__ cache_lens, const float* __restrict__ rc,
    const float* __restrict__ rs, float* __restrict__ o_part, float* __restrict__ m_part,
    float* __restrict__ l_part, int H, int Hkv, int T_max, int n_split, int per_split,
    float scale_log2) {
  using L = DecodeLayout<TIO, D>;
  constexpr int C = kDecodeChunk;
  constexpr int VEC = 16 / (int)sizeof(TIO);  // elements per 16-byte piece
  constexpr int NC = D / 32;                  // values per lane in the weighted sum
  constexpr int NW = kDecodeThreads / 32;
  constexpr int QP = D / VEC / 4;             // 16-byte pieces per quarter row
  extern __shared__ __align__(16) uint8_t sm[];
  const int G = H / Hkv;
  const int bhk = blockIdx.y, b = bhk / Hkv, hk = bhk - b * Hkv;
  const int split = blockIdx.x;
  int len = cache_lens[b];
  if (len < 1 || len > T_max) {
    if (threadIdx.x == 0 && split == 0 && hk == 0) report_status(ATTN_EDEVICE_INPUT);
    len = len < 1 ? 1 : T_max;
  }
  const int j0 = split * C;
  if (j0 >= len) return;  // uniform: this chunk is past the cache
  const int nk = min(C, len - j0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // 1. K and V rows of the chunk into shared memory (rows past the cache zero-filled)
  {
    const TIO* kb = k_cache + ((size_t)bhk * T_max + j0) * D;
    const TIO* vb = v_cache + ((size_t)bhk * T_max + j0) * D;
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(sm);
    for (int i = tid; i < C * D / VEC; i += kDecodeThreads) {
      const int r = i / (D / VEC), p = i - r * (D / VEC);
      const uint32_t nb = r < nk ? 16u : 0u;
      const size_t src = (size_t)(r < nk ? r : 0) * D + p * VEC;  // in bounds
      cp_async16(sbase + L::kK + r * L::kRowBytes + p * 16, kb + src, nb);
      cp_async16(sbase + L::kV + r * L::kRowBytes + p * 16, vb + src, nb);
    }
  }
  // 2. the G queries, rotated to position len-1 and scaled by scale*log2(e)
  float* qs = reinterpret_cast<float*>(sm + L::kQ);
  for (int i = tid; i < G * (D / 2); i += kDecodeThreads) {
    const int g = i / (D / 2), pi = i - g * (D / 2);
    float x[2];
    load_vec<2>(q + ((size_t)b * H + hk * G + g) * D + 2 * pi, x);
    if (rc) rope_pairs<2, D>(x, rc, rs, len - 1, 2 * pi, false);
    const int d = 2 * pi, at = g * 4 * L::kQuarter + (d / (D / 4)) * L::kQuarter + d % (D / 4);
    qs[at] = x[0] * scale_log2;
    qs[at + 1] = x[1] * scale_log2;
  }
  cp_async_wait_all();
  __syncthreads();

  // 3. scores: four threads per key (adjacent lanes), each a quarter of D for
  // every head, summed by two shuffles; each K row is read once
  float* ss = reinterpret_cast<float*>(sm + L::s_off(G));
  {
    const int j = tid >> 2, qd = tid & 3;
    const uint8_t* krow = sm + L::kK + j * L::kRowBytes + qd * QP * 16;
    float kv[QP][VEC];
#pragma unroll
    for (int p = 0; p < QP; ++p) {
      if constexpr (VEC == 8) {
        load_vec<4>(reinterpret_cast<const TIO*>(krow + p * 16), kv[p]);
        load_vec<4>(reinterpret_cast<const TIO*>(krow + p * 16) + 4, kv[p] + 4);
      } else {
        load_vec<4>(reinterpret_cast<const TIO*>(krow + p * 16), kv[p]);
      }
    }
    for (int g = 0; g < G; ++g) {
      const float4* qg = reinterpret_cast<const float4*>(qs + (g * 4 + qd) * L::kQuarter);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int p = 0; p < QP; ++p)
#pragma unroll
        for (int e4 = 0; e4 < VEC / 4; ++e4) {
          const float4 qq = qg[p * (VEC / 4) + e4];
          a0 = fmaf(qq.x, kv[p][4 * e4], a0);
          a1 = fmaf(qq.y, kv[p][4 * e4 + 1], a1);
          a0 = fmaf(qq.z, kv[p][4 * e4 + 2], a0);
          a1 = fmaf(qq.w, kv[p][4 * e4 + 3], a1);
        }
      float a = a0 + a1;
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      if (qd == 0) ss[g * C + j] = j < nk ? a : -INFINITY;
    }
  }
  __syncthreads();

  // 4. per head: chunk max, exponentials (base 2) in place, their sum
  float* ml = reinterpret_cast<float*>(sm + L::ml_off(G));
  for (int g = warp; g < G; g += NW) {
    const float m = warp_max(fmaxf(ss[g * C + lane], ss[g * C + lane + 32]));
    const float p0 = exp2f(ss[g * C + lane] - m);  // masked keys: exp2(-inf) = 0
    const float p1 = exp2f(ss[g * C + lane + 32] - m);
    ss[g * C + lane] = p0;
    ss[g * C + lane + 32] = p1;
    const float l = warp_sum(p0 + p1);
    if (lane == 0) {
      ml[g] = m;
      ml[G + g] = l;
    }
  }
  __syncthreads();

  // 5. weighted sums o_g = sum_j p_gj v_j, lanes over D (D/32 values each)
  auto store_part = [&](int g, const float* a) {
    const size_t slot = ((size_t)b * H + hk * G + g) * n_split + split;
    store_vec<NC>(o_part + slot * D + lane * NC, a);
    if (lane == 0) {
      m_part[slot] = ml[g];
      l_part[slot] = ml[G + g];
    }
  };
  if (G <= 8) {
    // warp w takes keys w, w+8, ... for every head (each V row read once),
    // then the eight slices are added through shared memory
    float acc[8][NC];
#pragma unroll
    for (int t = 0; t < 8; ++t)
#pragma unroll
      for (int e = 0; e < NC; ++e) acc[t][e] = 0.f;
    for (int j = warp; j < nk; j += NW) {
      float vv[NC];
      load_vec<NC>(reinterpret_cast<const TIO*>(sm + L::kV + j * L::kRowBytes) + lane * NC, vv);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (t < G) {
          const float pj = ss[t * C + j];
#pragma unroll
          for (int e = 0; e < NC; ++e) acc[t][e] = fmaf(pj, vv[e], acc[t][e]);
        }
      }
    }
    float* red = reinterpret_cast<float*>(sm + L::red_off(G));
#pragma unroll
    for (int t = 0; t < 8; ++t)
      if (t < G) store_vec<NC>(red + (warp * G + t) * D + lane * NC, acc[t]);
    __syncthreads();
    for (int g = warp; g < G; g += NW) {
      float a[NC];
#pragma unroll
      for (int e = 0; e < NC; ++e) a[e] = 0.f;
      for (int w = 0; w < NW; ++w) {
        float r[NC];
        load_vec<NC>(red + (w * G + g) * D + lane * NC, r);
#pragma unroll
        for (int e = 0; e < NC; ++e) a[e] += r[e];
      }
      store_part(g, a);
    }
  } else {
    // warp w owns heads w, w+8, ...: every key of the chunk
    for (int g = warp; g < G; g += NW) {
      float acc[NC];
#pragma unroll
      for (int e = 0; e < NC; ++e) acc[e] = 0.f;
      for (int j = 0; j < nk; ++j) {
        const float pj = ss[g * C + j];
        float vv[NC];
        load_vec<NC>(reinterpret_cast<const TIO*>(sm + L::kV + j * L::kRowBytes) + lane * NC, vv);
#pragma unroll
        for (int e = 0; e < NC; ++e) acc[e] = fmaf(pj, vv[e], acc[e]);
      }
      store_part(g, acc);
    }
  }
}

// Merge the chunk partials of one (b, h): M = max m_s, l = sum l_s 2^(m_s-M),
// o = sum o_s 2^(m_s-M) / l, lse = (M + log2 l) ln 2. One block of D threads
// per query head.
template <typename TIO, int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(
    const float* __restrict__ o_part, const float* __restrict__ m_part,
    const float* __restrict__ l_part, const int32_t* __restrict__ cache_lens, TIO* __restrict__ o,
    float* __restrict__ lse, int H, int T_max, int n_split, int per_split) {
  const int bh = blockIdx.x, d = threadIdx.x;
  int len = cache_lens[bh / H];
  len = len < 1 ? 1 : (len > T_max ? T_max : len);
  const int ns = (len + per_split - 1) / per_split;
  const size_t base = (size_t)bh * n_split;
  // eight independent loads in flight per thread in both passes
  float M = -INFINITY;
#pragma unroll 8
  for (int s = 0; s < ns; ++s) M = fmaxf(M, m_part[base + s]);
  float l = 0.f, acc = 0.f;
#pragma unroll 8
  for (int s = 0; s < ns; ++s) {
    const float w = exp2f(m_part[base + s] - M);
    l = fmaf(l_part[base + s], w, l);
    acc = fmaf(o_part[(base + s) * D + d], w, acc);
  }
  o[(size_t)bh * D + d] = from_f32<TIO>(acc / l);
  if (d == 0) lse[bh] = (M + log2f(l)) * 0.69314718055994531f;
}
