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
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's copy groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_pending() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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
  pdl_wait_and_trigger();
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

// ---------------------------------------------------------------------------
// Warp-level tensor-core helpers (mma.sync m16n8k16, ldmatrix) for the
// streaming variant below.
// ---------------------------------------------------------------------------
constexpr int kDecodeMmaThreads = 128;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
// D[16x8] += A[16x16] B[16x8], bf16 inputs, fp32 accumulators
__device__ __forceinline__ void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Streaming tensor-core variant (bf16 cache, G <= 16): the G query heads
// are the rows of a 16-row tile (zero rows past G). One CTA walks a range
// of the cache (per_split tokens, a multiple of kDecodePipeKeys) in stages of
// kDecodePipeKeys tokens through a kDecodePipeStages-deep cp.async pipeline,
// so loads stay in flight while earlier stages are scored and summed. Per
// stage: S = (Q_hi + Q_lo) K^T with each warp taking 8 keys (the scaled,
// rotated fp32 query is split into bf16 hi = bf16(q) and lo = bf16(q - hi),
// so the scores keep ~16 more bits than one bf16 query would, which the lse
// bound needs; the query fragments stay in registers), the row max combined across the warps, the
// running max / sum updated and the output accumulators (registers, warp w
// owning D/4 columns) rescaled by exp2(m_old - m_new) before P V of the
// stage is added.
// ---------------------------------------------------------------------------
constexpr int kDecodePipeKeys = 32;
constexpr int kDecodePipeStages = 2;

template <int D>
struct DecodePipeLayout {
  static constexpr int kRowBytes = D * 2 + 16;                 // padded bf16 rows
  static constexpr int kStageBytes = 2 * kDecodePipeKeys * kRowBytes;  // K rows, V rows
  static constexpr int kQhi = kDecodePipeStages * kStageBytes;
  static constexpr int kQlo = kQhi + 16 * kRowBytes;
  static constexpr int kPRowBytes = kDecodePipeKeys * 2 + 16;  // [16][32] bf16
  static constexpr int kP = kQlo + 16 * kRowBytes;
  static constexpr int kRed = kP + 16 * kPRowBytes;             // f32 [2][4 warps][16]
  static constexpr int kStat = kRed + 2 * 4 * 16 * 4;           // f32 running max [16], sum [16]
  static constexpr int kBytes = kStat + 2 * 16 * 4;
};
static_assert(DecodePipeLayout<128>::kP % 16 == 0 && DecodePipeLayout<64>::kRed % 16 == 0,
              "ldmatrix rows need 16-byte alignment");

template <int D>
__global__ void __launch_bounds__(kDecodeMmaThreads) decode_pipe_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_cache,
    const __nv_bfloat16* __restrict__ v_cache, const int32_t* __restrict__ cache_lens,
    const float* __restrict__ rc, const float* __restrict__ rs, float* __restrict__ o_part,
    float* __restrict__ m_part, float* __restrict__ l_part, int H, int Hkv, int T_max,
    int n_split, int per_split, float scale_log2) {
  pdl_wait_and_trigger();
  using L = DecodePipeLayout<D>;
  constexpr int C = kDecodePipeKeys;
  constexpr int NS = kDecodePipeStages;
  constexpr int NT = D / 32;  // n8 tiles of the weighted sum per warp
  constexpr int KS = D / 16;  // k-steps of the scores
  extern __shared__ __align__(16) uint8_t sm[];
  const int G = H / Hkv;
  const int bhk = blockIdx.y, b = bhk / Hkv, hk = bhk - b * Hkv;
  const int split = blockIdx.x;
  int len = cache_lens[b];
  if (len < 1 || len > T_max) {
    if (threadIdx.x == 0 && split == 0 && hk == 0) report_status(ATTN_EDEVICE_INPUT);
    len = len < 1 ? 1 : T_max;
  }
  const int t_lo = split * per_split;
  if (t_lo >= len) return;  // uniform: this range is past the cache
  const int t_hi = min(t_lo + per_split, len);
  const int n_st = (t_hi - t_lo + C - 1) / C;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = (uint32_t)__cvta_generic_to_shared(sm);
  const __nv_bfloat16* kb = k_cache + (size_t)bhk * T_max * D;
  const __nv_bfloat16* vb = v_cache + (size_t)bhk * T_max * D;

  // stage si's K and V rows into buffer si % NS (rows past the range
  // zero-filled); one commit per call, so the group counts line up
  auto issue_stage = [&](int si) {
    if (si < n_st) {
      const int j0 = t_lo + si * C, nk = min(C, t_hi - j0);
      const uint32_t st = sb + (si % NS) * L::kStageBytes;
      for (int i = tid; i < C * D / 8; i += kDecodeMmaThreads) {
        const int r = i / (D / 8), p = i - r * (D / 8);
        const uint32_t nb = r < nk ? 16u : 0u;
        const size_t src = (size_t)(j0 + (r < nk ? r : 0)) * D + p * 8;  // in bounds
        cp_async16(st + r * L::kRowBytes + p * 16, kb + src, nb);
        cp_async16(st + (C + r) * L::kRowBytes + p * 16, vb + src, nb);
      }
    }
    cp_async_commit();
  };
  for (int si = 0; si < NS - 1; ++si) issue_stage(si);

  // the queries: rotated to position len-1, scaled by scale*log2(e), split
  // into bf16 hi + lo; rows G..15 zero
  for (int i = tid; i < 16 * (D / 2); i += kDecodeMmaThreads) {
    const int g = i / (D / 2), pi = i - g * (D / 2);
    float x[2] = {0.f, 0.f};
    if (g < G) {
      load_vec<2>(q + ((size_t)b * H + hk * G + g) * D + 2 * pi, x);
      if (rc) rope_pairs<2, D>(x, rc, rs, len - 1, 2 * pi, false);
      x[0] *= scale_log2;
      x[1] *= scale_log2;
    }
    const __nv_bfloat162 hi = __floats2bfloat162_rn(x[0], x[1]);
    const __nv_bfloat162 lo =
        __floats2bfloat162_rn(x[0] - __low2float(hi), x[1] - __high2float(hi));
    *reinterpret_cast<__nv_bfloat162*>(sm + L::kQhi + g * L::kRowBytes + pi * 4) = hi;
    *reinterpret_cast<__nv_bfloat162*>(sm + L::kQlo + g * L::kRowBytes + pi * 4) = lo;
  }
  float* red = reinterpret_cast<float*>(sm + L::kRed);    // [0..63] maxima, [64..127] sums
  float* stm = reinterpret_cast<float*>(sm + L::kStat);   // running max [16]
  float* stl = stm + 16;                                  // running sum [16]
  if (tid < 16) {
    stm[tid] = -INFINITY;
    stl[tid] = 0.f;
  }
  __syncthreads();
  // query fragments (hi, lo) for all k-steps, kept in registers
  uint32_t qh[KS][4], ql[KS][4];
  {
    const int arow = lane & 15, acol = (lane >> 4) * 8;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      ldsm_x4(sb + L::kQhi + arow * L::kRowBytes + (ks * 16 + acol) * 2, qh[ks][0], qh[ks][1],
              qh[ks][2], qh[ks][3]);
      ldsm_x4(sb + L::kQlo + arow * L::kRowBytes + (ks * 16 + acol) * 2, ql[ks][0], ql[ks][1],
              ql[ks][2], ql[ks][3]);
    }
  }
  const int r0 = lane >> 2, r1 = r0 + 8;
  float oc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) oc[t][0] = oc[t][1] = oc[t][2] = oc[t][3] = 0.f;

  for (int si = 0; si < n_st; ++si) {
    issue_stage(si + NS - 1);
    cp_async_wait_pending<NS - 1>();
    __syncthreads();
    const uint32_t kst = sb + (si % NS) * L::kStageBytes;
    const uint32_t vst = kst + C * L::kRowBytes;
    const int nk = min(C, t_hi - (t_lo + si * C));
    // scores of this warp's 8 keys
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int brow = lane & 7, bcol = ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t b0, b1;
        ldsm_x2(kst + (warp * 8 + brow) * L::kRowBytes + (ks * 16 + bcol) * 2, b0, b1);
        mma_bf16_16816(sc, qh[ks][0], qh[ks][1], qh[ks][2], qh[ks][3], b0, b1);
        mma_bf16_16816(sc, ql[ks][0], ql[ks][1], ql[ks][2], ql[ks][3], b0, b1);
      }
    }
    const int key = warp * 8 + 2 * (lane & 3);  // this thread's two keys: key, key + 1
    if (key >= nk) sc[0] = sc[2] = -INFINITY;
    if (key + 1 >= nk) sc[1] = sc[3] = -INFINITY;
    float mx0 = fmaxf(sc[0], sc[1]), mx1 = fmaxf(sc[2], sc[3]);
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if ((lane & 3) == 0) {
      red[warp * 16 + r0] = mx0;
      red[warp * 16 + r1] = mx1;
    }
    __syncthreads();
    // new running max, rescale factor, P of this stage
    const float mo0 = stm[r0], mo1 = stm[r1];
    const float mn0 = fmaxf(mo0, fmaxf(fmaxf(red[r0], red[16 + r0]), fmaxf(red[32 + r0], red[48 + r0])));
    const float mn1 = fmaxf(mo1, fmaxf(fmaxf(red[r1], red[16 + r1]), fmaxf(red[32 + r1], red[48 + r1])));
    const float al0 = exp2f(mo0 - mn0), al1 = exp2f(mo1 - mn1);  // 0 on the first stage
    const float p0 = exp2f(sc[0] - mn0), p1 = exp2f(sc[1] - mn0);  // masked: 0
    const float p2 = exp2f(sc[2] - mn1), p3 = exp2f(sc[3] - mn1);
    *reinterpret_cast<__nv_bfloat162*>(sm + L::kP + r0 * L::kPRowBytes + key * 2) =
        __floats2bfloat162_rn(p0, p1);
    *reinterpret_cast<__nv_bfloat162*>(sm + L::kP + r1 * L::kPRowBytes + key * 2) =
        __floats2bfloat162_rn(p2, p3);
    float ls0 = p0 + p1, ls1 = p2 + p3;
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      ls0 += __shfl_xor_sync(0xffffffffu, ls0, o);
      ls1 += __shfl_xor_sync(0xffffffffu, ls1, o);
    }
    if ((lane & 3) == 0) {
      red[64 + warp * 16 + r0] = ls0;
      red[64 + warp * 16 + r1] = ls1;
    }
    __syncthreads();
    if (tid < 16) {  // running statistics of row tid
      const float mo = stm[tid];
      const float mn = fmaxf(mo, fmaxf(fmaxf(red[tid], red[16 + tid]), fmaxf(red[32 + tid], red[48 + tid])));
      stl[tid] = stl[tid] * exp2f(mo - mn) + (red[64 + tid] + red[80 + tid]) +
                 (red[96 + tid] + red[112 + tid]);
      stm[tid] = mn;
    }
    // O = O * alpha + P V (this warp's D/4 columns)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      oc[t][0] *= al0;
      oc[t][1] *= al0;
      oc[t][2] *= al1;
      oc[t][3] *= al1;
    }
    {
      const int arow = lane & 15, acol = (lane >> 4) * 8, vrow = lane & 15;
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sb + L::kP + arow * L::kPRowBytes + (ks * 16 + acol) * 2, a0, a1, a2, a3);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          uint32_t b0, b1;
          ldsm_x2_trans(vst + (ks * 16 + vrow) * L::kRowBytes + (warp * (D / 4) + t * 8) * 2, b0,
                        b1);
          mma_bf16_16816(oc[t], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    __syncthreads();  // buffer si % NS, P and the partial maxima / sums are reused
  }

  // partials of this range, rows < G
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int col = warp * (D / 4) + t * 8 + 2 * (lane & 3);
    if (r0 < G) {
      const size_t slot = ((size_t)b * H + hk * G + r0) * n_split + split;
      *reinterpret_cast<float2*>(o_part + slot * D + col) = make_float2(oc[t][0], oc[t][1]);
    }
    if (r1 < G) {
      const size_t slot = ((size_t)b * H + hk * G + r1) * n_split + split;
      *reinterpret_cast<float2*>(o_part + slot * D + col) = make_float2(oc[t][2], oc[t][3]);
    }
  }
  if (tid < G) {
    const size_t slot = ((size_t)b * H + hk * G + tid) * n_split + split;
    m_part[slot] = stm[tid];
    l_part[slot] = stl[tid];
  }
}

// Merge the chunk partials of one (b, h): M = max m_s, l = sum l_s 2^(m_s-M),
// o = sum o_s 2^(m_s-M) / l, lse = (M + log2 l) ln 2. One block of
// kDecodeCombineThreads threads per query head: the chunks are spread over
// the threads (block reductions through shared memory), then each of the
// kDecodeCombineThreads / D thread groups sums a share of the chunks for
// every column. Dynamic shared memory: n_split weights.
constexpr int kDecodeCombineThreads = 256;

template <typename TIO, int D>
__global__ void __launch_bounds__(kDecodeCombineThreads) decode_combine_kernel(
    const float* __restrict__ o_part, const float* __restrict__ m_part,
    const float* __restrict__ l_part, const int32_t* __restrict__ cache_lens, TIO* __restrict__ o,
    float* __restrict__ lse, int H, int T_max, int n_split, int per_split) {
  pdl_wait_and_trigger();
  constexpr int NT = kDecodeCombineThreads, NG = NT / D;
  extern __shared__ float wsh[];  // [n_split]
  __shared__ float red[NT / 32];
  __shared__ float part[NG][D];
  const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int len = cache_lens[bh / H];
  len = len < 1 ? 1 : (len > T_max ? T_max : len);
  const int ns = (len + per_split - 1) / per_split;
  const size_t base = (size_t)bh * n_split;
  // M
  float M = -INFINITY;
  for (int s = tid; s < ns; s += NT) M = fmaxf(M, m_part[base + s]);
  M = warp_max(M);
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  // weights and l
  float l = 0.f;
  for (int s = tid; s < ns; s += NT) {
    const float w = exp2f(m_part[base + s] - M);
    wsh[s] = w;
    l = fmaf(l_part[base + s], w, l);
  }
  l = warp_sum(l);
  if (lane == 0) red[warp] = l;
  __syncthreads();
  l = 0.f;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) l += red[w];
  // o: group gi of the threads sums chunks gi, gi + NG, ... for column d
  const int d = tid % D, gi = tid / D;
  float acc = 0.f;
#pragma unroll 4
  for (int s = gi; s < ns; s += NG) acc = fmaf(o_part[(base + s) * D + d], wsh[s], acc);
  part[gi][d] = acc;
  __syncthreads();
  if (gi == 0) {
#pragma unroll
    for (int g = 1; g < NG; ++g) acc += part[g][d];
    o[(size_t)bh * D + d] = from_f32<TIO>(acc / l);
    if (d == 0) lse[bh] = (M + log2f(l)) * 0.69314718055994531f;
  }
}
