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
#include "sm100.cuh"

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
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
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
// Transpose of an 8x8 b16 matrix held as one register per thread in the
// accumulator layout (row lane/4, columns 2 (lane%4), +1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void consumer_sync() {  // the eight consumer warps
  asm volatile("bar.sync 1, 256;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Streaming tensor-core variant (bf16 cache, G <= 8 NH query heads per cached
// head, NH = 1 or 2), for up to one cached head per SM. The cached tokens of
// all (b, cached head) pairs, laid end to end, are cut into gridDim.x equal
// spans, one per CTA (at most one CTA per SM), so every SM reads the same
// number of bytes whatever the length mix. A CTA's span covers pieces of one
// or more heads. One TMA warp streams the pieces in stages of 64 keys (K and
// V tiles, 128-byte swizzled boxes of 64 keys x 64 features) through a
// kDecStages-deep ring; eight consumer warps take the stages in turn, two
// groups of four (even and odd stages), each warp 16 keys of a stage with its
// own running max, sum and output for the G query heads, in transposed
// products (keys as the 16 rows of a tile, the heads as NH columns of 8):
//   S^T = K (Q_hi + Q_lo)^T    (the scaled, rotated fp32 query split into
//                               two bf16 parts, which keeps ~16 more bits
//                               of the scores than one bf16 query would)
//   O^T = O^T * 2^(m_old - m_new) + V^T P^T   (P^T from the score registers,
//                               moved to the operand layout by movmatrix)
// At the end of a piece the eight warps' states merge through shared memory.
// A head held whole by one CTA is written out at once; otherwise each CTA
// stores its partial (o unnormalised, max, sum) in slot (CTA + head), and
// the CTA that completes a head's count merges its partials into o and lse.
// Tile rows at or past the cache length are loaded with the tile but never
// contribute: their scores are masked and their V rows zeroed before P V.
// ---------------------------------------------------------------------------
constexpr int kDecKeys = 64;          // keys per stage
constexpr int kDecThreads = 288;      // 8 consumer warps + 1 TMA warp
constexpr int kDecConsumerWarps = 8;

template <int D>
struct DecStreamLayout {
  static constexpr int kTile = kDecKeys * D * 2;           // K or V tile of a stage
  static constexpr int kStageBytes = 2 * kTile;
  static constexpr int kStages = 196608 / kStageBytes;     // 6 (D = 128) or 12 (D = 64)
  static constexpr int kRing = 0;                          // 1024-aligned tiles
  static constexpr int kQRow = D * 2 + 16;                 // padded bf16 query rows
  static constexpr int kQhi = kStages * kStageBytes;
  static constexpr int kQlo = kQhi + 16 * kQRow;
  static constexpr int kOacc = kQlo + 16 * kQRow;          // f32 [16][D] merged output
  static constexpr int kLacc = kOacc + 16 * D * 4;         // f32 [16] merged sum
  static constexpr int kMw = kLacc + 16 * 4;               // f32 [8 warps][16] maxima
  static constexpr int kBars = kMw + kDecConsumerWarps * 16 * 4;  // full[S], empty[S]
  static constexpr int kMisc = kBars + 2 * kStages * 8;    // span, flags
  static constexpr int kBytes = kMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;             // slack to align the ring
};
static_assert(DecStreamLayout<128>::kAlloc <= 227 * 1024 && DecStreamLayout<64>::kAlloc <= 227 * 1024,
              "decode ring fits in shared memory");
static_assert(DecStreamLayout<128>::kQhi % 16 == 0 && DecStreamLayout<64>::kBars % 8 == 0,
              "aligned regions");

// Partial slots: o_part f32 [slots][16][D], ml_part f32 [slots][16][2]
// (max in log2 units, sum of exponentials); slots = gridDim.x + B * Hkv.
// cnt int32 [B * Hkv] is zero on entry (the caller clears it).
template <int D, int NH>
__global__ void __launch_bounds__(kDecThreads, 1) decode_stream_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ cache_lens,
    const float* __restrict__ rc, const float* __restrict__ rs, __nv_bfloat16* __restrict__ o,
    float* __restrict__ lse, float* __restrict__ o_part, float* __restrict__ ml_part,
    int* __restrict__ cnt, int B, int H, int Hkv, int T_max, float scale_log2) {
  using namespace sm100;
  if (threadIdx.x == kDecConsumerWarps * 32) {  // the TMA thread: descriptors are parameters
    prefetch_tensor_map(&tmK);
    prefetch_tensor_map(&tmV);
  }
  pdl_wait_and_trigger();
  using L = DecStreamLayout<D>;
  constexpr int NS = L::kStages;
  constexpr int KS = D / 16;  // k-steps of the scores, and 16-feature tiles of the output
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* sm = dsm_raw + ((1024 - (smem_u32(dsm_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = H / Hkv;
  auto bar_full = [&](int s) { return sb + L::kBars + 8u * s; };
  auto bar_empty = [&](int s) { return sb + L::kBars + 8u * (NS + s); };
  int* misc = reinterpret_cast<int*>(sm + L::kMisc);  // [0] start head, [1] start key, [2] last flag
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMisc + 16);
  auto clen = [&](int b) {
    const int v = cache_lens[b];
    return v < 1 ? 1 : (v > T_max ? T_max : v);
  };

  // ---- the span: tokens [x0, x1) of the concatenation; its first head and key ----
  long long total = 0;
  for (int b = lane; b < B; b += 32) total += (long long)clen(b) * Hkv;
#pragma unroll
  for (int o2 = 16; o2 >= 1; o2 >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o2);
  const long long W = (total + gridDim.x - 1) / gridDim.x;
  const long long x0 = (long long)blockIdx.x * W, x1 = min(x0 + W, total);
  if (warp == 0) {
    if (blockIdx.x == 0)  // out-of-range lengths are reported once
      for (int b = lane; b < B; b += 32) {
        const int v = cache_lens[b];
        if (v < 1 || v > T_max) report_status(ATTN_EDEVICE_INPUT);
      }
    if (x0 < x1) {
      // the row b whose tokens hold x0: a prefix sum over 32 rows at a time
      long long cum = 0;
      for (int base = 0; base < B; base += 32) {
        const int bb = base + lane;
        const long long seg = bb < B ? (long long)clen(bb) * Hkv : 0;
        long long inc = seg;
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) {
          const long long t = __shfl_up_sync(0xffffffffu, inc, o2);
          if (lane >= o2) inc += t;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, bb < B && x0 < cum + inc);
        if (hit) {
          if (lane == __ffs(hit) - 1) {
            const int len = clen(bb);
            const long long off = x0 - (cum + inc - seg);
            misc[0] = bb * Hkv + (int)(off / len);
            misc[1] = (int)(off % len);
          }
          break;
        }
        cum += __shfl_sync(0xffffffffu, inc, 31);
      }
    }
  }
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 4);  // the four warps of the group that takes the stage
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int i = tid; i < 16 * D + 16; i += kDecThreads)  // merged output and sums
    reinterpret_cast<float*>(sm + L::kOacc)[i] = 0.f;
  __syncthreads();
  if (x0 >= x1) return;  // uniform: an empty span (fewer tokens than CTAs)
  const int bhk_first = misc[0], j_first = misc[1];

  if (warp == kDecConsumerWarps) {
    // ---------------- TMA warp ----------------
    if (lane == 0) {
      int it = 0;
      long long x = x0;
      int bhk = bhk_first, j = j_first;
      while (x < x1) {
        const int len = clen(bhk / Hkv);
        const int n = (int)min((long long)(len - j), x1 - x);
        for (int k0 = 0; k0 < n; k0 += kDecKeys, ++it) {
          const int s = it % NS;
          if (it >= NS && !mbar_wait(bar_empty(s), ((it / NS) - 1) & 1, abort_flag)) return;
          mbar_arrive_expect_tx(bar_full(s), L::kStageBytes);
          const uint32_t kt = sb + L::kRing + s * L::kStageBytes, vt = kt + L::kTile;
#pragma unroll
          for (int fb = 0; fb < D / 64; ++fb) {
            tma_load_3d(kt + fb * 8192, &tmK, bar_full(s), 64 * fb, j + k0, bhk);
            tma_load_3d(vt + fb * 8192, &tmV, bar_full(s), 64 * fb, j + k0, bhk);
          }
        }
        x += n;
        ++bhk;
        j = 0;
      }
    }
    return;
  }

  // ---------------- consumer warps ----------------
  // Transposed products, keys as the rows of the tiles and the query heads
  // (NH tiles of 8) as the columns, so that no row of a tile is wasted:
  //   S^T[16 keys][8 heads] = K Q^T,   O^T[16 features][8 heads] += V^T P^T
  // (P^T moves from the accumulator layout into the operand layout with an
  // 8x8 transpose in registers).
  const int grp = warp >> 2, w4 = warp & 3;
  const int gq = lane >> 2, qd = lane & 3;  // fragment row, column pair
  float* oacc = reinterpret_cast<float*>(sm + L::kOacc);
  float* lacc = reinterpret_cast<float*>(sm + L::kLacc);
  float* mw = reinterpret_cast<float*>(sm + L::kMw);
  int it = 0;
  long long x = x0;
  int bhk = bhk_first, j = j_first;
  while (x < x1) {
    const int b = bhk / Hkv, hk = bhk - b * Hkv;
    const int len = clen(b);
    const int n = (int)min((long long)(len - j), x1 - x);
    const long long head_start = x - j;  // offset of this head's first key
    // the queries of this head: rotated to position len-1, scaled, split
    for (int i = tid; i < 8 * NH * (D / 2); i += 256) {
      const int g = i / (D / 2), pi = i - g * (D / 2);
      float xv[2] = {0.f, 0.f};
      if (g < G) {
        load_vec<2>(q + ((size_t)b * H + hk * G + g) * D + 2 * pi, xv);
        if (rc) rope_pairs<2, D>(xv, rc, rs, len - 1, 2 * pi, false);
        xv[0] *= scale_log2;
        xv[1] *= scale_log2;
      }
      const __nv_bfloat162 hi = __floats2bfloat162_rn(xv[0], xv[1]);
      const __nv_bfloat162 lo =
          __floats2bfloat162_rn(xv[0] - __low2float(hi), xv[1] - __high2float(hi));
      *reinterpret_cast<__nv_bfloat162*>(sm + L::kQhi + g * L::kQRow + pi * 4) = hi;
      *reinterpret_cast<__nv_bfloat162*>(sm + L::kQlo + g * L::kQRow + pi * 4) = lo;
    }
    consumer_sync();
    // Q^T operand fragments of k-steps 2 kp and 2 kp + 1, per head tile
    uint32_t qh[NH][KS][2], ql[NH][KS][2];
    {
      const int mi = lane >> 3, hrow = lane & 7;
#pragma unroll
      for (int nh = 0; nh < NH; ++nh)
#pragma unroll
        for (int kp = 0; kp < KS / 2; ++kp) {
          const int col = (4 * kp + mi) * 8;  // features of matrix mi
          const uint32_t ro = (nh * 8 + hrow) * L::kQRow + col * 2;
          ldsm_x4(sb + L::kQhi + ro, qh[nh][2 * kp][0], qh[nh][2 * kp][1], qh[nh][2 * kp + 1][0],
                  qh[nh][2 * kp + 1][1]);
          ldsm_x4(sb + L::kQlo + ro, ql[nh][2 * kp][0], ql[nh][2 * kp][1], ql[nh][2 * kp + 1][0],
                  ql[nh][2 * kp + 1][1]);
        }
    }
    float m[NH][2], l[NH][2], oc[KS][NH][4];
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) {
      m[nh][0] = m[nh][1] = -INFINITY;
      l[nh][0] = l[nh][1] = 0.f;
    }
#pragma unroll
    for (int t = 0; t < KS; ++t)
#pragma unroll
      for (int nh = 0; nh < NH; ++nh) oc[t][nh][0] = oc[t][nh][1] = oc[t][nh][2] = oc[t][nh][3] = 0.f;

    for (int k0 = 0; k0 < n; k0 += kDecKeys, ++it) {
      if ((it & 1) != grp) continue;
      const int s = it % NS;
      const uint32_t kt = sb + L::kRing + s * L::kStageBytes, vt = kt + L::kTile;
      // valid keys of this warp's 16; a wait that ran out (the status word
      // says so) skips the stage, so that all warps still meet at every
      // consumer barrier
      int nk = min(kDecKeys, n - k0) - 16 * w4;
      if (!mbar_wait(bar_full(s), (it / NS) & 1, abort_flag)) nk = 0;
      if (nk > 0) {
        const int mi = lane >> 3, rr = lane & 7;
        // S^T for keys 16 w4 .. +15: the K rows are the A operand
        float sh[NH][4], sl[NH][4];
#pragma unroll
        for (int nh = 0; nh < NH; ++nh)
#pragma unroll
          for (int e = 0; e < 4; ++e) sh[nh][e] = sl[nh][e] = 0.f;
        {
          const int key = 16 * w4 + (mi & 1) * 8 + rr;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const int c16 = 2 * ks + (mi >> 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(kt + (c16 >> 3) * 8192 + key * 128 + (((c16 & 7) ^ (key & 7)) << 4), a0, a1,
                    a2, a3);
#pragma unroll
            for (int nh = 0; nh < NH; ++nh) {
              mma_bf16_16816(sh[nh], a0, a1, a2, a3, qh[nh][ks][0], qh[nh][ks][1]);
              mma_bf16_16816(sl[nh], a0, a1, a2, a3, ql[nh][ks][0], ql[nh][ks][1]);
            }
          }
        }
        // rows gq, gq + 8 (keys), columns 2 qd, 2 qd + 1 (heads)
        const bool v0 = gq < nk, v1 = gq + 8 < nk;
        if (nk < 16) {
          // zero the V rows of keys past the piece (they may hold anything:
          // rows past the cache length, or another head's)
          for (int i = lane; i < 16 * (D / 8); i += 32) {
            const int rrow = i / (D / 8), ch = i - rrow * (D / 8);
            if (rrow >= nk) {
              const int key = 16 * w4 + rrow;
              *reinterpret_cast<uint4*>(sm + (vt - sb) + (ch >> 3) * 8192 + key * 128 +
                                        ((ch & 7) << 4)) = make_uint4(0, 0, 0, 0);
            }
          }
          __syncwarp();
        }
        uint32_t pb[NH][2];  // P^T operand fragments
#pragma unroll
        for (int nh = 0; nh < NH; ++nh) {
          float sc[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[e] = sh[nh][e] + sl[nh][e];
          if (!v0) sc[0] = sc[1] = -INFINITY;
          if (!v1) sc[2] = sc[3] = -INFINITY;
          float mx0 = fmaxf(sc[0], sc[2]), mx1 = fmaxf(sc[1], sc[3]);
#pragma unroll
          for (int o2 = 4; o2 <= 16; o2 <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
          }
          const float mn0 = fmaxf(m[nh][0], mx0), mn1 = fmaxf(m[nh][1], mx1);  // finite
          const float al0 = exp2f(m[nh][0] - mn0), al1 = exp2f(m[nh][1] - mn1);
          m[nh][0] = mn0;
          m[nh][1] = mn1;
          const float p0 = exp2f(sc[0] - mn0), p1 = exp2f(sc[1] - mn1);
          const float p2 = exp2f(sc[2] - mn0), p3 = exp2f(sc[3] - mn1);
          l[nh][0] = l[nh][0] * al0 + (p0 + p2);
          l[nh][1] = l[nh][1] * al1 + (p1 + p3);
#pragma unroll
          for (int t = 0; t < KS; ++t) {
            oc[t][nh][0] *= al0;
            oc[t][nh][1] *= al1;
            oc[t][nh][2] *= al0;
            oc[t][nh][3] *= al1;
          }
          pb[nh][0] = movmatrix_trans(pack_bf16(p0, p1));
          pb[nh][1] = movmatrix_trans(pack_bf16(p2, p3));
        }
        // O^T += V^T P^T, feature tiles of 16: V rows through a transposing load
        {
          const int key = 16 * w4 + (mi >> 1) * 8 + rr;
#pragma unroll
          for (int t = 0; t < KS; ++t) {
            const int c16 = 2 * t + (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_trans(vt + (c16 >> 3) * 8192 + key * 128 + (((c16 & 7) ^ (key & 7)) << 4),
                          a0, a1, a2, a3);
#pragma unroll
            for (int nh = 0; nh < NH; ++nh)
              mma_bf16_16816(oc[t][nh], a0, a1, a2, a3, pb[nh][0], pb[nh][1]);
          }
        }
        if (nk < 16) fence_proxy_async_smem();  // zeroed rows before the next TMA write
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(s));
    }

    // ---- merge the eight warps' states of this piece ----
#pragma unroll
    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
      for (int o2 = 4; o2 <= 16; o2 <<= 1) {
        l[nh][0] += __shfl_xor_sync(0xffffffffu, l[nh][0], o2);
        l[nh][1] += __shfl_xor_sync(0xffffffffu, l[nh][1], o2);
      }
    if (gq == 0)
#pragma unroll
      for (int nh = 0; nh < NH; ++nh) {
        mw[warp * 16 + nh * 8 + 2 * qd] = m[nh][0];
        mw[warp * 16 + nh * 8 + 2 * qd + 1] = m[nh][1];
      }
    consumer_sync();
#pragma unroll
    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = nh * 8 + 2 * qd + e;  // this thread's head
        if (h >= G || m[nh][e] == -INFINITY) continue;  // a warp without keys adds nothing
        float M = mw[h];
#pragma unroll
        for (int w = 1; w < kDecConsumerWarps; ++w) M = fmaxf(M, mw[w * 16 + h]);
        const float f = exp2f(m[nh][e] - M);
#pragma unroll
        for (int t = 0; t < KS; ++t) {
          atomicAdd(oacc + h * D + 16 * t + gq, oc[t][nh][e] * f);
          atomicAdd(oacc + h * D + 16 * t + gq + 8, oc[t][nh][2 + e] * f);
        }
        if (gq == 0) atomicAdd(lacc + h, l[nh][e] * f);
      }
    consumer_sync();
    // a head held whole by this CTA is finished here; otherwise store the partial
    const long long W_ = W;
    const int c_first = (int)(head_start / W_), c_last = (int)((head_start + len - 1) / W_);
    const bool whole = c_first == c_last;
    const size_t slot = (size_t)blockIdx.x + bhk;
    for (int i = tid; i < G * D; i += 256) {
      const int g = i / D, d = i - g * D;
      const float v = oacc[i];
      if (whole) {
        o[((size_t)b * H + hk * G + g) * D + d] = __float2bfloat16_rn(v / lacc[g]);
      } else {
        o_part[(slot * 16 + g) * D + d] = v;
      }
    }
    if (tid < G) {
      float Mg = mw[tid];
#pragma unroll
      for (int w = 1; w < kDecConsumerWarps; ++w) Mg = fmaxf(Mg, mw[w * 16 + tid]);
      if (whole) {
        lse[(size_t)b * H + hk * G + tid] = (Mg + log2f(lacc[tid])) * 0.69314718055994531f;
      } else {
        ml_part[(slot * 16 + tid) * 2] = Mg;
        ml_part[(slot * 16 + tid) * 2 + 1] = lacc[tid];
      }
    }
    consumer_sync();  // every read of oacc, lacc and mw is done
    for (int i = tid; i < 16 * D + 16; i += 256) oacc[i] = 0.f;  // lacc follows oacc
    if (!whole) {
      __threadfence();
      consumer_sync();
      if (tid == 0) misc[2] = atomicAdd(cnt + bhk, 1) == c_last - c_first;
      consumer_sync();
      if (misc[2]) {
        // the last of the head's CTAs: merge its partials (slots c + bhk)
        __threadfence();
        const int np = c_last - c_first + 1;
        const size_t s0 = (size_t)c_first + bhk;
        for (int i = tid; i < G * D; i += 256) {
          const int g = i / D, d = i - g * D;
          // one pass with a running maximum: every partial's loads are
          // independent of the others
          float Mg = -INFINITY, lg = 0.f, og = 0.f;
          for (int pi = 0; pi < np; ++pi) {
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(ml_part) + (s0 + pi) * 16 + g);
            const float op = __ldcg(o_part + ((s0 + pi) * 16 + g) * D + d);
            const float mn = fmaxf(Mg, ml.x);
            const float a = exp2f(Mg - mn), w = exp2f(ml.x - mn);  // Mg = -inf first: a = 0
            lg = lg * a + ml.y * w;
            og = og * a + op * w;
            Mg = mn;
          }
          o[((size_t)b * H + hk * G + g) * D + d] = __float2bfloat16_rn(og / lg);
          if (d == 0) lse[(size_t)b * H + hk * G + g] = (Mg + log2f(lg)) * 0.69314718055994531f;
        }
      }
    }
    x += n;
    ++bhk;
    j = 0;
  }
}

constexpr int kDecodeMmaThreads = 128;

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

// ---------------------------------------------------------------------------
// Split tensor-core variant (bf16 cache, G <= 16), for many short heads
// (more cached heads than SMs, where the persistent kernel's spans would
// each hold several heads and pay a query setup and merge per piece): the G
// query heads are the rows of a 16-row tile (zero rows past G), and the
// hardware schedules many short CTAs. One CTA walks a range
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
