// fwd_sm100.cuh -- tensor-core (tcgen05) attention forward for bf16 storage.
//
// One CTA computes two 128-row query tiles (A = rows [256t, 256t+128), B =
// the next 128) of one (b, h) slice; both share every K and V tile it loads.
//   warps 0-15 softmax: warpgroup g takes tile g & 1 and key columns
//              [64 (g >> 1), +64) of its S; thread t of a warpgroup owns query
//              row t (= TMEM lane t), so each row is shared by two threads,
//              which agree on the row's reference max through a small
//              shared-memory exchange (double-buffered by key-tile parity,
//              bounded mbarrier) and add their row sums at the end;
//   warp 16    TMA producer: both Q tiles once, then K and V tiles through a
//              ring of shared-memory stages;
//   warp 17    TMEM owner and MMA issuer (one thread).
// TMEM (512 columns): per tile an S column block (P, bf16, is written back
// over its first half) and an O accumulator. Per key tile j the MMA thread
// issues PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so the tensor pipe works on one
// tile while the other tile's softmax runs. S_t(j+1) is issued only after
// PV_t(j) completed (it overwrites the P that PV_t(j) reads); since a tcgen05
// commit covers every earlier MMA of the issuing thread, a softmax warp that
// has seen S_t(j) may rescale O_t without a further wait.
//
// Online softmax in log2 units with a lazy rescale: a row's reference max
// moves (and O, l are rescaled) only when the max grows by more than 8, so P
// stays <= 2^8 and O is rarely touched; the final O / l and lse = (m +
// log2 l) ln 2 use the same reference, so the result is exact up to rounding.
//
// Masking is per element only on tiles that cross the diagonal or the start
// of a row's document; key tiles wholly before the first row's document are
// never loaded (block skipping), nor are tiles past the diagonal.
//
// Sources (page, section): ARK README, "Accelerated forward pass (GPU)" (SDPA
// with the causal mask fused in) and aten.metal entry (scores, softmax,
// weighted sum, fused causal kernel); Forge README, "Acknowledgements"
// (FlashAttention-2-style tiling) and roadmap (attention tile sweep). The
// tiling, TMEM plan and warp roles are this library's own design.
#pragma once

#include "sm100.cuh"

namespace fwd100 {

using namespace sm100;

template <int D>
struct Layout {
  static constexpr int kTileBytes = 128 * D * 2;  // 128 rows x D 16-bit values
  static constexpr int kBlockBytes = 128 * 128;   // one 64-column block: 128 rows x 128 B
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kQ = 0;                    // Q_A, Q_B
  static constexpr int kK = kQ + 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBars = kV + kStages * kTileBytes;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bKFull = 1;
  static constexpr int bKEmpty = bKFull + kStages;
  static constexpr int bVFull = bKEmpty + kStages;
  static constexpr int bVEmpty = bVFull + kStages;
  static constexpr int bSFull = bVEmpty + kStages;  // [tile]
  static constexpr int bPFull = bSFull + 2;         // [tile], 128 arrivals
  static constexpr int bPVDone = bPFull + 2;        // [tile]
  static constexpr int bOFinal = bPVDone + 2;       // [tile]
  static constexpr int bXch = bOFinal + 2;          // [tile], 256 arrivals: row maxima exchanged
  static constexpr int kNumBars = bXch + 2;
  // row-max exchange between the two halves of a row: f32 [2 parities][2 tiles][2 halves][128]
  static constexpr int kXch = kBars + kNumBars * 8;
  static constexpr int kMisc = (kXch + 2 * 2 * 2 * 128 * 4 + 15) / 16 * 16;  // [0] TMEM base, [1] abort flag
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kSmemAlloc = kBytes;  // the window is 1024-byte aligned (checked)
  // TMEM columns: tile t uses [256t, 256t+128) for S/P and [256t+128, ...) for O
  static constexpr uint32_t kTmemCols = 512;
  // softmax warps 0-15 (warpgroup g: tile g & 1, key columns [64 (g >> 1), +64)),
  // then the TMA producer and the MMA issuer
  static constexpr int kSoftmaxThreads = 512;
  static constexpr int kThreads = kSoftmaxThreads + 64;
  static constexpr int kProducerWarp = 16, kMmaWarp = 17;
};

struct Params {
  int T, H, Hkv, BH, n_pairs, n_qtiles;  // H query heads read Hkv key/value heads
  float scale_log2;          // scale * log2(e)
  uint32_t idesc_s;          // instruction descriptor of S = Q K^T
  const float* q_fac;        // inverse power-of-two factor per (query head, tile) of the
                             // stored rotated q, one 16-byte record each (value first),
                             // or null (q as given)
  const float* k_fac;        // the same per (key/value head, tile) for k
  const int32_t* doc_start;  // flattened document starts, or null
  __nv_bfloat16* o;
  float* lse;
};

template <int D>
__global__ void __launch_bounds__(Layout<D>::kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const Params p) {
  pdl_wait_and_trigger();
  using L = Layout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sb0 = smem_u32(smem_raw);
  if (sb0 & 1023u) {  // uniform across the CTA: nothing has been issued yet
    if (threadIdx.x == 0) report_status(ATTN_ECUDA_LAYOUT);
    return;
  }
  uint8_t* sg = smem_raw;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sg + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + L::kMisc + 4);
  auto bar = [&](int i) -> uint32_t { return sb0 + L::kBars + 8u * i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  // Flattened grid, tile-major from the last tile pair: the longest rows (most
  // key tiles) are scheduled first.
  const int bh = (int)blockIdx.x % p.BH, b = bh / p.H;
  const int bhk = b * p.Hkv + (bh - b * p.H) / (p.H / p.Hkv);  // its key/value head
  const int pr = p.n_pairs - 1 - (int)blockIdx.x / p.BH;
  const int qtA = 2 * pr, qtB = 2 * pr + 1;
  const bool hasB = qtB * 128 < T;
  const int row0 = b * T;
  // Key tiles are numbered from kv_t0, the tile holding the start of tile A's
  // first row's document; tile A takes key tiles [0, nA) of that range, tile
  // B [jB0, n_kv): from the tile holding its own first row's document start
  // to its diagonal. Every key tile of a range holds a key some row of the
  // query tile may see (a query tile's allowed keys form one interval).
  const int ds0 = p.doc_start ? p.doc_start[row0 + qtA * 128] - row0 : 0;
  const int kv_t0 = ds0 >> 7;
  const int nA = qtA - kv_t0 + 1;           // key tiles tile A needs
  const int n_kv = hasB ? nA + 1 : nA;      // tile B needs one more (its diagonal)
  const int jB0 = (hasB && p.doc_start) ? ((p.doc_start[row0 + qtB * 128] - row0) >> 7) - kv_t0 : 0;
  auto t_lo = [&](int t) -> int { return t == 0 ? 0 : jB0; };
  auto t_hi = [&](int t) -> int { return t == 0 ? nA : (hasB ? n_kv : 0); };

  if (threadIdx.x == 0) {
    mbar_init(bar(L::bQFull), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::bKFull + s), 1);
      mbar_init(bar(L::bKEmpty + s), 1);
      mbar_init(bar(L::bVFull + s), 1);
      mbar_init(bar(L::bVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::bSFull + t), 1);
      mbar_init(bar(L::bPFull + t), 256);
      mbar_init(bar(L::bXch + t), 256);
      mbar_init(bar(L::bPVDone + t), 1);
      mbar_init(bar(L::bOFinal + t), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
    atomicAdd(&g_attn_tiles[0], (unsigned long long)(nA + (hasB ? n_kv - jB0 : 0)));
  }
  if (warp == L::kMmaWarp) {
    tmem_alloc(sb0 + L::kMisc, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == L::kProducerWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tensor_map(&tmQ);
      prefetch_tensor_map(&tmK);
      prefetch_tensor_map(&tmV);
      mbar_arrive_expect_tx(bar(L::bQFull), (hasB ? 2 : 1) * L::kTileBytes);
      for (int t = 0; t < (hasB ? 2 : 1); ++t)
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kQ + t * L::kTileBytes + cb * L::kBlockBytes, &tmQ,
                      bar(L::bQFull), cb * 64, (qtA + t) * 128, bh);
      for (int it = 0; it < n_kv; ++it) {
        const int st = it % L::kStages, round = it / L::kStages;
        const int kvrow = (kv_t0 + it) * 128;
        if (it >= L::kStages && !mbar_wait(bar(L::bKEmpty + st), (round - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::bKFull + st), L::kTileBytes);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kK + st * L::kTileBytes + cb * L::kBlockBytes, &tmK,
                      bar(L::bKFull + st), cb * 64, kvrow, bhk);
#ifdef ATTN_DEBUG_HOOKS
        if (it == 0 && g_attn_withhold == 1) continue;  // V(0) never arrives
#endif
        if (it >= L::kStages && !mbar_wait(bar(L::bVEmpty + st), (round - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::bVFull + st), L::kTileBytes);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kV + st * L::kTileBytes + cb * L::kBlockBytes, &tmV,
                      bar(L::bVFull + st), cb * 64, kvrow, bhk);
      }
    }
  } else if (warp == L::kMmaWarp) {
    // ---------------- MMA issuer ----------------
    // Issue order: S of each tile whose range starts at key tile 0, then per
    // key tile j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), each only where tile
    // t's range holds j (a tile whose range starts at j+1 gets its first S
    // there). Each tile's S(j+1) follows its own PV(j) (it overwrites the P
    // that PV(j) reads, so it waits for PV(j) to finish), and never waits for
    // the other tile's softmax: the two chains S -> softmax -> PV run
    // independently and fill each other's gaps. Barrier phases of tile t count
    // its own key tiles (j - t_lo(t)).
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_f16(128, D, true, true, false, true);
      const int t1 = hasB ? 2 : 1;
      auto active = [&](int t, int j) -> bool { return t < t1 && j >= t_lo(t) && j < t_hi(t); };
      auto issue_S = [&](int t, int j) {
        const uint32_t kbase = sb0 + L::kK + (j % L::kStages) * L::kTileBytes;
        const uint32_t qbase = sb0 + L::kQ + t * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBlockBytes + (kk & 3) * 32;
          mma_ss(tmem + 256 * t, smem_desc_sw128(qbase + off, 16, 1024),
                 smem_desc_sw128(kbase + off, 16, 1024), p.idesc_s, kk > 0);
        }
        mma_commit(bar(L::bSFull + t));
      };
      bool ok = mbar_wait(bar(L::bQFull), 0, abort_flag) && mbar_wait(bar(L::bKFull), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < t1; ++t)
          if (active(t, 0)) issue_S(t, 0);
        mma_commit(bar(L::bKEmpty));
      }
      for (int it = 0; ok && it < n_kv; ++it) {
        const int st = it % L::kStages, nst = (it + 1) % L::kStages;
        if (!mbar_wait(bar(L::bVFull + st), (it / L::kStages) & 1, abort_flag)) break;
        const uint32_t vbase = sb0 + L::kV + st * L::kTileBytes;
        bool issued_next = false;
        for (int t = 0; ok && t < t1; ++t) {
          if (!active(t, it)) {
            if (active(t, it + 1)) {  // tile t's range starts at it + 1
              if (!mbar_wait(bar(L::bKFull + nst), ((it + 1) / L::kStages) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              issue_S(t, it + 1);
              issued_next = true;
            }
            continue;
          }
          const int li = it - t_lo(t);  // this tile's own key-tile count
          if (!mbar_wait(bar(L::bPFull + t), li & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t aP = tmem + 256 * t;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + 256 * t + 128, aP + kk * 8,
                   smem_desc_sw128(vbase + kk * 2048, L::kBlockBytes, 1024), idesc_o,
                   (li > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::bPVDone + t));
          if (active(t, it + 1)) {
            if (!mbar_wait(bar(L::bKFull + nst), ((it + 1) / L::kStages) & 1, abort_flag) ||
                !mbar_wait(bar(L::bPVDone + t), li & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_S(t, it + 1);
            issued_next = true;
          }
        }
        if (!ok) break;
        mma_commit(bar(L::bVEmpty + st));
        if (issued_next) mma_commit(bar(L::bKEmpty + nst));
      }
      if (ok) {
        mma_commit(bar(L::bOFinal + 0));
        mma_commit(bar(L::bOFinal + 1));
      }
    }
  } else {
    // ---------------- softmax warpgroups ----------------
    const int t = (warp >> 2) & 1;   // tile
    const int hf = warp >> 3;        // key columns [64 hf, 64 hf + 64) of the tile's S
    const int r = (warp & 3) * 32 + lane;  // row within the tile = TMEM lane
    const int qt = qtA + t;
    const int i = qt * 128 + r;
    const bool active = (t == 0) || hasB;
    const int n_t = t_hi(t) - t_lo(t);  // key tiles this tile processes
    const int kt_first = kv_t0 + t_lo(t);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + 256 * t;
    const uint32_t tO = tS + 128;
    float* xch = reinterpret_cast<float*>(sg + L::kXch);  // [parity][tile][half][row]
    const int ds_i = p.doc_start ? p.doc_start[row0 + min(i, T - 1)] - row0 : 0;
    const float fq = p.q_fac ? p.q_fac[((size_t)bh * p.n_qtiles + min(qt, p.n_qtiles - 1)) * 4] : 1.f;
    float m = -INFINITY, l = 0.f;
    bool ok = active;
    for (int it = 0; ok && it < n_t; ++it) {
      const int kt = kt_first + it, j0 = kt * 128 + 64 * hf;  // first key of this half
      if (!mbar_wait(bar(L::bSFull + t), it & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      // scale of this key tile's scores (q, k tiles may carry power-of-two
      // factors). A zero scale (uniform attention) is evaluated with the
      // smallest normal scale instead: a score below 2^100 in magnitude then
      // scales to below 2^-26, so each kept probability rounds to exactly 1
      // as it should, while a masked score still becomes -inf rather than
      // inf * 0 = NaN.
      float sc = p.scale_log2 * fq * (p.k_fac ? p.k_fac[bhk * p.n_qtiles + kt] : 1.f);
      if (sc == 0.f) sc = 1.17549435e-38f;
      const bool pos_scale = sc > 0.f;
      uint32_t s[64];
      tmem_ld32(tS + 64 * hf, s);
      tmem_ld32(tS + 64 * hf + 32, s + 32);
      tmem_wait_ld();
      const bool need_mask = (j0 + 63 > i) || (j0 < ds_i);
      const float masked = pos_scale ? -INFINITY : INFINITY;
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (j0 + c > i || j0 + c < ds_i) s[c] = __float_as_uint(masked);
      }
      // extreme of this half's raw scores (max for a positive scale)
      float e4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) e4[q] = __uint_as_float(s[q]);
      float ext;
      if (pos_scale) {
#pragma unroll
        for (int c = 4; c < 64; c += 2)
          e4[(c >> 1) & 3] = max3f(e4[(c >> 1) & 3], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
        ext = max3f(fmaxf(e4[0], e4[1]), e4[2], e4[3]);
      } else {
#pragma unroll
        for (int c = 4; c < 64; c += 2)
          e4[(c >> 1) & 3] = min3f(e4[(c >> 1) & 3], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
        ext = min3f(fminf(e4[0], e4[1]), e4[2], e4[3]);
      }
      // the row max of the scaled scores: this half's and the other half's
      // (-inf for a half that is all masked, so both halves see the same value)
      float* xs = xch + ((it & 1) * 4 + t * 2) * 128;
      xs[hf * 128 + r] = ext * sc;
      mbar_arrive(bar(L::bXch + t));
      if (!mbar_wait(bar(L::bXch + t), it & 1, abort_flag)) { ok = false; break; }
      const float mx = fmaxf(xs[r], xs[128 + r]);
      // Move the reference max only when it grows by more than 8 (log2
      // units); the first key a row sees always moves it (m = -inf). Both
      // halves compute the same m from the same inputs.
      const bool move = mx > m + 8.f;
      const float alpha = move ? ex2(m - mx) : 1.f;
      // O needs rescaling only if it already holds a non-zero partial sum;
      // PV_t(it-1) is complete (it precedes S_t(it) in the commit order).
      const bool scale_o = move && m != -INFINITY && it > 0;
      if (move) {
        l *= alpha;
        m = mx;
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      // p = 2^(s * sc - m) two at a time; P (bf16) goes over the first half
      // of the S columns: this half's keys at columns [32 hf, 32 hf + 32),
      // which both halves have read by now (they passed the exchange)
      const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(-mref, -mref);
      float2 l2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 sv = make_float2(__uint_as_float(s[32 * c + 2 * e]),
                                        __uint_as_float(s[32 * c + 2 * e + 1]));
          const float2 x = __ffma2_rn(sv, sc2, nm2);
          const float2 pv = make_float2(ex2(x.x), ex2(x.y));
          l2[e & 3] = __fadd2_rn(l2[e & 3], pv);
          pk[e] = pack_bf16(pv.x, pv.y);
        }
        tmem_st16(tS + 32 * hf + 16 * c, pk);
      }
      const float2 la = __fadd2_rn(l2[0], l2[1]), lb = __fadd2_rn(l2[2], l2[3]);
      l += (la.x + la.y) + (lb.x + lb.y);
      // rescale this half's O columns (warp-collective: each lane by its own
      // factor, 1 for lanes that kept their max) before PV_t(it) runs
      if (__any_sync(0xffffffffu, scale_o)) {
        const float f = scale_o ? alpha : 1.f;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t ov[32];
          tmem_ld32(tO + (D / 2) * hf + 32 * c, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st32(tO + (D / 2) * hf + 32 * c, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::bPFull + t));
    }
    // row sum: this half's plus the other half's (through the exchange area,
    // parity n_t; both halves ran the same number of key tiles)
    float lt = l;
    if (ok) {
      float* xs = xch + ((n_t & 1) * 4 + t * 2) * 128;
      xs[hf * 128 + r] = l;
      mbar_arrive(bar(L::bXch + t));
      if (!mbar_wait(bar(L::bXch + t), n_t & 1, abort_flag)) ok = false;
      else lt = xs[r] + xs[128 + r];
    }
    if (ok && mbar_wait(bar(L::bOFinal + t), 0, abort_flag)) {
      tc_fence_after();
      const float inv = 1.f / lt;
      __nv_bfloat16* orow = p.o + ((size_t)bh * T + min(i, T - 1)) * D + (D / 2) * hf;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t ov[32];
        tmem_ld32(tO + (D / 2) * hf + 32 * c, ov);  // warp-collective
        tmem_wait_ld();
        if (i < T) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (i < T && hf == 0) p.lse[(size_t)bh * T + i] = (m + __log2f(lt)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fwd100
