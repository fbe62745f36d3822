// fwd_sm100.cuh -- tensor-core (tcgen05) attention forward for bf16 storage.
//
// One CTA computes two 128-row query tiles (A = rows [256t, 256t+128), B =
// the next 128) of one (b, h) slice; both share every K and V block it loads.
// Keys advance in blocks of 64, which keeps the scores of a block small
// enough (64 TMEM columns per tile) that S, P and O of both tiles live in
// TMEM side by side:
//   columns [64 t, +64)            S_t   = Q_t K_j^T (fp32)
//   columns [128 + 64 t + 32 b, +32) P_t, buffer b = j & 1 (bf16 pairs)
//   columns [256 + 128 t, +D)      O_t   (fp32 accumulator)
// so S_t(j+1) is computed while the softmax of block j still runs (it only
// has to wait until that softmax has copied S_t(j) into registers), and the
// softmax never waits for a PV product except to reuse a P buffer two blocks
// later. Per query tile the work is one chain of softmax blocks kept fed by
// the tensor pipe, and the two tiles' chains run side by side.
//
// Warp roles (352 threads):
//   warps 0-7  softmax: warp w serves tile w >> 2, thread = query row
//              32 (w & 3) + lane (= TMEM lane), all 64 columns of a block;
//   warp 8     TMA producer: both Q tiles once, then K and V blocks through
//              rings of shared-memory stages;
//   warps 9,10 MMA issuers, one per tile (one elected thread each): S_t(0),
//              then per block j: S_t(j+1) once the softmax released S_t(j),
//              PV_t(j) once P_t(j) is in TMEM. A K or V stage is released by
//              a commit (or, for a block the tile does not use, an arrive) of
//              each issuer, so the ring cannot be overrun by either.
//
// O / l leaves as bf16 through the tile's Q buffer (no product reads it once
// O is final) and TMA stores; lse is written per row.
//
// Online softmax in log2 units with a lazy rescale: a row's reference max
// moves (and O, l are rescaled) only when the max grows by more than 8, so P
// stays <= 2^8 and O is rarely touched; the final O / l and lse = (m +
// log2 l) ln 2 use the same reference, so the result is exact up to rounding.
// A fixed share of the exponentials (kPolyPairs pairs of every 32) runs as a
// polynomial on the FMA pipe, the rest on MUFU, so that neither unit alone
// sets the pace of the softmax; the share was measured per head size (0, 2,
// 4, 6, 8 pairs: 2 best at D = 128, 3 % faster than 8; 8 best at D = 64).
//
// Masking is per element only on blocks that cross the diagonal or the start
// of a row's document; key blocks wholly before the document of a tile's
// first row are never loaded (block skipping, per query tile), nor are
// blocks past the diagonal or past the sequence end.
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
  static constexpr int kQTileBytes = 128 * D * 2;  // 128 rows x D 16-bit values
  static constexpr int kQBlockBytes = 128 * 128;   // one 64-column block of a Q tile
  static constexpr int kKV = 64;                   // keys per block
  static constexpr int kKVBytes = kKV * D * 2;     // one K or V block
  static constexpr int kKVBlockBytes = kKV * 128;  // one 64-column block of it
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kQ = 0;  // Q_A, Q_B
  static constexpr int kK = kQ + 2 * kQTileBytes;
  static constexpr int kV = kK + kStages * kKVBytes;
  static constexpr int kBars = kV + kStages * kKVBytes;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bKFull = 1;
  static constexpr int bKEmpty = bKFull + kStages;
  static constexpr int bVFull = bKEmpty + kStages;
  static constexpr int bVEmpty = bVFull + kStages;
  static constexpr int bSFull = bVEmpty + kStages;  // [tile]: S_t(j) in TMEM
  static constexpr int bSFree = bSFull + 2;         // [tile], 4 warps: S_t(j) copied out
  static constexpr int bPFull = bSFree + 2;         // [tile][j & 1], 4 warps: P_t(j) stored
  static constexpr int bPVDone = bPFull + 4;        // [tile][j & 1]: PV_t(j) complete
  static constexpr int bOFinal = bPVDone + 4;       // [tile]
  static constexpr int kNumBars = bOFinal + 2;
  static constexpr int kMisc = (kBars + kNumBars * 8 + 15) / 16 * 16;  // [0] TMEM base, [1] abort flag
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kSmemAlloc = kBytes;  // the window is 1024-byte aligned (checked)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColP = 128, kColO = 256;
  static constexpr int kSoftmaxThreads = 256;
  static constexpr int kThreads = kSoftmaxThreads + 96;
  static constexpr int kProducerWarp = 8, kMmaWarp0 = 9;
  static constexpr int kPolyPairs = D == 128 ? 2 : 8;  // of the 32 pairs of a block row
  static_assert(kBytes <= 232448, "shared memory");
  static_assert(kQTileBytes % 1024 == 0 && kKVBytes % 1024 == 0, "swizzle atoms stay aligned");
  static_assert(kPolyPairs >= 0 && kPolyPairs <= 32, "poly share");
};

// Byte offset of 16-byte chunk `ch` (0..7 within a 64-column block) of row r
// in a 128-byte-swizzled tile block (the layout of the tensor maps' boxes).
__device__ __forceinline__ uint32_t sw128(int r, int ch) {
  return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
}

struct Params {
  int T, H, Hkv, BH, n_pairs, n_qtiles;  // H query heads read Hkv key/value heads
  float scale_log2;          // scale * log2(e)
  uint32_t idesc_s;          // instruction descriptor of S = Q K^T (M = 128, N = 64)
  const float* q_fac;        // inverse power-of-two factor per (query head, tile) of the
                             // stored rotated q, one 16-byte record each (value first),
                             // or null (q as given)
  const float* k_fac;        // the same per (key/value head, 128-key tile) for k, plain floats
  const int32_t* doc_start;  // flattened document starts, or null
  __nv_bfloat16* o;
  float* lse;
};

template <int D>
__global__ void __launch_bounds__(Layout<D>::kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const Params p) {
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
  // key blocks) are scheduled first.
  const int bh = (int)blockIdx.x % p.BH, b = bh / p.H;
  const int bhk = b * p.Hkv + (bh - b * p.H) / (p.H / p.Hkv);  // its key/value head
  const int pr = p.n_pairs - 1 - (int)blockIdx.x / p.BH;
  const int qtA = 2 * pr;
  const bool hasB = (qtA + 1) * 128 < T;
  const int row0 = b * T;
  const int n64 = (T + 63) >> 6;
  // Key blocks of tile t: [lo(t), hi(t)), from the block holding the start of
  // the document of the tile's first row to the block holding its last row's
  // key (its diagonal), clipped to the sequence. Every block of the range
  // holds a key some row of the tile may see (a query tile's allowed keys
  // form one interval). The producer loads the union [lo(0), hi_u).
  auto first_block = [&](int qt) -> int {
    return p.doc_start ? ((p.doc_start[row0 + qt * 128] - row0) >> 6) : 0;
  };
  const int lo0 = first_block(qtA);
  const int hi0 = min(2 * qtA + 2, n64);
  const int lo1 = hasB ? first_block(qtA + 1) : hi0;
  const int hi1 = hasB ? min(2 * qtA + 4, n64) : hi0;
  const int hi_u = hasB ? hi1 : hi0;
  auto lo_of = [&](int t) -> int { return t == 0 ? lo0 : lo1; };
  auto hi_of = [&](int t) -> int { return t == 0 ? hi0 : hi1; };

  if (threadIdx.x == 0) {
    const uint32_t users = hasB ? 2 : 1;  // issuers that release each K / V stage
    mbar_init(bar(L::bQFull), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::bKFull + s), 1);
      mbar_init(bar(L::bKEmpty + s), users);
      mbar_init(bar(L::bVFull + s), 1);
      mbar_init(bar(L::bVEmpty + s), users);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::bSFull + t), 1);
      mbar_init(bar(L::bSFree + t), 4);
      mbar_init(bar(L::bOFinal + t), 1);
      for (int e = 0; e < 2; ++e) {
        mbar_init(bar(L::bPFull + 2 * t + e), 4);
        mbar_init(bar(L::bPVDone + 2 * t + e), 1);
      }
    }
    *abort_flag = 0;
    fence_barrier_init();
    // 64-key blocks x 128 query rows processed (the tile counter's unit)
    atomicAdd(&g_attn_tiles[0], (unsigned long long)((hi0 - lo0) + (hasB ? hi1 - lo1 : 0)));
  }
  if (warp == L::kMmaWarp0) {
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
      mbar_arrive_expect_tx(bar(L::bQFull), (hasB ? 2 : 1) * L::kQTileBytes);
      for (int t = 0; t < (hasB ? 2 : 1); ++t)
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kQ + t * L::kQTileBytes + cb * L::kQBlockBytes, &tmQ,
                      bar(L::bQFull), cb * 64, (qtA + t) * 128, bh);
      for (int j = lo0; j < hi_u; ++j) {
        const int it = j - lo0, st = it % L::kStages, round = it / L::kStages;
        if (it >= L::kStages && !mbar_wait(bar(L::bKEmpty + st), (round - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::bKFull + st), L::kKVBytes);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kK + st * L::kKVBytes + cb * L::kKVBlockBytes, &tmK,
                      bar(L::bKFull + st), cb * 64, j * 64, bhk);
#ifdef ATTN_DEBUG_HOOKS
        if (it == 0 && g_attn_withhold == 1) continue;  // V(first block) never arrives
#endif
        if (it >= L::kStages && !mbar_wait(bar(L::bVEmpty + st), (round - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::bVFull + st), L::kKVBytes);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kV + st * L::kKVBytes + cb * L::kKVBlockBytes, &tmV,
                      bar(L::bVFull + st), cb * 64, j * 64, bhk);
      }
    }
  } else if (warp == L::kMmaWarp0 || warp == L::kMmaWarp0 + 1) {
    // ---------------- MMA issuers (one per tile) ----------------
    const int t = warp - L::kMmaWarp0;
    if (lane == 0 && (t == 0 || hasB)) {
      constexpr uint32_t idesc_o = idesc_f16(128, D, true, true, false, true);
      const int lo = lo_of(t), hi = hi_of(t), n = hi - lo;
      const uint32_t tS = tmem + L::kColS + 64 * t;
      const uint32_t tO = tmem + L::kColO + 128 * t;
      const uint32_t qbase = sb0 + L::kQ + t * L::kQTileBytes;
      auto stage = [&](int j) -> int { return (j - lo0) % L::kStages; };
      auto phase = [&](int j) -> uint32_t { return (uint32_t)((j - lo0) / L::kStages) & 1u; };
      // release a block this tile does not use (after it arrived, so that
      // the arrival counts toward that block's use of the stage)
      auto pass = [&](int j) -> bool {
        if (!mbar_wait(bar(L::bKFull + stage(j)), phase(j), abort_flag)) return false;
        mbar_arrive(bar(L::bKEmpty + stage(j)));
        if (!mbar_wait(bar(L::bVFull + stage(j)), phase(j), abort_flag)) return false;
        mbar_arrive(bar(L::bVEmpty + stage(j)));
        return true;
      };
      bool ok = true;
      for (int j = lo0; ok && j < lo; ++j) ok = pass(j);
      if (ok) ok = mbar_wait(bar(L::bQFull), 0, abort_flag);
      for (int li = 0; ok && li <= n; ++li) {
        if (li < n) {  // S_t(li) = Q_t K_j^T
          const int j = lo + li;
          const bool ready = li > 0 ? mbar_wait2(bar(L::bKFull + stage(j)), phase(j), bar(L::bSFree + t),
                                                 (li - 1) & 1, abort_flag)
                                    : mbar_wait(bar(L::bKFull + stage(j)), phase(j), abort_flag);
          if (!ready) { ok = false; break; }
          tc_fence_after();
          const uint32_t kbase = sb0 + L::kK + stage(j) * L::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tS,
                   smem_desc_sw128(qbase + (kk >> 2) * L::kQBlockBytes + (kk & 3) * 32, 16, 1024),
                   smem_desc_sw128(kbase + (kk >> 2) * L::kKVBlockBytes + (kk & 3) * 32, 16, 1024),
                   p.idesc_s, kk > 0);
          mma_commit(bar(L::bSFull + t));
          mma_commit(bar(L::bKEmpty + stage(j)));
        }
        if (li > 0) {  // O_t += P_t(lj) V_j
          const int lj = li - 1, j = lo + lj;
          if (!mbar_wait2(bar(L::bVFull + stage(j)), phase(j), bar(L::bPFull + 2 * t + (lj & 1)),
                          (lj >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t vbase = sb0 + L::kV + stage(j) * L::kKVBytes;
          const uint32_t aP = tmem + L::kColP + 64 * t + 32 * (lj & 1);
#pragma unroll
          for (int kk = 0; kk < L::kKV / 16; ++kk)
            mma_ts(tO, aP + kk * 8, smem_desc_sw128(vbase + kk * 2048, L::kKVBlockBytes, 1024),
                   idesc_o, (lj > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::bPVDone + 2 * t + (lj & 1)));
          mma_commit(bar(L::bVEmpty + stage(j)));
        }
      }
      if (ok) mma_commit(bar(L::bOFinal + t));
      for (int j = hi; ok && j < hi_u; ++j) ok = pass(j);
    }
  } else {
    // ---------------- softmax warps ----------------
    const int t = warp >> 2;
    const int r = (warp & 3) * 32 + lane;  // row within the tile = TMEM lane
    const int qt = qtA + t;
    const int i = qt * 128 + r;
    const bool active = (t == 0) || hasB;
    const int lo = lo_of(t), n = hi_of(t) - lo;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + L::kColS + 64 * t;
    const uint32_t tP = tmem + lane_base + L::kColP + 64 * t;
    const uint32_t tO = tmem + lane_base + L::kColO + 128 * t;
    const int ds_i = p.doc_start ? p.doc_start[row0 + min(i, T - 1)] - row0 : 0;
    const float fq = p.q_fac ? p.q_fac[((size_t)bh * p.n_qtiles + min(qt, p.n_qtiles - 1)) * 4] : 1.f;
    const float* kfp = p.k_fac ? p.k_fac + (size_t)bhk * p.n_qtiles : nullptr;
    float kf = (kfp && active) ? kfp[lo >> 1] : 1.f;  // this block's k factor (loaded a block ahead)
    float m = -INFINITY, l = 0.f;
    bool ok = active;
    for (int li = 0; ok && li < n; ++li) {
      const int j = lo + li, j0 = j * 64;  // first key of the block
      const float kf_next = (kfp && li + 1 < n) ? kfp[(j + 1) >> 1] : 1.f;
      if (!mbar_wait(bar(L::bSFull + t), li & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[64];
      tmem_ld32(tS, s);
      tmem_ld32(tS + 32, s + 32);
      tmem_wait_ld();
      // S_t(li) is in registers: the issuer may compute S_t(li+1) over it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::bSFree + t));
      // scale of this block's scores (q, k tiles may carry power-of-two
      // factors). A zero scale (uniform attention) is evaluated with the
      // smallest normal scale instead: a score below 2^100 in magnitude then
      // scales to below 2^-26, so each kept probability rounds to exactly 1
      // as it should, while a masked score still becomes -inf rather than
      // inf * 0 = NaN.
      float sc = p.scale_log2 * fq * kf;
      if (sc == 0.f) sc = 1.17549435e-38f;
      const bool pos_scale = sc > 0.f;
      const bool need_mask = (j0 + 63 > i) || (j0 < ds_i);
      const float masked = pos_scale ? -INFINITY : INFINITY;
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (j0 + c > i || j0 + c < ds_i) s[c] = __float_as_uint(masked);
      }
      // extreme of the raw scores (max for a positive scale)
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
      const float mx = ext * sc;  // -inf for a block the row may not see at all
      // Move the reference max only when it grows by more than 8 (log2
      // units); the first key a row sees always moves it (m = -inf).
      const bool move = mx > m + 8.f;
      const float alpha = move ? ex2(m - mx) : 1.f;
      // O needs rescaling only if it already holds a non-zero partial sum
      const bool scale_o = move && m != -INFINITY && li > 0;
      if (move) {
        l *= alpha;
        m = mx;
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      // P_t(li) goes to buffer li & 1, last read by PV_t(li - 2): asked now,
      // answered by the time P is formed
      const bool buf_free =
          li < 2 || mbar_test(bar(L::bPVDone + 2 * t + (li & 1)), ((li - 2) >> 1) & 1);
      // p = 2^(s * sc - m) two at a time, kPolyPairs of the 32 pairs on the
      // FMA pipe, the others on MUFU
      const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(-mref, -mref);
      float2 l2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 sv = make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1]));
        const float2 x = __ffma2_rn(sv, sc2, nm2);
        // pair e is a polynomial one when the running count e * share / 32
        // steps up at e (spreads kPolyPairs pairs evenly over the 32)
        const bool poly = (e * L::kPolyPairs) / 32 != ((e + 1) * L::kPolyPairs) / 32;
        const float2 pv = poly ? exp2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
        l2[e & 3] = __fadd2_rn(l2[e & 3], pv);
        pk[e] = pack_bf16(pv.x, pv.y);
      }
      const float2 la = __fadd2_rn(l2[0], l2[1]), lb = __fadd2_rn(l2[2], l2[3]);
      l += (la.x + la.y) + (lb.x + lb.y);
      if (!buf_free &&
          !mbar_wait(bar(L::bPVDone + 2 * t + (li & 1)), ((li - 2) >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      // rescale O (warp-collective: each lane by its own factor, 1 for lanes
      // that kept their max) once PV_t(li - 1), the last product into O, is done
      if (__any_sync(0xffffffffu, scale_o)) {
        if (!mbar_wait(bar(L::bPVDone + 2 * t + ((li - 1) & 1)), ((li - 1) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float f = scale_o ? alpha : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(tO + 32 * c, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st32(tO + 32 * c, ov);
        }
      }
      tc_fence_after();
      tmem_st32(tP + 32 * (li & 1), pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::bPFull + 2 * t + (li & 1)));
      kf = kf_next;
    }
    // O / l leaves as bf16 through this tile's Q buffer (no product reads
    // it once O is final) and TMA stores of 64-column boxes, rows past T
    // clipped by the map: stores to global memory from one query row per
    // lane took 32 cache lines per instruction.
    const bool epi = ok && mbar_wait(bar(L::bOFinal + t), 0, abort_flag);
    uint8_t* stage = sg + L::kQ + t * L::kQTileBytes;
    if (epi) {
      tc_fence_after();
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(tO + 32 * c, ov);  // warp-collective
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
        uint8_t* blk = stage + ((32 * c) >> 6) * L::kQBlockBytes;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4*>(blk + sw128(r, (((32 * c) & 63) >> 3) + e)) =
              make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
      fence_proxy_async_smem();
      if (i < T) p.lse[(size_t)bh * T + i] = (m + __log2f(l)) * 0.69314718055994531f;
    }
    // the tile's four warps all arrive (an aborted or idle one too, so none
    // waits for ever); before the CTA leaves the boxes must have been read,
    // the writes complete with the grid
    if (t == 0) asm volatile("barrier.sync 2, 128;" ::: "memory");
    else asm volatile("barrier.sync 3, 128;" ::: "memory");
    if ((warp & 3) == 0 && lane == 0 && epi) {
#pragma unroll
      for (int bcol = 0; bcol < D / 64; ++bcol)
        tma_store_3d(&tmO, smem_u32(stage) + bcol * L::kQBlockBytes, 64 * bcol, qt * 128, bh);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::kMmaWarp0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fwd100
