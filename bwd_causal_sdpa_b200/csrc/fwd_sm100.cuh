// fwd_sm100.cuh -- tensor-core (tcgen05) attention forward for bf16 storage.
//
// One CTA computes one 128-row query tile of one (b, h) slice:
//   warps 0-3  softmax: thread t owns query row t (= TMEM lane t), so the row
//              max and row sum are thread-local (no shuffles);
//   warp 4     TMA producer: Q once, then K and V tiles through a ring of
//              shared-memory stages;
//   warp 5     TMEM owner and MMA issuer (one thread): S = Q K^T into one of
//              two TMEM score buffers, O += P V with P read from TMEM.
// Per key tile j the MMA warp issues S_j while the softmax warps still work
// on S_{j-1}; the softmax writes P_j (bf16) back over the first half of S_j's
// columns and the PV MMA reads it from there (A operand in TMEM).
//
// Online softmax in log2 units with a lazy rescale: the running max is only
// moved (and O, l rescaled) when a row's max grows by more than 8, so P stays
// <= 2^8 and O is rarely touched; the final O / l and lse = (m + log2 l) ln 2
// use the same reference, which makes the result exact up to rounding.
//
// Masking is per element only on tiles that cross the diagonal or the start
// of a row's document; tiles wholly before the first row's document are never
// loaded (block skipping), nor are tiles past the diagonal.
//
// Sources (page, section): ARK README, "Accelerated forward pass (GPU)" (SDPA
// with the causal mask fused in) and aten.metal entry (scores, softmax,
// weighted sum, fused causal kernel); Forge README, "Acknowledgements"
// (FlashAttention-2-style tiling) and finding 3 (keep the kernel's live state
// small). The tiling, TMEM use and warp roles are this library's own design.
#pragma once

#include "sm100.cuh"

namespace fwd100 {

using namespace sm100;

template <int D>
struct Layout {
  static constexpr int kTileBytes = 128 * D * 2;  // 128 rows x D 16-bit values
  static constexpr int kBlockBytes = 128 * 128;   // one 64-column block: 128 rows x 128 B
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBars = kV + kStages * kTileBytes;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bKFull = 1;
  static constexpr int bKEmpty = bKFull + kStages;
  static constexpr int bVFull = bKEmpty + kStages;
  static constexpr int bVEmpty = bVFull + kStages;
  static constexpr int bSFull = bVEmpty + kStages;  // 2
  static constexpr int bPFull = bSFull + 2;         // 2
  static constexpr int bPVDone = bPFull + 2;        // 2
  static constexpr int bOFinal = bPVDone + 2;       // 1
  static constexpr int kNumBars = bOFinal + 1;
  static constexpr int kMisc = kBars + kNumBars * 8;  // [0] TMEM base, [1] abort flag
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;  // slack to align the base to 1024
  // TMEM columns
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
};

struct Params {
  int T, H, BH, n_qtiles;
  float scale_log2;          // scale * log2(e)
  uint32_t idesc_s;          // instruction descriptor of S = Q K^T
  const float* q_fac;        // per (bh, tile) power-of-two factor of the stored q tile, or null
  const float* k_fac;
  const int32_t* doc_start;  // flattened document starts, or null
  __nv_bfloat16* o;
  float* lse;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb0 = (raw + 1023u) & ~1023u;
  uint8_t* sg = smem_raw + (sb0 - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sg + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + L::kMisc + 4);
  auto bar = [&](int i) -> uint32_t { return sb0 + L::kBars + 8u * i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  // Flattened grid, tile-major from the last query tile: the longest rows
  // (most key tiles) are scheduled first.
  const int bh = (int)blockIdx.x % p.BH, b = bh / p.H;
  const int qt = p.n_qtiles - 1 - (int)blockIdx.x / p.BH;
  const int q0 = qt * 128;
  const int row0 = b * T;
  const int ds0 = p.doc_start ? p.doc_start[row0 + q0] - row0 : 0;
  const int kv_t0 = ds0 >> 7;
  const int n_kv = qt - kv_t0 + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::bQFull), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::bKFull + s), 1);
      mbar_init(bar(L::bKEmpty + s), 1);
      mbar_init(bar(L::bVFull + s), 1);
      mbar_init(bar(L::bVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::bSFull + s), 1);
      mbar_init(bar(L::bPFull + s), 128);
      mbar_init(bar(L::bPVDone + s), 1);
    }
    mbar_init(bar(L::bOFinal), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(sb0 + L::kMisc, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tensor_map(&tmQ);
      prefetch_tensor_map(&tmK);
      prefetch_tensor_map(&tmV);
      mbar_arrive_expect_tx(bar(L::bQFull), L::kTileBytes);
      for (int cb = 0; cb < D / 64; ++cb)
        tma_load_3d(sb0 + L::kQ + cb * L::kBlockBytes, &tmQ, bar(L::bQFull), cb * 64, q0, bh);
      for (int it = 0; it < n_kv; ++it) {
        const int st = it % L::kStages, round = it / L::kStages;
        const int kvrow = (kv_t0 + it) * 128;
        if (it >= L::kStages && !mbar_wait(bar(L::bKEmpty + st), (round - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::bKFull + st), L::kTileBytes);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kK + st * L::kTileBytes + cb * L::kBlockBytes, &tmK,
                      bar(L::bKFull + st), cb * 64, kvrow, bh);
        if (it >= L::kStages && !mbar_wait(bar(L::bVEmpty + st), (round - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::bVFull + st), L::kTileBytes);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kV + st * L::kTileBytes + cb * L::kBlockBytes, &tmV,
                      bar(L::bVFull + st), cb * 64, kvrow, bh);
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_f16(128, D, true, true, false, true);
      bool ok = mbar_wait(bar(L::bQFull), 0, abort_flag);
      for (int it = 0; ok && it <= n_kv; ++it) {
        if (it < n_kv) {
          const int sbuf = it & 1, st = it % L::kStages;
          if (!mbar_wait(bar(L::bKFull + st), (it / L::kStages) & 1, abort_flag)) break;
          if (it >= 2 && !mbar_wait(bar(L::bPVDone + sbuf), ((it - 2) >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t dS = tmem + (sbuf ? L::kColS1 : L::kColS0);
          const uint32_t kbase = sb0 + L::kK + st * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBlockBytes + (kk & 3) * 32;
            mma_ss(dS, smem_desc_sw128(sb0 + L::kQ + off, 16, 1024),
                   smem_desc_sw128(kbase + off, 16, 1024), p.idesc_s, kk > 0);
          }
          mma_commit(bar(L::bSFull + sbuf));
          mma_commit(bar(L::bKEmpty + st));
        }
        if (it >= 1) {
          const int j = it - 1, pb = j & 1, vst = j % L::kStages;
          if (!mbar_wait(bar(L::bPFull + pb), (j >> 1) & 1, abort_flag)) break;
          if (!mbar_wait(bar(L::bVFull + vst), (j / L::kStages) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t aP = tmem + (pb ? L::kColS1 : L::kColS0);
          const uint32_t vbase = sb0 + L::kV + vst * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            mma_ts(tmem + L::kColO, aP + kk * 8,
                   smem_desc_sw128(vbase + kk * 2048, L::kBlockBytes, 1024), idesc_o,
                   (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(L::bPVDone + pb));
          mma_commit(bar(L::bVEmpty + vst));
          if (j == n_kv - 1) mma_commit(bar(L::bOFinal));
        }
      }
    }
  } else {
    // ---------------- softmax warps 0-3 ----------------
    const int r = threadIdx.x;  // row within the tile, TMEM lane
    const int i = q0 + r;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int ds_i = p.doc_start ? p.doc_start[row0 + min(i, T - 1)] - row0 : 0;
    const float fq = p.q_fac ? p.q_fac[bh * p.n_qtiles + qt] : 1.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int it = 0; it < n_kv; ++it) {
      const int sbuf = it & 1;
      const int kt = kv_t0 + it, j0 = kt * 128;
      if (!mbar_wait(bar(L::bSFull + sbuf), (it >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const float sc = p.scale_log2 * fq * (p.k_fac ? p.k_fac[bh * p.n_qtiles + kt] : 1.f);
      const uint32_t tS = tmem + lane_base + (sbuf ? L::kColS1 : L::kColS0);
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, s + 32 * c);
      tmem_wait_ld();
      const bool need_mask = (j0 + 127 > i) || (j0 < ds_i);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float x = __uint_as_float(s[c]) * sc;
        if (need_mask && (j0 + c > i || j0 + c < ds_i)) x = -INFINITY;
        s[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      // Move the reference max only when it grows by more than 8 (log2
      // units); the first key a row sees always moves it (m = -inf).
      const bool move = mx > m + 8.f;
      const float alpha = move ? ex2(m - mx) : 1.f;
      // O needs rescaling only if it already holds a non-zero partial sum.
      const bool scale_o = move && m != -INFINITY && it > 0;
      if (__any_sync(0xffffffffu, scale_o)) {
        // Warp-collective: wait for PV_{it-1}, then scale each lane's row by
        // its own factor (1 for lanes that keep their max).
        if (!mbar_wait(bar(L::bPVDone + ((it - 1) & 1)), ((it - 1) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float f = scale_o ? alpha : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_base + L::kColO + 32 * c, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st32(tmem + lane_base + L::kColO + 32 * c, ov);
        }
      }
      if (move) {
        l *= alpha;
        m = mx;
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(__uint_as_float(s[32 * c + 2 * e]) - mref);
          const float p1 = ex2(__uint_as_float(s[32 * c + 2 * e + 1]) - mref);
          l += p0 + p1;
          pk[e] = pack_bf16(p0, p1);
        }
        tmem_st16(tS + 16 * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::bPFull + sbuf));
    }
    if (ok && mbar_wait(bar(L::bOFinal), 0, abort_flag)) {
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.o + ((size_t)bh * T + min(i, T - 1)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(tmem + lane_base + L::kColO + 32 * c, ov);  // warp-collective
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
      if (i < T) p.lse[(size_t)bh * T + i] = (m + __log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fwd100
