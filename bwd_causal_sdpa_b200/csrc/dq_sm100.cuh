// dq_sm100.cuh -- the backward's query-tile pass: dQ of one 128-row query tile
// of one query head on the tensor cores (tcgen05), for bf16 storage.
//
// The key-tile kernel (bwd_sm100.cuh) forms dK and dV; this pass forms dQ
// without atomics: per query tile it recomputes, for every key tile the tile
// can see (from its first row's document start to its diagonal),
//   S  = Q K^T            (TMEM, lane = query row)
//   dP = dO V^T           (TMEM)
//   P  = exp2(S * scale*log2e - lse2), masked
//   dS = P (dP - Delta), into a shared tile (query rows, key columns)
//   dQ += dS K            (TMEM accumulator)
// and the epilogue stores dq = R^T (scale * dQ) as bf16, so the path needs no
// fp32 accumulator, no zeroing and no finishing pass. It costs two more
// products per tile pair than forming dQ beside dK and dV (S and dP are
// computed twice); which of the two ways is faster is a measured choice made
// by the host.
//
// Operand types follow the key-tile kernel: without RoPE q, k as given and dS
// in bf16; with RoPE (kF16) the rotated q, k as fp16 tiles with power-of-two
// factors (the forward's own values) and dS stored as dS * C * kinv_j, where
// kinv_j is key tile j's inverse factor (it cancels that tile's factor in dQ,
// which therefore accumulates C dS K over all key tiles) and C a power of two
// per CTA that keeps every stored value below 2^14 (from |dS_ij| <= |dO_i|
// max_j |v_j| + |Delta_i|, per-head maxima the preprocessing recorded); the
// epilogue divides by C.
//
// Warp roles: four elementwise warpgroups; warpgroup g takes key columns
// [32g, 32g + 32) of S and dP, thread t of a warpgroup owns query row t (TMEM
// lane t) and, in the epilogue, dQ columns [g D/4, (g + 1) D/4) of that row.
// One TMA warp (Q, dO, the row terms and the factor record once; then K and V
// through a ring of stages) and one MMA warp, which owns TMEM and issues each
// product as soon as its inputs are ready.
//
// Sources (page, section): ARK README, "Backward pass (AutoGrad)" (attention
// gradients inside training); Forge README, finding 3 (split backward
// kernels) and "What this is" (fused flash-attention backward). Tiling, TMEM
// plan and warp roles are this library's own.
#pragma once

#include "sm100.cuh"

namespace dq100 {

using namespace sm100;

template <int D>
struct Layout {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kStages = (D == 128) ? 2 : 3;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kTileBytes;
  static constexpr int kDS = kDO + kTileBytes;          // dS: 128 query rows x 128 keys, 16-bit
  static constexpr int kK = kDS + 128 * 128 * 2;        // kStages stages
  static constexpr int kV = kK + kStages * kTileBytes;  // kStages stages
  // -lse2[128], -delta[128] (f32) of the tile's rows, then the query tile's
  // inverse factor record (16 bytes, value first)
  static constexpr int kLD = kV + kStages * kTileBytes;
  static constexpr int kStats = kLD + 1024 + 16;        // per elementwise warp: largest kinv
  static constexpr int kBars = kStats + 16 * 4;
  static constexpr int bQ = 0;
  static constexpr int bKFull = 1, bKEmpty = bKFull + kStages, bVFull = bKEmpty + kStages,
                       bVEmpty = bVFull + kStages;
  static constexpr int bSFull = bVEmpty + kStages, bSFree = bSFull + 1, bDPFull = bSFree + 1,
                       bDPFree = bDPFull + 1, bDSFull = bDPFree + 1, bDSFree = bDSFull + 1,
                       bFinal = bDSFree + 1, bStats = bFinal + 1;
  static constexpr int kNumBars = bStats + 1;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kSmemAlloc = kBytes;  // the window is 1024-byte aligned (checked)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256;
  static constexpr int kEwThreads = 512;
  static constexpr int kProducerWarp = 16, kMmaWarp = 17;
  static constexpr int kThreads = kEwThreads + 64;
  static_assert(kK % 1024 == 0 && kV % 1024 == 0 && kDS % 1024 == 0, "128-byte swizzle atoms");
  static_assert(kBytes <= 232448, "more shared memory than a CTA may use");
};

struct Params {
  int T, H, Hkv, BH, n_tiles, Tpad;
  float scale_log2;        // scale * log2(e)
  float scale;
  const float* lse2;       // [B*H][Tpad] -lse * log2(e), zero-padded
  const float* delta;      // [B*H][Tpad] -Delta, zero-padded
  const int32_t* doc_start;  // flattened, or null
  const float* rope_cos;   // [T][D/2] or null
  const float* rope_sin;
  // fp16 operands: inverse factors of the stored q (16-byte records,
  // [B*H][n_tiles]) and k ([B*Hkv][n_tiles]); per query head the largest
  // |dO_i| and |Delta_i|, per key/value head the largest |v_j| ([B*H][4]:
  // dO, Delta, v, unused)
  const float* qinv;
  const float* kinv;
  const float* hstat;
  __nv_bfloat16* dq;       // [B*H][T][D]
};

// Byte offset of 16-byte chunk `ch` (0..7 within a 64-column block) of row r
// in a 128-byte-swizzled tile block.
__device__ __forceinline__ uint32_t sw128(int r, int ch) {
  return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
}

// C from X >= max |dS_ij| kinv_j (see bwd_sm100.cuh): every stored value
// stays below 2^14; 1 when X is zero.
__device__ __forceinline__ float dq_ds_scale(float X) {
  if (!(X > 0.f && X <= 3.0e38f)) return 1.f;
  return ldexpf(1.f, max(-100, min(100, 13 - ilogbf(X))));
}

template <int D, bool kF16>
__global__ void __launch_bounds__(Layout<D>::kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
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
  // Flattened grid, the last query tiles (which see the most keys) first.
  const int bh = (int)blockIdx.x % p.BH, b = bh / p.H;
  const int bhk = b * p.Hkv + (bh - b * p.H) / (p.H / p.Hkv);  // its key/value head
  const int qt = p.n_tiles - 1 - (int)blockIdx.x / p.BH;
  const int row0 = b * T;
  // key tiles [kt_lo, qt]: from the tile holding the start of the first row's
  // document (a query tile's allowed keys form one interval) to the diagonal
  // document ranges clamped into the row (they may come from the caller's saved buffer)
  const int kt_lo =
      p.doc_start ? (min(max(p.doc_start[row0 + qt * 128] - row0, 0), qt * 128) >> 7) : 0;
  const int n_kv = qt - kt_lo + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::bQ), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::bKFull + s), 1);
      mbar_init(bar(L::bKEmpty + s), 1);
      mbar_init(bar(L::bVFull + s), 1);
      mbar_init(bar(L::bVEmpty + s), 1);
    }
    mbar_init(bar(L::bSFull), 1);
    mbar_init(bar(L::bSFree), L::kEwThreads);
    mbar_init(bar(L::bDPFull), 1);
    mbar_init(bar(L::bDPFree), L::kEwThreads);
    mbar_init(bar(L::bDSFull), L::kEwThreads);
    mbar_init(bar(L::bDSFree), 1);
    mbar_init(bar(L::bFinal), 1);
    mbar_init(bar(L::bStats), L::kEwThreads);
    *abort_flag = 0;
    fence_barrier_init();
    atomicAdd(&g_attn_tiles[2], (unsigned long long)n_kv);
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
      prefetch_tensor_map(&tmDO);
      const int qrow = qt * 128;
      mbar_arrive_expect_tx(bar(L::bQ), 2 * L::kTileBytes + 1024 + (kF16 ? 16 : 0));
      for (int cb = 0; cb < D / 64; ++cb) {
        tma_load_3d(sb0 + L::kQ + cb * L::kBlockBytes, &tmQ, bar(L::bQ), cb * 64, qrow, bh);
        tma_load_3d(sb0 + L::kDO + cb * L::kBlockBytes, &tmDO, bar(L::bQ), cb * 64, qrow, bh);
      }
      bulk_load(sb0 + L::kLD, p.lse2 + (size_t)bh * p.Tpad + qrow, 512, bar(L::bQ));
      bulk_load(sb0 + L::kLD + 512, p.delta + (size_t)bh * p.Tpad + qrow, 512, bar(L::bQ));
      if (kF16)
        bulk_load(sb0 + L::kLD + 1024, p.qinv + ((size_t)bh * p.n_tiles + qt) * 4, 16, bar(L::bQ));
      for (int it = 0; it < n_kv; ++it) {
        const int st = it % L::kStages, round = it / L::kStages;
        const int kvrow = (kt_lo + it) * 128;
        if (it >= L::kStages && !mbar_wait(bar(L::bKEmpty + st), (round - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::bKFull + st), L::kTileBytes);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kK + st * L::kTileBytes + cb * L::kBlockBytes, &tmK,
                      bar(L::bKFull + st), cb * 64, kvrow, bhk);
        if (it >= L::kStages && !mbar_wait(bar(L::bVEmpty + st), (round - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::bVFull + st), L::kTileBytes);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kV + st * L::kTileBytes + cb * L::kBlockBytes, &tmV,
                      bar(L::bVFull + st), cb * 64, kvrow, bhk);
      }
    }
  } else if (warp == L::kMmaWarp) {
    // ---------------- MMA issuer ----------------
    // Three groups per key tile i: S(i), dP(i), dQ(i), each in tile order,
    // issued as soon as ready (non-blocking probes), in the priority S, dP,
    // dQ. Readiness:
    //   S(i):  K(i) loaded; the S columns free (S(0) always, else the
    //          elementwise warps have read S(i-1))
    //   dP(i): V(i) loaded; the dP columns free (likewise)
    //   dQ(i): dS(i) in the shared tile (S(i) was issued before it)
    // Commits: S(i) -> SFull; dP(i) -> DPFull and V(i)'s stage free; dQ(i)
    // -> the dS tile free and K(i)'s stage free (dQ(i) is K(i)'s last reader).
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16(128, 128, !kF16, !kF16, false, false);
      constexpr uint32_t id_dp = idesc_f16(128, 128, true, true, false, false);
      constexpr uint32_t id_dq = idesc_f16(128, D, !kF16, !kF16, false, true);
      const uint32_t tS = tmem + L::kColS, tDP = tmem + L::kColDP, tDQ = tmem + L::kColDQ;
      const uint32_t ds = sb0 + L::kDS;
      int nS = 0, nP = 0, nQ = 0;
      bool ok = mbar_wait(bar(L::bQ), 0, abort_flag);
      long long t_last = clock64();
      while (ok && nQ < n_kv) {
        if (nS < n_kv &&
            mbar_test(bar(L::bKFull + nS % L::kStages), (nS / L::kStages) & 1) &&
            (nS == 0 || mbar_test(bar(L::bSFree), (nS - 1) & 1))) {
          // S(i) = Q K(i)^T
          tc_fence_after();
          const uint32_t kbase = sb0 + L::kK + (nS % L::kStages) * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBlockBytes + (kk & 3) * 32;
            mma_ss(tS, smem_desc_sw128(sb0 + L::kQ + off, 16, 1024),
                   smem_desc_sw128(kbase + off, 16, 1024), id_s, kk > 0);
          }
          mma_commit(bar(L::bSFull));
          ++nS;
        } else if (nP < n_kv &&
                   mbar_test(bar(L::bVFull + nP % L::kStages), (nP / L::kStages) & 1) &&
                   (nP == 0 || mbar_test(bar(L::bDPFree), (nP - 1) & 1))) {
          // dP(i) = dO V(i)^T
          tc_fence_after();
          const uint32_t vbase = sb0 + L::kV + (nP % L::kStages) * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBlockBytes + (kk & 3) * 32;
            mma_ss(tDP, smem_desc_sw128(sb0 + L::kDO + off, 16, 1024),
                   smem_desc_sw128(vbase + off, 16, 1024), id_dp, kk > 0);
          }
          mma_commit(bar(L::bDPFull));
          mma_commit(bar(L::bVEmpty + nP % L::kStages));
          ++nP;
        } else if (nQ < nS && mbar_test(bar(L::bDSFull), nQ & 1)) {
          // dQ += dS(i) K(i) (dS K-major, K read MN-major)
          tc_fence_after();
          const uint32_t kbase = sb0 + L::kK + (nQ % L::kStages) * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tDQ, smem_desc_sw128(ds + (kk >> 2) * L::kBlockBytes + (kk & 3) * 32, 16, 1024),
                   smem_desc_sw128(kbase + kk * 2048, L::kBlockBytes, 1024), id_dq,
                   (nQ > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::bDSFree));
          mma_commit(bar(L::bKEmpty + nQ % L::kStages));
          if (nQ == n_kv - 1) mma_commit(bar(L::bFinal));
          ++nQ;
        } else {
          // nothing ready: keep probing; give up like mbar_wait does
          if (*abort_flag) break;
          if (clock64() - t_last > kWaitLimitCycles) {
            *abort_flag = 1;
            report_status(ATTN_ETIMEOUT);
            break;
          }
          continue;
        }
        t_last = clock64();
      }
    }
  } else {
    // ---------------- elementwise warps ----------------
    constexpr int QC = 32;      // key columns of S / dP per warpgroup
    constexpr int DC = D / 4;   // dQ columns per warpgroup in the epilogue
    const int wg = warp >> 2, sub = warp & 3;
    const int r = sub * 32 + lane;      // query row in the tile = TMEM lane
    const int i = qt * 128 + r;         // query index in the row
    const int kc0 = QC * wg;            // key columns handled here
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const uint32_t tS = tmem + lane_base + L::kColS + kc0;
    const uint32_t tDP = tmem + lane_base + L::kColDP + kc0;
    const int ds_i = p.doc_start ? min(max(p.doc_start[row0 + min(i, T - 1)] - row0, 0), min(i, T - 1)) : 0;
    uint8_t* dsb = sg + L::kDS + (kc0 >> 6) * L::kBlockBytes;
    const int ch0 = (kc0 & 63) >> 3;
    bool ok = mbar_wait(bar(L::bQ), 0, abort_flag);
    const float* ld = reinterpret_cast<const float*>(sg + L::kLD);
    const float nl = ok ? ld[r] : 0.f;          // -lse_i log2(e)
    const float nd = ok ? ld[128 + r] : 0.f;    // -Delta_i
    const float qinv = (kF16 && ok) ? ld[256] : 1.f;
    float cscale = 1.f;
    // C (fp16 operands): the largest kinv over this CTA's key tiles, with the
    // per-head maxima of |dO_i|, |Delta_i| and |v_j|; posted after the first P
    // (C is first needed by the first dS)
    auto post_stats = [&]() -> bool {
      float km = 0.f;
      for (int e = threadIdx.x; e < n_kv; e += L::kEwThreads)
        km = fmaxf(km, p.kinv[(size_t)bhk * p.n_tiles + kt_lo + e]);
      km = warp_max(km);
      float* st = reinterpret_cast<float*>(sg + L::kStats);
      if (lane == 0) st[warp] = km;
      mbar_arrive(bar(L::bStats));
      if (!mbar_wait(bar(L::bStats), 0, abort_flag)) return false;
      float kmax = st[0];
#pragma unroll
      for (int w = 1; w < 16; ++w) kmax = fmaxf(kmax, st[w]);
      const float dom = p.hstat[4 * bh], dlm = p.hstat[4 * bh + 1], vm = p.hstat[4 * bhk + 2];
      cscale = dq_ds_scale(kmax * fmaf(dom, vm, dlm));
      return true;
    };
    float pf[QC];
    for (int it = 0; ok && it < n_kv; ++it) {
      const int kt = kt_lo + it;
      const int j0 = kt * 128 + kc0;  // first key of this thread's columns
      const float kinv = kF16 ? p.kinv[(size_t)bhk * p.n_tiles + kt] : 1.f;
      // ---- P = exp2(S * scale log2e - lse2), masked ----
      if (!mbar_wait(bar(L::bSFull), it & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[QC];
      tmem_ld32(tS, s);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(L::bSFree));
      const float sc = p.scale_log2 * qinv * kinv;
      const bool need_mask = (j0 + QC - 1 > i) || (j0 < ds_i);
#pragma unroll
      for (int e = 0; e < QC; ++e) {
        const float x = fmaf(__uint_as_float(s[e]), sc, nl);
        float pv = ex2(x);
        if (need_mask && (j0 + e > i || j0 + e < ds_i)) pv = 0.f;
        pf[e] = pv;
      }
      if (kF16 && it == 0 && !post_stats()) { ok = false; break; }
      // ---- dS = P (dP - Delta), into the shared tile once dQ(i-1) read it ----
      if (!mbar_wait(bar(L::bDPFull), it & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t dpv[QC];
      tmem_ld32(tDP, dpv);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(L::bDPFree));
      const float dsm = cscale * kinv;  // 1 for bf16 operands
      uint32_t w[QC / 2];
#pragma unroll
      for (int e = 0; e < QC / 2; ++e) {
        const float a0 = pf[2 * e] * ((__uint_as_float(dpv[2 * e]) + nd) * dsm);
        const float a1 = pf[2 * e + 1] * ((__uint_as_float(dpv[2 * e + 1]) + nd) * dsm);
        w[e] = kF16 ? pack_half(a0, a1) : pack_bf16(a0, a1);
      }
      if (it > 0 && !mbar_wait(bar(L::bDSFree), (it - 1) & 1, abort_flag)) { ok = false; break; }
#pragma unroll
      for (int e = 0; e < 4; ++e)
        *reinterpret_cast<uint4*>(dsb + sw128(r, ch0 + e)) =
            make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
      fence_proxy_async_smem();
      mbar_arrive(bar(L::bDSFull));
    }
    // ---- epilogue: dq = R^T (scale / C * dQ), bf16 ----
    if (ok && mbar_wait(bar(L::bFinal), 0, abort_flag)) {
      tc_fence_after();
      const int ii = min(i, T - 1);
      const int pos = ii - (p.doc_start ? min(max(p.doc_start[row0 + ii] - row0, 0), ii) : 0);
      __nv_bfloat16* dqrow = p.dq + ((size_t)bh * T + ii) * D;
      const float f = p.scale / cscale;
      constexpr int CW = DC < 32 ? DC : 32;  // columns per TMEM load
#pragma unroll
      for (int c = 0; c < DC / CW; ++c) {
        const int col = DC * wg + CW * c;
        uint32_t v[CW];
        if constexpr (CW == 32) tmem_ld32(tmem + lane_base + L::kColDQ + col, v);
        else tmem_ld16(tmem + lane_base + L::kColDQ + col, v);
        tmem_wait_ld();
        float x[CW];
#pragma unroll
        for (int e = 0; e < CW; ++e) x[e] = __uint_as_float(v[e]) * f;
        if (p.rope_cos) rope_pairs<CW, D>(x, p.rope_cos, p.rope_sin, pos, col, true);
        if (i < T) {
#pragma unroll
          for (int e = 0; e < CW / 8; ++e)
            reinterpret_cast<uint4*>(dqrow + col)[e] =
                make_uint4(pack_bf16(x[8 * e], x[8 * e + 1]), pack_bf16(x[8 * e + 2], x[8 * e + 3]),
                           pack_bf16(x[8 * e + 4], x[8 * e + 5]), pack_bf16(x[8 * e + 6], x[8 * e + 7]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace dq100
