// bwd_sm100.cuh -- tensor-core (tcgen05) attention backward, key-tile
// parallel, for bf16 storage.
//
// One CTA owns one 128-key tile of one (b, h) slice; K and V stay in shared
// memory and the dK, dV accumulators stay in TMEM while the query tiles that
// can see these keys stream through (from the diagonal tile to the end of the
// last key's document). Per query tile i (keys are TMEM lanes, queries are
// columns):
//   S^T  = K Q^T           (TMEM)      dP^T = V dO^T        (TMEM)
//   P^T  = exp2(S^T * scale*log2e - lse2_i), masked; written back to TMEM (bf16)
//   dV  += P^T dO          (A = P^T from TMEM)
//   dS^T = P^T (dP^T - Delta_i), written to shared memory (bf16, 128-B swizzle)
//   dK  += dS^T Q          (A = dS^T read K-major from shared memory)
//   dQ_i = dS K            (A = the same tile read MN-major), into the dP^T
//                          columns; read out, staged in shared memory and
//                          added to the fp32 dq accumulator in global memory by
//                          bulk reduce-add operations of the TMA unit.
// The elementwise work runs in kNWG warpgroups (4 at D = 128, 2 at D = 64):
// warpgroup g takes query columns [g*kQC, (g+1)*kQC) of S^T and dP^T (its P^T
// goes to the first half of its own S^T columns, so warpgroups never touch
// each other's TMEM) and feature columns [g*kDC, (g+1)*kDC) of dQ_i, dK and
// dV; thread t of a warpgroup owns TMEM lane t (a key row, or a query row for
// dQ_i). The next warp streams Q (two stages, with lse2 and Delta riding on
// the same barrier) and dO with TMA after loading K and V once; the last warp
// owns TMEM and issues the MMAs. dK is
// scaled and rotated back (R^T) in the epilogue; dq is finished by a separate
// kernel once every key tile has added its part.
//
// Sources (page, section): ARK README, "Backward pass (AutoGrad)" (attention
// gradients inside training); Forge README, finding 3 (key-tile-parallel dK/dV
// kernels, the dK/dV split and register pressure) and "What this is" (fused
// flash-attention backward). The dQ accumulation follows the measurement
// contract's "atomic dQ" option (reduce-add in L2). Tiling, TMEM plan and warp
// roles are this library's own.
#pragma once

#include "sm100.cuh"

namespace bwd100 {

using namespace sm100;

template <int D>
struct Layout {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kDOStages = (D == 128) ? 1 : 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTileBytes;
  static constexpr int kQ = kV + kTileBytes;                  // 2 stages
  static constexpr int kDO = kQ + 2 * kTileBytes;             // kDOStages stages
  static constexpr int kDS = kDO + kDOStages * kTileBytes;    // 128 keys x 128 queries bf16
  static constexpr int kLD = kDS + 128 * 128 * 2;             // 2 x {-lse2[128], -delta[128]} f32
  // dQ_i staging: 32 x 32 fp32 boxes (4 KB), D/32 x 4 of them per tile: the
  // first 8 in the (then free) dS tile, the rest (D = 128) in this area.
  static constexpr int kXS = kLD + 2 * 1024;
  static constexpr int kBars = kXS + (D == 128 ? 8 * 4096 : 0);
  static constexpr int bKV = 0;
  static constexpr int bQFull = 1, bQEmpty = 3, bDOFull = 5, bDOEmpty = 7;  // 2 each
  static constexpr int bSFull = 9, bPFull = 10, bDPFull = 11, bDSFull = 12, bDVDone = 13,
                       bDQFull = 14, bDQFree = 15, bFinal = 16, bStageFree = 17;
  static constexpr int kNumBars = 18;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  // The dynamic shared-memory window starts 1024-byte aligned on sm_100 (after
  // the 1 KB the system reserves per block); the kernel checks this and
  // reports an error instead of running misaligned.
  static constexpr int kSmemAlloc = kBytes;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM columns: S^T (P^T over the first half of each warpgroup's 64), dP^T
  // (dQ_i after dS), dV, dK
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  // Elementwise warpgroups: 4 at D = 128 (16 warps), 2 at D = 64; each owns
  // kQC query columns of S^T / dP^T and kDC feature columns of dQ_i, dK, dV.
  static constexpr int kNWG = (D == 128) ? 4 : 2;
  static constexpr int kQC = 128 / kNWG;
  static constexpr int kDC = D / kNWG;
  static constexpr int kEwThreads = 128 * kNWG;
  static constexpr int kProducerWarp = 4 * kNWG, kMmaWarp = 4 * kNWG + 1;
  static constexpr int kThreads = kEwThreads + 64;
};

struct Params {
  int T, H, Hkv, BHkv, n_tiles, Tpad;  // H query heads read Hkv key/value heads
  float scale_log2;  // scale * log2(e)
  float scale;
  const float* lse2;       // [B*H][Tpad] -lse * log2(e), zero-padded
  const float* delta;      // [B*H][Tpad] -Delta, zero-padded
  const int32_t* doc_start;
  const int32_t* doc_end;  // flattened, or null
  const float* rope_cos;   // [T][D/2] or null
  const float* rope_sin;
  float* dq_acc;           // [B*H][T][D] fp32
  __nv_bfloat16* dk;       // [B*Hkv][T][D]
  __nv_bfloat16* dv;
};

// Byte offset of 16-byte chunk `ch` (0..7 within a 64-column block) of row r
// in a 128-byte-swizzled tile block.
__device__ __forceinline__ uint32_t sw128(int r, int ch) {
  return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(Layout<D>::kThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                const __grid_constant__ CUtensorMap tmDQ, const Params p) {
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
  // Flattened grid, heaviest key tiles (the earliest, which see the most
  // query tiles) first. One CTA per (key/value head, key tile); it walks the
  // query tiles of every query head reading that key/value head (G of them),
  // head by head: step `it` is query tile qt0 + it % n_q of the group's
  // it / n_q-th head.
  const int bhk = (int)blockIdx.x % p.BHkv, b = bhk / p.Hkv;
  const int kt = (int)blockIdx.x / p.BHkv;
  const int G = p.H / p.Hkv;
  const int bhq0 = b * p.H + (bhk - b * p.Hkv) * G;  // first query head of the group
  const int j0 = kt * 128;
  const int row0 = b * T;
  const int jlast = min(j0 + 127, T - 1);
  const int q_end = p.doc_end ? p.doc_end[row0 + jlast] - row0 : T;  // exclusive
  const int qt0 = kt;
  const int n_q = (q_end + 127) / 128 - qt0;
  const int n_it = G * n_q;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::bKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::bQFull + s), 1);
      mbar_init(bar(L::bQEmpty + s), 1);
      mbar_init(bar(L::bDOFull + s), 1);
      mbar_init(bar(L::bDOEmpty + s), 1);
    }
    mbar_init(bar(L::bSFull), 1);
    mbar_init(bar(L::bPFull), L::kEwThreads);
    mbar_init(bar(L::bDPFull), 1);
    mbar_init(bar(L::bDSFull), L::kEwThreads);
    mbar_init(bar(L::bDVDone), 1);
    mbar_init(bar(L::bDQFull), 1);
    mbar_init(bar(L::bDQFree), L::kEwThreads);
    mbar_init(bar(L::bFinal), 1);
    mbar_init(bar(L::bStageFree), L::kEwThreads);
    *abort_flag = 0;
    fence_barrier_init();
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
      mbar_arrive_expect_tx(bar(L::bKV), 2 * L::kTileBytes);
      for (int cb = 0; cb < D / 64; ++cb) {
        tma_load_3d(sb0 + L::kK + cb * L::kBlockBytes, &tmK, bar(L::bKV), cb * 64, j0, bhk);
        tma_load_3d(sb0 + L::kV + cb * L::kBlockBytes, &tmV, bar(L::bKV), cb * 64, j0, bhk);
      }
      for (int it = 0; it < n_it; ++it) {
        const int st = it & 1;
        const int so = it % L::kDOStages;
        const int gi = it / n_q;
        const int bh = bhq0 + gi;
        const int qrow = (qt0 + it - gi * n_q) * 128;
        const float* lse2_bh = p.lse2 + (size_t)bh * p.Tpad;
        const float* delta_bh = p.delta + (size_t)bh * p.Tpad;
        if (it >= 2 && !mbar_wait(bar(L::bQEmpty + st), ((it >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::bQFull + st), L::kTileBytes + 1024);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kQ + st * L::kTileBytes + cb * L::kBlockBytes, &tmQ,
                      bar(L::bQFull + st), cb * 64, qrow, bh);
        bulk_load(sb0 + L::kLD + st * 1024, lse2_bh + qrow, 512, bar(L::bQFull + st));
        bulk_load(sb0 + L::kLD + st * 1024 + 512, delta_bh + qrow, 512, bar(L::bQFull + st));
        if (it >= L::kDOStages &&
            !mbar_wait(bar(L::bDOEmpty + so), ((it / L::kDOStages) - 1) & 1, abort_flag))
          break;
        mbar_arrive_expect_tx(bar(L::bDOFull + so), L::kTileBytes);
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_3d(sb0 + L::kDO + so * L::kTileBytes + cb * L::kBlockBytes, &tmDO,
                      bar(L::bDOFull + so), cb * 64, qrow, bh);
      }
    }
  } else if (warp == L::kMmaWarp) {
    // ---------------- MMA issuer ----------------
    // Issue order per query tile i: dV(i), S(i+1), dK(i), dQ(i), dP(i+1), so
    // the tensor pipe has S(i+1) to run while the elementwise warps form dS(i),
    // and dK/dQ(i) while they form P(i+1). TMEM reuse: S(i+1) waits for dV(i)
    // (which reads P^T(i) from the S columns); dP(i+1) waits until dQ(i) has
    // been read out of the dP columns.
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16(128, 128, true, true, false, false);
      constexpr uint32_t id_dv = idesc_f16(128, D, true, true, false, true);
      constexpr uint32_t id_dk = idesc_f16(128, D, true, true, false, true);
      constexpr uint32_t id_dq = idesc_f16(128, D, true, true, true, true);
      const uint32_t tS = tmem + L::kColS, tDP = tmem + L::kColDP;
      const uint32_t tDV = tmem + L::kColDV, tDK = tmem + L::kColDK;
      auto qbuf = [&](int i) -> uint32_t { return sb0 + L::kQ + (i & 1) * L::kTileBytes; };
      auto obuf = [&](int i) -> uint32_t {
        return sb0 + L::kDO + (i % L::kDOStages) * L::kTileBytes;
      };
      // S^T(i) = K Q(i)^T
      auto issue_S = [&](int i) -> bool {
        if (!mbar_wait(bar(L::bQFull + (i & 1)), (i >> 1) & 1, abort_flag)) return false;
        if (i > 0 && !mbar_wait(bar(L::bDVDone), (i - 1) & 1, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBlockBytes + (kk & 3) * 32;
          mma_ss(tS, smem_desc_sw128(sb0 + L::kK + off, 16, 1024),
                 smem_desc_sw128(qbuf(i) + off, 16, 1024), id_s, kk > 0);
        }
        mma_commit(bar(L::bSFull));
        return true;
      };
      // dP^T(i) = V dO(i)^T
      auto issue_dP = [&](int i) -> bool {
        if (!mbar_wait(bar(L::bDOFull + i % L::kDOStages), (i / L::kDOStages) & 1, abort_flag))
          return false;
        if (i > 0 && !mbar_wait(bar(L::bDQFree), (i - 1) & 1, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBlockBytes + (kk & 3) * 32;
          mma_ss(tDP, smem_desc_sw128(sb0 + L::kV + off, 16, 1024),
                 smem_desc_sw128(obuf(i) + off, 16, 1024), id_s, kk > 0);
        }
        mma_commit(bar(L::bDPFull));
        return true;
      };
      bool ok = mbar_wait(bar(L::bKV), 0, abort_flag) && issue_S(0) && issue_dP(0);
      for (int it = 0; ok && it < n_it; ++it) {
        const int ph = it & 1;
        // dV += P^T dO; P^T of warpgroup g's query columns [g*kQC, (g+1)*kQC)
        // sits in TMEM columns [g*kQC, g*kQC + kQC/2), so the 16 queries of
        // k-step kk start at column 8*kk + (kQC/2) * (16*kk / kQC)
        if (!mbar_wait(bar(L::bPFull), ph, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tDV, tS + 8 * kk + (L::kQC / 2) * ((16 * kk) / L::kQC),
                 smem_desc_sw128(obuf(it) + kk * 2048, L::kBlockBytes, 1024), id_dv,
                 (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(L::bDVDone));
        mma_commit(bar(L::bDOEmpty + it % L::kDOStages));
        if (it + 1 < n_it && !issue_S(it + 1)) break;
        // dK += dS^T Q ; dQ_i = dS K
        if (!mbar_wait(bar(L::bDSFull), ph, abort_flag)) break;
        tc_fence_after();
        const uint32_t ds = sb0 + L::kDS;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tDK, smem_desc_sw128(ds + (kk >> 2) * L::kBlockBytes + (kk & 3) * 32, 16, 1024),
                 smem_desc_sw128(qbuf(it) + kk * 2048, L::kBlockBytes, 1024), id_dk,
                 (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tDP, smem_desc_sw128(ds + kk * 2048, L::kBlockBytes, 1024),
                 smem_desc_sw128(sb0 + L::kK + kk * 2048, L::kBlockBytes, 1024), id_dq, kk > 0);
        mma_commit(bar(L::bDQFull));
        mma_commit(bar(L::bQEmpty + (it & 1)));
        if (it == n_it - 1) mma_commit(bar(L::bFinal));
        if (it + 1 < n_it && !issue_dP(it + 1)) break;
      }
    }
  } else {
    // ---------------- elementwise warps ----------------
    constexpr int QC = L::kQC, DC = L::kDC;
    const int wg = warp >> 2, sub = warp & 3;
    const int r = sub * 32 + lane;  // TMEM lane: key row (S^T, dP^T, dK, dV) or query row (dQ_i)
    const int j = j0 + r;
    const int qc0 = QC * wg;        // query columns of S^T / dP^T handled here
    const int dc0 = DC * wg;        // feature columns of dQ_i / dK / dV handled here
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const int de_j = (j < T) ? (p.doc_end ? p.doc_end[row0 + j] - row0 : T) : T;
    const uint32_t tS = tmem + lane_base + L::kColS;
    const uint32_t tDP = tmem + lane_base + L::kColDP;
    uint8_t* dsb = sg + L::kDS;
    float pf[QC];  // P^T of this thread's key row, query columns [qc0, qc0 + QC)
    // ---- P^T(i) = exp2(S^T scale log2e - lse2), masked; bf16 copy to TMEM ----
    auto phase_P = [&](int i) -> bool {
      const int i0 = (qt0 + i % n_q) * 128;
      const bool need_mask = (i0 + qc0 < j) || (i0 + qc0 + QC - 1 >= de_j);
      const float* sl = reinterpret_cast<const float*>(sg + L::kLD + (i & 1) * 1024);
      if (!mbar_wait(bar(L::bQFull + (i & 1)), (i >> 1) & 1, abort_flag) ||
          !mbar_wait(bar(L::bSFull), i & 1, abort_flag))
        return false;
      tc_fence_after();
      uint32_t s[QC];
#pragma unroll
      for (int c = 0; c < QC / 32; ++c) tmem_ld32(tS + qc0 + 32 * c, s + 32 * c);
      tmem_wait_ld();
      const float2 scl2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
      for (int c = 0; c < QC / 32; ++c) {
        const int col = qc0 + 32 * c;
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 nl = reinterpret_cast<const float2*>(sl + col)[e];  // -lse2 pair
          const int i_a = i0 + col + 2 * e;
          const float2 sv = make_float2(__uint_as_float(s[32 * c + 2 * e]),
                                        __uint_as_float(s[32 * c + 2 * e + 1]));
          const float2 x = __ffma2_rn(sv, scl2, nl);
          // about a third of the pairs go to the FMA pipe
          float2 pv = (e % 3 == 2) ? exp2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
          if (need_mask) {
            if (i_a < j || i_a >= de_j) pv.x = 0.f;
            if (i_a + 1 < j || i_a + 1 >= de_j) pv.y = 0.f;
          }
          pf[32 * c + 2 * e] = pv.x;
          pf[32 * c + 2 * e + 1] = pv.y;
          pk[e] = pack_bf16(pv.x, pv.y);
        }
        tmem_st16(tS + qc0 + 16 * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::bPFull));
      return true;
    };
    // ---- dS^T(i) = P^T (dP^T - Delta) into the shared dS tile ----
    auto phase_dS = [&](int i) -> bool {
      const float* sd = reinterpret_cast<const float*>(sg + L::kLD + (i & 1) * 1024) + 128;
      // The dS tile doubled as dQ staging for tile i-1: every thread's bulk
      // reads of it must be done (a bounded barrier over the elementwise warps).
      bulk_wait_group_read0();
      mbar_arrive(bar(L::bStageFree));
      if (!mbar_wait(bar(L::bStageFree), i & 1, abort_flag) ||
          !mbar_wait(bar(L::bDPFull), i & 1, abort_flag))
        return false;
      tc_fence_after();
      uint32_t dpv[QC];
#pragma unroll
      for (int c = 0; c < QC / 32; ++c) tmem_ld32(tDP + qc0 + 32 * c, dpv + 32 * c);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < QC / 32; ++c) {
        const int col = qc0 + 32 * c;
        uint32_t dsk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 nd = reinterpret_cast<const float2*>(sd + col)[e];  // -Delta pair
          const float2 dpp = make_float2(__uint_as_float(dpv[32 * c + 2 * e]),
                                         __uint_as_float(dpv[32 * c + 2 * e + 1]));
          const float2 a = __fmul2_rn(make_float2(pf[32 * c + 2 * e], pf[32 * c + 2 * e + 1]),
                                      __fadd2_rn(dpp, nd));
          dsk[e] = pack_bf16(a.x, a.y);
        }
        // row r of the dS^T tile, query columns [col, col+32): block col/64,
        // 16-byte chunks (col%64)/8 .. +3
        uint8_t* blk = dsb + (col >> 6) * L::kBlockBytes;
        const int ch0 = (col & 63) >> 3;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4*>(blk + sw128(r, ch0 + e)) =
              make_uint4(dsk[4 * e], dsk[4 * e + 1], dsk[4 * e + 2], dsk[4 * e + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(L::bDSFull));
      return true;
    };
    // ---- dQ_i (lane = query row): release TMEM first, then reduce into global ----
    auto phase_dQ = [&](int i) -> bool {
      const int gi = i / n_q;
      const int i0 = (qt0 + i - gi * n_q) * 128;
      if (!mbar_wait(bar(L::bDQFull), i & 1, abort_flag)) return false;
      tc_fence_after();
      constexpr int NQC = DC / 32;  // 32-column chunks per warpgroup
      uint32_t dqv[NQC][32];
#pragma unroll
      for (int c = 0; c < NQC; ++c) tmem_ld32(tDP + dc0 + 32 * c, dqv[c]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(L::bDQFree));
      // Every thread has consumed the dS tile (dq_full implies the dK and dQ
      // MMAs are done), so it now serves as staging: one 32x32 fp32 box per
      // warp and chunk in the 128-byte-swizzled layout (conflict-free stores),
      // each added to the accumulator by one tensor reduce-add.
#pragma unroll
      for (int c = 0; c < NQC; ++c) {
        const int box = warp * NQC + c;
        uint8_t* bx = (box < 8) ? sg + L::kDS + box * 4096 : sg + L::kXS + (box - 8) * 4096;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<uint4*>(bx + sw128(lane, e)) =
              make_uint4(dqv[c][4 * e], dqv[c][4 * e + 1], dqv[c][4 * e + 2], dqv[c][4 * e + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && i0 + 32 * sub < T) {  // rows past T are clipped by the map
#pragma unroll
        for (int c = 0; c < NQC; ++c) {
          const int box = warp * NQC + c;
          const uint32_t bx = (box < 8) ? sb0 + L::kDS + box * 4096 : sb0 + L::kXS + (box - 8) * 4096;
          tma_reduce_add_3d(&tmDQ, bx, dc0 + 32 * c, i0 + 32 * sub, bhq0 + gi);
        }
        bulk_commit_group();
      }
      return true;
    };
    // Order: P(0); then per tile i: dS(i), P(i+1), dQ(i).
    bool ok = phase_P(0);
    for (int it = 0; ok && it < n_it; ++it) {
      ok = phase_dS(it) && (it + 1 >= n_it || phase_P(it + 1)) && phase_dQ(it);
    }
    bulk_wait_group0();
    // ---- epilogue: dK = R^T (scale * dK_r), dV ----
    if (ok && mbar_wait(bar(L::bFinal), 0, abort_flag)) {
      tc_fence_after();
      const int jj = min(j, T - 1);
      const int pos = jj - (p.doc_start ? p.doc_start[row0 + jj] - row0 : 0);
      __nv_bfloat16* dkrow = p.dk + ((size_t)bhk * T + jj) * D;
      __nv_bfloat16* dvrow = p.dv + ((size_t)bhk * T + jj) * D;
#pragma unroll
      for (int c = 0; c < DC / 32; ++c) {
        const int col = dc0 + 32 * c;
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + L::kColDK + col, v);
        tmem_wait_ld();
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]) * p.scale;
        if (p.rope_cos) rope_pairs<32, D>(f, p.rope_cos, p.rope_sin, pos, col, true);
        if (j < T) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            reinterpret_cast<uint4*>(dkrow + col)[e] =
                make_uint4(pack_bf16(f[8 * e], f[8 * e + 1]), pack_bf16(f[8 * e + 2], f[8 * e + 3]),
                           pack_bf16(f[8 * e + 4], f[8 * e + 5]), pack_bf16(f[8 * e + 6], f[8 * e + 7]));
        }
      }
#pragma unroll
      for (int c = 0; c < DC / 32; ++c) {
        const int col = dc0 + 32 * c;
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + L::kColDV + col, v);
        tmem_wait_ld();
        if (j < T) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            reinterpret_cast<uint4*>(dvrow + col)[e] = make_uint4(
                pack_bf16(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
                pack_bf16(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                pack_bf16(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                pack_bf16(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
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

}  // namespace bwd100
