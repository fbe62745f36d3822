// bwd_pair_sm100.cuh -- the key-tile backward (dK, dV) on a pair of CTAs:
// tcgen05 products with M = 256 keys (cta_group::2), D = 128.
//
// A cluster of two CTAs owns 256 consecutive keys of one key/value head:
// CTA r (its rank in the cluster) keeps keys [256 p + 128 r, +128) in its
// shared memory and the dK, dV rows of those keys in its TMEM, and both walk
// the same query tiles (from the pair's first diagonal tile to the end of
// the document of the pair's last key, for every query head of the group).
// Per query tile i, four products, each one instruction stream on the pair:
//   S^T  = K Q^T     A: each CTA's K rows       B: query rows split, CTA r
//                                                  holding rows [64 r, +64)
//   dP^T = V dO^T    A: each CTA's V rows       B: dO rows split likewise
//   dV  += P^T dO    A: each CTA's P^T rows     B: dO feature columns split,
//                                                  CTA r holding [64 r, +64)
//   dK  += dS^T Q    A: each CTA's dS^T rows    B: Q feature columns split
// so each SM reads half of every B operand from its own shared memory, and
// the pair's tensor work is issued by one thread of CTA 0 (the leader). dQ is
// formed by the query-tile pass (dq_sm100.cuh) instead: dQ_i = dS K sums over
// the pair's 256 keys, which no split of this product over the pair keeps
// local to one CTA.
//
// Synchronisation: every load of both CTAs signals the leader's barriers (the
// leader expects both CTAs' bytes), the elementwise warps of both CTAs arrive
// on the leader's barriers (one arrival per warp, over the cluster), and each
// product's commit arrives on the same barrier in both CTAs. Elementwise work,
// statistics and the epilogue follow the single-CTA kernel (bwd_sm100.cuh),
// each CTA on its own key rows; with fp16 operands each CTA's dS scale C is
// its own (its dK rows are divided by it), made from the preprocessing's
// per-head maxima.
//
// Sources (page, section): ARK README, "Backward pass (AutoGrad)"; Forge
// README, finding 3 (key-tile-parallel dK/dV kernels). The pairing of SMs on
// one product is this library's own B200 design (no page describes it).
#pragma once

#include "bwd_sm100.cuh"

namespace bwd2 {

using namespace sm100;
using bwd100::ds_scale;
using bwd100::Params;
using bwd100::sw128;

template <int D>
struct Layout {
  static_assert(D == 128, "the pair kernel splits 64-column halves of D = 128");
  static constexpr int kTileBytes = 128 * D * 2;   // 32 KB
  static constexpr int kHalfBytes = kTileBytes / 2;
  static constexpr int kBlockBytes = 128 * 128;    // 64 columns x 128 rows
  static constexpr int kRowHalfBlock = 64 * 128;   // 64 columns x 64 rows
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTileBytes;
  // Q and dO stages: [rows half: 64 rows x D][feature half: 128 rows x 64]
  static constexpr int kQ = kV + kTileBytes;
  static constexpr int kDO = kQ + 2 * kTileBytes;
  static constexpr int kPS = kDO + 2 * kTileBytes;  // P^T then dS^T, this CTA's 128 keys x 128 queries
  static constexpr int kLD = kPS + 128 * 128 * 2;   // 2 x {-lse2[128], -delta[128]} f32
  static constexpr int kStats = kLD + 2 * 1024;     // f32 [16 warps][4]
  static constexpr int kQInv = kStats + 16 * 4 * 4; // 2 x 16-byte records
  static constexpr int kBars = kQInv + 2 * 16;
  static constexpr int bKV = 0, bQFull = 1, bQEmpty = 3, bLDFull = 5, bDOFull = 7, bDOEmpty = 9,
                       bSFull = 11, bSFree = 12, bPFull = 13, bDPFull = 14, bDSFull = 15,
                       bDVDone = 16, bDSFree = 17, bFinal = 18, bStats = 19;
  static constexpr int kNumBars = 20;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kSmemAlloc = kBytes;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  static constexpr int kNWG = 4, kQC = 32, kDC = D / 4, kEwThreads = 512;
  static constexpr int kEwWarps = 16;
  static constexpr int kProducerWarp = 16, kMmaWarp = 17;
  static constexpr int kThreads = 576;
  static_assert(kBytes <= 232448, "more shared memory than a CTA may use");
  static_assert(kQ % 1024 == 0 && kDO % 1024 == 0 && kPS % 1024 == 0, "swizzle atoms aligned");
};

// Grid: two CTAs (a cluster) per (key/value head, pair of key tiles, part of
// the query-head group), heaviest pairs first. tmQr / tmOr: q, dO in boxes of
// 64 rows (the row halves), tmQc / tmOc: boxes of 128 rows (the feature
// halves), tmK / tmV: 128-row boxes.
template <int D, bool kF16>
__global__ void __launch_bounds__(Layout<D>::kThreads, 1)
    dkdv_pair_kernel(const __grid_constant__ CUtensorMap tmQr, const __grid_constant__ CUtensorMap tmQc,
                     const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmOr, const __grid_constant__ CUtensorMap tmOc,
                     const Params p) {
  pdl_wait_and_trigger();
  using L = Layout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sb0 = smem_u32(smem_raw);
  if (sb0 & 1023u) {  // the same in both CTAs: neither reaches a cluster barrier
    if (threadIdx.x == 0) report_status(ATTN_ECUDA_LAYOUT);
    return;
  }
  uint8_t* sg = smem_raw;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sg + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + L::kMisc + 4);
  auto bar = [&](int i) -> uint32_t { return sb0 + L::kBars + 8u * i; };
  const uint32_t rank = cluster_rank();
  auto lead = [&](int i) -> uint32_t { return map_rank(bar(i), 0); };  // the leader's barrier

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int pair = (int)blockIdx.x >> 1;
  const int bhk = pair % p.BHkv, b = bhk / p.Hkv;
  const int ktp = pair / (p.BHkv * p.n_split);
  const int part = (pair / p.BHkv) % p.n_split;
  const int G = p.H / p.Hkv / p.n_split;
  const int bhq0 = b * p.H + (bhk - b * p.Hkv) * (p.H / p.Hkv) + part * G;
  const int kt = 2 * ktp + (int)rank;  // this CTA's key tile (past the sequence: all keys masked)
  const int j0 = kt * 128;
  const int row0 = b * T;
  // the pair walks from its first diagonal tile to the end of its last key's document
  const int jlast = min(256 * ktp + 255, T - 1);
  const int q_end = p.doc_end ? min(max(p.doc_end[row0 + jlast] - row0, jlast + 1), T) : T;
  const int qt0 = 2 * ktp;
  const int n_q = (q_end + 127) / 128 - qt0;
  const int n_it = G * n_q;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::bKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::bQFull + s), 1);
      mbar_init(bar(L::bQEmpty + s), 1);
      mbar_init(bar(L::bLDFull + s), 1);
      mbar_init(bar(L::bDOFull + s), 1);
      mbar_init(bar(L::bDOEmpty + s), 1);
    }
    mbar_init(bar(L::bSFull), 1);
    mbar_init(bar(L::bSFree), 2 * L::kEwWarps);  // one arrival per elementwise warp of each CTA
    mbar_init(bar(L::bPFull), 2 * L::kEwWarps);
    mbar_init(bar(L::bDPFull), 1);
    mbar_init(bar(L::bDSFull), 2 * L::kEwWarps);
    mbar_init(bar(L::bDVDone), 1);
    mbar_init(bar(L::bDSFree), 1);
    mbar_init(bar(L::bFinal), 1);
    mbar_init(bar(L::bStats), L::kEwThreads);
    *abort_flag = 0;
    fence_barrier_init();
    atomicAdd(&g_attn_tiles[1], (unsigned long long)n_it);
  }
  if (warp == L::kMmaWarp) {  // the same warp in both CTAs, the same destination offset
    tmem_alloc_pair(sb0 + L::kMisc, L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const float kinv_cta = (kF16 && kt < p.n_tiles) ? p.kinv[(size_t)bhk * p.n_tiles + kt] : 1.f;
  float* stats = reinterpret_cast<float*>(sg + L::kStats);  // [warp][4]

  if (warp == L::kProducerWarp) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      prefetch_tensor_map(&tmQr);
      prefetch_tensor_map(&tmQc);
      prefetch_tensor_map(&tmK);
      prefetch_tensor_map(&tmV);
      prefetch_tensor_map(&tmOr);
      prefetch_tensor_map(&tmOc);
      if (rank == 0) mbar_arrive_expect_tx(bar(L::bKV), 4 * L::kTileBytes);  // K, V of both CTAs
      for (int cb = 0; cb < D / 64; ++cb) {
        tma_load_3d_pair(sb0 + L::kK + cb * L::kBlockBytes, &tmK, lead(L::bKV), cb * 64, j0, bhk);
        tma_load_3d_pair(sb0 + L::kV + cb * L::kBlockBytes, &tmV, lead(L::bKV), cb * 64, j0, bhk);
      }
      int nq = 0, no = 0;
      long long t_last = clock64();
      while (nq < n_it || no < n_it) {
        bool did = false;
        if (nq < n_it && (nq < 2 || mbar_test(bar(L::bQEmpty + (nq & 1)), ((nq >> 1) - 1) & 1))) {
          const int st = nq & 1, gi = nq / n_q, bh = bhq0 + gi;
          const int qrow = (qt0 + nq - gi * n_q) * 128;
          const uint32_t qb = sb0 + L::kQ + st * L::kTileBytes;
          if (rank == 0) mbar_arrive_expect_tx(bar(L::bQFull + st), 2 * L::kTileBytes);
          for (int cb = 0; cb < D / 64; ++cb)  // rows [64 rank, +64), every feature
            tma_load_3d_pair(qb + cb * L::kRowHalfBlock, &tmQr, lead(L::bQFull + st), cb * 64,
                             qrow + 64 * (int)rank, bh);
          // every row, features [64 rank, +64)
          tma_load_3d_pair(qb + L::kHalfBytes, &tmQc, lead(L::bQFull + st), 64 * (int)rank, qrow, bh);
          mbar_arrive_expect_tx(bar(L::bLDFull + st), 1024 + (kF16 ? 16 : 0));
          const uint32_t ld = sb0 + L::kLD + st * 1024;
          bulk_load(ld, p.lse2 + (size_t)bh * p.Tpad + qrow, 512, bar(L::bLDFull + st));
          bulk_load(ld + 512, p.delta + (size_t)bh * p.Tpad + qrow, 512, bar(L::bLDFull + st));
          if (kF16)
            bulk_load(sb0 + L::kQInv + st * 16, p.qinv + ((size_t)bh * p.n_tiles + (qrow >> 7)) * 4,
                      16, bar(L::bLDFull + st));
          ++nq;
          did = true;
        }
        if (no < n_it && (no < 2 || mbar_test(bar(L::bDOEmpty + (no & 1)), ((no >> 1) - 1) & 1))) {
          const int so = no & 1, gi = no / n_q, bh = bhq0 + gi;
          const int qrow = (qt0 + no - gi * n_q) * 128;
          const uint32_t ob = sb0 + L::kDO + so * L::kTileBytes;
          if (rank == 0) mbar_arrive_expect_tx(bar(L::bDOFull + so), 2 * L::kTileBytes);
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_3d_pair(ob + cb * L::kRowHalfBlock, &tmOr, lead(L::bDOFull + so), cb * 64,
                             qrow + 64 * (int)rank, bh);
          tma_load_3d_pair(ob + L::kHalfBytes, &tmOc, lead(L::bDOFull + so), 64 * (int)rank, qrow, bh);
          ++no;
          did = true;
        }
        if (did) {
          t_last = clock64();
          continue;
        }
        if (*abort_flag) break;
        if (clock64() - t_last > kWaitLimitCycles) {
          *abort_flag = 1;
          report_status(ATTN_ETIMEOUT);
          break;
        }
        __nanosleep(32);
      }
    }
  } else if (warp == L::kMmaWarp) {
    // ---------------- MMA issuer (the leader's, for the pair) ----------------
    // Fixed order: S(0) dP(0), then per query tile dV(i) S(i+1) dK(i)
    // dP(i+1), each after the wait for what it needs (waits on the leader's
    // barriers, which count both CTAs).
    if (rank == 0 && lane == 0) {
      constexpr uint32_t id_s = idesc_f16(256, 128, !kF16, !kF16, false, false);
      constexpr uint32_t id_dp = idesc_f16(256, 128, true, true, false, false);
      constexpr uint32_t id_dv = idesc_f16(256, D, true, true, false, true);
      constexpr uint32_t id_dk = idesc_f16(256, D, !kF16, !kF16, false, true);
      const uint32_t tS = tmem + L::kColS, tDP = tmem + L::kColDP;
      const uint32_t tDV = tmem + L::kColDV, tDK = tmem + L::kColDK;
      const uint32_t ps = sb0 + L::kPS;
      auto qb = [&](int i) -> uint32_t { return sb0 + L::kQ + (i & 1) * L::kTileBytes; };
      auto ob = [&](int i) -> uint32_t { return sb0 + L::kDO + (i & 1) * L::kTileBytes; };
      auto W = [&](int b1, int ph) { return mbar_wait_cl(bar(b1), ph & 1, abort_flag); };
      auto product_rows = [&](uint32_t d, uint32_t a_tile, uint32_t b_rows, uint32_t idesc) {
        // A: this CTA's 128 rows (K-major); B: the 64-row half (K-major)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_pair(d,
                      smem_desc_sw128(a_tile + (kk >> 2) * L::kBlockBytes + (kk & 3) * 32, 16, 1024),
                      smem_desc_sw128(b_rows + (kk >> 2) * L::kRowHalfBlock + (kk & 3) * 32, 16, 1024),
                      idesc, kk > 0);
      };
      auto product_feat = [&](uint32_t d, uint32_t b_feat, uint32_t idesc, bool first) {
        // A: the P/dS tile (K-major over 128 queries); B: the 64-feature half
        // (MN-major over 128 query rows)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss_pair(d, smem_desc_sw128(ps + (kk >> 2) * L::kBlockBytes + (kk & 3) * 32, 16, 1024),
                      smem_desc_sw128(b_feat + kk * 2048, L::kBlockBytes, 1024), idesc,
                      (!first || kk > 0) ? 1u : 0u);
      };
      auto group_S = [&](int i) -> bool {
        if (!W(L::bQFull + (i & 1), i >> 1) || (i > 0 && !W(L::bSFree, i - 1))) return false;
        tc_fence_after();
        product_rows(tS, sb0 + L::kK, qb(i), id_s);
        commit_pair(bar(L::bSFull));
        return true;
      };
      auto group_dP = [&](int i) -> bool {
        if (!W(L::bDOFull + (i & 1), i >> 1)) return false;
        tc_fence_after();
        product_rows(tDP, sb0 + L::kV, ob(i), id_dp);
        commit_pair(bar(L::bDPFull));
        return true;
      };
      auto group_dV = [&](int i) -> bool {
        if (!W(L::bPFull, i)) return false;
        tc_fence_after();
        product_feat(tDV, ob(i) + L::kHalfBytes, id_dv, i == 0);
        commit_pair(bar(L::bDVDone));
        commit_pair(bar(L::bDOEmpty + (i & 1)));
        return true;
      };
      auto group_dK = [&](int i) -> bool {
        if (!W(L::bDSFull, i)) return false;
        tc_fence_after();
        product_feat(tDK, qb(i) + L::kHalfBytes, id_dk, i == 0);
        commit_pair(bar(L::bQEmpty + (i & 1)));
        commit_pair(bar(L::bDSFree));
        if (i == n_it - 1) commit_pair(bar(L::bFinal));
        return true;
      };
      bool ok = W(L::bKV, 0) && group_S(0) && group_dP(0);
      for (int i = 0; ok && i < n_it; ++i)
        ok = group_dV(i) && (i + 1 == n_it || group_S(i + 1)) && group_dK(i) &&
             (i + 1 == n_it || group_dP(i + 1));
    }
  } else {
    // ---------------- elementwise warps (both CTAs, their own key rows) ----------------
    constexpr int QC = L::kQC, DC = L::kDC;
    const int wg = warp >> 2, sub = warp & 3;
    const int r = sub * 32 + lane;  // TMEM lane: key row
    const int j = j0 + r;
    const int qc0 = QC * wg, dc0 = DC * wg;
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const int de_j = (j < T) ? (p.doc_end ? min(max(p.doc_end[row0 + j] - row0, j + 1), T) : T) : T;
    const uint32_t tS = tmem + lane_base + L::kColS;
    const uint32_t tDP = tmem + lane_base + L::kColDP;
    uint8_t* psb = sg + L::kPS;
    float pf[QC];
    bool ok = true;
    float cscale = 1.f, qinv_i = 1.f;
    auto W = [&](int b1, int ph) { return mbar_wait_cl(bar(b1), ph & 1, abort_flag); };
    // one arrival per warp on the leader's barrier, after every lane's part
    auto warp_arrive_lead = [&](int b1) {
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(b1));
    };
    auto store_row = [&](const uint32_t* w) {
#pragma unroll
      for (int c = 0; c < QC / 32; ++c) {
        const int col = qc0 + 32 * c;
        uint8_t* blk = psb + (col >> 6) * L::kBlockBytes;
        const int ch0 = (col & 63) >> 3;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4*>(blk + sw128(r, ch0 + e)) =
              make_uint4(w[16 * c + 4 * e], w[16 * c + 4 * e + 1], w[16 * c + 4 * e + 2],
                         w[16 * c + 4 * e + 3]);
      }
    };
    // fp16 operands: C of this CTA from the largest qinv over the pair's query
    // tiles and the preprocessing's per-head maxima of |dO_i|, |Delta_i|
    // (this group's query heads) and |v_j| (this key/value head)
    auto make_c = [&]() -> bool {
      float qm = 0.f, dm = 0.f, dl = 0.f;
      for (int e = threadIdx.x; e < n_it; e += L::kEwThreads) {
        const int gi = e / n_q;
        qm = fmaxf(qm, p.qinv[((size_t)(bhq0 + gi) * p.n_tiles + qt0 + (e - gi * n_q)) * 4]);
      }
      for (int g = threadIdx.x; g < G; g += L::kEwThreads) {
        dm = fmaxf(dm, p.hstat[4 * (bhq0 + g)]);
        dl = fmaxf(dl, p.hstat[4 * (bhq0 + g) + 1]);
      }
      qm = warp_max(qm);
      dm = warp_max(dm);
      dl = warp_max(dl);
      if (lane == 0) {
        stats[4 * warp] = qm;
        stats[4 * warp + 1] = dm;
        stats[4 * warp + 2] = dl;
      }
      mbar_arrive(bar(L::bStats));
      if (!mbar_wait(bar(L::bStats), 0, abort_flag)) return false;
      float a = 0.f, c = 0.f, d = 0.f;
#pragma unroll
      for (int w = 0; w < L::kEwWarps; ++w) {
        a = fmaxf(a, stats[4 * w]);
        c = fmaxf(c, stats[4 * w + 1]);
        d = fmaxf(d, stats[4 * w + 2]);
      }
      cscale = ds_scale(a * fmaf(c, p.hstat[4 * bhk + 2], d));
      return true;
    };
    // ---- P^T(i) = exp2(S^T * scale*log2e - lse2), masked, into the P/dS tile ----
    auto phase_P = [&](int i) -> bool {
      const int i0 = (qt0 + i % n_q) * 128;
      const bool need_mask = (i0 + qc0 < j) || (i0 + qc0 + QC - 1 >= de_j);
      const float* sl = reinterpret_cast<const float*>(sg + L::kLD + (i & 1) * 1024);
      if (!W(L::bLDFull + (i & 1), i >> 1) || !W(L::bSFull, i)) return false;
      tc_fence_after();
      uint32_t s[QC];
      tmem_ld32(tS + qc0, s);
      tmem_wait_ld();
      tc_fence_before();
      warp_arrive_lead(L::bSFree);  // the S^T columns may take the next tile
      float scl = p.scale_log2;
      if constexpr (kF16) {
        qinv_i = *reinterpret_cast<const float*>(sg + L::kQInv + (i & 1) * 16);
        scl *= kinv_cta * qinv_i;
      }
      const float2 scl2 = make_float2(scl, scl);
#pragma unroll
      for (int e = 0; e < QC / 2; ++e) {
        const int col = qc0 + 2 * e;
        const float2 nl = reinterpret_cast<const float2*>(sl + col)[0];
        const int i_a = i0 + col;
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])),
                                    scl2, nl);
        float2 pv = (e % 3 == 2) ? exp2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
        if (need_mask) {
          if (i_a < j || i_a >= de_j) pv.x = 0.f;
          if (i_a + 1 < j || i_a + 1 >= de_j) pv.y = 0.f;
        }
        pf[2 * e] = pv.x;
        pf[2 * e + 1] = pv.y;
      }
      // dK(i-1) must be done reading dS^T(i-1) from the tile
      if (i > 0 && !W(L::bDSFree, i - 1)) return false;
      uint32_t w[QC / 2];
#pragma unroll
      for (int e = 0; e < QC / 2; ++e) w[e] = pack_bf16(pf[2 * e], pf[2 * e + 1]);
      store_row(w);
      fence_proxy_async_smem();
      warp_arrive_lead(L::bPFull);
      return true;
    };
    // ---- dS^T(i) = P^T (dP^T - Delta), over P^T once dV(i) ran ----
    auto phase_dS = [&](int i) -> bool {
      const float* sd = reinterpret_cast<const float*>(sg + L::kLD + (i & 1) * 1024) + 128;
      if (!W(L::bDPFull, i)) return false;
      tc_fence_after();
      uint32_t w[QC / 2];
      const float dsm = cscale * qinv_i;
      const float2 dsm2 = make_float2(dsm, dsm);
#pragma unroll
      for (int h = 0; h < QC / 16; ++h) {
        uint32_t dpv[16];
        tmem_ld16(tDP + qc0 + 16 * h, dpv);
        tmem_wait_ld();
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const int e = 8 * h + e2;
          const float2 nd = reinterpret_cast<const float2*>(sd + qc0)[e];
          const float2 dpp = make_float2(__uint_as_float(dpv[2 * e2]), __uint_as_float(dpv[2 * e2 + 1]));
          if constexpr (kF16) {
            const float2 a = __fmul2_rn(make_float2(pf[2 * e], pf[2 * e + 1]),
                                        __fmul2_rn(__fadd2_rn(dpp, nd), dsm2));
            w[e] = pack_half(a.x, a.y);
          } else {
            const float2 a = __fmul2_rn(make_float2(pf[2 * e], pf[2 * e + 1]), __fadd2_rn(dpp, nd));
            w[e] = pack_bf16(a.x, a.y);
          }
        }
      }
      if (!W(L::bDVDone, i)) return false;
      store_row(w);
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive_lead(L::bDSFull);
      return true;
    };
    ok = phase_P(0);
    if constexpr (kF16) ok = make_c() && ok;  // every thread arrives, even after a failed wait
    ok = ok && phase_dS(0);
    for (int it = 1; ok && it < n_it; ++it) ok = phase_P(it) && phase_dS(it);
    // ---- epilogue: dK = R^T (scale * dK_r), dV (this CTA's key rows) ----
    if (ok && W(L::bFinal, 0)) {
      tc_fence_after();
      const int jj = min(j, T - 1);
      const int pos = jj - (p.doc_start ? min(max(p.doc_start[row0 + jj] - row0, 0), jj) : 0);
      const float inv_c = 1.f / cscale;
      if (p.n_split > 1) {
        float* dka = p.dk_acc + ((size_t)bhk * T + jj) * D;
        float* dva = p.dv_acc + ((size_t)bhk * T + jj) * D;
#pragma unroll
        for (int c = 0; c < DC / 32; ++c) {
          const int col = dc0 + 32 * c;
          uint32_t v[32], u[32];
          tmem_ld32(tmem + lane_base + L::kColDK + col, v);
          tmem_ld32(tmem + lane_base + L::kColDV + col, u);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * inv_c);
          if (j < T) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              red_add_v4(dka + col + 4 * e, v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
              red_add_v4(dva + col + 4 * e, u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
            }
          }
        }
      } else {
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
          for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]) * (p.scale * inv_c);
          if (p.rope_cos) rope_pairs<32, D>(f, p.rope_cos, p.rope_sin, pos, col, true);
          if (j < T) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              reinterpret_cast<uint4*>(dkrow + col)[e] =
                  make_uint4(pack_bf16(f[8 * e], f[8 * e + 1]), pack_bf16(f[8 * e + 2], f[8 * e + 3]),
                             pack_bf16(f[8 * e + 4], f[8 * e + 5]), pack_bf16(f[8 * e + 6], f[8 * e + 7]));
          }
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
  }
  // Neither CTA leaves (or frees TMEM) while the other may still signal its
  // barriers or the pair's products may still write its TMEM.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == L::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, L::kTmemCols);
  }
}

}  // namespace bwd2
