// bwd_sm100.cuh -- tensor-core (tcgen05) attention backward, key-tile
// parallel, for bf16 storage.
//
// One CTA owns one 128-key tile of one key/value head; K and V stay in shared
// memory and the dK, dV accumulators stay in TMEM while the query tiles that
// can see these keys stream through (from the diagonal tile to the end of the
// last key's document, for every query head reading this key/value head).
// Per query tile i (keys are TMEM lanes, queries are columns):
//   S^T  = K Q^T           (TMEM)      dP^T = V dO^T        (TMEM)
//   P^T  = exp2(S^T * scale*log2e - lse2_i), masked; written to the shared
//          P/dS tile (bf16, 128-byte swizzle)
//   dV  += P^T dO          (A = P^T, K-major, from shared memory)
//   dS^T = P^T (dP^T - Delta_i), written over P^T in the same tile once dV
//          has read it
//   dQ_i = dS K            (A = the tile read MN-major), into the S^T
//                          columns once S^T of the next tile has been read
//   dK  += dS^T Q          (A = the tile read K-major)
// Because P^T lives in shared memory rather than in the S^T columns, S^T of
// the next query tile is issued as soon as the elementwise warps have read
// S^T of this one into registers, so the tensor pipe computes it while they
// form P. The MMA warp issues the products in one fixed order, each group
// after one wait that has normally completed already (probing readiness
// instead cost more than it saved). At D = 64 (kPT) TMEM has room for P^T and
// dQ_i in columns of their own, and dV reads P^T from TMEM. dQ_i is drained
// by its own warpgroup: read out of TMEM in 32-column chunks, staged through
// a two-buffer shared ring and added to the fp32 dq accumulator in global
// memory by TMA bulk reduce-adds, off the elementwise warps' path.
//
// Warp roles: four elementwise warpgroups; warpgroup g takes query columns [g*kQC, (g+1)*kQC) of S^T and dP^T and
// feature columns [g*kDC, (g+1)*kDC) of dK and dV; thread t of a warpgroup
// owns TMEM lane t (a key row). Then the dQ warpgroup (lane = query row),
// one TMA warp (K and V once, then Q with lse2 and Delta on the same barrier,
// and dO) and one MMA warp, which owns TMEM. dK is scaled and rotated back
// (R^T) in the epilogue; dK and dV leave as bf16 through shared memory (the
// Q stages) and TMA stores, and a key tile inside one document takes its
// RoPE table rows by TMA into stages the last products no longer read. dq is
// finished by a separate kernel once every key tile has added its part.
//
// Operand types. Without RoPE every product reads bf16 (q, k as given, P^T
// and dS^T rounded to bf16). With RoPE (kF16) the scores are recomputed from
// the forward's own operands: the rotated q, k stored as fp16 times a
// power-of-two factor per 128-row tile (the preprocessing writes the same
// values the forward computed), so P matches the forward's lse. The products
// that pair dS with those operands (dK = dS^T Q, dQ = dS K) then need dS in
// fp16 as well, stored as dS * C * qinv_i: qinv_i (the inverse of query tile
// i's factor) cancels that tile's factor in dK, which therefore accumulates
// C dS^T Q over all tiles, and C, a power of two per CTA, keeps every stored
// value below 2^14 (from |dS_ij| <= |dO_i| max_j |v_j| + |Delta_i|). With the
// dQ warpgroup, C = Cg * kinv (kinv: this key tile's inverse factor, Cg one
// power of two per key/value head), so every key tile adds Cg qinv_i dS K to
// query tile i's dQ and the finishing pass divides that out; without it
// (dQ from the query-tile pass), C is this CTA's own. dK is divided by C in
// the epilogue. P^T and dO stay bf16 for dV, and V, dO for dP.
//
// Sources (page, section): ARK README, "Backward pass (AutoGrad)" (attention
// gradients inside training); Forge README, finding 3 (key-tile-parallel dK/dV
// kernels, the dK/dV split and register pressure) and "What this is" (fused
// flash-attention backward). dQ is accumulated by reduce-adds in L2 rather
// than by a separate query-tile pass, which would recompute S and dP (two more
// products per tile). Tiling, TMEM plan and warp roles are this library's own.
#pragma once

#include "sm100.cuh"

namespace bwd100 {

using namespace sm100;

// kDQ: the kernel also forms dQ_i = dS K per query tile and adds it into the
// fp32 accumulator (its own warpgroup and staging ring); without it dQ comes
// from the query-tile pass (dq_sm100.cuh) and the freed shared memory holds a
// second dO stage at D = 128.
template <int D, bool kDQ = true>
struct Layout {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kDOStages = (D == 128 && kDQ) ? 1 : 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTileBytes;
  static constexpr int kQ = kV + kTileBytes;                  // 2 stages
  static constexpr int kDO = kQ + 2 * kTileBytes;             // kDOStages stages
  static constexpr int kPS = kDO + kDOStages * kTileBytes;    // P^T then dS^T: 128 keys x 128 queries bf16
  static constexpr int kLD = kPS + 128 * 128 * 2;             // 2 x {-lse2[128], -delta[128]} f32
  // dQ_i staging ring: two buffers of 128 query rows x 32 fp32 columns, each
  // four 32 x 32 boxes (4 KB, 128-byte swizzle), one per dQ warp.
  static constexpr int kXS = kLD + 2 * 1024;  // 1024-byte aligned (128-byte swizzle)
  static constexpr int kXSBuf = kDQ ? 128 * 32 * 4 : 0;
  // per warp that makes C: largest qinv, |dO_i|, |Delta_i| of this CTA's
  // query tiles and of its key rows' value norms (f32 [16][4]); with the dQ
  // warpgroup, C itself in the last slot
  static constexpr int kStats = kXS + 2 * kXSBuf;
  // per Q stage: the query tile's inverse factor record (16 bytes, qinv first)
  static constexpr int kQInv = kStats + 16 * 4 * 4;
  static constexpr int kBars = kQInv + 2 * 16;
  static constexpr int bKV = 0;
  static constexpr int bQFull = 1, bQEmpty = 3, bDOFull = 5, bDOEmpty = 7;  // 2 each
  static constexpr int bSFull = 9, bSFree = 10, bPFull = 11, bDPFull = 12, bDSFull = 13,
                       bDVDone = 14, bDQFull = 15, bDSFree = 16, bDQFree = 17, bFinal = 18,
                       bStats = 19, bTab = 20;
  static constexpr int kNumBars = 21;
  // RoPE table rows of a key tile that lies in one document, for the dK
  // epilogue: cos into the V tile, sin into the dO stages (both unread once
  // the last dV product is done), 128 rows x D/2 floats each in boxes of
  // 32 floats with the 128-byte swizzle.
  static constexpr int kTabBytes = 128 * (D / 2) * 4;
  static_assert(kTabBytes <= kTileBytes && kTabBytes <= kDOStages * kTileBytes, "table rows fit");
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  // The dynamic shared-memory window starts 1024-byte aligned on sm_100 (after
  // the 1 KB the system reserves per block); the kernel checks this and
  // reports an error instead of running misaligned.
  static constexpr int kSmemAlloc = kBytes;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM columns: S^T (dQ_{i-1} once S^T(i) has been read), dP^T, dV, dK.
  // kPT (D = 64 with the dQ warpgroup, where TMEM has room): P^T (bf16, two
  // queries per column) and dQ have columns of their own instead, so dV reads
  // P^T from TMEM and no product waits for another to free its columns.
  static constexpr bool kPT = kDQ && D == 64;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  static constexpr uint32_t kColP = 256 + 2 * D, kColDQ = kColP + 64;
  static_assert(!kPT || kColDQ + D <= kTmemCols, "P^T and dQ columns fit");
  // Four elementwise warpgroups (16 warps); each owns kQC = 32 query columns
  // of S^T / dP^T and kDC = D/4 feature columns of dK, dV.
  static constexpr int kNWG = 4;
  static constexpr int kQC = 128 / kNWG;
  static constexpr int kDC = D / kNWG;
  static constexpr int kEwThreads = 128 * kNWG;
  static constexpr int kDqWarp0 = 4 * kNWG;  // the dQ warpgroup: warps kDqWarp0 .. +3 (kDQ)
  static constexpr int kProducerWarp = 4 * kNWG + (kDQ ? 4 : 0), kMmaWarp = kProducerWarp + 1;
  static constexpr int kThreads = kEwThreads + (kDQ ? 128 : 0) + 64;
  static_assert(kXS % 1024 == 0, "the dQ staging boxes use the 128-byte swizzle");
  static_assert(kDQ || kThreads == 576, "without dQ: 16 elementwise warps, TMA and MMA warps");
  static_assert(kBytes <= 232448, "more shared memory than a CTA may use");
};

struct Params {
  int T, H, Hkv, BHkv, n_tiles, Tpad;  // H query heads read Hkv key/value heads
  int n_split;  // CTAs sharing one (key/value head, key tile): each takes H/Hkv/n_split query heads
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
  float* dk_acc;           // [B*Hkv][T][D] fp32 (n_split > 1: the parts are added here)
  float* dv_acc;
  // fp16 operands (RoPE): inverse tile factors of the stored q, one 16-byte
  // record per tile ([B*H][n_tiles][4], value first), and of the stored k
  // ([B*Hkv][n_tiles]), and per query head the largest |dO_i| and |Delta_i|
  // ([B*H][4]: dO, Delta, then v of the key/value head of that index)
  const float* qinv;
  const float* kinv;
  float* hstat;  // with the dQ warpgroup, slot 3 of each key/value head receives Cg
};

// The power of two C that keeps every stored dS * C * qinv_i below 2^14,
// from X = max qinv_i * (max |dO_i| * max |v_j| + max |Delta_i|) >= max
// |dS_ij| qinv_i (maxima over this CTA's query tiles, its query heads and its
// key rows); 1 when X is zero (dS is then zero too).
__device__ __forceinline__ float ds_scale(float X) {
  if (!(X > 0.f && X <= 3.0e38f)) return 1.f;
  return ldexpf(1.f, max(-100, min(100, 13 - ilogbf(X))));
}

// Byte offset of 16-byte chunk `ch` (0..7 within a 64-column block) of row r
// in a 128-byte-swizzled tile block.
__device__ __forceinline__ uint32_t sw128(int r, int ch) {
  return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
}

template <int D, bool kF16, bool kDQ>
__global__ void __launch_bounds__(Layout<D, kDQ>::kThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
                const __grid_constant__ CUtensorMap tmDV, const __grid_constant__ CUtensorMap tmRC,
                const __grid_constant__ CUtensorMap tmRS, const Params p) {
  pdl_wait_and_trigger();
  using L = Layout<D, kDQ>;
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
  // query tiles) first. n_split CTAs per (key/value head, key tile); each
  // walks the query tiles of G = H/Hkv/n_split query heads reading that
  // key/value head, head by head: step `it` is query tile qt0 + it % n_q of
  // its it / n_q-th head.
  const int bhk = (int)blockIdx.x % p.BHkv, b = bhk / p.Hkv;
  const int kt = (int)blockIdx.x / (p.BHkv * p.n_split);
  const int part = ((int)blockIdx.x / p.BHkv) % p.n_split;
  const int G = p.H / p.Hkv / p.n_split;
  const int bhq0 = b * p.H + (bhk - b * p.Hkv) * (p.H / p.Hkv) + part * G;  // first query head
  const int j0 = kt * 128;
  const int row0 = b * T;
  const int jlast = min(j0 + 127, T - 1);
  // exclusive; document ranges are clamped into the row wherever they are
  // read (they may come from the caller's saved buffer)
  const int q_end = p.doc_end ? min(max(p.doc_end[row0 + jlast] - row0, jlast + 1), T) : T;
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
    mbar_init(bar(L::bSFree), L::kEwThreads);
    mbar_init(bar(L::bPFull), L::kEwThreads);
    mbar_init(bar(L::bDPFull), 1);
    mbar_init(bar(L::bDSFull), L::kEwThreads);
    mbar_init(bar(L::bDVDone), 1);
    mbar_init(bar(L::bDQFull), 1);
    mbar_init(bar(L::bDSFree), 1);
    mbar_init(bar(L::bDQFree), 128);
    mbar_init(bar(L::bFinal), 1);
    mbar_init(bar(L::bTab), 1);
    // C is made by the dQ warpgroup when there is one (it is idle until the
    // first dQ), else by the elementwise warps
    mbar_init(bar(L::bStats), kDQ ? 128 : L::kEwThreads);
    *abort_flag = 0;
    fence_barrier_init();
    atomicAdd(&g_attn_tiles[1], (unsigned long long)n_it);
  }
  if (warp == L::kMmaWarp) {
    tmem_alloc(sb0 + L::kMisc, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // fp16 operands: this key tile's inverse factor, and C from the posted
  // statistics (every thread that needs it derives the same value)
  const float kinv_cta = kF16 ? p.kinv[(size_t)bhk * p.n_tiles + kt] : 1.f;
  float* stats = reinterpret_cast<float*>(sg + L::kStats);  // [warp][4]
  auto cta_ds_scale = [&]() -> float {
    float qm = 0.f, dm = 0.f, dl = 0.f, vb = 0.f;
#pragma unroll
    for (int g = 0; g < L::kNWG; ++g) {
      float vg = 0.f;
#pragma unroll
      for (int w4 = 0; w4 < 4; ++w4) {
        const float* e = stats + 4 * (4 * g + w4);
        qm = fmaxf(qm, e[0]);
        dm = fmaxf(dm, e[1]);
        dl = fmaxf(dl, e[2]);
        vg = fmaxf(vg, e[3]);
      }
      vb += vg;  // |v_j| <= sum over the column groups of their largest partial norms
    }
    return ds_scale(qm * fmaf(dm, vb, dl));
  };

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
      // Q (with its lse2 / Delta rows) and dO stream independently: each is
      // loaded as soon as its buffer is free, in tile order.
      int nq = 0, no = 0;
      long long t_last = clock64();
      while (nq < n_it || no < n_it) {
        bool did = false;
        if (nq < n_it && (nq < 2 || mbar_test(bar(L::bQEmpty + (nq & 1)), ((nq >> 1) - 1) & 1))) {
          const int st = nq & 1;
          const int gi = nq / n_q;
          const int bh = bhq0 + gi;
          const int qrow = (qt0 + nq - gi * n_q) * 128;
          mbar_arrive_expect_tx(bar(L::bQFull + st), L::kTileBytes + 1024 + (kF16 ? 16 : 0));
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_3d(sb0 + L::kQ + st * L::kTileBytes + cb * L::kBlockBytes, &tmQ,
                        bar(L::bQFull + st), cb * 64, qrow, bh);
          const uint32_t ld = sb0 + L::kLD + st * 1024;
          bulk_load(ld, p.lse2 + (size_t)bh * p.Tpad + qrow, 512, bar(L::bQFull + st));
          bulk_load(ld + 512, p.delta + (size_t)bh * p.Tpad + qrow, 512, bar(L::bQFull + st));
          if (kF16)
            bulk_load(sb0 + L::kQInv + st * 16, p.qinv + ((size_t)bh * p.n_tiles + (qrow >> 7)) * 4,
                      16, bar(L::bQFull + st));
          ++nq;
          did = true;
        }
        if (no < n_it && (no < L::kDOStages ||
                          mbar_test(bar(L::bDOEmpty + no % L::kDOStages),
                                    ((no / L::kDOStages) - 1) & 1))) {
          const int so = no % L::kDOStages;
          const int gi = no / n_q;
          const int qrow = (qt0 + no - gi * n_q) * 128;
          mbar_arrive_expect_tx(bar(L::bDOFull + so), L::kTileBytes);
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_3d(sb0 + L::kDO + so * L::kTileBytes + cb * L::kBlockBytes, &tmDO,
                        bar(L::bDOFull + so), cb * 64, qrow, bhq0 + gi);
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
    // ---------------- MMA issuer ----------------
    // Five groups per query tile i: S(i), dP(i), dV(i), dK(i), dQ(i). TMEM:
    // S^T(i) and then dQ(i-1) share the S^T columns, dP^T has its own.
    // With dQ formed here the issuer follows one fixed order, S(0) dP(0),
    // then per tile dV(i) S(i+1) dK(i) dQ(i) dP(i+1), each group after a
    // blocking wait for what it needs. That wait is normally complete already
    // and its answer then arrives while the previous group's products are
    // still queued on the tensor pipe; probing several groups for readiness
    // instead costs the probes' answer time before every issue, with the pipe
    // draining meanwhile (measured at 8K: 767 against 886 us). Without dQ
    // the issuer takes whichever group is ready, probing in the priority dV,
    // S, dK, dP. Readiness:
    //   S(i):  Q(i) loaded; the S^T columns free: S(0) always, S(1) once the
    //          elementwise warps have read S(0), S(i >= 2) once dQ(i-2) has
    //          been read out
    //   dP(i): dO(i) loaded; dS^T(i-1) formed (so dP^T(i-1) has been read)
    //   dV(i): P^T(i) in the P/dS tile; dP(i) issued (dO(i) is loaded and the
    //          commit after dV(i) covers both readers of dO(i))
    //   dK(i): dS^T(i) in the tile
    //   dQ(i): dK(i) issued; the elementwise warps have read S(i+1) (or i is
    //          the last tile). The tile is free again after dQ(i).
    // Every barrier probed for phase k has been seen complete for phase k-1,
    // so the parity probes are unambiguous.
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16(128, 128, !kF16, !kF16, false, false);
      constexpr uint32_t id_dp = idesc_f16(128, 128, true, true, false, false);
      constexpr uint32_t id_dv = idesc_f16(128, D, true, true, false, true);
      constexpr uint32_t id_dk = idesc_f16(128, D, !kF16, !kF16, false, true);
      constexpr uint32_t id_dq = idesc_f16(128, D, !kF16, !kF16, true, true);
      const uint32_t tS = tmem + L::kColS, tDP = tmem + L::kColDP;
      const uint32_t tDV = tmem + L::kColDV, tDK = tmem + L::kColDK;
      const uint32_t ps = sb0 + L::kPS;
      auto qbuf = [&](int i) -> uint32_t { return sb0 + L::kQ + (i & 1) * L::kTileBytes; };
      auto obuf = [&](int i) -> uint32_t {
        return sb0 + L::kDO + (i % L::kDOStages) * L::kTileBytes;
      };
      int nS = 0, nP = 0, nV = 0, nK = 0, nQ = 0;  // next tile of each group
      bool ok = mbar_wait(bar(L::bKV), 0, abort_flag);
      if constexpr (kDQ) {
        // Every barrier is waited on for its phases in order, and its next
        // phase needs a group issued after the wait, so the parity is exact.
        auto wait1 = [&](int b1, int ph1) { return mbar_wait(bar(b1), ph1 & 1, abort_flag); };
        auto wait2 = [&](int b1, int ph1, int b2, int ph2) {
          return mbar_wait2(bar(b1), ph1 & 1, bar(b2), ph2 & 1, abort_flag);
        };
        auto group_S = [&](int i) -> bool {
          // kPT: S(i-1) has been read (P(i-1) formed, which dV(i-1) waited for)
          const bool r = (i == 0 || L::kPT) ? wait1(L::bQFull + (i & 1), i >> 1)
                         : i == 1 ? wait2(L::bQFull + 1, 0, L::bSFree, 0)
                                  : wait2(L::bQFull + (i & 1), i >> 1, L::bDQFree, i - 2);
          if (!r) return false;
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
        auto group_dP = [&](int i) -> bool {
          if (!wait1(L::bDOFull + i % L::kDOStages, i / L::kDOStages)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBlockBytes + (kk & 3) * 32;
            mma_ss(tDP, smem_desc_sw128(sb0 + L::kV + off, 16, 1024),
                   smem_desc_sw128(obuf(i) + off, 16, 1024), id_dp, kk > 0);
          }
          mma_commit(bar(L::bDPFull));
          return true;
        };
        auto group_dV = [&](int i) -> bool {
          if (!wait1(L::bPFull, i)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t db = smem_desc_sw128(obuf(i) + kk * 2048, L::kBlockBytes, 1024);
            const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
            if constexpr (L::kPT)  // A = P^T from TMEM, 8 columns per K step
              mma_ts(tDV, tmem + L::kColP + 8 * kk, db, id_dv, acc);
            else
              mma_ss(tDV,
                     smem_desc_sw128(ps + (kk >> 2) * L::kBlockBytes + (kk & 3) * 32, 16, 1024),
                     db, id_dv, acc);
          }
          mma_commit(bar(L::bDVDone));
          mma_commit(bar(L::bDOEmpty + i % L::kDOStages));
          return true;
        };
        auto group_dK = [&](int i) -> bool {
          if (!wait1(L::bDSFull, i)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tDK, smem_desc_sw128(ps + (kk >> 2) * L::kBlockBytes + (kk & 3) * 32, 16, 1024),
                   smem_desc_sw128(qbuf(i) + kk * 2048, L::kBlockBytes, 1024), id_dk,
                   (i > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::bQEmpty + (i & 1)));
          if (i == n_it - 1) mma_commit(bar(L::bFinal));
          return true;
        };
        auto group_dQ = [&](int i) -> bool {
          // into the S^T columns once the elementwise warps have read S(i+1);
          // kPT: into its own columns once the dQ warps have read dQ(i-1) out
          if (L::kPT ? (i > 0 && !wait1(L::bDQFree, i - 1))
                     : (i < n_it - 1 && !wait1(L::bSFree, i + 1)))
            return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(L::kPT ? tmem + L::kColDQ : tS, smem_desc_sw128(ps + kk * 2048, L::kBlockBytes, 1024),
                   smem_desc_sw128(sb0 + L::kK + kk * 2048, L::kBlockBytes, 1024), id_dq, kk > 0);
          mma_commit(bar(L::bDQFull));
          mma_commit(bar(L::bDSFree));  // the P/dS tile is free again (dK(i) is covered too)
          return true;
        };
        ok = ok && group_S(0) && group_dP(0);
        for (int i = 0; ok && i < n_it; ++i)
          ok = group_dV(i) && (i + 1 == n_it || group_S(i + 1)) && group_dK(i) && group_dQ(i) &&
               (i + 1 == n_it || group_dP(i + 1));
      }
      long long t_last = clock64();
      while (!kDQ && ok && nK < n_it) {
        if (nV < nP && mbar_test(bar(L::bPFull), nV & 1)) {
          // dV += P^T dO (P^T K-major in the P/dS tile, dO MN-major)
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tDV, smem_desc_sw128(ps + (kk >> 2) * L::kBlockBytes + (kk & 3) * 32, 16, 1024),
                   smem_desc_sw128(obuf(nV) + kk * 2048, L::kBlockBytes, 1024), id_dv,
                   (nV > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::bDVDone));
          mma_commit(bar(L::bDOEmpty + nV % L::kDOStages));
          ++nV;
        } else if (nS < n_it && mbar_test(bar(L::bQFull + (nS & 1)), (nS >> 1) & 1) &&
                   (nS == 0 ||
                    (kDQ ? (nS == 1 ? mbar_test(bar(L::bSFree), 0)
                                    : (nQ > nS - 2 && mbar_test(bar(L::bDQFree), nS & 1)))
                         : mbar_test(bar(L::bSFree), (nS - 1) & 1)))) {
          // S^T(i) = K Q(i)^T
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBlockBytes + (kk & 3) * 32;
            mma_ss(tS, smem_desc_sw128(sb0 + L::kK + off, 16, 1024),
                   smem_desc_sw128(qbuf(nS) + off, 16, 1024), id_s, kk > 0);
          }
          mma_commit(bar(L::bSFull));
          ++nS;
        } else if (nK < nV && mbar_test(bar(L::bDSFull), nK & 1)) {
          // dK += dS^T Q (dS^T K-major)
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tDK, smem_desc_sw128(ps + (kk >> 2) * L::kBlockBytes + (kk & 3) * 32, 16, 1024),
                   smem_desc_sw128(qbuf(nK) + kk * 2048, L::kBlockBytes, 1024), id_dk,
                   (nK > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::bQEmpty + (nK & 1)));
          if (!kDQ) mma_commit(bar(L::bDSFree));  // the P/dS tile is free again
          if (nK == n_it - 1) mma_commit(bar(L::bFinal));
          ++nK;
        } else if (kDQ && nQ < nK && (nQ == n_it - 1 ||
                               (nS > nQ + 1 && mbar_test(bar(L::bSFree), (nQ + 1) & 1)))) {
          // dQ_i = dS K (dS read MN-major), into the S^T columns
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tS, smem_desc_sw128(ps + kk * 2048, L::kBlockBytes, 1024),
                   smem_desc_sw128(sb0 + L::kK + kk * 2048, L::kBlockBytes, 1024), id_dq, kk > 0);
          mma_commit(bar(L::bDQFull));
          mma_commit(bar(L::bDSFree));
          ++nQ;
        } else if (nP < n_it && nP <= nK &&
                   mbar_test(bar(L::bDOFull + nP % L::kDOStages), (nP / L::kDOStages) & 1)) {
          // dP^T(i) = V dO(i)^T
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBlockBytes + (kk & 3) * 32;
            mma_ss(tDP, smem_desc_sw128(sb0 + L::kV + off, 16, 1024),
                   smem_desc_sw128(obuf(nP) + off, 16, 1024), id_dp, kk > 0);
          }
          mma_commit(bar(L::bDPFull));
          ++nP;
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
  } else if (kDQ && warp >= L::kDqWarp0) {
    // ---------------- dQ warpgroup (lane = query row) ----------------
    // Per query tile: read dQ_i out of the S^T columns in 32-column chunks
    // (releasing the columns after the last read), stage each chunk as this
    // warp's 32 x 32 box in the next ring buffer and reduce-add it into the
    // accumulator. A buffer is rewritten only after the reduce that last used
    // it (two chunks back) has read it.
    const int sub = warp & 3;
    const uint32_t tq = tmem + ((uint32_t)(sub * 32) << 16) + (L::kPT ? L::kColDQ : L::kColS);
    constexpr int NCH = D / 32;
    int chunk = 0;
    bool prev_issued = false;  // did this warp reduce the previous chunk
    float cscale = 1.f;
    bool okq = true;
    if constexpr (kF16) {
      // C for this CTA, made here. Every CTA that adds into a query head's
      // dQ accumulator must carry the same factor per query tile, so C is
      // Cg * kinv (this key tile's inverse factor, which then cancels in dQ),
      // with Cg one power of two per key/value head: from the largest qinv
      // and kinv over all of that head's tiles, |dO_i| and |Delta_i| over its
      // query heads and |v_j| over its keys (the preprocessing's per-head
      // maxima). dQ then accumulates Cg qinv_i dS K for query tile i, which
      // the finishing pass divides out; Cg is left in the head's fourth
      // statistics slot for it. Published to the elementwise warps in the
      // last statistics slot.
      const int tq = threadIdx.x - 32 * L::kDqWarp0;  // 0..127
      const int Gf = p.H / p.Hkv;
      const int bhq_first = b * p.H + (bhk - b * p.Hkv) * Gf;  // the group's query heads follow
      float qm = 0.f, km = 0.f, dm = 0.f, dl = 0.f;
      for (int e = tq; e < Gf * p.n_tiles; e += 128)
        qm = fmaxf(qm, p.qinv[((size_t)bhq_first * p.n_tiles + e) * 4]);
      for (int e = tq; e < p.n_tiles; e += 128) km = fmaxf(km, p.kinv[(size_t)bhk * p.n_tiles + e]);
      for (int g = tq; g < Gf; g += 128) {
        dm = fmaxf(dm, p.hstat[4 * (bhq_first + g)]);
        dl = fmaxf(dl, p.hstat[4 * (bhq_first + g) + 1]);
      }
      qm = warp_max(qm);
      km = warp_max(km);
      dm = warp_max(dm);
      dl = warp_max(dl);
      if (lane == 0) {
        float* e = stats + 4 * sub;
        e[0] = qm;
        e[1] = km;
        e[2] = dm;
        e[3] = dl;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the four dQ warps, none exits early
#pragma unroll
      for (int w4 = 0; w4 < 4; ++w4) {
        qm = fmaxf(qm, stats[4 * w4]);
        km = fmaxf(km, stats[4 * w4 + 1]);
        dm = fmaxf(dm, stats[4 * w4 + 2]);
        dl = fmaxf(dl, stats[4 * w4 + 3]);
      }
      const float cg = ds_scale(qm * km * fmaf(dm, p.hstat[4 * bhk + 2], dl));
      cscale = cg * kinv_cta;
      if (tq == 0) {
        stats[63] = cscale;
        if (kt == 0 && part == 0) p.hstat[4 * bhk + 3] = cg;
      }
      mbar_arrive(bar(L::bStats));
    }
    for (int it = 0; okq && it < n_it; ++it) {
      const int gi = it / n_q;
      const int i0 = (qt0 + it - gi * n_q) * 128;
      const bool rows_in = i0 + 32 * sub < T;  // rows past T are clipped by the map
      if (!mbar_wait(bar(L::bDQFull), it & 1, abort_flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < NCH; ++c, ++chunk) {
        uint32_t v[32];
        tmem_ld32(tq + 32 * c, v);
        tmem_wait_ld();
        if (c == NCH - 1) {
          tc_fence_before();
          mbar_arrive(bar(L::bDQFree));
        }
        const int buf = chunk & 1;
        if (lane == 0) {
          if (prev_issued) bulk_wait_group_read1();
          else bulk_wait_group_read0();
        }
        __syncwarp();
        uint8_t* bx = sg + L::kXS + buf * L::kXSBuf + sub * 4096;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<uint4*>(bx + sw128(lane, e)) =
              make_uint4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && rows_in) {
          tma_reduce_add_3d(&tmDQ, sb0 + L::kXS + buf * L::kXSBuf + sub * 4096, 32 * c,
                            i0 + 32 * sub, bhq0 + gi);
          bulk_commit_group();
        }
        prev_issued = rows_in;
      }
    }
    // before the CTA leaves, the staging ring must have been read; the adds
    // themselves complete with the grid, before any later kernel reads dq
    if (lane == 0) bulk_wait_group_read0();
  } else {
    // ---------------- elementwise warps ----------------
    constexpr int QC = L::kQC, DC = L::kDC;
    const int wg = warp >> 2, sub = warp & 3;
    const int r = sub * 32 + lane;  // TMEM lane: key row of S^T, dP^T, dK, dV
    const int j = j0 + r;
    const int qc0 = QC * wg;        // query columns of S^T / dP^T handled here
    const int dc0 = DC * wg;        // feature columns of dK / dV handled here
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const int de_j = (j < T) ? (p.doc_end ? min(max(p.doc_end[row0 + j] - row0, j + 1), T) : T) : T;
    const uint32_t tS = tmem + lane_base + L::kColS;
    const uint32_t tDP = tmem + lane_base + L::kColDP;
    uint8_t* psb = sg + L::kPS;
    float pf[QC];  // P^T of this thread's key row, query columns [qc0, qc0 + QC)
    bool ok = true;
    float cscale = 1.f;  // C (fp16 operands)
    float qinv_i = 1.f;  // inverse factor of the current query tile (fp16 operands)
    // fp16 operands: this warp's share of the statistics C is made from (the
    // largest qinv over this CTA's query tiles, |dO_i| and |Delta_i| over its
    // query heads, and the largest norm of this warpgroup's columns of the
    // value rows) is posted after the first P tile (C is needed from the
    // first dS tile on); the per-tile values are prefetched into L1 here.
    auto stat_index = [&](int e) -> size_t {
      const int gi = e / n_q;
      return (size_t)(bhq0 + gi) * p.n_tiles + qt0 + (e - gi * n_q);
    };
    if constexpr (kF16 && !kDQ) {
      for (int e = threadIdx.x; e < n_it; e += L::kEwThreads)
        asm volatile("prefetch.global.L1 [%0];" ::"l"(p.qinv + stat_index(e) * 4));
    }
    auto post_stats = [&]() -> bool {
      float qm = 0.f, dm = 0.f, dl = 0.f;
      for (int e = threadIdx.x; e < n_it; e += L::kEwThreads) qm = fmaxf(qm, p.qinv[stat_index(e) * 4]);
      for (int g = threadIdx.x; g < G; g += L::kEwThreads) {
        dm = fmaxf(dm, p.hstat[4 * (bhq0 + g)]);
        dl = fmaxf(dl, p.hstat[4 * (bhq0 + g) + 1]);
      }
      float vn = 0.f;
      bool okv = mbar_wait(bar(L::bKV), 0, abort_flag);
      if (okv) {
        const uint8_t* vb = sg + L::kV + (dc0 >> 6) * L::kBlockBytes;
#pragma unroll
        for (int e = 0; e < DC / 8; ++e) {
          const uint4 raw = *reinterpret_cast<const uint4*>(vb + sw128(r, ((dc0 & 63) >> 3) + e));
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int q2 = 0; q2 < 4; ++q2) {
            const float a = __low2float(h[q2]), b2 = __high2float(h[q2]);
            vn = fmaf(a, a, fmaf(b2, b2, vn));
          }
        }
        vn = sqrtf(vn);
      }
      qm = warp_max(qm);
      dm = warp_max(dm);
      dl = warp_max(dl);
      vn = warp_max(vn);
      if (lane == 0) {
        float* e = stats + 4 * warp;
        e[0] = qm;
        e[1] = dm;
        e[2] = dl;
        e[3] = vn;
      }
      mbar_arrive(bar(L::bStats));
      okv = okv && mbar_wait(bar(L::bStats), 0, abort_flag);
      if (okv) cscale = cta_ds_scale();
      return okv;
    };
    // Row r, query columns [qc0, qc0 + QC) of the P/dS tile (bf16 pairs in
    // w[]): 64-column block col/64, 16-byte chunks (col%64)/8 onwards.
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
    // ---- P^T(i) = exp2(S^T scale log2e - lse2), masked; bf16 into the tile ----
    auto phase_P = [&](int i) -> bool {
      const int i0 = (qt0 + i % n_q) * 128;
      const bool need_mask = (i0 + qc0 < j) || (i0 + qc0 + QC - 1 >= de_j);
      const float* sl = reinterpret_cast<const float*>(sg + L::kLD + (i & 1) * 1024);
      if (!mbar_wait2(bar(L::bQFull + (i & 1)), (i >> 1) & 1, bar(L::bSFull), i & 1, abort_flag))
        return false;
      tc_fence_after();
      uint32_t s[QC];
#pragma unroll
      for (int c = 0; c < QC / 32; ++c) tmem_ld32(tS + qc0 + 32 * c, s + 32 * c);
      tmem_wait_ld();
      tc_fence_before();
      if constexpr (!L::kPT) mbar_arrive(bar(L::bSFree));  // the S^T columns may take the next tile
      // asked now, answered by the time P is formed (see the wait below):
      // kPT, dV(i-1) done reading P^T(i-1) from TMEM; else dQ(i-1) and
      // dK(i-1) done reading dS^T(i-1) from the tile
      const bool p_free = i == 0 || (L::kPT ? mbar_test(bar(L::bDVDone), (i - 1) & 1)
                                            : mbar_test(bar(L::bDSFree), (i - 1) & 1));
      float scl = p.scale_log2;
      if constexpr (kF16) {
        // loaded with this tile's lse2 and Delta rows
        qinv_i = *reinterpret_cast<const float*>(sg + L::kQInv + (i & 1) * 16);
        scl *= kinv_cta * qinv_i;  // the stored operands carry the tile factors
      }
      const float2 scl2 = make_float2(scl, scl);
#pragma unroll
      for (int e = 0; e < QC / 2; ++e) {
        const int col = qc0 + 2 * e;
        const float2 nl = reinterpret_cast<const float2*>(sl + col)[0];  // -lse2 pair
        const int i_a = i0 + col;
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * e]),
                                                __uint_as_float(s[2 * e + 1])),
                                    scl2, nl);
        // kPolyPairs of the QC/2 pairs go to the FMA pipe (measured: at
        // D = 128 every pair on MUFU is fastest, 2.5 % on the 8K kernel, since
        // dS and the products' epilogue keep the FMA pipe busy; at D = 64 five
        // pairs of sixteen)
        constexpr int kPolyPairs = D == 128 ? 0 : 5;
        const bool poly = (e * kPolyPairs) / (QC / 2) != ((e + 1) * kPolyPairs) / (QC / 2);
        float2 pv = poly ? exp2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
        if (need_mask) {
          if (i_a < j || i_a >= de_j) pv.x = 0.f;
          if (i_a + 1 < j || i_a + 1 >= de_j) pv.y = 0.f;
        }
        pf[2 * e] = pv.x;
        pf[2 * e + 1] = pv.y;
      }
      if (!p_free && !mbar_wait(bar(L::kPT ? L::bDVDone : L::bDSFree), (i - 1) & 1, abort_flag))
        return false;
      uint32_t w[QC / 2];
#pragma unroll
      for (int e = 0; e < QC / 2; ++e) w[e] = pack_bf16(pf[2 * e], pf[2 * e + 1]);
      if constexpr (L::kPT) {
        // this thread's 32 query columns as 16 packed columns of P^T
        tc_fence_after();
        tmem_st16(tmem + lane_base + L::kColP + (qc0 >> 1), w);
        tmem_wait_st();
        tc_fence_before();
      } else {
        store_row(w);
        fence_proxy_async_smem();
      }
      mbar_arrive(bar(L::bPFull));
      return true;
    };
    // ---- dS^T(i) = P^T (dP^T - Delta), over P^T in the tile once dV(i) ran ----
    auto phase_dS = [&](int i) -> bool {
      const float* sd = reinterpret_cast<const float*>(sg + L::kLD + (i & 1) * 1024) + 128;
      if (!mbar_wait(bar(L::bDPFull), i & 1, abort_flag)) return false;
      tc_fence_after();
      // 16 columns of dP^T at a time: fewer registers live next to P
      uint32_t w[QC / 2];
      bool dv_done = false;
      const float dsm = cscale * qinv_i;  // 1 for bf16 operands
      const float2 dsm2 = make_float2(dsm, dsm);
#pragma unroll
      for (int h = 0; h < QC / 16; ++h) {
        uint32_t dpv[16];
        tmem_ld16(tDP + qc0 + 16 * h, dpv);
        tmem_wait_ld();
        if (h == 0)  // answered by the store below
          dv_done = L::kPT ? (i == 0 || mbar_test(bar(L::bDSFree), (i - 1) & 1))
                           : mbar_test(bar(L::bDVDone), i & 1);
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const int e = 8 * h + e2;
          const float2 nd = reinterpret_cast<const float2*>(sd + qc0)[e];  // -Delta pair
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
      // the tile must be free: dV(i) done reading P^T(i) from it, or (kPT, P^T
      // in TMEM) dK(i-1) and dQ(i-1) done reading dS^T(i-1)
      if (!dv_done && !(L::kPT ? mbar_wait(bar(L::bDSFree), (i - 1) & 1, abort_flag)
                               : mbar_wait(bar(L::bDVDone), i & 1, abort_flag)))
        return false;
      store_row(w);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(L::bDSFull));
      return true;
    };
    // the first tile is peeled: C is made (without the dQ warpgroup) or picked
    // up (with it) between its P and dS
    ok = phase_P(0);
    if constexpr (kF16) {
      if constexpr (kDQ) {
        ok = ok && mbar_wait(bar(L::bStats), 0, abort_flag);
        if (ok) cscale = stats[63];
      } else {
        ok = post_stats() && ok;  // every thread arrives, even after a failed wait
      }
    }
    ok = ok && phase_dS(0);
    for (int it = 1; ok && it < n_it; ++it) ok = phase_P(it) && phase_dS(it);
    // ---- epilogue: dK = R^T (scale * dK_r), dV ----
    // Once dV of the last tile is done, V, the dO stages and the Q stage that
    // does not hold the last Q tile are unread (dK and dQ of the last tile
    // may still run): the RoPE table rows come in and dV is staged then.
    const bool dv_fin = ok && mbar_wait(bar(L::bDVDone), (n_it - 1) & 1, abort_flag);
    const uint32_t off_dv = L::kQ + (n_it & 1) * L::kTileBytes;        // free from here on
    const uint32_t off_dk = L::kQ + ((n_it - 1) & 1) * L::kTileBytes;  // free after the last dK
    // one document over the whole key tile (uniform across the CTA): its
    // table rows are consecutive from pos0
    const int jl = min(j0 + 127, T - 1);
    const int ds0 = p.doc_start ? min(max(p.doc_start[row0 + j0] - row0, 0), j0) : 0;
    const bool tab_tma = p.rope_cos != nullptr && p.n_split <= 1 &&
                         (!p.doc_start || min(max(p.doc_start[row0 + jl] - row0, 0), jl) == ds0);
    constexpr int HC = 16;  // columns per TMEM load in the staged epilogue
    static_assert(DC % HC == 0, "16-column pieces");
    if (tab_tma && warp == 0 && lane == 0 && dv_fin) {
      mbar_arrive_expect_tx(bar(L::bTab), 2 * L::kTabBytes);
#pragma unroll
      for (int bx = 0; bx < D / 64; ++bx) {
        tma_load_3d(sb0 + L::kV + bx * (128 * 128), &tmRC, bar(L::bTab), 32 * bx, j0 - ds0, 0);
        tma_load_3d(sb0 + L::kDO + bx * (128 * 128), &tmRS, bar(L::bTab), 32 * bx, j0 - ds0, 0);
      }
    }
    if (dv_fin && p.n_split <= 1) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < DC / HC; ++c) {
        const int col = dc0 + HC * c;
        uint32_t v[HC];
        tmem_ld16(tmem + lane_base + L::kColDV + col, v);
        tmem_wait_ld();
        uint8_t* blk = sg + off_dv + (col >> 6) * L::kBlockBytes;
#pragma unroll
        for (int e = 0; e < HC / 8; ++e)
          *reinterpret_cast<uint4*>(blk + sw128(r, ((col & 63) >> 3) + e)) = make_uint4(
              pack_bf16(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
              pack_bf16(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
              pack_bf16(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
              pack_bf16(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
      }
    }
    const bool epi = dv_fin && mbar_wait(bar(L::bFinal), 0, abort_flag);
    if (epi) {
      tc_fence_after();
      const int jj = min(j, T - 1);
      const int pos = jj - (p.doc_start ? min(max(p.doc_start[row0 + jj] - row0, 0), jj) : 0);
      constexpr int CW = DC < 32 ? DC : 32;  // columns per TMEM load
      auto ld = [&](uint32_t taddr, uint32_t* v) {
        if constexpr (CW == 32) tmem_ld32(taddr, v);
        else tmem_ld16(taddr, v);
      };
      const float inv_c = 1.f / cscale;  // dK accumulated C dS^T Q (exact power of two)
      if (p.n_split > 1) {
        // this CTA's part of dK_r and dV: added into the fp32 accumulators
        // (scale and R^T are applied by the finishing pass)
        float* dka = p.dk_acc + ((size_t)bhk * T + jj) * D;
        float* dva = p.dv_acc + ((size_t)bhk * T + jj) * D;
#pragma unroll
        for (int c = 0; c < DC / CW; ++c) {
          const int col = dc0 + CW * c;
          uint32_t v[CW], u[CW];
          ld(tmem + lane_base + L::kColDK + col, v);
          ld(tmem + lane_base + L::kColDV + col, u);
          tmem_wait_ld();
          if constexpr (kF16) {
#pragma unroll
            for (int e = 0; e < CW; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * inv_c);
          }
          if (j < T) {
#pragma unroll
            for (int e = 0; e < CW / 4; ++e) {
              red_add_v4(dka + col + 4 * e, v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
              red_add_v4(dva + col + 4 * e, u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
            }
          }
        }
      } else {
      // dK and dV leave as bf16 through the two Q stages and TMA stores: one
      // 16-byte chunk per lane and key row into the maps' 128-byte swizzle,
      // where stores to global memory from one key row per lane took 32
      // cache lines per instruction and, with the RoPE table loads, held up
      // the dQ warps' last drain on the shared load/store path. A key tile
      // in one document reads consecutive table rows, which came in by TMA
      // while dV was staged (other tiles load this row's entries directly).
      // 16 columns per TMEM load keep the table entries and the accumulator
      // values within the register budget.
      float4 rcos[DC / 8], rsin[DC / 8];
      if (p.rope_cos && !tab_tma) {
        const float4* c4 = reinterpret_cast<const float4*>(p.rope_cos + (size_t)pos * (D / 2) + (dc0 >> 1));
        const float4* s4 = reinterpret_cast<const float4*>(p.rope_sin + (size_t)pos * (D / 2) + (dc0 >> 1));
#pragma unroll
        for (int q = 0; q < DC / 8; ++q) {
          rcos[q] = c4[q];
          rsin[q] = s4[q];
        }
      }
      if (tab_tma) {
        // this row's entries from the swizzled table boxes (4 floats per
        // 16-byte chunk, 32 per 128-byte box row); a wait that gives up has
        // raised the abort flag, and the results are not used then
        mbar_wait(bar(L::bTab), 0, abort_flag);
#pragma unroll
        for (int q = 0; q < DC / 8; ++q) {
          const int fc = (dc0 >> 1) + 4 * q;  // first float of the chunk
          const uint32_t off = (uint32_t)((fc >> 5) * (128 * 128)) + sw128(r, (fc & 31) >> 2);
          rcos[q] = *reinterpret_cast<const float4*>(sg + L::kV + off);
          rsin[q] = *reinterpret_cast<const float4*>(sg + L::kDO + off);
        }
      }
#pragma unroll
      for (int c = 0; c < DC / HC; ++c) {
        const int col = dc0 + HC * c;
        uint32_t v[HC];
        tmem_ld16(tmem + lane_base + L::kColDK + col, v);
        tmem_wait_ld();
        float f[HC];
#pragma unroll
        for (int e = 0; e < HC; ++e) f[e] = __uint_as_float(v[e]) * (p.scale * inv_c);
        if (p.rope_cos) {
          // inverse rotation, the same roundings as rope_pairs
#pragma unroll
          for (int q = 0; q < HC / 8; ++q) {
            const float4 cq = rcos[c * (HC / 8) + q], sq = rsin[c * (HC / 8) + q];
            const float cs[4] = {cq.x, cq.y, cq.z, cq.w};
            const float sn[4] = {-sq.x, -sq.y, -sq.z, -sq.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = f[8 * q + 2 * e], x1 = f[8 * q + 2 * e + 1];
              f[8 * q + 2 * e] = fmaf(x0, cs[e], -__fmul_rn(x1, sn[e]));
              f[8 * q + 2 * e + 1] = fmaf(x0, sn[e], __fmul_rn(x1, cs[e]));
            }
          }
        }
        uint8_t* blk = sg + off_dk + (col >> 6) * L::kBlockBytes;
#pragma unroll
        for (int e = 0; e < HC / 8; ++e)
          *reinterpret_cast<uint4*>(blk + sw128(r, ((col & 63) >> 3) + e)) =
              make_uint4(pack_bf16(f[8 * e], f[8 * e + 1]), pack_bf16(f[8 * e + 2], f[8 * e + 3]),
                         pack_bf16(f[8 * e + 4], f[8 * e + 5]), pack_bf16(f[8 * e + 6], f[8 * e + 7]));
      }
      fence_proxy_async_smem();
      }
    }
    if (p.n_split <= 1) {
      // every elementwise thread arrives (an aborted one too, so none waits
      // for ever); the staged rows then leave in 64-column boxes, rows past
      // T clipped by the maps. Before the CTA leaves its boxes must have
      // been read; the writes complete with the grid.
      asm volatile("barrier.sync 2, %0;" ::"n"(L::kEwThreads) : "memory");
      if (warp == 0 && lane == 0 && epi) {
#pragma unroll
        for (int bcol = 0; bcol < D / 64; ++bcol) {
          tma_store_3d(&tmDK, sb0 + off_dk + bcol * L::kBlockBytes, 64 * bcol, j0, bhk);
          tma_store_3d(&tmDV, sb0 + off_dv + bcol * L::kBlockBytes, 64 * bcol, j0, bhk);
        }
        bulk_commit_group();
        bulk_wait_group_read0();
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
