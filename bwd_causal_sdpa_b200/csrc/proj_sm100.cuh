// proj_sm100.cuh -- tensor-core (tcgen05) GEMM for the projections around the
// attention: C[M][N] = sum_k A[m][k] B[n][k], bf16 operands, fp32 accumulate.
//
// The three products of a linear layer (Forge README, "Benchmarks": forward
// X W^T, backward dX = dY W and dW = dY^T X) and the layer around the
// attention (ARK README, "Inference architecture (EKO)" and "Backward pass
// (AutoGrad)": q, k, v and output projections with the weight gradients dwq,
// dwk, dwv, dwo; Forge README, "Architecture": attention with GQA and RoPE on
// interleaved pairs) all map onto this one kernel:
//   * an operand is read either from a plain row-major matrix or from up to
//     three [B*heads][T][D] head-major tensors (q, k, v: a feature index
//     runs over q's heads, then k's, then v's, D features each), and either
//     K-major (K contiguous) or MN-major (M or N contiguous); TMA moves it
//     into 128-byte-swizzled shared tiles, so no transpose is ever written;
//   * the epilogue writes bf16 rows, fp32 rows (added with reductions when K
//     is split over several CTAs), or scatters the columns into the
//     head-major q, k, v tensors, rotating q and k by RoPE on the way.
// Persistent: each CTA (at most one per SM) walks a strided list of work
// units, a unit being one 128 x 128 output tile over one share of K. 256-wide
// tiles run on clusters of two CTAs instead: a unit is a 256 x 256 tile, each
// CTA loads its 128 rows of A and half of the B tile, and CTA 0 issues
// products of M = 256 (cta_group::2) that read both CTAs' tiles and write
// both CTAs' accumulators. K moves through a three-stage ring of 128-wide
// stages (two K blocks of 64) that runs across units; the accumulator alternates
// between two TMEM buffers, so the epilogue of one unit overlaps the main
// loop of the next. Warps: TMA, MMA (one elected thread issues tcgen05.mma)
// and four epilogue warps (thread = TMEM lane = output row).
#pragma once

#include "common.cuh"
#include "prep.cuh"
#include "sm100.cuh"

namespace proj100 {

using namespace sm100;

constexpr int kBM = 128, kBK = 64;  // kBK: the K block of the unit split

// kPair: the CTA is one of a cluster of two that computes a 256 x BN tile
// (this CTA's 128 rows), loading only its half of every B tile (BN / 2 rows)
// while the pair's products (M = 256, issued by CTA 0) read both halves.
// KB: K values per ring stage (64, or 128 = two K blocks, which lets an
// MN-major operand arrive in boxes of 128 K rows: TMA moves 64-row boxes
// markedly slower per byte; K-major GEMMs gain a few per cent too).
template <int BN, bool kPair = false, int KB = 128>
struct Layout {
  static constexpr int kBLocal = kPair ? BN / 2 : BN;  // B rows this CTA loads
  static constexpr int kABytes = kBM * KB * 2;
  static constexpr int kBBytes = kBLocal * KB * 2;
  static constexpr int kStages = 196608 / (kABytes + kBBytes) > 8 ? 8 : 196608 / (kABytes + kBBytes);
  static constexpr int kA = 0;
  static constexpr int kB = kStages * kABytes;
  static constexpr int kBars = kB + kStages * kBBytes;
  static constexpr int bFull = 0, bEmpty = kStages, bAccFull = 2 * kStages,
                       bAccEmpty = 2 * kStages + 2;
  static constexpr int kNumBars = 2 * kStages + 4;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kSmemAlloc = kMisc + 16;
  static constexpr int kProducerWarp = 0, kMmaWarp = 1;
  static constexpr int kThreads = 192;  // + four epilogue warps
  static constexpr uint32_t kTmemCols = 2 * BN;  // two accumulators
};

enum Src : int { SRC_ROWS = 0, SRC_HEADS = 1 };
enum Epi : int { EPI_ROWS_BF16 = 0, EPI_ROWS_F32 = 1, EPI_HEADS = 2 };

// One operand. SRC_ROWS: a row-major matrix, [MN][K] when K-major, [K][MN]
// when MN-major. SRC_HEADS: tensors [B*heads[s]][T][D]; the token index
// b*T + t runs along MN when K-major, along K when MN-major, and the feature
// index along the other.
struct Operand {
  int src;
  int mn_major;
  int heads[3];
};

struct Params {
  int M, N, K;
  int tiles_m, tiles_n, splits;  // work units: tiles_m * tiles_n * splits
  int kb_per_split;     // 64-wide K blocks per unit
  int T, D;             // token rows per batch row; head dimension
  Operand a, b;
  int epi;
  int out_heads[3];     // EPI_HEADS: head counts of the output tensors
  void* out[3];         // EPI_HEADS: q, k, v (absent ones null); else out[0]
  int reduce;           // EPI_ROWS_F32: add into out[0] instead of storing
  int rope_segs;        // EPI_HEADS: rotate the first rope_segs tensors
  const float* rope_cos;
  const float* rope_sin;
  const int32_t* doc_start;  // flattened document starts, or null
};

// Feature index f of a head-major operand -> (tensor, head, d).
__device__ __forceinline__ void split_feature(const int* heads, int D, int f, int& seg, int& h,
                                              int& d) {
  seg = 0;
  while (seg < 2 && f >= heads[seg] * D) {
    f -= heads[seg] * D;
    ++seg;
  }
  h = f / D;
  d = f - h * D;
}

// One K-major box: BMN rows x the 64 K values from k0.
template <int BMN, bool kPairLoad>
__device__ __forceinline__ void operand_box_kmajor(bool issue, const Operand& o,
                                                   const CUtensorMap* m0, const CUtensorMap* m1,
                                                   const CUtensorMap* m2, int T, int D, int mn0,
                                                   int k0, uint32_t dst, uint32_t bar) {
  if (!issue) return;
  if (o.src == SRC_ROWS) {
    if (kPairLoad) tma_load_2d_pair(dst, m0, bar, k0, mn0);
    else tma_load_2d(dst, m0, bar, k0, mn0);
  } else {
    int seg, h, d;
    split_feature(o.heads, D, k0, seg, h, d);
    const int b = mn0 / T, t = mn0 - b * T;
    const CUtensorMap* mp = seg == 0 ? m0 : (seg == 1 ? m1 : m2);
    if (kPairLoad) tma_load_3d_pair(dst, mp, bar, d, t, b * o.heads[seg] + h);
    else tma_load_3d(dst, mp, bar, d, t, b * o.heads[seg] + h);
  }
}

// Issue (or, with issue = false, only count the bytes of) the TMA boxes of
// one operand tile: MN rows [mn0, mn0 + BMN) and the nsub (1 or KB / 64)
// K blocks from kb on, into dst.
template <int BMN, int KB, bool kPairLoad = false>
__device__ __forceinline__ uint32_t operand_boxes(bool issue, const Operand& o,
                                                  const CUtensorMap* m0, const CUtensorMap* m1,
                                                  const CUtensorMap* m2, int mn_total, int T,
                                                  int D, int mn0, int kb, int nsub, uint32_t dst,
                                                  uint32_t bar) {
  if (!o.mn_major) {
    // per K block one box of BMN rows x 64 K values, BMN * 128 bytes apart
    for (int sb = 0; sb < nsub; ++sb)
      operand_box_kmajor<BMN, kPairLoad>(issue, o, m0, m1, m2, T, D, mn0, (kb + sb) * kBK,
                                         dst + sb * BMN * 128, bar);
    return nsub * BMN * kBK * 2;
  }
  // MN-major: BMN / 64 boxes of 64 MN values x KB K rows, KB * 128 bytes
  // apart (a box reads all KB rows; those of a missing second block are
  // never multiplied)
  const int k0 = kb * kBK;
  uint32_t bytes = 0;
#pragma unroll
  for (int j = 0; j < BMN / 64; ++j) {
    const int f = mn0 + 64 * j;
    if (f >= mn_total) break;
    if (issue) {
      if (o.src == SRC_ROWS) {
        if (kPairLoad) tma_load_2d_pair(dst + j * KB * 128, m0, bar, f, k0);
        else tma_load_2d(dst + j * KB * 128, m0, bar, f, k0);
      } else {
        int seg, h, d;
        split_feature(o.heads, D, f, seg, h, d);
        const int b = k0 / T, t = k0 - b * T;
        const CUtensorMap* mp = seg == 0 ? m0 : (seg == 1 ? m1 : m2);
        if (kPairLoad) tma_load_3d_pair(dst + j * KB * 128, mp, bar, d, t, b * o.heads[seg] + h);
        else tma_load_3d(dst + j * KB * 128, mp, bar, d, t, b * o.heads[seg] + h);
      }
    }
    bytes += KB * 128;
  }
  return bytes;
}

// K step kk (16 K values) of an operand tile of BMN rows and KB K values.
template <int BMN, int KB>
__device__ __forceinline__ uint64_t operand_desc(bool mn_major, uint32_t base, int kk) {
  return mn_major ? smem_desc_sw128(base + kk * 2048, KB * 128, 1024)
                  : smem_desc_sw128(base + (kk >> 2) * (BMN * 128) + (kk & 3) * 32, 16, 1024);
}

// kPair: launched in clusters of two; p.tiles_m then counts 256-row tiles.
// KB = 128: p.kb_per_split is even (a stage never straddles two units' K
// ranges); only the last stage of K may hold one K block.
template <int BN, bool kPair = false, int KB = 128>
__global__ void __launch_bounds__(Layout<BN, kPair, KB>::kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB,
                const Params p) {
  pdl_wait_and_trigger();
  using L = Layout<BN, kPair, KB>;
  constexpr int kStages = L::kStages;
  constexpr int kSub = KB / kBK;  // K blocks per stage
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
  const int rank = kPair ? (int)cluster_rank() : 0;
  auto lead = [&](int i) -> uint32_t { return kPair ? map_rank(bar(i), 0) : bar(i); };
  const int nkb_total = (p.K + kBK - 1) / kBK;
  const int tiles = p.tiles_m * p.tiles_n;
  const int n_units = tiles * p.splits;
  // Work unit u (this CTA, or this pair, takes u = its index, + the number
  // of CTAs or pairs, ...): split u / tiles, then the tile, M fastest so that
  // CTAs running at the same time share the B tile (the weights) in L2. A
  // pair's CTA r takes rows [256 tm + 128 r, +128) of tile tm.
  const int u_first = kPair ? (int)blockIdx.x >> 1 : (int)blockIdx.x;
  const int u_step = kPair ? (int)gridDim.x >> 1 : (int)gridDim.x;
  auto unit = [&](int u, int& m0, int& n0, int& kb0, int& nkb) {
    const int z = u / tiles, r = u - z * tiles;
    const int tn = r / p.tiles_m;
    m0 = kPair ? (r - tn * p.tiles_m) * 2 * kBM + rank * kBM : (r - tn * p.tiles_m) * kBM;
    n0 = tn * BN;
    kb0 = z * p.kb_per_split;
    nkb = min(nkb_total, kb0 + p.kb_per_split) - kb0;  // >= 1: the host sizes the split so
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(L::bFull + s), 1);
      mbar_init(bar(L::bEmpty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(L::bAccFull + a), 1);
      // the epilogue threads that read the accumulator out (for a pair, one
      // arrival per epilogue warp of either CTA, on CTA 0's barrier)
      mbar_init(bar(L::bAccEmpty + a), kPair ? 8 : 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == L::kMmaWarp) {
    if constexpr (kPair) {
      tmem_alloc_pair(sb0 + L::kMisc, L::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(sb0 + L::kMisc, L::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync_all();  // both CTAs' barriers ready before cross-CTA signals
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == L::kProducerWarp) {
    if (lane == 0) {
      prefetch_tensor_map(&tmA0);
      prefetch_tensor_map(&tmB);
      int it = 0;  // stages loaded so far by this CTA, over all its units
      bool ok = true;
      constexpr int BL = L::kBLocal;
      for (int u = u_first; ok && u < n_units; u += u_step) {
        int m0, n0, kb0, nkb;
        unit(u, m0, n0, kb0, nkb);
        const int nb = n0 + rank * BL;  // this CTA's B rows
        for (int jb = 0; jb < nkb; jb += kSub, ++it) {
          const int ns = min(kSub, nkb - jb);  // K blocks in this stage
          const int s = it % kStages, round = it / kStages;
          if (it >= kStages && !mbar_wait(bar(L::bEmpty + s), (round - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t sa = sb0 + L::kA + s * L::kABytes, sbb = sb0 + L::kB + s * L::kBBytes;
          if (rank == 0) {
            // CTA 0's barrier counts the bytes of both CTAs' boxes
            uint32_t bytes = 0;
            for (int q = 0; q < (kPair ? 2 : 1); ++q)
              bytes += operand_boxes<kBM, KB>(false, p.a, &tmA0, &tmA1, &tmA2, p.M, p.T, p.D,
                                              m0 + q * kBM, kb0 + jb, ns, sa, 0) +
                       operand_boxes<BL, KB>(false, p.b, &tmB, &tmB, &tmB, p.N, p.T, p.D,
                                             n0 + q * BL, kb0 + jb, ns, sbb, 0);
            mbar_arrive_expect_tx(bar(L::bFull + s), bytes);
          }
          operand_boxes<kBM, KB, kPair>(true, p.a, &tmA0, &tmA1, &tmA2, p.M, p.T, p.D, m0,
                                        kb0 + jb, ns, sa, lead(L::bFull + s));
          operand_boxes<BL, KB, kPair>(true, p.b, &tmB, &tmB, &tmB, p.N, p.T, p.D, nb, kb0 + jb,
                                       ns, sbb, lead(L::bFull + s));
        }
      }
    }
  } else if (warp == L::kMmaWarp) {
    // one instruction stream: this CTA's, or for a pair CTA 0's, whose
    // products (M = 256) read both CTAs' tiles and write both accumulators
    if (lane == 0 && rank == 0) {
      const uint32_t idesc =
          idesc_f16(kPair ? 2 * kBM : kBM, BN, true, true, p.a.mn_major != 0, p.b.mn_major != 0);
      auto wait = [&](uint32_t b, uint32_t par) {
        return kPair ? mbar_wait_cl(b, par, abort_flag) : mbar_wait(b, par, abort_flag);
      };
      auto commit = [&](uint32_t b) {
        if constexpr (kPair) commit_pair(b);
        else mma_commit(b);
      };
      int it = 0, n = 0;  // stages consumed, units finished by this CTA
      bool ok = true;
      for (int u = u_first; ok && u < n_units; u += u_step, ++n) {
        int m0, n0, kb0, nkb;
        unit(u, m0, n0, kb0, nkb);
        const int a = n & 1;
        // the epilogue must have read this accumulator's previous unit out
        if (n >= 2 && !wait(bar(L::bAccEmpty + a), ((n >> 1) - 1) & 1)) break;
        tc_fence_after();
        const uint32_t acc = tmem + a * BN;
        for (int jb = 0; jb < nkb; jb += kSub, ++it) {
          const int s = it % kStages;
          if (!wait(bar(L::bFull + s), (it / kStages) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sb0 + L::kA + s * L::kABytes, sbb = sb0 + L::kB + s * L::kBBytes;
          const int nk = (kSub == 1 || jb + kSub <= nkb) ? KB / 16 : (nkb - jb) * (kBK / 16);
#pragma unroll
          for (int kk = 0; kk < KB / 16; ++kk) {
            if (kk >= nk) break;
            const uint64_t da = operand_desc<kBM, KB>(p.a.mn_major, sa, kk),
                           db = operand_desc<L::kBLocal, KB>(p.b.mn_major, sbb, kk);
            const uint32_t acc_on = (jb > 0 || kk > 0) ? 1u : 0u;
            if constexpr (kPair) mma_ss_pair(acc, da, db, idesc, acc_on);
            else mma_ss(acc, da, db, idesc, acc_on);
          }
          commit(bar(L::bEmpty + s));
        }
        if (ok) commit(bar(L::bAccFull + a));
      }
    }
  } else {
    // ---------------- epilogue: thread = TMEM lane = output row ----------------
    const int sub = warp & 3;
    const int r = sub * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(sub * 32) << 16);
    const int T = p.T, D = p.D;
    int n = 0;
    for (int u = u_first; u < n_units; u += u_step, ++n) {
      int m0, n0, kb0, nkb;
      unit(u, m0, n0, kb0, nkb);
      const int a = n & 1;
      if (!mbar_wait(bar(L::bAccFull + a), (n >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      const int m = m0 + r;
      const int b = m / T, t = m - b * T;
      int pos = t;
      if (p.epi == EPI_HEADS && p.rope_segs > 0 && m < p.M && p.doc_start)
        pos = m - p.doc_start[m];
      const int nch = min(BN, p.N - n0 + 31) / 32;  // chunks holding columns < N
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        const int nc = n0 + 32 * c;
        uint32_t v[32];
        tmem_ld32(tl + a * BN + 32 * c, v);
        tmem_wait_ld();
        if (c == nch - 1) {
          // every column of this accumulator that is used has been read
          tc_fence_before();
          if constexpr (kPair) {
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead(L::bAccEmpty + a));
          } else {
            mbar_arrive(bar(L::bAccEmpty + a));
          }
        }
        if (m >= p.M) continue;
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
        if (p.epi == EPI_HEADS) {
          int seg, h, d;
          split_feature(p.out_heads, D, nc, seg, h, d);  // 32 | D: the chunk stays in one head
          if (seg < p.rope_segs) {
            if (D == 64) rope_pairs<32, 64>(f, p.rope_cos, p.rope_sin, pos, d, false);
            else rope_pairs<32, 128>(f, p.rope_cos, p.rope_sin, pos, d, false);
          }
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out[seg]) +
                               ((size_t)(b * p.out_heads[seg] + h) * T + t) * D + d;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            reinterpret_cast<uint4*>(dst)[e] =
                make_uint4(pack_bf16(f[8 * e], f[8 * e + 1]), pack_bf16(f[8 * e + 2], f[8 * e + 3]),
                           pack_bf16(f[8 * e + 4], f[8 * e + 5]),
                           pack_bf16(f[8 * e + 6], f[8 * e + 7]));
        } else if (p.epi == EPI_ROWS_BF16) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out[0]) + (size_t)m * p.N + nc;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (nc + 8 * e < p.N)  // N % 8 == 0
              reinterpret_cast<uint4*>(dst)[e] = make_uint4(
                  pack_bf16(f[8 * e], f[8 * e + 1]), pack_bf16(f[8 * e + 2], f[8 * e + 3]),
                  pack_bf16(f[8 * e + 4], f[8 * e + 5]), pack_bf16(f[8 * e + 6], f[8 * e + 7]));
        } else {
          float* dst = reinterpret_cast<float*>(p.out[0]) + (size_t)m * p.N + nc;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (nc + 4 * e >= p.N) break;  // N % 4 == 0
            if (p.reduce)
              red_add_v4(dst + 4 * e, v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
            else
              reinterpret_cast<float4*>(dst)[e] =
                  make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // a pair: no CTA leaves (or frees TMEM) while the other may still signal it
  if constexpr (kPair) cluster_sync_all();
  if (warp == L::kMmaWarp) {
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(tmem, L::kTmemCols);
    else tmem_dealloc(tmem, L::kTmemCols);
  }
}

// R(pos)^T applied to a [B*heads][T][D] bf16 gradient (taken with respect to
// rotated vectors), written to dst: 8 values per thread.
template <int D>
__global__ void __launch_bounds__(256) rope_grad_kernel(const __nv_bfloat16* __restrict__ g,
                                                        const float* __restrict__ rc,
                                                        const float* __restrict__ rs,
                                                        const int32_t* __restrict__ doc_start,
                                                        __nv_bfloat16* __restrict__ dst, int heads,
                                                        int T, long n8) {
  pdl_wait_and_trigger();
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const long e0 = i * 8;
  const int d0 = (int)(e0 % D);
  const long row = e0 / D;  // (b * heads + h) * T + t
  const int t = (int)(row % T);
  const int b = (int)(row / T / heads);
  const int m = b * T + t;
  const int pos = doc_start ? m - doc_start[m] : t;
  float v[8];
  load8_bf16(g + e0, v);
  rope_pairs<8, D>(v, rc, rs, pos, d0, true);
  store8_bf16(dst + e0, v);
}

}  // namespace proj100
