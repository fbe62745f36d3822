// attn_api.cu -- the C ABI of libattn.so (declared in include/attn.h):
// host-side validation, the workspace plan, kernel launches and the device
// status word. No function here allocates or frees device memory.
#include <math.h>
#include <stdint.h>

#include <mutex>
#include <type_traits>

#include "attn.h"
#include "common.cuh"
#include "bwd_sm100.cuh"
#include "bwd_pair_sm100.cuh"
#include "dq_sm100.cuh"
#include "decode.cuh"
#include "fwd_sm100.cuh"
#include "prep.cuh"
#include "simt.cuh"
#include "trace.cuh"

namespace {

constexpr size_t kAlign = 256;
inline size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Workspace layout (byte offsets from the caller's base pointer).
struct WsPlan {
  size_t doc_start = 0, doc_end = 0;  // int32 [B*T] each
  size_t delta = 0;                   // f32 [B*H*T] (f32 backward) or [B*H*Tpad] (bf16 backward)
  size_t lse2 = 0;                    // f32 [B*H*Tpad] lse*log2(e) (bf16 backward)
  size_t dq_acc = 0;                  // f32 [B*H*T*D] dq accumulator (bf16 backward)
  size_t q16 = 0, k16 = 0;            // rotated q, k as fp16 [B*H*T*D] each (bf16 storage)
  size_t qfac = 0, kfac = 0;          // inverse tile factors (bf16, both passes): q as f32
                                      // [B*H*ceil(T/128)][4] records, k as f32 [B*H*ceil(T/128)]
  size_t hstat = 0;                   // f32 [B*H][4] per-head max |dO_i|, |Delta_i|, |v_j| (bf16 backward)
  size_t dk_acc = 0, dv_acc = 0;      // f32 [B*Hkv*T*D] each when the backward splits groups
  int split = 1;                      // query-head groups split over this many CTAs
  size_t total = 0;
};

// Grouped-query backward: one CTA per (key/value head, key tile) walks the G
// query heads of its group. When that gives too few CTAs to fill the GPU, the
// group is split over S CTAs (S the smallest divisor of G reaching about two
// CTAs per SM of a B200), which then add their dK, dV parts into fp32
// accumulators.
constexpr long kSplitTargetCtas = 2 * 148;
int choose_split(int B, int H, int Hkv, int T) {
  const int G = H / Hkv;
  const long base = (long)B * Hkv * ((T + 127) / 128);
  if (G == 1 || base >= kSplitTargetCtas) return 1;
  for (int S = 2; S < G; ++S)
    if (G % S == 0 && base * S >= kSplitTargetCtas) return S;
  return G;
}

bool sizes_ok(int B, int H, int T, int D) {
  if (B <= 0 || H <= 0 || T <= 0) return false;
  if (D != 64 && D != 128) return false;
  const int64_t bt = (int64_t)B * T;
  const int64_t n = bt * H * D;
  return bt < INT32_MAX && n < INT32_MAX;
}

WsPlan plan(int B, int H, int T, int D, int dtype, int is_bwd, int Hkv = 0) {
  WsPlan p;
  if (Hkv <= 0) Hkv = H;
  size_t off = 0;
  const size_t bt = (size_t)B * T, rows = bt * H, n = rows * D;
  const size_t tiles = (size_t)B * H * ((T + 127) / 128);
  const size_t rows_pad = tiles * 128;
  p.doc_start = off; off += round_up(bt * sizeof(int32_t));
  p.doc_end = off;   off += round_up(bt * sizeof(int32_t));
  if (is_bwd && dtype == ATTN_F32) { p.delta = off; off += round_up(rows * sizeof(float)); }
  if (is_bwd && dtype == ATTN_BF16) {
    p.delta = off;  off += round_up(rows_pad * sizeof(float));
    p.lse2 = off;   off += round_up(rows_pad * sizeof(float));
    p.dq_acc = off; off += round_up(n * sizeof(float));
    p.q16 = off;    off += round_up(n * 2);
    p.k16 = off;    off += round_up(n * 2);
    p.qfac = off;   off += round_up(tiles * 4 * sizeof(float));
    p.kfac = off;   off += round_up(tiles * sizeof(float));
    p.hstat = off;  off += round_up((size_t)B * H * 4 * sizeof(float));
    p.split = choose_split(B, H, Hkv, T);
    if (p.split > 1) {
      const size_t nkv = bt * Hkv * D;
      p.dk_acc = off; off += round_up(nkv * sizeof(float));
      p.dv_acc = off; off += round_up(nkv * sizeof(float));
    }
  }
  if (dtype == ATTN_BF16 && !is_bwd) {
    p.q16 = off;  off += round_up(n * 2);
    p.k16 = off;  off += round_up(n * 2);
    p.qfac = off; off += round_up(tiles * 4 * sizeof(float));
    p.kfac = off; off += round_up(tiles * sizeof(float));
  }
  p.total = off;
  return p;
}

// The forward's rotated operands kept for the backward (attn_fwd_save /
// attn_bwd_saved): rotated q, k as fp16 and their inverse tile factors, in the
// layout rope_prep writes them.
struct SavedPlan {
  size_t q16 = 0, k16 = 0, qfac = 0, kfac = 0, docs = 0, total = 0;
};

SavedPlan saved_plan(int B, int H, int Hkv, int T, int D) {
  SavedPlan p;
  const size_t nt = (size_t)((T + 127) / 128);
  size_t off = 0;
  p.q16 = off;  off += round_up((size_t)B * H * T * D * 2);
  p.k16 = off;  off += round_up((size_t)B * Hkv * T * D * 2);
  p.qfac = off; off += round_up((size_t)B * H * nt * 4 * sizeof(float));
  p.kfac = off; off += round_up((size_t)B * Hkv * nt * sizeof(float));
  // per-token document start and end (int32 [B*T] each), with cu_seqlens
  p.docs = off; off += round_up((size_t)2 * B * T * sizeof(int32_t));
  p.total = off;
  return p;
}

// ---- TMA descriptors (driver entry point fetched through the runtime) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)f;
  }
  return fn;
}

// A [B*H][T][D] 16-bit tensor seen in boxes of 128 rows x 64 columns with the
// 128-byte swizzle; rows past T read as zeros.
bool make_tile_map(CUtensorMap* m, const void* base, bool is_f16, int D, int T, int BH,
                   int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, is_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A RoPE table ([T][D/2] fp32) seen in boxes of 128 rows x 32 floats with the
// 128-byte swizzle; rows past T read as zeros.
bool make_table_map(CUtensorMap* m, const float* base, int D, int T) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)(D / 2), (cuuint64_t)T, 1};
  cuuint64_t strides[2] = {(cuuint64_t)(D / 2) * 4, (cuuint64_t)T * (D / 2) * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The fp32 [B*H][T][D] dq accumulator seen in boxes of 32 rows x 32 columns
// (128-byte swizzle) for tensor reduce-add; rows past T are clipped.
bool make_acc_map(CUtensorMap* m, float* base, int D, int T, int BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)T * D * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Opt a kernel into its dynamic shared memory once per device.
template <typename K>
bool ensure_smem(K kernel, int bytes, bool* done_per_device) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!done_per_device[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
      return false;
    done_per_device[dev] = true;
  }
  return true;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int check_common(const void* q, const void* k, const void* v, const float* rc, const float* rs,
                 const int32_t* cu, int B, int H, int H_kv, int T, int D, float scale, int dtype,
                 void* ws, size_t ws_bytes, int is_bwd) {
  if (!q || !k || !v) return ATTN_EINVAL;
  if (dtype != ATTN_BF16 && dtype != ATTN_F32) return ATTN_EINVAL;
  if (B <= 0 || H <= 0 || T <= 0) return ATTN_EINVAL;
  if (H_kv <= 0 || H % H_kv != 0) return ATTN_EINVAL;
  if (!isfinite(scale)) return ATTN_EINVAL;
  if ((rc == nullptr) != (rs == nullptr)) return ATTN_EINVAL;
  if (!sizes_ok(B, H, T, D)) return ATTN_EUNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return ATTN_EALIGN;
  if ((rc && !aligned(rc, 16)) || (rs && !aligned(rs, 16)) || (cu && !aligned(cu, 4))) return ATTN_EALIGN;
  const WsPlan p = plan(B, H, T, D, dtype, is_bwd, H_kv);
  if (p.total > 0) {
    if (!ws) return ATTN_EWORKSPACE;
    if (!aligned(ws, 16)) return ATTN_EALIGN;
    if (ws_bytes < p.total) return ATTN_EWORKSPACE;
  }
  return ATTN_OK;
}

int launch_status() {
  const cudaError_t pe = pdl_launch_error();
  pdl_launch_error() = cudaSuccess;
  return (cudaGetLastError() == cudaSuccess && pe == cudaSuccess) ? ATTN_OK : ATTN_ECUDA;
}

template <typename TIO, int D>
int fwd_simt(const void* q, const void* k, const void* v, const float* rc, const float* rs,
             const int32_t* ds, void* o, float* lse, int B, int H, int Hkv, int T, float scale,
             cudaStream_t st) {
  dim3 grid(B * H, (T + 15) / 16);
  ATTN_LAUNCH(KK_FWD, st, pdl_launch(simt_fwd_kernel<TIO, D>, grid, 128, 0, st, (const TIO*)q, (const TIO*)k,
                                                            (const TIO*)v, rc, rs, ds, (TIO*)o,
                                                            lse, H, Hkv, T, scale));
  return launch_status();
}

template <typename TIO, int D>
int bwd_simt(const void* q, const void* k, const void* v, const void* o, const void* dO,
             const float* lse, const float* rc, const float* rs, const int32_t* ds,
             const int32_t* de, float* delta, void* dq, void* dk, void* dv, int B, int H, int Hkv,
             int T, float scale, cudaStream_t st) {
  const long rows = (long)B * H * T;
  ATTN_LAUNCH(KK_DELTA, st, pdl_launch(delta_kernel<TIO, D>, (unsigned)((rows + 7) / 8), 256, 0, st, (const TIO*)o, (const TIO*)dO, delta, rows));
  if (launch_status()) return ATTN_ECUDA;
  dim3 g1(B * Hkv, (T + 31) / 32), g2(B * H, (T + 31) / 32);
  ATTN_LAUNCH(KK_DKDV, st, pdl_launch(simt_dkdv_kernel<TIO, D>, g1, 128, 0, st, (const TIO*)q, (const TIO*)k, (const TIO*)v, (const TIO*)dO, lse, delta, rc, rs,
                  ds, de, (TIO*)dk, (TIO*)dv, H, Hkv, T, scale));
  if (launch_status()) return ATTN_ECUDA;
  ATTN_LAUNCH(KK_DQ, st, pdl_launch(simt_dq_kernel<TIO, D>, g2, 128, 0, st, (const TIO*)q, (const TIO*)k, (const TIO*)v, (const TIO*)dO, lse, delta, rc, rs,
                  ds, (TIO*)dq, H, Hkv, T, scale));
  return launch_status();
}

// The RoPE pre-pass over q and k (see prep.cuh): one block per tile, batch
// and head.
template <int D>
int launch_rope_prep(const void* q, const void* k, const float* rc, const float* rs,
                     const int32_t* ds, __half* qo, __half* ko, float* qf, float* kf, float* hstat,
                     int B, int H, int Hkv, int T, int nt, cudaStream_t st) {
  const dim3 grid(nt, B, H + Hkv);
  ATTN_LAUNCH(KK_ROPE_PREP, st, pdl_launch(rope_prep_kernel<D>, grid, kRopePrepThreads, 0, st,
                                           (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, rc, rs,
                                           ds, qo, ko, qf, kf, hstat, B, H, Hkv, T, nt));
  return launch_status();
}

template <int D>
int fwd_tc(const void* q, const void* k, const void* v, const float* rc, const float* rs,
           const int32_t* ds, void* o, float* lse, int B, int H, int Hkv, int T, float scale,
           char* ws, const WsPlan& wp, char* saved, cudaStream_t st) {
  using L = fwd100::Layout<D>;
  const int nt = (T + 127) / 128, BH = B * H, BHkv = B * Hkv;
  // With RoPE q and k are rotated once into fp16 tiles with power-of-two
  // factors (rope_prep); without it the kernel reads them as given (bf16).
  const void* qs = q;
  const void* ks = k;
  float *qf = nullptr, *kf = nullptr;
  if (rc) {
    // into the caller's saved buffer when it keeps them for the backward
    const SavedPlan sp = saved_plan(B, H, Hkv, T, D);
    __half* qh = (__half*)(saved ? saved + sp.q16 : ws + wp.q16);
    __half* kh = (__half*)(saved ? saved + sp.k16 : ws + wp.k16);
    qf = (float*)(saved ? saved + sp.qfac : ws + wp.qfac);
    kf = (float*)(saved ? saved + sp.kfac : ws + wp.kfac);
    if (launch_rope_prep<D>(q, k, rc, rs, ds, qh, kh, qf, kf, nullptr, B, H, Hkv, T, nt, st))
      return ATTN_ECUDA;
    qs = qh;
    ks = kh;
  }
  const bool f16 = rc != nullptr;
  CUtensorMap mq, mk, mv, mo;
  if (!make_tile_map(&mq, qs, f16, D, T, BH) || !make_tile_map(&mk, ks, f16, D, T, BHkv, L::kKV) ||
      !make_tile_map(&mv, v, false, D, T, BHkv, L::kKV) || !make_tile_map(&mo, o, false, D, T, BH))
    return ATTN_ECUDA;
  static bool smem_set[64] = {};
  if (!ensure_smem(fwd100::fwd_kernel<D>, L::kSmemAlloc, smem_set)) return ATTN_ECUDA;
  fwd100::Params prm;
  const int n_pairs = (nt + 1) / 2;
  prm.T = T;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.BH = BH;
  prm.n_pairs = n_pairs;
  prm.n_qtiles = nt;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.idesc_s = sm100::idesc_f16(128, L::kKV, !f16, !f16, false, false);
  prm.q_fac = qf;
  prm.k_fac = kf;
  prm.doc_start = ds;
  prm.o = (__nv_bfloat16*)o;
  prm.lse = lse;
  ATTN_LAUNCH(KK_FWD, st, pdl_launch(fwd100::fwd_kernel<D>, (unsigned)(n_pairs * BH), L::kThreads, L::kSmemAlloc, st, mq, mk, mv, mo, prm));
  return launch_status();
}

template <int D, bool kF16, bool kDQ>
int launch_dkdv(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                const CUtensorMap& mo, const CUtensorMap& mdq, const CUtensorMap& mdk,
                const CUtensorMap& mdv, const CUtensorMap& mrc, const CUtensorMap& mrs,
                const bwd100::Params& prm, unsigned grid, cudaStream_t st) {
  using L = bwd100::Layout<D, kDQ>;
  static bool smem_set[64] = {};
  if (!ensure_smem(bwd100::dkdv_kernel<D, kF16, kDQ>, L::kSmemAlloc, smem_set)) return ATTN_ECUDA;
  ATTN_LAUNCH(KK_DKDV, st, pdl_launch(bwd100::dkdv_kernel<D, kF16, kDQ>, grid, L::kThreads,
                                       L::kSmemAlloc, st, mq, mk, mv, mo, mdq, mdk, mdv, mrc, mrs, prm));
  return launch_status();
}

template <int D, bool kF16>
int launch_dq(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
              const CUtensorMap& mo, const dq100::Params& prm, unsigned grid, cudaStream_t st) {
  using L = dq100::Layout<D>;
  static bool smem_set[64] = {};
  if (!ensure_smem(dq100::dq_kernel<D, kF16>, L::kSmemAlloc, smem_set)) return ATTN_ECUDA;
  ATTN_LAUNCH(KK_DQ, st, pdl_launch(dq100::dq_kernel<D, kF16>, grid, L::kThreads, L::kSmemAlloc,
                                     st, mq, mk, mv, mo, prm));
  return launch_status();
}

// dQ by the query-tile pass (dq_sm100.cuh: two more products per tile pair,
// no fp32 accumulator, no atomics, no zeroing or finishing pass) or by
// reduce-adds from the key-tile kernel: a per-head-size choice, set by
// measuring both on the B200 (the measurement is recorded with the library's
// design notes).
// The test build (build.py --debug) takes the other route, so the GPU tests
// cover both.
#ifndef ATTN_DQ_PASS_D64
#define ATTN_DQ_PASS_D64 0
#endif
#ifndef ATTN_DQ_PASS_D128
#define ATTN_DQ_PASS_D128 0
#endif
#ifdef ATTN_DQ_ROUTE_SWAPPED
constexpr bool kDqRouteSwapped = true;
#else
constexpr bool kDqRouteSwapped = false;
#endif
constexpr bool use_dq_pass(int D) {
  return (D == 64 ? ATTN_DQ_PASS_D64 : ATTN_DQ_PASS_D128) != kDqRouteSwapped;
}

// The tensor-core backward's route, chosen at run time by
// attn_set_backward_route: 0 = the default above, 1 = key-tile kernel without
// dQ + query-tile dQ pass, 2 = the CTA-pair key-tile kernel (D = 128; D = 64
// takes route 1) + query-tile dQ pass.
int g_bwd_route = 0;
int backward_route(int D) {
  if (g_bwd_route == 2) return D == 128 ? 2 : 1;
  if (g_bwd_route == 1) return 1;
  return use_dq_pass(D) ? 1 : 0;
}

template <bool kF16>
int launch_dkdv_pair(const void* qs, const void* dO, const CUtensorMap& mq, const CUtensorMap& mk,
                     const CUtensorMap& mv, const CUtensorMap& mo, const bwd100::Params& prm,
                     int T, int BH, cudaStream_t st) {
  using L = bwd2::Layout<128>;
  CUtensorMap mqr, mor;  // 64-row boxes: the row halves of q and dO
  if (!make_tile_map(&mqr, qs, kF16, 128, T, BH, 64) || !make_tile_map(&mor, dO, false, 128, T, BH, 64))
    return ATTN_ECUDA;
  static bool smem_set[64] = {};
  if (!ensure_smem(bwd2::dkdv_pair_kernel<128, kF16>, L::kSmemAlloc, smem_set)) return ATTN_ECUDA;
  const unsigned grid = 2u * (unsigned)(prm.BHkv * prm.n_split * ((prm.n_tiles + 1) / 2));
  ATTN_LAUNCH(KK_DKDV, st, pdl_cluster_launch(bwd2::dkdv_pair_kernel<128, kF16>, grid, L::kThreads,
                                              L::kSmemAlloc, st, 2u, mqr, mq, mk, mv, mor, mo, prm));
  return launch_status();
}

template <int D>
int bwd_tc(const void* q, const void* k, const void* v, const void* o, const void* dO,
           const float* lse, const float* rc, const float* rs, const int32_t* ds,
           const int32_t* de, void* dq, void* dk, void* dv, int B, int H, int Hkv, int T,
           float scale, char* ws, const WsPlan& wp, const char* saved, cudaStream_t st) {
  const int nt = (T + 127) / 128, BH = B * H, BHkv = B * Hkv, Tpad = nt * 128;
  // With RoPE the scores are recomputed from fp16 operands (the rotated q, k
  // with per-tile factors, as the forward computed them); without it from q,
  // k as given (bf16).
  const bool f16 = rc != nullptr;
  // the forward's rotated operands: from the caller's saved buffer when given
  // (attn_bwd_saved), else made again here
  const bool reuse = f16 && saved != nullptr;
  const SavedPlan sp = saved_plan(B, H, Hkv, T, D);
  __half* q16 = reuse ? (__half*)(saved + sp.q16) : (__half*)(ws + wp.q16);
  __half* k16 = reuse ? (__half*)(saved + sp.k16) : (__half*)(ws + wp.k16);
  const void* qs = f16 ? (const void*)q16 : q;
  const void* ks = f16 ? (const void*)k16 : k;
  float* delta = (float*)(ws + wp.delta);
  float* lse2 = (float*)(ws + wp.lse2);
  float* dq_acc = (float*)(ws + wp.dq_acc);
  float* qinv = reuse ? (float*)(saved + sp.qfac) : (float*)(ws + wp.qfac);
  float* kinv = reuse ? (float*)(saved + sp.kfac) : (float*)(ws + wp.kfac);
  float* hstat = f16 ? (float*)(ws + wp.hstat) : nullptr;
  const int split = wp.split;
  float* dk_acc = split > 1 ? (float*)(ws + wp.dk_acc) : nullptr;
  float* dv_acc = split > 1 ? (float*)(ws + wp.dv_acc) : nullptr;
  if (reuse) {
    // the statistics slots the row pass fills with atomic maxima start at 0
    // (rope_prep zeroes them when it runs)
    if (cudaMemsetAsync(hstat, 0, (size_t)BH * 4 * sizeof(float), st) != cudaSuccess) return ATTN_ECUDA;
  } else if (f16) {
    // the forward's rotation, factors included (same kernel, same values)
    if (launch_rope_prep<D>(q, k, rc, rs, ds, q16, k16, qinv, kinv, hstat, B, H, Hkv, T, nt, st))
      return ATTN_ECUDA;
  }
  const int route = backward_route(D);
  const bool dq_pass = route != 0;
  const long rows_pad = (long)BH * Tpad;
  ATTN_LAUNCH(KK_DELTA, st, pdl_launch(bwd_prep_kernel<D>, (unsigned)(rows_pad * (D / 8) / 256), 256, 0, st,
                                       (const __nv_bfloat16*)o, (const __nv_bfloat16*)dO, lse, delta, lse2,
                                       dq_pass ? nullptr : dq_acc, dk_acc, dv_acc,
                                       (const __nv_bfloat16*)v, hstat, H, Hkv, T, Tpad, rows_pad));
  if (launch_status()) return ATTN_ECUDA;
  CUtensorMap mq, mk, mv, mo, mdq, mdk, mdv;
  if (!make_tile_map(&mq, qs, f16, D, T, BH) || !make_tile_map(&mk, ks, f16, D, T, BHkv) ||
      !make_tile_map(&mv, v, false, D, T, BHkv) || !make_tile_map(&mo, dO, false, D, T, BH) ||
      !make_acc_map(&mdq, dq_acc, D, T, BH) || !make_tile_map(&mdk, dk, false, D, T, BHkv) ||
      !make_tile_map(&mdv, dv, false, D, T, BHkv))
    return ATTN_ECUDA;
  // the RoPE tables for the key-tile epilogue (without RoPE the kernel does
  // not read them: any valid map stands in)
  CUtensorMap mrc = mdk, mrs = mdk;
  if (rc && (!make_table_map(&mrc, rc, D, T) || !make_table_map(&mrs, rs, D, T))) return ATTN_ECUDA;
  bwd100::Params prm;
  prm.T = T;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.BHkv = BHkv;
  prm.n_split = split;
  prm.n_tiles = nt;
  prm.Tpad = Tpad;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.scale = scale;
  prm.lse2 = lse2;
  prm.delta = delta;
  prm.doc_start = ds;
  prm.doc_end = de;
  prm.rope_cos = rc;
  prm.rope_sin = rs;
  prm.dq_acc = dq_acc;
  prm.dk = (__nv_bfloat16*)dk;
  prm.dv = (__nv_bfloat16*)dv;
  prm.dk_acc = dk_acc;
  prm.dv_acc = dv_acc;
  prm.qinv = qinv;
  prm.kinv = kinv;
  prm.hstat = hstat;
  const unsigned grid = (unsigned)(nt * BHkv * split);
  int rc_k = ATTN_ECUDA;
  if (route == 2) {  // backward_route gives 2 only at D = 128
    if constexpr (D == 128)
      rc_k = f16 ? launch_dkdv_pair<true>(qs, dO, mq, mk, mv, mo, prm, T, BH, st)
                 : launch_dkdv_pair<false>(qs, dO, mq, mk, mv, mo, prm, T, BH, st);
  } else if (dq_pass)
    rc_k = f16 ? launch_dkdv<D, true, false>(mq, mk, mv, mo, mdq, mdk, mdv, mrc, mrs, prm, grid, st)
               : launch_dkdv<D, false, false>(mq, mk, mv, mo, mdq, mdk, mdv, mrc, mrs, prm, grid, st);
  else
    rc_k = f16 ? launch_dkdv<D, true, true>(mq, mk, mv, mo, mdq, mdk, mdv, mrc, mrs, prm, grid, st)
               : launch_dkdv<D, false, true>(mq, mk, mv, mo, mdq, mdk, mdv, mrc, mrs, prm, grid, st);
  if (rc_k) return rc_k;
  if (split > 1) {
    // dk = R^T (scale * sum of the parts), dv = sum of the parts
    const long n8kv = (long)BHkv * T * D / 8;
    ATTN_LAUNCH(KK_DQ_FINALIZE, st, pdl_launch(dq_finalize_kernel<D>, (unsigned)(((n8kv + 1) / 2 + 255) / 256), 256, 0, st, dk_acc, rc, rs, ds, (__nv_bfloat16*)dk, Hkv, T, scale, n8kv, (const float*)nullptr, (const float*)nullptr, Hkv, nt));
    if (launch_status()) return ATTN_ECUDA;
    ATTN_LAUNCH(KK_DQ_FINALIZE, st, pdl_launch(dq_finalize_kernel<D>, (unsigned)(((n8kv + 1) / 2 + 255) / 256), 256, 0, st, dv_acc, nullptr, nullptr, nullptr, (__nv_bfloat16*)dv, Hkv, T, 1.0f, n8kv, (const float*)nullptr, (const float*)nullptr, Hkv, nt));
    if (launch_status()) return ATTN_ECUDA;
  }
  if (dq_pass) {
    dq100::Params qp;
    qp.T = T;
    qp.H = H;
    qp.Hkv = Hkv;
    qp.BH = BH;
    qp.n_tiles = nt;
    qp.Tpad = Tpad;
    qp.scale_log2 = scale * 1.4426950408889634f;
    qp.scale = scale;
    qp.lse2 = lse2;
    qp.delta = delta;
    qp.doc_start = ds;
    qp.rope_cos = rc;
    qp.rope_sin = rs;
    qp.qinv = qinv;
    qp.kinv = kinv;
    qp.hstat = hstat;
    qp.dq = (__nv_bfloat16*)dq;
    const unsigned qgrid = (unsigned)(nt * BH);
    return f16 ? launch_dq<D, true>(mq, mk, mv, mo, qp, qgrid, st)
               : launch_dq<D, false>(mq, mk, mv, mo, qp, qgrid, st);
  }
  const long n8 = (long)BH * T * D / 8;
  ATTN_LAUNCH(KK_DQ_FINALIZE, st, pdl_launch(dq_finalize_kernel<D>, (unsigned)(((n8 + 1) / 2 + 255) / 256), 256, 0, st, dq_acc, rc, rs, ds, (__nv_bfloat16*)dq, H, T, scale, n8, f16 ? (const float*)qinv : nullptr, (const float*)hstat, Hkv, nt));
  return launch_status();
}

__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = sm100::exp2_fma(x[i]);
}

}  // namespace

extern "C" {

size_t attn_workspace_bytes(int B, int H, int T, int D, int dtype, int is_bwd) {
  if (!sizes_ok(B, H, T, D) || (dtype != ATTN_BF16 && dtype != ATTN_F32)) return 0;
  return plan(B, H, T, D, dtype, is_bwd).total;
}

size_t attn_workspace_bytes_gqa(int B, int H, int H_kv, int T, int D, int dtype, int is_bwd) {
  if (!sizes_ok(B, H, T, D) || (dtype != ATTN_BF16 && dtype != ATTN_F32)) return 0;
  if (H_kv <= 0 || H % H_kv != 0) return 0;
  return plan(B, H, T, D, dtype, is_bwd, H_kv).total;
}

size_t attn_saved_bytes(int B, int H, int H_kv, int T, int D, int dtype, int has_rope) {
  if (!sizes_ok(B, H, T, D) || dtype != ATTN_BF16 || !has_rope) return 0;
  if (H_kv <= 0 || H % H_kv != 0) return 0;
  return saved_plan(B, H, H_kv, T, D).total;
}

}  // extern "C"

namespace {

// A saved buffer is used only where there is something to keep (bf16
// storage with RoPE); elsewhere it may be null and is ignored.
int check_saved(const void* saved, size_t saved_bytes, int B, int H, int H_kv, int T, int D,
                int dtype, const float* rope_cos) {
  const size_t need = attn_saved_bytes(B, H, H_kv, T, D, dtype, rope_cos != nullptr);
  if (need == 0 || saved == nullptr) return ATTN_OK;  // nothing kept: the plain call
  if (!aligned(saved, 16)) return ATTN_EALIGN;
  if (saved_bytes < need) return ATTN_EWORKSPACE;
  return ATTN_OK;
}

int fwd_impl(const void* q, const void* k, const void* v, const float* rope_cos,
             const float* rope_sin, const int32_t* cu_seqlens, void* o, float* lse, int B, int H,
             int H_kv, int T, int D, float scale, int dtype, void* workspace, size_t ws_bytes,
             void* saved, void* stream) {
  int rc = check_common(q, k, v, rope_cos, rope_sin, cu_seqlens, B, H, H_kv, T, D, scale, dtype,
                        workspace, ws_bytes, 0);
  if (rc) return rc;
  if (!o || !lse) return ATTN_EINVAL;
  if (!aligned(o, 16) || !aligned(lse, 4)) return ATTN_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  const WsPlan p = plan(B, H, T, D, dtype, 0);
  char* ws = (char*)workspace;
  char* sv = (dtype == ATTN_BF16 && rope_cos && saved) ? (char*)saved : nullptr;
  int32_t* ds = nullptr;
  if (cu_seqlens) {
    // kept with the saved operands when there are any: the backward reuses them
    int32_t* de;
    if (sv) {
      ds = (int32_t*)(sv + saved_plan(B, H, H_kv, T, D).docs);
      de = ds + (size_t)B * T;
    } else {
      ds = (int32_t*)(ws + p.doc_start);
      de = (int32_t*)(ws + p.doc_end);
    }
    ATTN_LAUNCH(KK_DOC_RANGES, st, pdl_launch(doc_ranges_kernel, doc_ranges_blocks(B, T), 1024, 0, st, cu_seqlens, B, T, ds, de));
    if (launch_status()) return ATTN_ECUDA;
  }
  if (dtype == ATTN_F32) {
    return D == 64 ? fwd_simt<float, 64>(q, k, v, rope_cos, rope_sin, ds, o, lse, B, H, H_kv, T,
                                         scale, st)
                   : fwd_simt<float, 128>(q, k, v, rope_cos, rope_sin, ds, o, lse, B, H, H_kv, T,
                                          scale, st);
  }
  return D == 64 ? fwd_tc<64>(q, k, v, rope_cos, rope_sin, ds, o, lse, B, H, H_kv, T, scale, ws,
                              p, sv, st)
                 : fwd_tc<128>(q, k, v, rope_cos, rope_sin, ds, o, lse, B, H, H_kv, T, scale, ws,
                               p, sv, st);
}

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dO,
             const float* lse, const float* rope_cos, const float* rope_sin,
             const int32_t* cu_seqlens, int B, int H, int H_kv, int T, int D, float scale,
             int dtype, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
             const void* saved, void* stream);

}  // namespace

extern "C" {

int attn_fwd_gqa(const void* q, const void* k, const void* v, const float* rope_cos,
                 const float* rope_sin, const int32_t* cu_seqlens, void* o, float* lse, int B,
                 int H, int H_kv, int T, int D, float scale, int dtype, void* workspace,
                 size_t ws_bytes, void* stream) {
  return fwd_impl(q, k, v, rope_cos, rope_sin, cu_seqlens, o, lse, B, H, H_kv, T, D, scale,
                  dtype, workspace, ws_bytes, nullptr, stream);
}

int attn_fwd_save(const void* q, const void* k, const void* v, const float* rope_cos,
                  const float* rope_sin, const int32_t* cu_seqlens, void* o, float* lse, int B,
                  int H, int H_kv, int T, int D, float scale, int dtype, void* workspace,
                  size_t ws_bytes, void* saved, size_t saved_bytes, void* stream) {
  const int rc = check_saved(saved, saved_bytes, B, H, H_kv, T, D, dtype, rope_cos);
  if (rc) return rc;
  return fwd_impl(q, k, v, rope_cos, rope_sin, cu_seqlens, o, lse, B, H, H_kv, T, D, scale,
                  dtype, workspace, ws_bytes, saved, stream);
}

int attn_fwd(const void* q, const void* k, const void* v, const float* rope_cos,
             const float* rope_sin, const int32_t* cu_seqlens, void* o, float* lse, int B, int H,
             int T, int D, float scale, int dtype, void* workspace, size_t ws_bytes,
             void* stream) {
  return attn_fwd_gqa(q, k, v, rope_cos, rope_sin, cu_seqlens, o, lse, B, H, H, T, D, scale,
                      dtype, workspace, ws_bytes, stream);
}

int attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, const float* rope_cos, const float* rope_sin,
                 const int32_t* cu_seqlens, int B, int H, int H_kv, int T, int D, float scale,
                 int dtype, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                 void* stream) {
  return bwd_impl(q, k, v, o, dO, lse, rope_cos, rope_sin, cu_seqlens, B, H, H_kv, T, D, scale,
                  dtype, dq, dk, dv, workspace, ws_bytes, nullptr, stream);
}

int attn_bwd_saved(const void* q, const void* k, const void* v, const void* o, const void* dO,
                   const float* lse, const float* rope_cos, const float* rope_sin,
                   const int32_t* cu_seqlens, int B, int H, int H_kv, int T, int D, float scale,
                   int dtype, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                   const void* saved, size_t saved_bytes, void* stream) {
  const int rc = check_saved(saved, saved_bytes, B, H, H_kv, T, D, dtype, rope_cos);
  if (rc) return rc;
  return bwd_impl(q, k, v, o, dO, lse, rope_cos, rope_sin, cu_seqlens, B, H, H_kv, T, D, scale,
                  dtype, dq, dk, dv, workspace, ws_bytes, saved, stream);
}

}  // extern "C"

namespace {

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dO,
             const float* lse, const float* rope_cos, const float* rope_sin,
             const int32_t* cu_seqlens, int B, int H, int H_kv, int T, int D, float scale,
             int dtype, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
             const void* saved, void* stream) {
  int rc = check_common(q, k, v, rope_cos, rope_sin, cu_seqlens, B, H, H_kv, T, D, scale, dtype,
                        workspace, ws_bytes, 1);
  if (rc) return rc;
  if (!o || !dO || !lse || !dq || !dk || !dv) return ATTN_EINVAL;
  if (!aligned(o, 16) || !aligned(dO, 16) || !aligned(dq, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16) || !aligned(lse, 4))
    return ATTN_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  const WsPlan p = plan(B, H, T, D, dtype, 1, H_kv);
  char* ws = (char*)workspace;
  const char* sv = (dtype == ATTN_BF16 && rope_cos && saved) ? (const char*)saved : nullptr;
  int32_t *ds = nullptr, *de = nullptr;
  if (cu_seqlens && sv) {
    // the forward left them with the saved operands
    ds = (int32_t*)(sv + saved_plan(B, H, H_kv, T, D).docs);
    de = ds + (size_t)B * T;
  } else if (cu_seqlens) {
    ds = (int32_t*)(ws + p.doc_start);
    de = (int32_t*)(ws + p.doc_end);
    ATTN_LAUNCH(KK_DOC_RANGES, st, pdl_launch(doc_ranges_kernel, doc_ranges_blocks(B, T), 1024, 0, st, cu_seqlens, B, T, ds, de));
    if (launch_status()) return ATTN_ECUDA;
  }
  float* delta = (float*)(ws + p.delta);
  if (dtype == ATTN_F32) {
    return D == 64 ? bwd_simt<float, 64>(q, k, v, o, dO, lse, rope_cos, rope_sin, ds, de, delta,
                                         dq, dk, dv, B, H, H_kv, T, scale, st)
                   : bwd_simt<float, 128>(q, k, v, o, dO, lse, rope_cos, rope_sin, ds, de, delta,
                                          dq, dk, dv, B, H, H_kv, T, scale, st);
  }
  return D == 64 ? bwd_tc<64>(q, k, v, o, dO, lse, rope_cos, rope_sin, ds, de, dq, dk, dv, B, H,
                              H_kv, T, scale, ws, p, sv, st)
                 : bwd_tc<128>(q, k, v, o, dO, lse, rope_cos, rope_sin, ds, de, dq, dk, dv, B, H,
                               H_kv, T, scale, ws, p, sv, st);
}

}  // namespace

extern "C" {

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
             const float* lse, const float* rope_cos, const float* rope_sin,
             const int32_t* cu_seqlens, int B, int H, int T, int D, float scale, int dtype,
             void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, void* stream) {
  return attn_bwd_gqa(q, k, v, o, dO, lse, rope_cos, rope_sin, cu_seqlens, B, H, H, T, D, scale,
                      dtype, dq, dk, dv, workspace, ws_bytes, stream);
}

int attn_set_backward_route(int route) {
  if (route < 0 || route > 2) return ATTN_EINVAL;
  g_bwd_route = route;
  return ATTN_OK;
}

int attn_get_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return ATTN_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ECUDA;
  if (v != 0) {
    const int z = 0;
    if (cudaMemcpyToSymbol(g_attn_status, &z, sizeof(int)) != cudaSuccess) return ATTN_ECUDA;
  }
  return v;
}

const char* attn_error_string(int code) {
  switch (code) {
    case ATTN_OK: return "ok";
    case ATTN_EINVAL: return "invalid argument (null pointer, non-positive size, bad dtype or scale)";
    case ATTN_EUNSUPPORTED: return "unsupported size (D must be 64 or 128; indices must fit int32)";
    case ATTN_EALIGN: return "misaligned pointer (tensors and workspace need 16 bytes)";
    case ATTN_EWORKSPACE: return "workspace missing or smaller than attn_workspace_bytes()";
    case ATTN_ECUDA: return "CUDA launch or runtime error";
    case ATTN_EDEVICE_INPUT: return "malformed cu_seqlens detected on the device";
    case ATTN_ETIMEOUT: return "a bounded device-side wait timed out";
    case ATTN_ESCRATCH:
      return "problem needs more scratch than attn_bwd_noalloc's fixed array "
             "(ATTN_NOALLOC_SCRATCH_BYTES)";
    default: return "unknown attn status code";
  }
}

unsigned long long attn_launch_count(void) { return trace::launches(); }

int attn_tile_counts(unsigned long long* fwd_tiles, unsigned long long* bwd_tiles,
                     unsigned long long* dq_tiles) {
  if (!fwd_tiles || !bwd_tiles || !dq_tiles) return ATTN_EINVAL;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ECUDA;
  unsigned long long v[3] = {0, 0, 0};
  if (cudaMemcpyFromSymbol(v, g_attn_tiles, sizeof(v)) != cudaSuccess) return ATTN_ECUDA;
  const unsigned long long z[3] = {0, 0, 0};
  if (cudaMemcpyToSymbol(g_attn_tiles, z, sizeof(z)) != cudaSuccess) return ATTN_ECUDA;
  *fwd_tiles = v[0];
  *bwd_tiles = v[1];
  *dq_tiles = v[2];
  return ATTN_OK;
}

int attn_exp2_selftest(const float* x, float* y, int n, void* stream) {
  if (!x || !y || n < 0) return ATTN_EINVAL;
  if (n == 0) return ATTN_OK;
  exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>(x, y, n);
  return launch_status();
}

int attn_debug_withhold(int what) {
#ifdef ATTN_DEBUG_HOOKS
  if (what < 0 || what > 1) return ATTN_EINVAL;
  return cudaMemcpyToSymbol(g_attn_withhold, &what, sizeof(int)) == cudaSuccess ? ATTN_OK
                                                                              : ATTN_ECUDA;
#else
  (void)what;
  return ATTN_EUNSUPPORTED;
#endif
}

int attn_profile_enable(int on) { return trace::enable(on != 0) == 0 ? ATTN_OK : ATTN_ECUDA; }

int attn_profile_kinds(void) { return KK_COUNT; }

int attn_profile_read(int kind, const char** name, int* launches, double* total_ms) {
  if (kind < 0 || kind >= KK_COUNT || !name || !launches || !total_ms) return ATTN_EINVAL;
  *name = kKernelNames[kind];
  return trace::read(kind, launches, total_ms) == 0 ? ATTN_OK : ATTN_ECUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// attn_decode: one new token per sequence against a key/value cache
// ---------------------------------------------------------------------------
namespace {

// bf16 caches with up to 16 query heads per cached head take a tensor-core
// kernel: with at most kDecodeStreamCtas cached heads the persistent
// streaming one (one CTA per SM over equal spans of all cached tokens;
// workspace: partial slots f32 [slots][16][D], then f32 [slots][16][2] max
// and sum, slots = kDecodeStreamCtas + B*H_kv, and one int32 count per cached
// head); with more, each span would hold several short heads, so the split
// one (cache ranges sized for about sixteen CTAs per SM over the grid, a
// two-deep cp.async pipeline, then a combine launch) measured faster. The
// split kernels (and f32 caches and larger groups: one 64-token chunk per
// CTA) use per (query head, range) the unnormalised partial sum
// (f32 [B*H][n_split][D]), then its max and sum of exponentials
// (f32 [B*H][n_split] each). n_split == 0 marks the persistent kernel.
struct DecodePlan {
  size_t o_part = 0, m_part = 0, l_part = 0, cnt = 0, total = 0;
  int n_split = 0, per_split = 0;
};

bool decode_streams(int H, int H_kv, int dtype) { return dtype == ATTN_BF16 && H / H_kv <= 16; }
constexpr int kDecodeStreamCtas = 148;
constexpr long kDecodePipeCtas = 16 * 148;

DecodePlan decode_plan(int B, int H, int H_kv, int T_max, int D, int dtype) {
  DecodePlan p;
  if (decode_streams(H, H_kv, dtype) && (long)B * H_kv > kDecodeStreamCtas) {
    const long stages = (T_max + kDecodePipeKeys - 1) / kDecodePipeKeys;
    long want = (kDecodePipeCtas + (long)B * H_kv - 1) / ((long)B * H_kv);
    want = want < 1 ? 1 : (want > stages ? stages : want);
    const long per = (stages + want - 1) / want;  // stages per range
    p.per_split = (int)(per * kDecodePipeKeys);
    p.n_split = (int)((stages + per - 1) / per);
  } else if (decode_streams(H, H_kv, dtype)) {
    const size_t slots = (size_t)kDecodeStreamCtas + (size_t)B * H_kv;
    p.o_part = 0;
    p.m_part = round_up(slots * 16 * D * sizeof(float));  // (max, sum) pairs
    p.cnt = p.m_part + round_up(slots * 16 * 2 * sizeof(float));
    p.total = p.cnt + round_up((size_t)B * H_kv * sizeof(int));
    return p;
  }
  p.per_split = kDecodeChunk;
  p.n_split = (T_max + kDecodeChunk - 1) / kDecodeChunk;
  const size_t slots = (size_t)B * H * p.n_split;
  p.o_part = 0;
  p.m_part = round_up(slots * D * sizeof(float));
  p.l_part = p.m_part + round_up(slots * sizeof(float));
  p.total = p.l_part + round_up(slots * sizeof(float));
  return p;
}

bool decode_sizes_ok(int B, int H, int H_kv, int T_max, int D) {
  if (B <= 0 || H <= 0 || H_kv <= 0 || T_max <= 0 || H % H_kv) return false;
  if (D != 64 && D != 128) return false;
  if (H / H_kv > kDecodeMaxGroup) return false;
  if ((int64_t)B * H_kv > 65535) return false;  // grid y
  if ((T_max + kDecodeChunk - 1) / kDecodeChunk > 8192) return false;  // combine weights in shared memory
  return (int64_t)B * H_kv * T_max * D < ((int64_t)1 << 40);
}

template <typename TIO, int D>
int decode_launch(const void* q, const void* k, const void* v, const int32_t* lens,
                  const float* rc, const float* rs, void* o, float* lse, int B, int H, int H_kv,
                  int T_max, float scale, char* ws, const DecodePlan& dp, cudaStream_t st) {
  using L = DecodeLayout<TIO, D>;
  static bool smem_set[64] = {};
  if (!ensure_smem(decode_split_kernel<TIO, D>, L::bytes(kDecodeMaxGroup), smem_set))
    return ATTN_ECUDA;
  float* op = (float*)(ws + dp.o_part);
  float* mp = (float*)(ws + dp.m_part);
  float* lp = (float*)(ws + dp.l_part);
  const int G = H / H_kv;
  if (std::is_same<TIO, __nv_bfloat16>::value && G <= 16 && dp.n_split > 0) {
    // split tensor-core variant (many short heads), then the combine
    static bool pipe_smem_set[64] = {};
    if (!ensure_smem(decode_pipe_kernel<D>, DecodePipeLayout<D>::kBytes, pipe_smem_set))
      return ATTN_ECUDA;
    ATTN_LAUNCH(KK_DECODE, st, pdl_launch(decode_pipe_kernel<D>, dim3(dp.n_split, B * H_kv), kDecodeMmaThreads,
                                          DecodePipeLayout<D>::kBytes, st, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                          (const __nv_bfloat16*)v, lens, rc, rs, op, mp, lp, H, H_kv, T_max,
                                          dp.n_split, dp.per_split, scale * 1.4426950408889634f));
  } else if (std::is_same<TIO, __nv_bfloat16>::value && G <= 16) {
    // persistent streaming tensor-core variant (up to 16 query heads per
    // cached head): one launch, the heads split over CTAs merged by their
    // last CTA
    using SL = DecStreamLayout<D>;
    static bool stream_smem_set[2][64] = {};
    auto kern = G <= 8 ? decode_stream_kernel<D, 1> : decode_stream_kernel<D, 2>;
    if (!ensure_smem(kern, SL::kAlloc, stream_smem_set[G <= 8 ? 0 : 1])) return ATTN_ECUDA;
    CUtensorMap mk, mv;
    if (!make_tile_map(&mk, k, false, D, T_max, B * H_kv, kDecKeys) ||
        !make_tile_map(&mv, v, false, D, T_max, B * H_kv, kDecKeys))
      return ATTN_ECUDA;
    int* cnt = (int*)(ws + dp.cnt);
    if (cudaMemsetAsync(cnt, 0, (size_t)B * H_kv * sizeof(int), st) != cudaSuccess)
      return ATTN_ECUDA;
    ATTN_LAUNCH(KK_DECODE, st, pdl_launch(kern, kDecodeStreamCtas, kDecThreads,
                                          SL::kAlloc, st, mk, mv, (const __nv_bfloat16*)q, lens,
                                          rc, rs, (__nv_bfloat16*)o, lse, op, mp, cnt, B, H,
                                          H_kv, T_max, scale * 1.4426950408889634f));
    return launch_status();
  } else {
    ATTN_LAUNCH(KK_DECODE, st, pdl_launch(decode_split_kernel<TIO, D>, dim3(dp.n_split, B * H_kv), kDecodeThreads,
                                          L::bytes(G), st, (const TIO*)q, (const TIO*)k, (const TIO*)v, lens, rc, rs, op, mp, lp, H,
                                          H_kv, T_max, dp.n_split, dp.per_split, scale * 1.4426950408889634f));
  }
  if (launch_status()) return ATTN_ECUDA;
  ATTN_LAUNCH(KK_DECODE_COMBINE, st, pdl_launch(decode_combine_kernel<TIO, D>, B * H, kDecodeCombineThreads,
                                              dp.n_split * sizeof(float), st, op, mp, lp, lens, (TIO*)o, lse, H, T_max, dp.n_split, dp.per_split));
  return launch_status();
}

}  // namespace

extern "C" size_t attn_decode_workspace_bytes(int B, int H, int H_kv, int T_max, int D,
                                              int dtype) {
  if (!decode_sizes_ok(B, H, H_kv, T_max, D) || (dtype != ATTN_BF16 && dtype != ATTN_F32))
    return 0;
  return decode_plan(B, H, H_kv, T_max, D, dtype).total;
}

extern "C" int attn_decode(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* cache_lens, const float* rope_cos,
                           const float* rope_sin, void* o, float* lse, int B, int H, int H_kv,
                           int T_max, int D, float scale, int dtype, void* workspace,
                           size_t ws_bytes, void* stream) {
  if (!q || !k_cache || !v_cache || !cache_lens || !o || !lse) return ATTN_EINVAL;
  if (dtype != ATTN_BF16 && dtype != ATTN_F32) return ATTN_EINVAL;
  if (B <= 0 || H <= 0 || T_max <= 0 || !isfinite(scale)) return ATTN_EINVAL;
  if (H_kv <= 0 || H % H_kv) return ATTN_EINVAL;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return ATTN_EINVAL;
  if (!decode_sizes_ok(B, H, H_kv, T_max, D)) return ATTN_EUNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(cache_lens, 4) || (rope_cos && !aligned(rope_cos, 16)) ||
      (rope_sin && !aligned(rope_sin, 16)))
    return ATTN_EALIGN;
  const DecodePlan dp = decode_plan(B, H, H_kv, T_max, D, dtype);
  if (!workspace) return ATTN_EWORKSPACE;
  if (!aligned(workspace, 16)) return ATTN_EALIGN;
  if (ws_bytes < dp.total) return ATTN_EWORKSPACE;
  char* ws = (char*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == ATTN_F32)
    return D == 64 ? decode_launch<float, 64>(q, k_cache, v_cache, cache_lens, rope_cos, rope_sin,
                                              o, lse, B, H, H_kv, T_max, scale, ws, dp, st)
                   : decode_launch<float, 128>(q, k_cache, v_cache, cache_lens, rope_cos,
                                               rope_sin, o, lse, B, H, H_kv, T_max, scale, ws, dp,
                                               st);
  return D == 64 ? decode_launch<__nv_bfloat16, 64>(q, k_cache, v_cache, cache_lens, rope_cos,
                                                    rope_sin, o, lse, B, H, H_kv, T_max, scale, ws,
                                                    dp, st)
                 : decode_launch<__nv_bfloat16, 128>(q, k_cache, v_cache, cache_lens, rope_cos,
                                                     rope_sin, o, lse, B, H, H_kv, T_max, scale,
                                                     ws, dp, st);
}

// ---------------------------------------------------------------------------
// attn_bwd_noalloc: the backward for callers that cannot allocate device
// memory. Its scratch is this file-scope device array. In host code the name
// g_noalloc_scratch is only a host-side stand-in for the symbol, never a
// device address: the device address is looked up once per device with
// cudaGetSymbolAddress and that pointer is what the kernels receive.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocBytes = ATTN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_dev_ptr[kNoAllocMaxDevices] = {};
CUcontext g_noalloc_ctx[kNoAllocMaxDevices] = {};

// Scratch layout: Delta (f32 [B*H*T]) at offset 0, then, only when documents
// are packed (cu_seqlens given), the document starts and ends (int32 [B*T]
// each); each part starts on a 256-byte boundary.
struct NoAllocPlan {
  size_t delta, doc_start, doc_end, total;
};

NoAllocPlan noalloc_plan(int B, int H, int T, bool packed) {
  NoAllocPlan p;
  const size_t bt = (size_t)B * T;
  p.delta = 0;
  p.total = round_up(bt * (size_t)H * sizeof(float));
  p.doc_start = p.doc_end = 0;
  if (packed) {
    p.doc_start = p.total;
    p.doc_end = p.doc_start + round_up(bt * sizeof(int32_t));
    p.total = p.doc_end + round_up(bt * sizeof(int32_t));
  }
  return p;
}

// The current context, through the driver entry point the runtime exposes
// (the library links no driver library); null if it cannot be queried.
CUcontext current_context() {
  typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
  static CtxGetCurrentFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (CtxGetCurrentFn)f;
  }
  CUcontext c = nullptr;
  if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}

// Device address of the scratch array on the current device. The lookup is
// done once per device, with that device current, and again whenever the
// device's context has changed since (after a cudaDeviceReset the module is
// loaded anew and the array may sit at a new address).
int noalloc_scratch(char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
    return ATTN_ECUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  CUcontext ctx = current_context();
  if (g_noalloc_dev_ptr[dev] == nullptr || ctx == nullptr || g_noalloc_ctx[dev] != ctx) {
    // (also makes the device's primary context current if none is yet)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return ATTN_ECUDA;
    g_noalloc_dev_ptr[dev] = p;
    g_noalloc_ctx[dev] = current_context();
  }
  *out = (char*)g_noalloc_dev_ptr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const void* dO, const float* lse, const float* rope_cos,
                                const float* rope_sin, const int32_t* cu_seqlens, int B, int H,
                                int T, int D, float scale, int dtype, void* dq, void* dk,
                                void* dv, void* stream) {
  // Host-side checks, as attn_bwd makes them (minus the workspace).
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return ATTN_EINVAL;
  if (dtype != ATTN_BF16 && dtype != ATTN_F32) return ATTN_EINVAL;
  if (B <= 0 || H <= 0 || T <= 0 || !isfinite(scale)) return ATTN_EINVAL;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return ATTN_EINVAL;
  if (!sizes_ok(B, H, T, D)) return ATTN_EUNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dO, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4) || (rope_cos && !aligned(rope_cos, 16)) ||
      (rope_sin && !aligned(rope_sin, 16)) || (cu_seqlens && !aligned(cu_seqlens, 4)))
    return ATTN_EALIGN;
  const NoAllocPlan p = noalloc_plan(B, H, T, cu_seqlens != nullptr);
  if (p.total > kNoAllocBytes) return ATTN_ESCRATCH;

  char* ws = nullptr;
  if (int rc = noalloc_scratch(&ws)) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  int32_t *ds = nullptr, *de = nullptr;
  if (cu_seqlens) {
    // doc_ranges_kernel writes every entry of both arrays.
    ds = (int32_t*)(ws + p.doc_start);
    de = (int32_t*)(ws + p.doc_end);
    ATTN_LAUNCH(KK_DOC_RANGES, st, pdl_launch(doc_ranges_kernel, doc_ranges_blocks(B, T), 1024, 0, st, cu_seqlens, B, T, ds, de));
    if (launch_status()) return ATTN_ECUDA;
  }
  // delta_kernel writes every row of Delta before the two passes read it.
  float* delta = (float*)(ws + p.delta);
  if (dtype == ATTN_F32) {
    return D == 64 ? bwd_simt<float, 64>(q, k, v, o, dO, lse, rope_cos, rope_sin, ds, de, delta,
                                         dq, dk, dv, B, H, H, T, scale, st)
                   : bwd_simt<float, 128>(q, k, v, o, dO, lse, rope_cos, rope_sin, ds, de, delta,
                                          dq, dk, dv, B, H, H, T, scale, st);
  }
  return D == 64 ? bwd_simt<__nv_bfloat16, 64>(q, k, v, o, dO, lse, rope_cos, rope_sin, ds, de,
                                               delta, dq, dk, dv, B, H, H, T, scale, st)
                 : bwd_simt<__nv_bfloat16, 128>(q, k, v, o, dO, lse, rope_cos, rope_sin, ds, de,
                                                delta, dq, dk, dv, B, H, H, T, scale, st);
}

// The projections around the attention (tensor-core GEMMs).
#include "proj_api.cuh"
