// proj_api.cuh -- host side of the projection GEMMs (included at the end of
// attn_api.cu, whose helpers it uses): operand maps, tile and split choice,
// and the four projection entry points of include/attn.h.
#pragma once

#include <algorithm>

#include "proj_sm100.cuh"

namespace {

// A row-major bf16 matrix [rows][cols] seen in boxes of box_rows x 64 columns
// (128-byte swizzle); boxes past the edges read zeros.
bool make_rows_map(CUtensorMap* m, const void* base, long rows, long cols, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A head-major bf16 tensor [BH][T][D] in boxes of box_t tokens x 64 features.
bool make_heads_map(CUtensorMap* m, const void* base, int D, int T, long BH, int box_t) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_t, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__global__ void __launch_bounds__(256) fill_zero_kernel(float4* __restrict__ p, long n4) {
  pdl_wait_and_trigger();
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long)gridDim.x * blockDim.x)
    p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

constexpr int kProjSms = 148;

// Tile width and K split of one GEMM. fp32 outputs may split K over work
// units; the split is chosen by a small cost model in microseconds: rounds of
// persistent CTAs times the K blocks of one unit (at the per-SM share of the
// measured bf16 tensor rate, about 11 TFLOP/s) plus a pipeline fill per
// round, plus, for a split, zeroing the output and one more fp32 reduce of it
// per part (at ~2.5 TB/s of L2 reductions, half of which overlaps the main
// loops).
struct GemmPlan {
  int bn, tiles_m, tiles_n, splits, kb_per_split;
  long units, ctas;
};
// The K blocks per split are even: the kernel's ring stages hold two.
GemmPlan plan_gemm(int M, int N, int K, bool f32_out) {
  using namespace proj100;
  GemmPlan g;
  g.bn = N >= 256 ? 256 : 128;
  g.tiles_m = (M + kBM - 1) / kBM;
  g.tiles_n = (N + g.bn - 1) / g.bn;
  const int nkb = (K + kBK - 1) / kBK;
  auto per_of = [&](int s) {
    const int per = (nkb + s - 1) / s;
    return per + (per & 1);
  };
  auto rounded = [&](int s) {
    const int per = per_of(s);
    return (nkb + per - 1) / per;  // every split gets >= 1 block
  };
  auto cost_us = [&](int s) {
    const int sr = rounded(s), per = per_of(s);
    const long units = (long)g.tiles_m * g.tiles_n * sr;
    const long rounds = (units + kProjSms - 1) / kProjSms;
    const double kb_us = 2.0 * kBM * g.bn * kBK / 11.2e6;
    const double out_mb = (double)M * N * 4 / 1e6;
    double t = rounds * (per * kb_us + 1.0);
    if (sr > 1) t += out_mb / 6.0 + 0.5 * sr * out_mb / 2.5;  // MB at MB/us
    return t;
  };
  int split = 1;
  if (f32_out) {
    double best = cost_us(1);
    for (int s = 2; s <= 32 && nkb / s >= 4; ++s) {
      const double c = cost_us(s);
      if (c < best) {
        best = c;
        split = s;
      }
    }
  }
  g.splits = rounded(split);
  g.kb_per_split = per_of(split);
  g.units = (long)g.tiles_m * g.tiles_n * g.splits;
  g.ctas = std::min<long>(g.units, kProjSms);  // persistent: at most one CTA per SM
  return g;
}

// Rows of a K-major B operand's TMA box for an N-column product: 256-wide
// tiles run on CTA pairs (a 256 x 256 tile per pair), each CTA loading half
// of the B tile, so every box is 128 rows high.
int gemm_b_box_rows(int) { return 128; }

// TMA box rows of an MN-major operand: its K extent per ring stage.
constexpr int kMnBoxRows = 128;

template <int BN, bool kPair, int KB>
int gemm_kernel_launch(dim3 grid, const CUtensorMap& a0, const CUtensorMap& a1,
                       const CUtensorMap& a2, const CUtensorMap& b, const proj100::Params& p,
                       cudaStream_t st) {
  using namespace proj100;
  using L = Layout<BN, kPair, KB>;
  static bool smem_done[64];
  if (!ensure_smem(gemm_kernel<BN, kPair, KB>, L::kSmemAlloc, smem_done)) return ATTN_ECUDA;
  if (kPair)
    ATTN_LAUNCH(KK_GEMM, st, pdl_cluster_launch(gemm_kernel<BN, kPair, KB>, grid, L::kThreads,
                                                L::kSmemAlloc, st, 2u, a0, a1, a2, b, p));
  else
    ATTN_LAUNCH(KK_GEMM, st, pdl_launch(gemm_kernel<BN, kPair, KB>, grid, L::kThreads,
                                        L::kSmemAlloc, st, a0, a1, a2, b, p));
  return launch_status();
}

// One GEMM launch: the operands' maps are built by the caller (an MN-major
// operand's boxes kMnBoxRows high). With a K split the fp32 output is zeroed
// first and the parts are added into it.
int gemm_launch(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2,
                const CUtensorMap& b, proj100::Params p, cudaStream_t st) {
  using namespace proj100;
  const GemmPlan g = plan_gemm(p.M, p.N, p.K, p.epi == EPI_ROWS_F32);
  if (g.units >= (1L << 31)) return ATTN_EUNSUPPORTED;
  p.tiles_m = g.tiles_m;
  p.tiles_n = g.tiles_n;
  p.splits = g.splits;
  p.kb_per_split = g.kb_per_split;
  p.reduce = g.splits > 1;
  if (p.reduce) {
    const long n4 = (long)p.M * p.N / 4;
    ATTN_LAUNCH(KK_FILL, st, pdl_launch(fill_zero_kernel, (unsigned)std::min<long>((n4 + 255) / 256, 4L * kProjSms),
                                        256, 0, st, (float4*)p.out[0], n4));
  }
  const dim3 grid((unsigned)g.ctas);
  if (g.bn == 256) {
    // measured on the two projection workloads: 15 % and 6 % faster than
    // one CTA per 128 x 256 tile (the per-SM tile loads halve for B)
    p.tiles_m = (p.M + 2 * kBM - 1) / (2 * kBM);  // 256-row tiles, one per pair
    const long units = (long)p.tiles_m * p.tiles_n * p.splits;
    const dim3 pgrid((unsigned)(2 * std::min<long>(units, kProjSms / 2)));
    return gemm_kernel_launch<256, true, 128>(pgrid, a0, a1, a2, b, p, st);
  }
  return gemm_kernel_launch<128, false, 128>(grid, a0, a1, a2, b, p, st);
}

struct ProjWs {
  size_t doc_start = 0, doc_end = 0, gq = 0, gk = 0, total = 0;
};
ProjWs proj_plan(int B, int T, int H, int H_kv, int D) {
  ProjWs w;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = round_up(off + bytes);
    return at;
  };
  const size_t bt = (size_t)B * T;
  w.doc_start = take(bt * 4);
  w.doc_end = take(bt * 4);
  w.gq = take(bt * H * D * 2);
  w.gk = take(bt * H_kv * D * 2);
  w.total = off;
  return w;
}

bool proj_sizes_ok(int B, int T, int C, int H, int H_kv, int D) {
  if (B <= 0 || T <= 0 || C <= 0 || H <= 0 || H_kv < 0) return false;
  if (D != 64 && D != 128) return false;
  if (T % 128 != 0 || C % 8 != 0) return false;
  const long bt = (long)B * T, feats = (long)(H + 2L * H_kv) * D;
  return bt < (1L << 31) && feats < (1L << 31) && bt * std::max<long>(C, feats) < (1L << 40);
}

int doc_positions(const int32_t* cu, int B, int T, char* ws, const ProjWs& w, cudaStream_t st,
                  const int32_t** ds) {
  *ds = nullptr;
  if (!cu) return ATTN_OK;
  int32_t* s = (int32_t*)(ws + w.doc_start);
  ATTN_LAUNCH(KK_DOC_RANGES, st, pdl_launch(doc_ranges_kernel, doc_ranges_blocks(B, T), 1024, 0, st, cu, B, T, s,
                                            (int32_t*)(ws + w.doc_end)));
  *ds = s;
  return launch_status();
}

proj100::Params base_params(int M, int N, int K, int T, int D) {
  proj100::Params p = {};
  p.M = M;
  p.N = N;
  p.K = K;
  p.T = T;
  p.D = D;
  return p;
}

}  // namespace

extern "C" {

int attn_proj_gemm_plan(int M, int N, int K, int f32_out, int* out) {
  if (!out || M <= 0 || N <= 0 || K <= 0) return ATTN_EINVAL;
  const GemmPlan g = plan_gemm(M, N, K, f32_out != 0);
  if (g.units >= (1L << 31)) return ATTN_EUNSUPPORTED;
  out[0] = g.bn;
  out[1] = g.tiles_m;
  out[2] = g.tiles_n;
  out[3] = g.splits;
  out[4] = g.kb_per_split;
  out[5] = (int)g.ctas;
  return ATTN_OK;
}

size_t attn_proj_workspace_bytes(int B, int T, int H, int H_kv, int D) {
  if (!proj_sizes_ok(B, T, 8, H, H_kv, D)) return 0;
  return proj_plan(B, T, H, H_kv, D).total;
}

int attn_qkv_proj(const void* x, const void* w_qkv, const float* rope_cos, const float* rope_sin,
                  const int32_t* cu_seqlens, void* q, void* k, void* v, int B, int T, int C,
                  int H, int H_kv, int D, void* workspace, size_t ws_bytes, void* stream) {
  using namespace proj100;
  if (!x || !w_qkv || !q || !k || !v || H_kv <= 0) return ATTN_EINVAL;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return ATTN_EINVAL;
  if (!proj_sizes_ok(B, T, C, H, H_kv, D)) return ATTN_EUNSUPPORTED;
  if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(q, 16) || !aligned(k, 16) ||
      !aligned(v, 16) || (rope_cos && (!aligned(rope_cos, 16) || !aligned(rope_sin, 16))) ||
      (cu_seqlens && !aligned(cu_seqlens, 4)))
    return ATTN_EALIGN;
  const ProjWs w = proj_plan(B, T, H, H_kv, D);
  const bool need_ws = cu_seqlens && rope_cos;
  if (need_ws && (!workspace || ws_bytes < w.total)) return ATTN_EWORKSPACE;
  if (need_ws && !aligned(workspace, 16)) return ATTN_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  const int F = (H + 2 * H_kv) * D;
  CUtensorMap ma, mb;
  if (!make_rows_map(&ma, x, (long)B * T, C, kBM) ||
      !make_rows_map(&mb, w_qkv, F, C, gemm_b_box_rows(F)))
    return ATTN_ECUDA;
  Params p = base_params(B * T, F, C, T, D);
  p.a = {SRC_ROWS, 0, {0, 0, 0}};
  p.b = {SRC_ROWS, 0, {0, 0, 0}};
  p.epi = EPI_HEADS;
  p.out_heads[0] = H;
  p.out_heads[1] = H_kv;
  p.out_heads[2] = H_kv;
  p.out[0] = q;
  p.out[1] = k;
  p.out[2] = v;
  if (rope_cos) {
    p.rope_segs = 2;
    p.rope_cos = rope_cos;
    p.rope_sin = rope_sin;
    if (int rc = doc_positions(need_ws ? cu_seqlens : nullptr, B, T, (char*)workspace, w, st,
                               &p.doc_start))
      return rc;
  }
  return gemm_launch(ma, ma, ma, mb, p, st);
}

int attn_qkv_proj_bwd(const void* dq, const void* dk, const void* dv, const void* x,
                      const void* w_qkv, const float* rope_cos, const float* rope_sin,
                      const int32_t* cu_seqlens, void* dx, float* dw_qkv, int B, int T, int C,
                      int H, int H_kv, int D, void* workspace, size_t ws_bytes, void* stream) {
  using namespace proj100;
  if (!dq || !dk || !dv || !x || !w_qkv || !dx || !dw_qkv || H_kv <= 0) return ATTN_EINVAL;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return ATTN_EINVAL;
  if (!proj_sizes_ok(B, T, C, H, H_kv, D)) return ATTN_EUNSUPPORTED;
  if (!aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(x, 16) ||
      !aligned(w_qkv, 16) || !aligned(dx, 16) || !aligned(dw_qkv, 16) ||
      (rope_cos && (!aligned(rope_cos, 16) || !aligned(rope_sin, 16))) ||
      (cu_seqlens && !aligned(cu_seqlens, 4)))
    return ATTN_EALIGN;
  const ProjWs w = proj_plan(B, T, H, H_kv, D);
  if (rope_cos && (!workspace || ws_bytes < w.total)) return ATTN_EWORKSPACE;
  if (rope_cos && !aligned(workspace, 16)) return ATTN_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  const void* gq = dq;
  const void* gk = dk;
  if (rope_cos) {
    // gradients with respect to the rotated q, k -> the un-rotated projection
    const int32_t* ds = nullptr;
    if (int rc = doc_positions(cu_seqlens, B, T, ws, w, st, &ds)) return rc;
    const long nq8 = (long)B * H * T * D / 8, nk8 = (long)B * H_kv * T * D / 8;
    auto launch_rg = [&](const void* g, void* dst, int heads, long n8) {
      if (D == 64)
        ATTN_LAUNCH(KK_ROPE_GRAD, st, pdl_launch(rope_grad_kernel<64>, (unsigned)((n8 + 255) / 256), 256, 0, st,
                                                 (const __nv_bfloat16*)g, rope_cos, rope_sin, ds,
                                                 (__nv_bfloat16*)dst, heads, T, n8));
      else
        ATTN_LAUNCH(KK_ROPE_GRAD, st, pdl_launch(rope_grad_kernel<128>, (unsigned)((n8 + 255) / 256), 256, 0, st,
                                                 (const __nv_bfloat16*)g, rope_cos, rope_sin, ds,
                                                 (__nv_bfloat16*)dst, heads, T, n8));
    };
    launch_rg(dq, ws + w.gq, H, nq8);
    launch_rg(dk, ws + w.gk, H_kv, nk8);
    if (launch_status()) return ATTN_ECUDA;
    gq = ws + w.gq;
    gk = ws + w.gk;
  }
  const int F = (H + 2 * H_kv) * D;
  const long BT = (long)B * T;
  // dx = dY W_qkv: A = the gradients K-major (tokens x features), B = W_qkv
  // read MN-major ([F][C]: C contiguous)
  {
    CUtensorMap a0, a1, a2, mb;
    if (!make_heads_map(&a0, gq, D, T, (long)B * H, kBM) ||
        !make_heads_map(&a1, gk, D, T, (long)B * H_kv, kBM) ||
        !make_heads_map(&a2, dv, D, T, (long)B * H_kv, kBM) ||
        !make_rows_map(&mb, w_qkv, F, C, kMnBoxRows))
      return ATTN_ECUDA;
    Params p = base_params((int)BT, C, F, T, D);
    p.a = {SRC_HEADS, 0, {H, H_kv, H_kv}};
    p.b = {SRC_ROWS, 1, {0, 0, 0}};
    p.epi = EPI_ROWS_BF16;
    p.out[0] = dx;
    if (int rc = gemm_launch(a0, a1, a2, mb, p, st)) return rc;
  }
  // dW_qkv = dY^T x: A = the gradients MN-major (features contiguous within a
  // head, tokens along K), B = x read MN-major ([BT][C])
  {
    CUtensorMap a0, a1, a2, mb;
    if (!make_heads_map(&a0, gq, D, T, (long)B * H, kMnBoxRows) ||
        !make_heads_map(&a1, gk, D, T, (long)B * H_kv, kMnBoxRows) ||
        !make_heads_map(&a2, dv, D, T, (long)B * H_kv, kMnBoxRows) ||
        !make_rows_map(&mb, x, BT, C, kMnBoxRows))
      return ATTN_ECUDA;
    Params p = base_params(F, C, (int)BT, T, D);
    p.a = {SRC_HEADS, 1, {H, H_kv, H_kv}};
    p.b = {SRC_ROWS, 1, {0, 0, 0}};
    p.epi = EPI_ROWS_F32;
    p.out[0] = dw_qkv;
    if (int rc = gemm_launch(a0, a1, a2, mb, p, st)) return rc;
  }
  return ATTN_OK;
}

int attn_out_proj(const void* o, const void* w_o, void* y, int B, int T, int C, int H, int D,
                  void* stream) {
  using namespace proj100;
  if (!o || !w_o || !y) return ATTN_EINVAL;
  if (!proj_sizes_ok(B, T, C, H, 0, D)) return ATTN_EUNSUPPORTED;
  if (!aligned(o, 16) || !aligned(w_o, 16) || !aligned(y, 16)) return ATTN_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  CUtensorMap ma, mb;
  if (!make_heads_map(&ma, o, D, T, (long)B * H, kBM) ||
      !make_rows_map(&mb, w_o, C, (long)H * D, gemm_b_box_rows(C)))
    return ATTN_ECUDA;
  Params p = base_params(B * T, C, H * D, T, D);
  p.a = {SRC_HEADS, 0, {H, 0, 0}};
  p.b = {SRC_ROWS, 0, {0, 0, 0}};
  p.epi = EPI_ROWS_BF16;
  p.out[0] = y;
  return gemm_launch(ma, ma, ma, mb, p, st);
}

int attn_out_proj_bwd(const void* dy, const void* o, const void* w_o, void* d_o, float* dw_o,
                      int B, int T, int C, int H, int D, void* stream) {
  using namespace proj100;
  if (!dy || !o || !w_o || !d_o || !dw_o) return ATTN_EINVAL;
  if (!proj_sizes_ok(B, T, C, H, 0, D)) return ATTN_EUNSUPPORTED;
  if (!aligned(dy, 16) || !aligned(o, 16) || !aligned(w_o, 16) || !aligned(d_o, 16) ||
      !aligned(dw_o, 16))
    return ATTN_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  const long BT = (long)B * T;
  const int HD = H * D;
  // d_o = dy W_o: A = dy K-major, B = W_o read MN-major ([C][HD]: HD contiguous)
  {
    CUtensorMap ma, mb;
    if (!make_rows_map(&ma, dy, BT, C, kBM) || !make_rows_map(&mb, w_o, C, HD, kMnBoxRows))
      return ATTN_ECUDA;
    Params p = base_params((int)BT, HD, C, T, D);
    p.a = {SRC_ROWS, 0, {0, 0, 0}};
    p.b = {SRC_ROWS, 1, {0, 0, 0}};
    p.epi = EPI_HEADS;
    p.out_heads[0] = H;
    p.out[0] = d_o;
    if (int rc = gemm_launch(ma, ma, ma, mb, p, st)) return rc;
  }
  // dW_o = dy^T o: A = dy read MN-major ([BT][C]), B = o read MN-major
  {
    CUtensorMap ma, mb;
    if (!make_rows_map(&ma, dy, BT, C, kMnBoxRows) ||
        !make_heads_map(&mb, o, D, T, (long)B * H, kMnBoxRows))
      return ATTN_ECUDA;
    Params p = base_params(C, HD, (int)BT, T, D);
    p.a = {SRC_ROWS, 1, {0, 0, 0}};
    p.b = {SRC_HEADS, 1, {H, 0, 0}};
    p.epi = EPI_ROWS_F32;
    p.out[0] = dw_o;
    if (int rc = gemm_launch(ma, ma, ma, mb, p, st)) return rc;
  }
  return ATTN_OK;
}

}  // extern "C"
