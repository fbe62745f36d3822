/*
 * attn.h -- C ABI of libattn.so: causal multi-head scaled-dot-product
 * attention (forward and backward) for NVIDIA B200 (sm_100a).
 *
 * What it computes. For every batch row b and head h, with q_r = R(pos) q and
 * k_r = R(pos) k (RoPE, optional):
 *     S   = scale * q_r k_r^T,  keeping S[i][j] only where j <= i and j is in
 *           i's document; every other entry is -inf
 *     P   = softmax over each row of S;   o = P v
 *     lse = log(sum_j exp(S[i][j]))  (natural log)
 * and the backward of L = sum(o * dO):
 *     Delta_i = sum_d dO[i][d] * o[i][d];  dP = dO v^T;  dS = P * (dP - Delta)
 *     dv = P^T dO;  dq = R(pos)^T (scale * dS k_r);  dk = R(pos)^T (scale * dS^T q_r)
 * Sources, by page and section: ARK README, "Accelerated forward pass (GPU)"
 * (multi-head SDPA with the causal mask fused in) and "Inference architecture
 * (EKO)" (RoPE from precomputed sin/cos tables); ARK README, "Backward pass
 * (AutoGrad)" (gradients of the attention inside training); Forge README,
 * "What this is" (flash attention forward and backward) and "Architecture",
 * Model line (RoPE on interleaved pairs); Cort33x, "Preserving context in the
 * data" (short documents packed into one training window).
 *
 * Conventions shared by every call:
 *   - Tensors q, k, v, o, dO, dq, dk, dv are [B, H, T, D], contiguous, D
 *     fastest, in the storage type `dtype` (ATTN_BF16 or ATTN_F32). lse is
 *     [B, H, T] float32. All are DEVICE pointers on the current CUDA device,
 *     owned by the caller; the library never allocates or frees memory.
 *   - q, k, v, o, dO, dq, dk, dv, the rope tables and the workspace must be
 *     16-byte aligned (the kernels move tiles with TMA and read the tables in
 *     16-byte groups); lse and cu_seqlens must be 4-byte aligned.
 *   - D must be 64 or 128. B, H, T >= 1. B*T and B*H*T*D must fit in int32.
 *   - RoPE: rope_cos and rope_sin are both NULL (no RoPE) or both [T, D/2]
 *     float32 with row p holding cos/sin(p * theta_i) for position p. Pairs
 *     (x[2i], x[2i+1]) of q and k are rotated by the angle of pair i; v is not
 *     rotated. The position of token t is t minus the start of its document.
 *   - Packed documents: cu_seqlens is NULL (each row is one document) or an
 *     int32 device array over the flattened B*T token axis: strictly rising,
 *     starting at 0, containing every row boundary r*T and ending with the
 *     value B*T, which marks its end (the array holds at most B*T+1 entries;
 *     the device reads it up to that end marker and no further). A malformed
 *     array is detected on the device: the call then computes as if
 *     cu_seqlens were NULL and the status word reports ATTN_EDEVICE_INPUT.
 *   - Every call is asynchronous and stream ordered on `stream` (a
 *     cudaStream_t; NULL = the legacy default stream). Host-side validation
 *     errors return before anything is launched.
 *   - The workspace is caller-owned device scratch of at least
 *     attn_workspace_bytes(...) bytes; its contents on entry do not matter
 *     and are undefined on return. Two calls that overlap in time must not
 *     share one workspace.
 *
 * Return codes: ATTN_OK or one of the negative ATTN_E* values below.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* storage types */
#define ATTN_BF16 0
#define ATTN_F32 1

/* return / status codes */
#define ATTN_OK 0
#define ATTN_EINVAL (-1)        /* null pointer, B/H/T <= 0, non-finite scale, bad dtype */
#define ATTN_EUNSUPPORTED (-2)  /* D not 64/128, or sizes beyond the int32 index range */
#define ATTN_EALIGN (-3)        /* a pointer violates the alignment rules above */
#define ATTN_EWORKSPACE (-4)    /* ws_bytes smaller than attn_workspace_bytes(...) */
#define ATTN_ECUDA (-5)         /* a CUDA launch or runtime call failed */
#define ATTN_EDEVICE_INPUT (-6) /* device-detected malformed cu_seqlens */
#define ATTN_ETIMEOUT (-7)      /* a bounded device-side wait gave up */
#define ATTN_ESCRATCH (-8)      /* too large for attn_bwd_noalloc's fixed scratch array */

/*
 * attn_fwd -- forward pass.
 * In:  q, k, v [B,H,T,D] (dtype); rope_cos, rope_sin [T,D/2] f32 or NULL;
 *      cu_seqlens (see above) or NULL; scale (usually 1/sqrt(D)).
 * Out: o [B,H,T,D] (dtype); lse [B,H,T] f32, natural log, saved for attn_bwd.
 * Workspace: attn_workspace_bytes(B,H,T,D,dtype,0) bytes.
 */
int attn_fwd(const void* q, const void* k, const void* v,
             const float* rope_cos, const float* rope_sin,
             const int32_t* cu_seqlens,
             void* o, float* lse,
             int B, int H, int T, int D, float scale,
             int dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_bwd -- backward pass of L = sum(o * dO).
 * In:  q, k, v (the same un-rotated inputs given to attn_fwd), o and lse as
 *      attn_fwd returned them, dO [B,H,T,D] (dtype), the same RoPE tables,
 *      cu_seqlens and scale as the forward.
 * Out: dq, dk, dv [B,H,T,D] (dtype): gradients with respect to the
 *      un-rotated q and k, and v.
 * Workspace: attn_workspace_bytes(B,H,T,D,dtype,1) bytes.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o,
             const void* dO, const float* lse,
             const float* rope_cos, const float* rope_sin,
             const int32_t* cu_seqlens,
             int B, int H, int T, int D, float scale, int dtype,
             void* dq, void* dk, void* dv,
             void* workspace, size_t ws_bytes, void* stream);

/*
 * Grouped-query attention (Forge README, "Architecture", Model line: the
 * attention is GQA with RoPE). k and v have H_kv heads, H_kv dividing H; query
 * head h reads key/value head h / (H / H_kv), and the gradient of a shared
 * key/value head is the sum over the H / H_kv query heads that read it.
 *
 * attn_fwd_gqa / attn_bwd_gqa take the arguments of attn_fwd / attn_bwd plus
 * H_kv (after H) and follow their rules, with these shapes:
 *   q, o, dO, dq [B, H, T, D]; k, v, dk, dv [B, H_kv, T, D]; lse [B, H, T].
 * Workspace: attn_workspace_bytes_gqa(B, H, H_kv, T, D, dtype, is_bwd) bytes.
 * (When the key/value heads times the 128-key tiles are too few to fill the
 * GPU, the bf16 backward splits each group of query heads over several CTAs
 * and needs room for fp32 dk, dv accumulators; the size includes it.)
 * H_kv <= 0 or H not a multiple of H_kv: ATTN_EINVAL. attn_fwd and attn_bwd
 * are these calls with H_kv = H.
 */
int attn_fwd_gqa(const void* q, const void* k, const void* v,
                 const float* rope_cos, const float* rope_sin,
                 const int32_t* cu_seqlens,
                 void* o, float* lse,
                 int B, int H, int H_kv, int T, int D, float scale,
                 int dtype, void* workspace, size_t ws_bytes, void* stream);

int attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                 const void* dO, const float* lse,
                 const float* rope_cos, const float* rope_sin,
                 const int32_t* cu_seqlens,
                 int B, int H, int H_kv, int T, int D, float scale, int dtype,
                 void* dq, void* dk, void* dv,
                 void* workspace, size_t ws_bytes, void* stream);

/* Bytes of workspace attn_fwd (is_bwd = 0) or attn_bwd (is_bwd = 1) needs for
 * these sizes; 0 for invalid sizes. Pure host function, no CUDA call. */
size_t attn_workspace_bytes(int B, int H, int T, int D, int dtype, int is_bwd);

/* The same for attn_fwd_gqa / attn_bwd_gqa (H_kv key/value heads); 0 for
 * invalid sizes, including H_kv not dividing H. Pure host function. */
size_t attn_workspace_bytes_gqa(int B, int H, int H_kv, int T, int D, int dtype, int is_bwd);

/*
 * Keeping the forward's rotated operands for the backward (the saved
 * activations of a training step). With bf16 storage and RoPE tables the
 * forward rotates q and k once (interleaved pairs at document positions,
 * ARK README, "Inference architecture (EKO)"; Forge README, "Architecture")
 * into fp16 tiles with power-of-two tile factors, and the backward recomputes
 * the scores from exactly those operands. attn_fwd_save leaves them in the
 * caller's buffer `saved`; attn_bwd_saved reads them from there instead of
 * rotating q and k again (one pass over q and k fewer per step). With
 * cu_seqlens the per-token document ranges are kept there too, so the
 * backward does not rebuild them.
 *
 * attn_saved_bytes: bytes of that buffer; 0 when there is nothing to keep
 * (dtype ATTN_F32, has_rope = 0, or invalid sizes). Pure host function.
 * attn_fwd_save: attn_fwd_gqa plus `saved` (device, 16-byte aligned,
 * saved_bytes >= attn_saved_bytes(...), written by the call).
 * attn_bwd_saved: attn_bwd_gqa plus `saved` (read only): it must hold what
 * attn_fwd_save wrote for the same q, k, rope tables, cu_seqlens and sizes,
 * unchanged since; results are then identical to attn_bwd_gqa's. That
 * correspondence is the caller's contract and is not checked; the kernels
 * clamp every document range they read from it into its own row, so a buffer
 * that breaks the contract gives wrong results, never an out-of-range access.
 * For both: when attn_saved_bytes is 0, or saved is NULL, the call is the
 * plain attn_fwd_gqa / attn_bwd_gqa and `saved` is not touched. Misaligned
 * saved: ATTN_EALIGN; saved_bytes too small: ATTN_EWORKSPACE. The buffer
 * stays owned by the caller; workspaces are sized as for the plain calls.
 */
size_t attn_saved_bytes(int B, int H, int H_kv, int T, int D, int dtype, int has_rope);

int attn_fwd_save(const void* q, const void* k, const void* v,
                  const float* rope_cos, const float* rope_sin,
                  const int32_t* cu_seqlens,
                  void* o, float* lse,
                  int B, int H, int H_kv, int T, int D, float scale,
                  int dtype, void* workspace, size_t ws_bytes,
                  void* saved, size_t saved_bytes, void* stream);

int attn_bwd_saved(const void* q, const void* k, const void* v, const void* o,
                   const void* dO, const float* lse,
                   const float* rope_cos, const float* rope_sin,
                   const int32_t* cu_seqlens,
                   int B, int H, int H_kv, int T, int D, float scale, int dtype,
                   void* dq, void* dk, void* dv,
                   void* workspace, size_t ws_bytes,
                   const void* saved, size_t saved_bytes, void* stream);

/*
 * attn_decode -- decode attention: one new token per sequence against a
 * key/value cache (Forge README, "Roadmap": a KV cache for generation on the
 * training attention module; ARK README, "Inference architecture (EKO)":
 * RoPE from precomputed tables).
 * In:  q [B, H, D] (dtype): the new token's queries, un-rotated;
 *      k_cache, v_cache [B, H_kv, T_max, D] (dtype): row b holds
 *      cache_lens[b] tokens at positions 0 .. cache_lens[b]-1, the new
 *      token's own key and value included; keys are stored already rotated
 *      by their positions (as attn_fwd rotates k); rows past cache_lens[b]
 *      never affect the result (their values may be anything, NaN
 *      included: a tile load may fetch some of them, and they are masked
 *      and zeroed before use; no byte past the [B, H_kv, T_max, D] arrays is
 *      read);
 *      cache_lens [B] int32 device array, each in [1, T_max] (a value out of
 *      range is clamped into it and the status word reports
 *      ATTN_EDEVICE_INPUT);
 *      rope_cos, rope_sin [T_max, D/2] f32 or NULL: the query is rotated at
 *      position cache_lens[b]-1;
 *      H_kv divides H (query head h reads cache head h / (H / H_kv)), at
 *      most 64 query heads per key/value head; B * H_kv <= 65535.
 * Out: o [B, H, D] (dtype) = softmax_j(scale * q_r . k_j) v_j over the
 *      cached tokens; lse [B, H] f32, natural log.
 * Workspace: attn_decode_workspace_bytes(B, H, H_kv, T_max, D, dtype) bytes;
 *      the call clears what it needs of it on `stream` (no initial contents
 *      are assumed).
 * Alignment, ownership, asynchrony and return codes as for attn_fwd.
 */
int attn_decode(const void* q, const void* k_cache, const void* v_cache,
                const int32_t* cache_lens, const float* rope_cos, const float* rope_sin,
                void* o, float* lse, int B, int H, int H_kv, int T_max, int D, float scale,
                int dtype, void* workspace, size_t ws_bytes, void* stream);

/* Bytes of workspace attn_decode needs; 0 for invalid or unsupported sizes.
 * Pure host function, no CUDA call. */
size_t attn_decode_workspace_bytes(int B, int H, int H_kv, int T_max, int D, int dtype);

/* Synchronises `stream`, then returns and clears the current device's status
 * word: ATTN_OK, ATTN_EDEVICE_INPUT or ATTN_ETIMEOUT (first error recorded
 * since the last call), or ATTN_ECUDA if the synchronisation itself failed. */
int attn_get_status(void* stream);

/* Static, human-readable text for a return or status code. */
const char* attn_error_string(int code);

/*
 * attn_bwd_noalloc -- the backward pass for callers that cannot allocate
 * device memory. (The source pages have no counterpart: this is an
 * integration variant, not part of the method.)
 *
 * Some callers cannot hand the library a workspace: code embedded in a host
 * runtime that has already reserved the whole device for its own memory pool
 * (so a cudaMalloc would fail or fight that pool), or code on a hot path where
 * a cudaMalloc/cudaFree is not allowed because it can synchronise the device
 * and stall every other stream. This entry point takes the same arguments as
 * attn_bwd minus the workspace and calls no allocating function at all: its
 * scratch (the per-row Delta_i and the per-token document ranges) lives in one
 * static device array of ATTN_NOALLOC_SCRATCH_BYTES, which every GPU that
 * loads the library holds until the process exits.
 *
 * It runs the CUDA-core (fp32 arithmetic) backward kernels, for either dtype,
 * and needs 4*B*H*T bytes of scratch, plus 8*B*T more when cu_seqlens is
 * given (each part rounded up to 256); larger problems are rejected with
 * ATTN_ESCRATCH before anything is launched. The first call on each device
 * looks up the array's device address with cudaGetSymbolAddress (no
 * allocation), and so does the first call after that device's context was
 * reset (cudaDeviceReset); make those calls before any stream capture. All calls share the one array and it keeps the previous call's
 * contents; every byte a call reads is written earlier in the same call, so
 * nothing needs clearing, but two calls that overlap on the GPU (on different
 * streams, or from different threads) race on it and must be serialised by the
 * caller. Other arguments, rules and return codes are those of attn_bwd.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (8u << 20)
int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                     const void* dO, const float* lse,
                     const float* rope_cos, const float* rope_sin,
                     const int32_t* cu_seqlens,
                     int B, int H, int T, int D, float scale, int dtype,
                     void* dq, void* dk, void* dv, void* stream);

/*
 * ---- Projections around the attention (tensor-core GEMMs) ----
 *
 * The linear layers on either side of the attention in the pages' training
 * layer: q, k, v = heads of x W_qkv^T (RoPE optionally applied to q and k in
 * the same kernel) and y = o W_o^T, with their backward products dX = dY W and
 * dW = dY^T X (ARK README, "Inference architecture (EKO)" and "Backward pass
 * (AutoGrad)", whose per-layer gradients include dwq, dwk, dwv, dwo; Forge
 * README, "Benchmarks" (the forward X W^T and the two backward products of a
 * linear layer) and "Architecture" (Linear layers, attention with GQA and
 * RoPE on interleaved pairs)). All operands and activations are bf16;
 * accumulation is fp32; weight gradients are written in fp32.
 *
 * Layouts (row-major, contiguous, device pointers owned by the caller, each
 * 16-byte aligned):
 *   x, dx:        [B, T, C] bf16          y, dy:      [B, T, C] bf16
 *   w_qkv:        [(H + 2 H_kv) D, C] bf16: rows of the H query heads, then
 *                 the H_kv key heads, then the H_kv value heads, D per head
 *   dw_qkv:       [(H + 2 H_kv) D, C] float32
 *   q, dq:        [B, H, T, D] bf16       k, v, dk, dv: [B, H_kv, T, D] bf16
 *   o, d_o:       [B, H, T, D] bf16 (feature index h D + d for W_o)
 *   w_o:          [C, H D] bf16           dw_o:       [C, H D] float32
 * Sizes: D is 64 or 128; T a multiple of 128; C a multiple of 8; B, T, C,
 * H, H_kv >= 1; B*T < 2^31. Otherwise ATTN_EUNSUPPORTED (ATTN_EINVAL for a
 * null pointer or H_kv <= 0, ATTN_EALIGN for a misaligned pointer).
 * Every output is overwritten (weight gradients are not accumulated into).
 * Asynchronous on `stream`, like the attention calls.
 *
 * attn_qkv_proj: with rope_cos/rope_sin NULL, q, k, v are the projection;
 * with tables ([T, D/2] float32, as for attn_fwd) q and k are rotated at each
 * token's position in its document (cu_seqlens as for attn_fwd, or NULL), so
 * that attn_fwd is then called without tables. Workspace: needed only when
 * both tables and cu_seqlens are given, attn_proj_workspace_bytes(...) bytes.
 *
 * attn_qkv_proj_bwd: dq, dk, dv are the gradients with respect to the
 * outputs of attn_qkv_proj (with tables: with respect to the rotated q, k;
 * they are rotated back first, in the workspace, which is then required).
 * Writes dx and dw_qkv.
 *
 * attn_out_proj / attn_out_proj_bwd: y = o W_o^T; d_o = dy W_o (written in
 * the attention's layout) and dw_o = dy^T o. No workspace.
 */
size_t attn_proj_workspace_bytes(int B, int T, int H, int H_kv, int D);
/* attn_proj_gemm_plan: how the projection GEMM C[M][N] = sum over K runs
 * (host arithmetic only, no CUDA call): out[0..5] = tile width BN (128 or
 * 256), tiles along M and N, K parts (> 1 only for the fp32 weight gradients,
 * f32_out != 0, whose parts are added into a zeroed output), 64-wide K blocks
 * per part, and persistent CTAs launched (at most one per SM of a B200).
 * Returns ATTN_OK, ATTN_EINVAL (null out, a size <= 0) or ATTN_EUNSUPPORTED. */
int attn_proj_gemm_plan(int M, int N, int K, int f32_out, int* out);
int attn_qkv_proj(const void* x, const void* w_qkv, const float* rope_cos, const float* rope_sin,
                  const int32_t* cu_seqlens, void* q, void* k, void* v, int B, int T, int C,
                  int H, int H_kv, int D, void* workspace, size_t ws_bytes, void* stream);
int attn_qkv_proj_bwd(const void* dq, const void* dk, const void* dv, const void* x,
                      const void* w_qkv, const float* rope_cos, const float* rope_sin,
                      const int32_t* cu_seqlens, void* dx, float* dw_qkv, int B, int T, int C,
                      int H, int H_kv, int D, void* workspace, size_t ws_bytes, void* stream);
int attn_out_proj(const void* o, const void* w_o, void* y, int B, int T, int C, int H, int D,
                  void* stream);
int attn_out_proj_bwd(const void* dy, const void* o, const void* w_o, void* d_o, float* dw_o,
                      int B, int T, int C, int H, int D, void* stream);

/*
 * Tracing aids (the source pages define no counterpart; they support
 * measurement only). Not thread safe: call them from the thread that
 * launches the attention calls.
 *
 * attn_launch_count: number of kernels this library has launched in this
 * process so far (all devices, all streams).
 *
 * attn_profile_enable(1) clears earlier records and starts recording a pair
 * of CUDA events around every kernel the library launches (on the stream of
 * that launch; up to 16384 launches, later ones are counted but not timed);
 * attn_profile_enable(0) stops recording. Returns ATTN_OK or ATTN_ECUDA.
 *
 * attn_profile_read(kind, ...): for kernel kind 0 <= kind < attn_profile_kinds(),
 * waits for the recorded events and stores the kind's name (static string),
 * the number of timed launches and their summed duration in milliseconds.
 * Returns ATTN_OK, ATTN_EINVAL (kind out of range or a null output pointer)
 * or ATTN_ECUDA.
 *
 * attn_tile_counts: the block products the tensor-core forward (fwd_tiles:
 * 128 queries x 64 keys each), key-tile backward (bwd_tiles: 128 x 128) and
 * query-tile dQ pass (dq_tiles: 128 x 128; zero when dQ is formed in the
 * key-tile kernel) executed on the current device since the previous read,
 * counted on the device (one atomic add per CTA; the CUDA-core float32 path
 * is not counted); resets the counters. Block skipping makes each equal to
 * the blocks of its size that hold at least one allowed (query, key) pair.
 * Synchronises the device. Returns ATTN_OK, ATTN_EINVAL (a null pointer) or
 * ATTN_ECUDA.
 */
/* attn_exp2_selftest: y[i] = the forward/backward kernels' software 2^x
 * (FMA-pipe polynomial) of x[i], for 0 <= i < n; x, y device f32 arrays,
 * asynchronous on `stream`. A test hook for checking that routine against
 * CUDA's exp2f. Returns ATTN_OK, ATTN_EINVAL or ATTN_ECUDA. */
int attn_exp2_selftest(const float* x, float* y, int n, void* stream);

/* attn_debug_withhold: watchdog test hook. In a library built with the debug
 * hooks (libattn_debug.so: bounded waits cut to about 10 ms), what = 1 makes
 * every later attn_fwd / attn_fwd_gqa on the tensor-core path withhold the
 * load of its first value tile, so the waits for it run out: the call
 * completes, leaves o and lse undefined and the status word reports
 * ATTN_ETIMEOUT; what = 0 restores normal loads. Synchronous (device-wide).
 * Returns ATTN_OK, ATTN_EINVAL (what not 0 or 1), ATTN_ECUDA, or
 * ATTN_EUNSUPPORTED in a library built without the hooks (libattn.so). */
int attn_debug_withhold(int what);

/* attn_set_backward_route: which tensor-core backward the attn_bwd* calls
 * of this process run (bf16 storage; float32 is unaffected). 0 = the
 * library's default (the key-tile kernel forms dQ by reduce-adds into an fp32
 * accumulator); 1 = the key-tile kernel for dK, dV and the query-tile pass
 * for dQ; 2 = the key-tile kernel on CTA pairs (clusters of two CTAs,
 * tcgen05 products of M = 256 keys issued for both SMs by one thread) for
 * dK, dV at D = 128 (D = 64 takes route 1) and the query-tile pass for dQ.
 * All routes compute the same gradients within the bf16 tolerance. A global
 * setting for tuning and tests: calls already enqueued keep their route.
 * Returns ATTN_OK or ATTN_EINVAL (route not 0, 1 or 2). Host only. */
int attn_set_backward_route(int route);

unsigned long long attn_launch_count(void);
int attn_tile_counts(unsigned long long* fwd_tiles, unsigned long long* bwd_tiles,
                     unsigned long long* dq_tiles);
int attn_profile_enable(int on);
int attn_profile_kinds(void);
int attn_profile_read(int kind, const char** name, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
