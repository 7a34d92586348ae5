/*
 * dsa.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * The path has three stages, each a call below, plus one call that runs all
 * three for a decode step:
 *
 *   1. dsa_indexer_scores  lightning-indexer scores with the causal mask
 *        I[t,s] = sum_h w[t,h] * ReLU(q_I[t,h,:] . k_I[s,:])
 *      ("DeepSeek-V3.2-Exp - Keep top-k positions", Indexer.forward listing,
 *       the fp8_index call and "index_score += mask"; the head sum is the fix
 *       in "[WIP] deepseek v32", mlx-lm PR #512).
 *   2. dsa_topk  keep each query's min(k, valid) highest-scoring positions
 *      (same page, the M^sel formula and "topk(min(index_topk, end_pos))").
 *   3. dsa_sparse_mla  absorbed MLA over only the selected latent rows
 *      ("DeepSeek-V3.2-Exp - Apply sparse mask", MQA decode listing:
 *       scores = q.[kv||pe] * scale, the -inf index mask, softmax, P.kv).
 *
 * Shapes and layouts (all device pointers, row-major, no padding unless said):
 *   H_I = 64 indexer heads, D_I = 128 indexer dim, D_QK = 576 (512 latent ||
 *   64 rope), D_V = 512, H = MLA heads (1..128).
 *   offsets  int32 [B+1], device.  Sequence b owns rows [offsets[b],
 *            offsets[b+1]) of BOTH caches; end_pos_b = offsets[b+1]-offsets[b].
 *            Its T query rows sit at absolute positions end_pos_b - T + t.
 *   kv_rows  number of rows the caches were allocated with (>= offsets[B]);
 *            bounds every cache read.
 *   q_idx    [B,T,64,128] bf16, or e4m3 codes (uint8) when idx_dtype=DSA_E4M3
 *   w        [B,T,64] fp32 per-head weights; for e4m3 the per-(t,h) q scale
 *            is already multiplied in, as the listing does before fp8_index
 *   k_idx    [kv_rows,128] bf16 or e4m3 codes;  k_scale [kv_rows] fp32 (e4m3 only)
 *   scores   fp32, row (b,t) starts at scores + (b*T+t)*ld_scores
 *   indices  int32 [B,T,k], sequence-local positions, ascending, -1 padded
 *   q        [B,T,H,576] bf16 absorbed query;  kv [kv_rows,576] bf16
 *   out      [B,T,H,512] bf16 or fp32;  lse [B,T,H] fp32 natural-log, optional
 *
 * Ownership and errors.  The caller allocates and owns every buffer, the
 * workspace included; the library allocates nothing and keeps no state between
 * calls.  Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 * legacy default stream).  Argument errors are returned before anything is
 * launched.  A launch failure returns DSA_ERR_CUDA.  Problems only the device
 * can see (offsets that break the bounds above, an index outside [0,end_pos),
 * a pipeline wait that ran out of time) are written as a DSA status code into
 * *dev_status (device int32, optional, never cleared by the library) and the
 * affected row is skipped or zeroed; read it after synchronising.
 * Device pointers must be 16-byte aligned.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or enum       */
  DSA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. H > 128)  */
  DSA_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than required   */
  DSA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed         */
  DSA_ERR_TIMEOUT = 5,     /* device: a pipeline wait ran out of time   */
  DSA_ERR_BAD_INDEX = 6,   /* device: an index outside [0, end_pos)     */
  DSA_ERR_BAD_OFFSETS = 7  /* device: offsets exceed kv_rows / ld / T   */
} dsa_status_t;

enum { DSA_BF16 = 0, DSA_E4M3 = 1, DSA_F32 = 2 };

/* Largest k accepted by dsa_topk / dsa_sparse_mla (index_topk = 2048). */
#define DSA_MAX_TOPK 2048
/* Largest MLA head count (the 128 heads of the decode listing). */
#define DSA_MAX_HEADS 128

/* Human-readable name of a status code; never NULL. */
const char* dsa_status_string(int status);

/* ABI version of this library (major*100 + minor). */
int dsa_version(void);

/*
 * Stage 1 -- indexer scores ("Keep top-k positions", Indexer.forward: the
 * fp8_index call over k_cache[:end_pos] and "index_score += mask").
 * Writes, for every row (b,t) and every s < end_pos_b:
 *   scores[(b*T+t)*ld_scores + s] = s <= end_pos_b-T+t
 *       ? sum_h w[b,t,h] * ReLU(q_I[b,t,h,:] . k_I[offsets[b]+s,:]) (* k_scale for e4m3)
 *       : -inf
 * Entries at s >= end_pos_b are not touched.  ld_scores >= max end_pos, a
 * multiple of 4.  Bytes read: the key cache once, q_I and w once.
 */
int dsa_indexer_scores(const void* q_idx, const float* w, const void* k_idx,
                       const float* k_scale, int idx_dtype, const int32_t* offsets,
                       int B, int T, int64_t kv_rows, float* scores, int64_t ld_scores,
                       int32_t* dev_status, void* stream);

/*
 * Stage 2 -- top-k ("Keep top-k positions": topk(min(index_topk, end_pos))
 * and M^sel).  For row (b,t) the valid positions are s < min(end_pos_b,
 * end_pos_b-T+t+1) (the causal prefix); it keeps k_eff = min(k, #valid) of
 * them, ordered by larger score first and then lower position (-0.0 == +0.0),
 * and writes them ascending into indices[(b*T+t)*k ...], then -1 up to k.
 * Deterministic: the same scores always give the same indices.  1 <= k <= 2048.
 */
int dsa_topk(const float* scores, int64_t ld_scores, const int32_t* offsets, int B, int T,
             int k, int32_t* indices, int32_t* dev_status, void* stream);

/*
 * Stage 3 -- sparse absorbed MLA ("Apply sparse mask", MQA decode listing).
 * For each row r=(b,t), head h, the selected positions j (indices >= 0):
 *   l_j = scale * q[r,h,:576] . kv[offsets[b]+j, :576];  p = softmax_j(l)
 *   out[r,h,:] = sum_j p_j * kv[offsets[b]+j, :512];  lse[r,h] = log sum_j exp(l_j)
 * Rows with no selected position get out = 0, lse = -inf.  Indices outside
 * [0,end_pos_b) are treated as empty and reported as DSA_ERR_BAD_INDEX.
 * workspace: dsa_sparse_mla_workspace_size(B,T,H,k) bytes (may be 0 -> NULL ok).
 */
size_t dsa_sparse_mla_workspace_size(int B, int T, int H, int k);
int dsa_sparse_mla(const void* q, const void* kv, const int32_t* offsets, const int32_t* indices,
                   int B, int T, int H, int k, float scale, int64_t kv_rows, void* out,
                   int out_dtype, float* lse, void* workspace, size_t ws_bytes,
                   int32_t* dev_status, void* stream);

/*
 * The whole decode step (T = 1): stages 1 -> 2 -> 3 on `stream`, scores and
 * indices kept in the workspace.  max_end_pos bounds every end_pos_b (it sets
 * the workspace's score pitch).  Same layouts as above with T = 1.  When
 * max_end_pos <= k every sequence keeps all of its positions, so stages 1 and
 * 2 are skipped (the workspace's scores and indices are then not written) and
 * stage 3 attends to each whole cache.
 * workspace: dsa_decode_step_workspace_size(B, max_end_pos, k, H) bytes.
 */
size_t dsa_decode_step_workspace_size(int B, int max_end_pos, int k, int H);
/*
 * Kernels one dsa_decode_step call launches for these sizes (the indexer and
 * the selection are skipped when max_end_pos <= k: every position is then
 * kept whatever the scores, as the MLX port does below the top-k size).
 * -1 for invalid sizes.  Useful to budget CUDA-graph nodes.
 */
int dsa_decode_step_launches(int B, int max_end_pos, int k, int H);
int dsa_decode_step(const void* q_idx, const float* w, const void* k_idx, const float* k_scale,
                    int idx_dtype, const void* q, const void* kv, const int32_t* offsets, int B,
                    int max_end_pos, int64_t kv_rows, int k, int H, float scale, void* out,
                    int out_dtype, float* lse, void* workspace, size_t ws_bytes,
                    int32_t* dev_status, void* stream);

/*
 * Cache write of the newest tokens ("Keep top-k positions", Indexer.forward:
 * k_cache[start:end] = k after act_quant; the latent cache write of the MLA
 * listing).  For every sequence b and new token t < T, the row
 * offsets[b+1] - T + t (the sequence's last T rows) of each cache gets:
 *   kv_cache  <- kv_new[b,t,:576] (bf16 copy)                 if kv_new != NULL
 *   k_idx_cache <- k_new[b,t,:128]                            if k_new  != NULL
 *     bf16 (idx_dtype DSA_BF16): copied;
 *     e4m3 (DSA_E4M3): act_quant of the 128-vector -- scale = amax/448 in fp32
 *     (1 when amax = 0), codes = nearest e4m3 of x/scale (ties to even,
 *     saturating), the scale stored in k_scale_cache[row].
 * k_new [B,T,128] bf16, kv_new [B,T,576] bf16 (device, 16-byte aligned).
 * Offsets that break the bounds are reported in *dev_status and skipped.
 */
int dsa_cache_append(const void* k_new, const void* kv_new, const int32_t* offsets, int B, int T,
                     int idx_dtype, void* k_idx_cache, float* k_scale_cache, void* kv_cache,
                     int64_t kv_rows, int32_t* dev_status, void* stream);

/*
 * Indexer pre-stage ("Keep top-k positions", Indexer.forward, before
 * act_quant): for every 128-vector x[r, v, :] (bf16; r < n_rows, v <
 * vec_per_row -- the 64 heads of a query row, or one key per row)
 *   1. rotary embedding of the rope part, entries 0..63, not interleaved:
 *      entry i < 32 pairs with entry i + 32 and (a, b) becomes
 *      (a*cos - b*sin, a*sin + b*cos), cos/sin = rope_cos/rope_sin[pos[r], i]
 *      (the freqs_cis table, [rope_len, 32] fp32, row-major); the result is
 *      rounded to bf16;
 *   2. rotate_activation: the Walsh-Hadamard transform of the 128 entries in
 *      Sylvester order, scaled by 128^-1/2, rounded to bf16 into y[r, v, :].
 * y may equal x.  x, y, rope_cos, rope_sin 16-byte aligned (device).  A
 * position outside [0, rope_len) leaves that row's vectors untouched and is
 * reported in *dev_status as DSA_ERR_BAD_INDEX.
 */
int dsa_indexer_prestage(const void* x, const int32_t* pos, int n_rows, int vec_per_row, const float* rope_cos,
                         const float* rope_sin, int rope_len, void* y, int32_t* dev_status, void* stream);

/*
 * act_quant of the indexer queries for the e4m3 path (Indexer.forward:
 * q_fp8, q_scale = act_quant(q) and weights * q_scale): for every row and
 * head the 128-vector q_idx[row,h,:] (bf16) becomes e4m3 codes
 * q_idx_e4m3[row,h,:] with the rule of dsa_cache_append, and
 * w_out[row,h] = w[row,h] * scale (fp32).  n_rows = B*T.
 */
int dsa_quantize_queries(const void* q_idx, const float* w, int n_rows, void* q_idx_e4m3, float* w_out,
                         void* stream);

/*
 * Host <-> device copies done by a kernel (not a copy engine), so that a step
 * fed from host buffers stays one chain of kernel launches on `stream`.
 * dsa_copy_host_to_device: dst (device) <- src_host; dsa_copy_device_to_host:
 * dst_host <- src (device).  The host buffer must be page-locked and mapped
 * into the device's address space as one allocation (cudaHostAlloc, or
 * torch's pin_memory); this is checked at both ends of the range and anything
 * else returns DSA_ERR_INVALID_ARG, as do null pointers, pointers not 16-byte
 * aligned and sizes that are not a multiple of 16.  bytes = 0 does nothing.
 * The copy waits for the previous kernel in the stream; the host may read
 * dst_host once the stream has been synchronised.  The caller keeps
 * ownership of both buffers.
 */
int dsa_copy_host_to_device(void* dst, const void* src_host, size_t bytes, void* stream);
int dsa_copy_device_to_host(void* dst_host, const void* src, size_t bytes, void* stream);

/*
 * Stage 3 without a caller workspace.  The paper has no counterpart: this is
 * a convenience of this library, not a step of the method.
 *
 * For callers that cannot allocate device memory where they issue the step
 * (a plugin inside a runtime that owns all device memory and offers no
 * allocator, a serving loop whose memory is fixed at start-up, code that may
 * not call cudaMalloc on that path).  Same arguments, layouts and results as
 * dsa_sparse_mla, minus the workspace: the split partials live in a scratch
 * array of DSA_NOALLOC_SCRATCH_BYTES (32 MiB) built into the library, which
 * every GPU that loads the library holds until the process exits.
 *   - A call that needs more scratch than that (dsa_sparse_mla_workspace_size
 *     above the limit; e.g. 128..147 rows at H = 128, k = 2048) returns
 *     DSA_ERR_WORKSPACE before launching anything.
 *   - The first call on each device looks the scratch address up with
 *     cudaGetSymbolAddress (with that device current); make that first call
 *     before any stream capture.  It allocates nothing, ever.
 *   - All calls on a device share the one scratch array: calls that may run
 *     concurrently on the GPU (different streams, no ordering between them)
 *     race and corrupt each other's results.  Order them on one stream.
 *   - Nothing in the scratch needs to start at zero: every value a call reads
 *     was written earlier in the same call.
 */
#define DSA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int dsa_sparse_mla_noalloc(const void* q, const void* kv, const int32_t* offsets,
                           const int32_t* indices, int B, int T, int H, int k, float scale,
                           int64_t kv_rows, void* out, int out_dtype, float* lse,
                           int32_t* dev_status, void* stream);

/*
 * Test hook for the device-side timeout path.  The paper has no counterpart:
 * it exists so that a test can make a pipeline wait run out on purpose
 * without faulting or hanging the GPU.
 *
 * The next n_launches attention-stage launches in this process (from
 * dsa_sparse_mla, dsa_decode_step or dsa_sparse_mla_noalloc) initialise their
 * query barrier with one expected arrival more than will ever come, and limit
 * every pipeline wait to wait_limit_ns (1 ms to 1 s).  The wait runs out; the
 * kernel stops its pipeline, waits (bounded) for its own copies and tensor
 * core work, releases its tensor memory and writes DSA_ERR_TIMEOUT into
 * *dev_status.  The output of such a launch is undefined; the launches after
 * it run normally.  n_launches = 0 cancels.  Returns DSA_ERR_INVALID_ARG for
 * a negative count or a limit outside the range.  Launches captured in a
 * CUDA graph keep the setting they were captured with.
 */
int dsa_debug_stall_attention(int n_launches, uint64_t wait_limit_ns);

/*
 * Where, inside a decode-step workspace, the step leaves its intermediates
 * (byte offsets; the scores pitch is returned in *ld_scores).  For tests and
 * tools that want to look at stage outputs; the layout may change between
 * versions.
 */
int dsa_decode_step_workspace_layout(int B, int max_end_pos, int k, int H, size_t* scores_off,
                                     int64_t* ld_scores, size_t* indices_off, size_t* mla_off);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
