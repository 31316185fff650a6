/*
 * sga.h - C ABI of libsga, the B200 (sm_100a) hot path of Sparse Gated
 * Attention (SGA), the attention of the A.X K2 model.
 *
 * For each query the path scores every causal past position with a DSA-style
 * indexer, keeps the top K (= 2048) positions, runs MLA-style attention in the
 * latent form (64 heads sharing one 576-wide latent row per token; the first
 * 512 dims are the value) over only those positions, and multiplies each
 * head's output by a sigmoid gate.  Sources:
 *   - archdb "A.X K2", token-selection field: DSA-style indexer, top-2048
 *     tokens per query, 64 indexer heads of dim 128, ReLU-scored;
 *     indexer-key-width field: 128 per token.
 *   - archdb "A.X K2", attention fields: 64 query heads, qk head dim 192
 *     (128 nope + 64 rope), v head dim 128, KV latent 512, shared rope key 64.
 *   - archdb "A.X K2", gate field: head-specific sigmoid gate on the attention
 *     output before o_proj.
 *   - arXiv abstract "A.X K2 Technical Report": each query reads only 2,048
 *     positions.
 * The indexer score is the DSA-style reading
 *     score(t,s) = sum_j w[t,j] * max(0, q_idx[t,j,:] . k_idx[s,:]),
 * since the pages name the parts but print no formula.
 *
 * Conventions shared by every call
 *   - All tensors are dense, row-major, innermost dimension contiguous, and live
 *     in device memory owned by the caller.  bf16 tensors are passed as their
 *     16-bit patterns (sga_bf16_t).  Pointers to bf16 inputs must be 16-byte
 *     aligned (they are read by the Tensor Memory Accelerator).
 *   - B = dims.batch sequences, T = dims.n_q queries per sequence,
 *     L = dims.kv_stride cache rows per sequence, K = dims.top_k.
 *     q_pos[b*T + i] is the absolute position t of query i of sequence b;
 *     positions 0..t are its candidates, so 0 <= t < L is required.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream), allocates nothing, and does not synchronise.
 *   - The return value reports host-side validation and launch errors only.
 *     Errors found on the device (a position or index out of range, a
 *     bounded wait that ran out) are written to a status word at the start of
 *     the workspace; read it with sga_get_device_status.  The first device
 *     error is kept until sga_clear_device_status.
 *   - Workspace: caller-allocated device memory of at least
 *     sga_workspace_size(dims, op) bytes, 256-byte aligned.  A zero-filled
 *     workspace starts with a clear status.  sga_forward (and its variants)
 *     also keeps per-query histograms and counters in it: its workspace must
 *     be zero-filled before the first call, and every call leaves them zeroed
 *     for the next one.  After a
 *     device error, zero the whole workspace before using it again.  Calls
 *     that share a workspace must be ordered on one stream.
 *   - No C++ exception crosses this interface.
 */
#ifndef SGA_H_
#define SGA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SGA_API __attribute__((visibility("default")))
#else
#define SGA_API
#endif

typedef uint16_t sga_bf16_t; /* bfloat16 bit pattern */
typedef uint8_t sga_fp8_e4m3_t; /* FP8 E4M3 bit pattern: 1 sign, 4 exponent (bias 7), 3 mantissa bits;
                                  no infinities, 0x7F / 0xFF are NaN, largest finite 448 */
typedef void* sga_stream_t;  /* cudaStream_t */

typedef enum {
  SGA_OK = 0,
  SGA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, unsupported shape */
  SGA_ERR_UNSUPPORTED = 2, /* no sm_100 device, or a size beyond the compiled limits */
  SGA_ERR_WORKSPACE = 3,   /* workspace null, misaligned or too small */
  SGA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  SGA_ERR_TIMEOUT = 5,     /* device: a bounded wait inside a kernel ran out */
  SGA_ERR_DEVICE_ARG = 6,  /* device: a position or index outside its range */
  SGA_ERR_INTERNAL = 7     /* device: an internal invariant check failed (libsga_debug.so only) */
} sga_status_t;

typedef enum {
  SGA_OP_INDEX_SCORES = 0,
  SGA_OP_TOPK_SELECT = 1,
  SGA_OP_SPARSE_MLA_ATTEND = 2,
  SGA_OP_FORWARD = 3,
  SGA_OP_FORWARD_FUSED = 4 /* sga_forward_fused and sga_forward_fused_fp8 */
} sga_op_t;

typedef struct {
  int32_t batch;     /* B >= 1 */
  int32_t n_q;       /* T >= 1 queries per sequence */
  int32_t kv_stride; /* L >= 1 cache rows per sequence (capacity) */
  int32_t top_k;     /* K: a multiple of 64 in [64, 2048]; the method uses 2048 */
} sga_dims_t;

/* Compiled model constants (archdb "A.X K2" attention, indexer and gate fields). */
#define SGA_INDEX_HEADS 64 /* Hi */
#define SGA_INDEX_DIM 128  /* Di */
#define SGA_HEADS 64       /* H */
#define SGA_QK_DIM 576     /* Dq = 512 latent + 64 rope */
#define SGA_V_DIM 512      /* Dv: the latent part is the value */
#define SGA_TOP_K 2048
#define SGA_MAX_TOP_K 2048
/* Softmax scale 192^-0.5 (qk head dim 192 = 128 nope + 64 rope). */
#define SGA_SOFTMAX_SCALE 0.07216878364870322
#define SGA_MAX_KV_STRIDE (1 << 30) /* positions are int32; rows * L must fit in int32 */

/* ABI version of this header (bumped on any incompatible change). */
SGA_API int32_t sga_abi_version(void);

/* Human-readable name of a status code (static string). */
SGA_API const char* sga_status_string(sga_status_t status);

/* Bytes of workspace `op` needs for `dims`.  SGA_OP_FORWARD covers ops 0-3;
 * SGA_OP_FORWARD_FUSED covers only the fused forward calls.
 * Returns SGA_ERR_INVALID_ARG for bad dims or a null `bytes`. */
SGA_API sga_status_t sga_workspace_size(const sga_dims_t* dims, sga_op_t op, size_t* bytes);

/* Step 1, the indexer (archdb "A.X K2", token-selection field):
 *   scores[b,i,s] = sum_j w[b,i,j] * max(0, sum_d q_idx[b,i,j,d] * k_idx[b,s,d])
 * for 0 <= s <= t = q_pos[b,i].  Entries with s > t are left unwritten.
 *   q_idx  [B][T][64][128] bf16     w      [B][T][64] bf16
 *   k_idx  [B][L][128] bf16         q_pos  [B][T] int32
 *   scores [B][T][L] fp32 (output; 16-byte aligned)
 * Accumulation is fp32; integer-valued inputs whose scores stay below 2^24
 * give exact scores.  Device error: t outside [0, L) (the row is skipped). */
SGA_API sga_status_t sga_index_scores(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                              const sga_bf16_t* k_idx, const int32_t* q_pos, float* scores, void* ws,
                              size_t ws_bytes, sga_stream_t stream);

/* Step 2, top-K selection (archdb "A.X K2", token-selection field; arXiv
 * abstract "A.X K2 Technical Report": each query reads 2,048 positions):
 * for each query, the K positions s <= t with the largest scores[b,i,s],
 * equal scores going to the lower position (-0.0 counts as +0.0); if t+1 <= K
 * every position 0..t is kept.  idx[b,i,:] lists them in ascending order,
 * followed by -1 in unused slots.
 *   scores [B][T][L] fp32 (entries s > t are not read)   q_pos [B][T] int32
 *   idx    [B][T][K] int32 (output)
 * NaN scores give an unspecified selection.  Device error: t outside [0, L):
 * that row's idx is all -1, the error goes only to the workspace status word
 * and the call itself still returns SGA_OK, so read the status (or validate
 * q_pos on the host) before trusting a row of -1. */
SGA_API sga_status_t sga_topk_select(const sga_dims_t* dims, const float* scores, const int32_t* q_pos, int32_t* idx,
                             void* ws, size_t ws_bytes, sga_stream_t stream);

/* Steps 3 and 4, sparse MLA attention in latent form plus the head gate
 * (archdb "A.X K2", attention and gate fields): for each query and head h,
 *   z_s   = (q[b,i,h,:] . kv[b,s,:]) * 192^-0.5     for s in idx[b,i,:], s >= 0
 *   o     = sum_s softmax(z)_s * kv[b,s,0:512]
 *   out[b,i,h,:] = o / (1 + exp(-gate[b,i,h]))      (gate == NULL: no gate)
 *   q    [B][T][64][576] bf16        kv  [B][L][576] bf16
 *   idx  [B][T][K] int32, any order, -1 = empty slot (positions are not
 *        compared with q_pos here; duplicates count twice)
 *   gate [B][T][64] bf16 or NULL     out [B][T][64][512] fp32 (output)
 * A query with no valid slot gets zeros.  Device error: an index outside
 * [-1, L) (the slot is treated as empty). */
SGA_API sga_status_t sga_sparse_mla_attend(const sga_dims_t* dims, const sga_bf16_t* q, const sga_bf16_t* kv,
                                   const int32_t* idx, const sga_bf16_t* gate, float* out, void* ws,
                                   size_t ws_bytes, sga_stream_t stream);

/* The whole path: sga_index_scores -> sga_topk_select -> sga_sparse_mla_attend,
 * with the scores and (when idx_out is NULL) the indices kept in the workspace.
 * idx_out [B][T][K] int32 may be NULL; other arguments as above. */
SGA_API sga_status_t sga_forward(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                         const sga_bf16_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                         const sga_bf16_t* gate, const int32_t* q_pos, int32_t* idx_out, float* out, void* ws,
                         size_t ws_bytes, sga_stream_t stream);

/* The indexer and the whole path with an E4M3 indexer-key cache (archdb "A.X
 * K2": the indexer key is the 128 values per token cached beside the KV;
 * its pretraining-precision field gives E4M3 matmuls; nlp.com.ai "A.X K2 FP8"
 * releases the model in FP8).  q_idx [B][T][64][128] and k_idx [B][L][128]
 * hold E4M3 bytes, used as their exact values with no block scale (so a key
 * row is 128 B instead of 256 B); everything else, the workspace and the
 * results are as for sga_index_scores / sga_forward.  Products of E4M3 values
 * are exact in fp32, and integer-valued inputs keep exact scores. */
SGA_API sga_status_t sga_index_scores_fp8(const sga_dims_t* dims, const sga_fp8_e4m3_t* q_idx, const sga_bf16_t* w,
                                  const sga_fp8_e4m3_t* k_idx, const int32_t* q_pos, float* scores, void* ws,
                                  size_t ws_bytes, sga_stream_t stream);
SGA_API sga_status_t sga_forward_fp8(const sga_dims_t* dims, const sga_fp8_e4m3_t* q_idx, const sga_bf16_t* w,
                             const sga_fp8_e4m3_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                             const sga_bf16_t* gate, const int32_t* q_pos, int32_t* idx_out, float* out, void* ws,
                             size_t ws_bytes, sga_stream_t stream);

/* The whole path with the selection fused into the indexer (archdb "A.X K2",
 * token-selection field: the top 2,048 positions by indexer score).  The
 * results are those of sga_forward / sga_forward_fp8 (the same indices, bit
 * for bit, and the same outputs); only the work differs.  For queries of
 * decode (T < 8) over L <= 262,144 positions the indexer writes no scores: it
 * counts the first radix level of each query's selection as it goes, raises a
 * per-query threshold from the counts so far (every key below it has at least
 * K larger keys already counted), and appends only the keys at or above it,
 * with their positions, to a candidate list in the workspace; the selection
 * then reads the candidates instead of L scores.  Other dims take the path of
 * sga_forward.  The workspace is sga_workspace_size(dims, SGA_OP_FORWARD_FUSED)
 * bytes, zero-filled before the first call, as for sga_forward. */
SGA_API sga_status_t sga_forward_fused(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                                       const sga_bf16_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                                       const sga_bf16_t* gate, const int32_t* q_pos, int32_t* idx_out, float* out,
                                       void* ws, size_t ws_bytes, sga_stream_t stream);
SGA_API sga_status_t sga_forward_fused_fp8(const sga_dims_t* dims, const sga_fp8_e4m3_t* q_idx,
                                           const sga_bf16_t* w, const sga_fp8_e4m3_t* k_idx, const sga_bf16_t* q,
                                           const sga_bf16_t* kv, const sga_bf16_t* gate, const int32_t* q_pos,
                                           int32_t* idx_out, float* out, void* ws, size_t ws_bytes,
                                           sga_stream_t stream);

/* Synchronises `stream` and returns in *device_status the first device-side
 * error recorded in the workspace (an sga_status_t value, SGA_OK if none). */
SGA_API sga_status_t sga_get_device_status(const void* ws, sga_stream_t stream, int32_t* device_status);

/* Clears the workspace status word (asynchronously on `stream`). */
SGA_API sga_status_t sga_clear_device_status(void* ws, sga_stream_t stream);

/* Diagnostic of the device-side failure path; no counterpart on the pages.
 * Every wait inside the kernels of this library gives up after a cycle
 * budget: the waiting thread writes SGA_ERR_TIMEOUT to the workspace status
 * word and raises an abort flag that releases every other wait of its thread
 * block, which then frees its tensor memory and exits, leaving the CUDA
 * context usable.  This call runs that sequence in one small kernel on a
 * shared-memory barrier that nothing completes (no copy is in flight): one
 * thread waits `budget_cycles` SM clock cycles, a second waits with the
 * kernels' own budget (about one second) and is released by the abort flag.
 * Afterwards the status word holds SGA_ERR_TIMEOUT and the second 32-bit word
 * of the workspace holds the number of waits that gave up (2; it is added to,
 * so zero it first).  budget_cycles in [1, 2^31); ws: at least 256 bytes,
 * 256-byte aligned.  Asynchronous on `stream`. */
SGA_API sga_status_t sga_selftest_bounded_wait(int64_t budget_cycles, void* ws, size_t ws_bytes,
                                               sga_stream_t stream);

/* Bytes of device memory inside the library that sga_topk_select_noalloc uses
 * as its scratch (a status word plus the selection bitmaps). */
#define SGA_NOALLOC_SCRATCH_BYTES (256 + 4 * 1024 * 1024)

/* sga_topk_select without a caller workspace.  No counterpart on the pages:
 * this entry point exists for callers that cannot allocate device memory,
 * for example a custom operator inside another inference engine whose plugin
 * interface hands over only its input and output buffers: it cannot lend a
 * workspace and must not call cudaMalloc, which would synchronise the device
 * and step outside the engine's memory budget.
 *   The scratch is one static device array of SGA_NOALLOC_SCRATCH_BYTES that
 * every GPU which loads the library keeps until the process exits.  The
 * selection bitmaps need 2 * B * T * ceil(L / 32) * 4 bytes; larger sizes are
 * rejected with SGA_ERR_WORKSPACE before anything is launched.  This call
 * allocates nothing and calls no allocating routine.  The first call on each
 * device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture.  Every call
 * shares the array, which keeps the last call's contents; each call clears
 * what must start at zero (the status word; the kernel zeroes its bitmap
 * words before use).  Calls that overlap on the GPU race on the array, so
 * order them on one stream.  Device-side errors are not reported (the status
 * word is private to the library): a row whose q_pos lies outside [0, L)
 * comes back as all -1 while the call returns SGA_OK, so validate q_pos on the
 * host.  All other arguments, results and errors are as for sga_topk_select.
 * A failed look-up of the array's address returns SGA_ERR_CUDA, and the next
 * call on that device looks it up again. */
SGA_API sga_status_t sga_topk_select_noalloc(const sga_dims_t* dims, const float* scores, const int32_t* q_pos,
                                             int32_t* idx, sga_stream_t stream);

/* ------------------------------------------------------------------------
 * One SGA attention layer: the projections either side of the path.
 * Sources: archdb "A.X K2", attention fields (64 heads; qk head dim 192 = 128
 * nope + 64 rope; v head dim 128; KV latent 512; q low-rank width 1536; a
 * 64-dim decoupled RoPE key shared across heads; partial RoPE with base 1e6;
 * no per-head QK norm; no projection bias), gate field (head-specific sigmoid
 * gate on the attention output before o_proj, projected jointly with the
 * query) and token-selection field (DSA-style indexer, 64 heads of dim 128).
 * For new tokens h [B][T][D] at positions q_pos:
 *   c_q = W_DQ h;  [q_nope_h, q_rope_h] = W_UQ_h c_q;  g = W_G c_q
 *   [c_kv, k_rope] = W_DKV h;  k_idx = W_IK h;  w = W_IW h;  q_idx = W_IQ c_q
 *   q_rope, k_rope rotated by RoPE at the token's position: interleaved pairs
 *     (2i, 2i+1), angle q_pos * 1e6^(-i/32), i < 32 (no YaRN factor)
 *   q_h = [W_UK_h^T q_nope_h, q_rope_h]   (W_UK absorbed into the query)
 *   kv_cache[b, q_pos] = [c_kv, k_rope];  k_idx_cache[b, q_pos] = k_idx
 *   idx, out = sga_forward(q_idx, w, k_idx_cache, q, kv_cache, g, q_pos)
 *   o_h = W_UV_h out_h;  y = W_O [o_1; ...; o_64]
 * Every activation between two contractions is rounded to bf16 (to nearest,
 * ties to even); the contractions accumulate in fp32; y is fp32.  The GEMMs
 * are this library's tcgen05 kernels (the weights streamed once, the new
 * tokens in the MMA's N dimension); when one splits K for parallelism its fp32
 * partial sums are added in a fixed order, so results do not depend on the
 * schedule.  Layer calls are thread-safe across distinct workspaces.
 *
 * Weights: bf16, row-major, `out = W in` (torch Linear layout), packed so the
 * projections that read the same input are one GEMM:
 *   w_hq [R + 768][D]:        rows W_DQ (R) | W_DKV (576: c_kv then k_rope)
 *                             | W_IK (128) | W_IW (64)
 *   w_cq [20544][R]:          rows W_UQ (head h: rows 192h .. 192h+191, the 128
 *                             nope rows first) | W_G (64) | W_IQ (head j: rows
 *                             12352 + 128j ..)
 *   w_uk [64][128][512]:      k_nope_h = w_uk[h] c_kv
 *   w_uv [64][128][512]:      o_h = w_uv[h] out_h
 *   w_o  [D][8192]
 * D = d_model (7168 in A.X K2) and R = q_rank (1536) are multiples of 8; every
 * weight pointer is 16-byte aligned.  The new tokens of one sequence must
 * have distinct positions.                                                   */

typedef struct {
  int32_t d_model; /* D */
  int32_t q_rank;  /* R */
  const sga_bf16_t* w_hq;
  const sga_bf16_t* w_cq;
  const sga_bf16_t* w_uk;
  const sga_bf16_t* w_uv;
  const sga_bf16_t* w_o;
} sga_layer_weights_t;

typedef enum {
  SGA_LAYER_PROJECT = 0, /* sga_layer_project */
  SGA_LAYER_OUTPUT = 1,  /* sga_layer_output */
  SGA_LAYER_FORWARD = 2  /* sga_layer_forward (covers both) */
} sga_layer_op_t;

/* Bytes of workspace a layer call needs (256-byte aligned, zero-filled before
 * the first sga_layer_forward, as for sga_forward; the layer's status word is
 * at its start).  Depends on dims and on weights->d_model / q_rank only.
 * SGA_ERR_INVALID_ARG for bad dims, sizes or a null `bytes`. */
SGA_API sga_status_t sga_layer_workspace_size(const sga_dims_t* dims, const sga_layer_weights_t* weights,
                                              sga_layer_op_t op, size_t* bytes);

/* The projections in front of the path for new tokens:
 *   h      [B][T][D] bf16              q_pos [B][T] int32, 0 <= q_pos < L
 *   kv_cache [B][L][576] bf16, k_idx_cache [B][L][128] bf16: the rows at
 *          (b, q_pos[b,i]) are overwritten with the new tokens' rows; no
 *          other row is touched
 *   q [B][T][64][576], gate [B][T][64], q_idx [B][T][64][128], w [B][T][64]
 *          bf16 (outputs): the inputs sga_forward takes for these tokens
 * Device error: a position outside [0, L) (that token's cache rows are not
 * written). */
SGA_API sga_status_t sga_layer_project(const sga_dims_t* dims, const sga_layer_weights_t* weights,
                                       const sga_bf16_t* h, const int32_t* q_pos, sga_bf16_t* kv_cache,
                                       sga_bf16_t* k_idx_cache, sga_bf16_t* q, sga_bf16_t* gate, sga_bf16_t* q_idx,
                                       sga_bf16_t* w, void* ws, size_t ws_bytes, sga_stream_t stream);

/* The projections after the path: out [B][T][64][512] fp32 (the gated
 * attention output sga_forward writes) -> y [B][T][D] fp32. */
SGA_API sga_status_t sga_layer_output(const sga_dims_t* dims, const sga_layer_weights_t* weights, const float* out,
                                      float* y, void* ws, size_t ws_bytes, sga_stream_t stream);

/* The whole layer: sga_layer_project -> sga_forward -> sga_layer_output, with
 * every intermediate in the workspace.  idx_out [B][T][K] int32 may be NULL;
 * dims->top_k as for sga_forward. */
SGA_API sga_status_t sga_layer_forward(const sga_dims_t* dims, const sga_layer_weights_t* weights,
                                       const sga_bf16_t* h, const int32_t* q_pos, sga_bf16_t* kv_cache,
                                       sga_bf16_t* k_idx_cache, int32_t* idx_out, float* y, void* ws, size_t ws_bytes,
                                       sga_stream_t stream);

/* ------------------------------------------------------------------------
 * The indexer's sparse warm-up objective and its gradients (arXiv abstract
 * "A.X K2 Technical Report": the indexer is optimised against its own sparse
 * top-k selection rather than the dense attention distribution; archdb
 * "A.X K2", stage notes: indexer-only training with the backbone frozen).
 * The pages give no formula; the reading, for query t with its selection S =
 * the valid entries of idx[b,i,:] (as sga_forward returns them):
 *   p(s)  = (1/64) sum_h softmax_{s in S}((q[b,i,h,:] . kv[b,s,:]) * 192^-0.5)
 *           the frozen attention's distribution (a target: no gradient)
 *   r(s)  = softmax_{s in S}(score(s)), score as in sga_index_scores
 *   loss[b,i] = KL(p || r)
 * and the gradients of the loss with respect to the indexer's inputs:
 *   grad_q_idx [B][T][64][128] fp32 (8-byte aligned), grad_w [B][T][64]
 *   fp32 (overwritten);
 *   grad_k_idx [B][L][128] fp32 (8-byte aligned): ADDED to (zero it before
 *   the first call; a position selected by several queries receives all
 *   their terms).  The gradients are summed with float atomics, so their last
 *   bits depend on the order in which the terms arrive.
 * The ReLU passes no gradient at 0.  Inputs as for sga_forward; loss [B][T]
 * fp32 (its terms summed in a fixed order).  Workspace: sga_indexer_warmup_workspace_size bytes, 256-byte aligned,
 * its status word at the start (zero-filled before the first call).  B*T is
 * at most 65535.  Device error: an index outside [-1, L) (treated as empty). */
SGA_API sga_status_t sga_indexer_warmup_workspace_size(const sga_dims_t* dims, size_t* bytes);
SGA_API sga_status_t sga_indexer_warmup(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                                        const sga_bf16_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                                        const int32_t* idx, float* loss, float* grad_q_idx, float* grad_w,
                                        float* grad_k_idx, void* ws, size_t ws_bytes, sga_stream_t stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* SGA_H_ */
