/*
 * mla.h -- C ABI of libmla_b200.so: absorbed Multi-head Latent Attention (MLA) decode on B200.
 *
 * The method (cited by page title and section):
 *   [rs]  "ferrox-core 0.23.0 src/mla_absorbed.rs", module docs "What it is" and the doc comment
 *         of causal_mla_absorbed_attention: the query is pushed into the latent
 *         (q_abs[h] = W_UK[h]^T q_nope[h]), attention runs as multi-query attention over ONE shared
 *         key row concat(c_t, k_pe_t) and ONE shared value c_t per position,
 *         score = (q_abs . c + q_pe . k_pe) * kq_scale, kq_scale = 1/sqrt(qk_nope + rope_dim),
 *         out_lat = softmax(score) . c, and v[h] = W_UV[h] out_lat[h].
 *   [nb]  "MLA_RoPE-less.ipynb": cache update before attention, matrix absorption
 *         (W_aQK = W_uQ W_uK^T, W_aVO = W_uV W_O), the adding trick over heads.
 *   [lab] "Lab 01 - Ejercicio matematico de MLA" (lynx-cortex), Bloque B: the matmul identity
 *         q^T W_UK c = (W_UK^T q)^T c.
 *   [fm]  "preacher-1/MLA_tutorial formula.md", Part 3, inference-form equation: o_t is the
 *         concatenation of o^(s) W_v^(s), followed by the output projection; the query comes from
 *         the low-rank latent c'_i = x_i W'_c as [c'_i W_qc^(s) W_kc^(s)T, c'_i W_qr^(s) R_i] and the
 *         key from c_i = x_i W_c and the rotary part x_i W_kr R_i (from x_i, not c_i).
 *   [gm]  "Gated MLA" (tensortonic, Kimi K3 step 2 of 11): Y = [sigmoid(X Wg^T) * O] Wo^T,
 *         causal mask removing later positions, the Requirements (inputs are not mutated).
 *
 * Conventions shared by every entry point
 *   - All tensors are caller-owned DEVICE memory, dense, row-major, in the dtype named by the call
 *     (MLA_F32 or MLA_BF16), except where a parameter says float / int32 / int64 explicitly, and
 *     except the host buffers of mla_decode_step with MLA_IO_HOST.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call is asynchronous
 *     with respect to the host and enqueues its kernels on that stream only.
 *   - Inputs are never written. Outputs are written only where documented.
 *   - Host-side validation runs before any launch; on a violation the call returns an error and
 *     launches nothing. A failed launch returns MLA_ERR_CUDA. Nothing aborts the process.
 *   - The library allocates no device memory. Scratch memory is the caller's `workspace`.
 *   - bf16 values are rounded to nearest-even wherever the library stores bf16.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point (int32_t). */
enum {
  MLA_OK = 0,
  MLA_ERR_NULL = 1,        /* a required pointer is NULL                                        */
  MLA_ERR_SHAPE = 2,       /* a size is negative, zero where it must be positive, or inconsistent */
  MLA_ERR_DTYPE = 3,       /* unknown dtype code, or a dtype the operation does not take         */
  MLA_ERR_ALIGN = 4,       /* a pointer is not aligned as the operation requires (16 B for bf16) */
  MLA_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than the size query returned             */
  MLA_ERR_CUDA = 6,        /* a CUDA runtime call or a kernel launch failed                      */
  MLA_ERR_TIMEOUT = 7,     /* a bounded device-side wait gave up (reported by mla_check_status)  */
  MLA_ERR_UNSUPPORTED = 8, /* a valid request this build does not implement                      */
  MLA_ERR_MODE = 9         /* unknown mode or flag bit                                           */
};

/* Element types. All floating-point tensors of one call share the call's dtype ([gm] Constraints),
 * except the fp8 latent cache of the *_fp8 entry points (MLA_FP8_E4M3: 1 byte, 4 exponent and 3
 * mantissa bits, no infinities, largest finite value 448). */
enum { MLA_F32 = 0, MLA_BF16 = 1, MLA_FP8_E4M3 = 2 };

/* Model dimensions. kq_scale == 0 selects the default 1/sqrt(qk_nope + rope_dim): the width of the
 * UN-absorbed head, not of the latent ([rs] module docs, the kq_scale paragraph). */
typedef struct mla_dims {
  int32_t n_heads;      /* H                                                        */
  int32_t kv_lora_rank; /* d_c: width of the latent c_t, also the value width        */
  int32_t rope_dim;     /* d_r: width of the decoupled rotary key k_pe_t (may be 0)   */
  int32_t qk_nope;      /* n: per-head width of the non-rotary query / key            */
  int32_t v_head;       /* d_v: per-head width of the value after W_UV                */
  int32_t d_model;      /* D: width of the layer output                               */
  float kq_scale;       /* score scale; 0 => 1/sqrt(qk_nope + rope_dim)               */
} mla_dims;

/* modes of mla_absorb_weights */
enum { MLA_ABSORB_QUERY = 0, MLA_FOLD_QK = 1, MLA_FOLD_VO = 2 };
/* flags of mla_append_latent */
enum { MLA_APPEND_NORM = 1u, MLA_APPEND_ROPE = 2u };
/* flags of mla_decode_absorbed */
enum { MLA_DECODE_CAUSAL = 1u, MLA_DECODE_OUT_BF16 = 2u };
/* flags of mla_linear */
enum { MLA_LINEAR_SIGMOID = 1u, MLA_LINEAR_W_KN = 2u };
/* where the step's x, y and index arrays live (mla_decode_step) */
enum { MLA_IO_DEVICE = 0, MLA_IO_HOST = 1 };

/* The weights of one decode step, all DEVICE memory in the step's dtype, PyTorch Linear convention
 * ([out, in], row-major) for the dense projections. */
typedef struct mla_step_weights {
  const void* w_cq;   /* W'_c^T  [q_rank, d_model]                       query down-projection     */
  const void* w_qc;   /* W_qc^T  [n_heads * qk_nope, q_rank]             head h: rows h*qk_nope..  */
  const void* w_qr;   /* W_qr^T  [n_heads * rope_dim, q_rank]            head h: rows h*rope_dim.. */
  const void* w_dkv;  /* [W_c, W_kr]^T [kv_lora_rank + rope_dim, d_model] latent rows, then rotary */
  const void* w_uk;   /* W_UK    [n_heads, qk_nope, kv_lora_rank]        (W_kc^(h) transposed)     */
  const void* w_uv;   /* W_UV    [n_heads, v_head, kv_lora_rank]                                   */
  const void* w_o;    /* W_O     [d_model, n_heads * v_head]                                       */
} mla_step_weights;

/* Human-readable name of a status code (static string, never NULL). */
MLA_API const char* mla_status_string(int32_t status);

/* ABI version of this header (increments on any signature change). */
MLA_API int32_t mla_abi_version(void);

/*
 * mla_append_latent -- write new latent-cache rows ([nb] "update cache": the new latent is
 * stacked onto the cache before attention; [rs] fn docs: a row is the normed compressed KV
 * followed by the roped k_pe, i.e. concat(c, k_pe)).
 *
 *   cache      [cache_rows, d_c + d_r] in cache_dtype; only rows row_idx[k] are written.
 *   row_idx    int64 [n_new], each in [0, cache_rows); duplicates give an unspecified winner.
 *   c_new      float [n_new, d_c];  kpe_new float [n_new, d_r] (may be NULL when d_r == 0).
 *   positions  int32 [n_new] rotary positions (read only with MLA_APPEND_ROPE).
 *   flags      MLA_APPEND_NORM: c <- c / sqrt(mean(c^2) + eps) (unit weight);
 *              MLA_APPEND_ROPE: k_pe pair (2i, 2i+1) turns by positions[k] * rope_theta^(-2i/d_r).
 * Errors: MLA_ERR_NULL, MLA_ERR_SHAPE (d_r odd with ROPE, n_new < 0), MLA_ERR_DTYPE, MLA_ERR_MODE.
 */
MLA_API int32_t mla_append_latent(const mla_dims* dims, int32_t cache_dtype, void* cache, int64_t cache_rows,
                          const int64_t* row_idx, const float* c_new, const float* kpe_new,
                          const int32_t* positions, int64_t n_new, uint32_t flags, float eps,
                          float rope_theta, void* stream);

/*
 * mla_append_latent_fp8 -- mla_append_latent into an e4m3 latent cache (cache [cache_rows, d_c + d_r]
 * bytes). The row is built as there, in fp32; each value is then stored as the e4m3 code nearest to
 * value / cache_scale (an fp32 division; ties to even; saturating at +-448). One scale per cache: 1
 * suits RMS-normed latents and N(0, 1) rotary keys, whose values stay far below 448.
 * Errors: those of mla_append_latent; MLA_ERR_SHAPE for a scale that is not positive and finite.
 */
MLA_API int32_t mla_append_latent_fp8(const mla_dims* dims, uint8_t* cache, int64_t cache_rows,
                                      const int64_t* row_idx, const float* c_new, const float* kpe_new,
                                      const int32_t* positions, int64_t n_new, uint32_t flags, float eps,
                                      float rope_theta, float cache_scale, void* stream);

/*
 * mla_absorb_weights -- per-head products of the absorbed form.
 *
 * MLA_ABSORB_QUERY ([rs] module docs: q_nope_absorbed[h] = wk_b[h] . q_nope[h]; [lab] Bloque B:
 *   q^T W_UK c = (W_UK^T q)^T c):
 *     x    = q_nope [n_rows, H, qk_nope];  x_pe = q_pe [n_rows, H, d_r] (NULL allowed if d_r == 0);
 *     w    = W_UK   [H, qk_nope, d_c];
 *     out  = q_abs  [n_rows, H, d_c + d_r]:  out[t,h,j] = sum_i x[t,h,i] w[h,i,j] (j < d_c),
 *            out[t,h,d_c + r] = x_pe[t,h,r].
 * MLA_FOLD_QK ([nb] matrix absorption, W_aQK = W_uQ W_uK^T):
 *     x = W_uQ heads [H, n_rows, qk_nope], w = W_uK heads [H, d_c, qk_nope],
 *     out = W_aQK [H, n_rows, d_c] = x[h] . w[h]^T.
 * MLA_FOLD_VO ([nb] matrix absorption, W_aVO = W_uV W_O):
 *     x = W_uV heads [H, d_c, v_head], w = W_O heads [H, v_head, d_model],
 *     out = W_aVO [H, d_c, d_model] = x[h] . w[h]   (n_rows must equal d_c).
 * All operands in `dtype`; accumulation in fp32; out in `dtype`.
 */
MLA_API int32_t mla_absorb_weights(const mla_dims* dims, int32_t dtype, int32_t mode, const void* x,
                           const void* x_pe, const void* w, int64_t n_rows, void* out, void* stream);

/*
 * mla_decode_workspace_size -- bytes of scratch mla_decode_absorbed needs for these sizes.
 *   batch        number of sequences B;  n_q_per_seq  query tokens per sequence (>= 1);
 *   max_seqlen   an upper bound on every T_b (a requirement: see mla_decode_absorbed);
 *   total_rows   sum of T_b (rows of the packed cache).
 *   dtype MLA_FP8_E4M3 returns the scratch of mla_decode_absorbed_fp8 (for either query dtype).
 */
MLA_API int32_t mla_decode_workspace_size(const mla_dims* dims, int32_t dtype, int32_t batch,
                                  int32_t n_q_per_seq, int64_t max_seqlen, int64_t total_rows,
                                  uint32_t flags, size_t* bytes);

/*
 * mla_decode_absorbed -- attention of the absorbed queries over the shared latent cache
 * ([rs] module docs and fn: score[h][t] = (q_abs[h] . c[t] + q_pe[h] . k_pe[t]) * kq_scale,
 * out_lat[h] = sum_t softmax(score[h])[t] c[t], returned before W_UV; [gm] causal mask).
 *
 *   q_abs       [B * n_q, H, d_c + d_r]; row b*n_q + j is query j of sequence b.
 *   cache       [total_rows, d_c + d_r]; sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1.
 *   cu_seqlens  DEVICE int32 [B + 1], non-decreasing, cu_seqlens[0] = 0, cu_seqlens[B] = total_rows.
 *   flags       MLA_DECODE_CAUSAL: query j of sequence b (the n_q newest tokens sit at its last
 *               n_q rows) sees positions t <= T_b - n_q + j; otherwise it sees all T_b positions.
 *               MLA_DECODE_OUT_BF16: out_lat is written in bf16 instead (the operand of
 *               mla_out_project_bf16); tensor-core route only, else MLA_ERR_UNSUPPORTED.
 *   out_lat     float [B * n_q, H, d_c] (bf16 under MLA_DECODE_OUT_BF16): the softmax-weighted latent
 *               (zeros when nothing is seen).
 *   lse         float [B * n_q, H] or NULL: natural-log sum-exp of the scaled scores (-inf if empty).
 *   workspace   caller scratch of at least mla_decode_workspace_size() bytes, 256-byte aligned.
 * Requirements: T_b <= max_seqlen for every b (not checked on the device: the plan assumes it
 * when it sizes the split of each sequence), T_b >= n_q when causal.
 * bf16 calls with d_c = 512 and d_r in {0, 64} run the tensor-core (tcgen05) kernel; every other
 * supported shape runs the CUDA-core kernel. Both accumulate in fp32. In the tensor-core kernel the
 * scores are fp32 from the MMA to the exponential (no range limit below fp32's); the softmax weights
 * enter the P . C product as bf16 (round to nearest even), and the row sums add the same values.
 * Cache rows read past the end of a sequence are multiplied by zero weights: they must hold finite
 * values (rows of other sequences, or rows the caller keeps finite).
 */
MLA_API int32_t mla_decode_absorbed(const mla_dims* dims, int32_t dtype, const void* q_abs, const void* cache,
                            const int32_t* cu_seqlens, int32_t batch, int32_t n_q_per_seq,
                            int64_t max_seqlen, int64_t total_rows, uint32_t flags, float* out_lat,
                            float* lse, void* workspace, size_t workspace_bytes, void* stream);

/*
 * mla_decode_absorbed_fp8 -- mla_decode_absorbed over an e4m3 latent cache (value = code * cache_scale,
 * the cache of mla_append_latent_fp8) with a bf16 or fp32 absorbed query (q_dtype): half the cache bytes
 * of a bf16 cache. Same arguments, layouts and results otherwise; scratch of at least
 * mla_decode_workspace_size(dims, MLA_FP8_E4M3, ...) bytes. With a bf16 query at d_c 512 (d_r 0 or
 * 64) it runs on the tensor cores: QK^T as e4m3 MMAs against the query split into two e4m3 parts with
 * a per-row power-of-two scale (about 2^-8 relative), P.C in f16 over the codes converted exactly;
 * the cache base must then be 16-byte aligned (otherwise the CUDA-core route runs). With an fp32 query
 * it runs on CUDA cores in fp32 arithmetic (decoded cache values, fp32 scores and softmax).
 */
MLA_API int32_t mla_decode_absorbed_fp8(const mla_dims* dims, int32_t q_dtype, const void* q_abs,
                                        const uint8_t* cache, float cache_scale, const int32_t* cu_seqlens,
                                        int32_t batch, int32_t n_q_per_seq, int64_t max_seqlen, int64_t total_rows,
                                        uint32_t flags, float* out_lat, float* lse, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Bytes of scratch mla_out_project needs for n_rows query rows. */
MLA_API int32_t mla_out_project_workspace_size(const mla_dims* dims, int32_t dtype, int64_t n_rows,
                                       size_t* bytes);

/*
 * mla_out_project -- v[t,h] = W_UV[h] out_lat[t,h] ([rs] v = wv_b . out_lat), optional channel
 * gate ([gm]: sigmoid(X Wg^T) * O), then y[t] = W_O concat_h v[t,h] ([fm] inference form;
 * [nb] the adding trick is the same sum over heads).
 *
 *   out_lat  float [n_rows, H, d_c];  w_uv [H, v_head, d_c];  w_o [d_model, H * v_head];
 *   gate     [n_rows, H * v_head] in `dtype`, or NULL for no gate (values are used as given: pass
 *            sigmoid(X Wg^T), e.g. from mla_linear with MLA_LINEAR_SIGMOID);
 *   y        [n_rows, d_model] in `dtype`.
 */
MLA_API int32_t mla_out_project(const mla_dims* dims, int32_t dtype, const float* out_lat, const void* w_uv,
                        const void* w_o, const void* gate, int64_t n_rows, void* y,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * mla_out_project_bf16 -- mla_out_project (dtype MLA_BF16) with out_lat in bf16 [n_rows, H, d_c], as
 * mla_decode_absorbed writes it under MLA_DECODE_OUT_BF16: the W_UV product reads it directly (no
 * fp32 -> bf16 conversion pass). out_lat 16-byte aligned; scratch as for mla_out_project.
 */
MLA_API int32_t mla_out_project_bf16(const mla_dims* dims, const void* out_lat, const void* w_uv, const void* w_o,
                                     const void* gate, int64_t n_rows, void* y, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * mla_linear -- Y = X W^T ([gm] problem equations, PyTorch Linear convention W = [n, k]).
 *   x [m, k], w [n, k] (or [k, n] with MLA_LINEAR_W_KN), y [m, n]; all in `dtype`, fp32 accumulate.
 *   MLA_LINEAR_SIGMOID applies sigmoid to Y before it is stored.
 */
MLA_API int32_t mla_linear(int32_t dtype, const void* x, const void* w, int64_t m, int64_t n, int64_t k,
                   uint32_t flags, void* y, void* stream);

/* Bytes of scratch mla_project_inputs needs for n_rows tokens. */
MLA_API int32_t mla_project_workspace_size(const mla_dims* dims, int32_t dtype, int32_t q_rank, int64_t n_rows,
                                           size_t* bytes);

/*
 * mla_project_inputs -- the input projections of n_rows new tokens ([fm] Part 3, inference-form
 * equation, the terms computed from x), fused with the latent append:
 *     c'_t         = x_t W'_c                        (q_rank wide; scratch, in `dtype`)
 *     q_nope[t, h] = c'_t W_qc^(h)                   (absorbed next by MLA_ABSORB_QUERY)
 *     q_pe[t, h]   = c'_t W_qr^(h), turned by R_{positions[t]} when flags has MLA_APPEND_ROPE
 *     c_t, k_t     = x_t W_c, x_t W_kr               (fp32 scratch; never rounded before the append)
 *     cache row row_idx[t] = concat(c_t, k_t) with mla_append_latent's flags (norm of c_t, rotation
 *     of k_t at positions[t]).
 *   x        [n_rows, d_model]; w_cq, w_qc, w_qr, w_dkv as in mla_step_weights (w_qr may be NULL
 *            when rope_dim == 0); q_nope [n_rows, H, qk_nope] and q_pe [n_rows, H, rope_dim] written;
 *   cache, cache_rows, row_idx, positions, eps, rope_theta: as mla_append_latent, with the cache in
 *   `dtype`. The rotation is the append's: pair (2i, 2i+1) turns by pos * rope_theta^(-2i/rope_dim).
 *   Products accumulate in fp32; bf16 operands go through the tensor cores when d_model and q_rank
 *   are multiples of 64 (c'_t is then rounded to bf16 once, as the next product's operand).
 * Errors: MLA_ERR_NULL, MLA_ERR_SHAPE (q_rank <= 0, qk_nope <= 0, d_model <= 0, rope_dim odd with
 * ROPE), MLA_ERR_DTYPE, MLA_ERR_MODE (unknown flag), MLA_ERR_ALIGN (16 B for bf16 tensors, 256 B for
 * the workspace), MLA_ERR_WORKSPACE; a row index outside the cache is skipped and reported through
 * mla_check_status (MLA_ERR_SHAPE).
 */
MLA_API int32_t mla_project_inputs(const mla_dims* dims, int32_t dtype, int32_t q_rank, const void* x,
                                   const void* w_cq, const void* w_qc, const void* w_qr, const void* w_dkv,
                                   int64_t n_rows, const int32_t* positions, void* q_nope, void* q_pe, void* cache,
                                   int64_t cache_rows, const int64_t* row_idx, uint32_t flags, float eps,
                                   float rope_theta, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of scratch mla_decode_step needs (the same for both io modes). */
MLA_API int32_t mla_decode_step_workspace_size(const mla_dims* dims, int32_t dtype, int32_t q_rank,
                                               int32_t batch, int64_t max_seqlen, int64_t total_rows,
                                               size_t* bytes);

/*
 * mla_decode_step -- one whole decode step for `batch` sequences with one new token each:
 * mla_project_inputs (append included) -> MLA_ABSORB_QUERY -> mla_decode_absorbed (n_q = 1) ->
 * mla_out_project without a gate ([fm] Part 3, inference form, end to end: y_t from x_t).
 *   x [batch, d_model] -> y [batch, d_model], both in `dtype`;
 *   cache [total_rows, d_c + d_r] (sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1], which
 *   already count the new token; row_idx[b] is where its latent goes, normally the last of those);
 *   cu_seqlens int32 [batch + 1], row_idx int64 [batch], positions int32 [batch] (read with
 *   MLA_APPEND_ROPE), append_flags / eps / rope_theta as mla_append_latent.
 *   io = MLA_IO_DEVICE: every pointer is device memory.
 *   io = MLA_IO_HOST: x, y, cu_seqlens, row_idx and positions are HOST memory. The call copies x
 *   into the workspace and y back with cudaMemcpyAsync on `stream`. The index arrays are read when
 *   the call is made, and passed on in a kernel's launch parameters (up to 240 sequences; beyond
 *   that, or while `stream` is being captured into a CUDA graph, they are copied like x, so that a
 *   graph's replays read them again). With page-locked host memory the call returns once all is
 *   enqueued: x and y must then stay untouched until the stream has passed this step (y holds the
 *   result after a synchronisation). The weights and the cache are device memory in both modes.
 * Errors: those of the four stages, checked before the first launch where they concern sizes;
 * MLA_ERR_MODE for an unknown io; MLA_ERR_CUDA when a copy cannot be enqueued.
 */
MLA_API int32_t mla_decode_step(const mla_dims* dims, int32_t dtype, int32_t q_rank, const mla_step_weights* w,
                                const void* x, void* cache, const int32_t* cu_seqlens, int32_t batch,
                                int64_t max_seqlen, int64_t total_rows, const int64_t* row_idx,
                                const int32_t* positions, uint32_t append_flags, float eps, float rope_theta,
                                void* y, int32_t io, void* workspace, size_t workspace_bytes, void* stream);

/*
 * mla_prefill_attention -- attention of UN-absorbed heads over whole prompts (prefill): per sequence b
 * and head h, O = softmax(scale * Q K^T) V with the causal mask under MLA_DECODE_CAUSAL (query s
 * sees keys t <= s), optionally times a gate ([gm] problem equations: Q = X Wq^T, K = C Wk^T,
 * V = C Wv^T, heads of D_h, causal mask, Y = [sigmoid(X Wg^T) * O] Wo^T; [fm] Part 3, training-form
 * equation). With every query of a prompt present, materialising K and V per head costs less than the
 * absorbed route, whose heads are d_c wide ([fm] Part 3, the note after the inference form).
 *   q, k, v, out  [batch * seq, n_heads * head_dim] row-major in `dtype` (sequence b owns rows
 *                 b*seq .. b*seq + seq - 1; head h owns columns h*head_dim ..);
 *   gate          same shape, multiplied into out (pass sigmoid(X Wg^T)), or NULL;
 *   scale         0 => 1/sqrt(head_dim).
 * Tensor cores: bf16 with head_dim 128; other requests return MLA_ERR_UNSUPPORTED (the absorbed route,
 * mla_decode_absorbed with n_q = seq, computes the same attention for any width). P is rounded to bf16
 * for the P V product; scores, the softmax and the output accumulate in fp32.
 * Errors: MLA_ERR_NULL, MLA_ERR_SHAPE, MLA_ERR_DTYPE, MLA_ERR_MODE, MLA_ERR_ALIGN (16 B),
 * MLA_ERR_UNSUPPORTED; a bounded device wait that gives up reports MLA_ERR_TIMEOUT (mla_check_status).
 */
MLA_API int32_t mla_prefill_attention(int32_t dtype, const void* q, const void* k, const void* v, const void* gate,
                                      int32_t batch, int32_t seq, int32_t n_heads, int32_t head_dim, float scale,
                                      uint32_t flags, void* out, void* stream);

/*
 * mla_lse_merge -- merge partial decode results computed over disjoint slices of every sequence's
 * positions (split-KV across devices: each device holds a contiguous slice of the latent cache and runs
 * mla_decode_absorbed on it). For each query row and head, with m = max_r lse_r and
 * w_r = exp(lse_r - m):  out_lat = sum_r w_r out_lat_r / sum_r w_r,  lse = m + log(sum_r w_r); the
 * softmax over the union of the slices, restated by its log-sum-exp ([rs] fn body: max-subtracted
 * exponentials, their sum and the weighted sum of latent rows). Parts whose lse is -inf (a slice
 * with no visible position) take no part; if every part is -inf the row is 0 and its lse -inf.
 *   n_parts         1 .. MLA_MERGE_MAX_PARTS;
 *   out_lat_parts   HOST array of n_parts pointers, each to float [rows_total, H, d_c] (16-byte
 *                   aligned; a whole buffer even for a part whose slice is empty: its values may be
 *                   read, never used); lse_parts likewise to float [rows_total, H]. They may point into other
 *                   devices' memory that this device can load from (peer access or symmetric memory):
 *                   the kernel only reads them, so the merge is also the exchange;
 *   row_begin, n_rows  the query rows merged: rows row_begin .. row_begin + n_rows of every part;
 *   out_lat float [n_rows, H, d_c] and lse float [n_rows, H] (lse may be NULL) receive them.
 * Sums run over r in index order: the result does not depend on timing or on the device that runs it.
 * Errors: MLA_ERR_NULL, MLA_ERR_SHAPE (n_parts out of range, n_rows or row_begin < 0), MLA_ERR_ALIGN.
 */
#define MLA_MERGE_MAX_PARTS 16
MLA_API int32_t mla_lse_merge(const mla_dims* dims, int32_t n_parts, const float* const* out_lat_parts,
                              const float* const* lse_parts, int64_t row_begin, int64_t n_rows, float* out_lat,
                              float* lse, void* stream);

/*
 * mla_check_status -- synchronise `stream`, then report and clear the library's device status
 * word: MLA_OK, or MLA_ERR_TIMEOUT when a bounded device wait gave up, or MLA_ERR_SHAPE when a kernel skipped an out-of-range row index, since the last check.
 */
MLA_API int32_t mla_check_status(void* stream, int32_t* device_status);

/* Tuning hook: number of 2-CTA clusters the tensor-core decode spreads its work over (0 = one per
 * pair of SMs, the default). Affects only the work split, never the result beyond rounding. */
MLA_API int32_t mla_set_decode_clusters(int32_t n);

/* Number of kernels this library has launched in this process (all devices, all streams). */
MLA_API int64_t mla_launch_count(void);

/* Test hook: time limit, in nanoseconds of the device's global timer, of every bounded device-side
 * wait (0 restores the default of 2 s; negative: MLA_ERR_SHAPE). Applies to kernels launched after
 * the call. A wait that runs out sets MLA_ERR_TIMEOUT in the status word and its kernel abandons its
 * work (outputs undefined) after its own copies and tensor-core operations in flight have ended. */
MLA_API int32_t mla_set_wait_limit(int64_t limit_ns);

/*
 * mla_wait_selftest -- diagnostic with no counterpart in the method: launches one CTA on `stream`
 * that allocates tensor memory, waits on an mbarrier that nothing completes (through the same
 * bounded wait as the tensor-core kernels), gives up after the current wait limit, releases its
 * tensor memory and returns. The status word then reads MLA_ERR_TIMEOUT (mla_check_status) and the
 * context stays usable. Returns MLA_ERR_CUDA if the launch fails.
 */
MLA_API int32_t mla_wait_selftest(void* stream);

/*
 * mla_decode_absorbed_noalloc -- an addition of this library with no counterpart in the method: the
 * same decode as mla_decode_absorbed (same arguments, layouts and results), with its scratch in a
 * fixed array of MLA_DECODE_NOALLOC_MAX_BYTES inside the library's device image instead of a
 * caller workspace. It allocates no memory (no cudaMalloc / cudaFree, no allocating library call);
 * the array's address is looked up once per device, with that device current.
 *   Errors: those of mla_decode_absorbed; MLA_ERR_WORKSPACE when the problem needs more scratch than
 *   MLA_DECODE_NOALLOC_MAX_BYTES (mla_decode_workspace_size reports the need); MLA_ERR_CUDA when the
 *   array's address cannot be obtained, or when `stream` belongs to a device other than the current
 *   one (the array is looked up on the current device; no launch happens then).
 *   Nothing in the scratch has to start at zero. All calls on one device share the one array: calls
 *   whose executions overlap on the GPU (different streams without ordering between them) race on
 *   it and give undefined results; calls ordered on one stream do not.
 */
#define MLA_DECODE_NOALLOC_MAX_BYTES ((size_t)40 << 20)
MLA_API int32_t mla_decode_absorbed_noalloc(const mla_dims* dims, int32_t dtype, const void* q_abs,
                                            const void* cache, const int32_t* cu_seqlens, int32_t batch,
                                            int32_t n_q, int64_t max_seqlen, int64_t total_rows,
                                            uint32_t flags, float* out_lat, float* lse, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
