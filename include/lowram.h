/*
 * lowram.h -- C ABI of liblowram.so: LowRAM's encode and decode-time hot path on one
 * B200 (sm_100a).
 *
 * The method ("LowRAM: Low-Rank Keys and Amortised Values for Composable KV Cache
 * Compression at Test-Time"; summary on agihunt.info, overview "LowRAM Exploits
 * Key-Value Predictability to Compress the KV Cache" on cctest.ai, and the abstract):
 *   - keys: RoPE is inverted, then every token's key (all KV heads of a layer, flattened
 *     to D = H_kv*d) is projected onto a low-rank basis shared by two adjacent layers
 *     (xKV); the prefix is cut into chunks whose mean key is kept as a landmark;
 *   - values: a small per-head key->value MLP predicts V from the rebuilt key; residual
 *     corrections are stored only for the tokens it predicts worst;
 *   - decode: the query scores the chunk landmarks, the top-k chunks are selected, only
 *     their keys (low rank, RoPE re-applied) and values (MLP + residuals) are rebuilt,
 *     and GQA attention runs over that subset.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers on the context's device unless stated.
 *     Arrays are dense, row-major, in the order of the brackets given.
 *   - Element type: every cache, weight, query and output array is stored in
 *     cfg->dtype (fp32 or bf16); index arrays are int32. Arithmetic is fp32 with fp64
 *     used to settle selections near their threshold.
 *   - The caller owns every buffer (inputs, cache, outputs, workspace). The context owns
 *     tables (RoPE cos/sin, a status word, work counters) and the landmark scores
 *     of one decode step (B*H_kv*N_c floats: 4 MiB at batch 8, 8 KV heads, 128K tokens,
 *     chunk 8), which it keeps in a reset state between calls. Calls allocate nothing.
 *   - Calls are asynchronous on the given stream (a cudaStream_t passed as void*; NULL =
 *     the legacy default stream). Arguments are validated on the host first; on any
 *     error nothing is launched and the status says why.
 *   - Alignment: every pointer must be 16-byte aligned (LOWRAM_ERR_ALIGN otherwise).
 *   - One context serves one stream at a time: concurrent calls with the same context
 *     on different streams race on its counters. Use one context per stream.
 *   - The ABI is per layer. Two layers of one xKV group pass the same basis pointer.
 */
#ifndef LOWRAM_H
#define LOWRAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lowram_status {
  LOWRAM_OK = 0,
  LOWRAM_ERR_INVALID_ARG = 1,  /* null pointer, unknown enum value                    */
  LOWRAM_ERR_SHAPE = 2,        /* sizes inconsistent with each other                  */
  LOWRAM_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned                    */
  LOWRAM_ERR_UNSUPPORTED = 4,  /* valid sizes this build does not implement           */
  LOWRAM_ERR_WORKSPACE = 5,    /* workspace smaller than lowram_workspace_size()      */
  LOWRAM_ERR_CUDA = 6,         /* a CUDA runtime call or launch failed                */
  LOWRAM_ERR_DEVICE_CHECK = 7, /* a kernel found malformed cache contents (reported by
                                  lowram_last_error)                                   */
  LOWRAM_ERR_TIMEOUT = 8       /* a kernel's bounded wait gave up (lowram_last_error)  */
} lowram_status;

enum { LOWRAM_DTYPE_F32 = 0, LOWRAM_DTYPE_BF16 = 1 };
enum { LOWRAM_ACT_SILU = 0, LOWRAM_ACT_GELU_ERF = 1 };
/* Which reconstruct-and-attend kernel decode uses. AUTO picks the tcgen05 tensor-core
 * kernel where it applies (bf16, d = 128, F = 256, r % 32 == 0, r <= 160, G = 4) and the
 * CUDA-core kernel otherwise (always for fp32, whose 1e-4 tolerance tensor cores cannot
 * meet). */
enum { LOWRAM_DECODE_AUTO = 0, LOWRAM_DECODE_SIMT = 1, LOWRAM_DECODE_TCGEN05 = 2 };
enum { LOWRAM_OP_ENCODE = 0, LOWRAM_OP_DECODE = 1, LOWRAM_OP_DENSE = 2, LOWRAM_OP_EVICT = 3 };
/* How residual rows are stored. STORE: in cfg->dtype. INT4_G32 (LowRAM-Q, the residuals
 * stored at low precision of the agihunt summary's composition paragraph): symmetric
 * int4 codes, two per byte (element 2i in the low nibble), with one fp16 scale per 32
 * elements, s = fp16(max|x| / 7), q = clamp(round-half-even(x / s), -8, 7); the row's
 * value is q * s. bf16 caches with the tensor-core encode's sizes only. */
enum { LOWRAM_RES_STORE = 0, LOWRAM_RES_INT4_G32 = 1 };

/* Sizes of one layer call. T % chunk == 0; n_q_heads % n_kv_heads == 0. */
typedef struct lowram_config {
  int32_t batch;          /* B                                                          */
  int32_t n_tokens;       /* T, prefix length (token positions 0 .. T-1)               */
  int32_t n_kv_heads;     /* H_kv                                                       */
  int32_t n_q_heads;      /* H_q; G = H_q / H_kv query heads share a KV head (GQA)      */
  int32_t head_dim;       /* d: 64 or 128                                               */
  int32_t rank;           /* r: xKV rank, multiple of 16, 16 .. 256                      */
  int32_t chunk;          /* C: tokens per chunk, one of 1, 2, 4, 8, 16, 32             */
  int32_t mlp_hidden;     /* F: predictor hidden width, 128 or 256                      */
  int32_t top_k;          /* chunks selected per step, >= 1; >= T/C selects all         */
  int32_t n_res;          /* residual rows per (batch, KV head), 0 .. T                 */
  int32_t act;            /* LOWRAM_ACT_*                                               */
  int32_t dtype;          /* LOWRAM_DTYPE_*                                             */
  int32_t decode_variant; /* LOWRAM_DECODE_*                                            */
  int32_t res_format;     /* LOWRAM_RES_*                                               */
  int32_t n_positions;    /* RoPE positions of the original prefix, 0 .. n_positions-1;
                             0 means n_tokens. Larger than n_tokens only for a cache whose
                             chunks were evicted (lowram_evict): the cache then holds
                             n_tokens tokens of kept chunks and cache->chunk_pos gives each
                             stored chunk's original index. A multiple of chunk.          */
  int32_t reserved;       /* must be 0                                                  */
  double rope_theta;      /* RoPE base; theta_i = rope_theta^(-2i/d)                    */
} lowram_config;

/* One layer's parameters (inputs; never written).
 *   basis [H_kv*d][r]   columns orthonormal (precondition, not checked); shared by the two
 *                       layers of an xKV group ("adjacent layers share the SVD basis")
 *   w1 [H_kv][F][d], b1 [H_kv][F], w2 [H_kv][d][F], b2 [H_kv][d]:
 *                       per-head predictor V_hat = w2 act(w1 x + b1) + b2 (x = pre-RoPE key)
 */
typedef struct lowram_layer_params {
  const void* basis;
  const void* w1;
  const void* b1;
  const void* w2;
  const void* b2;
} lowram_layer_params;

/* One layer's compressed cache (written by lowram_encode, read by lowram_decode_step).
 *   coef      [B][T][r]          low-rank key coefficients c_t = basis^T RoPE^-1(K_t)
 *   landmark  [B][H_kv][T/C][d]  mean post-RoPE key of each chunk
 *   res_idx   [B][H_kv][n_res]   int32 token indices of the residual rows, ascending
 *   res_val   [B][H_kv][n_res][d] residual corrections V_t - V_hat_t
 *   chunk_ptr [B][H_kv][T/C + 1] int32 CSR: rows of chunk c are ptr[c] .. ptr[c+1]-1
 *   landmark_norm [B][H_kv]      fp32 upper bound of max_c |landmark_c|_2 of each (b, h).
 *                                Not part of the method: decode uses it to bound the fp32
 *                                score error near the top-k threshold. lowram_encode
 *                                writes it; lowram_landmark_norms recomputes it for a
 *                                cache built elsewhere. A value below the true maximum
 *                                can change the selection.
 *   chunk_pos [B][T/C]           int32 original chunk index of each stored chunk,
 *                                ascending (eviction; RoPE is re-applied at position
 *                                chunk_pos*C + j). NULL when n_positions == n_tokens.
 *   res_scale [B][H_kv][n_res][d/32] fp16 scales of int4 residual rows (res_format
 *                                INT4_G32; res_val then holds [B][H_kv][n_res][d/2] bytes
 *                                of codes). NULL otherwise.
 * The layout is fixed by these shapes, so a cache can be saved and restored byte for
 * byte (lowram_cache_layout gives the eight sizes). res_idx, res_val and res_scale may be
 * NULL when n_res == 0. With eviction, decode selects among the stored chunks: sel_out
 * holds stored-chunk indices (map them through chunk_pos). */
typedef struct lowram_cache {
  void* coef;
  void* landmark;
  int32_t* res_idx;
  void* res_val;
  int32_t* chunk_ptr;
  float* landmark_norm;
  int32_t* chunk_pos;
  void* res_scale;
} lowram_cache;

typedef struct lowram_ctx lowram_ctx;

/* Validate a configuration on the host only (no CUDA call). Returns LOWRAM_OK or the
 * first failing check's status. */
lowram_status lowram_check_config(const lowram_config* cfg);

/* Create a context on `device`: checks cfg, builds the RoPE tables (two-level cos/sin of
 * t*theta_i, and the chunk-base cos/sin of c*C*theta_i for every chunk c < N_c:
 * N_c*d/2 fp32 pairs, 8 MiB at 128K tokens, chunk 8, d 128; all computed in fp64 on the
 * host, stored fp32 and fp64 on the device) and the counters. *out is set only on
 * success. Destroy with lowram_destroy. */
lowram_status lowram_create(const lowram_config* cfg, int device, lowram_ctx** out);

/* Free the context's tables. Waits for nothing: the caller must have synchronised any
 * stream still using the context. NULL is accepted. */
void lowram_destroy(lowram_ctx* ctx);

/* Host only. bytes_out[0..7] = sizes of coef, landmark, res_idx, res_val, chunk_ptr,
 * landmark_norm, chunk_pos (0 without eviction), res_scale (0 unless int4 residuals). */
lowram_status lowram_cache_layout(const lowram_config* cfg, size_t bytes_out[8]);

/* Host only. Workspace bytes needed by op (LOWRAM_OP_ENCODE or LOWRAM_OP_DECODE). The
 * workspace needs no initialisation and holds nothing between calls. */
lowram_status lowram_workspace_size(const lowram_config* cfg, int op, size_t* bytes);

/* Encode one layer's prefix into `out` (all five arrays written).
 *   k_cache [B][T][H_kv][d]  post-RoPE keys;  v [B][T][H_kv][d] values.
 * Steps (agihunt summary, key paragraph and value-amortisation paragraph; cctest "How
 * the method works": Low-rank keys, Amortised values, Residuals for difficult tokens):
 * invert RoPE, project onto the basis (coef stored rounded), landmarks = chunk means of
 * the original keys, squared predictor error of every token with the unrounded
 * coefficients, per (batch, KV head) the n_res largest errors (ties to the lower token;
 * candidates near the threshold re-scored in fp64), residual rows against the stored
 * coefficients, chunk CSR. */
lowram_status lowram_encode(lowram_ctx* ctx, const void* k_cache, const void* v,
                            const lowram_layer_params* params, const lowram_cache* out,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Eviction before compression (LowRAM-E / LowRAM-EQ: eviction composes with the method,
 * agihunt summary, composition paragraph). For every batch element, keeps the
 * n_tokens / C chunks of the n_positions-token prefix with the largest all-head landmark
 * norm (sum over KV heads of |landmark|^2, landmarks as lowram_encode stores them: the
 * fp32 chunk mean rounded to the cache dtype; norms summed in fp64), ties to the lower
 * chunk, and copies their keys and values out in ascending order.
 *   k_full, v_full [B][n_positions][H_kv][d] (post-RoPE keys, values; inputs);
 *   k_kept, v_kept [B][n_tokens][H_kv][d] (written);
 *   chunk_pos [B][n_tokens / C] int32 (written): the kept chunks' original indices,
 *   ascending; pass it as cache->chunk_pos to lowram_encode and to decode.
 * Workspace: lowram_workspace_size(cfg, LOWRAM_OP_EVICT). Needs n_positions > n_tokens. */
lowram_status lowram_evict(lowram_ctx* ctx, const void* k_full, const void* v_full,
                           void* k_kept, void* v_kept, int32_t* chunk_pos, void* workspace,
                           size_t workspace_bytes, void* stream);

/* The xKV basis of one layer group from its keys, by a randomised range finder with
 * Cholesky-QR in place of an exact SVD (agihunt summary, key paragraph: adjacent layers
 * share one SVD basis, computed by a randomised Cholesky-QR instead of the exact SVD).
 * With A the group's pre-RoPE key rows (every token of every layer and batch element,
 * flattened over D = H_kv*d):
 *   Y = A^T A omega;  Q = CholQR2(Y);  n_power times: Q = CholQR2(A^T A Q);
 *   S = Q^T A^T A Q = U diag(lambda) U^T (Rayleigh-Ritz);  basis = Q U[:, :r]
 * with the columns of U by decreasing lambda (ties to the lower index), CholQR2 = Q from
 * Cholesky-QR applied twice (Y^T Y = R^T R, Q = Y R^-1). All in fp64 (A^T A formed once
 * as a D x D Gram matrix; the eigenproblem by Jacobi rotations). Each column of the
 * result is defined up to its sign.
 *   k_layers  HOST array of n_layers (1..8) device pointers, each [B][T][H_kv][d] post-RoPE
 *             keys of one layer of the group (the context's sizes; no eviction);
 *   omega     [D][l] fp64 random test matrix (input), r <= l <= min(D, 256);
 *   basis_out [D][r] in cfg->dtype (written): orthonormal columns.
 * Workspace: lowram_fit_basis_workspace_size. Cholesky-QR needs Y of full column rank:
 * keys of rank below l make a pivot non-positive, which lowram_last_error reports as
 * LOWRAM_ERR_DEVICE_CHECK (the result is then not valid). */
lowram_status lowram_fit_basis(lowram_ctx* ctx, const void* const* k_layers, int32_t n_layers,
                               const double* omega, int32_t l, int32_t n_power,
                               void* basis_out, void* workspace, size_t workspace_bytes,
                               void* stream);
lowram_status lowram_fit_basis_workspace_size(const lowram_config* cfg, int32_t l,
                                              size_t* bytes);

/* One decode step of one layer.
 *   q   [B][H_q][d]  post-RoPE queries (input)
 *   out [B][H_q][d]  attention output (written)
 *   sel_out [B][H_kv][k] int32, k = min(top_k, T/C): the selected chunks, ascending
 *           (written when not NULL)
 * Steps (agihunt summary, key paragraph; cctest "Selective reconstruction"; abstract):
 * score every chunk by max over the GQA group of q . landmark, select the top-k (ties to
 * the lower chunk; candidates near the threshold re-scored in fp64), rebuild the selected
 * chunks' keys from coef and basis and re-apply RoPE, predict their values with the
 * per-head MLP plus the stored residuals, and attend over them with scale 1/sqrt(d).
 * Rebuilt keys and values never reach global memory. */
lowram_status lowram_decode_step(lowram_ctx* ctx, const lowram_cache* cache,
                                 const lowram_layer_params* params, const void* q,
                                 void* out, int32_t* sel_out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* One decode step over the compressed prefix plus an uncompressed suffix of generated
 * tokens (long generation keeps recent tokens uncompressed until they are compressed in
 * turn; agihunt summary, limitations paragraph). One softmax spans the selected chunks'
 * rebuilt tokens and every suffix token:
 *   k_suffix, v_suffix [B][s_max][H_kv][d] (post-RoPE keys, values; bf16), rows
 *   0 .. n_suffix-1 valid (0 <= n_suffix <= s_max; NULL allowed when n_suffix == 0);
 *   q, out, sel_out as in lowram_decode_step.
 * The compressed part runs as in lowram_decode_step with its output kept in fp32; the
 * suffix is attended by the dense flash-decode kernel and the two merged by their
 * softmax statistics. Workspace: lowram_suffix_workspace_size(cfg, s_max). bf16 with
 * d = 128 and G = 4 only (LOWRAM_ERR_UNSUPPORTED otherwise). */
lowram_status lowram_decode_step_suffix(lowram_ctx* ctx, const lowram_cache* cache,
                                        const lowram_layer_params* params, const void* q,
                                        const void* k_suffix, const void* v_suffix,
                                        int32_t s_max, int32_t n_suffix, void* out,
                                        int32_t* sel_out, void* workspace,
                                        size_t workspace_bytes, void* stream);
lowram_status lowram_suffix_workspace_size(const lowram_config* cfg, int32_t s_max,
                                           size_t* bytes);

/* Periodic re-compression of the generated suffix (agihunt summary, limitations
 * paragraph: long generation keeps the generated suffix dense and compresses it
 * periodically). A block of whole chunks of generated tokens is compressed with
 * lowram_encode under its own context (same basis and predictor; configuration
 * n_tokens = the block's tokens, n_positions > n_tokens, and cache->chunk_pos = the
 * block's chunk positions, so RoPE is inverted at the tokens' true positions; its own
 * n_res residual rows chosen within the block). lowram_append then writes into `dst` the
 * cache of the prefix followed by the block:
 *   coef, landmark: the prefix's tokens / chunks, then the block's;
 *   res_idx, res_val, res_scale: per (b, h) the prefix's n_res_p rows, then the block's
 *   (token indices moved by the prefix's n_tokens);
 *   chunk_ptr: the prefix's offsets, then the block's moved by n_res_p;
 *   landmark_norm: the larger of the two bounds;
 *   chunk_pos (written when dst's configuration has n_positions > n_tokens): the
 *   prefix's (0, 1, ... when it has none), then the block's.
 * When dst has no chunk_pos, the block's chunk_pos must be N_p, N_p + 1, ... (N_p the
 * prefix's chunk count): checked on the device, LOWRAM_ERR_DEVICE_CHECK through
 * lowram_last_error(dst_ctx) otherwise, the copies still made.
 * The three configurations must agree in batch, heads, head_dim, rank, chunk,
 * mlp_hidden, act, dtype and res_format, with dst n_tokens = prefix n_tokens + block
 * n_tokens and dst n_res = prefix n_res + block n_res (LOWRAM_ERR_SHAPE otherwise).
 * dst must not overlap the sources. coef, landmark and res_val of all three 16-byte
 * aligned. Asynchronous on `stream`; no workspace. */
lowram_status lowram_append(lowram_ctx* dst_ctx, const lowram_cache* dst,
                            const lowram_ctx* prefix_ctx, const lowram_cache* prefix,
                            const lowram_ctx* block_ctx, const lowram_cache* block,
                            void* stream);

/* Decode sub-step 1 (kernel (a) alone): score every chunk by max over the GQA group of
 * q . landmark and write the top-k chunks per (batch, KV head), ascending, ties to the
 * lower chunk (agihunt summary, key paragraph; cctest "Selective reconstruction").
 *   landmark [B][H_kv][T/C][d]; landmark_norm [B][H_kv] fp32 (the cache field);
 *   q [B][H_q][d]; sel_out [B][H_kv][k] int32 (written).
 * Uses the decode workspace. lowram_decode_step = this + lowram_attend_selected. */
lowram_status lowram_select_chunks(lowram_ctx* ctx, const void* landmark,
                                   const float* landmark_norm, const void* q, int32_t* sel_out,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Write landmark_norm [B][H_kv] (fp32, rounded up) = max over chunks c of |landmark_c|_2,
 * summed in fp64, for a cache whose landmarks were produced outside lowram_encode (which
 * writes the field itself). landmark [B][H_kv][T/C][d] is read only. */
lowram_status lowram_landmark_norms(lowram_ctx* ctx, const void* landmark, float* landmark_norm,
                                    void* stream);

/* Decode sub-step 2 (kernel (b) + split-K combine): rebuild the chunks listed in sel
 * ([B][H_kv][k] int32, k = min(top_k, T/C), each entry in 0 .. T/C-1; out-of-range
 * entries are skipped and reported through lowram_last_error) and attend over them.
 *   q [B][H_q][d] (input); out [B][H_q][d] (written). Uses the decode workspace. */
lowram_status lowram_attend_selected(lowram_ctx* ctx, const lowram_cache* cache,
                                     const lowram_layer_params* params, const void* q,
                                     const int32_t* sel, void* out, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* lowram_decode_step with its scratch in a fixed device array of the library instead of
 * a caller workspace. The paper has no counterpart: it is an interface for callers that
 * cannot allocate device memory where they decode (a fully reserved memory pool, a
 * runtime that forbids allocation after start-up, a plugin without an allocator). The
 * call itself allocates nothing; arguments and results are those of lowram_decode_step.
 *   - The array holds 32 MiB and lives on every device that loads the library until the
 *     process exits (or the device's context is destroyed, e.g. by cudaDeviceReset). A
 *     configuration whose decode workspace (lowram_workspace_size) is larger is refused
 *     with LOWRAM_ERR_WORKSPACE, before anything else is checked and with nothing
 *     launched.
 *   - The first call on a device, and the first call after that device's context was
 *     destroyed and created again, looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); the address is cached with the
 *     context's unique id. Make such a first call before any stream capture.
 *   - Every call on a device shares the one array, which keeps whatever the last call
 *     left. The decode step needs none of it zeroed: it writes all it reads. Calls that
 *     overlap on the GPU (other streams, other threads, other contexts) race on it:
 *     serialise them. */
lowram_status lowram_decode_step_static(lowram_ctx* ctx, const lowram_cache* cache,
                                        const lowram_layer_params* params, const void* q,
                                        void* out, int32_t* sel_out, void* stream);

/* The uncompressed baseline the method is measured against (the pages compare decode
 * throughput with the uncompressed model and report about five times its peak decode
 * throughput at 262K tokens: agihunt summary, efficiency paragraph; cctest "How the
 * method works", Selective reconstruction; abstract): exact GQA decode attention over the
 * full bf16 cache, out_g = sum_t softmax_t(q_g . K_t / sqrt(d)) V_t over every position
 * t < T, for each query head g.
 *   k_cache [B][T][H_kv][d], v [B][T][H_kv][d] (post-RoPE keys and values, bf16, as
 *   lowram_encode takes them); q [B][H_q][d]; out [B][H_q][d] (written).
 * Uses the context's sizes and device only (rank, chunk, predictor and residual settings
 * are ignored). Workspace: lowram_workspace_size(cfg, LOWRAM_OP_DENSE). bf16 with d = 128
 * and G = 4 only (LOWRAM_ERR_UNSUPPORTED otherwise). */
lowram_status lowram_dense_decode(lowram_ctx* ctx, const void* k_cache, const void* v,
                                  const void* q, void* out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Synchronise the device, then return and clear the context's status word: LOWRAM_OK,
 * LOWRAM_ERR_DEVICE_CHECK (a kernel met a residual index outside its chunk or a CSR
 * offset out of range, and skipped it) or LOWRAM_ERR_TIMEOUT (a bounded wait expired;
 * the kernel returned early and its outputs are not valid). */
lowram_status lowram_last_error(lowram_ctx* ctx);

/* Static string naming a status. */
const char* lowram_status_string(lowram_status status);

/* Test only: lowram_attend_selected on the tensor-core kernel (LOWRAM_ERR_UNSUPPORTED
 * where it does not apply) that also stores the rows it rebuilds, at the points where its
 * epilogue holds them, so they can be compared element by element with the method's
 * rebuilt keys and values (only the top-k chunks are rebuilt: agihunt summary, key
 * paragraph; cctest "Residuals for difficult tokens"). Rows are in selection order:
 * row = (b*H_kv + h)*k*C + s*C + j for token j of the chunk sel[b][h][s]; rows = B*H_kv*k*C
 * with k = min(top_k, T/C). All three outputs are device fp32 arrays, zeroed first:
 *   k_rot [rows][d]  the rebuilt key with RoPE re-applied (epilogue part A);
 *   h_act [rows][F]  act(W1 K~_pre + b1), the hidden layer (epilogue part B);
 *   v_rec [rows][d]  the rebuilt value W2 h_act + b2 + R_t (R_t: the token's stored
 *                    residual row, read where part B reads it; W2 and b2 applied by a
 *                    small separate kernel, since the decode kernel applies W2 only after
 *                    the attention sum).
 * out is written as by lowram_attend_selected. */
lowram_status lowram_debug_reconstruct(lowram_ctx* ctx, const lowram_cache* cache,
                                      const lowram_layer_params* params, const void* q,
                                      const int32_t* sel, void* out, float* k_rot,
                                      float* h_act, float* v_rec, void* workspace,
                                      size_t workspace_bytes, void* stream);

/* Test only: the tensor-core attend kernel launched as if it followed a selection launch
 * in the same decode step, so it waits on every (batch, KV head)'s ready flag; no
 * selection runs in this call and the flags stay clear, so its first wait gives up after
 * its bound (about 2 s), the kernel drains its own copies and MMAs, frees its Tensor
 * Memory and returns. lowram_last_error then reports LOWRAM_ERR_TIMEOUT, out is not
 * valid, and the context serves the next call normally. LOWRAM_ERR_UNSUPPORTED where the
 * tensor-core kernel does not apply. */
lowram_status lowram_debug_attend_unpublished(lowram_ctx* ctx, const lowram_cache* cache,
                                              const lowram_layer_params* params, const void* q,
                                              const int32_t* sel, void* out, void* workspace,
                                              size_t workspace_bytes, void* stream);

/* Test only (no counterpart in the method): one 128 x 128 tcgen05 tile product
 * d[m][n] = sum_k a[m][k] * b[n][k] with a [128][K], b [128][K] bf16 row-major (device)
 * and d [128][128] fp32 (device), staged through the same shared-memory layouts and
 * descriptors as the tensor-core decode kernel.
 *   mode 0: K % 32 == 0, 32 <= K <= 256; a and b TMA-loaded with the 64-byte swizzle
 *           (a in 8-row boxes like the gathered coefficients, b like the basis);
 *   mode 1: K == 128; a TMA-loaded with the 128-byte swizzle (like W1), b stored by
 *           threads in the 128-byte-swizzled layout (like the rebuilt keys);
 *   mode 2: K == 128; a stored by threads into Tensor Memory (row m in lane m, two bf16
 *           per column) and used as the MMA's A operand, b rows 0..15 stored by threads
 *           with the 128-byte swizzle; only d[m][0..15] is written.
 * Synchronous: returns after the kernel finished. */
lowram_status lowram_debug_tc_tile(const void* a, const void* b, float* d, int32_t k,
                                   int32_t mode, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* LOWRAM_H */
