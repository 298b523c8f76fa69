/*
 * rest.h -- C ABI of the ReST encode-once / decode-many ranking forward on
 * NVIDIA B200 (sm_100a).
 *
 * The method is the one described in "From Language to Behavior" (a close
 * reading of the ReST paper, arXiv 2609.01240): a causal Dual-Gated-Attention
 * encoder T run once per user history (§3.2, eqs. 3-6) and a projection-free,
 * token-specific cross decoder C run for every candidate against T's output
 * (§3.3, eqs. 7-8), served with a shared prefix (§3.5).
 *
 * Conventions for every entry point
 *   - Matrices are row-major; a projection is x . W with W stored [d_in, d_out].
 *   - "dev" pointers are CUDA device memory owned by the caller (for example
 *     allocated by PyTorch); "host" pointers are ordinary host memory read
 *     before the call returns. The library never frees or keeps any pointer,
 *     and allocates no device memory: all scratch lives in the caller's
 *     workspace `ws` of at least rest_workspace_size() bytes.
 *   - Every dev pointer must be 16-byte aligned.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream). Host-detectable errors are returned
 *     synchronously before anything is enqueued. Errors found on the device
 *     (decreasing timestamps, a bounded wait that ran out) are written to the
 *     int32 word `*dev_err` (dev, may be NULL to ignore them). Each call
 *     clears the word on `stream` before its first kernel, so after
 *     synchronizing it holds this call's status (0 = no device error).
 *   - An empty batch (no tokens, or no candidates) is a successful no-op.
 *   - No C++ exception crosses this boundary.
 *   - REST_F32 computes with fp32 storage throughout. REST_BF16 takes bf16
 *     inputs and weights, multiplies bf16 operands with fp32 accumulation,
 *     keeps the residual stream, softmax statistics and gates in fp32, and
 *     stores the activations that feed a matrix product in bf16.
 */
#ifndef REST_H_
#define REST_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  REST_OK = 0,
  REST_ERR_INVALID_ARG = 1,   /* a shape, pointer, alignment or index argument is invalid */
  REST_ERR_UNSORTED_TIME = 2, /* (device) a user's timestamps decrease */
  REST_ERR_UNSUPPORTED = 3,   /* valid but not supported (e.g. head_dim outside the built set) */
  REST_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch, copy, device query) */
  REST_ERR_TIMEOUT = 5,       /* (device) a bounded wait inside a kernel ran out */
  REST_ERR_WORKSPACE = 6,     /* ws is NULL or smaller than rest_workspace_size() */
  REST_ERR_NO_DEVICE = 7,     /* no CUDA device of compute capability 10.0 is current */
  REST_ERR_RANGE = 8          /* (device) a decoder query or memory value is beyond the fp16 range
                                 (|v| > 65504) that the bf16 tensor-core decoder computes in */
} rest_status;

typedef enum { REST_F32 = 0, REST_BF16 = 1 } rest_dtype;

/* Attention-head split (§3.2.2, eq. 5). Head h owns columns
 * h*head_dim .. (h+1)*head_dim-1 of every d-wide activation. */
typedef struct {
  int d;               /* model width, == n_heads * head_dim */
  int n_heads;
  int head_dim;        /* even; REST_BF16 supports 32 and 64, REST_F32 16, 32 and 64 */
  const int64_t* tau;  /* host [n_heads]: 0 = RoPE head (ordinal position),
                          > 0 = RoTE head with time buckets of tau seconds */
  double rope_base;    /* theta_j = rope_base^(-2j/head_dim), normally 10000 */
} rest_heads;

/* Packed, padding-free histories: user u owns rows cu_seqlens[u] ..
 * cu_seqlens[u+1]-1 of every [T, *] array, T = cu_seqlens[n_users]. */
typedef struct {
  int n_users;
  const int32_t* cu_seqlens;  /* host [n_users+1]; cu_seqlens[0] == 0, non-decreasing */
} rest_batch;

/* Gates of the attention sublayer. The DGA layer gates the value stream and
 * the attention output (eqs. 3-4). The other two are the variants of the
 * page's gated-attention ablation (§4 ablations, "gated attention"): the
 * output gate alone, and gates on Q, K and V as well as the output, with
 * q = sigmoid(y W_gq) * (y W_Q) and k = sigmoid(y W_gk) * (y W_K) taken
 * before the rotation of eq. 5 (so that scores still depend only on the
 * index difference, eq. 14). */
typedef enum {
  REST_GATES_VALUE_OUTPUT = 0, /* w_qkvgg [d, 5d]: W_Q | W_K | W_V | W_gv | W_go */
  REST_GATES_OUTPUT = 1,       /* w_qkvgg [d, 4d]: W_Q | W_K | W_V | W_go */
  REST_GATES_QKV_OUTPUT = 2    /* w_qkvgg [d, 7d]: W_Q | W_K | W_V | W_gv | W_go | W_gq | W_gk */
} rest_gates;

/* One encoder layer (Fig. 1 left): a DGA sublayer and an optional SwiGLU FFN
 * sublayer, each wrapped by SRN (eq. 6). Weights have the dtype of the call. */
typedef struct {
  const void* w_qkvgg;   /* dev [d, 5d]: column blocks W_Q | W_K | W_V | W_gv | W_go (eqs. 3-4);
                            other widths and blocks with the gate variants (rest_gates) */
  const void* w_o;       /* dev [d, d] */
  const void* w_ffn13;   /* dev [d, 2*d_ff]: W_1 | W_3, or NULL for an attention-only layer */
  const void* w_ffn2;    /* dev [d_ff, d] (ignored when w_ffn13 is NULL) */
  const float* ln_attn_g; /* dev [d] fp32 LayerNorm gain/bias of the attention sublayer */
  const float* ln_attn_b;
  const float* ln_ffn_g;  /* dev [d] fp32, of the FFN sublayer (ignored without FFN) */
  const float* ln_ffn_b;
  float alpha_attn;      /* SRN residual scale of each sublayer */
  float alpha_ffn;
  int d_ff;              /* FFN width, a multiple of 64 (0 without FFN) */
  int gates;             /* a rest_gates value; 0 is the DGA layer */
} rest_enc_layer;

/* Cross-decoder parameters (§3.3): token-specific W_Q and W_go (eq. 8), a
 * shared W_o. Weights have the dtype of the call. */
typedef struct {
  int K;              /* query tokens per candidate, 1..8 ([CLS], ad, user: K = 3) */
  const void* w_q;    /* dev [K, d, d] */
  const void* w_go;   /* dev [K, d, d] */
  const void* w_o;    /* dev [d, d] */
} rest_dec_params;

/* Ranking requests sharing encoded prefixes (§3.5). Request r belongs to user
 * req_user[r], reads the first req_cutoff[r] rows of that user's encoder
 * output, and scores candidates cu_cands[r] .. cu_cands[r+1]-1. */
typedef struct {
  int n_req;
  const int32_t* req_user;    /* host [n_req], 0 .. n_users-1 */
  const int32_t* req_cutoff;  /* host [n_req], 1 .. L_user */
  const int32_t* cu_cands;    /* host [n_req+1]; cu_cands[0] == 0, non-decreasing */
} rest_requests;

/* Bytes of workspace that rest_rank_request (and therefore each of the
 * entry points below) needs for this batch. `reqs` may be NULL (encoder
 * only); `n_layers`/`layers` may be 0/NULL (decoder only). Returns
 * REST_ERR_INVALID_ARG for invalid shapes. */
rest_status rest_workspace_size(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                                const rest_enc_layer* layers, int n_layers,
                                const rest_requests* reqs, int K, size_t* bytes);

/* Rotation index and table of §3.2.2 / eq. 5, the first step of the encoder.
 * For row i of user u (position p = i - cu_seqlens[u]) and head h:
 *   idx[i,h] = p                                   if tau_h == 0 (RoPE)
 *   idx[i,h] = floor((ts[i] - ts[cu_seqlens[u]]) / tau_h)   otherwise (RoTE)
 * and for j < head_dim/2, with phi = idx * rope_base^(-2j/head_dim) in fp64:
 *   cos_out[i,h,j] = cos(phi), sin_out[i,h,j] = sin(phi)   (stored fp32).
 *   ts:      dev [T] int64 seconds, non-decreasing within each user
 *            (a decrease sets *dev_err = REST_ERR_UNSORTED_TIME)
 *   idx_out: dev [T, n_heads] int64 (may be NULL)
 *   cos_out, sin_out: dev [T, n_heads, head_dim/2] fp32 (both or neither NULL)
 * Needs no workspace beyond the batch index copy: ws as for the encoder. */
rest_status rest_rotation_table(const rest_heads* heads, const rest_batch* batch, const int64_t* ts,
                                int64_t* idx_out, float* cos_out, float* sin_out,
                                void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* Encoder T (§3.2, eqs. 3-6; Fig. 1 left): n_layers layers over the packed
 * histories. Layer l (1-based) uses post-LN when l <= l_switch and pre-LN
 * otherwise (eq. 6). Each DGA sublayer computes, per head and per user,
 * causal softmax(q k^T / sqrt(head_dim)) over rotated q, k (eq. 5) against the
 * value-gated V' = sigmoid(x W_gv) * (x W_V), then the output gate
 * sigmoid(x W_go) and W_o (eqs. 3-4).
 *   x:     dev [T, d] (dtype of the call)  history features s_i
 *   ts:    dev [T] int64 timestamps t_i in seconds
 *   layers: host [n_layers]
 *   h_out: dev [T, d] (dtype of the call)  the encoder memory H
 */
rest_status rest_encoder_attn(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                              const void* x, const int64_t* ts,
                              const rest_enc_layer* layers, int n_layers, int l_switch,
                              void* h_out, void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* Cross decoder C (§3.3, eq. 7 with the token-specific weights of eq. 8).
 * For every request r, candidate n, query token k:
 *   q = z[n,k] W_Q^(k),  g = sigmoid(z[n,k] W_go^(k)),
 *   per head: o_h = softmax(q_h H_h^T / sqrt(head_dim)) H_h over the first
 *   req_cutoff[r] rows of the user's H (keys and values are H itself),
 *   y[n,k] = (o * g) W_o.
 * Every H tile is staged once per request and head and read by all of the
 * request's candidate query rows (the shared prefix).
 *   h:     dev [T, d] (dtype of the call)  encoder memory
 *   z:     dev [N_total, K, d] (dtype of the call)  candidate query tokens
 *   y_out: dev [N_total, K, d] fp32
 */
rest_status rest_cross_decode(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                              const void* h, const rest_requests* reqs, const void* z,
                              const rest_dec_params* dec, float* y_out,
                              void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* Size in bytes of the scratch array that rest_cross_decode_static_ws uses. */
#define REST_STATIC_WS_BYTES (32u * 1024u * 1024u)

/* REST_STATIC_WS_BYTES as the library was built with it (for bindings that
 * cannot read this header). */
size_t rest_static_ws_bytes(void);

/* rest_cross_decode without a workspace argument. The paper has no
 * counterpart to this entry point; it exists for callers that cannot
 * allocate device memory themselves. Examples: a plain-C host program
 * linking only this library (it has no device allocator of its own), and a
 * serving process whose device memory is all handed to a fixed arena at
 * start-up, after which nothing may call cudaMalloc.
 *
 * The decoder's scratch (index/tile lists and the per-row q, g and o
 * buffers) lives in one REST_STATIC_WS_BYTES array in the library's device
 * image instead. The caller still passes inputs and outputs exactly as for
 * rest_cross_decode, with the same meaning, and the same results.
 *   - The CUDA runtime loads the library's device image, and with it the
 *     array, on a device's first call of this entry point (lazy module
 *     loading). From then on that GPU holds the array until the process
 *     exits. A call with no candidates (n_req = 0, or no candidates in any
 *     request) loads it too and does nothing else: make one such call per
 *     device, with that device current, before handing device memory to an
 *     arena and before any CUDA stream capture.
 *   - Every call looks up the array's address in the current device's
 *     context, so `stream` must belong to the current device.
 *   - A batch whose scratch would exceed the array returns
 *     REST_ERR_WORKSPACE; rest_workspace_size() with n_layers = 0 tells the
 *     bytes a batch needs.
 *   - This entry point calls no cudaMalloc, cudaFree or other allocating
 *     routine.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Nothing in it needs to start at zero. Calls whose work overlaps on the
 *     GPU (different streams, or different host threads without ordering)
 *     race on it: order them on one stream. */
rest_status rest_cross_decode_static_ws(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                                        const void* h, const rest_requests* reqs, const void* z,
                                        const rest_dec_params* dec, float* y_out, int32_t* dev_err,
                                        void* stream);

/* Shared-prefix serving (§3.5): the encoder runs once over the packed
 * histories and the decoder scores every candidate of every request against
 * its output: FLOPs(T) + N * FLOPs(C) instead of N * (FLOPs(T) + FLOPs(C)).
 * Arguments as in rest_encoder_attn and rest_cross_decode; h_out receives H. */
rest_status rest_rank_request(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                              const void* x, const int64_t* ts,
                              const rest_enc_layer* layers, int n_layers, int l_switch,
                              const rest_requests* reqs, const void* z, const rest_dec_params* dec,
                              void* h_out, float* y_out,
                              void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* Append-only encoder cache. The encoder's attention is causal (eqs. 3-5),
 * its other steps act row by row, and RoTE counts time from a history's first
 * timestamp (§3.2.2), which appending leaves in place; so the encoder state of
 * a history's first c tokens does not change when tokens are appended after
 * them (§3.5 uses the same fact for the prefix a request reads). The cache
 * keeps, for every layer and cached token, the rotated key R k and the gated
 * value V' = sigmoid(y W_gv) * (y W_V) that later tokens attend to, and
 * optionally the token's row of H.
 *
 * User u owns rows cu_cap[u] .. cu_cap[u+1]-1 of every cache array; its first
 * len[u] rows hold positions 0 .. len[u]-1 of its history. The arrays are
 * caller-owned device memory in the call's dtype, [rows, d] each. Rows that
 * hold no cached token must hold finite values (allocate the arrays
 * zero-filled): the attention reads keys in blocks of 128 rows and weights the
 * rows past a user's last key by zero, and zero times a NaN is NaN.
 *
 * With h set, the cache's H rows serve rest_cross_decode directly: pass
 * {n_users, cu_cap} as its batch and keep every cutoff within len[u]. */
typedef struct {
  void* const* k;          /* host [n_layers]: dev [rows, d] arrays, R k of layer l */
  void* const* v;          /* host [n_layers]: dev [rows, d] arrays, V' of layer l */
  void* h;                 /* dev [rows, d]: H rows, or NULL */
  long long rows;          /* rows of each array, < 2^31 */
  const int32_t* cu_cap;   /* host [n_users+1]: cu_cap[0] == 0, non-decreasing, cu_cap[n_users] <= rows */
  const int32_t* len;      /* host [n_users]: cached tokens of each user */
  const int64_t* t_first;  /* host [n_users]: timestamp of the user's first cached token (read when len[u] > 0) */
  const int64_t* t_last;   /* host [n_users]: timestamp of the user's last cached token (read when len[u] > 0) */
} rest_kv_cache;

/* Workspace bytes rest_encoder_append needs for these new tokens. */
rest_status rest_append_workspace_size(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                                       const rest_enc_layer* layers, int n_layers, size_t* bytes);

/* Encodes tokens appended to cached histories, computing only their rows:
 * the result equals rows len[u] .. len[u]+n_u-1 of rest_encoder_attn over
 * each user's whole history (positions continue after the cached ones and
 * RoTE time counts from t_first[u]).
 *   batch: the new tokens, packed: user u's n_u new tokens are rows
 *          cu_seqlens[u] .. cu_seqlens[u+1]-1 of x and ts
 *   x:     dev [T_new, d] (dtype of the call)
 *   ts:    dev [T_new] int64 seconds, non-decreasing within each user and not
 *          below t_last[u] (a decrease sets *dev_err = REST_ERR_UNSORTED_TIME)
 *   cache: len[u] + n_u must fit user u's region (else REST_ERR_INVALID_ARG);
 *          cache->k and cache->v hold n_layers arrays
 *   h_out: dev [T_new, d] (dtype of the call)  the new rows of H
 * For every layer the call writes the new tokens' R k and V' into the cache
 * at rows cu_cap[u] + len[u] + i (and H there too when cache->h is set). It
 * changes none of the host arrays: afterwards user u has len[u] + n_u cached
 * tokens, whose first timestamp is t_first[u] (the first new one when len[u]
 * was 0) and whose last is the last new one. */
rest_status rest_encoder_append(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                                const void* x, const int64_t* ts,
                                const rest_enc_layer* layers, int n_layers, int l_switch,
                                const rest_kv_cache* cache, void* h_out,
                                void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* The causal attention core of a DGA sublayer for training, forward and
 * backward (ULT, §3.5: the union history of a user's training samples is
 * encoded once under a prefix-valid causal mask; a sample ending at row c
 * reads rows < c, and with row i seeing rows j <= i only that mask is the
 * causal mask on the union sequence). Per user (batch) and head h:
 *   S = q k^T / sqrt(head_dim) over j <= i,  P = softmax(S),  O = P V,
 * with q, k the rotated queries and keys and V the gated values V' (eq. 3);
 * the output gate is not part of it. */

/* Workspace bytes rest_attn_forward and rest_attn_backward need. */
rest_status rest_attn_workspace_size(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                                     size_t* bytes);

/*   q, k, v: dev [T, d] (dtype of the call)
 *   o:       dev [T, d] (dtype of the call)  O
 *   o_lo:    dev [T, d] bf16, or NULL: with REST_BF16, the low part of O
 *            (O = o + o_lo to about 2^-16 relative), for the backward
 *   lse:     dev fp32 [T, n_heads]  log sum_{j <= i} exp(S_ij), the statistic the backward reuses */
rest_status rest_attn_forward(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                              const void* q, const void* k, const void* v, void* o, void* o_lo, float* lse,
                              void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* Gradients of a scalar loss L through the core, from d_o = dL/dO (dev [T, d],
 * dtype of the call) and the forward's o, o_lo (may be NULL) and lse:
 *   dV = P^T dO,  dS = P * (dO V^T - rowsum(dO * O)),
 *   dq = dS k / sqrt(head_dim),  dk = dS^T q / sqrt(head_dim).
 * rowsum(dO * O) takes O = o + o_lo when o_lo is given: a row with few keys
 * subtracts nearly equal terms in dS, and O's bf16 rounding alone would show.
 *   dq, dk, dv: dev fp32 [T, d], overwritten. */
rest_status rest_attn_backward(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                               const void* q, const void* k, const void* v, const void* o, const void* o_lo,
                               const float* lse, const void* d_o, float* dq, float* dk, float* dv,
                               void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* Decoder block and candidate score ("From Language to Behavior", §3.3.2
 * eq. 8 and Fig. 1 right; the wiring the page leaves open is fixed as: a
 * residual on the query token, a pre-LN feed-forward sublayer whose LN and
 * SwiGLU weights are specific to the token type, and a linear logit on
 * token 0, [CLS]). For candidate n and token k:
 *   a = z[n,k] + y[n,k];  u = LN_k(a);
 *   f[n,k] = a + (SiLU(u W_1^(k)) * (u W_3^(k))) W_2^(k);
 *   score[n] = f[n,0] . w_s + b_s.
 * All weights are device memory: w_ffn13 [K, d, 2 d_ff] in the call's dtype
 * (W_1^(k) in the first d_ff columns of block k, W_3^(k) after), w_ffn2
 * [K, d_ff, d] in the call's dtype, ln_g and ln_b fp32 [K, d], w_s fp32 [d]. */
typedef struct {
  const void* w_ffn13;
  const void* w_ffn2;
  const float* ln_g;
  const float* ln_b;
  const float* w_s;
  float b_s;
  int d_ff;            /* > 0, a multiple of 8 */
} rest_score_params;

/* Workspace bytes rest_score_head needs for n_cands candidates of K tokens. */
rest_status rest_score_workspace_size(rest_dtype dt, int d, int K, long long n_cands, int d_ff, size_t* bytes);

/* z: dev [n_cands, K, d] in the call's dtype (the decoder's query tokens);
 * y: dev fp32 [n_cands, K, d] (rest_cross_decode's or rest_rank_request's
 * y_out); f_out: dev fp32 [n_cands, K, d] receives f (it also holds a while
 * the block runs); score_out: dev fp32 [n_cands]. d is a multiple of 8 and at
 * most 1024, 1 <= K <= 8. Errors as for the other calls; an empty batch is a
 * no-op. */
rest_status rest_score_head(rest_dtype dt, int d, int K, long long n_cands, const void* z, const float* y,
                            const rest_score_params* sp, float* f_out, float* score_out,
                            void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* Failure-detection self-test (no GPU fault): launches n_ctas (1..1024) CTAs
 * whose threads wait, with the bounded wait every library kernel uses, on a
 * barrier that nothing completes. CTA 0 gives up after limit_cycles SM clock
 * cycles (1e6 .. 4e9) and writes REST_ERR_TIMEOUT to *dev_err (dev, required);
 * the other CTAs give up as soon as they see it. After synchronizing, the
 * word holds REST_ERR_TIMEOUT and the context is usable. */
rest_status rest_selftest_wait_timeout(int n_ctas, long long limit_cycles, int32_t* dev_err, void* stream);

/* Static description of a status code. */
const char* rest_status_string(rest_status s);

/* Number of kernel launches the library enqueued on this host thread since
 * the last call with reset != 0 (instrumentation for benchmarks). */
long long rest_launch_count(int reset);

/* Per-kernel timing (instrumentation for benchmarks; not part of the method).
 * Between rest_profile_begin() and rest_profile_end(), every kernel the
 * library launches from this host thread is bracketed by two CUDA events on
 * its own stream. rest_profile_end() waits for those events, aggregates them
 * by kernel name and writes up to max_out records to `out` (host), returning
 * the number of distinct kernels. `flops` and `bytes` are the algorithmic
 * work of the launches (the FLOPs and the bytes that must cross HBM once),
 * computed from the shapes; `name` points to a static string. */
typedef struct {
  const char* name;
  int launches;
  double ms;
  double flops;
  double bytes;
} rest_kernel_stat;
void rest_profile_begin(void);
int rest_profile_end(rest_kernel_stat* out, int max_out);

#ifdef __cplusplus
}
#endif

#endif /* REST_H_ */
