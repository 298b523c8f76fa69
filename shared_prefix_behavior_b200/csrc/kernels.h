// Internal launcher interface between the C-ABI layer (rest_api.cu) and the
// kernel translation units. Host-side C++ only; not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace rest {

// ---------------------------------------------------------------- table
struct TableParams {
  int n_heads, half;            // half = head_dim / 2
  long long tau[32];            // per head, 0 = RoPE
  double theta[64];             // theta_j = base^(-2j/head_dim)
  // fractional turns of 2^(16 k) theta_j / (2 pi), k = 0, 1, 2 (extended precision
  // on the host): idx theta_j mod 2 pi from the 16-bit pieces of idx
  double turn[3][64];
};
// Appending to cached histories: per user, the part of its history already in
// the cache. The call's packed rows cu[u] .. cu[u+1]-1 are the user's new
// tokens, at positions cached .. cached + n - 1 of its history.
struct UserAppend {
  long long t_origin;  // timestamp of the history's first token (RoTE's t_1), when cached > 0
  long long t_prev;    // timestamp of the last cached token (order check), when cached > 0
  int cached;          // tokens already cached
  int key0;            // cache row of position 0
};

// app (nullable): positions and time origins of appended tokens, as above.
cudaError_t launch_rotation_table(const int64_t* ts, const int32_t* cu, int n_users,
                                  int T, const TableParams& p, int64_t* idx_out, float* cos_out,
                                  float* sin_out, int32_t* err, cudaStream_t s,
                                  const UserAppend* app = nullptr);
// Copies row i of user u (packed by cu) of src0 / src1 to row
// app[u].key0 + app[u].cached + (i - cu[u]) of dst0 / dst1; src1, dst1 may be
// null. row_bytes is a multiple of 16.
cudaError_t launch_append_rows(const void* src0, void* dst0, const void* src1, void* dst1, const int32_t* cu,
                               const UserAppend* app, int n_users, long long T, int row_bytes, cudaStream_t s);

// ---------------------------------------------------------------- casts / norms
// The encoder's first launch, bf16 with d a multiple of 128 (up to 1024): the
// rotation table (as launch_rotation_table, without idx_out), x_res = fp32(x),
// and with y non-null y = bf16(LN(x)) with g, b (a pre-LN first sublayer's input).
cudaError_t launch_table_cast_ln(const int64_t* ts, const int32_t* cu, int n_users, int T, const TableParams& p,
                                 float* cos_out, float* sin_out, int32_t* err, const UserAppend* app,
                                 const void* x, float* xres, void* y, const float* g, const float* b, int d,
                                 cudaStream_t s);
// mode 0: y = dt(LN(x))  (pre-LN input of a sublayer)
// mode 1: x = LN(x); y = dt(x)  (post-LN after the residual add)
// mode 2: y = dt(x)  (post-LN sublayer input, no norm)
// mode 3: x = LN(x)  (post-LN, y not written)
// mode 4: x = LN(x); y = dt(LN2(x))  (post-LN, then the next sublayer's pre-LN with g2, b2)
cudaError_t launch_layernorm(bool bf16, float* x, void* y, const float* g, const float* b, int T, int d,
                             int mode, cudaStream_t s, const float* g2 = nullptr, const float* b2 = nullptr);
// Decoder block input: a = z + y (fp32, into f) and u = dt(LN_k(a)) with the
// parameters of token type k = row % K (ln_g, ln_b are [K, d]); in bf16 with
// u_lo also the low part, u_lo = bf16(LN_k(a) - u); with u16, u in fp16 instead
// (a value beyond fp16's range sets REST_ERR_RANGE in err). One warp per row.
cudaError_t launch_score_ln(bool bf16, const void* z, const float* y, float* f, void* u, void* u_lo,
                            const float* ln_g, const float* ln_b, long long rows, int d, int K, cudaStream_t s,
                            bool u16 = false, int32_t* err = nullptr);
// score[n] = f[n, 0, :] . w_s + b_s; one warp per candidate.
cudaError_t launch_score_readout(const float* f, const float* w_s, float b_s, float* score, long long n, int d, int K,
                                 cudaStream_t s);
// x_res = float(x_in)
cudaError_t launch_to_f32(bool bf16, const void* x_in, float* x_res, long long n, cudaStream_t s);
// hi = bf16(x), lo = bf16(x - hi): x as an unevaluated sum of two bf16 numbers
cudaError_t launch_split_bf16(const float* x, void* hi, void* lo, long long n, cudaStream_t s);
// hb = bf16(x) and h16 = fp16(x) (the memory of the tensor-core decoder); a
// value beyond fp16's range sets REST_ERR_RANGE in err. n a multiple of 8,
// pointers 16-byte aligned.
cudaError_t launch_split_h16(const float* x, void* hb, void* h16, long long n, int32_t* err, cudaStream_t s);
// dst = fp16(src) for a bf16 src, with the same range check
cudaError_t launch_bf16_to_f16(const void* src, void* dst, long long n, int32_t* err, cudaStream_t s);

// ---------------------------------------------------------------- GEMM
enum Epilogue {
  EPI_F32 = 0,      // out0[m, n] = acc (fp32)
  EPI_DT = 1,       // out0[m, n] = dt(acc)
  EPI_SIGMOID = 2,  // out0[m, n] = sigmoid(acc) (fp32)
  EPI_RESID = 3,    // out0[m, n] += alpha * acc (fp32 residual stream)
  EPI_QKVG = 4,     // the DGA projection epilogue (rotation, value gate, output gate)
  EPI_SWIGLU = 5,   // out0[m, j] = dt(SiLU(acc_1) * acc_3); with out1 (bf16) also its low part,
                    // out1 = bf16(value - out0)
  EPI_DECQG = 6     // decoder token-specific projections, all token types in one launch:
                    // q[n, k] = z[n, k] W_Q^(k) -> out0, sigmoid(z[n, k] W_go^(k)) -> out1
};
// Gates of the DGA projection (EPI_QKVG), with the column blocks of its weight:
//   GATES_VO    Q | K | V | Gv | Go             value and output gates (the DGA layer)
//   GATES_O     Q | K | V | Go                  output gate only
//   GATES_QKVO  Q | K | V | Gv | Go | Gq | Gk   gates on Q, K, V and the output;
//               Q and K are gated before the rotation
enum GateMode { GATES_VO = 0, GATES_O = 1, GATES_QKVO = 2 };
inline int gate_blocks(int mode) { return mode == GATES_O ? 4 : mode == GATES_QKVO ? 7 : 5; }

struct GemmArgs {
  const void* A; long long lda;   // [M, K], row stride lda elements
  const void* B; long long ldb;   // [K, N] row-major, row stride ldb elements
  int M, N, K;
  int epi;
  void* out0; void* out1; void* out2; void* out3;
  long long ldo;                  // row stride of the outputs (elements)
  const float* cos_t; const float* sin_t;  // [M, d/2] rotation table (EPI_QKVG)
  float alpha;
  int d;                          // model width (EPI_QKVG) or d_ff (EPI_SWIGLU)
  int a_f32;                      // A is fp32 even when the call's dtype is bf16
  const void* A2;                 // bf16 low part of A (A = A + A2, same layout), or null
  const void* B2;                 // EPI_DECQG: the stacked W_go [K_tok * K, N] (B is W_Q)
  int k_tok;                      // EPI_DECQG: number of token types
  // EPI_SWIGLU / EPI_RESID / EPI_F32: `groups` independent products in one
  // launch; group g reads A columns [g K, g K + K), B rows [g K, g K + K) (the
  // groups' weights stacked) and writes output columns [g W, g W + W), W the
  // output width (d_ff, resp. N). 0 or 1: one product.
  int groups;
  int gate_mode;                  // EPI_QKVG: a GateMode
  // A and B are fp16 (kind::f16 with fp16 operands); EPI_SWIGLU then writes out0
  // in fp16, and a value beyond fp16's range sets REST_ERR_RANGE
  int f16;
  // EPI_DECQG (bf16 A and B): q * alpha and sigmoid(g) written in fp16 (for the
  // tensor-core decoder's fp16 products; a value beyond fp16's range sets
  // REST_ERR_RANGE)
  int out16;
};
// Logical output columns of EPI_QKVG are [Q | K | V,Gv interleaved | Go]
// (GATES_O: [Q | K | V | Go]; GATES_QKVO: [Q,Gq | K,Gk | V,Gv interleaved | Go])
// and of EPI_SWIGLU [W1,W3 interleaved]: every group of 4 interleaved logical
// columns holds columns (2p, 2p+1) of the first block then of the second.
cudaError_t launch_gemm_simt(bool bf16, const GemmArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- attention
// Encoder work item: query positions [q0, q0 + rows) of a user. With kb1 > 0
// (appending, keys split across CTAs) it covers only the 128-key blocks
// [kb0, kb1) of the user's keys and writes partial results as split `split`.
struct EncTile { int user; int q0; int kb0; int kb1; int split; };
// Decoder work item: query rows [row0, row0 + nrows) against the first nkeys
// rows of H starting at key0; it covers the 128-key blocks [kb0, kb1) and, when
// the launch splits keys, writes partial results as split number `split`.
struct DecTile { int row0; int nrows; int key0; int nkeys; int kb0; int kb1; int split; int pad; };
struct EncAttnArgs {
  const void* q; const void* k; const void* v;  // [T, d] rotated Q, K and gated V'
  const float* gate;                            // [T, d] sigmoid(Go), or null (no output gate)
  void* out;                                    // [T, d] dt(O * gate)
  void* out_lo;                                 // [T, d] bf16 low part of the output (out + out_lo), or null
  float* lse;                                   // [T, n_heads] log sum_j exp(q k_j / sqrt(d_h)), or null
  const int32_t* cu;                            // [n_users+1]
  const EncTile* tiles; int n_tiles;
  int n_heads, d;
  float scale_log2;                             // log2(e) / sqrt(head_dim)
  long long rows;                               // T, rows of the packed arrays
  // tensor-core kernel: CTA c runs the work items (tile * n_heads + head)
  // sched[n_cta + 1 + k] for k in [sched[c], sched[c + 1])
  const int* sched; int n_cta;
  // Appending (app non-null): q, gate and out hold the new rows (packed by cu);
  // k and v are the cache arrays of key_rows rows, where user u's keys are rows
  // app[u].key0 .. app[u].key0 + app[u].cached + n_u - 1 and its new row i sits
  // at position app[u].cached + i.
  const UserAppend* app;
  long long key_rows;
  // Keys split across CTAs (tensor-core kernel, appending): per split the
  // unnormalised fp32 output [n_split, rows, d] and its reference max m (log2
  // domain) and sum l [n_split, rows, n_heads, 2]; launch_enc_combine merges
  // them, normalises, applies the gate and writes out.
  float* part_o; float* part_ml; int n_split;
};
cudaError_t launch_enc_attn_simt(bool bf16, int hd, const EncAttnArgs& a, cudaStream_t s);
cudaError_t launch_enc_combine(int hd, const EncAttnArgs& a, cudaStream_t s);

// Backward of the causal attention core (training; the forward wrote o and lse
// with the gate left out): dq, dk, dv from d_o = dL/dO.
struct AttnBwdArgs {
  const void* q; const void* k; const void* v; const void* o; const void* d_o;  // [T, d], the call's dtype
  const void* o_lo;    // [T, d] bf16 low part of o (o + o_lo), or null
  const float* lse;    // [T, n_heads]
  float* delta;        // [T, n_heads]: rowsum(dO * O) per head, written by the first kernel
  float* dq; float* dk; float* dv;  // [T, d] fp32
  const int32_t* cu;
  const EncTile* tiles; int n_tiles;  // 128-row tiles of every user (query rows, or key rows)
  int n_heads, d;
  float scale_log2;    // log2(e) / sqrt(head_dim)
  long long rows;
  // tensor-core kernel: CTA c runs the work items (key tile * n_heads + head)
  // sched[n_cta + 1 + k] for k in [sched[c], sched[c + 1]); dq starts at zero
  const int* sched; int n_cta;
};
// part 0: delta; part 1: dq (one thread per query row); part 2: dk and dv (one thread per key row)
cudaError_t launch_attn_bwd_simt(bool bf16, int hd, int part, const AttnBwdArgs& a, cudaStream_t s);

struct DecAttnArgs {
  const float* q;      // [NK, d] decoder queries (fp32; CUDA-core decoder)
  const float* g;      // [NK, d] sigmoid output gate (fp32; CUDA-core decoder)
  // the tensor-core decoder's query rows, scaled by log2(e) / sqrt(head_dim), and
  // output gate, [NK, d] fp16 each
  const void* q16; const void* g16;
  const void* h;       // [T, d] encoder memory: keys and values (the tensor-core decoder: fp16)
  const void* h_lo;    // [T, d] bf16 low part of H (H = h + h_lo), or null (CUDA-core decoder)
  void* out;           // [NK, d] o * g: fp32 (CUDA-core decoder) or fp16 (tensor-core decoder)
  void* out_lo;        // unused (null)
  const DecTile* tiles; int n_tiles;
  int n_heads, d;
  float scale_log2;
  long long key_rows;  // T, rows of h
  // split keys (n_split > 1): per split, the unnormalized O [NK, d] and the
  // reference max m (log2 domain) and sum l [NK, n_heads, 2]; combined by
  // launch_dec_combine into out (tensor-core decoder: fp16, with the fp16 gate).
  int n_split;
  long long nk_rows;   // NK
  float* part_o;
  float* part_ml;
  const int* sched; int n_cta;  // as in EncAttnArgs
};
cudaError_t launch_dec_attn_simt(bool bf16, int hd, const DecAttnArgs& a, cudaStream_t s);
cudaError_t launch_dec_combine(int hd, const DecAttnArgs& a, cudaStream_t s);

}  // namespace rest
