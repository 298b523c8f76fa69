// Plain CUDA-core kernels of the ReST forward: the rotation table, LayerNorm,
// a tiled fp32-accumulating GEMM with the fused epilogues of the encoder and
// decoder, and a thread-per-query-row flash attention for the causal
// encoder and the shared-prefix decoder. These carry the fp32 path (the
// tolerance there, 1e-4, rules out tf32/bf16 tensor cores) and every shape
// the tensor-core kernels do not cover.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace rest {

// ============================================================================
// Rotation index and cos/sin table (ReST §3.2.2, bucket definition and eq. 5)
// ============================================================================

__device__ __forceinline__ int find_user(const int32_t* cu, int n_users, int i) {
  // largest u with cu[u] <= i (empty users share their start with the next one)
  int lo = 0, hi = n_users;  // invariant: cu[lo] <= i < cu[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (cu[mid] <= i) lo = mid; else hi = mid;
  }
  return lo;
}

// floor(rel / tau) for tau > 0, exact: a double quotient corrected by integer steps
__device__ __forceinline__ long long floor_div(long long rel, long long tau) {
  long long q = (long long)floor((double)rel / (double)tau);
  while (q * tau > rel) --q;
  while ((q + 1) * tau <= rel) ++q;
  return q;
}

// sin and cos of idx * theta_j: the angle in turns is reduced modulo 1 in fp64
// from the three 16-bit pieces of idx and the host's fractional turns of
// 2^(16 k) theta_j. The reduced turns r (|r| <= 1/2) split into an fp32 part
// r_hi and a remainder r_lo (|r_lo| <= 2^-25); the library's fp32 sincospi of
// 2 r_hi (exact) is corrected to first order in the remaining angle
// d = 2 pi r_lo (|d| < 2e-7 rad, so the dropped d^2 / 2 term is below 2e-14):
// sin(a + d) ~ sin a + d cos a, cos(a + d) ~ cos a - d sin a. The result is the
// fp32 table value within about 1.5 ulp, without fp64 transcendental work.
__device__ __forceinline__ void rotation(long long idx, const TableParams& p, int j, float* sv, float* cv) {
  const double h2 = (double)(idx >> 32), h1 = (double)((idx >> 16) & 0xffff), h0 = (double)(idx & 0xffff);
  double tr = fma(h2, p.turn[2][j], fma(h1, p.turn[1][j], h0 * p.turn[0][j]));
  tr -= rint(tr);
  const float hi = (float)tr;
  const float d = 6.28318530717958648f * (float)(tr - (double)hi);
  float sa, ca;
  sincospif(2.0f * hi, &sa, &ca);
  *sv = fmaf(d, ca, sa);
  *cv = fmaf(-d, sa, ca);
}

// A block takes TB = min(256 / half, 128) consecutive tokens. Its first threads find
// each token's user and, per (token, head), the rotation index (one exact
// integer division per time head, shared by all the head's frequencies);
// then one thread per (token, frequency j) loops over the heads, so that
// consecutive threads write consecutive table entries. With `app` the rows
// are tokens appended to cached histories: positions continue after the
// cached ones and time still counts from the history's first timestamp.
constexpr int ROT_THREADS = 256;
constexpr int ROT_MAX_HEADS = 32;  // TableParams::tau
constexpr int ROT_TB_MAX = 32;     // tokens per block (256 / half from head_dim 16 on)

__host__ __device__ __forceinline__ int rot_tokens_per_block(int half) {
  return ROT_THREADS / half < ROT_TB_MAX ? ROT_THREADS / half : ROT_TB_MAX;
}

// The table's block `blk` (all threads of a block of ROT_THREADS take part).
__device__ __forceinline__ void rotation_table_block(int blk, const int64_t* __restrict__ ts,
                                                     const int32_t* __restrict__ cu, int n_users, int T,
                                                     const TableParams& p, int64_t* idx_out, float* cos_out,
                                                     float* sin_out, int32_t* err, const UserAppend* __restrict__ app) {
  __shared__ long long s_idx[ROT_TB_MAX][ROT_MAX_HEADS];
  __shared__ long long s_rel[ROT_TB_MAX], s_pos[ROT_TB_MAX];
  const int TB = rot_tokens_per_block(p.half);
  const int i0 = blk * TB;
  const int nt = min(TB, T - i0);
  const int H = p.n_heads;
  for (int k = threadIdx.x; k < nt; k += blockDim.x) {  // per token: user, time since its first token, position
    const int i = i0 + k;
    const int u = find_user(cu, n_users, i);
    const int s = cu[u];
    const int cached = app ? app[u].cached : 0;
    const long long t = ts[i];
    if (i > s ? ts[i - 1] > t : (cached > 0 && app[u].t_prev > t)) set_error(err, REST_ERR_UNSORTED_TIME);
    s_rel[k] = t - (cached > 0 ? app[u].t_origin : ts[s]);  // exact int64
    s_pos[k] = (long long)(i - s) + cached;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < nt * H; k += blockDim.x) {  // per (token, head): the rotation index
    const int tk = k / H, h = k % H;
    const long long tau = p.tau[h];
    const long long idx = tau == 0 ? s_pos[tk] : floor_div(s_rel[tk], tau);
    s_idx[tk][h] = idx;
    if (idx_out) idx_out[(long long)(i0 + tk) * H + h] = idx;
  }
  __syncthreads();
  if (!cos_out) return;
  const int tk = threadIdx.x / p.half, j = threadIdx.x % p.half;
  if (tk >= nt) return;
  const long long i = i0 + tk;
  for (int h = 0; h < H; ++h) {
    float sv, cv;
    rotation(s_idx[tk][h], p, j, &sv, &cv);
    const long long o = (i * H + h) * p.half + j;
    cos_out[o] = cv;
    sin_out[o] = sv;
  }
}

__global__ void __launch_bounds__(ROT_THREADS)
    rotation_table_kernel(const int64_t* __restrict__ ts, const int32_t* __restrict__ cu, int n_users, int T,
                          TableParams p, int64_t* idx_out, float* cos_out, float* sin_out, int32_t* err,
                          const UserAppend* __restrict__ app) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  rotation_table_block(blockIdx.x, ts, cu, n_users, T, p, idx_out, cos_out, sin_out, err, app);
}

cudaError_t launch_rotation_table(const int64_t* ts, const int32_t* cu, int n_users, int T,
                                    const TableParams& p, int64_t* idx_out, float* cos_out,
                                    float* sin_out, int32_t* err, cudaStream_t s, const UserAppend* app) {
  if (T == 0) return cudaSuccess;
  if (p.half < 1 || p.half > 64 || p.n_heads < 1 || p.n_heads > ROT_MAX_HEADS) return cudaErrorInvalidValue;
  const int tb = rot_tokens_per_block(p.half);
  const long long blocks = ((long long)T + tb - 1) / tb;
  if (cudaError_t e_ = launch_k(rotation_table_kernel, (unsigned)blocks, ROT_THREADS, 0, s, ts, cu, n_users, T, p,
                                idx_out, cos_out, sin_out, err, app)) return e_;
  return cudaGetLastError();
}

// One thread per 16 bytes of a row; rows of a user stay contiguous in the
// cache, so consecutive threads write consecutive addresses.
__global__ void append_rows_kernel(const uint4* __restrict__ src0, uint4* __restrict__ dst0,
                                   const uint4* __restrict__ src1, uint4* __restrict__ dst1,
                                   const int32_t* __restrict__ cu, const UserAppend* __restrict__ app, int n_users,
                                   long long T, int row_vecs) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= T * row_vecs) return;
  const long long i = gid / row_vecs;
  const int c = (int)(gid % row_vecs);
  const int u = find_user(cu, n_users, (int)i);
  const long long dst_row = (long long)app[u].key0 + app[u].cached + (i - cu[u]);
  dst0[dst_row * row_vecs + c] = src0[gid];
  if (src1) dst1[dst_row * row_vecs + c] = src1[gid];
}

cudaError_t launch_append_rows(const void* src0, void* dst0, const void* src1, void* dst1, const int32_t* cu,
                               const UserAppend* app, int n_users, long long T, int row_bytes, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (row_bytes % 16 != 0) return cudaErrorInvalidValue;
  const int row_vecs = row_bytes / 16;
  const long long n = T * row_vecs;
  const int threads = 256;
  if (cudaError_t e_ = launch_k(append_rows_kernel, (unsigned)((n + threads - 1) / threads), threads, 0, s, (const uint4*)src0, (uint4*)dst0, (const uint4*)src1, (uint4*)dst1, cu, app, n_users, T, row_vecs)) return e_;
  return cudaGetLastError();
}

// ============================================================================
// LayerNorm / casts (ReST §3.2.3, eq. 6)
// ============================================================================

// One warp per row; lane l holds columns 4l + 128k (k < d/128) as float4s.
// One row per warp at a time: the normalisation of a row already in registers
// (lane holds columns 128 k + 4 lane .. + 3).
template <typename T, int NV>
__device__ __forceinline__ void ln_row(float* __restrict__ xr, T* __restrict__ yr, const float* __restrict__ g,
                                       const float* __restrict__ b, const float* __restrict__ g2,
                                       const float* __restrict__ b2, int d, int mode, int lane, float (&v)[NV][4]) {
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) sum += v[k][0] + v[k][1] + v[k][2] + v[k][3];
  if (mode == 2) {
#pragma unroll
    for (int k = 0; k < NV; ++k) store4(yr + 128 * k + 4 * lane, v[k]);
    return;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / d;
  float sq = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float t = v[k][i] - mean;
      sq += t * t;
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = 1.0f / sqrtf(sq / d + 1e-5f);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = 128 * k + 4 * lane;
    float gg[4], bb[4], n[4];
    load4(g + c, gg);
    load4(b + c, bb);
#pragma unroll
    for (int i = 0; i < 4; ++i) n[i] = (v[k][i] - mean) * rstd * gg[i] + bb[i];
    if (mode == 1 || mode == 3 || mode == 4) store4(xr + c, n);
    if (mode == 0 || mode == 1) store4(yr + c, n);
    if (mode == 4) {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[k][i] = n[i];
    }
  }
  if (mode != 4) return;
  // mode 4: the next sublayer's pre-LN of the row just normalized
  float sum2 = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) sum2 += v[k][0] + v[k][1] + v[k][2] + v[k][3];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum2 += __shfl_xor_sync(0xffffffffu, sum2, o);
  const float mean2 = sum2 / d;
  float sq2 = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float t = v[k][i] - mean2;
      sq2 += t * t;
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq2 += __shfl_xor_sync(0xffffffffu, sq2, o);
  const float rstd2 = 1.0f / sqrtf(sq2 / d + 1e-5f);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = 128 * k + 4 * lane;
    float gg[4], bb[4], n[4];
    load4(g2 + c, gg);
    load4(b2 + c, bb);
#pragma unroll
    for (int i = 0; i < 4; ++i) n[i] = (v[k][i] - mean2) * rstd2 * gg[i] + bb[i];
    store4(yr + c, n);
  }
}


// Grid-stride over rows; each warp loads its next row before normalising the
// current one, so the load latency of one row hides behind the work of another.
template <typename T, int NV>
__global__ void layernorm_kernel(float* __restrict__ x, T* __restrict__ y, const float* __restrict__ g,
                                 const float* __restrict__ b, const float* __restrict__ g2,
                                 const float* __restrict__ b2, int rows, int d, int mode) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  const int lane = threadIdx.x & 31;
  const int n_warps = gridDim.x * (blockDim.x >> 5);
  int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  float v[NV][4], nx[NV][4];
  if (row < rows) {
#pragma unroll
    for (int k = 0; k < NV; ++k) load4(x + (long long)row * d + 128 * k + 4 * lane, v[k]);
  }
  for (; row < rows; row += n_warps) {
    const int next = row + n_warps;
    if (next < rows) {
#pragma unroll
      for (int k = 0; k < NV; ++k) load4(x + (long long)next * d + 128 * k + 4 * lane, nx[k]);
    }
    ln_row<T, NV>(x + (long long)row * d, y ? y + (long long)row * d : nullptr, g, b, g2, b2, d, mode, lane, v);
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
      for (int i = 0; i < 4; ++i) v[k][i] = nx[k][i];
  }
}

template <typename T>
static cudaError_t layernorm_dispatch(float* x, T* y, const float* g, const float* b, const float* g2,
                                      const float* b2, int rows, int d, int mode, cudaStream_t s) {
  int threads = 256;
  int blocks = (rows * 32 + threads - 1) / threads;
  static int cap = 0;
  if (cap == 0) {
    int dev = 0, n_sm = 0;
    cap = (cudaGetDevice(&dev) == cudaSuccess &&
           cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n_sm > 0)
              ? 8 * n_sm
              : 1184;
  }
  if (blocks > cap) blocks = cap;
  switch (d / 128) {
    case 1: if (cudaError_t e_ = launch_k(layernorm_kernel<T, 1>, blocks, threads, 0, s, x, y, g, b, g2, b2, rows, d, mode)) return e_; break;
    case 2: if (cudaError_t e_ = launch_k(layernorm_kernel<T, 2>, blocks, threads, 0, s, x, y, g, b, g2, b2, rows, d, mode)) return e_; break;
    case 3: if (cudaError_t e_ = launch_k(layernorm_kernel<T, 3>, blocks, threads, 0, s, x, y, g, b, g2, b2, rows, d, mode)) return e_; break;
    case 4: if (cudaError_t e_ = launch_k(layernorm_kernel<T, 4>, blocks, threads, 0, s, x, y, g, b, g2, b2, rows, d, mode)) return e_; break;
    case 5: if (cudaError_t e_ = launch_k(layernorm_kernel<T, 5>, blocks, threads, 0, s, x, y, g, b, g2, b2, rows, d, mode)) return e_; break;
    case 6: if (cudaError_t e_ = launch_k(layernorm_kernel<T, 6>, blocks, threads, 0, s, x, y, g, b, g2, b2, rows, d, mode)) return e_; break;
    case 7: if (cudaError_t e_ = launch_k(layernorm_kernel<T, 7>, blocks, threads, 0, s, x, y, g, b, g2, b2, rows, d, mode)) return e_; break;
    case 8: if (cudaError_t e_ = launch_k(layernorm_kernel<T, 8>, blocks, threads, 0, s, x, y, g, b, g2, b2, rows, d, mode)) return e_; break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// Rows whose width is not a multiple of 128 (d = 32, 64, 96, ...): one warp
// per row, one column per lane and step.
template <typename T>
__global__ void layernorm_narrow_kernel(float* __restrict__ x, T* __restrict__ y, const float* __restrict__ g,
                                        const float* __restrict__ b, const float* __restrict__ g2,
                                        const float* __restrict__ b2, int rows, int d, int mode) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  constexpr int VMAX = 32;  // d <= 1024
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  float* xr = x + (long long)warp * d;
  float v[VMAX];
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < VMAX; ++k) {
    int c = k * 32 + lane;
    v[k] = (c < d) ? xr[c] : 0.f;
    sum += v[k];
  }
  if (mode == 2) {
    T* yr = y + (long long)warp * d;
#pragma unroll
    for (int k = 0; k < VMAX; ++k) {
      int c = k * 32 + lane;
      if (c < d) yr[c] = from_f<T>(v[k]);
    }
    return;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  float mean = sum / d;
  float sq = 0.f;
#pragma unroll
  for (int k = 0; k < VMAX; ++k) {
    int c = k * 32 + lane;
    float t = (c < d) ? v[k] - mean : 0.f;
    sq += t * t;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  float rstd = 1.0f / sqrtf(sq / d + 1e-5f);
#pragma unroll
  for (int k = 0; k < VMAX; ++k) {
    int c = k * 32 + lane;
    if (c < d) {
      float n = (v[k] - mean) * rstd * g[c] + b[c];
      if (mode == 1 || mode == 3 || mode == 4) xr[c] = n;
      if (mode == 0 || mode == 1) y[(long long)warp * d + c] = from_f<T>(n);
      v[k] = n;
    }
  }
  if (mode != 4) return;
  // mode 4: the next sublayer's pre-LN of the row just normalized
  float sum2 = 0.f;
#pragma unroll
  for (int k = 0; k < VMAX; ++k) sum2 += (k * 32 + lane < d) ? v[k] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum2 += __shfl_xor_sync(0xffffffffu, sum2, o);
  const float mean2 = sum2 / d;
  float sq2 = 0.f;
#pragma unroll
  for (int k = 0; k < VMAX; ++k) {
    float t = (k * 32 + lane < d) ? v[k] - mean2 : 0.f;
    sq2 += t * t;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq2 += __shfl_xor_sync(0xffffffffu, sq2, o);
  const float rstd2 = 1.0f / sqrtf(sq2 / d + 1e-5f);
#pragma unroll
  for (int k = 0; k < VMAX; ++k) {
    int c = k * 32 + lane;
    if (c < d) y[(long long)warp * d + c] = from_f<T>((v[k] - mean2) * rstd2 * g2[c] + b2[c]);
  }
}

cudaError_t launch_layernorm(bool bf16m, float* x, void* y, const float* g, const float* b, int T, int d,
                             int mode, cudaStream_t s, const float* g2, const float* b2) {
  if (T == 0) return cudaSuccess;
  if (mode == 4 && (!g2 || !b2)) return cudaErrorInvalidValue;
  if (d % 128 == 0 && d <= 1024)
    return bf16m ? layernorm_dispatch<bf16>(x, (bf16*)y, g, b, g2, b2, T, d, mode, s)
                 : layernorm_dispatch<float>(x, (float*)y, g, b, g2, b2, T, d, mode, s);
  int threads = 256;
  int blocks = (T * 32 + threads - 1) / threads;
  if (bf16m) {
    if (cudaError_t e_ = launch_k(layernorm_narrow_kernel<bf16>, blocks, threads, 0, s, x, (bf16*)y, g, b, g2, b2, T, d, mode)) return e_;
  } else {
    if (cudaError_t e_ = launch_k(layernorm_narrow_kernel<float>, blocks, threads, 0, s, x, (float*)y, g, b, g2, b2, T, d, mode)) return e_;
  }
  return cudaGetLastError();
}

// The encoder's first launch: the rotation table (blocks n_cast ..) and, in blocks
// 0 .. n_cast - 1, the bf16 input into the fp32 residual stream with, for a
// pre-LN first sublayer, that sublayer's input y = bf16(LN(x)). The table is
// bound by its arithmetic and the rows by HBM, so the two kinds of block share
// the SMs: the row blocks, few and grid-striding, take two of each SM's block
// slots and the table's blocks the rest. A row's arithmetic is the LayerNorm
// kernel's (mode 0) on the same values, bf16 -> fp32 being exact.
template <int NV>
__global__ void __launch_bounds__(ROT_THREADS)
    table_cast_ln_kernel(const int64_t* __restrict__ ts, const int32_t* __restrict__ cu, int n_users, int T,
                         TableParams p, float* cos_out, float* sin_out, int32_t* err,
                         const UserAppend* __restrict__ app, const bf16* __restrict__ x, float* __restrict__ xres,
                         bf16* __restrict__ y, const float* __restrict__ g, const float* __restrict__ b, int d,
                         int n_cast) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  if ((int)blockIdx.x >= n_cast) {
    rotation_table_block(blockIdx.x - n_cast, ts, cu, n_users, T, p, nullptr, cos_out, sin_out, err, app);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int n_warps = n_cast * (blockDim.x >> 5);
  int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  float v[NV][4], nx[NV][4];
  if (row < T) {
#pragma unroll
    for (int k = 0; k < NV; ++k) load4(x + (long long)row * d + 128 * k + 4 * lane, v[k]);
  }
  for (; row < T; row += n_warps) {  // the next row's loads in flight during this row's work
    const int next = row + n_warps;
    if (next < T) {
#pragma unroll
      for (int k = 0; k < NV; ++k) load4(x + (long long)next * d + 128 * k + 4 * lane, nx[k]);
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) store4(xres + (long long)row * d + 128 * k + 4 * lane, v[k]);
    if (y) ln_row<bf16, NV>(nullptr, y + (long long)row * d, g, b, nullptr, nullptr, d, 0, lane, v);
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
      for (int i = 0; i < 4; ++i) v[k][i] = nx[k][i];
  }
}

cudaError_t launch_table_cast_ln(const int64_t* ts, const int32_t* cu, int n_users, int T, const TableParams& p,
                                 float* cos_out, float* sin_out, int32_t* err, const UserAppend* app,
                                 const void* x, float* xres, void* y, const float* g, const float* b, int d,
                                 cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (p.half < 1 || p.half > 64 || p.n_heads < 1 || p.n_heads > ROT_MAX_HEADS) return cudaErrorInvalidValue;
  if (d % 128 != 0 || d > 1024 || (y && (!g || !b))) return cudaErrorInvalidValue;
  if (((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 7) != 0 ||
      (reinterpret_cast<uintptr_t>(xres) & 15) != 0)
    return cudaErrorInvalidValue;
  static int n_sm = 0;
  if (n_sm == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0)
      n_sm = 148;
  }
  const long long rot_blocks = ((long long)T + rot_tokens_per_block(p.half) - 1) / rot_tokens_per_block(p.half);
  const long long row_blocks = ((long long)T * 32 + ROT_THREADS - 1) / ROT_THREADS;
  const int n_cast = (int)(row_blocks < 2LL * n_sm ? row_blocks : 2LL * n_sm);
  const unsigned grid = (unsigned)(n_cast + rot_blocks);
  const bf16* xb = static_cast<const bf16*>(x);
  bf16* yb = static_cast<bf16*>(y);
  cudaError_t e_ = cudaSuccess;
  switch (d / 128) {
    case 1: e_ = launch_k(table_cast_ln_kernel<1>, grid, ROT_THREADS, 0, s, ts, cu, n_users, T, p, cos_out, sin_out, err, app, xb, xres, yb, g, b, d, n_cast); break;
    case 2: e_ = launch_k(table_cast_ln_kernel<2>, grid, ROT_THREADS, 0, s, ts, cu, n_users, T, p, cos_out, sin_out, err, app, xb, xres, yb, g, b, d, n_cast); break;
    case 3: e_ = launch_k(table_cast_ln_kernel<3>, grid, ROT_THREADS, 0, s, ts, cu, n_users, T, p, cos_out, sin_out, err, app, xb, xres, yb, g, b, d, n_cast); break;
    case 4: e_ = launch_k(table_cast_ln_kernel<4>, grid, ROT_THREADS, 0, s, ts, cu, n_users, T, p, cos_out, sin_out, err, app, xb, xres, yb, g, b, d, n_cast); break;
    case 5: e_ = launch_k(table_cast_ln_kernel<5>, grid, ROT_THREADS, 0, s, ts, cu, n_users, T, p, cos_out, sin_out, err, app, xb, xres, yb, g, b, d, n_cast); break;
    case 6: e_ = launch_k(table_cast_ln_kernel<6>, grid, ROT_THREADS, 0, s, ts, cu, n_users, T, p, cos_out, sin_out, err, app, xb, xres, yb, g, b, d, n_cast); break;
    case 7: e_ = launch_k(table_cast_ln_kernel<7>, grid, ROT_THREADS, 0, s, ts, cu, n_users, T, p, cos_out, sin_out, err, app, xb, xres, yb, g, b, d, n_cast); break;
    case 8: e_ = launch_k(table_cast_ln_kernel<8>, grid, ROT_THREADS, 0, s, ts, cu, n_users, T, p, cos_out, sin_out, err, app, xb, xres, yb, g, b, d, n_cast); break;
    default: return cudaErrorInvalidValue;
  }
  if (e_ != cudaSuccess) return e_;
  return cudaGetLastError();
}

// ============================================================================
// Decoder block and candidate score (ReST §3.3.2 eq. 8, Fig. 1 right)
// ============================================================================

// a = z + y into f; u = dt(LN_k(a)) with token type k = row % K (U16: u in
// fp16, for an fp16 product; a value beyond fp16's range sets REST_ERR_RANGE).
// One warp per row; lane holds columns 128 i + 4 lane .. + 3 (d a multiple of
// 128, NV = d / 128) or, for other widths, columns lane, lane + 32, ... (NV = 0).
template <typename T, int NV, bool U16 = false>
__global__ void score_ln_kernel(const T* __restrict__ z, const float* __restrict__ y, float* __restrict__ f,
                                T* __restrict__ u, T* __restrict__ u_lo, const float* __restrict__ ln_g,
                                const float* __restrict__ ln_b, long long rows, int d, int K, int32_t* err) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  constexpr int VN = NV > 0 ? 4 * NV : 32;  // values per lane
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int k = (int)(row % K);
  const long long o = row * d;
  auto col = [&](int i) { return NV > 0 ? 128 * (i >> 2) + 4 * lane + (i & 3) : 32 * i + lane; };
  float v[VN];
  float sum = 0.f;
  if (NV > 0) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float zz[4], yy[4];
      load4(z + o + 128 * i + 4 * lane, zz);
      load4(y + o + 128 * i + 4 * lane, yy);
#pragma unroll
      for (int e = 0; e < 4; ++e) v[4 * i + e] = zz[e] + yy[e];
      store4(f + o + 128 * i + 4 * lane, &v[4 * i]);
    }
#pragma unroll
    for (int i = 0; i < VN; ++i) sum += v[i];
  } else {
#pragma unroll
    for (int i = 0; i < VN; ++i) {
      const int c = col(i);
      v[i] = c < d ? to_f<T>(z[o + c]) + y[o + c] : 0.f;
      if (c < d) f[o + c] = v[i];
      sum += v[i];
    }
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
  const float mean = sum / d;
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < VN; ++i) {
    const float t = col(i) < d ? v[i] - mean : 0.f;
    sq += t * t;
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, m);
  const float rstd = 1.0f / sqrtf(sq / d + 1e-5f);
  const float* g = ln_g + (long long)k * d;
  const float* b = ln_b + (long long)k * d;
  if (NV > 0 && U16) {
    bool ok = true;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = 128 * i + 4 * lane;
      float gg[4], bb[4], n[4];
      load4(g + c, gg);
      load4(b + c, bb);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        n[e] = (v[4 * i + e] - mean) * rstd * gg[e] + bb[e];
        ok = ok && fits_f16(n[e]);
      }
      *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(u) + o + c) =
          make_uint2(pack_f16x2(n[0], n[1]), pack_f16x2(n[2], n[3]));
    }
    if (!ok) set_error(err, REST_ERR_RANGE);
  } else if (NV > 0) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = 128 * i + 4 * lane;
      float gg[4], bb[4], hi[4], lo[4];
      load4(g + c, gg);
      load4(b + c, bb);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float n = (v[4 * i + e] - mean) * rstd * gg[e] + bb[e];
        hi[e] = to_f<T>(from_f<T>(n));
        lo[e] = n - hi[e];
      }
      store4(u + o + c, hi);
      if (u_lo) store4(u_lo + o + c, lo);
    }
  } else {
#pragma unroll
    for (int i = 0; i < VN; ++i) {
      const int c = col(i);
      if (c < d) {
        const float n = (v[i] - mean) * rstd * g[c] + b[c];
        const T hi = from_f<T>(n);
        u[o + c] = hi;
        if (u_lo) u_lo[o + c] = from_f<T>(n - to_f<T>(hi));
      }
    }
  }
}

template <typename T, bool U16 = false>
static cudaError_t score_ln_dispatch(const T* z, const float* y, float* f, T* u, T* u_lo, const float* ln_g,
                                    const float* ln_b, long long rows, int d, int K, cudaStream_t s, int32_t* err) {
  const int threads = 256;
  const long long blocks = (rows * 32 + threads - 1) / threads;
  const unsigned nb = (unsigned)blocks;
  switch (d % 128 == 0 ? d / 128 : 0) {
    case 1: if (cudaError_t e_ = launch_k(score_ln_kernel<T, 1, U16>, nb, threads, 0, s, z, y, f, u, u_lo, ln_g, ln_b, rows, d, K, err)) return e_; break;
    case 2: if (cudaError_t e_ = launch_k(score_ln_kernel<T, 2, U16>, nb, threads, 0, s, z, y, f, u, u_lo, ln_g, ln_b, rows, d, K, err)) return e_; break;
    case 4: if (cudaError_t e_ = launch_k(score_ln_kernel<T, 4, U16>, nb, threads, 0, s, z, y, f, u, u_lo, ln_g, ln_b, rows, d, K, err)) return e_; break;
    case 8: if (cudaError_t e_ = launch_k(score_ln_kernel<T, 8, U16>, nb, threads, 0, s, z, y, f, u, u_lo, ln_g, ln_b, rows, d, K, err)) return e_; break;
    default:
      if (U16) return cudaErrorInvalidValue;  // the fp16 output takes d a multiple of 128
      if (cudaError_t e_ = launch_k(score_ln_kernel<T, 0>, nb, threads, 0, s, z, y, f, u, u_lo, ln_g, ln_b, rows, d, K, err)) return e_; break;
  }
  return cudaGetLastError();
}

cudaError_t launch_score_ln(bool bf16m, const void* z, const float* y, float* f, void* u, void* u_lo,
                            const float* ln_g, const float* ln_b, long long rows, int d, int K, cudaStream_t s,
                            bool u16, int32_t* err) {
  if (rows == 0) return cudaSuccess;
  if (d > 1024 || K < 1) return cudaErrorInvalidValue;
  if (bf16m && u16)
    return score_ln_dispatch<bf16, true>((const bf16*)z, y, f, (bf16*)u, nullptr, ln_g, ln_b, rows, d, K, s, err);
  if (bf16m)
    return score_ln_dispatch<bf16>((const bf16*)z, y, f, (bf16*)u, (bf16*)u_lo, ln_g, ln_b, rows, d, K, s, err);
  return score_ln_dispatch<float>((const float*)z, y, f, (float*)u, nullptr, ln_g, ln_b, rows, d, K, s, err);
}

// score[n] = f[n, 0, :] . w_s + b_s (token 0 is [CLS]); one warp per candidate.
__global__ void score_readout_kernel(const float* __restrict__ f, const float* __restrict__ w_s, float b_s,
                                     float* __restrict__ score, long long n, int d, int K) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  const long long c = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (c >= n) return;
  const float* row = f + c * K * d;
  float acc = 0.f;
  if ((d & 127) == 0 && ((reinterpret_cast<uintptr_t>(f) | reinterpret_cast<uintptr_t>(w_s)) & 15) == 0) {
    // 16 bytes a lane: a row's loads are in flight together
    for (int i = 4 * lane; i < d; i += 128) {
      const float4 a = *reinterpret_cast<const float4*>(row + i), w = *reinterpret_cast<const float4*>(w_s + i);
      acc = fmaf(a.x, w.x, fmaf(a.y, w.y, fmaf(a.z, w.z, fmaf(a.w, w.w, acc))));
    }
  } else {
    for (int i = lane; i < d; i += 32) acc = fmaf(row[i], w_s[i], acc);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (lane == 0) score[c] = acc + b_s;
}

cudaError_t launch_score_readout(const float* f, const float* w_s, float b_s, float* score, long long n, int d, int K,
                                 cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = (n * 32 + threads - 1) / threads;
  if (cudaError_t e_ = launch_k(score_readout_kernel, (unsigned)blocks, threads, 0, s, f, w_s, b_s, score, n, d, K)) return e_;
  return cudaGetLastError();
}

template <typename T>
__global__ void to_f32_kernel(const T* __restrict__ in, float* __restrict__ out, long long n) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = to_f<T>(in[i]);
}
// 8 bf16 values (16 bytes) per thread in, 32 bytes out
__global__ void bf16_to_f32_x8_kernel(const uint4* __restrict__ in, float4* __restrict__ out, long long n8) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const uint4 u = in[i];
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  float f[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
  out[2 * i] = make_float4(f[0], f[1], f[2], f[3]);
  out[2 * i + 1] = make_float4(f[4], f[5], f[6], f[7]);
}

cudaError_t launch_to_f32(bool bf16m, const void* x_in, float* x_res, long long n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  int threads = 256;
  if (bf16m && n % 8 == 0 && (reinterpret_cast<uintptr_t>(x_in) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(x_res) & 15) == 0) {
    const long long n8 = n / 8;
    if (cudaError_t e_ = launch_k(bf16_to_f32_x8_kernel, (unsigned)((n8 + threads - 1) / threads), threads, 0, s, static_cast<const uint4*>(x_in), reinterpret_cast<float4*>(x_res), n8)) return e_;
    return cudaGetLastError();
  }
  long long blocks = (n + threads - 1) / threads;
  if (bf16m) {
    if (cudaError_t e_ = launch_k(to_f32_kernel<bf16>, (unsigned)blocks, threads, 0, s, (const bf16*)x_in, x_res, n)) return e_;
  } else {
    if (cudaError_t e_ = launch_k(to_f32_kernel<float>, (unsigned)blocks, threads, 0, s, (const float*)x_in, x_res, n)) return e_;
  }
  return cudaGetLastError();
}

// 8 values per thread: two 16-byte loads, a 16-byte store of each part
__global__ void split_bf16_kernel(const float4* __restrict__ x, uint4* __restrict__ hi, uint4* __restrict__ lo,
                                  long long n8) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = x[2 * i], b = x[2 * i + 1];
  const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    const float2 hf = __bfloat1622float2(h2);
    const __nv_bfloat162 l2 = __floats2bfloat162_rn(v[2 * k] - hf.x, v[2 * k + 1] - hf.y);
    h[k] = *reinterpret_cast<const uint32_t*>(&h2);
    l[k] = *reinterpret_cast<const uint32_t*>(&l2);
  }
  hi[i] = make_uint4(h[0], h[1], h[2], h[3]);
  lo[i] = make_uint4(l[0], l[1], l[2], l[3]);
}

// one value per thread, for sizes or addresses the vector form does not take
__global__ void split_bf16_scalar_kernel(const float* __restrict__ x, bf16* __restrict__ hi, bf16* __restrict__ lo,
                                         long long n) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    float v = x[i];
    bf16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

cudaError_t launch_split_bf16(const float* x, void* hi, void* lo, long long n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const bool vec = n % 8 == 0 && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(hi) |
                                   reinterpret_cast<uintptr_t>(lo)) & 15) == 0;
  if (vec) {
    const long long n8 = n / 8;
    return launch_k(split_bf16_kernel, (unsigned)((n8 + threads - 1) / threads), threads, 0, s,
                    reinterpret_cast<const float4*>(x), static_cast<uint4*>(hi), static_cast<uint4*>(lo), n8);
  }
  const long long blocks = (n + threads - 1) / threads;
  return launch_k(split_bf16_scalar_kernel, (unsigned)blocks, threads, 0, s, x, (bf16*)hi, (bf16*)lo, n);
}

// H for the tensor-core decoder, which multiplies in fp16: from the fp32
// residual stream, H in bf16 (the call's output) and an fp16 copy, 8 values per
// thread; a value beyond fp16's range sets REST_ERR_RANGE.
__global__ void split_h16_kernel(const float4* __restrict__ x, uint4* __restrict__ hb, uint4* __restrict__ h16,
                                 long long n8, int32_t* err) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = x[2 * i], b = x[2 * i + 1];
  const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t hh[4], hf[4];
  bool ok = true;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    hh[k] = pack_bf16x2(v[2 * k], v[2 * k + 1]);
    hf[k] = pack_f16x2(v[2 * k], v[2 * k + 1]);
    ok = ok && fits_f16(v[2 * k]) && fits_f16(v[2 * k + 1]);
  }
  hb[i] = make_uint4(hh[0], hh[1], hh[2], hh[3]);
  h16[i] = make_uint4(hf[0], hf[1], hf[2], hf[3]);
  if (!ok) set_error(err, REST_ERR_RANGE);
}

// The caller's bf16 H as fp16 for the tensor-core decoder, 8 values per thread
// (exact within fp16's range; a value beyond it sets REST_ERR_RANGE).
__global__ void bf16_to_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, long long n8,
                                   int32_t* err) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const uint4 w4 = src[i];
  const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
  uint32_t hf[4];
  bool ok = true;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xffff0000u);
    hf[k] = pack_f16x2(lo, hi);
    ok = ok && fits_f16(lo) && fits_f16(hi);
  }
  dst[i] = make_uint4(hf[0], hf[1], hf[2], hf[3]);
  if (!ok) set_error(err, REST_ERR_RANGE);
}

cudaError_t launch_split_h16(const float* x, void* hb, void* h16, long long n, int32_t* err, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (n % 8 != 0 || ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(hb) |
                      reinterpret_cast<uintptr_t>(h16)) & 15) != 0)
    return cudaErrorInvalidValue;  // d is a multiple of 32 and the buffers 16-byte aligned
  const int threads = 256;
  const long long n8 = n / 8;
  return launch_k(split_h16_kernel, (unsigned)((n8 + threads - 1) / threads), threads, 0, s,
                  reinterpret_cast<const float4*>(x), static_cast<uint4*>(hb), static_cast<uint4*>(h16), n8, err);
}

cudaError_t launch_bf16_to_f16(const void* src, void* dst, long long n, int32_t* err, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (n % 8 != 0 || ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) != 0)
    return cudaErrorInvalidValue;
  const int threads = 256;
  const long long n8 = n / 8;
  return launch_k(bf16_to_f16_kernel, (unsigned)((n8 + threads - 1) / threads), threads, 0, s,
                  static_cast<const uint4*>(src), static_cast<uint4*>(dst), n8, err);
}

// ============================================================================
// Tiled GEMM with the fused epilogues
// ============================================================================

// Physical column of logical column n for the interleaved epilogues: every
// group of 4 logical columns from `lbase` on is (2p, 2p+1) of the block at
// physical column `pbase`, then (2p, 2p+1) of the block `width` columns after it.
__device__ __forceinline__ int interleave_col(int n, int lbase, int pbase, int width) {
  int r = n - lbase, p = r >> 2, w = r & 3;
  return pbase + (w < 2 ? 2 * p + w : width + 2 * p + w - 2);
}

__device__ __forceinline__ int physical_col(const GemmArgs& a, int n) {
  const int d = a.d;
  if (a.epi == EPI_QKVG) {
    if (a.gate_mode == GATES_O) return n;                       // Q | K | V | Go
    if (a.gate_mode == GATES_QKVO) {                            // Q,Gq | K,Gk | V,Gv | Go
      if (n < 2 * d) return interleave_col(n, 0, 0, 5 * d);
      if (n < 4 * d) return interleave_col(n, 2 * d, d, 5 * d);
      if (n < 6 * d) return interleave_col(n, 4 * d, 2 * d, d);
      return n - 2 * d;
    }
    if (n >= 2 * d && n < 4 * d) return interleave_col(n, 2 * d, 2 * d, d);  // Q | K | V,Gv | Go
    return n;
  }
  if (a.epi == EPI_SWIGLU) return interleave_col(n, 0, 0, a.d);
  return n;
}

// Rotate the pair (x0, x1) of Q or K at column `col` of row m (eq. 5).
__device__ __forceinline__ void rotate_pair(const GemmArgs& a, long long m, int col, float x0, float x1, float* out) {
  const float c = a.cos_t[m * (a.d / 2) + col / 2], s = a.sin_t[m * (a.d / 2) + col / 2];
  out[0] = x0 * c - x1 * s;
  out[1] = x0 * s + x1 * c;
}

// TA: type of A; T: the call's dtype (B and the dtype outputs).
template <typename TA, typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs a) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN];
  const TA* A = (const TA*)a.A;
  const T* B = (const T*)a.B;
  int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  int ar = tid >> 2, ak = (tid & 3) * 4;
  int bk = tid >> 4, bn = (tid & 15) * 4;
  int bcol[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int ln = n0 + bn + i;
    bcol[i] = (ln < a.N) ? physical_col(a, ln) : -1;
  }
  for (int k0 = 0; k0 < a.K; k0 += BK) {
    float av[4] = {0.f, 0.f, 0.f, 0.f};
    int gm = m0 + ar;
    if (gm < a.M) {
      load4(A + (long long)gm * a.lda + k0 + ak, av);
      if (a.A2) {  // A = A + A2 (a bf16 hi + lo pair)
        float lv[4];
        load4((const TA*)a.A2 + (long long)gm * a.lda + k0 + ak, lv);
        for (int i = 0; i < 4; ++i) av[i] += lv[i];
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) As[ak + i][ar] = av[i];
    const T* brow = B + (long long)(k0 + bk) * a.ldb;
#pragma unroll
    for (int i = 0; i < 4; ++i) Bs[bk][bn + i] = (bcol[i] >= 0) ? to_f<T>(brow[bcol[i]]) : 0.f;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float4 a4 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      float4 b4 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      float av2[4] = {a4.x, a4.y, a4.z, a4.w}, bv2[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av2[i], bv2[j], acc[i][j]);
    }
    __syncthreads();
  }

  int n = n0 + tx * 4;
  if (n >= a.N) return;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int m = m0 + ty * 4 + i;
    if (m >= a.M) break;
    float* c = acc[i];
    long long ro = (long long)m * a.ldo;
    switch (a.epi) {
      case EPI_F32: store4((float*)a.out0 + ro + n, c); break;
      case EPI_DT: store4((T*)a.out0 + ro + n, c); break;
      case EPI_SIGMOID: {
        float v[4] = {sigmoid_f(c[0]), sigmoid_f(c[1]), sigmoid_f(c[2]), sigmoid_f(c[3])};
        store4((float*)a.out0 + ro + n, v);
        break;
      }
      case EPI_RESID: {
        float* p = (float*)a.out0 + ro + n;
        float v[4];
        load4(p, v);
        for (int j = 0; j < 4; ++j) v[j] = fmaf(a.alpha, c[j], v[j]);
        store4(p, v);
        break;
      }
      case EPI_QKVG: {
        int d = a.d;
        if (a.gate_mode == GATES_QKVO) {
          if (n < 4 * d) {  // gated Q or K pair (2p, 2p+1), then its rotation (eq. 5)
            const int blk = n < 2 * d ? 0 : 1, col = ((n - 2 * d * blk) >> 2) * 2;
            float v[2];
            rotate_pair(a, m, col, c[0] * sigmoid_f(c[2]), c[1] * sigmoid_f(c[3]), v);
            store2((T*)(blk == 0 ? a.out0 : a.out1) + ro + col, v[0], v[1]);
          } else if (n < 6 * d) {  // value gate
            int col = ((n - 4 * d) >> 2) * 2;
            store2((T*)a.out2 + ro + col, c[0] * sigmoid_f(c[2]), c[1] * sigmoid_f(c[3]));
          } else {  // output gate
            float v[4] = {sigmoid_f(c[0]), sigmoid_f(c[1]), sigmoid_f(c[2]), sigmoid_f(c[3])};
            store4((float*)a.out3 + ro + (n - 6 * d), v);
          }
          break;
        }
        if (a.gate_mode == GATES_O && n >= 2 * d) {
          if (n < 3 * d) {  // V without a gate
            store4((T*)a.out2 + ro + (n - 2 * d), c);
          } else {  // output gate
            float v[4] = {sigmoid_f(c[0]), sigmoid_f(c[1]), sigmoid_f(c[2]), sigmoid_f(c[3])};
            store4((float*)a.out3 + ro + (n - 3 * d), v);
          }
          break;
        }
        if (n < 2 * d) {  // Q or K: rotate the pairs (eq. 5)
          int col = n < d ? n : n - d;
          const float* ct = a.cos_t + (long long)m * (d / 2) + col / 2;
          const float* st = a.sin_t + (long long)m * (d / 2) + col / 2;
          float v[4];
          v[0] = c[0] * ct[0] - c[1] * st[0];
          v[1] = c[0] * st[0] + c[1] * ct[0];
          v[2] = c[2] * ct[1] - c[3] * st[1];
          v[3] = c[2] * st[1] + c[3] * ct[1];
          store4((T*)(n < d ? a.out0 : a.out1) + ro + col, v);
        } else if (n < 4 * d) {  // value gate: V' = sigmoid(Gv) * V (eq. 3)
          int col = ((n - 2 * d) >> 2) * 2;
          store2((T*)a.out2 + ro + col, c[0] * sigmoid_f(c[2]), c[1] * sigmoid_f(c[3]));
        } else {  // output gate sigmoid(Go) (eq. 4), kept in fp32
          float v[4] = {sigmoid_f(c[0]), sigmoid_f(c[1]), sigmoid_f(c[2]), sigmoid_f(c[3])};
          store4((float*)a.out3 + ro + (n - 4 * d), v);
        }
        break;
      }
      case EPI_SWIGLU: {
        int col = (n >> 2) * 2;
        const float h0 = c[0] * sigmoid_f(c[0]) * c[2], h1 = c[1] * sigmoid_f(c[1]) * c[3];
        store2((T*)a.out0 + ro + col, h0, h1);
        if (a.out1)  // the low part of a bf16 hi + lo pair
          store2((T*)a.out1 + ro + col, h0 - to_f<T>(from_f<T>(h0)), h1 - to_f<T>(from_f<T>(h1)));
        break;
      }
    }
  }
}

cudaError_t launch_gemm_simt(bool bf16m, const GemmArgs& a, cudaStream_t s) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  dim3 grid((a.N + 63) / 64, (a.M + 63) / 64);
  if (bf16m && a.a_f32) {
    if (cudaError_t e_ = launch_k(gemm_simt_kernel<float, bf16>, grid, 256, 0, s, a)) return e_;
  } else if (bf16m) {
    if (cudaError_t e_ = launch_k(gemm_simt_kernel<bf16, bf16>, grid, 256, 0, s, a)) return e_;
  } else {
    if (cudaError_t e_ = launch_k(gemm_simt_kernel<float, float>, grid, 256, 0, s, a)) return e_;
  }
  return cudaGetLastError();
}

// ============================================================================
// Attention: one thread per query row, K/V tiles staged in shared memory.
// Online softmax in base 2 (scores pre-scaled by log2(e)/sqrt(head_dim)).
// ============================================================================

template <int HD>
struct RowState {
  float q[HD];
  float o[HD];
  float m, l;
};

// Decoder: keys and values are both the rows of H (+ its low part when given).
template <typename T, int HD, int BK>
__device__ __forceinline__ void stage_h(float (*Ks)[HD], float (*Vs)[HD], const T* hbase, const T* lobase,
                                        long long ld, int nvalid) {
  for (int e = threadIdx.x * 4; e < BK * HD; e += blockDim.x * 4) {
    int r = e / HD, c = e % HD;
    float hv[4] = {0.f, 0.f, 0.f, 0.f};
    if (r < nvalid) {
      load4(hbase + r * ld + c, hv);
      if (lobase) {
        float lv[4];
        load4(lobase + r * ld + c, lv);
        for (int i = 0; i < 4; ++i) hv[i] += lv[i];
      }
    }
    *reinterpret_cast<float4*>(&Ks[r][c]) = make_float4(hv[0], hv[1], hv[2], hv[3]);
    *reinterpret_cast<float4*>(&Vs[r][c]) = make_float4(hv[0], hv[1], hv[2], hv[3]);
  }
}

template <typename T, int HD, int BK>
__device__ __forceinline__ void stage_kv(float (*Ks)[HD], float (*Vs)[HD], const T* kbase, const T* vbase,
                                         long long ld, int nvalid) {
  for (int e = threadIdx.x * 4; e < BK * HD; e += blockDim.x * 4) {
    int r = e / HD, c = e % HD;
    float kv[4] = {0.f, 0.f, 0.f, 0.f}, vv[4] = {0.f, 0.f, 0.f, 0.f};
    if (r < nvalid) {
      load4(kbase + r * ld + c, kv);
      load4(vbase + r * ld + c, vv);
    }
    *reinterpret_cast<float4*>(&Ks[r][c]) = make_float4(kv[0], kv[1], kv[2], kv[3]);
    *reinterpret_cast<float4*>(&Vs[r][c]) = make_float4(vv[0], vv[1], vv[2], vv[3]);
  }
}

// Process one staged tile for one row: keys j < jmax are visible.
template <int HD, int BK>
__device__ __forceinline__ void row_tile(RowState<HD>& st, const float (*Ks)[HD], const float (*Vs)[HD], int jmax) {
  float sc[BK];
  float mt = st.m;
#pragma unroll
  for (int j = 0; j < BK; ++j) {
    float dot = 0.f;
#pragma unroll
    for (int c = 0; c < HD; c += 4) {
      float4 k4 = *reinterpret_cast<const float4*>(&Ks[j][c]);
      dot = fmaf(st.q[c], k4.x, dot);
      dot = fmaf(st.q[c + 1], k4.y, dot);
      dot = fmaf(st.q[c + 2], k4.z, dot);
      dot = fmaf(st.q[c + 3], k4.w, dot);
    }
    sc[j] = (j < jmax) ? dot : -INFINITY;
    mt = fmaxf(mt, sc[j]);
  }
  float alpha = exp2_approx(st.m - mt);
  st.l *= alpha;
#pragma unroll
  for (int c = 0; c < HD; ++c) st.o[c] *= alpha;
  st.m = mt;
#pragma unroll
  for (int j = 0; j < BK; ++j) {
    float p = exp2_approx(sc[j] - mt);
    st.l += p;
#pragma unroll
    for (int c = 0; c < HD; c += 4) {
      float4 v4 = *reinterpret_cast<const float4*>(&Vs[j][c]);
      st.o[c] = fmaf(p, v4.x, st.o[c]);
      st.o[c + 1] = fmaf(p, v4.y, st.o[c + 1]);
      st.o[c + 2] = fmaf(p, v4.z, st.o[c + 2]);
      st.o[c + 3] = fmaf(p, v4.w, st.o[c + 3]);
    }
  }
}

template <typename T, int HD>
__device__ __forceinline__ void load_q(RowState<HD>& st, const T* q, float scale) {
#pragma unroll
  for (int c = 0; c < HD; c += 4) {
    float v[4];
    load4(q + c, v);
    st.q[c] = v[0] * scale; st.q[c + 1] = v[1] * scale; st.q[c + 2] = v[2] * scale; st.q[c + 3] = v[3] * scale;
  }
#pragma unroll
  for (int c = 0; c < HD; ++c) st.o[c] = 0.f;
  st.m = -INFINITY;
  st.l = 0.f;
}

// O / l times the output gate (gate null: no gate); with out_lo (bf16 outputs)
// also the low part, out + out_lo
template <typename T, int HD>
__device__ __forceinline__ void store_row(const RowState<HD>& st, const float* gate, T* out, T* out_lo = nullptr) {
  float inv = 1.0f / st.l;
#pragma unroll
  for (int c = 0; c < HD; c += 4) {
    float g[4] = {1.f, 1.f, 1.f, 1.f};
    if (gate) load4(gate + c, g);
    float v[4] = {st.o[c] * inv * g[0], st.o[c + 1] * inv * g[1], st.o[c + 2] * inv * g[2], st.o[c + 3] * inv * g[3]};
    store4(out + c, v);
    if (out_lo) {
      float lo[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) lo[i] = v[i] - to_f<T>(from_f<T>(v[i]));
      store4(out_lo + c, lo);
    }
  }
}

constexpr int ATT_ROWS = 128;  // query rows per block (one per thread)
constexpr int ATT_BK = 16;     // keys per staged tile

template <typename T, int HD>
__global__ void __launch_bounds__(ATT_ROWS) enc_attn_simt_kernel(EncAttnArgs a) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  __shared__ __align__(16) float Ks[ATT_BK][HD];
  __shared__ __align__(16) float Vs[ATT_BK][HD];
  EncTile tile = a.tiles[blockIdx.x];
  int h = blockIdx.y;
  int s = a.cu[tile.user];                  // packed row of the user's first query row
  int n = a.cu[tile.user + 1] - s;          // the user's query rows
  int off = a.app ? a.app[tile.user].cached : 0;  // position of query row 0 in the history
  int key0 = a.app ? a.app[tile.user].key0 : s;   // row of the history's first key
  int i = tile.q0 + threadIdx.x;
  bool valid = i < n;
  int pos = off + i;
  long long hoff = (long long)h * HD;
  RowState<HD> st;
  load_q<T, HD>(st, (const T*)a.q + (long long)(s + (valid ? i : 0)) * a.d + hoff, a.scale_log2);
  int kv_end = min(off + n, off + tile.q0 + ATT_ROWS);
  const T* K = (const T*)a.k + (long long)key0 * a.d + hoff;
  const T* V = (const T*)a.v + (long long)key0 * a.d + hoff;
  for (int kb = 0; kb < kv_end; kb += ATT_BK) {
    __syncthreads();
    stage_kv<T, HD, ATT_BK>(Ks, Vs, K + (long long)kb * a.d, V + (long long)kb * a.d, a.d, kv_end - kb);
    __syncthreads();
    if (valid && kb <= pos) row_tile<HD, ATT_BK>(st, Ks, Vs, pos - kb + 1);  // causal: key <= pos
  }
  if (valid) {
    long long ro = (long long)(s + i) * a.d + hoff;
    store_row<T, HD>(st, a.gate ? a.gate + ro : nullptr, (T*)a.out + ro, a.out_lo ? (T*)a.out_lo + ro : nullptr);
    // log sum_j exp(score): the running max is kept in the scaled log2 domain
    if (a.lse) a.lse[(long long)(s + i) * a.n_heads + h] = (st.m + log2f(st.l)) * 0.69314718055994531f;
  }
}

template <typename T, int HD>
__global__ void __launch_bounds__(ATT_ROWS) dec_attn_simt_kernel(DecAttnArgs a) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  __shared__ __align__(16) float Ks[ATT_BK][HD];
  __shared__ __align__(16) float Vs[ATT_BK][HD];
  DecTile tile = a.tiles[blockIdx.x];
  int h = blockIdx.y;
  long long hoff = (long long)h * HD;
  bool valid = threadIdx.x < tile.nrows;
  long long row = tile.row0 + (valid ? threadIdx.x : 0);
  RowState<HD> st;
  load_q<float, HD>(st, a.q + row * a.d + hoff, a.scale_log2);
  const T* Hm = (const T*)a.h + (long long)tile.key0 * a.d + hoff;
  const T* Hlo = a.h_lo ? (const T*)a.h_lo + (long long)tile.key0 * a.d + hoff : nullptr;
  for (int kb = 0; kb < tile.nkeys; kb += ATT_BK) {
    __syncthreads();
    // keys and values are the same rows of H (projection-free, ReST eq. 7)
    stage_h<T, HD, ATT_BK>(Ks, Vs, Hm + (long long)kb * a.d, Hlo ? Hlo + (long long)kb * a.d : nullptr, a.d,
                           tile.nkeys - kb);
    __syncthreads();
    if (valid) row_tile<HD, ATT_BK>(st, Ks, Vs, tile.nkeys - kb);
  }
  if (valid) {
    long long ro = row * a.d + hoff;
    store_row<float, HD>(st, a.g + ro, (float*)a.out + ro);
  }
}

template <typename T>
static cudaError_t enc_dispatch(int hd, const EncAttnArgs& a, cudaStream_t s) {
  dim3 grid(a.n_tiles, a.n_heads);
  switch (hd) {
    case 16: if (cudaError_t e_ = launch_k(enc_attn_simt_kernel<T, 16>, grid, ATT_ROWS, 0, s, a)) return e_; break;
    case 32: if (cudaError_t e_ = launch_k(enc_attn_simt_kernel<T, 32>, grid, ATT_ROWS, 0, s, a)) return e_; break;
    case 64: if (cudaError_t e_ = launch_k(enc_attn_simt_kernel<T, 64>, grid, ATT_ROWS, 0, s, a)) return e_; break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T>
static cudaError_t dec_dispatch(int hd, const DecAttnArgs& a, cudaStream_t s) {
  dim3 grid(a.n_tiles, a.n_heads);
  switch (hd) {
    case 16: if (cudaError_t e_ = launch_k(dec_attn_simt_kernel<T, 16>, grid, ATT_ROWS, 0, s, a)) return e_; break;
    case 32: if (cudaError_t e_ = launch_k(dec_attn_simt_kernel<T, 32>, grid, ATT_ROWS, 0, s, a)) return e_; break;
    case 64: if (cudaError_t e_ = launch_k(dec_attn_simt_kernel<T, 64>, grid, ATT_ROWS, 0, s, a)) return e_; break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// Split-key decoder (after the tensor-core decoder): out = (sum_s 2^(m_s - M) O_s)
// / (sum_s 2^(m_s - M) l_s) * g in fp16, g the fp16 gate, M = max_s m_s; one
// thread per 4 output columns of a row.
__global__ void dec_combine_kernel(DecAttnArgs a, int hd) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int cols4 = a.d / 4;
  if (gid >= a.nk_rows * cols4) return;
  const long long row = gid / cols4;
  const int c = (int)(gid % cols4) * 4;
  const int h = c / hd;
  float M = -INFINITY;
  for (int s = 0; s < a.n_split; ++s) M = fmaxf(M, a.part_ml[((s * a.nk_rows + row) * a.n_heads + h) * 2]);
  float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < a.n_split; ++s) {
    const float* ml = a.part_ml + ((s * a.nk_rows + row) * a.n_heads + h) * 2;
    if (ml[0] == -INFINITY) continue;  // a split with no keys
    const float w = exp2f(ml[0] - M);
    L = fmaf(w, ml[1], L);
    float v[4];
    load4(a.part_o + (s * a.nk_rows + row) * a.d + c, v);
    for (int i = 0; i < 4; ++i) o[i] = fmaf(w, v[i], o[i]);
  }
  // the tensor-core decoder's gate and o * g are fp16
  float g[4];
  load4_f16(static_cast<const __half*>(a.g16) + row * a.d + c, g);
  const float inv = 1.0f / L;
  *reinterpret_cast<uint2*>(static_cast<__half*>(a.out) + row * a.d + c) =
      make_uint2(pack_f16x2(o[0] * inv * g[0], o[1] * inv * g[1]), pack_f16x2(o[2] * inv * g[2], o[3] * inv * g[3]));
}

cudaError_t launch_dec_combine(int hd, const DecAttnArgs& a, cudaStream_t s) {
  const long long n = a.nk_rows * (a.d / 4);
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  if (cudaError_t e_ = launch_k(dec_combine_kernel, (unsigned)((n + threads - 1) / threads), threads, 0, s, a, hd)) return e_;
  return cudaGetLastError();
}

// Split-key encoder (appending): out = dt((sum_s 2^(m_s - M) O_s) / (sum_s 2^(m_s - M) l_s) * gate),
// M = max_s m_s; one thread per 4 output columns of a row. Every split of a
// valid row holds at least one visible key, so M is finite.
__global__ void enc_combine_kernel(EncAttnArgs a, int hd) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int cols4 = a.d / 4;
  if (gid >= a.rows * cols4) return;
  const long long row = gid / cols4;
  const int c = (int)(gid % cols4) * 4;
  const int h = c / hd;
  float M = -INFINITY;
  for (int s = 0; s < a.n_split; ++s) M = fmaxf(M, a.part_ml[((s * a.rows + row) * a.n_heads + h) * 2]);
  float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < a.n_split; ++s) {
    const float* ml = a.part_ml + ((s * a.rows + row) * a.n_heads + h) * 2;
    if (ml[0] == -INFINITY) continue;  // a split with no keys
    const float w = exp2f(ml[0] - M);
    L = fmaf(w, ml[1], L);
    float v[4];
    load4(a.part_o + (s * a.rows + row) * a.d + c, v);
    for (int i = 0; i < 4; ++i) o[i] = fmaf(w, v[i], o[i]);
  }
  float g[4] = {1.f, 1.f, 1.f, 1.f};
  if (a.gate) load4(a.gate + row * a.d + c, g);
  const float inv = 1.0f / L;
  float r[4] = {o[0] * inv * g[0], o[1] * inv * g[1], o[2] * inv * g[2], o[3] * inv * g[3]};
  store4((bf16*)a.out + row * a.d + c, r);
}

cudaError_t launch_enc_combine(int hd, const EncAttnArgs& a, cudaStream_t s) {
  const long long n = a.rows * (a.d / 4);
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  if (cudaError_t e_ = launch_k(enc_combine_kernel, (unsigned)((n + threads - 1) / threads), threads, 0, s, a, hd)) return e_;
  return cudaGetLastError();
}

// ---------------------------------------------------------------- attention backward
// delta[i, h] = sum over the head's columns of dO * O (one thread per row and head)
template <typename T>
__global__ void attn_bwd_delta_kernel(AttnBwdArgs a, int hd) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= a.rows * a.n_heads) return;
  const long long i = gid / a.n_heads;
  const int h = (int)(gid % a.n_heads);
  const T* o = (const T*)a.o + i * a.d + (long long)h * hd;
  const T* olo = a.o_lo ? (const T*)a.o_lo + i * a.d + (long long)h * hd : nullptr;
  const T* g = (const T*)a.d_o + i * a.d + (long long)h * hd;
  float acc = 0.f;
  for (int c = 0; c < hd; c += 4) {
    float ov[4], gv[4];
    load4(o + c, ov);
    load4(g + c, gv);
    if (olo) {  // O = o + o_lo
      float lv[4];
      load4(olo + c, lv);
      for (int e = 0; e < 4; ++e) ov[e] += lv[e];
    }
    acc += ov[0] * gv[0] + ov[1] * gv[1] + ov[2] * gv[2] + ov[3] * gv[3];
  }
  a.delta[gid] = acc;
}

// dq: one thread per query row i, over the keys j <= i staged in shared memory:
// p = exp(s - lse), ds = p (dO_i . v_j - delta_i), dq_i += ds k_j, times 1/sqrt(d_h).
template <typename T, int HD>
__global__ void __launch_bounds__(ATT_ROWS) attn_bwd_dq_simt_kernel(AttnBwdArgs a) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  __shared__ __align__(16) float Ks[ATT_BK][HD];
  __shared__ __align__(16) float Vs[ATT_BK][HD];
  const EncTile tile = a.tiles[blockIdx.x];
  const int h = blockIdx.y;
  const int s = a.cu[tile.user], L = a.cu[tile.user + 1] - s;
  const int i = tile.q0 + threadIdx.x;
  const bool valid = i < L;
  const long long ro = (long long)(s + (valid ? i : 0)) * a.d + (long long)h * HD;
  float q[HD], go[HD], dq[HD];
#pragma unroll
  for (int c = 0; c < HD; c += 4) {
    load4((const T*)a.q + ro + c, &q[c]);
    load4((const T*)a.d_o + ro + c, &go[c]);
  }
#pragma unroll
  for (int c = 0; c < HD; ++c) {
    q[c] *= a.scale_log2;
    dq[c] = 0.f;
  }
  const long long ri = (long long)(s + (valid ? i : 0)) * a.n_heads + h;
  const float lse2 = a.lse[ri] * 1.4426950408889634f, dlt = a.delta[ri];
  const int kv_end = min(L, tile.q0 + ATT_ROWS);
  const T* K = (const T*)a.k + (long long)s * a.d + (long long)h * HD;
  const T* V = (const T*)a.v + (long long)s * a.d + (long long)h * HD;
  for (int kb = 0; kb < kv_end; kb += ATT_BK) {
    __syncthreads();
    stage_kv<T, HD, ATT_BK>(Ks, Vs, K + (long long)kb * a.d, V + (long long)kb * a.d, a.d, kv_end - kb);
    __syncthreads();
    if (!valid || kb > i) continue;
    const int jmax = min(ATT_BK, i - kb + 1);
    for (int j = 0; j < jmax; ++j) {
      float sc = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < HD; ++c) {
        sc = fmaf(q[c], Ks[j][c], sc);
        dp = fmaf(go[c], Vs[j][c], dp);
      }
      const float ds = exp2f(sc - lse2) * (dp - dlt);
#pragma unroll
      for (int c = 0; c < HD; ++c) dq[c] = fmaf(ds, Ks[j][c], dq[c]);
    }
  }
  if (valid) {
    const float sc = a.scale_log2 * 0.69314718055994531f;  // 1 / sqrt(d_h)
#pragma unroll
    for (int c = 0; c < HD; ++c) dq[c] *= sc;
#pragma unroll
    for (int c = 0; c < HD; c += 4) store4(a.dq + ro + c, &dq[c]);
  }
}

// dk, dv: one thread per key row j, over the queries i >= j staged in shared
// memory: dv_j += p dO_i, dk_j += p (dO_i . v_j - delta_i) q_i, times 1/sqrt(d_h).
template <typename T, int HD>
__global__ void __launch_bounds__(ATT_ROWS) attn_bwd_dkdv_simt_kernel(AttnBwdArgs a) {
  pdl_wait();  // the previous kernel of the stream has completed
  pdl_release();
  __shared__ __align__(16) float Qs[ATT_BK][HD];
  __shared__ __align__(16) float Gs[ATT_BK][HD];
  __shared__ float Ls[ATT_BK], Ds[ATT_BK];
  const EncTile tile = a.tiles[blockIdx.x];
  const int h = blockIdx.y;
  const int s = a.cu[tile.user], L = a.cu[tile.user + 1] - s;
  const int j = tile.q0 + threadIdx.x;
  const bool valid = j < L;
  const long long ro = (long long)(s + (valid ? j : 0)) * a.d + (long long)h * HD;
  float k[HD], v[HD], dk[HD], dv[HD];
#pragma unroll
  for (int c = 0; c < HD; c += 4) {
    load4((const T*)a.k + ro + c, &k[c]);
    load4((const T*)a.v + ro + c, &v[c]);
  }
#pragma unroll
  for (int c = 0; c < HD; ++c) {
    k[c] *= a.scale_log2;
    dk[c] = 0.f;
    dv[c] = 0.f;
  }
  const T* Q = (const T*)a.q + (long long)s * a.d + (long long)h * HD;
  const T* G = (const T*)a.d_o + (long long)s * a.d + (long long)h * HD;
  for (int qb = tile.q0; qb < L; qb += ATT_BK) {
    __syncthreads();
    stage_kv<T, HD, ATT_BK>(Qs, Gs, Q + (long long)qb * a.d, G + (long long)qb * a.d, a.d, L - qb);
    if (threadIdx.x < ATT_BK && qb + (int)threadIdx.x < L) {
      const long long r = (long long)(s + qb + threadIdx.x) * a.n_heads + h;
      Ls[threadIdx.x] = a.lse[r] * 1.4426950408889634f;
      Ds[threadIdx.x] = a.delta[r];
    }
    __syncthreads();
    if (!valid) continue;
    const int imax = min(ATT_BK, L - qb);
    for (int ii = max(0, j - qb); ii < imax; ++ii) {  // causal: query qb + ii >= j
      float sc = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < HD; ++c) {
        sc = fmaf(k[c], Qs[ii][c], sc);
        dp = fmaf(v[c], Gs[ii][c], dp);
      }
      const float p = exp2f(sc - Ls[ii]);
      const float ds = p * (dp - Ds[ii]);
#pragma unroll
      for (int c = 0; c < HD; ++c) {
        dv[c] = fmaf(p, Gs[ii][c], dv[c]);
        dk[c] = fmaf(ds, Qs[ii][c], dk[c]);
      }
    }
  }
  if (valid) {
    const float sc = a.scale_log2 * 0.69314718055994531f;  // 1 / sqrt(d_h)
#pragma unroll
    for (int c = 0; c < HD; ++c) dk[c] *= sc;
#pragma unroll
    for (int c = 0; c < HD; c += 4) {
      store4(a.dk + ro + c, &dk[c]);
      store4(a.dv + ro + c, &dv[c]);
    }
  }
}

template <typename T, int HD>
static cudaError_t attn_bwd_part(int part, const AttnBwdArgs& a, cudaStream_t s) {
  const dim3 grid(a.n_tiles, a.n_heads);
  if (part == 1) return launch_k(attn_bwd_dq_simt_kernel<T, HD>, grid, ATT_ROWS, 0, s, a);
  return launch_k(attn_bwd_dkdv_simt_kernel<T, HD>, grid, ATT_ROWS, 0, s, a);
}

template <typename T>
static cudaError_t attn_bwd_dispatch(int hd, int part, const AttnBwdArgs& a, cudaStream_t s) {
  if (part == 0) {
    const long long n = a.rows * a.n_heads;
    return launch_k(attn_bwd_delta_kernel<T>, (unsigned)((n + 255) / 256), 256, 0, s, a, hd);
  }
  switch (hd) {
    case 16: return attn_bwd_part<T, 16>(part, a, s);
    case 32: return attn_bwd_part<T, 32>(part, a, s);
    case 64: return attn_bwd_part<T, 64>(part, a, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd_simt(bool bf16m, int hd, int part, const AttnBwdArgs& a, cudaStream_t s) {
  if (a.n_tiles == 0) return cudaSuccess;
  return bf16m ? attn_bwd_dispatch<bf16>(hd, part, a, s) : attn_bwd_dispatch<float>(hd, part, a, s);
}

cudaError_t launch_enc_attn_simt(bool bf16m, int hd, const EncAttnArgs& a, cudaStream_t s) {
  if (a.n_tiles == 0) return cudaSuccess;
  return bf16m ? enc_dispatch<bf16>(hd, a, s) : enc_dispatch<float>(hd, a, s);
}

cudaError_t launch_dec_attn_simt(bool bf16m, int hd, const DecAttnArgs& a, cudaStream_t s) {
  if (a.n_tiles == 0) return cudaSuccess;
  return bf16m ? dec_dispatch<bf16>(hd, a, s) : dec_dispatch<float>(hd, a, s);
}

}  // namespace rest
