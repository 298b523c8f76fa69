// tcgen05 GEMM for sm_100a with the fused epilogues of the ReST encoder and
// decoder (bf16 operands, fp32 accumulation in TMEM).
//
// One CTA computes a 128 x BN tile of C = A . B:
//   warp 0       TMA producer: A box [128 rows x 64 K] (K-major, 128B swizzle)
//                and BN/64 boxes of B [64 K rows x 64 N] (N-major, 128B swizzle)
//                per stage, into a STAGES-deep ring;
//   warp 1       allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN,
//                K=16) over the ring and commits each stage back to the producer;
//   warps 2..5   epilogue: tcgen05.ld of the accumulator rows (warp w owns TMEM
//                lanes 32*(w%4)..), the fused epilogue, and the global stores.
// B is read directly from the weight as stored ([K, N] row-major, x . W
// layout), so no transposed copy of any weight is made. The column blocks an
// epilogue must pair (V with its gate Gv; W_1 with W_3) are brought into the
// same tile by choosing which 64-column box of B each slot of the tile loads.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.h"
#include "sm100_common.cuh"

namespace rest {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int NUM_THREADS = 320;  // TMA warp, MMA warp, 8 epilogue warps
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int BOX_B_BYTES = 64 * BK * 2;  // one 64-column box of B: 8 KB

// Global column of B loaded into box b of N-tile t.
__device__ __forceinline__ int b_box_col(const GemmArgs& a, int BN, int t, int b) {
  const int nbh = BN / 128;  // boxes per half tile (paired epilogues)
  const int half = BN / 2;
  if (a.epi == EPI_QKVG) {
    const int d = a.d, nQ = d / BN, nV = d / half;
    if (t < 2 * nQ) return t * BN + 64 * b;
    if (t < 2 * nQ + nV) {
      int u = t - 2 * nQ;
      return b < nbh ? 2 * d + u * half + 64 * b : 3 * d + u * half + 64 * (b - nbh);
    }
    return 4 * d + (t - 2 * nQ - nV) * BN + 64 * b;
  }
  if (a.epi == EPI_SWIGLU) return b < nbh ? t * half + 64 * b : a.d + t * half + 64 * (b - nbh);
  return t * BN + 64 * b;
}

__device__ __forceinline__ void store32(float* p, const float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 4) store4(p + i, &v[i]);
}
// 32 bf16 values as four 16-byte stores
__device__ __forceinline__ void store32(bf16* p, const float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    uint4 u;
    __nv_bfloat162 t0 = __floats2bfloat162_rn(v[i], v[i + 1]), t1 = __floats2bfloat162_rn(v[i + 2], v[i + 3]);
    __nv_bfloat162 t2 = __floats2bfloat162_rn(v[i + 4], v[i + 5]), t3 = __floats2bfloat162_rn(v[i + 6], v[i + 7]);
    u.x = *reinterpret_cast<uint32_t*>(&t0);
    u.y = *reinterpret_cast<uint32_t*>(&t1);
    u.z = *reinterpret_cast<uint32_t*>(&t2);
    u.w = *reinterpret_cast<uint32_t*>(&t3);
    *reinterpret_cast<uint4*>(p + i) = u;
  }
}
// sigmoid from the hardware base-2 exponential and reciprocal (relative
// error about 3e-7; every consumer of these gates rounds to bf16 or feeds a
// bf16 product)
__device__ __forceinline__ float sigmoid_fast(float x) {
  const float e = exp2_approx(-1.4426950408889634f * x);
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
  return r;
}

// Every lane executes the (warp-collective) TMEM loads; only rows < M touch
// global memory.
// The epilogue of one 128 x BN tile, split between two warps per TMEM lane
// quarter (part 0: the first half of the columns, part 1: the second half;
// for the paired epilogues, of each half). Inputs that do not depend on the
// accumulator (the residual row, the rotation table) are loaded by
// epi_prefetch before the accumulator is waited for, so their latency hides
// behind the tile's MMAs. Every lane executes the (warp-collective) TMEM
// loads; only rows < M touch global memory.
template <int BN>
struct EpiIn {
  float v[BN / 2];
};

template <int BN>
__device__ __forceinline__ void epi_prefetch(const GemmArgs& a, int m, int t, bool valid, int part, EpiIn<BN>& in) {
  if (!valid) return;
  const long long ro = (long long)m * a.ldo;
  if (a.epi == EPI_RESID) {
    const float* p = (const float*)a.out0 + ro + t * BN + part * (BN / 2);
#pragma unroll
    for (int j = 0; j < BN / 2; j += 4) load4(p + j, &in.v[j]);
  } else if (a.epi == EPI_QKVG) {
    const int d = a.d, nQ = d / BN;
    if (t < 2 * nQ) {  // cos and sin of the BN/4 column pairs of this part
      const int col0 = (t < nQ ? t : t - nQ) * BN + part * (BN / 2);
      const float* ct = a.cos_t + (long long)m * (d / 2) + col0 / 2;
      const float* st = a.sin_t + (long long)m * (d / 2) + col0 / 2;
#pragma unroll
      for (int j = 0; j < BN / 4; j += 4) {
        load4(ct + j, &in.v[j]);
        load4(st + j, &in.v[BN / 4 + j]);
      }
    }
  }
}

template <int BN>
__device__ __forceinline__ void epilogue(const GemmArgs& a, uint32_t tmem_row, int m, int t, bool valid, int part,
                                         const EpiIn<BN>& in) {
  float v[32];
  const long long ro = (long long)m * a.ldo;
  const int half = BN / 2;
  if (a.epi == EPI_QKVG) {
    const int d = a.d, nQ = d / BN, nV = d / half;
    if (t < 2 * nQ) {  // Q or K: rotate the pairs (ReST eq. 5)
      const bool isq = t < nQ;
      const int col0 = (isq ? t : t - nQ) * BN + part * half;
      bf16* out = (bf16*)(isq ? a.out0 : a.out1) + ro + col0;
#pragma unroll
      for (int c0 = 0; c0 < half; c0 += 32) {
        tmem_ld32(tmem_row + part * half + c0, v);
        if (!valid) continue;
        float w[32];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const float c = in.v[c0 / 2 + jj], sn = in.v[BN / 4 + c0 / 2 + jj];
          w[2 * jj] = v[2 * jj] * c - v[2 * jj + 1] * sn;
          w[2 * jj + 1] = v[2 * jj] * sn + v[2 * jj + 1] * c;
        }
        store32(out + c0, w);
      }
      return;
    }
    if (t < 2 * nQ + nV) {  // value gate: V' = sigmoid(Gv) * V (eq. 3)
      const int col0 = (t - 2 * nQ) * half + part * (half / 2);
      bf16* out = (bf16*)a.out2 + ro + col0;
#pragma unroll
      for (int c0 = 0; c0 < half / 2; c0 += 32) {
        float g[32];
        tmem_ld32(tmem_row + part * (half / 2) + c0, v);
        tmem_ld32(tmem_row + half + part * (half / 2) + c0, g);
        if (!valid) continue;
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= sigmoid_fast(g[j]);
        store32(out + c0, v);
      }
      return;
    }
    // output gate sigmoid(Go) (eq. 4), fp32
    float* out = (float*)a.out3 + ro + (t - 2 * nQ - nV) * BN + part * half;
#pragma unroll
    for (int c0 = 0; c0 < half; c0 += 32) {
      tmem_ld32(tmem_row + part * half + c0, v);
      if (!valid) continue;
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = sigmoid_fast(v[j]);
      store32(out + c0, v);
    }
    return;
  }
  if (a.epi == EPI_SWIGLU) {  // SiLU(x W_1) * (x W_3)
    bf16* out = (bf16*)a.out0 + ro + t * half + part * (half / 2);
#pragma unroll
    for (int c0 = 0; c0 < half / 2; c0 += 32) {
      float u[32];
      tmem_ld32(tmem_row + part * (half / 2) + c0, v);
      tmem_ld32(tmem_row + half + part * (half / 2) + c0, u);
      if (!valid) continue;
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = v[j] * sigmoid_fast(v[j]) * u[j];
      store32(out + c0, v);
    }
    return;
  }
  if (a.epi == EPI_DECQG) {  // q (fp32) or the sigmoid gate (fp32) of token k
    const int per = a.N / BN, g = t / per, nt = t % per, k = g % a.k_tok;
    float* out = (float*)(g < a.k_tok ? a.out0 : a.out1) + ro + (long long)k * a.N + nt * BN + part * half;
#pragma unroll
    for (int c0 = 0; c0 < half; c0 += 32) {
      tmem_ld32(tmem_row + part * half + c0, v);
      if (!valid) continue;
      if (g >= a.k_tok) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = sigmoid_fast(v[j]);
      }
      store32(out + c0, v);
    }
    return;
  }
  const int n0 = t * BN + part * half;
#pragma unroll
  for (int c0 = 0; c0 < half; c0 += 32) {
    tmem_ld32(tmem_row + part * half + c0, v);
    if (!valid) continue;
    switch (a.epi) {
      case EPI_F32: store32((float*)a.out0 + ro + n0 + c0, v); break;
      case EPI_DT: store32((bf16*)a.out0 + ro + n0 + c0, v); break;
      case EPI_SIGMOID: {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = sigmoid_fast(v[j]);
        store32((float*)a.out0 + ro + n0 + c0, v);
        break;
      }
      case EPI_RESID: {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = fmaf(a.alpha, v[j], in.v[c0 + j]);
        store32((float*)a.out0 + ro + n0 + c0, v);
        break;
      }
    }
  }
}

// Persistent kernel: one CTA per SM walks the tiles t = blockIdx.x, +gridDim.x,
// ... (N-tiles of one 128-row block adjacent, so concurrent CTAs share A and
// B in L2). The accumulator is double-buffered in TMEM: the epilogue of tile
// i runs while the MMAs of tile i+1 proceed.
template <int BN, int STAGES>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB2, const GemmArgs a,
                   int num_kb, int n_tiles_n, int n_tiles, int32_t* err) {
  // with a low part A2, the K loop runs twice: A . B, then A2 . B
  const int nkb = a.A2 ? 2 * num_kb : num_kb;
  constexpr int STAGE_BYTES = A_BYTES + BN * BK * 2;
  constexpr int EPI_THREADS = NUM_THREADS - 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tslot;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_THREADS);
    }
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tslot, 2 * BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    prefetch_tmap(&tmA);
    if (a.A2) prefetch_tmap(&tmA2);
    prefetch_tmap(&tmB);
    if (a.B2) prefetch_tmap(&tmB2);
    int it = 0, issued = 0;
    for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x) {
      const int t = tile % n_tiles_n, mt = tile / n_tiles_n;
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % STAGES;
        const int kk = kb < num_kb ? kb : kb - num_kb;
        if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, err, &abort_flag)) break;
        uint8_t* st = smem + s * STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        if (a.epi == EPI_DECQG) {
          // tile t: group g (q of token k = g, or the gate of token k = g - k_tok), N-tile nt
          const int per = a.N / BN, g = t / per, nt = t % per, k = g % a.k_tok;
          tma_load_2d(st, &tmA, k * a.K + kk * BK, mt * BM, &full[s]);
#pragma unroll
          for (int b = 0; b < BN / 64; ++b)
            tma_load_2d(st + A_BYTES + b * BOX_B_BYTES, g < a.k_tok ? &tmB : &tmB2, nt * BN + 64 * b,
                        k * a.K + kk * BK, &full[s]);
        } else {
          tma_load_2d(st, kb < num_kb ? &tmA : &tmA2, kk * BK, mt * BM, &full[s]);
#pragma unroll
          for (int b = 0; b < BN / 64; ++b)
            tma_load_2d(st + A_BYTES + b * BOX_B_BYTES, &tmB, b_box_col(a, BN, t, b), kk * BK, &full[s]);
        }
        issued = it + 1;
      }
    }
    if (abort_flag) {  // let the copies already in flight land before the CTA exits
      volatile int no_abort = 0;
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, nullptr, &no_abort);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16(BN, 1);
    int it = 0, i = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++i) {
      const int b = i & 1;
      // the epilogue has drained this accumulator (tile i-2)
      if (!mbar_wait(&acc_empty[b], ((i >> 1) & 1) ^ 1, err, &abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t acc = tmem + b * BN;
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&full[s], (it / STAGES) & 1, err, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * STAGE_BYTES);
        const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          // A: K-major, 128B swizzle; a K step of 16 is 32 bytes inside the swizzle row
          const uint64_t ad = smem_desc(a_base + k * 32, 16, 1024, 2);
          // B: N-major, 128B swizzle; 8-row K groups 1024 B apart, 64-column boxes 8 KB apart
          const uint64_t bd = smem_desc(b_base + k * 2048, BOX_B_BYTES, 1024, 2);
          mma_bf16(acc, ad, bd, idesc, (kb | k) != 0);
        }
        mma_commit(&empty[s]);
      }
      if (ok) mma_commit(&acc_full[b]);
    }
    mma_commit(&drain);
    volatile int no_abort = 0;
    mbar_wait(&drain, 0, nullptr, &no_abort);
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue (two warps per TMEM lane quarter)
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;  // warps 2..5: first half of the columns, 6..9: second half
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    int i = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
      const int b = i & 1;
      const int t = tile % n_tiles_n, mt = tile / n_tiles_n;
      const int m = mt * BM + q * 32 + lane;
      EpiIn<BN> in;
      epi_prefetch<BN>(a, m, t, m < a.M, part, in);
      if (!mbar_wait(&acc_full[b], (i >> 1) & 1, err, &abort_flag)) break;
      tc_fence_after();
      epilogue<BN>(a, tmem + b * BN + lane_off, m, t, m < a.M, part, in);
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

// 2-D bf16 tensor map over rows x cols (row stride in elements), box of
// box_cols x box_rows, swizzle of 128 or 64 bytes; out-of-range elements
// read as zero.
bool make_tmap_bf16(CUtensorMap* m, const void* base, long long rows, long long cols, long long stride,
                    int box_cols, int box_rows, int swizzle_bytes) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)stride * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

constexpr int TC_BN = 128;
constexpr int TC_STAGES = 6;  // 192 KB of shared memory, one persistent CTA per SM

template <int BN, int STAGES>
cudaError_t launch_bn(const GemmArgs& a, cudaStream_t s, int32_t* err) {
  CUtensorMap ma, ma2, mb, mb2;
  if (a.epi == EPI_DECQG) {
    // A: z as [M, k_tok * K]; B, B2: the stacked [k_tok * K, N] weights
    if (!make_tmap_bf16(&ma, a.A, a.M, (long long)a.k_tok * a.K, a.lda, BK, BM, 128) ||
        !make_tmap_bf16(&mb, a.B, (long long)a.k_tok * a.K, a.N, a.ldb, 64, BK, 128) ||
        !make_tmap_bf16(&mb2, a.B2, (long long)a.k_tok * a.K, a.N, a.ldb, 64, BK, 128))
      return cudaErrorInvalidValue;
    ma2 = ma;
  } else {
    if (!make_tmap_bf16(&ma, a.A, a.M, a.K, a.lda, BK, BM, 128)) return cudaErrorInvalidValue;
    ma2 = ma;
    if (a.A2 && !make_tmap_bf16(&ma2, a.A2, a.M, a.K, a.lda, BK, BM, 128)) return cudaErrorInvalidValue;
    // B is [K, Ncols] with Ncols = ldb (the full weight width)
    if (!make_tmap_bf16(&mb, a.B, a.K, a.ldb, a.ldb, 64, BK, 128)) return cudaErrorInvalidValue;
    mb2 = mb;
  }
  constexpr int smem = STAGES * (A_BYTES + BN * BK * 2) + 1024;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int n_tiles_n = a.N / BN;
  if (a.epi == EPI_QKVG) n_tiles_n = 5 * a.d / BN;
  if (a.epi == EPI_DECQG) n_tiles_n = 2 * a.k_tok * (a.N / BN);
  const int n_tiles = n_tiles_n * ((a.M + BM - 1) / BM);
  static int n_sm = 0;
  if (n_sm == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      n_sm = 148;
  }
  const int grid = n_tiles < n_sm ? n_tiles : n_sm;
  gemm_tc_kernel<BN, STAGES><<<grid, NUM_THREADS, smem, s>>>(ma, ma2, mb, mb2, a, a.K / BK, n_tiles_n, n_tiles, err);
  return cudaGetLastError();
}

}  // namespace

bool sm100_gemm_supported(const GemmArgs& a) {
  if (a.a_f32) return false;
  if (a.M <= 0 || a.K % BK != 0 || a.K <= 0) return false;
  if ((a.lda % 8) || (a.ldb % 8) || (a.ldo % 8)) return false;
  switch (a.epi) {
    case EPI_QKVG: return a.d % TC_BN == 0 && a.N == 5 * a.d && a.ldb == 5LL * a.d;
    case EPI_SWIGLU: return a.d % (TC_BN / 2) == 0 && a.N == 2 * a.d && a.ldb == 2LL * a.d;
    case EPI_DECQG: return a.N % TC_BN == 0 && a.ldb == a.N && a.B2 != nullptr && a.k_tok >= 1;
    default: return a.N % TC_BN == 0 && a.ldb == a.N;
  }
}

cudaError_t launch_gemm_sm100(const GemmArgs& a, cudaStream_t s, int32_t* err) {
  return launch_bn<TC_BN, TC_STAGES>(a, s, err);
}

}  // namespace rest
