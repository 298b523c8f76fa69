// tcgen05 GEMM for sm_100a with the fused epilogues of the ReST encoder and
// decoder (bf16 operands, or fp16 for the decoder's output projection and the
// score head; fp32 accumulation in TMEM).
//
// CTA pairs (clusters of two CTAs on two SMs) walk tiles of 256 rows of C =
// A . B; each pair tile is one M=256 tcgen05 MMA chain issued by rank 0, with
// rank r holding rows [128 r, 128 r + 128) of A and half of the tile's B
// columns in its own shared memory, and receiving its 128 accumulator rows
// in its own TMEM. Per CTA and K block that is 16 KB of A and 8 or 16 KB of
// B for a 128 x 128 or 128 x 256 output block, half the L2 traffic of a
// single-CTA tile of the same output. In each CTA:
//   warp 0       TMA producer: the CTA's A box [128 rows x 64 K] (K-major,
//                128B swizzle) and its 64-column boxes of B [64 K x 64 N]
//                (N-major, 128B swizzle) into a STAGES-deep ring, completing
//                on rank 0's barriers;
//   warp 1       allocates the pair's TMEM (two accumulators of 256 columns);
//                on rank 0 one thread issues the pair MMAs (M=256, K=16) and
//                commits each stage back to both producers;
//   warps 2..9   epilogue, two warps per TMEM lane quarter: tcgen05.ld of the
//                CTA's rows, the fused epilogue, the result written into a
//                swizzled shared-memory box and sent to global memory by a
//                TMA store; the residual sublayers add into the fp32 residual
//                stream with a TMA reduce-add, so the residual is never loaded;
//   warp 10      for the DGA projection, the tile's rows of the rotation table
//                (cos, sin) into a side slot by TMA, one tile ahead of the
//                epilogue that uses them.
// Tiles are 256 columns wide for the epilogues that pair two column blocks
// (rotated Q with K of the same heads, V with its gate Gv, W_1 with W_3) and
// 128 wide for the fp32 outputs. B is read directly from the weight as stored
// ([K, N] row-major, x . W layout), so no transposed copy of any weight is
// made.
#include <cudaTypedefs.h>

#include <cstring>

#include "kernels.h"
#include "sm100.h"
#include "sm100_common.cuh"

namespace rest {
namespace {

using namespace sm100;

constexpr int BM = 128;  // rows per CTA; a pair tile has 256
constexpr int BK = 64;
constexpr int NUM_THREADS = 352;  // TMA warp, MMA warp, 8 epilogue warps, side-input TMA warp
constexpr int EPI_WARPS = 8;
constexpr int A_BYTES = BM * BK * 2;      // 16 KB
constexpr int BOX_B_BYTES = 64 * BK * 2;  // one 64-column box of B: 8 KB
constexpr int STAGE_BYTES = A_BYTES + 2 * BOX_B_BYTES;
constexpr int ACC_COLS = 256;     // TMEM columns of one accumulator
constexpr int BOX128 = BM * 128;  // a [128 rows x 128 bytes] staging box: 16 KB

// The tensor maps of one launch: operands, side inputs (rotation table) and
// up to four outputs.
struct GemmMaps {
  CUtensorMap a, a2, b, b2;
  CUtensorMap s0, s1;  // EPI_QKVG: cos, sin [M, d/2] fp32, boxes of 32 columns x 128 rows
  CUtensorMap o[4];    // outputs, boxes of 32 rows (see setup_maps)
};

// Width (MMA N) of the tiles: 256 columns (128 per CTA of the pair), 128 for
// the plain bf16 copy. EPI_QKVG tiles (DGA gates): [0, nH) rotated Q and K of
// head group t (128 columns each), [nH, 2 nH) V and Gv, then Go in 256-column
// tiles, with nH = d / 128; the gate variants are laid out by qkvg_tiles().
__host__ __device__ __forceinline__ int tile_n(const GemmArgs& a) { return a.epi == EPI_DT ? 128 : 256; }
// Output columns of a 256-column tile of an fp32 output; the last tile may end past the width.
__host__ __device__ __forceinline__ int f32_tiles(int width) { return (width + 255) / 256; }

// Grouped products: N-tiles per group and the group of N-tile t.
__host__ __device__ __forceinline__ int tiles_per_group(const GemmArgs& a) {
  return a.epi == EPI_SWIGLU ? (a.d + 127) / 128 : f32_tiles(a.N);
}
__host__ __device__ __forceinline__ bool grouped(const GemmArgs& a) {
  return a.groups > 1 && (a.epi == EPI_SWIGLU || a.epi == EPI_RESID || a.epi == EPI_F32);
}

// N-tiles of the DGA projection by gate mode: rotation tiles [0, rot_end),
// value tiles [rot_end, val_end), output-gate tiles after. A rotation tile is
// Q | K of head group t (128 columns each), or with GATES_QKVO X | G_X, X = Q
// for t < nH and K after; a value tile is V | Gv (128 columns each), or 256
// columns of V with GATES_O.
struct QkvgTiles {
  int nH, rot_end, val_end;
};
__host__ __device__ __forceinline__ QkvgTiles qkvg_tiles(const GemmArgs& a) {
  QkvgTiles q;
  q.nH = a.d / 128;
  q.rot_end = a.gate_mode == GATES_QKVO ? 2 * q.nH : q.nH;
  q.val_end = q.rot_end + (a.gate_mode == GATES_O ? (a.d + 255) / 256 : q.nH);
  return q;
}
// First column of the output-gate block W_go in the projection weight.
__host__ __device__ __forceinline__ int go_col(const GemmArgs& a) { return (a.gate_mode == GATES_O ? 3 : 4) * a.d; }

// Global column (in the B map that box_map selects) of the 64-column box b
// that CTA `rank` loads for N-tile t.
__device__ __forceinline__ int b_box_col(const GemmArgs& a, int t, int rank, int b, bool* second_map) {
  *second_map = false;
  if (a.epi == EPI_QKVG) {
    const int d = a.d;
    const QkvgTiles g = qkvg_tiles(a);
    if (t < g.rot_end) {
      if (a.gate_mode == GATES_QKVO) {  // Q | Gq or K | Gk
        const int k = t >= g.nH ? 1 : 0;
        return (rank ? (5 + k) * d : k * d) + (t - k * g.nH) * 128 + 64 * b;
      }
      return (rank ? d : 0) + t * 128 + 64 * b;  // Q | K
    }
    if (t < g.val_end) {
      if (a.gate_mode == GATES_O) return 2 * d + (t - g.rot_end) * 256 + 128 * rank + 64 * b;  // V
      return (rank ? 3 * d : 2 * d) + (t - g.rot_end) * 128 + 64 * b;                          // V | Gv
    }
    *second_map = true;  // Go, through its [K, d] view
    return (t - g.val_end) * 256 + 128 * rank + 64 * b;
  }
  if (grouped(a)) t %= tiles_per_group(a);  // the group's rows of B come from the K offset
  if (a.epi == EPI_SWIGLU) {  // W_1 | W_3, each through its own [K, d_ff] view
    *second_map = rank != 0;
    return t * 128 + 64 * b;
  }
  if (a.epi == EPI_DECQG) {
    const int per = f32_tiles(a.N), g = t / per, nt = t % per;
    *second_map = g >= a.k_tok;
    return nt * 256 + 128 * rank + 64 * b;
  }
  if (a.epi == EPI_DT) return t * 128 + 64 * rank;
  return t * 256 + 128 * rank + 64 * b;
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

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// 32 fp32 values: one 128-byte row (row r) of a 128B-swizzled box
__device__ __forceinline__ void stage_f32(uint8_t* box, int r, const float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 8; ++k)
    *reinterpret_cast<float4*>(box + sw128_off(r, k)) = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
}
// 32 values as bf16 into half (chunks k0..k0+3) of a 128-byte row of a 128B-swizzled box
__device__ __forceinline__ void stage_bf16_sw128(uint8_t* box, int r, int k0, const float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint4 u;
    u.x = pack_bf16(v[8 * k], v[8 * k + 1]);
    u.y = pack_bf16(v[8 * k + 2], v[8 * k + 3]);
    u.z = pack_bf16(v[8 * k + 4], v[8 * k + 5]);
    u.w = pack_bf16(v[8 * k + 6], v[8 * k + 7]);
    *reinterpret_cast<uint4*>(box + sw128_off(r, k0 + k)) = u;
  }
}

// 32 values as fp16 into half (chunks k0..k0+3) of a 128-byte row of a
// 128B-swizzled box; false if one is beyond fp16's range
__device__ __forceinline__ bool stage_f16_sw128(uint8_t* box, int r, int k0, const float (&v)[32]) {
  bool ok = true;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint4 u;
    u.x = pack_f16x2(v[8 * k], v[8 * k + 1]);
    u.y = pack_f16x2(v[8 * k + 2], v[8 * k + 3]);
    u.z = pack_f16x2(v[8 * k + 4], v[8 * k + 5]);
    u.w = pack_f16x2(v[8 * k + 6], v[8 * k + 7]);
    *reinterpret_cast<uint4*>(box + sw128_off(r, k0 + k)) = u;
#pragma unroll
    for (int i = 0; i < 8; ++i) ok = ok && fits_f16(v[8 * k + i]);
  }
  return ok;
}

// Q and K columns of four rotation pairs (ReST eq. 5): outputs 8 bf16 each.
__device__ __forceinline__ uint4 rotate4(const float* p, float4 c, float4 s) {
  uint4 u;
  u.x = pack_bf16(p[0] * c.x - p[1] * s.x, p[0] * s.x + p[1] * c.x);
  u.y = pack_bf16(p[2] * c.y - p[3] * s.y, p[2] * s.y + p[3] * c.y);
  u.z = pack_bf16(p[4] * c.z - p[5] * s.z, p[4] * s.z + p[5] * c.z);
  u.w = pack_bf16(p[6] * c.w - p[7] * s.w, p[6] * s.w + p[7] * c.w);
  return u;
}

// The epilogue of one tile for one epilogue warp: rows r = 32 q + lane of
// the CTA's 128 rows (global rows from y0), a part of the accumulator's
// columns. The result is written into the tile's shared-memory slot as
// 32-row TMA boxes and lane 0 issues their stores. With SIDE (the DGA
// projection) the slot already holds this tile's rotation table rows and is
// known to be free; otherwise the warp first waits until its own stores of
// the previous tile have left the slot.
template <bool SIDE, int NSLOT>
__device__ __forceinline__ void epilogue(const GemmArgs& a, const GemmMaps& mp, uint32_t trow, uint8_t* slot, int t,
                                         int m0, int q, int lane, int part, uint32_t acc_empty_addr, int32_t* err) {
  const int r = q * 32 + lane;
  const int y0 = m0 + q * 32;
  float v[32], w[32];
  auto slot_ready = [&]() {
    if (!SIDE) {
      if (lane == 0) bulk_wait_read<NSLOT - 1>();  // the stores of this slot's previous tile
      __syncwarp();
    }
  };
  auto issue = [&]() {
    fence_async_smem();
    __syncwarp();
  };
  // the accumulator is free for the next MMAs as soon as its last columns are in registers
  auto release = [&]() {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(acc_empty_addr);
  };
  // SIDE holds exactly for the DGA projection (EPI_QKVG): testing it instead of
  // a.epi keeps each instantiation's code to its own epilogues
  const QkvgTiles qt = qkvg_tiles(a);
  if (SIDE && t < qt.rot_end && a.gate_mode == GATES_QKVO) {
    // X = Q or K of head group t % nH, gated by sigmoid(G_X), then rotated; this warp
    // takes pairs [32 part, 32 part + 32), and the output takes the bytes of the cos values
    uint8_t* cb = slot + part * BOX128;
    const uint8_t* sb = slot + (2 + part) * BOX128;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      tmem_ld32x2(trow + part * 64 + 32 * j, v, trow + 128 + part * 64 + 32 * j, w);  // X and G_X columns
      if (j == 1) release();
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= sigmoid_fast(w[i]);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t off = sw128_off(r, 4 * j + kk);
        const float4 c = *reinterpret_cast<const float4*>(cb + off);
        const float4 s = *reinterpret_cast<const float4*>(sb + off);
        *reinterpret_cast<uint4*>(cb + off) = rotate4(v + 8 * kk, c, s);
      }
    }
    issue();
    if (lane == 0) {
      const int k = t >= qt.nH ? 1 : 0;
      tma_store_2d(&mp.o[k], cb + q * 32 * 128, (t - k * qt.nH) * 128 + 64 * part, y0);
      bulk_commit();
    }
    return;
  }
  if (SIDE && t < qt.rot_end) {
    // rotated Q and K of head group t; this warp takes pairs [32 part, 32 part + 32) of both,
    // and the outputs take the bytes of the cos (Q) and sin (K) values they were made from
    uint8_t* cb = slot + part * BOX128;
    uint8_t* sb = slot + (2 + part) * BOX128;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      tmem_ld32x2(trow + part * 64 + 32 * j, v, trow + 128 + part * 64 + 32 * j, w);  // Q and K columns
      if (j == 1) release();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t off = sw128_off(r, 4 * j + kk);
        const float4 c = *reinterpret_cast<const float4*>(cb + off);
        const float4 s = *reinterpret_cast<const float4*>(sb + off);
        const uint4 uq = rotate4(v + 8 * kk, c, s);
        const uint4 uk = rotate4(w + 8 * kk, c, s);
        *reinterpret_cast<uint4*>(cb + off) = uq;
        *reinterpret_cast<uint4*>(sb + off) = uk;
      }
    }
    issue();
    if (lane == 0) {
      tma_store_2d(&mp.o[0], cb + q * 32 * 128, t * 128 + 64 * part, y0);
      tma_store_2d(&mp.o[1], sb + q * 32 * 128, t * 128 + 64 * part, y0);
      bulk_commit();
    }
    return;
  }
  if (SIDE && t < qt.val_end && a.gate_mode == GATES_O) {
    // V without a gate: this warp's 128 accumulator columns as bf16, in two 64-column boxes
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(trow + part * 128 + 32 * c, v);
      if (c == 3) release();
      if (c == 0) slot_ready();
      stage_bf16_sw128(slot + (2 * part + (c >> 1)) * BOX128, r, 4 * (c & 1), v);
    }
    issue();
    if (lane == 0) {
#pragma unroll
      for (int bx = 0; bx < 2; ++bx) {
        const int x = (t - qt.rot_end) * 256 + 128 * part + 64 * bx;
        if (x < a.d) tma_store_2d(&mp.o[2], slot + (2 * part + bx) * BOX128 + q * 32 * 128, x, y0);
      }
      bulk_commit();
    }
    return;
  }
  if ((SIDE && t < qt.val_end) || (!SIDE && a.epi == EPI_SWIGLU)) {
    // V' = sigmoid(Gv) * V (eq. 3) or SiLU(x W_1) * (x W_3): accumulator columns
    // [0, 128) and [128, 256) pair up; this warp makes output columns [64 part, 64 part + 64)
    const bool gate = SIDE;
    const bool lo = !SIDE && a.out1 != nullptr;  // SwiGLU output as a bf16 hi + lo pair (out0, out1)
    uint8_t* box = slot + part * BOX128;
    uint8_t* box_lo = slot + (2 + part) * BOX128;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      tmem_ld32x2(trow + part * 64 + 32 * j, v, trow + 128 + part * 64 + 32 * j, w);
      if (j == 1) release();
      if (gate) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= sigmoid_fast(w[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = v[i] * sigmoid_fast(v[i]) * w[i];
      }
      if (j == 0) slot_ready();
      if (!SIDE && a.f16) {  // the hidden state for an fp16 product
        if (!stage_f16_sw128(box, r, 4 * j, v)) set_error(err, REST_ERR_RANGE);
      } else {
        stage_bf16_sw128(box, r, 4 * j, v);
      }
      if (lo) {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = v[i] - __bfloat162float(__float2bfloat16_rn(v[i]));
        stage_bf16_sw128(box_lo, r, 4 * j, w);
      }
    }
    issue();
    const int tl = SIDE ? t - qt.rot_end : grouped(a) ? t % tiles_per_group(a) : t;
    const int gofs = SIDE || !grouped(a) ? 0 : (t / tiles_per_group(a)) * a.d;
    const int x = tl * 128 + 64 * part;
    if (lane == 0 && x < a.d) {  // the last SwiGLU tile may end past d_ff
      tma_store_2d(&mp.o[gate ? 2 : 0], box + q * 32 * 128, gofs + x, y0);
      if (lo) tma_store_2d(&mp.o[1], box_lo + q * 32 * 128, gofs + x, y0);
      bulk_commit();
    }
    return;
  }
  if (!SIDE && a.epi == EPI_DT) {  // bf16 copy of the accumulator
    uint8_t* box = slot + part * BOX128;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      tmem_ld32(trow + part * 64 + 32 * j, v);
      if (j == 1) release();
      if (j == 0) slot_ready();
      stage_bf16_sw128(box, r, 4 * j, v);
    }
    issue();
    if (lane == 0) {
      tma_store_2d(&mp.o[0], box + q * 32 * 128, t * 128 + 64 * part, y0);
      bulk_commit();
    }
    return;
  }
  if (!SIDE && a.epi == EPI_DECQG && a.out16) {
    // the decoder's q (scaled by alpha) and sigmoid gate in fp16: this warp's 128
    // columns of the 256-column tile as two 64-column fp16 boxes
    const int per = f32_tiles(a.N), g = t / per, nt = t % per, k = g % a.k_tok;
    const bool gate = g >= a.k_tok;
    const int x0 = k * a.N + nt * 256, width = k * a.N + a.N;
    bool in_range = true;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(trow + part * 128 + 32 * c, v);
      if (c == 3) release();
      if (gate) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = sigmoid_fast(v[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= a.alpha;
      }
      if (c == 0) slot_ready();
      in_range = stage_f16_sw128(slot + (2 * part + (c >> 1)) * BOX128, r, 4 * (c & 1), v) && in_range;
    }
    if (!in_range) set_error(err, REST_ERR_RANGE);
    issue();
    if (lane == 0) {
#pragma unroll
      for (int bx = 0; bx < 2; ++bx) {
        const int x = x0 + part * 128 + 64 * bx;
        if (x < width) tma_store_2d(&mp.o[gate ? 1 : 0], slot + (2 * part + bx) * BOX128 + q * 32 * 128, x, y0);
      }
      bulk_commit();
    }
    return;
  }
  // fp32 outputs (256-column tiles, this warp's 128 columns in four 32-column
  // chunks through two staging boxes): the output gate sigmoid(Go) (eq. 4),
  // plain, sigmoid, the decoder's q / gate, or the residual add
  const CUtensorMap* om = &mp.o[0];
  int x0 = t * 256, width = a.N;
  if (!SIDE && grouped(a)) {  // group g writes columns [g N, g N + N)
    const int g = t / tiles_per_group(a);
    x0 = g * a.N + (t % tiles_per_group(a)) * 256;
    width = g * a.N + a.N;
  }
  bool sig = !SIDE && a.epi == EPI_SIGMOID;
  if (SIDE) {
    om = &mp.o[3];
    x0 = (t - qt.val_end) * 256;
    width = a.d;
    sig = true;
  } else if (a.epi == EPI_DECQG) {  // tile t: group g (q of token k = g, or the gate of token k = g - k_tok), N-tile nt
    const int per = f32_tiles(a.N), g = t / per, nt = t % per, k = g % a.k_tok;
    om = g < a.k_tok ? &mp.o[0] : &mp.o[1];
    x0 = k * a.N + nt * 256;
    width = k * a.N + a.N;
    sig = g >= a.k_tok;
  }
  const bool resid = !SIDE && a.epi == EPI_RESID;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    tmem_ld32(trow + part * 128 + 32 * c, v);
    if (c == 3) release();
    if (resid) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= a.alpha;
    } else if (sig) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = sigmoid_fast(v[i]);
    }
    uint8_t* box = slot + (2 * part + (c & 1)) * BOX128;
    if (c >= 2 || !SIDE) {  // the store that last read this box (two chunks back) is done
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
    }
    stage_f32(box, r, v);
    issue();
    const int x = x0 + part * 128 + 32 * c;
    if (lane == 0 && x < width) {
      const uint8_t* src = box + q * 32 * 128;
      // x_res += alpha * acc: the add happens at the residual's home in memory
      if (resid) tma_reduce_add_2d(om, src, x, y0);
      else tma_store_2d(om, src, x, y0);
    }
    if (lane == 0) bulk_commit();
  }
}

// Persistent kernel: pair c walks the pair tiles c, c + n_pairs, ... (N-tiles
// of one 256-row block adjacent, so concurrent pairs share A and B in L2).
// The accumulator is double-buffered in TMEM: the epilogue of tile i runs
// while the MMAs of tile i+1 proceed. NSLOT shared-memory slots of SLOT
// bytes hold the epilogue's side inputs and staged outputs; with SIDE the
// producer fills slot i % 2 for tile i once every epilogue warp of its CTA
// has released it (after the stores of tile i - 2 have read it out).
// Barriers: full[s] and acc_empty[b] of rank 0 collect both CTAs (the TMA
// bytes of both, the epilogue warps of both); empty[s], acc_full[b] and the
// side barriers are per CTA, the MMA commits arriving on both CTAs' copies.
template <int STAGES, int NSLOT, int SLOT, bool SIDE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ GemmMaps mp, const GemmArgs a, int num_kb, int n_tiles_n, int n_tiles,
                   int32_t* err) {
  static_assert(!SIDE || NSLOT == 2, "side inputs are double-buffered");
  // with a low part A2, the K loop runs twice: A . B, then A2 . B
  const int nkb = a.A2 ? 2 * num_kb : num_kb;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* slots = smem + STAGES * STAGE_BYTES;
  __shared__ uint64_t full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], side_full[2], side_empty[2], drain;
  __shared__ uint32_t tslot;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster_rank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const QkvgTiles qt = qkvg_tiles(a);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * EPI_WARPS);
      mbar_init(&side_full[b], 1);
      mbar_init(&side_empty[b], EPI_WARPS);
    }
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(&tslot, 2 * ACC_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or complete_tx
  tc_fence_after();
  const uint32_t tmem = tslot;
  pdl_wait();  // the previous kernel of the stream has completed: its outputs may be read
  pdl_release();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    prefetch_tmap(&mp.a);
    if (a.A2) prefetch_tmap(&mp.a2);
    prefetch_tmap(&mp.b);
    if (a.B2 || a.epi == EPI_SWIGLU || a.epi == EPI_QKVG) prefetch_tmap(&mp.b2);
    int it = 0, issued = 0;
    for (int tile = pair; tile < n_tiles && !abort_flag; tile += n_pairs) {
      const int t = tile % n_tiles_n;
      const int m0 = (tile / n_tiles_n) * 2 * BM + rank * BM;
      const int nb = tile_n(a) / 128;  // 64-column boxes of B per CTA
      const uint32_t tx = 2 * (A_BYTES + nb * BOX_B_BYTES);
      // decoder projections: token type k selects the column block of z and the row block of the weights
      const int kofs = a.epi == EPI_DECQG ? ((t / f32_tiles(a.N)) % a.k_tok) * a.K
                       : grouped(a)       ? (t / tiles_per_group(a)) * a.K
                                          : 0;
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % STAGES;
        const int kk = kb < num_kb ? kb : kb - num_kb;
        if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, err, &abort_flag)) break;
        uint8_t* st = smem + s * STAGE_BYTES;
        if (rank == 0) mbar_arrive_expect_tx(&full[s], tx);
        const uint32_t fb = peer_addr(&full[s], 0);
        tma_load_2d_pair(st, kb < num_kb ? &mp.a : &mp.a2, kofs + kk * BK, m0, fb);
        for (int b = 0; b < nb; ++b) {
          bool second;
          const int col = b_box_col(a, t, rank, b, &second);
          tma_load_2d_pair(st + A_BYTES + b * BOX_B_BYTES, second ? &mp.b2 : &mp.b, col, kofs + kk * BK, fb);
        }
        issued = it + 1;
      }
    }
    if (abort_flag) {  // let the copies already in flight land before the CTA exits
      volatile int no_abort = 0;
      for (int j = (issued > STAGES ? issued - STAGES : 0); rank == 0 && j < issued; ++j)
        mbar_wait(&full[j % STAGES], (j / STAGES) & 1, nullptr, &no_abort);
    }
  } else if (SIDE && warp == 10 && lane == 0) {
    // ------------------------------------------------ side-input TMA (DGA projection)
    // the rotation table rows of a Q/K tile into slot i % 2 once every epilogue
    // warp has released it; other tiles only pass the slot on
    prefetch_tmap(&mp.s0);
    prefetch_tmap(&mp.s1);
    int i = 0, side_issued = 0;
    for (int tile = pair; tile < n_tiles && !abort_flag; tile += n_pairs, ++i) {
      const int t = tile % n_tiles_n;
      const int m0 = (tile / n_tiles_n) * 2 * BM + rank * BM;
      const int s = i & 1;
      if (!mbar_wait(&side_empty[s], ((i >> 1) & 1) ^ 1, err, &abort_flag)) break;
      if (t < qt.rot_end) {
        const int hg = t % qt.nH;  // head group of the tile's columns
        uint8_t* sl = slots + s * SLOT;
        mbar_arrive_expect_tx(&side_full[s], 4 * BOX128);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          tma_load_2d(sl + p * BOX128, &mp.s0, hg * 64 + 32 * p, m0, &side_full[s]);
          tma_load_2d(sl + (2 + p) * BOX128, &mp.s1, hg * 64 + 32 * p, m0, &side_full[s]);
        }
        side_issued = i + 1;
      } else {
        mbar_arrive(&side_full[s]);
      }
    }
    if (abort_flag) {  // let the copies already in flight land before the CTA exits
      volatile int no_abort = 0;
      for (int j = (side_issued > 2 ? side_issued - 2 : 0); j < side_issued; ++j)
        mbar_wait(&side_full[j & 1], (j >> 1) & 1, nullptr, &no_abort);
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------ MMA issuer (rank 0 only)
    // The whole warp runs the loop and one elected lane issues: a lone lane of a
    // diverged warp took about 160 cycles per N = 256 pair MMA, a whole warp about
    // 127, against about 128 of tensor work per SM (measured).
    int it = 0, i = 0;
    bool ok = true;
    for (int tile = pair; tile < n_tiles && ok; tile += n_pairs, ++i) {
      const uint32_t idesc = a.f16 ? idesc_f16_pair(tile_n(a)) : idesc_bf16_pair(tile_n(a));
      const int b = i & 1;
      // both CTAs' epilogues have drained this accumulator (tile i-2)
      if (!mbar_wait(&acc_empty[b], ((i >> 1) & 1) ^ 1, err, &abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t acc = tmem + b * ACC_COLS;
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
          mma_bf16_pair_e(acc, ad, bd, idesc, (kb | k) != 0);
        }
        mma_commit_pair_e(&empty[s]);
      }
      if (ok) mma_commit_pair_e(&acc_full[b]);
    }
    mma_commit_pair_e(&drain);
    volatile int no_abort = 0;
    mbar_wait(&drain, 0, nullptr, &no_abort);
  } else if (warp >= 2 && warp < 10) {
    // ------------------------------------------------ epilogue (two warps per TMEM lane quarter)
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;  // warps 2..5: first half of the columns, 6..9: second half
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t acc_empty0[2] = {peer_addr(&acc_empty[0], 0), peer_addr(&acc_empty[1], 0)};
    int i = 0;
    for (int tile = pair; tile < n_tiles; tile += n_pairs, ++i) {
      const int b = i & 1;
      const int t = tile % n_tiles_n;
      const int m0 = (tile / n_tiles_n) * 2 * BM + rank * BM;
      if (SIDE) {
        // release the previous tile's slot once this warp's stores have read it out
        if (i > 0 && lane == 0) {
          bulk_wait_read<0>();
          mbar_arrive(&side_empty[(i - 1) & 1]);
        }
        if (!mbar_wait(&side_full[i & 1], (i >> 1) & 1, err, &abort_flag)) break;
      }
      if (!mbar_wait(&acc_full[b], (i >> 1) & 1, err, &abort_flag)) break;
      tc_fence_after();
      epilogue<SIDE, NSLOT>(a, mp, tmem + b * ACC_COLS + lane_off, slots + (i % NSLOT) * SLOT, t, m0, q, lane, part,
                            acc_empty0[b], err);
    }
    if (lane == 0) bulk_wait<0>();  // every store has completed before the CTA's shared memory goes away
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs, remote arrivals and TMEM reads are all done
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 2 * ACC_COLS);
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

// 2-D tensor map over a row-major [rows, cols] array of 2- or 4-byte
// elements (row stride in elements), box of box_cols x box_rows, swizzle of
// 128, 64 or 0 bytes; out-of-range elements read as zero and are not written.
bool make_tmap(CUtensorMap* m, bool f32, const void* base, long long rows, long long cols, long long stride,
               int box_cols, int box_rows, int swizzle_bytes) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)stride * es};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Operand, side-input and output maps of one launch (unused maps stay zero).
bool setup_maps(const GemmArgs& a, GemmMaps& mp) {
  memset(&mp, 0, sizeof(mp));
  bool ok = true;
  if (a.epi == EPI_DECQG) {
    // A: z as [M, k_tok * K]; B, B2: the stacked [k_tok * K, N] weights
    const long long kk = (long long)a.k_tok * a.K;
    ok = make_tmap(&mp.a, false, a.A, a.M, kk, a.lda, BK, BM, 128) &&
         make_tmap(&mp.b, false, a.B, kk, a.N, a.ldb, 64, BK, 128) &&
         make_tmap(&mp.b2, false, a.B2, kk, a.N, a.ldb, 64, BK, 128);
    mp.a2 = mp.a;
  } else {
    const long long G = grouped(a) ? a.groups : 1, KG = G * a.K;  // grouped: the groups' K blocks side by side
    ok = make_tmap(&mp.a, false, a.A, a.M, KG, a.lda, BK, BM, 128);
    mp.a2 = mp.a;
    if (ok && a.A2) ok = make_tmap(&mp.a2, false, a.A2, a.M, KG, a.lda, BK, BM, 128);
    if (a.epi == EPI_SWIGLU) {
      // W_1 and W_3 as two [K, d_ff] views of the [K, 2 d_ff] weight, so that a
      // ragged last tile reads zeros past d_ff rather than the other block
      const bf16* w = static_cast<const bf16*>(a.B);
      ok = ok && make_tmap(&mp.b, false, w, KG, a.d, a.ldb, 64, BK, 128) &&
           make_tmap(&mp.b2, false, w + a.d, KG, a.d, a.ldb, 64, BK, 128);
    } else {
      // B is [K, Ncols] with Ncols = ldb (the full weight width)
      ok = ok && make_tmap(&mp.b, false, a.B, KG, a.ldb, a.ldb, 64, BK, 128);
      mp.b2 = mp.b;
      // the output-gate block W_go as its own [K, d] view (a ragged last Go tile reads zeros)
      if (ok && a.epi == EPI_QKVG)
        ok = make_tmap(&mp.b2, false, static_cast<const bf16*>(a.B) + go_col(a), a.K, a.d, a.ldb, 64, BK, 128);
    }
  }
  if (!ok) return false;
  switch (a.epi) {
    case EPI_QKVG: {
      const int d = a.d;
      return make_tmap(&mp.s0, true, a.cos_t, a.M, d / 2, d / 2, 32, BM, 128) &&
             make_tmap(&mp.s1, true, a.sin_t, a.M, d / 2, d / 2, 32, BM, 128) &&
             make_tmap(&mp.o[0], false, a.out0, a.M, d, a.ldo, 64, 32, 128) &&
             make_tmap(&mp.o[1], false, a.out1, a.M, d, a.ldo, 64, 32, 128) &&
             make_tmap(&mp.o[2], false, a.out2, a.M, d, a.ldo, 64, 32, 128) &&
             make_tmap(&mp.o[3], true, a.out3, a.M, d, a.ldo, 32, 32, 128);
    }
    case EPI_SWIGLU: {
      const long long wd = (grouped(a) ? a.groups : 1) * (long long)a.d;
      return make_tmap(&mp.o[0], false, a.out0, a.M, wd, a.ldo, 64, 32, 128) &&
             (!a.out1 || make_tmap(&mp.o[1], false, a.out1, a.M, wd, a.ldo, 64, 32, 128));
    }
    case EPI_DT: return make_tmap(&mp.o[0], false, a.out0, a.M, a.N, a.ldo, 64, 32, 128);
    case EPI_DECQG: {
      const long long w = (long long)a.k_tok * a.N;
      if (a.out16)  // fp16 q and gate, 64-column boxes
        return make_tmap(&mp.o[0], false, a.out0, a.M, w, a.ldo, 64, 32, 128) &&
               make_tmap(&mp.o[1], false, a.out1, a.M, w, a.ldo, 64, 32, 128);
      return make_tmap(&mp.o[0], true, a.out0, a.M, w, a.ldo, 32, 32, 128) &&
             make_tmap(&mp.o[1], true, a.out1, a.M, w, a.ldo, 32, 32, 128);
    }
    default: return make_tmap(&mp.o[0], true, a.out0, a.M, (grouped(a) ? a.groups : 1) * (long long)a.N, a.ldo, 32,
                              32, 128);
  }
}

template <int STAGES, int NSLOT, int SLOT, bool SIDE>
cudaError_t launch_cfg(const GemmArgs& a, cudaStream_t s, int32_t* err) {
  if (SIDE != (a.epi == EPI_QKVG)) return cudaErrorInvalidValue;  // the epilogue relies on it
  GemmMaps mp;
  if (!setup_maps(a, mp)) return cudaErrorInvalidValue;
  auto kern = gemm_tc_kernel<STAGES, NSLOT, SLOT, SIDE>;
  constexpr int smem = STAGES * STAGE_BYTES + NSLOT * SLOT + 1024;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait()
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // pairs that can be resident at once (one CTA per SM)
  static int max_pairs = 0;
  if (max_pairs == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(2 * 74);
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    max_pairs = n;
  }
  int n_tiles_n = f32_tiles(a.N);
  if (a.epi == EPI_DT) n_tiles_n = a.N / 128;
  if (a.epi == EPI_QKVG) n_tiles_n = qkvg_tiles(a).val_end + f32_tiles(a.d);
  if (a.epi == EPI_SWIGLU) n_tiles_n = (a.d + 127) / 128;
  if (a.epi == EPI_DECQG) n_tiles_n = 2 * a.k_tok * f32_tiles(a.N);
  if (grouped(a)) n_tiles_n = a.groups * tiles_per_group(a);
  const int n_tiles = n_tiles_n * ((a.M + 2 * BM - 1) / (2 * BM));
  cfg.gridDim = dim3(2 * (n_tiles < max_pairs ? n_tiles : max_pairs));
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, mp, a, a.K / BK, n_tiles_n, n_tiles, err);
}

}  // namespace

bool make_tmap_bf16(CUtensorMap* m, const void* base, long long rows, long long cols, long long stride,
                    int box_cols, int box_rows, int swizzle_bytes) {
  return make_tmap(m, false, base, rows, cols, stride, box_cols, box_rows, swizzle_bytes);
}

bool sm100_gemm_supported(const GemmArgs& a) {
  if (a.a_f32) return false;
  if (a.f16 && (a.A2 || a.out1 || (a.epi != EPI_SWIGLU && a.epi != EPI_RESID && a.epi != EPI_F32))) return false;
  if (a.out16 && (a.f16 || a.epi != EPI_DECQG)) return false;
  if (a.M <= 0 || a.K % BK != 0 || a.K <= 0) return false;
  if ((a.lda % 8) || (a.ldb % 8) || (a.ldo % 8)) return false;
  switch (a.epi) {
    case EPI_QKVG:
      return a.d % 128 == 0 && a.N == gate_blocks(a.gate_mode) * a.d && a.ldb == (long long)a.N;
    case EPI_SWIGLU: return a.d % 64 == 0 && a.N == 2 * a.d && a.ldb == 2LL * a.d;
    case EPI_DECQG: return a.N % 128 == 0 && a.ldb == a.N && a.B2 != nullptr && a.k_tok >= 1;
    default: return a.N % 128 == 0 && a.ldb == a.N;
  }
}

// Shared memory per configuration: stages of 32 KB plus the epilogue slots
// (224 KB in each case, one CTA per SM).
cudaError_t launch_gemm_sm100(const GemmArgs& a, cudaStream_t s, int32_t* err) {
  switch (a.epi) {
    case EPI_QKVG: return launch_cfg<3, 2, 65536, true>(a, s, err);                  // cos + sin in, double-buffered
    case EPI_SWIGLU:
      if (a.out1) return launch_cfg<5, 1, 65536, false>(a, s, err);  // bf16 hi + lo out
      return launch_cfg<5, 2, 32768, false>(a, s, err);               // bf16 out, double-buffered
    case EPI_DT: return launch_cfg<5, 2, 32768, false>(a, s, err);
    default: return launch_cfg<5, 1, 65536, false>(a, s, err);                       // fp32 out (store or residual add)
  }
}

}  // namespace rest
