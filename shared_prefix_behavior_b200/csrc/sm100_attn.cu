// tcgen05 / TMEM / TMA attention for sm_100a: the causal Dual-Gated
// Attention of the ReST encoder (§3.2.1 eqs. 3-4) and the shared-prefix,
// projection-free cross attention of the decoder (§3.3.1 eq. 7, §3.5).
//
// One CTA owns 128 query rows of one head (one thread per row in the
// softmax warpgroup) and streams 128-key blocks:
//   warp 0       TMA producer. Encoder: Q once, then K and V' tiles per
//                block. Decoder: one H tile per block, which serves as both
//                the keys (K-major operand of S = q H^T) and the values
//                (N-major operand of O = P H): H crosses HBM once per
//                (request, head) and is staged once per block.
//   warp 1       TMEM owner and MMA issuer: S_j = Q K_j^T into one of two
//                128-column TMEM buffers, O_j = P_j V_j into one of two
//                head_dim-column buffers; commits release smem stages.
//   warps 2..5   softmax: a thread reads its row of S_j from TMEM, masks,
//                takes the running max, exponentiates in base 2, writes P_j
//                (bf16) to shared memory in the 128B-swizzled K-major layout
//                the MMA reads, and folds O_{j-1} into fp32 registers.
// The decoder's query comes in fp32; it is staged as a hi + lo pair of bf16
// tiles and S accumulates q_hi H^T + q_lo H^T. When the encoder ran in the
// same call, the decoder also reads H's low part (H = H_hi + H_lo, from the
// encoder's fp32 residual stream): S adds q_hi H_lo^T and O adds P H_lo.
//
// MODE 0: encoder; 1: decoder over H; 2: decoder over H_hi + H_lo.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.h"
#include "sm100_common.cuh"

namespace rest {
namespace {

using namespace sm100;

constexpr int ROWS = 128;      // query rows per CTA
constexpr int KB = 128;        // keys per block
constexpr int NTHREADS = 192;
constexpr int KV_STAGES = 3;

template <int HD>
struct Cfg {
  static constexpr int ROW_BYTES = HD * 2;                   // one bf16 row of a head slice
  static constexpr int TILE_BYTES = ROWS * ROW_BYTES;        // 128 rows
  static constexpr int SWZ = HD == 64 ? 2 : 4;               // descriptor code: 128B / 64B swizzle
  static constexpr int ATOM = 8 * ROW_BYTES;                 // bytes of 8 swizzled rows
  static constexpr int P_BYTES = ROWS * KB * 2;              // 32 KB
  static constexpr uint32_t TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O0 = 256, TMEM_O1 = 256 + HD;
};

// byte offset of 16-byte chunk u (0..ROW_BYTES/16-1) of row r in a swizzled tile
template <int HD>
__device__ __forceinline__ uint32_t swz_off(int r, int u) {
  constexpr int CH = Cfg<HD>::ROW_BYTES / 16;  // chunks per row: 8 (128B) or 4 (64B)
  return r * Cfg<HD>::ROW_BYTES + ((u ^ ((r >> (HD == 64 ? 0 : 1)) & (CH - 1))) * 16);
}

template <int HD, int MODE>
struct SmemLayout {
  // [Q (hi) | Q lo (decoder) | KV stages | P x2], every block 1024-aligned.
  // A stage holds K and V' (encoder), H (decoder), or H_hi and H_lo.
  static constexpr int Q = 0;
  static constexpr int QLO = Cfg<HD>::TILE_BYTES;
  static constexpr int KV = (MODE >= 1 ? 2 : 1) * Cfg<HD>::TILE_BYTES;
  static constexpr int STAGE = (MODE == 1 ? 1 : 2) * Cfg<HD>::TILE_BYTES;
  static constexpr int P = KV + KV_STAGES * STAGE;
  static constexpr int TOTAL = P + 2 * Cfg<HD>::P_BYTES;
};

struct AttnWork {
  int q_row0;     // first query row (packed row index: encoder token / decoder q row)
  int nrows;      // valid query rows (<= 128)
  int key_row0;   // first key row in the packed [T, d] array
  int nkeys;      // keys visible to the last query row (encoder: causal bound)
  int causal_off; // encoder: position of query row 0 minus position of key row 0
};

template <int HD, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, EncAttnArgs ea, DecAttnArgs da, int32_t* err) {
  constexpr bool DEC = MODE >= 1, HLO = MODE == 2;
  using C = Cfg<HD>;
  using L = SmemLayout<HD, MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t q_full, kv_full[KV_STAGES], kv_empty[KV_STAGES], s_full[2], p_full[2], p_free[2], o_full[2],
      o_free[2], drain;
  __shared__ uint32_t tslot;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_heads = DEC ? da.n_heads : ea.n_heads;
  const int d = DEC ? da.d : ea.d;
  const int tile = blockIdx.x / n_heads, h = blockIdx.x % n_heads;

  // ---------------------------------------------------------------- work item
  AttnWork w;
  if (DEC) {
    DecTile t = da.tiles[tile];
    w = AttnWork{t.row0, t.nrows, t.key0, t.nkeys, 0};
  } else {
    EncTile t = ea.tiles[tile];
    int s = ea.cu[t.user], Lu = ea.cu[t.user + 1] - s;
    w = AttnWork{s + t.q0, min(ROWS, Lu - t.q0), s, min(Lu, t.q0 + ROWS), t.q0};
  }
  const int nblk = (w.nkeys + KB - 1) / KB;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, DEC ? 128 : 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&p_free[b], 1);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], 128);
    }
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      if (!DEC) {
        mbar_arrive_expect_tx(&q_full, C::TILE_BYTES);
        tma_load_2d(smem + L::Q, &tmQ, h * HD, w.q_row0, &q_full);
      }
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int st = j % KV_STAGES;
        if (!mbar_wait(&kv_empty[st], ((j / KV_STAGES) & 1) ^ 1, err, &abort_flag)) break;
        uint8_t* base = smem + L::KV + st * L::STAGE;
        mbar_arrive_expect_tx(&kv_full[st], L::STAGE);
        tma_load_2d(base, &tmK, h * HD, w.key_row0 + j * KB, &kv_full[st]);
        if (MODE != 1) tma_load_2d(base + C::TILE_BYTES, &tmV, h * HD, w.key_row0 + j * KB, &kv_full[st]);
        issued = j + 1;
      }
      if (abort_flag) {
        volatile int no_abort = 0;
        if (!DEC) mbar_wait(&q_full, 0, nullptr, &no_abort);
        for (int j = (issued > KV_STAGES ? issued - KV_STAGES : 0); j < issued; ++j)
          mbar_wait(&kv_full[j % KV_STAGES], (j / KV_STAGES) & 1, nullptr, &no_abort);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idS = idesc_bf16(KB, 0);   // N = 128 keys, B (keys) K-major
      constexpr uint32_t idO = idesc_bf16(HD, 1);   // N = head_dim, B (values) N-major
      bool ok = mbar_wait(&q_full, 0, err, &abort_flag);
      tc_fence_after();
      const uint32_t q_base = smem_u32(smem + L::Q);
      const uint32_t qlo_base = smem_u32(smem + L::QLO);
      for (int j = 0; ok && j <= nblk; ++j) {
        if (j < nblk) {
          const int st = j % KV_STAGES;
          if (!mbar_wait(&kv_full[st], (j / KV_STAGES) & 1, err, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_base = smem_u32(smem + L::KV + st * L::STAGE);
          const uint32_t tS = tmem + ((j & 1) ? C::TMEM_S1 : C::TMEM_S0);
#pragma unroll
          for (int k = 0; k < HD / 16; ++k) {
            const uint64_t ad = smem_desc(q_base + k * 32, 16, C::ATOM, C::SWZ);
            const uint64_t bd = smem_desc(k_base + k * 32, 16, C::ATOM, C::SWZ);
            mma_bf16(tS, ad, bd, idS, k != 0);
          }
          if (DEC) {  // + q_lo . H^T
#pragma unroll
            for (int k = 0; k < HD / 16; ++k) {
              const uint64_t ad = smem_desc(qlo_base + k * 32, 16, C::ATOM, C::SWZ);
              const uint64_t bd = smem_desc(k_base + k * 32, 16, C::ATOM, C::SWZ);
              mma_bf16(tS, ad, bd, idS, 1);
            }
          }
          if (HLO) {  // + q_hi . H_lo^T
#pragma unroll
            for (int k = 0; k < HD / 16; ++k) {
              const uint64_t ad = smem_desc(q_base + k * 32, 16, C::ATOM, C::SWZ);
              const uint64_t bd = smem_desc(k_base + C::TILE_BYTES + k * 32, 16, C::ATOM, C::SWZ);
              mma_bf16(tS, ad, bd, idS, 1);
            }
          }
          mma_commit(&s_full[j & 1]);
        }
        if (j >= 1) {
          const int i = j - 1, b = i & 1, st = i % KV_STAGES;
          if (!mbar_wait(&p_full[b], (i >> 1) & 1, err, &abort_flag)) { ok = false; break; }
          if (i >= 2 && !mbar_wait(&o_free[b], ((i - 2) >> 1) & 1, err, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t p_base = smem_u32(smem + L::P + b * C::P_BYTES);
          const uint32_t v_base = smem_u32(smem + L::KV + st * L::STAGE + (DEC ? 0 : C::TILE_BYTES));
          const uint32_t tO = tmem + (b ? C::TMEM_O1 : C::TMEM_O0);
#pragma unroll
          for (int k = 0; k < KB / 16; ++k) {
            const uint64_t ad = smem_desc(p_base + (k >> 2) * (ROWS * 128) + (k & 3) * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(v_base + k * 2 * C::ATOM, 64 * KB * 2, C::ATOM, C::SWZ);
            mma_bf16(tO, ad, bd, idO, k != 0);
          }
          if (HLO) {  // + P . H_lo
#pragma unroll
            for (int k = 0; k < KB / 16; ++k) {
              const uint64_t ad = smem_desc(p_base + (k >> 2) * (ROWS * 128) + (k & 3) * 32, 16, 1024, 2);
              const uint64_t bd = smem_desc(v_base + C::TILE_BYTES + k * 2 * C::ATOM, 64 * KB * 2, C::ATOM, C::SWZ);
              mma_bf16(tO, ad, bd, idO, 1);
            }
          }
          mma_commit(&o_full[b]);
          mma_commit(&p_free[b]);
          mma_commit(&kv_empty[st]);
        }
      }
      mma_commit(&drain);
      volatile int no_abort = 0;
      mbar_wait(&drain, 0, nullptr, &no_abort);
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int q = warp & 3;
    const int r = q * 32 + lane;                  // row within the tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool valid = r < w.nrows;
    const float sl2 = DEC ? da.scale_log2 : ea.scale_log2;

    if (DEC) {  // stage q (fp32) as hi + lo bf16 tiles in the swizzled K-major layout
      const float* qrow = da.q + (long long)(w.q_row0 + (valid ? r : 0)) * d + h * HD;
#pragma unroll
      for (int u = 0; u < HD / 8; ++u) {
        float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (valid) {
          load4(qrow + 8 * u, v);
          load4(qrow + 8 * u + 4, v + 4);
        }
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
          float2 hf = __bfloat1622float2(h2);
          __nv_bfloat162 l2 = __floats2bfloat162_rn(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
          hi[e] = *reinterpret_cast<uint32_t*>(&h2);
          lo[e] = *reinterpret_cast<uint32_t*>(&l2);
        }
        const uint32_t off = swz_off<HD>(r, u);
        *reinterpret_cast<uint4*>(smem + L::Q + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(smem + L::QLO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_async_smem();
      mbar_arrive(&q_full);
    }

    float acc[HD];
#pragma unroll
    for (int c = 0; c < HD; ++c) acc[c] = 0.f;
    float m_run = -INFINITY;  // running max after the last block (log2 domain)
    float l_run = 0.f;        // running sum of exponentials, relative to m_run
    float m_acc = -INFINITY;  // max that acc is expressed relative to
    bool ok = true;
    // O_i (relative to m_i) folded into acc: acc = acc * 2^(m_acc - m_i) + O_i
    auto fold = [&](int i, float m_i) -> bool {
      const int bo = i & 1;
      if (!mbar_wait(&o_full[bo], (i >> 1) & 1, err, &abort_flag)) return false;
      tc_fence_after();
      const uint32_t tO = tmem + lane_off + (bo ? C::TMEM_O1 : C::TMEM_O0);
      const float f = exp2_approx(m_acc - m_i);
#pragma unroll
      for (int c0 = 0; c0 < HD; c0 += 32) {
        float t32[32];
        tmem_ld32(tO + c0, t32);
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[c0 + e] = fmaf(acc[c0 + e], f, t32[e]);
      }
      tc_fence_before();
      mbar_arrive(&o_free[bo]);
      m_acc = m_i;
      return true;
    };
    for (int j = 0; j < nblk; ++j) {
      const int b = j & 1;
      if (!mbar_wait(&s_full[b], (j >> 1) & 1, err, &abort_flag)) { ok = false; break; }
      tc_fence_after();
      float s[KB];
      const uint32_t tS = tmem + lane_off + (b ? C::TMEM_S1 : C::TMEM_S0);
#pragma unroll
      for (int c0 = 0; c0 < KB; c0 += 32) {
        float t32[32];
        tmem_ld32(tS + c0, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c0 + i] = t32[i];
      }
      // keys visible to this row in block j: index < lim (the tail; and causality in the encoder)
      int lim = w.nkeys - j * KB;
      if (!DEC) lim = min(lim, w.causal_off + r + 1 - j * KB);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < KB; ++c) {
        s[c] = (c < lim) ? s[c] * sl2 : -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      const float m_old = m_run;
      const float m_new = fmaxf(m_run, mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < KB; ++c) {
        s[c] = exp2_approx(s[c] - m_use);
        sum += s[c];
      }
      l_run = l_run * exp2_approx(m_old - m_use) + sum;
      m_run = m_use;
      // P_j -> shared memory, once PV_{j-2} has finished reading this buffer
      if (j >= 2 && !mbar_wait(&p_free[b], ((j - 2) >> 1) & 1, err, &abort_flag)) { ok = false; break; }
      uint8_t* pb = smem + L::P + b * C::P_BYTES;
#pragma unroll
      for (int u = 0; u < KB / 8; ++u) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __nv_bfloat162 t2 = __floats2bfloat162_rn(s[8 * u + 2 * e], s[8 * u + 2 * e + 1]);
          pk[e] = *reinterpret_cast<uint32_t*>(&t2);
        }
        const int chunk = u >> 3, uu = u & 7;
        *reinterpret_cast<uint4*>(pb + chunk * (ROWS * 128) + r * 128 + ((uu ^ (r & 7)) * 16)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
      if (j >= 1 && !fold(j - 1, m_old)) { ok = false; break; }
    }
    if (ok && nblk > 0) ok = fold(nblk - 1, m_run);
    if (ok && valid) {
      const float inv = 1.0f / l_run;
      const long long ro = (long long)(w.q_row0 + r) * d + h * HD;
      const float* gate = (DEC ? da.g : ea.gate) + ro;
#pragma unroll
      for (int c = 0; c < HD; c += 4) {
        float g[4];
        load4(gate + c, g);
        float v[4] = {acc[c] * inv * g[0], acc[c + 1] * inv * g[1], acc[c + 2] * inv * g[2], acc[c + 3] * inv * g[3]};
        if (DEC)
          store4(da.out + ro + c, v);
        else
          store4((bf16*)ea.out + ro + c, v);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int HD, int MODE>
cudaError_t launch_attn(const EncAttnArgs* ea, const DecAttnArgs* da, cudaStream_t s, int32_t* err) {
  constexpr bool DEC = MODE >= 1;
  const int swz = HD == 64 ? 128 : 64;
  CUtensorMap mq, mk, mv;
  const int n_tiles = DEC ? da->n_tiles : ea->n_tiles;
  const int n_heads = DEC ? da->n_heads : ea->n_heads;
  const int d = DEC ? da->d : ea->d;
  if (n_tiles == 0) return cudaSuccess;
  // the packed [T, d] arrays: T is not needed by the kernel; the maps cover every row the tiles name
  const long long rows = DEC ? da->key_rows : ea->rows;
  if (DEC) {
    if (!make_tmap_bf16(&mk, da->h, rows, d, d, HD, ROWS, swz)) return cudaErrorInvalidValue;
    mq = mk;
    mv = mk;
    if (MODE == 2 && !make_tmap_bf16(&mv, da->h_lo, rows, d, d, HD, ROWS, swz)) return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_bf16(&mq, ea->q, rows, d, d, HD, ROWS, swz) ||
        !make_tmap_bf16(&mk, ea->k, rows, d, d, HD, ROWS, swz) ||
        !make_tmap_bf16(&mv, ea->v, rows, d, d, HD, ROWS, swz))
      return cudaErrorInvalidValue;
  }
  // at least 120 KB so that one CTA (which takes all 512 TMEM columns) runs per SM
  constexpr int smem_need = SmemLayout<HD, MODE>::TOTAL + 1024;
  constexpr int smem = smem_need > 120 * 1024 ? smem_need : 120 * 1024;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  EncAttnArgs e0 = ea ? *ea : EncAttnArgs{};
  DecAttnArgs d0 = da ? *da : DecAttnArgs{};
  attn_tc_kernel<HD, MODE><<<n_tiles * n_heads, NTHREADS, smem, s>>>(mq, mk, mv, e0, d0, err);
  return cudaGetLastError();
}

}  // namespace

bool sm100_attn_supported(int head_dim) { return head_dim == 32 || head_dim == 64; }

cudaError_t launch_enc_attn_sm100(int hd, const EncAttnArgs& a, cudaStream_t s, int32_t* err) {
  return hd == 64 ? launch_attn<64, 0>(&a, nullptr, s, err) : launch_attn<32, 0>(&a, nullptr, s, err);
}

cudaError_t launch_dec_attn_sm100(int hd, const DecAttnArgs& a, cudaStream_t s, int32_t* err) {
  if (a.h_lo) return hd == 64 ? launch_attn<64, 2>(nullptr, &a, s, err) : launch_attn<32, 2>(nullptr, &a, s, err);
  return hd == 64 ? launch_attn<64, 1>(nullptr, &a, s, err) : launch_attn<32, 1>(nullptr, &a, s, err);
}

}  // namespace rest
