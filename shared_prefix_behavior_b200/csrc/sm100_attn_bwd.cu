// tcgen05 / TMEM / TMA backward of the causal attention core for sm_100a
// (bf16, head_dim 32 or 64): the gradients a training step needs when a
// user's samples are encoded once as their union history (ULT, ReST §3.5).
//
// One work item is one 128-key block of one user and head. Its K and V tiles
// stay in shared memory while the query blocks from the diagonal to the
// user's end stream through two Q / dO stages. Per query block, with the
// block's keys in the TMEM lanes:
//   S^T  = K Q^T,  dP^T = V dO^T                 (128 x 128, operands in shared memory)
//   P^T  = exp(S^T - lse) under the causal mask,  dS^T = P^T * (dP^T - delta),
//          written as bf16 into shared memory by the key-row warpgroup
//   dV  += P^T dO,  dK += dS^T Q                  (accumulated in TMEM over the item)
//   dQ   = dS K                                   (the dS^T tile read MN-major)
// and a query-row warpgroup adds dQ into the fp32 dq with vector reductions.
//   warp 0       TMA producer (K, V per item; Q, dO per block, two stages)
//   warp 1       TMEM owner and MMA issuer. Order per block g: dV(g) once P^T(g)
//                is written, S^T(g+1), then dK(g) and dQ(g) once dS^T(g) is
//                written, dP^T(g+1): the next block's products run while this
//                block's dS is computed.
//   warps 4..11  two warpgroups, a thread per key row and half of the block's
//                queries: P^T, dS^T, and the item's dV (first) or dK (second)
//   warps 12..15 a thread per query row of the block: dQ out of TMEM
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.h"
#include "sm100_common.cuh"

namespace rest {
namespace {

using namespace sm100;

constexpr int BR = 128;  // keys per item, queries per block
constexpr int NTHREADS = 512;
constexpr int NKEY = 256;  // threads of the two key-row warpgroups
constexpr int PBOX = BR * 128;  // one 64-column box of a [128 x 128] bf16 tile (128-byte swizzle)

template <int HD>
struct BwdCfg {
  static constexpr int ROW_BYTES = HD * 2;
  static constexpr int TILE = BR * ROW_BYTES;   // one [128 x head_dim] bf16 tile
  static constexpr int SWZ = HD == 64 ? 2 : 4;  // descriptor swizzle of the head tiles: 128B / 64B
  static constexpr int ATOM = 8 * ROW_BYTES;    // bytes of 8 swizzled rows
  // shared memory: K | V | Q[2] | dO[2] | P^T | dS^T; the last two are [128 x 128] bf16 tiles
  // kept as two 64-column boxes of 128 rows with 128-byte swizzle (queries 0..63, 64..127)
  static constexpr int K_OFF = 0, V_OFF = TILE, Q_OFF = 2 * TILE, G_OFF = 4 * TILE, P_OFF = 6 * TILE;
  static constexpr int DS_OFF = P_OFF + 2 * PBOX;
  static constexpr int TOTAL = DS_OFF + 2 * PBOX;
  // TMEM columns: S^T | dP^T | dV | dK | dQ
  static constexpr uint32_t S_COL = 0, DP_COL = 128, DV_COL = 256, DK_COL = 256 + HD, DQ_COL = 256 + 2 * HD;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

__device__ __forceinline__ void named_sync_keys() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// dst[0..3] += v (fp32 reduction in L2, no value returned)
__device__ __forceinline__ void red_add4(float* dst, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// One work item: keys kb*128 .. of user `user`, head h, against query blocks kb .. nqb-1.
struct BwdItem {
  int row0;  // packed row of the user's position 0
  int len;   // the user's length
  int kb;    // key block
  int n;     // query blocks (kb .. kb + n - 1)
  int h;
};

__device__ __forceinline__ BwdItem decode_bwd(const AttnBwdArgs& a, int item) {
  BwdItem w;
  const EncTile t = a.tiles[item / a.n_heads];
  w.h = item % a.n_heads;
  w.row0 = a.cu[t.user];
  w.len = a.cu[t.user + 1] - w.row0;
  w.kb = t.q0 / BR;
  w.n = (w.len + BR - 1) / BR - w.kb;
  return w;
}

// Persistent: CTA c walks its items sched[n_cta + 1 + k], k in [sched[c], sched[c+1]),
// in decreasing cost. Barrier phases follow from the running counts of items
// (kit) and query blocks (g) every role keeps.
template <int HD>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                       AttnBwdArgs a, int32_t* err) {
  using C = BwdCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // kv_full / kv_empty: the item's K, V loaded / no longer read; q_full[s] / q_empty[s]: stage s
  // loaded / read by every product of its block; s_full, dp_full: S^T(g), dP^T(g) in TMEM;
  // p_ready / p_free: P^T(g) written / read by dV(g); ds_ready / ds_free: dS^T(g) written / read
  // by dK(g) and dQ(g); dq_full / dq_empty: dQ(g) in TMEM / read out; acc_full / acc_empty: the
  // item's dK, dV complete / read out.
  __shared__ uint64_t kv_full, kv_empty, q_full[2], q_empty[2], s_full, dp_full, p_ready, p_free, ds_ready,
      ds_free, dq_full, dq_empty, acc_full, acc_empty, drain;
  __shared__ uint32_t tslot;
  __shared__ volatile int abort_flag;
  __shared__ float lse_s[2][BR], dlt_s[2][BR];  // log2-domain lse and delta of a block's queries

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int* items = a.sched + a.n_cta + 1;
  const int k_begin = a.sched[blockIdx.x], k_end = a.sched[blockIdx.x + 1];

  if (threadIdx.x == 0) {
    mbar_init(&kv_full, 1);
    mbar_init(&kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(&s_full, 1);
    mbar_init(&dp_full, 1);
    mbar_init(&p_ready, NKEY);
    mbar_init(&p_free, 1);
    mbar_init(&ds_ready, NKEY);
    mbar_init(&ds_free, 1);
    mbar_init(&dq_full, 1);
    mbar_init(&dq_empty, BR);
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, NKEY);
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  pdl_wait();  // the previous kernel of the stream has completed: its outputs may be read
  pdl_release();

  if (warp < 4) {
    // 4 x 32 x 64 (control) + 8 x 32 x 168 (key rows) + 4 x 32 x 112 (query rows) = 512 x 128
    asm volatile("setmaxnreg.dec.sync.aligned.u32 64;");
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int g = 0, kv_issued = 0, q_issued = 0;
      bool ok = true;
      for (int k = k_begin; k < k_end && ok; ++k) {
        const BwdItem w = decode_bwd(a, items[k]);
        if (kv_issued >= 1 && !mbar_wait(&kv_empty, (kv_issued - 1) & 1, err, &abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&kv_full, 2 * C::TILE);
        tma_load_2d(smem + C::K_OFF, &tmK, w.h * HD, w.row0 + w.kb * BR, &kv_full);
        tma_load_2d(smem + C::V_OFF, &tmV, w.h * HD, w.row0 + w.kb * BR, &kv_full);
        ++kv_issued;
        for (int i = 0; i < w.n; ++i, ++g) {
          const int st = g & 1, u = g >> 1;
          if (u >= 1 && !mbar_wait(&q_empty[st], (u - 1) & 1, err, &abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[st], 2 * C::TILE);
          const int row = w.row0 + (w.kb + i) * BR;
          tma_load_2d(smem + C::Q_OFF + st * C::TILE, &tmQ, w.h * HD, row, &q_full[st]);
          tma_load_2d(smem + C::G_OFF + st * C::TILE, &tmG, w.h * HD, row, &q_full[st]);
          q_issued = g + 1;
        }
      }
      if (!ok) {  // let the copies in flight land before the CTA exits
        volatile int no_abort = 0;
        if (kv_issued >= 1) mbar_wait(&kv_full, (kv_issued - 1) & 1, nullptr, &no_abort);
        for (int j = (q_issued > 2 ? q_issued - 2 : 0); j < q_issued; ++j)
          mbar_wait(&q_full[j & 1], (j >> 1) & 1, nullptr, &no_abort);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idS = idesc_bf16_ab(BR, 0, 0);  // S^T, dP^T: A, B K-major, N = 128 queries
      constexpr uint32_t idKV = idesc_bf16_ab(HD, 0, 1);  // dV, dK: A = P^T / dS^T K-major, B = dO / Q MN-major
      constexpr uint32_t idQ = idesc_bf16_ab(HD, 1, 1);   // dQ: A = dS (the dS^T tile) MN-major, B = K MN-major
      const uint32_t k_base = smem_u32(smem + C::K_OFF), v_base = smem_u32(smem + C::V_OFF);
      const uint32_t p_base = smem_u32(smem + C::P_OFF), ds_base = smem_u32(smem + C::DS_OFF);
      bool ok = true;
      // S^T(gg) = K Q(gg)^T and dP^T(gg) = V dO(gg)^T; the caller has waited for what they overwrite
      auto issue_s = [&](int gg) -> bool {
        const int st = gg & 1;
        if (!mbar_wait(&q_full[st], (gg >> 1) & 1, err, &abort_flag)) return false;
        tc_fence_after();
        const uint32_t q_base = smem_u32(smem + C::Q_OFF + st * C::TILE);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          mma_bf16(tmem + C::S_COL, smem_desc(k_base + kk * 32, 16, C::ATOM, C::SWZ),
                   smem_desc(q_base + kk * 32, 16, C::ATOM, C::SWZ), idS, kk != 0);
        mma_commit(&s_full);
        return true;
      };
      auto issue_dp = [&](int gg) {
        const uint32_t g_base = smem_u32(smem + C::G_OFF + (gg & 1) * C::TILE);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          mma_bf16(tmem + C::DP_COL, smem_desc(v_base + kk * 32, 16, C::ATOM, C::SWZ),
                   smem_desc(g_base + kk * 32, 16, C::ATOM, C::SWZ), idS, kk != 0);
        mma_commit(&dp_full);
      };
      int g = 0, kit = 0;
      for (int k = k_begin; k < k_end && ok; ++k, ++kit) {
        const BwdItem w = decode_bwd(a, items[k]);
        if (!mbar_wait(&kv_full, kit & 1, err, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (!issue_s(g)) { ok = false; break; }
        issue_dp(g);
        for (int i = 0; i < w.n && ok; ++i, ++g) {
          const int st = g & 1;
          const uint32_t q_base = smem_u32(smem + C::Q_OFF + st * C::TILE);
          const uint32_t g_base = smem_u32(smem + C::G_OFF + st * C::TILE);
          // dV += P^T(g) dO(g); the item's first product starts the accumulator over,
          // once the previous item's dK, dV have been read out
          if (!mbar_wait(&p_ready, g & 1, err, &abort_flag)) { ok = false; break; }
          if (i == 0 && kit >= 1 && !mbar_wait(&acc_empty, (kit - 1) & 1, err, &abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BR / 16; ++kk)
            mma_bf16(tmem + C::DV_COL, smem_desc(p_base + (kk >> 2) * PBOX + (kk & 3) * 32, 16, 1024, 2),
                     smem_desc(g_base + kk * 2 * C::ATOM, 64 * BR * 2, C::ATOM, C::SWZ), idKV, (i | kk) != 0);
          mma_commit(&p_free);
          // S^T(g) has been read (P^T(g) is written): the next block's scores
          if (i + 1 < w.n && !issue_s(g + 1)) { ok = false; break; }
          // dK += dS^T(g) Q(g) and dQ(g) = dS(g) K, once dQ(g-1) has been read out
          if (!mbar_wait(&ds_ready, g & 1, err, &abort_flag)) { ok = false; break; }
          if (g >= 1 && !mbar_wait(&dq_empty, (g - 1) & 1, err, &abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BR / 16; ++kk)
            mma_bf16(tmem + C::DK_COL, smem_desc(ds_base + (kk >> 2) * PBOX + (kk & 3) * 32, 16, 1024, 2),
                     smem_desc(q_base + kk * 2 * C::ATOM, 64 * BR * 2, C::ATOM, C::SWZ), idKV, (i | kk) != 0);
#pragma unroll
          for (int kk = 0; kk < BR / 16; ++kk)
            mma_bf16(tmem + C::DQ_COL, smem_desc(ds_base + kk * 2 * 1024, PBOX, 1024, 2),
                     smem_desc(k_base + kk * 2 * C::ATOM, 64 * BR * 2, C::ATOM, C::SWZ), idQ, kk != 0);
          mma_commit(&ds_free);
          mma_commit(&dq_full);
          mma_commit(&q_empty[st]);
          // dP^T(g) has been read (dS^T(g) is written)
          if (i + 1 < w.n) issue_dp(g + 1);
        }
        if (!ok) break;
        mma_commit(&acc_full);  // the item's dK and dV
        mma_commit(&kv_empty);
      }
      mma_commit(&drain);
      volatile int no_abort = 0;
      mbar_wait(&drain, 0, nullptr, &no_abort);
    }
  } else if (warp < 12) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 168;");
    // -------------------------------------------------------------- key rows: P^T, dS^T, dK, dV
    // two warpgroups on the same TMEM lanes: warpgroup hf takes query columns [64 hf, 64 hf + 64)
    // of every block (box hf of the P^T and dS^T tiles) and, at the item's end, dV (hf 0) or dK (hf 1)
    const int r = (warp & 3) * 32 + lane;  // the key row (TMEM lane)
    const int hf = (warp - 4) >> 2, c0 = 64 * hf;
    const int tid = threadIdx.x - 128;     // 0 .. 255
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    bool ok = true;
    int g = 0, kit = 0;
    // the lse (log2 domain) and delta of query qb * 128 + tid, loaded one block ahead (tid < 128)
    auto stats = [&](const BwdItem& w, int qb, float& l2, float& dl) {
      const int qp = qb * BR + tid;
      l2 = 0.f;
      dl = 0.f;
      if (tid < BR && qp < w.len) {
        const long long ri = (long long)(w.row0 + qp) * a.n_heads + w.h;
        l2 = a.lse[ri] * 1.4426950408889634f;
        dl = a.delta[ri];
      }
    };
    for (int k = k_begin; k < k_end && ok; ++k, ++kit) {
      const BwdItem w = decode_bwd(a, items[k]);
      const int kpos = w.kb * BR + r;  // this thread's key position in the history
      float l2_next, dl_next;
      stats(w, w.kb, l2_next, dl_next);
      for (int i = 0; i < w.n; ++i, ++g) {
        const int qb = w.kb + i, b = g & 1;
        if (tid < BR) {
          lse_s[b][tid] = l2_next;
          dlt_s[b][tid] = dl_next;
        }
        if (i + 1 < w.n) stats(w, qb + 1, l2_next, dl_next);
        named_sync_keys();
        if (!mbar_wait(&s_full, g & 1, err, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        // this half's query column c is visible when kpos <= qb*128 + c0 + c < len
        const int first = kpos - qb * BR - c0, lim = (kpos < w.len ? w.len - qb * BR : 0) - c0;
        const bool open = first <= 0 && lim >= 64;  // no masked column in this half
        float p[64];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float sv[32];
          tmem_ld32(tmem + lane_off + C::S_COL + c0 + 32 * c, sv);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(&lse_s[b][c0 + 32 * c + e]);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const int col = 32 * c + e + t;
              const float pv = exp2_approx(fmaf(sv[e + t], sl2, -lv[t]));
              p[col] = (open || (col >= first && col < lim)) ? pv : 0.f;
            }
          }
        }
        // P^T(g) into shared memory once dV(g-1) has read P^T(g-1)
        if (g >= 1 && !mbar_wait(&p_free, (g - 1) & 1, err, &abort_flag)) { ok = false; break; }
        uint8_t* pt = smem + C::P_OFF + hf * PBOX;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<uint4*>(pt + sw128_off(r, u)) =
              make_uint4(pack_bf16x2(p[8 * u], p[8 * u + 1]), pack_bf16x2(p[8 * u + 2], p[8 * u + 3]),
                         pack_bf16x2(p[8 * u + 4], p[8 * u + 5]), pack_bf16x2(p[8 * u + 6], p[8 * u + 7]));
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&p_ready);
        // dS^T(g) = P^T (dP^T - delta), once dK(g-1), dQ(g-1) have read dS^T(g-1)
        if (!mbar_wait(&dp_full, g & 1, err, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (g >= 1 && !mbar_wait(&ds_free, (g - 1) & 1, err, &abort_flag)) { ok = false; break; }
        uint8_t* dst = smem + C::DS_OFF + hf * PBOX;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float dp[32];
          tmem_ld32(tmem + lane_off + C::DP_COL + c0 + 32 * c, dp);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(&dlt_s[b][c0 + 32 * c + e]);
            dp[e] = p[32 * c + e] * (dp[e] - d4.x);
            dp[e + 1] = p[32 * c + e + 1] * (dp[e + 1] - d4.y);
            dp[e + 2] = p[32 * c + e + 2] * (dp[e + 2] - d4.z);
            dp[e + 3] = p[32 * c + e + 3] * (dp[e + 3] - d4.w);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(dst + sw128_off(r, 4 * c + u)) =
                make_uint4(pack_bf16x2(dp[8 * u], dp[8 * u + 1]), pack_bf16x2(dp[8 * u + 2], dp[8 * u + 3]),
                           pack_bf16x2(dp[8 * u + 4], dp[8 * u + 5]), pack_bf16x2(dp[8 * u + 6], dp[8 * u + 7]));
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&ds_ready);
      }
      if (!ok) break;
      // the item's dV (warpgroup 0) or dK (warpgroup 1) rows
      if (!mbar_wait(&acc_full, kit & 1, err, &abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t col = hf ? C::DK_COL : C::DV_COL;
      const float mul = hf ? sl2 * 0.69314718055994531f : 1.f;  // dK carries 1 / sqrt(head_dim)
      float* out = (hf ? a.dk : a.dv) + (long long)(w.row0 + kpos) * a.d + w.h * HD;
      float acc[HD];
#pragma unroll
      for (int cc = 0; cc < HD; cc += 32) {
        float t[32];
        tmem_ld32(tmem + lane_off + col + cc, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[cc + e] = t[e] * mul;
      }
      tc_fence_before();
      mbar_arrive(&acc_empty);  // the accumulators may be started over
      if (kpos < w.len) {
#pragma unroll
        for (int c = 0; c < HD; c += 4) store4(out + c, &acc[c]);
      }
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 112;");
    // -------------------------------------------------------------- query rows: dQ += dS K
    const int r = (warp & 3) * 32 + lane;  // the query row of the block (TMEM lane)
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float scale = a.scale_log2 * 0.69314718055994531f;  // 1 / sqrt(head_dim)
    bool ok = true;
    int g = 0;
    for (int k = k_begin; k < k_end && ok; ++k) {
      const BwdItem w = decode_bwd(a, items[k]);
      for (int i = 0; i < w.n; ++i, ++g) {
        const int qpos = (w.kb + i) * BR + r;
        if (!mbar_wait(&dq_full, g & 1, err, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        float v[HD];
#pragma unroll
        for (int cc = 0; cc < HD; cc += 32) {
          float t[32];
          tmem_ld32(tmem + lane_off + C::DQ_COL + cc, t);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[cc + e] = t[e] * scale;
        }
        tc_fence_before();
        mbar_arrive(&dq_empty);
        if (qpos < w.len) {
          float* dst = a.dq + (long long)(w.row0 + qpos) * a.d + w.h * HD;
#pragma unroll
          for (int c = 0; c < HD; c += 4) red_add4(dst + c, v[c], v[c + 1], v[c + 2], v[c + 3]);
        }
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

template <int HD>
cudaError_t launch_bwd(const AttnBwdArgs& a, cudaStream_t s, int32_t* err) {
  if (a.n_tiles == 0) return cudaSuccess;
  if (a.n_cta <= 0) return cudaErrorInvalidValue;
  const int swz = HD == 64 ? 128 : 64;
  CUtensorMap mq, mk, mv, mg;
  if (!make_tmap_bf16(&mq, a.q, a.rows, a.d, a.d, HD, BR, swz) ||
      !make_tmap_bf16(&mk, a.k, a.rows, a.d, a.d, HD, BR, swz) ||
      !make_tmap_bf16(&mv, a.v, a.rows, a.d, a.d, HD, BR, swz) ||
      !make_tmap_bf16(&mg, a.d_o, a.rows, a.d, a.d, HD, BR, swz))
    return cudaErrorInvalidValue;
  // at least 120 KB so that exactly one CTA (which takes all 512 TMEM columns) runs per SM
  constexpr int need = BwdCfg<HD>::TOTAL + 1024;
  constexpr int smem = need > 120 * 1024 ? need : 120 * 1024;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_k(attn_bwd_tc_kernel<HD>, a.n_cta, NTHREADS, smem, s, mq, mk, mv, mg, a, err);
}

}  // namespace

cudaError_t launch_attn_bwd_sm100(int hd, const AttnBwdArgs& a, cudaStream_t s, int32_t* err) {
  return hd == 64 ? launch_bwd<64>(a, s, err) : launch_bwd<32>(a, s, err);
}

}  // namespace rest
