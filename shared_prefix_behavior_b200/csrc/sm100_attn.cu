// tcgen05 / TMEM / TMA attention for sm_100a: the causal Dual-Gated
// Attention of the ReST encoder (§3.2.1 eqs. 3-4) and the shared-prefix,
// projection-free cross attention of the decoder (§3.3.1 eq. 7, §3.5).
//
// One CTA owns NT x 128 query rows of one head as NT 128-row tiles that share
// every staged key block (so each K/V (or H) block crosses to shared memory
// once per NT x 128 query rows), with one softmax warpgroup per tile. NT = 2
// with 128-key blocks at head_dim 64, NT = 3 with 64-key blocks at head_dim 32
// (see Geo):
//   warp 0       TMA producer. Encoder: Q tiles once, then K and V' per key
//                block. Decoder: the fp16 q tiles, then H per block; one H
//                tile is both the keys (K-major operand of S = q H^T) and the
//                values (N-major operand of O = P H).
//   warps 1..NT  MMA issuers of tiles 0..NT-1 (warp 1 also owns TMEM): per
//                block j, S_t(j) = Q_t K_j^T into the tile's TMEM S buffer as
//                soon as its softmax has read S_t(j-1), then
//                O_t += P_t(j-1) V_{j-1} into the tile's head_dim-column
//                accumulator once P_t(j-1) is written. A warp issues one
//                tcgen05.mma about every hundred cycles whatever its size
//                (measured), so each tile has its own issuing warp, running
//                whole with one elected lane.
//   warp 3       head_dim 32: first decodes the CTA's work items into a
//                shared-memory table (a lane per item), then issues tile 2.
//   warps 4..    softmax, four warps per tile (warps 4..7 tile 0, 8..11 tile 1,
//                12..15 tile 2): a thread owns a query row; it reads its row
//                of S from TMEM, masks, keeps the running max, exponentiates in
//                base 2, and writes P (bf16 pairs) back to the tile's P columns
//                of TMEM, from where the P V MMA takes its A operand; the
//                exponentials are computed before the wait for the previous
//                P V, which only their store needs. O stays in TMEM: when a
//                row's max grows by more than 2^8 the warp rescales its O rows
//                in TMEM (after the previous P V has completed); otherwise P is
//                taken relative to the old max (values up to 2^8, exact in fp32
//                accumulation). At head_dim 64 the two tiles' warps of a lane
//                quarter, which share a sub-partition's special-function unit,
//                take turns at the exponentials block by block. The encoder's
//                output rows go out through a per-warp staging area in shared
//                memory.
// The decoder multiplies in fp16 (kind::f16 with fp16 operands, fp32
// accumulation): H comes as an fp16 copy, the query as the fp16 rows the
// projection wrote (scaled by log2(e) / sqrt(head_dim) there, so S is in the
// base-2 domain), and P is written as fp16 pairs; o * g goes out in fp16.
// fp16's 11-bit significand rounds q, H and P 8 times finer than bf16; the
// producers of H and q report values beyond fp16's range (REST_ERR_RANGE).
//
// MODE 0: encoder; 1: decoder; 3: encoder over a range of key blocks
// (appending with split keys), writing partials.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.h"
#include "sm100_common.cuh"

namespace rest {
namespace {

using namespace sm100;

constexpr int ROWS = 128;  // query rows per tile
constexpr int HKB = 128;   // keys per block in the host's work items (their kb0, kb1)
constexpr int MAXNT = 3;   // most tiles per work item
constexpr int ITEM_CACHE = 64;  // work items per CTA decoded into shared memory up front
constexpr float RESCALE_LOG2 = 8.0f;  // rescale O when the row max grows by more than 2^8

// The shape of a CTA by head size. head_dim 64: two query tiles, 128-key blocks,
// 384 threads. head_dim 32: three query tiles and 64-key blocks (S, P and O of a
// tile then take 64 + 32 + 32 TMEM columns, 384 for the three), 512 threads, so
// that three softmax warps share each SM sub-partition's special-function unit
// where two did.
template <int HD>
struct Geo {
  static constexpr int NT = HD <= 32 ? 3 : 2;     // query tiles per work item
  static constexpr int KB = HD <= 32 ? 64 : 128;  // keys per block
  static constexpr int NTHREADS = 128 * (NT + 1);
  // registers per thread after setmaxnreg: warps 0-3, then the softmax warpgroups
  // (4 x 32 x REG_CTRL + NT x 128 x REG_SOFT stays within the 65,536 of the SM)
  static constexpr int REG_CTRL = HD <= 32 ? 56 : 72;
  static constexpr int REG_SOFT = HD <= 32 ? 152 : 216;
  static_assert(4 * 32 * REG_CTRL + NT * 128 * REG_SOFT <= 65536, "register split");
  static_assert(NT <= MAXNT && HKB % KB == 0, "tile shape");
};

template <int HD>
struct Cfg {
  static constexpr int ROW_BYTES = HD * 2;             // one bf16 row of a head slice
  static constexpr int TILE_BYTES = ROWS * ROW_BYTES;  // a query tile: 128 rows
  static constexpr int KV_TILE_BYTES = Geo<HD>::KB * ROW_BYTES;  // a key block
  static constexpr int SWZ = HD == 64 ? 2 : 4;         // descriptor code: 128B / 64B swizzle
  static constexpr int ATOM = 8 * ROW_BYTES;           // bytes of 8 swizzled rows
};
// TMEM columns: S_0 .. S_{NT-1} (KB each) | O_0 .. (HD each) | P_0 .. (KB bf16
// keys packed in KB / 2 columns each)
template <int HD>
__device__ __forceinline__ uint32_t s_col(int t) { return (uint32_t)(t * Geo<HD>::KB); }
template <int HD>
__device__ __forceinline__ uint32_t o_col(int t) { return (uint32_t)(Geo<HD>::NT * Geo<HD>::KB + t * HD); }
template <int HD>
__device__ __forceinline__ uint32_t p_col(int t) {
  return (uint32_t)(Geo<HD>::NT * (Geo<HD>::KB + HD) + t * (Geo<HD>::KB / 2));
}

// byte offset of 16-byte chunk u of row r in a swizzled [128 x HD] bf16 tile
template <int HD>
__device__ __forceinline__ uint32_t swz_off(int r, int u) {
  constexpr int CH = Cfg<HD>::ROW_BYTES / 16;  // 16B chunks per row: 8 (128B rows) or 4 (64B rows)
  return r * Cfg<HD>::ROW_BYTES + ((u ^ ((r >> (HD == 64 ? 0 : 1)) & (CH - 1))) * 16);
}

template <int HD, int MODE>
struct SmemLayout {
  // [Q_0 .. Q_{NT-1} | KV stages], 1024-aligned blocks
  static constexpr int STAGES = HD <= 32 ? 6 : 3;
  static constexpr int Q = 0;
  static constexpr int KV = Geo<HD>::NT * Cfg<HD>::TILE_BYTES;
  // a stage holds K and V' (encoder) or H (decoder)
  static constexpr int STAGE = (MODE == 1 ? 1 : 2) * Cfg<HD>::KV_TILE_BYTES;
  // per softmax warp, its 32 output rows in 2-byte values (rows padded by 16
  // bytes): the encoder's O (bf16) or the decoder's o * g (fp16)
  static constexpr bool DEC = MODE == 1;
  static constexpr int STG_ROW = HD * 2 + 16;
  static constexpr int STG = KV + STAGES * STAGE;
  static constexpr bool STAGED_OUT = MODE == 0 || (DEC && HD <= 32);
  // head_dim 32: every softmax thread's output-gate row (fp32; decoding fp16)
  // fetched ahead by cp.async, rows padded by 16 bytes
  static constexpr bool PREFETCH = HD <= 32 && MODE != 3;
  static constexpr int PF_ROW = HD * (DEC ? 2 : 4) + 16;
  static constexpr int PF = STG + (STAGED_OUT ? Geo<HD>::NT * 4 * 32 * STG_ROW : 0);
  static constexpr int TOTAL = PF + (PREFETCH ? Geo<HD>::NT * ROWS * PF_ROW : 0);
  static_assert(KV % 1024 == 0 && STAGE % 1024 == 0, "1024-aligned tiles");
};

// Asynchronous 16-byte copies global -> shared memory (no TMA): a thread
// fetches its own rows ahead of their use and waits for its own groups.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Packed fp32 pair arithmetic of sm_100 (one instruction for two lanes of work).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// 2^x for two values on the FMA and integer pipes instead of the special-function
// unit. x = n + f with n the nearest integer (adding 1.5 * 2^23 leaves n in the
// low bits of the sum) and f in [-1/2, 1/2]; 2^f from a degree-3 polynomial
// fitted here for least maximum relative error on that interval (Remez
// exchange: 7.5e-5, below the bf16 or fp16 rounding P gets), times 2^n built in
// the exponent field. x is first raised to -127, where 2^n's bits are those of
// +0: a masked score (minus infinity) gives an exact 0, as the special-function
// unit does, and so does anything below 2^-127.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.99992806f, c1 = 0.69326097f, c2 = 0.24261113f, c3 = 0.05517167f;
  x = make_float2(fmaxf(x.x, -127.0f), fmaxf(x.y, -127.0f));
  const float2 t = fadd2(x, make_float2(kRound, kRound));
  const float2 n = fadd2(t, make_float2(-kRound, -kRound));
  const float2 f = ffma2(n, make_float2(-1.0f, -1.0f), x);
  float2 p = ffma2(f, make_float2(c3, c3), make_float2(c2, c2));
  p = ffma2(p, f, make_float2(c1, c1));
  p = ffma2(p, f, make_float2(c0, c0));
  // t's bits are 0x4B400000 + n, which shifted by 23 leave n << 23 (mod 2^32):
  // 2^n's bits are (n + 127) << 23, zero for n = -127
  const float2 e2 = make_float2(__uint_as_float((__float_as_uint(t.x) << 23) + (127u << 23)),
                                __uint_as_float((__float_as_uint(t.y) << 23) + (127u << 23)));
  return make_float2(p.x * e2.x, p.y * e2.y);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int N>
__device__ __forceinline__ void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

// One work item: NT x 128 query rows (NT 128-row tiles) of one head.
template <int NT>
struct AttnItem {
  int q_row0;     // packed row of query row 0 of tile 0
  int key_row0;   // packed row of the item's first key
  int nrow[NT];   // valid query rows of each tile
  int nblk[NT];   // key blocks (of the kernel's KB keys) each tile reads
  int user_len;   // encoder: keys of the user's history (cached and new rows)
  int q_pos0;     // encoder: position of query row 0 within the user's history
  int nkeys;      // keys from key_row0 visible to the item (decoder: cutoff minus the split start)
  int key_off;    // encoder with split keys: position of key_row0 within the user's keys
  int split;      // split index of the partial result
  int h;          // head
};

// The host's items count keys in blocks of HKB (128); the kernel walks them in
// blocks of KB (64 at head_dim 32, 128 at 64).
template <int HD, bool DEC, bool SPLITK>
__device__ __forceinline__ AttnItem<Geo<HD>::NT> decode_item(const EncAttnArgs& ea, const DecAttnArgs& da, int item) {
  constexpr int NT = Geo<HD>::NT, KB = Geo<HD>::KB;
  AttnItem<NT> w;
  const int n_heads = DEC ? da.n_heads : ea.n_heads;
  const int tile = item / n_heads;
  w.h = item % n_heads;
  if (DEC) {
    const DecTile t = da.tiles[tile];
    w.q_row0 = t.row0;
    w.key_row0 = t.key0 + t.kb0 * HKB;  // this item's keys: host blocks kb0 .. kb1-1
    w.nkeys = t.nkeys - t.kb0 * HKB;
    w.user_len = 0;
    w.q_pos0 = 0;
    w.split = t.split;
    w.key_off = 0;
    // key blocks of the item's range (with KB = HKB, its host blocks)
    const int nk = min(t.nkeys, t.kb1 * HKB) - t.kb0 * HKB;
    const int nbk = KB == HKB ? t.kb1 - t.kb0 : nk > 0 ? (nk + KB - 1) / KB : 0;
    for (int i = 0; i < NT; ++i) {
      w.nrow[i] = max(0, min(ROWS, t.nrows - i * ROWS));
      w.nblk[i] = w.nrow[i] > 0 ? nbk : 0;
    }
  } else {
    const EncTile t = ea.tiles[tile];
    const int s = ea.cu[t.user];
    const int n = ea.cu[t.user + 1] - s;  // the user's query rows
    // appending: the query rows follow `cached` positions held in the cache arrays
    const int off = ea.app ? ea.app[t.user].cached : 0;
    w.key_row0 = ea.app ? ea.app[t.user].key0 : s;
    w.user_len = off + n;
    w.q_pos0 = off + t.q0;
    w.q_row0 = s + t.q0;
    w.nkeys = 0;
    w.split = SPLITK ? t.split : 0;
    // split keys: host blocks [kb0, kb1) of the user's keys only
    const int kb0 = SPLITK ? t.kb0 * (HKB / KB) : 0;
    w.key_off = kb0 * KB;
    w.key_row0 += w.key_off;
    for (int i = 0; i < NT; ++i) {
      const int r0 = t.q0 + i * ROWS;
      w.nrow[i] = max(0, min(ROWS, n - r0));
      const int nb = (min(w.user_len, off + r0 + ROWS) + KB - 1) / KB;
      w.nblk[i] = w.nrow[i] > 0 ? (SPLITK ? max(0, min(nb, t.kb1 * (HKB / KB)) - kb0) : nb) : 0;
    }
  }
  return w;
}

// key blocks of the item's longest tile (the blocks the producer loads)
template <int NT>
__device__ __forceinline__ int max_blocks(const AttnItem<NT>& w) {
  int m = 0;
#pragma unroll
  for (int i = 0; i < NT; ++i) m = max(m, w.nblk[i]);
  return m;
}

// Persistent: one CTA per SM walks its own list of work items (a
// longest-processing-time schedule built on the host: sched[n_cta + 1 + k] for
// k in [sched[c], sched[c + 1])). TMEM, barriers and the pipelines persist
// across items; every role keeps, per tile, the count of key blocks (cb) and of
// items with work (qn) processed so far, from which all barrier parities follow.
template <int HD, int MODE>
__global__ void __launch_bounds__(Geo<HD>::NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, EncAttnArgs ea, DecAttnArgs da, int32_t* err) {
  constexpr bool DEC = MODE == 1, ESPLIT = MODE == 3;
  constexpr int NT = Geo<HD>::NT, KB = Geo<HD>::KB;
  // head_dim 64: the two tiles' softmax warps of a lane quarter take turns at the
  // exponentials block by block (see the softmax); at 32 they do not.
  constexpr bool TURNS = HD >= 64;
  using C = Cfg<HD>;
  using L = SmemLayout<HD, MODE>;
  constexpr int STAGES = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // q_full: Q_t staged; q_empty: the item's last S_t has read Q_t; s_full / p_full /
  // p_free: S_t(j) ready / P_t(j) written / O_t += P_t(j) V done; o_empty: the
  // item's O_t has been read out of TMEM.
  __shared__ uint64_t q_full[NT], q_empty[NT], kv_full[STAGES], kv_empty[STAGES], s_full[NT], s_free[NT], p_full[NT],
      p_free[NT], o_empty[NT], drain;
  // xe[t][q][n & 1]: tile t's softmax warp of TMEM lane quarter q has issued the
  // exponentials of its n-th key block (two barriers per pair so that a warp one
  // or two blocks ahead never completes the phase its partner still waits for)
  __shared__ uint64_t xe[NT][4][2];
  __shared__ AttnItem<NT> s_items[HD <= 32 ? ITEM_CACHE : 1];
  __shared__ uint32_t tslot;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_heads = DEC ? da.n_heads : ea.n_heads;
  const int d = DEC ? da.d : ea.d;
  const int* sched = DEC ? da.sched : ea.sched;
  const int* items = sched + (DEC ? da.n_cta : ea.n_cta) + 1;

  if (threadIdx.x == 0) {
    for (int t = 0; t < NT; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&q_empty[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&s_free[t], 128);
      mbar_init(&p_full[t], 128);
      mbar_init(&p_free[t], 1);
      mbar_init(&o_empty[t], 128);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], NT);  // one arrival per MMA-issuing warp
    }
    mbar_init(&drain, NT);
    for (int t = 0; t < NT; ++t)
      for (int q = 0; q < 4; ++q) {
        mbar_init(&xe[t][q][0], 1);
        mbar_init(&xe[t][q][1], 1);
      }
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
  // head_dim 32: the CTA's first ITEM_CACHE work items, decoded once by warp 3
  // (a lane per item, so their chains of dependent loads overlap) for every
  // role to read from shared memory; later items are decoded where they are
  // used. Items there are short (a few key blocks), and each role's decode, three
  // dependent global loads, was about 5 % of an item. head_dim 64 decodes in
  // place: its items are long, and the table cost registers in its softmax.
  constexpr bool CACHE_ITEMS = HD <= 32;
  const int k_first = sched[blockIdx.x];
  if (CACHE_ITEMS && warp == 3) {
    const int n = min(sched[blockIdx.x + 1] - k_first, ITEM_CACHE);
    for (int i = lane; i < n; i += 32) s_items[i] = decode_item<HD, DEC, ESPLIT>(ea, da, items[k_first + i]);
  }
  __syncthreads();
  auto item_at = [&](int k) -> AttnItem<NT> {
    return CACHE_ITEMS && k - k_first < ITEM_CACHE ? s_items[k - k_first]
                                                   : decode_item<HD, DEC, ESPLIT>(ea, da, items[k]);
  };

  if (warp < 4) {
    setmaxnreg_dec<Geo<HD>::REG_CTRL>();
    // Warp 0, lane 0 loads (the other lanes of warp 0 have no role and wait at
    // the end); warps 1 .. NT issue the MMAs of tiles 0 .. NT-1 (with two tiles,
    // warp 3 has no role after the item table). The issuing warps run whole:
    // their elect.sync needs every lane.
    if (warp == 0 && lane == 0) {
      // -------------------------------------------------------- TMA producer
      int g = 0, issued = 0, qn[NT] = {};
      bool ok = true;
      for (int k = sched[blockIdx.x]; k < sched[blockIdx.x + 1] && ok; ++k) {
        const AttnItem<NT> w = item_at(k);
        // the query tiles (decoding: fp16, scaled to the base-2 domain by the projection)
        for (int t = 0; t < NT && ok; ++t) {
          if (w.nblk[t] == 0) continue;
          if (qn[t] >= 1 && !mbar_wait(&q_empty[t], (qn[t] - 1) & 1, err, &abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[t], C::TILE_BYTES);
          tma_load_2d(smem + L::Q + t * C::TILE_BYTES, &tmQ, w.h * HD, w.q_row0 + t * ROWS, &q_full[t]);
          ++qn[t];
        }
        const int nblk_all = max_blocks<NT>(w);
        for (int j = 0; j < nblk_all && ok; ++j, ++g) {
          const int st = g % STAGES;
          if (!mbar_wait(&kv_empty[st], ((g / STAGES) & 1) ^ 1, err, &abort_flag)) { ok = false; break; }
          uint8_t* base = smem + L::KV + st * L::STAGE;
          mbar_arrive_expect_tx(&kv_full[st], L::STAGE);
          tma_load_2d(base, &tmK, w.h * HD, w.key_row0 + j * KB, &kv_full[st]);
          if (MODE != 1) tma_load_2d(base + C::KV_TILE_BYTES, &tmV, w.h * HD, w.key_row0 + j * KB, &kv_full[st]);
          issued = g + 1;
        }
      }
      if (!ok) {  // let the copies in flight land before the CTA exits
        volatile int no_abort = 0;
        for (int t = 0; t < NT; ++t)
            if (qn[t] >= 1) mbar_wait(&q_full[t], (qn[t] - 1) & 1, nullptr, &no_abort);
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          mbar_wait(&kv_full[i % STAGES], (i / STAGES) & 1, nullptr, &no_abort);
      }
    } else if (warp >= 1 && warp <= NT) {
      // -------------------------------------------------------- MMA issuers
      // Warp 1 + t for tile t: S_t(j) = Q_t K_j^T into the tile's S
      // buffer as soon as its softmax has loaded S_t(j-1) (s_free), then
      // O_t += P_t(j-1) V_{j-1} once P_t(j-1) is written (p_full). A warp issues one
      // tcgen05.mma about every hundred cycles whatever its size (measured), so
      // each tile has its own issuing warp, which also keeps one tile's softmax
      // from waiting on the other's. The whole warp runs the loop and one elected
      // lane issues. A block's K/V stage is released when every issuer has
      // committed it (kv_empty counts NT arrivals); a tile with fewer blocks in
      // the item still waits for each remaining block to land before releasing
      // it, so neither issuer can arrive for a later use of a stage before the
      // earlier use has completed.
      const int t = warp - 1;
      // the decoder's operands are fp16, the encoder's bf16
      constexpr uint32_t idS = DEC ? idesc_f16(KB, 0) : idesc_bf16(KB, 0);  // N = KB keys, B (keys) K-major
      constexpr uint32_t idO = DEC ? idesc_f16(HD, 1) : idesc_bf16(HD, 1);  // N = head_dim, B (values) N-major
      constexpr uint32_t V_STEP = (2 * C::ATOM) >> 4;  // 16 keys of V: two 8-row atoms
      const uint32_t tS = tmem + s_col<HD>(t), tO = tmem + o_col<HD>(t), tP = tmem + p_col<HD>(t);
      // Descriptors step along K: 16 elements are 32 bytes, 2 in the 16-byte address field.
      const uint64_t qd = smem_desc(smem_u32(smem + L::Q + t * C::TILE_BYTES), 16, C::ATOM, C::SWZ);
      int g = 0, cb = 0, qn = 0;
      bool ok = true;
      for (int k = sched[blockIdx.x]; k < sched[blockIdx.x + 1] && ok; ++k) {
        const AttnItem<NT> w = item_at(k);
        const int nblk_all = max_blocks<NT>(w);
        const int nb = w.nblk[t];
        if (nb > 0) ok = mbar_wait(&q_full[t], qn & 1, err, &abort_flag);
        tc_fence_after();
        for (int j = 0; ok && j <= nb; ++j) {
          if (j < nb) {  // S(j), overwriting the tile's S buffer
            const int st = (g + j) % STAGES;
            if (!mbar_wait(&kv_full[st], ((g + j) / STAGES) & 1, err, &abort_flag)) { ok = false; break; }
            if (cb + j >= 1 && !mbar_wait(&s_free[t], (cb + j - 1) & 1, err, &abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint64_t kd = smem_desc(smem_u32(smem + L::KV + st * L::STAGE), 16, C::ATOM, C::SWZ);
  #pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) mma_bf16_e(tS, qd + 2 * kk, kd + 2 * kk, idS, kk != 0);
            if (j == nb - 1) mma_commit_e(&q_empty[t]);  // the item's last read of Q_t
            mma_commit_e(&s_full[t]);
          }
          if (j >= 1) {  // O += P(j-1) V_{j-1}
            const int i = j - 1, st = (g + i) % STAGES;
            if (!mbar_wait(&p_full[t], (cb + i) & 1, err, &abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (i == 0 && qn >= 1) {  // the previous item's O_t has been read out
              if (!mbar_wait(&o_empty[t], (qn - 1) & 1, err, &abort_flag)) { ok = false; break; }
              tc_fence_after();
            }
            const uint64_t vd = smem_desc(smem_u32(smem + L::KV + st * L::STAGE + (DEC ? 0 : C::KV_TILE_BYTES)),
                                          64 * KB * 2, C::ATOM, C::SWZ);
            // A = P_t from TMEM, 8 columns per K step of 16
  #pragma unroll
            for (int kk = 0; kk < KB / 16; ++kk)
              mma_bf16_ts_e(tO, tP + kk * 8, vd + V_STEP * kk, idO, (i | kk) != 0);
            mma_commit_e(&p_free[t]);
            mma_commit_e(&kv_empty[st]);  // this tile is done with block i (its S and its P V)
          }
        }
        // the item's blocks this tile has no rows for: released once each has landed
        for (int j = nb; ok && j < nblk_all; ++j) {
          const int st = (g + j) % STAGES;
          if (!mbar_wait(&kv_full[st], ((g + j) / STAGES) & 1, err, &abort_flag)) { ok = false; break; }
          if (lane == 0) mbar_arrive(&kv_empty[st]);
        }
        g += nblk_all;
        if (nb > 0) {
          cb += nb;
          ++qn;
        }
      }
      mma_commit_e(&drain);
      volatile int no_abort = 0;
      mbar_wait(&drain, 0, nullptr, &no_abort);
    }
  } else {
    setmaxnreg_inc<Geo<HD>::REG_SOFT>();
    // -------------------------------------------------------------- softmax
    const int t = (warp - 4) >> 2;               // tile of this warpgroup
    const int q4 = warp & 3;                     // TMEM lane quarter
    const int r = q4 * 32 + lane;                // row within the tile
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    // the decoder's scores arrive in the base-2 domain (its query is staged pre-scaled)
    const float sl2 = DEC ? 1.0f : ea.scale_log2;
    const uint32_t tS = tmem + lane_off + s_col<HD>(t);
    const uint32_t tO = tmem + lane_off + o_col<HD>(t);
    const uint32_t tP = tmem + lane_off + p_col<HD>(t);
    const bool split = DEC ? da.n_split > 1 : ESPLIT;
    float* const part_o = DEC ? da.part_o : ea.part_o;       // split: partial results
    float* const part_ml = DEC ? da.part_ml : ea.part_ml;
    const long long part_rows = DEC ? da.nk_rows : ea.rows;
    int cb = 0, qn = 0, cbo = 0;  // cbo: the other tile's key blocks in earlier items
    // head_dim 32: this thread's output-gate row, fetched ahead (see SmemLayout::PREFETCH)
    const int tid = threadIdx.x - 128;
    uint8_t* const pf_gate = smem + L::PF + tid * L::PF_ROW;
    constexpr int GATE_ES = DEC ? 2 : 4;  // the gate's element size: fp16 decoding, fp32 encoding
    bool ok = true;
    for (int k = sched[blockIdx.x]; k < sched[blockIdx.x + 1] && ok; ++k) {
      const AttnItem<NT> w = item_at(k);
      const int nb = w.nblk[t];
      const bool valid = r < w.nrow[t];
      const long long row_g = (long long)(w.q_row0 + t * ROWS + r);
      const int h = w.h;
      if (nb == 0) {
        if (split && valid) {  // an empty key range: a partial that carries no weight
          float* po = part_o + ((long long)w.split * part_rows + row_g) * d + h * HD;
          const float z4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < HD; c += 4) store4(po + c, z4);
          float* pml = part_ml + (((long long)w.split * part_rows + row_g) * n_heads + h) * 2;
          pml[0] = -INFINITY;
          pml[1] = 0.f;
        }
        if constexpr (TURNS) cbo += w.nblk[1 - t];
        continue;
      }
      const long long ro = row_g * d + h * HD;
      const bool has_gate = DEC || ea.gate != nullptr;  // the encoder's gate may be left out (training core)
      const uint8_t* const gate_src = DEC ? static_cast<const uint8_t*>(da.g16) : reinterpret_cast<const uint8_t*>(ea.gate);
      if (L::PREFETCH) {  // this item's output gate row, in flight through the item's key blocks
        if (valid && !split && has_gate) {
#pragma unroll
          for (int u = 0; u < HD * GATE_ES / 16; ++u) cp_async16(pf_gate + 16 * u, gate_src + ro * GATE_ES + 16 * u);
        }
        cp_async_commit();
      }
      // visible keys: index < row_lim - KB j (the causal bound and the user end / cutoff)
      const int row_lim = DEC ? w.nkeys : min(w.q_pos0 + t * ROWS + r + 1, w.user_len) - (ESPLIT ? w.key_off : 0);
      float m_ref = -INFINITY;  // reference max (scaled, log2 domain) of P and O
      float l_run = 0.f;        // sum of exponentials relative to m_ref
      for (int j = 0; j < nb; ++j) {
        const int gj = cb + j;
        if (!mbar_wait(&s_full[t], gj & 1, err, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        float s[KB];
        {
          uint32_t raw[KB / 32][32];
#pragma unroll
          for (int c = 0; c < KB / 32; ++c) tmem_ld32_async(tS + 32 * c, raw[c]);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&s_free[t]);  // S_t may now be overwritten by the next block's scores
#pragma unroll
          for (int c = 0; c < KB / 32; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(raw[c][i]);
        }
        const int lim = row_lim - j * KB;
        if (lim < KB) {
#pragma unroll
          for (int c = 0; c < KB; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        // row max of the raw scores: 8 chains of three-input maxima
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmaxf(s[i], s[8 + i]);
#pragma unroll
        for (int c = 16; c < KB; c += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = fmax3(mx[i], s[c + i], s[c + 8 + i]);
        const float m_blk = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                  fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
        // P_t replaces the previous block's P once that block's O += P V has
        // completed (p_free). The wait comes after the exponentials, which need
        // only the reference max, unless the O row must be rescaled first.
        bool pv_done = gj == 0;
        if (j == 0) {
          m_ref = m_blk;
        } else if (__any_sync(0xffffffffu, m_blk > m_ref + RESCALE_LOG2)) {
          // Some row's max grew by more than 2^8: the warp rescales its O rows and
          // sums to their new maxima (a factor of 1 for the rows whose max did not
          // grow). Warp-wide, since the TMEM loads and stores are warp-collective.
          if (!mbar_wait(&p_free[t], (gj - 1) & 1, err, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          pv_done = true;
          const float m_new = fmaxf(m_ref, m_blk);
          const float f = exp2_approx(m_ref - m_new);
#pragma unroll
          for (int c0 = 0; c0 < HD; c0 += 32) {
            float o[32];
            tmem_ld32(tO + c0, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= f;
            tmem_st32(tO + c0, o);
          }
          l_run *= f;
          m_ref = m_new;
        }
        // The two tiles' warps of a lane quarter share an SM sub-partition and its
        // special-function unit: they take turns at the exponentials, block by block
        // (tile 0's block j, tile 1's block j, tile 0's block j + 1, ...), so each
        // one's loads, maxima and waits overlap the other's exponentials.
        if constexpr (TURNS) {
          const int oj = t == 0 ? j - 1 : j;  // the other tile's block that goes first
          if (oj >= 0 && oj < w.nblk[1 - t]) {
            const int n = cbo + oj;
            if (!mbar_wait(&xe[1 - t][q4][n & 1], (n >> 1) & 1, err, &abort_flag)) { ok = false; break; }
          }
        }
        float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 scale2 = make_float2(sl2, sl2), neg_m2 = make_float2(-m_ref, -m_ref);
        // P as bf16 (decoder: fp16) pairs, keys 2c, 2c+1 in column c, stored into the
        // tile's P columns of TMEM once the previous P V has completed
        uint32_t pk[KB / 2];
        // The pairs c with bit c % 8 of POLY_PAIRS set (two in eight) are
        // exponentiated on the FMA pipe, so the softmax warps queue less on the
        // special-function unit (measured, decoder attention: head_dim 32 on the
        // ragged workload, none 1.45 ms, one pair in eight 1.39, two 1.36; head_dim
        // 64 at 16k, none 0.155, one 0.152, two 0.151, three 0.161, four 0.166).
        // The choice follows the key's column alone, so a score gets the same P
        // whatever rows share its warp (appending equals re-encoding bit for bit).
        constexpr unsigned POLY_PAIRS = 0x88u;
#pragma unroll
        for (int c = 0; c < KB / 2; ++c) {
          const int e = 2 * c;
          const float2 x = ffma2(make_float2(s[e], s[e + 1]), scale2, neg_m2);
          const float2 p = (POLY_PAIRS >> (c & 7)) & 1u ? exp2_fma2(x)
                                                         : make_float2(exp2_approx(x.x), exp2_approx(x.y));
          sum2[c & 1] = fadd2(sum2[c & 1], p);
          pk[c] = DEC ? pack_f16x2(p.x, p.y) : pack_bf16x2(p.x, p.y);
        }
        if constexpr (TURNS) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&xe[t][q4][(cb + j) & 1]);
        }
        if (!pv_done) {
          if (!mbar_wait(&p_free[t], (gj - 1) & 1, err, &abort_flag)) { ok = false; break; }
          tc_fence_after();
        }
#pragma unroll
        for (int u = 0; u < KB / 64; ++u)
          tmem_st32_async(tP + 32 * u, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32 * u]));
        l_run += (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // the output gate of this row: fetched ahead into shared memory (head_dim 32),
      // or loaded here (64: the row would not fit the softmax warps' registers next to O)
      constexpr bool GATE_ROW = L::PREFETCH;
      float gate_row[GATE_ROW ? HD : 4];
      if (GATE_ROW && valid && !split && has_gate) {
        cp_async_wait<0>();
        if (DEC) {
#pragma unroll
          for (int c = 0; c < HD; c += 8) load8_f16(reinterpret_cast<const __half*>(pf_gate) + c, &gate_row[c]);
        } else {
#pragma unroll
          for (int c = 0; c < HD; c += 4) load4(reinterpret_cast<const float*>(pf_gate) + c, &gate_row[c]);
        }
      }
      if (!mbar_wait(&p_free[t], (cb + nb - 1) & 1, err, &abort_flag)) { ok = false; break; }  // the last P V
      tc_fence_after();
      // every lane takes part in the (warp-collective) TMEM loads
      float o[HD];
#pragma unroll
      for (int c0 = 0; c0 < HD; c0 += 32) {
        float v32[32];
        tmem_ld32(tO + c0, v32);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[c0 + e] = v32[e];
      }
      tc_fence_before();
      mbar_arrive(&o_empty[t]);  // O_t may now be overwritten by the next item
      if (L::STAGED_OUT && !split && (DEC || ea.out_lo == nullptr)) {
        // The output rows through shared memory: each lane writes its row's 2-byte
        // values (the encoder's O * gate in bf16, the decoder's o * g in fp16) into the
        // warp's staging rows, then the warp stores them 16 bytes a lane, HD / 8 lanes
        // to a row, so that a store instruction writes whole sectors of a few rows
        // instead of 8 bytes of each of 32 rows.
        const float inv = valid ? 1.0f / l_run : 0.f;
        if (!DEC && valid && ea.lse) ea.lse[row_g * n_heads + h] = (m_ref + log2f(l_run)) * 0.69314718055994531f;
        uint8_t* stg = smem + L::STG + (warp - 4) * 32 * L::STG_ROW;
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 8) {
          float gh[8];
          if (!has_gate || !valid) {
#pragma unroll
            for (int i = 0; i < 8; ++i) gh[i] = 1.f;
          } else if (GATE_ROW) {
#pragma unroll
            for (int i = 0; i < 8; ++i) gh[i] = gate_row[(c0 + i) % (GATE_ROW ? HD : 4)];
          } else if (DEC) {
            load8_f16(static_cast<const __half*>(da.g16) + ro + c0, gh);
          } else {
            load4(ea.gate + ro + c0, gh);
            load4(ea.gate + ro + c0 + 4, gh + 4);
          }
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float v0 = o[c0 + 2 * i] * inv * gh[2 * i], v1 = o[c0 + 2 * i + 1] * inv * gh[2 * i + 1];
            pk[i] = DEC ? pack_f16x2(v0, v1) : pack_bf16x2(v0, v1);
          }
          *reinterpret_cast<uint4*>(stg + lane * L::STG_ROW + c0 * 2) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        __syncwarp();
        constexpr int CPR = HD / 8;  // 16-byte chunks of a row
        uint8_t* const dst = static_cast<uint8_t*>(DEC ? da.out : ea.out);
#pragma unroll
        for (int rr = 0; rr < 32; rr += 32 / CPR) {
          const int r = rr + lane / CPR, ch = lane % CPR;
          const int tr = q4 * 32 + r;  // row within the tile
          if (tr < w.nrow[t]) {
            const uint4 val = *reinterpret_cast<const uint4*>(stg + r * L::STG_ROW + ch * 16);
            *reinterpret_cast<uint4*>(dst + ((long long)(w.q_row0 + t * ROWS + tr) * d + h * HD + ch * 8) * 2) = val;
          }
        }
        __syncwarp();  // the staging rows are free for the next item
      } else if (valid && split) {  // partial result of this key range, combined later
        float* po = part_o + ((long long)w.split * part_rows + row_g) * d + h * HD;
#pragma unroll
        for (int c = 0; c < HD; c += 4) store4(po + c, &o[c]);
        float* pml = part_ml + (((long long)w.split * part_rows + row_g) * n_heads + h) * 2;
        pml[0] = m_ref;
        pml[1] = l_run;
      } else if (valid) {
        const float inv = 1.0f / l_run;
        // log sum_j exp(score) for a backward pass: m_ref is in the scaled log2 domain
        if (!DEC && ea.lse) ea.lse[row_g * n_heads + h] = (m_ref + log2f(l_run)) * 0.69314718055994531f;
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 32) {  // 32 columns at a time, their gate loads in flight together
          float gh[32];
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            if (!has_gate) {
#pragma unroll
              for (int i = 0; i < 4; ++i) gh[c + i] = 1.f;
            } else if (GATE_ROW) {
#pragma unroll
              for (int i = 0; i < 4; ++i) gh[c + i] = gate_row[(c0 + c + i) % (GATE_ROW ? HD : 4)];
            } else if (DEC) {
              load4_f16(static_cast<const __half*>(da.g16) + ro + c0 + c, &gh[c]);
            } else {
              load4(ea.gate + ro + c0 + c, &gh[c]);
            }
          }
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const int cc = c0 + c;
            float v[4] = {o[cc] * inv * gh[c], o[cc + 1] * inv * gh[c + 1], o[cc + 2] * inv * gh[c + 2],
                          o[cc + 3] * inv * gh[c + 3]};
            if (DEC) {  // o * g in fp16 for the output projection's fp16 product
              *reinterpret_cast<uint2*>(static_cast<__half*>(da.out) + ro + cc) =
                  make_uint2(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]));
            } else {
              store4((bf16*)ea.out + ro + cc, v);
              if (ea.out_lo) {  // the low part, for a backward pass that needs O beyond bf16
                float lo[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) lo[i] = v[i] - __bfloat162float(__float2bfloat16_rn(v[i]));
                store4((bf16*)ea.out_lo + ro + cc, lo);
              }
            }
          }
        }
      }
      cb += nb;
      if constexpr (TURNS) cbo += w.nblk[1 - t];
      ++qn;
    }
    if (L::PREFETCH) cp_async_wait<0>();  // no copy into shared memory outlives the loop
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
  constexpr bool DEC = MODE == 1;
  constexpr int KB = Geo<HD>::KB;
  const int swz = HD == 64 ? 128 : 64;
  CUtensorMap mq, mk, mv;
  const int n_tiles = DEC ? da->n_tiles : ea->n_tiles;
  const int d = DEC ? da->d : ea->d;
  if (n_tiles == 0) return cudaSuccess;
  const long long rows = DEC ? da->key_rows : ea->rows;
  if (DEC) {  // fp16 H and queries, moved as 2-byte elements like bf16
    if (!make_tmap_bf16(&mk, da->h, rows, d, d, HD, KB, swz) ||
        !make_tmap_bf16(&mq, da->q16, da->nk_rows, d, d, HD, ROWS, swz))
      return cudaErrorInvalidValue;
    mv = mk;
  } else {
    const long long key_rows = ea->app ? ea->key_rows : rows;
    if (!make_tmap_bf16(&mq, ea->q, rows, d, d, HD, ROWS, swz) ||
        !make_tmap_bf16(&mk, ea->k, key_rows, d, d, HD, KB, swz) ||
        !make_tmap_bf16(&mv, ea->v, key_rows, d, d, HD, KB, swz))
      return cudaErrorInvalidValue;
  }
  // at least 120 KB so that exactly one CTA (which takes all 512 TMEM columns) runs per SM
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
  const int n_cta = DEC ? da->n_cta : ea->n_cta;
  if (n_cta <= 0) return cudaErrorInvalidValue;
  if (cudaError_t e_ = launch_k(attn_tc_kernel<HD, MODE>, n_cta, Geo<HD>::NTHREADS, smem, s, mq, mk, mv, e0, d0, err))
    return e_;
  return cudaGetLastError();
}

}  // namespace

bool sm100_attn_supported(int head_dim) { return head_dim == 32 || head_dim == 64; }
int sm100_attn_tile_rows(int head_dim) { return (head_dim <= 32 ? Geo<32>::NT : Geo<64>::NT) * ROWS; }

cudaError_t launch_enc_attn_sm100(int hd, const EncAttnArgs& a, cudaStream_t s, int32_t* err) {
  if (a.n_split > 1)  // appending with split keys: partial results for launch_enc_combine
    return hd == 64 ? launch_attn<64, 3>(&a, nullptr, s, err) : launch_attn<32, 3>(&a, nullptr, s, err);
  return hd == 64 ? launch_attn<64, 0>(&a, nullptr, s, err) : launch_attn<32, 0>(&a, nullptr, s, err);
}

cudaError_t launch_dec_attn_sm100(int hd, const DecAttnArgs& a, cudaStream_t s, int32_t* err) {
  return hd == 64 ? launch_attn<64, 1>(nullptr, &a, s, err) : launch_attn<32, 1>(nullptr, &a, s, err);
}

}  // namespace rest
