// C-ABI entry points of the ReST ranking forward: argument validation,
// workspace layout, work lists, and the launch sequence of the encoder
// (ReST §3.2) and the shared-prefix cross decoder (§3.3, §3.5).
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <queue>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "rest.h"
#include "sm100.h"

namespace rest {

static thread_local long long g_launches = 0;

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
static inline size_t dt_size(rest_dtype dt) { return dt == REST_BF16 ? 2 : 4; }

// ---------------------------------------------------------------- validation

static rest_status check_heads(rest_dtype dt, const rest_heads* hs) {
  if (dt != REST_F32 && dt != REST_BF16) return REST_ERR_INVALID_ARG;
  if (!hs || !hs->tau) return REST_ERR_INVALID_ARG;
  if (hs->n_heads < 1 || hs->n_heads > 32 || hs->head_dim < 2 || (hs->head_dim & 1)) return REST_ERR_INVALID_ARG;
  if (hs->d != hs->n_heads * hs->head_dim) return REST_ERR_INVALID_ARG;
  if (!(hs->rope_base > 0.0) || !isfinite(hs->rope_base)) return REST_ERR_INVALID_ARG;
  for (int h = 0; h < hs->n_heads; ++h)
    if (hs->tau[h] < 0) return REST_ERR_INVALID_ARG;
  if (hs->head_dim != 16 && hs->head_dim != 32 && hs->head_dim != 64) return REST_ERR_UNSUPPORTED;
  if (hs->d % 32 != 0 || hs->d > 1024) return REST_ERR_UNSUPPORTED;
  return REST_OK;
}

static rest_status check_batch(const rest_batch* b, long long* total) {
  if (!b || b->n_users < 0) return REST_ERR_INVALID_ARG;
  *total = 0;
  if (b->n_users == 0) return REST_OK;
  if (!b->cu_seqlens || b->cu_seqlens[0] != 0) return REST_ERR_INVALID_ARG;
  for (int u = 0; u < b->n_users; ++u)
    if (b->cu_seqlens[u + 1] < b->cu_seqlens[u]) return REST_ERR_INVALID_ARG;
  *total = b->cu_seqlens[b->n_users];
  return REST_OK;
}

static rest_status check_layers(const rest_enc_layer* layers, int n_layers, int l_switch, int* max_dff) {
  *max_dff = 0;
  if (n_layers < 0 || (n_layers > 0 && !layers)) return REST_ERR_INVALID_ARG;
  if (l_switch < 0 || l_switch > n_layers) return REST_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    const rest_enc_layer& L = layers[l];
    if (!L.w_qkvgg || !L.w_o || !L.ln_attn_g || !L.ln_attn_b) return REST_ERR_INVALID_ARG;
    if (!aligned16(L.w_qkvgg) || !aligned16(L.w_o) || !aligned16(L.ln_attn_g) || !aligned16(L.ln_attn_b))
      return REST_ERR_INVALID_ARG;
    if (!isfinite(L.alpha_attn) || !isfinite(L.alpha_ffn)) return REST_ERR_INVALID_ARG;
    if (L.gates != GATES_VO && L.gates != GATES_O && L.gates != GATES_QKVO) return REST_ERR_INVALID_ARG;
    if (L.w_ffn13) {
      if (!L.w_ffn2 || !L.ln_ffn_g || !L.ln_ffn_b || L.d_ff <= 0 || L.d_ff % 64 != 0 || L.d_ff > 16384)
        return REST_ERR_INVALID_ARG;
      if (!aligned16(L.w_ffn13) || !aligned16(L.w_ffn2) || !aligned16(L.ln_ffn_g) || !aligned16(L.ln_ffn_b))
        return REST_ERR_INVALID_ARG;
      *max_dff = std::max(*max_dff, L.d_ff);
    }
  }
  return REST_OK;
}

static rest_status check_requests(const rest_requests* r, const rest_batch* b, long long* n_cands) {
  if (!r || r->n_req < 0) return REST_ERR_INVALID_ARG;
  *n_cands = 0;
  if (r->n_req == 0) return REST_OK;
  if (!r->req_user || !r->req_cutoff || !r->cu_cands || r->cu_cands[0] != 0) return REST_ERR_INVALID_ARG;
  for (int i = 0; i < r->n_req; ++i) {
    int u = r->req_user[i];
    if (u < 0 || u >= b->n_users) return REST_ERR_INVALID_ARG;
    int L = b->cu_seqlens[u + 1] - b->cu_seqlens[u];
    if (r->req_cutoff[i] < 1 || r->req_cutoff[i] > L) return REST_ERR_INVALID_ARG;
    if (r->cu_cands[i + 1] < r->cu_cands[i]) return REST_ERR_INVALID_ARG;
  }
  *n_cands = r->cu_cands[r->n_req];
  return REST_OK;
}

static rest_status check_dec(const rest_dec_params* dec) {
  if (!dec || dec->K < 1 || dec->K > 8) return REST_ERR_INVALID_ARG;
  if (!dec->w_q || !dec->w_go || !dec->w_o) return REST_ERR_INVALID_ARG;
  if (!aligned16(dec->w_q) || !aligned16(dec->w_go) || !aligned16(dec->w_o)) return REST_ERR_INVALID_ARG;
  return REST_OK;
}

// ---------------------------------------------------------------- work lists

// Query rows per work item: 128 for the CUDA-core attention, the
// tensor-core kernel's own size otherwise (three 128-row tiles at head_dim 32,
// two at 64).
static int attn_tile_rows(rest_dtype dt, int head_dim) {
  return (dt == REST_BF16 && sm100_attn_supported(head_dim)) ? sm100_attn_tile_rows(head_dim) : 128;
}

static void build_enc_tiles(const rest_batch* b, int rows, std::vector<EncTile>& t) {
  t.clear();
  for (int u = 0; u < b->n_users; ++u) {
    int L = b->cu_seqlens[u + 1] - b->cu_seqlens[u];
    for (int q0 = 0; q0 < L; q0 += rows) t.push_back(EncTile{u, q0});
  }
  // longest causal rows first, so the tail of the grid holds the short tiles
  std::stable_sort(t.begin(), t.end(), [](const EncTile& a, const EncTile& c) { return a.q0 > c.q0; });
}

constexpr int KEY_BLOCK = 128;   // keys per block of the attention kernels
// In rank_request the CUDA-core decoder (fp32 arithmetic) reads H_lo (H =
// H_hi + H_lo) for requests with fewer keys than this: H's bf16 rounding reaches
// y through per-key perturbations that the attention average shrinks about as
// 1/sqrt(keys), while a cutoff of 1 key passes H's rounding straight into y.
// (The tensor-core decoder reads H in fp16, 8 times finer than bf16, for every
// request.)
constexpr int HLO_MAX_CUTOFF = 1024;
constexpr int TARGET_CTAS = 296;  // two waves of the B200's 148 SMs

// Decoder work items. With n_split > 1 every (request, row chunk) is split
// into n_split ranges of whole key blocks (some may be empty) whose partial
// results a combine kernel merges.
static void build_dec_tiles(const rest_batch* b, const rest_requests* r, int K, int rows, int n_split,
                            std::vector<DecTile>& t) {
  t.clear();
  if (!r) return;
  for (int i = 0; i < r->n_req; ++i) {
    long long rows0 = (long long)r->cu_cands[i] * K, rows1 = (long long)r->cu_cands[i + 1] * K;
    int key0 = b->cu_seqlens[r->req_user[i]];
    int c = r->req_cutoff[i];
    int nb = (c + KEY_BLOCK - 1) / KEY_BLOCK;
    for (long long p = rows0; p < rows1; p += rows)
      for (int sp = 0; sp < n_split; ++sp)
        t.push_back(DecTile{(int)p, (int)std::min<long long>(rows, rows1 - p), key0, c,
                            (int)((long long)nb * sp / n_split), (int)((long long)nb * (sp + 1) / n_split), sp,
                            c < HLO_MAX_CUTOFF ? 1 : 0});
  }
  // the tiles that read H_lo first (they run as a launch of their own), each group longest first
  std::stable_sort(t.begin(), t.end(), [](const DecTile& a, const DecTile& c) {
    if (a.pad != c.pad) return a.pad > c.pad;
    return a.kb1 - a.kb0 > c.kb1 - c.kb0;
  });
}

// Longest-processing-time assignment of attention work items to the
// tensor-core kernel's persistent CTAs: items by decreasing cost (key blocks
// times active query tiles), each to the least-loaded CTA. Returned as
// [n_cta + 1 offsets | item ids], each CTA's items in decreasing cost.
constexpr int SCHED_CTAS = 148;  // one persistent CTA per B200 SM

static std::vector<int> lpt_schedule(const std::vector<long long>& cost) {
  const int n = (int)cost.size();
  const int n_cta = std::min(n, SCHED_CTAS);
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  std::vector<std::vector<int>> lists(n_cta);
  std::vector<std::pair<long long, int>> heap;  // (load, cta), min-heap
  for (int c = 0; c < n_cta; ++c) heap.push_back({0, c});
  auto cmp = [](const std::pair<long long, int>& a, const std::pair<long long, int>& b) { return a > b; };
  std::make_heap(heap.begin(), heap.end(), cmp);
  for (int i : order) {
    std::pop_heap(heap.begin(), heap.end(), cmp);
    auto& top = heap.back();
    lists[top.second].push_back(i);
    top.first += std::max(1LL, cost[i]);
    std::push_heap(heap.begin(), heap.end(), cmp);
  }
  std::vector<int> out(n_cta + 1 + n);
  out[0] = 0;
  int k = n_cta + 1;
  for (int c = 0; c < n_cta; ++c) {
    for (int i : lists[c]) out[k++] = i;
    out[c + 1] = out[c] + (int)lists[c].size();
  }
  return out;
}

// Longest finishing time of the longest-first assignment of `cost` to n_cta CTAs.
static long long lpt_makespan(std::vector<long long> cost, int n_cta) {
  std::sort(cost.begin(), cost.end(), std::greater<long long>());
  std::priority_queue<long long, std::vector<long long>, std::greater<long long>> load;
  for (int c = 0; c < n_cta; ++c) load.push(0);
  long long most = 0;
  for (long long c : cost) {
    const long long l = load.top() + c;
    load.pop();
    load.push(l);
    most = std::max(most, l);
  }
  return most;
}

// Key splits of the decoder when its work items alone would leave SMs idle: the
// count (1..8, at least about 4 key blocks per split) whose longest-first schedule
// finishes first, counting an item as its key blocks times its query tiles plus a
// fixed cost in the same unit (q staging, pipeline fill, the output). The fixed
// cost, 7 blocks, fits the kernel's measured times at two split counts on two
// workloads (8 x 4096 and 2 x 16384 keys); a split count wins only when it is at
// least 5% shorter than every smaller one, since each split also writes a
// partial output that the combine reads back.
constexpr long long ITEM_COST_BLOCKS = 7;
static int choose_dec_split(const rest_batch* b, const rest_requests* r, int K, int rows, int n_heads) {
  std::vector<DecTile> t;
  build_dec_tiles(b, r, K, rows, 1, t);
  if (t.empty()) return 1;
  const long long base = (long long)t.size() * n_heads;
  if (base >= TARGET_CTAS) return 1;
  long long blocks = 0;
  for (const DecTile& x : t) blocks += x.kb1 - x.kb0;
  const long long most = std::min(8LL, std::max(1LL, blocks / (long long)t.size() / 4));
  int best = 1;
  long long best_t = -1;
  for (int ns = 1; ns <= most; ++ns) {
    build_dec_tiles(b, r, K, rows, ns, t);
    std::vector<long long> cost;
    for (const DecTile& x : t) {
      const long long c = (long long)(x.kb1 - x.kb0) * ((x.nrows + 127) / 128) + ITEM_COST_BLOCKS;
      for (int h = 0; h < n_heads; ++h) cost.push_back(c);
    }
    const long long m = lpt_makespan(cost, SCHED_CTAS);
    if (best_t < 0 || m * 20 < best_t * 19) {
      best = ns;
      best_t = m;
    }
  }
  return best;
}

// Key blocks an encoder item reads, summed over its 128-row query tiles (each
// reads every key up to its last row; with split keys only blocks [kb0, kb1)).
// app (may be empty): the cached positions before each user's rows.
static long long enc_item_cost(const rest_batch* b, const std::vector<UserAppend>& app, const EncTile& t, int rows) {
  const int n = b->cu_seqlens[t.user + 1] - b->cu_seqlens[t.user];
  const int off = app.empty() ? 0 : app[t.user].cached;
  long long c = 0;
  for (int r0 = t.q0; r0 < std::min(n, t.q0 + rows); r0 += 128) {
    int nb = (std::min(off + n, off + r0 + 128) + 127) / 128;
    if (t.kb1 > 0) nb = std::max(0, std::min(nb, t.kb1) - t.kb0);
    c += nb;
  }
  return c;
}

static std::vector<int> enc_schedule(const rest_batch* b, const std::vector<EncTile>& tiles, int n_heads, int rows,
                                     const std::vector<UserAppend>& app) {
  std::vector<long long> cost;
  for (const EncTile& t : tiles) {
    const long long c = enc_item_cost(b, app, t, rows);
    for (int h = 0; h < n_heads; ++h) cost.push_back(c);
  }
  return lpt_schedule(cost);
}

constexpr int MAX_ENC_SPLIT = 8;  // also bounds the workspace an append query reserves
// Appending on the tensor-core path: when the items alone would leave SMs idle
// (a few users' new rows against long cached prefixes), every tile's key blocks
// are split over n_split items whose partial results a combine kernel merges.
// The count is chosen as the decoder's is (longest-first makespan with the same
// per-item cost; a larger count must win by 5 %), among the counts where every
// split has at least two blocks and begins at or before the tile's first query
// position, so that each query row sees at least one key in every split.
static void split_enc_tiles(const rest_batch* b, const std::vector<UserAppend>& app, int rows, int n_heads,
                            std::vector<EncTile>& tiles, int* n_split) {
  *n_split = 1;
  if (app.empty() || tiles.empty() || (long long)tiles.size() * n_heads >= TARGET_CTAS) return;
  auto blocks_all = [&](const EncTile& t) {  // key blocks of the item's last query row
    const int n = b->cu_seqlens[t.user + 1] - b->cu_seqlens[t.user], off = app[t.user].cached;
    return (std::min(off + n, off + t.q0 + rows) + 127) / 128;
  };
  auto split_of = [&](int ns) {
    std::vector<EncTile> out;
    for (const EncTile& t : tiles) {
      const int nb = blocks_all(t);
      for (int sp = 0; sp < ns; ++sp)
        out.push_back(EncTile{t.user, t.q0, (int)((long long)nb * sp / ns), (int)((long long)nb * (sp + 1) / ns), sp});
    }
    return out;
  };
  auto makespan = [&](const std::vector<EncTile>& ts) {
    std::vector<long long> cost;
    for (const EncTile& t : ts) {
      const long long c = enc_item_cost(b, app, t, rows) + ITEM_COST_BLOCKS;
      for (int h = 0; h < n_heads; ++h) cost.push_back(c);
    }
    return lpt_makespan(cost, SCHED_CTAS);
  };
  int best = 1;
  long long best_t = makespan(tiles);
  for (int ns = 2; ns <= MAX_ENC_SPLIT; ++ns) {
    bool ok = true;
    for (const EncTile& t : tiles) {
      const int nb = blocks_all(t), first = app[t.user].cached + t.q0;
      if (nb / ns < 2 || (long long)nb * (ns - 1) / ns * 128 > first) ok = false;
    }
    if (!ok) continue;
    const long long m = makespan(split_of(ns));
    if (m * 20 < best_t * 19) {
      best = ns;
      best_t = m;
    }
  }
  if (best > 1) {
    tiles = split_of(best);
    *n_split = best;
  }
}

static std::vector<int> dec_schedule(const std::vector<DecTile>& tiles, int n_heads) {
  std::vector<long long> cost;
  for (const DecTile& t : tiles) {
    const long long c = (long long)(t.kb1 - t.kb0) * ((t.nrows + 127) / 128);
    for (int h = 0; h < n_heads; ++h) cost.push_back(c);
  }
  return lpt_schedule(cost);
}

// ---------------------------------------------------------------- workspace

struct Layout {
  size_t cu, enc_tiles, dec_tiles, enc_sched, dec_sched, app, bwd_tiles, bwd_sched, meta_end;
  size_t cos_t, sin_t, xres, y, q, k, v, g, o, hid;
  size_t dq, dg, dout, hx, wo16, part_o, part_ml, delta;
  size_t total;
  int n_enc_tiles, n_dec_tiles, n_bwd_tiles;
};

static Layout make_layout(rest_dtype dt, const rest_heads* hs, const rest_batch* b, long long T, bool enc,
                          int max_dff, long long NK, int n_enc_tiles, int n_dec_tiles, bool hx, int n_split,
                          size_t n_enc_sched, size_t n_dec_sched, bool append,
                          int n_bwd_tiles = 0, size_t n_bwd_sched = 0, int n_split_enc = 1) {
  Layout L;
  const size_t A = 256, e = dt_size(dt);
  const size_t d = (size_t)hs->d;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, A); return o; };
  L.n_enc_tiles = n_enc_tiles;
  L.n_dec_tiles = n_dec_tiles;
  L.cu = take(sizeof(int32_t) * (size_t)(b->n_users + 1));
  L.enc_tiles = take(sizeof(EncTile) * (size_t)n_enc_tiles);
  L.dec_tiles = take(sizeof(DecTile) * (size_t)n_dec_tiles);
  L.enc_sched = take(sizeof(int) * n_enc_sched);
  L.dec_sched = take(sizeof(int) * n_dec_sched);
  L.app = take(append ? sizeof(UserAppend) * (size_t)b->n_users : 0);
  L.n_bwd_tiles = n_bwd_tiles;
  L.bwd_tiles = take(sizeof(EncTile) * (size_t)n_bwd_tiles);
  L.bwd_sched = take(sizeof(int) * n_bwd_sched);
  L.meta_end = off;
  L.cos_t = take(enc ? 4 * (size_t)T * d / 2 : 0);
  L.sin_t = take(enc ? 4 * (size_t)T * d / 2 : 0);
  L.xres = take(enc ? 4 * (size_t)T * d : 0);
  L.y = take(enc ? e * (size_t)T * d : 0);
  L.q = take(enc ? e * (size_t)T * d : 0);
  L.k = take(enc ? e * (size_t)T * d : 0);
  L.v = take(enc ? e * (size_t)T * d : 0);
  L.g = take(enc ? 4 * (size_t)T * d : 0);
  L.o = take(enc ? e * (size_t)T * d : 0);
  L.hid = take(enc ? e * (size_t)T * (size_t)max_dff : 0);
  L.dq = take(4 * (size_t)NK * d);
  L.dg = take(4 * (size_t)NK * d);
  L.dout = take(4 * (size_t)NK * d);
  // H_lo for the CUDA-core decoder, or the fp16 H of the tensor-core decoder and
  // its fp16 copy of W_o
  L.hx = take(hx ? 2 * (size_t)T * d : 0);
  L.wo16 = take(hx ? 2 * d * d : 0);
  // split partial results: the decoder's [n_split, NK] or the appending encoder's [n_split_enc, T] rows
  const size_t part_rows = std::max(n_split > 1 ? (size_t)n_split * NK : 0,
                                    n_split_enc > 1 ? (size_t)n_split_enc * T : 0);
  L.part_o = take(4 * part_rows * d);
  L.part_ml = take(8 * part_rows * hs->n_heads);
  L.delta = take(n_bwd_tiles > 0 ? 4 * (size_t)T * hs->n_heads : 0);
  L.total = off;
  return L;
}

struct Plan {
  rest_dtype dt;
  const rest_heads* hs;
  const rest_batch* b;
  long long T, n_cands, NK;
  int max_dff, K;
  std::vector<EncTile> enc_tiles;
  std::vector<DecTile> dec_tiles;
  std::vector<int> enc_sched, dec_sched;  // tensor-core attention: per-CTA item lists
  std::vector<UserAppend> app;  // appending to a cache: each user's cached prefix
  std::vector<EncTile> bwd_tiles;  // attention core backward: 128-row tiles of every user
  std::vector<int> bwd_sched;      // tensor-core backward: per-CTA lists of (key tile, head) items
  int n_dec_hlo;  // decoder tiles that read H_lo (CUDA-core decoder in rank_request, bf16)
  Layout L;
  int32_t* err;
  bool hsplit;    // the CUDA-core decoder reads H as H_hi + H_lo (the workspace's hx)
  bool h16;       // the tensor-core decoder: it reads H in fp16 (the workspace's hx)
  int n_split;      // decoder key splits (tensor-core path)
  int n_split_enc;  // encoder key splits when appending (tensor-core path)
};

// The cache of an append: region bounds, cached lengths and their fit, the
// per-layer arrays. Fills `app` (one entry per user).
static rest_status check_cache(const rest_kv_cache* c, const rest_batch* b, int n_layers,
                               std::vector<UserAppend>& app) {
  app.clear();
  if (!c || c->rows < 0 || c->rows >= (1LL << 31)) return REST_ERR_INVALID_ARG;
  if (n_layers > 0 && (!c->k || !c->v)) return REST_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (!c->k[l] || !c->v[l] || !aligned16(c->k[l]) || !aligned16(c->v[l])) return REST_ERR_INVALID_ARG;
  if (c->h && !aligned16(c->h)) return REST_ERR_INVALID_ARG;
  if (b->n_users == 0) return REST_OK;
  if (!c->cu_cap || !c->len || c->cu_cap[0] != 0) return REST_ERR_INVALID_ARG;
  for (int u = 0; u < b->n_users; ++u) {
    const long long cap = (long long)c->cu_cap[u + 1] - c->cu_cap[u];
    const long long n = (long long)b->cu_seqlens[u + 1] - b->cu_seqlens[u];
    if (cap < 0 || c->len[u] < 0 || c->len[u] + n > cap) return REST_ERR_INVALID_ARG;
    UserAppend a{0, 0, c->len[u], c->cu_cap[u]};
    if (c->len[u] > 0) {
      if (!c->t_first || !c->t_last || c->t_last[u] < c->t_first[u]) return REST_ERR_INVALID_ARG;
      a.t_origin = c->t_first[u];
      a.t_prev = c->t_last[u];
    }
    app.push_back(a);
  }
  if (c->cu_cap[b->n_users] > c->rows) return REST_ERR_INVALID_ARG;
  return REST_OK;
}

static rest_status make_plan(Plan& p, rest_dtype dt, const rest_heads* hs, const rest_batch* b,
                             const rest_enc_layer* layers, int n_layers, int l_switch, const rest_requests* reqs,
                             int K, bool encoder_runs, const rest_kv_cache* cache = nullptr, bool append = false,
                             bool core = false) {
  rest_status st = check_heads(dt, hs);
  if (st != REST_OK) return st;
  if ((st = check_batch(b, &p.T)) != REST_OK) return st;
  p.app.clear();
  if (cache && (st = check_cache(cache, b, n_layers, p.app)) != REST_OK) return st;
  if ((st = check_layers(layers, n_layers, l_switch, &p.max_dff)) != REST_OK) return st;
  p.n_cands = 0;
  if (reqs) {
    if ((st = check_requests(reqs, b, &p.n_cands)) != REST_OK) return st;
    if (K < 1 || K > 8) return REST_ERR_INVALID_ARG;
  }
  p.dt = dt; p.hs = hs; p.b = b; p.K = K; p.err = nullptr; p.hsplit = false; p.h16 = false; p.n_split = 1;
  p.n_dec_hlo = 0;
  p.NK = p.n_cands * (reqs ? K : 0);
  if (p.T * (long long)hs->d >= (1LL << 40) || p.NK >= (1LL << 31)) return REST_ERR_UNSUPPORTED;
  const int tile_rows = attn_tile_rows(dt, hs->head_dim);
  if (encoder_runs) build_enc_tiles(b, tile_rows, p.enc_tiles);
  p.n_split_enc = 1;
  if (encoder_runs && append && tile_rows != 128) {
    if (cache) {
      split_enc_tiles(b, p.app, tile_rows, hs->n_heads, p.enc_tiles, &p.n_split_enc);
    } else if ((long long)p.enc_tiles.size() * hs->n_heads < TARGET_CTAS) {
      // the workspace query (no cache yet): room for the most splits a call can take
      std::vector<EncTile> most;
      for (const EncTile& t : p.enc_tiles)
        for (int sp = 0; sp < MAX_ENC_SPLIT; ++sp) most.push_back(EncTile{t.user, t.q0, 0, 1, sp});
      p.enc_tiles.swap(most);
      p.n_split_enc = MAX_ENC_SPLIT;
    }
  }
  // split the decoder's keys when its work items alone would leave SMs idle
  p.n_split = 1;
  if (reqs && tile_rows != 128) p.n_split = choose_dec_split(b, reqs, K, tile_rows, hs->n_heads);
  build_dec_tiles(b, reqs, K, tile_rows, p.n_split, p.dec_tiles);
  // The tensor-core decoder multiplies in fp16: it reads an fp16 copy of H that
  // the encoder's last launch writes beside H (rank_request) or that is converted
  // from the caller's bf16 H (cross_decode). The CUDA-core decoder after an
  // encoder in bf16 reads H as hi + lo for short prefixes.
  p.h16 = reqs != nullptr && tile_rows != 128 && p.NK > 0;
  p.n_dec_hlo = 0;
  if (!p.h16 && encoder_runs && reqs != nullptr && dt == REST_BF16)
    for (const DecTile& t : p.dec_tiles) p.n_dec_hlo += t.pad;
  p.hsplit = p.n_dec_hlo > 0;
  for (DecTile& t : p.dec_tiles) t.pad = 0;
  if (tile_rows != 128) {  // the tensor-core attention runs: schedule its persistent CTAs
    if (!p.enc_tiles.empty()) p.enc_sched = enc_schedule(b, p.enc_tiles, hs->n_heads, tile_rows, p.app);
    if (!p.dec_tiles.empty()) p.dec_sched = dec_schedule(p.dec_tiles, hs->n_heads);
  }
  // the attention core alone (training): no encoder buffers; the backward's 128-row tiles
  p.bwd_tiles.clear();
  p.bwd_sched.clear();
  if (core) {
    std::vector<long long> cost;  // tensor-core backward: a key tile meets the query blocks from its diagonal on
    for (int u = 0; u < b->n_users; ++u) {
      const int L = b->cu_seqlens[u + 1] - b->cu_seqlens[u];
      for (int r0 = 0; r0 < L; r0 += 128) {
        p.bwd_tiles.push_back(EncTile{u, r0});
        for (int h = 0; h < hs->n_heads; ++h) cost.push_back((L + 127) / 128 - r0 / 128);
      }
    }
    if (tile_rows != 128 && !cost.empty()) p.bwd_sched = lpt_schedule(cost);
  }
  p.L = make_layout(dt, hs, b, p.T, encoder_runs && !core, p.max_dff, p.NK, (int)p.enc_tiles.size(),
                    (int)p.dec_tiles.size(), p.hsplit || p.h16, p.n_split, p.enc_sched.size(), p.dec_sched.size(),
                    append, (int)p.bwd_tiles.size(), p.bwd_sched.size(), p.n_split_enc);
  return REST_OK;
}

static rest_status check_device() {
  static int checked[64] = {0};  // 0 unknown, 1 ok, 2 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return REST_ERR_NO_DEVICE; }
  if (dev < 0 || dev >= 64) return REST_ERR_NO_DEVICE;
  if (checked[dev] == 0) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      cudaGetLastError();
      return REST_ERR_NO_DEVICE;
    }
    checked[dev] = (major == 10) ? 1 : 2;
  }
  return checked[dev] == 1 ? REST_OK : REST_ERR_NO_DEVICE;
}

// ---------------------------------------------------------------- instrumentation
// When profiling is on, every launch is bracketed by a pair of CUDA events on
// its own stream and tagged with its algorithmic FLOPs and bytes.
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
  double flops, bytes;
};
static thread_local bool g_prof = false;
bool pdl_enabled() { return !g_prof; }
static thread_local std::vector<ProfRec>* g_recs = nullptr;
static thread_local std::vector<cudaEvent_t>* g_event_pool = nullptr;

static cudaEvent_t prof_event() {
  if (!g_event_pool) g_event_pool = new std::vector<cudaEvent_t>();
  if (!g_event_pool->empty()) {
    cudaEvent_t e = g_event_pool->back();
    g_event_pool->pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct LaunchScope {
  ProfRec rec;
  cudaStream_t s;
  bool on;
  LaunchScope(cudaStream_t s_, const char* name, double flops, double bytes) : s(s_), on(g_prof) {
    ++g_launches;
    if (on) {
      rec = ProfRec{name, prof_event(), prof_event(), flops, bytes};
      cudaEventRecord(rec.a, s);
    }
  }
  void done() {
    if (on) {
      cudaEventRecord(rec.b, s);
      if (!g_recs) g_recs = new std::vector<ProfRec>();
      g_recs->push_back(rec);
    }
  }
};

#define REST_KLAUNCH(stream, name, flops, bytes, call)        \
  do {                                                        \
    LaunchScope sc_((stream), (name), (flops), (bytes));      \
    cudaError_t e_ = (call);                                  \
    sc_.done();                                               \
    if (e_ != cudaSuccess) return REST_ERR_CUDA;              \
  } while (0)

template <typename P> static inline P* at(void* ws, size_t off) { return reinterpret_cast<P*>((char*)ws + off); }

static rest_status upload_meta(const Plan& p, void* ws, cudaStream_t s) {
  std::vector<char> host(p.L.meta_end, 0);
  memcpy(host.data() + p.L.cu, p.b->cu_seqlens ? p.b->cu_seqlens : (const int32_t*)"\0\0\0\0",
         sizeof(int32_t) * (size_t)(p.b->n_users + 1));
  if (!p.enc_tiles.empty())
    memcpy(host.data() + p.L.enc_tiles, p.enc_tiles.data(), sizeof(EncTile) * p.enc_tiles.size());
  if (!p.dec_tiles.empty())
    memcpy(host.data() + p.L.dec_tiles, p.dec_tiles.data(), sizeof(DecTile) * p.dec_tiles.size());
  if (!p.enc_sched.empty())
    memcpy(host.data() + p.L.enc_sched, p.enc_sched.data(), sizeof(int) * p.enc_sched.size());
  if (!p.dec_sched.empty())
    memcpy(host.data() + p.L.dec_sched, p.dec_sched.data(), sizeof(int) * p.dec_sched.size());
  if (!p.app.empty()) memcpy(host.data() + p.L.app, p.app.data(), sizeof(UserAppend) * p.app.size());
  if (!p.bwd_tiles.empty())
    memcpy(host.data() + p.L.bwd_tiles, p.bwd_tiles.data(), sizeof(EncTile) * p.bwd_tiles.size());
  if (!p.bwd_sched.empty())
    memcpy(host.data() + p.L.bwd_sched, p.bwd_sched.data(), sizeof(int) * p.bwd_sched.size());
  if (cudaMemcpyAsync(ws, host.data(), host.size(), cudaMemcpyHostToDevice, s) != cudaSuccess) return REST_ERR_CUDA;
  // the status word reports this call only
  if (p.err && cudaMemsetAsync(p.err, 0, sizeof(int32_t), s) != cudaSuccess) return REST_ERR_CUDA;
  return REST_OK;
}

static TableParams table_params(const rest_heads* hs) {
  TableParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.n_heads = hs->n_heads;
  tp.half = hs->head_dim / 2;
  for (int h = 0; h < hs->n_heads; ++h) tp.tau[h] = hs->tau[h];
  const long double two_pi = 2.0L * 3.141592653589793238462643383279502884L;
  for (int j = 0; j < tp.half; ++j) {
    tp.theta[j] = pow(hs->rope_base, -2.0 * j / hs->head_dim);
    for (int k = 0; k < 3; ++k) {
      const long double t = (long double)tp.theta[j] * ldexpl(1.0L, 16 * k) / two_pi;
      tp.turn[k][j] = (double)(t - floorl(t));
    }
  }
  return tp;
}

static GemmArgs gemm(const void* A, long long lda, const void* B, long long ldb, long long M, int N, int K, int epi,
                     void* out0, long long ldo) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.A = A; a.lda = lda; a.B = B; a.ldb = ldb; a.M = (int)M; a.N = N; a.K = K; a.epi = epi;
  a.out0 = out0; a.ldo = ldo;
  return a;
}

static double gemm_out_bytes(const GemmArgs& a, size_t e) {
  double MN = (double)a.M * a.N;
  switch (a.epi) {
    case EPI_F32: case EPI_SIGMOID: return 4 * MN;
    case EPI_DT: return e * MN;
    case EPI_RESID: return 8 * MN;
    case EPI_QKVG: return (double)a.M * a.d * (3 * e + 4) + 4.0 * a.M * a.d;  // + cos/sin reads
    case EPI_SWIGLU: return e * MN / 2;
    case EPI_DECQG: return (a.out16 ? 4.0 : 8.0) * a.k_tok * MN;  // q and g (fp16 or fp32), every token type
  }
  return 0;
}

static rest_status run_gemm(const Plan& p, const GemmArgs& a, const char* name, cudaStream_t s) {
  const bool bf = p.dt == REST_BF16;
  if (a.f16 && !(bf && sm100_gemm_supported(a))) return REST_ERR_UNSUPPORTED;  // fp16 products: tensor cores only
  const size_t e = dt_size(p.dt);
  const double groups = a.epi == EPI_DECQG ? 2.0 * a.k_tok : a.groups > 1 ? (double)a.groups : 1.0;
  const double flops = 2.0 * a.M * a.N * a.K * groups;
  const double a_sets = a.epi == EPI_DECQG ? a.k_tok : a.groups > 1 ? a.groups : 1;  // distinct A column blocks
  const double out_sets = a.epi != EPI_DECQG && a.groups > 1 ? a.groups : 1;
  const double bytes = (a.a_f32 || a.A2 ? 4 : e) * (double)a.M * a.K * a_sets + e * (double)a.K * a.N * groups +
                       gemm_out_bytes(a, e) * out_sets;
  if (bf && sm100_gemm_supported(a)) {
    REST_KLAUNCH(s, name, flops, bytes, launch_gemm_sm100(a, s, p.err));
  } else {
    REST_KLAUNCH(s, name, flops, bytes, launch_gemm_simt(bf, a, s));
  }
  return REST_OK;
}

// ---------------------------------------------------------------- encoder

// With `cache` the rows are tokens appended to cached histories: each layer
// adds their rotated keys and gated values to the cache and attends to the
// cached rows and the new ones.
static rest_status run_encoder(const Plan& p, const void* x, const int64_t* ts, const rest_enc_layer* layers,
                               int n_layers, int l_switch, void* h_out, void* ws, int32_t* err, cudaStream_t s,
                               const rest_kv_cache* cache = nullptr) {
  const bool bf = p.dt == REST_BF16;
  const int d = p.hs->d, hd = p.hs->head_dim, H = p.hs->n_heads;
  const long long T = p.T;
  const size_t e = dt_size(p.dt);
  const double Td = (double)T * d;
  const Layout& L = p.L;
  const int32_t* cu = at<int32_t>(ws, L.cu);
  float* cos_t = at<float>(ws, L.cos_t);
  float* sin_t = at<float>(ws, L.sin_t);
  float* xres = at<float>(ws, L.xres);
  void* y = at<void>(ws, L.y);
  void *q = at<void>(ws, L.q), *k = at<void>(ws, L.k), *v = at<void>(ws, L.v), *o = at<void>(ws, L.o);
  float* g = at<float>(ws, L.g);
  void* hid = at<void>(ws, L.hid);

  const UserAppend* app = cache ? at<UserAppend>(ws, L.app) : nullptr;
  double causal_pairs = 0;  // per user: n new rows after `off` cached ones see n off + n(n+1)/2 keys
  double key_rows = 0;      // keys read per head (cached and new)
  for (int u = 0; u < p.b->n_users; ++u) {
    const double n = p.b->cu_seqlens[u + 1] - p.b->cu_seqlens[u];
    const double off = cache ? p.app[u].cached : 0;
    causal_pairs += n * off + n * (n + 1) / 2;
    key_rows += n > 0 ? off + n : 0;
  }
  const double attn_flops = 4.0 * d * causal_pairs;  // QK^T and PV over every head
  const double attn_bytes = Td * (e + 4 + e) + 2.0 * e * key_rows * d;  // Q, gate, out; K and V'

  TableParams tp = table_params(p.hs);

  EncAttnArgs ea;
  memset(&ea, 0, sizeof(ea));  // optional outputs (lse, out_lo) stay null
  ea.q = q; ea.k = k; ea.v = v; ea.gate = g; ea.out = o; ea.cu = cu;
  ea.tiles = at<EncTile>(ws, L.enc_tiles); ea.n_tiles = L.n_enc_tiles;
  ea.sched = at<int>(ws, L.enc_sched);
  ea.n_cta = p.enc_sched.empty() ? 0 : std::min((int)p.enc_tiles.size() * H, SCHED_CTAS);
  ea.n_heads = H; ea.d = d;
  ea.scale_log2 = (float)(1.4426950408889634 / sqrt((double)hd));
  ea.rows = T;
  ea.app = app;
  ea.key_rows = cache ? cache->rows : T;
  ea.n_split = p.n_split_enc;
  if (p.n_split_enc > 1) {
    ea.part_o = at<float>(ws, L.part_o);
    ea.part_ml = at<float>(ws, L.part_ml);
  }

  // The sublayers in order (attention, then the FFN, per layer), each wrapped
  // by eq. 6: post-LN in the first l_switch layers, pre-LN after. One
  // normalisation launch follows each residual add: the post-LN of the
  // sublayer just finished (if any) merged with the next sublayer's input
  // (its pre-LN, or a plain cast), or with the cast of H.
  struct Sub {
    bool attn;
    int layer;
    bool post;
    const float* g;
    const float* b;
  };
  std::vector<Sub> subs;
  for (int l = 0; l < n_layers; ++l) {
    const bool post = (l + 1) <= l_switch;
    subs.push_back({true, l, post, layers[l].ln_attn_g, layers[l].ln_attn_b});
    if (layers[l].w_ffn13) subs.push_back({false, l, post, layers[l].ln_ffn_g, layers[l].ln_ffn_b});
  }
  auto norm = [&](void* out, const float* g, const float* b, int mode, const float* g2, const float* b2) -> rest_status {
    const double bytes = Td * (mode == 2 ? 4 + e : mode == 3 ? 8 : mode == 0 ? 4 + e : 8 + e);
    REST_KLAUNCH(s, "layernorm", 0, bytes, launch_layernorm(bf, xres, out, g, b, (int)T, d, mode, s, g2, b2));
    return REST_OK;
  };
  // The rotation table, x into the fp32 residual stream and (pre-LN) the first
  // sublayer's input: in bf16 one launch, whose table blocks (arithmetic-bound)
  // and row blocks (HBM-bound) share the SMs; otherwise three.
  const bool fuse_first = bf && d % 128 == 0 && d <= 1024;
  const bool pre0 = !subs.empty() && !subs[0].post;
  if (fuse_first) {
    REST_KLAUNCH(s, "table_cast_ln", 0, 8.0 * T + 4 * Td + Td * (e + 4) + (pre0 ? Td * e : 0),
                 launch_table_cast_ln(ts, cu, p.b->n_users, (int)T, tp, cos_t, sin_t, err, app, x, xres,
                                      pre0 ? y : nullptr, pre0 ? subs[0].g : nullptr, pre0 ? subs[0].b : nullptr,
                                      d, s));
  } else {
    REST_KLAUNCH(s, "rotation_table", 0, 8.0 * T + 4 * Td,
                 launch_rotation_table(ts, cu, p.b->n_users, (int)T, tp, nullptr, cos_t, sin_t, err, s, app));
    REST_KLAUNCH(s, "to_f32", 0, Td * (e + 4), launch_to_f32(bf, x, xres, T * d, s));
  }
  // input of the first sublayer: with post-LN it reads x itself, which in bf16
  // is the call's input as it stands
  // (with no layers H is x)
  const void* a_in = y;
  if (subs.empty()) {
  } else if (subs[0].post) {
    if (bf) a_in = x;
    else if (rest_status st = norm(y, nullptr, nullptr, 2, nullptr, nullptr)) return st;
  } else if (!fuse_first) {
    if (rest_status st = norm(y, subs[0].g, subs[0].b, 0, nullptr, nullptr)) return st;
  }
  bool h_written = false;
  for (size_t i = 0; i < subs.size(); ++i) {
    const Sub& S = subs[i];
    const rest_enc_layer& Ly = layers[S.layer];
    if (S.attn) {  // DGA sublayer (eqs. 3-5)
      const int nb = gate_blocks(Ly.gates);  // column blocks of the projection weight
      GemmArgs a = gemm(a_in, d, Ly.w_qkvgg, (long long)nb * d, T, nb * d, d, EPI_QKVG, q, d);
      a.out1 = k; a.out2 = v; a.out3 = g; a.cos_t = cos_t; a.sin_t = sin_t; a.d = d; a.gate_mode = Ly.gates;
      if (rest_status st = run_gemm(p, a, "gemm_qkvg", s)) return st;
      if (cache) {  // the new rows' R k and V' join the layer's cache; attention reads keys there
        REST_KLAUNCH(s, "append_kv", 0, 4.0 * e * Td,
                     launch_append_rows(k, cache->k[S.layer], v, cache->v[S.layer], cu, app, p.b->n_users, T,
                                        (int)(d * e), s));
        ea.k = cache->k[S.layer];
        ea.v = cache->v[S.layer];
      }
      if (bf && sm100_attn_supported(hd)) {
        REST_KLAUNCH(s, "enc_attn", attn_flops, attn_bytes, launch_enc_attn_sm100(hd, ea, s, err));
        if (p.n_split_enc > 1)
          REST_KLAUNCH(s, "enc_combine", 0, Td * (4.0 * (p.n_split_enc + 1) + e),
                       launch_enc_combine(hd, ea, s));
      } else {
        REST_KLAUNCH(s, "enc_attn", attn_flops, attn_bytes, launch_enc_attn_simt(bf, hd, ea, s));
      }
      a = gemm(o, d, Ly.w_o, d, T, d, d, EPI_RESID, xres, d);
      a.alpha = Ly.alpha_attn;
      if (rest_status st = run_gemm(p, a, "gemm_attn_out", s)) return st;
    } else {  // SwiGLU FFN sublayer
      const int dff = Ly.d_ff;
      GemmArgs a = gemm(a_in, d, Ly.w_ffn13, 2LL * dff, T, 2 * dff, d, EPI_SWIGLU, hid, dff);
      a.d = dff;
      if (rest_status st = run_gemm(p, a, "gemm_ffn13", s)) return st;
      a = gemm(hid, dff, Ly.w_ffn2, d, T, d, dff, EPI_RESID, xres, d);
      a.alpha = Ly.alpha_ffn;
      if (rest_status st = run_gemm(p, a, "gemm_ffn2", s)) return st;
    }
    a_in = y;
    rest_status st = REST_OK;
    if (i + 1 < subs.size()) {
      const Sub& N = subs[i + 1];  // post-LN sublayers come first, so a pre-LN one is followed by pre-LN
      if (S.post && N.post) st = norm(y, S.g, S.b, 1, nullptr, nullptr);        // x = LN(x), y = x
      else if (S.post) st = norm(y, S.g, S.b, 4, N.g, N.b);                     // x = LN(x), y = LN'(x)
      else st = norm(y, N.g, N.b, 0, nullptr, nullptr);                         // y = LN'(x)
    } else if (S.post) {
      if (p.hsplit || p.h16) {
        st = norm(nullptr, S.g, S.b, 3, nullptr, nullptr);  // x = LN(x)
      } else {
        st = norm(h_out, S.g, S.b, 1, nullptr, nullptr);    // x = LN(x), H = x
        h_written = true;
      }
    }
    if (st != REST_OK) return st;
  }
  // H: the residual stream after the last layer, in the call's dtype (no final norm).
  // When the tensor-core decoder follows, also H in fp16 (what it multiplies in);
  // when the CUDA-core decoder follows in bf16, H's low part: H = h_out + h_lo.
  if (p.h16) {
    REST_KLAUNCH(s, "split_h", 0, Td * 8, launch_split_h16(xres, h_out, at<void>(ws, L.hx), T * d, err, s));
  } else if (p.hsplit) {
    REST_KLAUNCH(s, "split_h", 0, Td * 8, launch_split_bf16(xres, h_out, at<void>(ws, L.hx), T * d, s));
  } else if (!h_written) {
    if (rest_status st = norm(h_out, nullptr, nullptr, 2, nullptr, nullptr)) return st;
  }
  if (cache && cache->h)
    REST_KLAUNCH(s, "append_h", 0, 2.0 * e * Td,
                 launch_append_rows(h_out, cache->h, nullptr, nullptr, cu, app, p.b->n_users, T, (int)(d * e), s));
  return REST_OK;
}

// ---------------------------------------------------------------- decoder

// h: the caller's H (the call's dtype). from_encoder: the encoder ran in the
// same call and left the workspace's hx as the decoder needs it (the fp16 H of
// the tensor-core decoder, or H_lo of the CUDA-core one).
static rest_status run_decoder(const Plan& p, const rest_requests* reqs, const void* h, bool from_encoder,
                               const void* z, const rest_dec_params* dec, float* y_out, void* ws, int32_t* err,
                               cudaStream_t s) {
  const bool bf = p.dt == REST_BF16;
  const int d = p.hs->d, hd = p.hs->head_dim, K = dec->K;
  const size_t e = dt_size(p.dt);
  const Layout& L = p.L;
  float* dq = at<float>(ws, L.dq);
  float* dg = at<float>(ws, L.dg);
  float* dout = at<float>(ws, L.dout);
  const long long N = p.n_cands;
  const bool tc = bf && sm100_attn_supported(hd);
  // token-specific projections (eq. 8): rows n*K + k use W_Q^(k), W_go^(k);
  // the tensor-core GEMM does all token types and both weights in one launch. For
  // the tensor-core decoder it writes q, already scaled by log2(e) / sqrt(d_h),
  // and the gate in fp16 (in the fp32 buffers' bytes).
  GemmArgs qg = gemm(z, (long long)K * d, dec->w_q, d, N, d, d, EPI_DECQG, dq, (long long)K * d);
  qg.out1 = dg;
  qg.B2 = dec->w_go;
  qg.k_tok = K;
  if (tc) {
    qg.out16 = 1;
    qg.alpha = (float)(1.4426950408889634 / sqrt((double)hd));
  }
  if (bf && sm100_gemm_supported(qg)) {
    if (rest_status st = run_gemm(p, qg, "gemm_dec_qg", s)) return st;
  } else if (tc) {
    return REST_ERR_UNSUPPORTED;  // the fp16 queries come from the tensor-core projection only
  } else
  for (int kk = 0; kk < K; ++kk) {
    const char* zk = (const char*)z + e * (size_t)kk * d;
    GemmArgs a = gemm(zk, (long long)K * d, (const char*)dec->w_q + e * (size_t)kk * d * d, d, N, d, d, EPI_F32,
                      dq + (size_t)kk * d, (long long)K * d);
    if (rest_status st = run_gemm(p, a, "gemm_dec_q", s)) return st;
    a = gemm(zk, (long long)K * d, (const char*)dec->w_go + e * (size_t)kk * d * d, d, N, d, d, EPI_SIGMOID,
             dg + (size_t)kk * d, (long long)K * d);
    if (rest_status st = run_gemm(p, a, "gemm_dec_g", s)) return st;
  }
  // The tensor-core decoder multiplies in fp16 (H, q and P): its H is the fp16
  // copy in the workspace, converted here unless the encoder wrote it.
  const void* h_lo = !tc && from_encoder && p.hsplit ? at<void>(ws, L.hx) : nullptr;
  if (tc) {
    if (!from_encoder)
      REST_KLAUNCH(s, "h_to_f16", 0, 4.0 * p.T * d, launch_bf16_to_f16(h, at<void>(ws, L.hx), p.T * d, err, s));
    h = at<void>(ws, L.hx);
  }
  // every H prefix is read once per request; each candidate row reads q, g and writes o
  double flops = 0, hbytes = 0;
  for (int r = 0; r < reqs->n_req; ++r) {
    double rows = (double)(reqs->cu_cands[r + 1] - reqs->cu_cands[r]) * K;
    if (rows == 0) continue;
    flops += 4.0 * d * rows * reqs->req_cutoff[r];
    hbytes += (double)e * reqs->req_cutoff[r] * d * (h_lo ? 2 : 1);
  }
  // q and g in, o * g out: fp16 each for the tensor-core decoder, fp32 for the
  // CUDA-core one; with split keys the tensor-core decoder reads q and writes
  // one fp32 partial o per split, and the combine reads g
  const double bytes = hbytes + (double)p.NK * d * (!tc ? 12 : p.n_split > 1 ? 2 + 4.0 * p.n_split : 6);
  // The tensor-core decoder hands o * g to the output projection in fp16, the
  // CUDA-core one in fp32.
  DecAttnArgs da;
  memset(&da, 0, sizeof(da));
  da.q = dq; da.g = dg; da.h = h; da.h_lo = h_lo; da.out = dout;
  da.q16 = dq; da.g16 = dg;
  da.tiles = at<DecTile>(ws, L.dec_tiles); da.n_tiles = L.n_dec_tiles;

  da.n_heads = p.hs->n_heads; da.d = d;
  da.scale_log2 = (float)(1.4426950408889634 / sqrt((double)hd));
  da.key_rows = p.T;
  da.n_split = p.n_split;
  da.nk_rows = p.NK;
  da.part_o = at<float>(ws, L.part_o);
  da.part_ml = at<float>(ws, L.part_ml);
  if (tc) {
    da.sched = at<int>(ws, L.dec_sched);
    da.n_cta = std::min(L.n_dec_tiles * p.hs->n_heads, SCHED_CTAS);
    if (L.n_dec_tiles > 0) REST_KLAUNCH(s, "dec_attn", flops, bytes, launch_dec_attn_sm100(hd, da, s, err));
    if (p.n_split > 1)
      REST_KLAUNCH(s, "dec_combine", 0, (double)p.NK * d * (4.0 * p.n_split + 4),
                   launch_dec_combine(hd, da, s));
  } else {
    REST_KLAUNCH(s, "dec_attn", flops, bytes, launch_dec_attn_simt(bf, hd, da, s));
  }
  // y = (o * g) W_o: one fp16 product for the tensor-core decoder (W_o copied to
  // fp16 per call), fp32 A otherwise
  const void* wo = dec->w_o;
  if (tc) {
    REST_KLAUNCH(s, "w_o_f16", 0, 4.0 * d * d, launch_bf16_to_f16(dec->w_o, at<void>(ws, L.wo16), (long long)d * d, err, s));
    wo = at<void>(ws, L.wo16);
  }
  GemmArgs a = gemm(dout, d, wo, d, p.NK, d, d, EPI_F32, y_out, d);
  if (tc)
    a.f16 = 1;
  else
    a.a_f32 = 1;
  if (rest_status st = run_gemm(p, a, "gemm_dec_out", s)) return st;
  return REST_OK;
}

}  // namespace rest

using namespace rest;

extern "C" {

const char* rest_status_string(rest_status s) {
  switch (s) {
    case REST_OK: return "ok";
    case REST_ERR_INVALID_ARG: return "invalid argument";
    case REST_ERR_UNSORTED_TIME: return "timestamps decrease within a user";
    case REST_ERR_UNSUPPORTED: return "unsupported shape";
    case REST_ERR_CUDA: return "CUDA runtime error";
    case REST_ERR_TIMEOUT: return "bounded device wait ran out";
    case REST_ERR_WORKSPACE: return "workspace missing or too small";
    case REST_ERR_NO_DEVICE: return "no sm_100 CUDA device is current";
    case REST_ERR_RANGE: return "decoder value beyond the fp16 range";
  }
  return "unknown status";
}

void rest_profile_begin(void) {
  g_prof = true;
  if (!g_recs) g_recs = new std::vector<ProfRec>();
  g_recs->clear();
}

int rest_profile_end(rest_kernel_stat* out, int max_out) {
  g_prof = false;
  if (!g_recs) return 0;
  std::vector<rest_kernel_stat> agg;
  for (ProfRec& r : *g_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
      cudaGetLastError();
      ms = 0.f;
    }
    size_t i = 0;
    while (i < agg.size() && strcmp(agg[i].name, r.name) != 0) ++i;
    if (i == agg.size()) agg.push_back(rest_kernel_stat{r.name, 0, 0.0, 0.0, 0.0});
    agg[i].launches += 1;
    agg[i].ms += ms;
    agg[i].flops += r.flops;
    agg[i].bytes += r.bytes;
    if (!g_event_pool) g_event_pool = new std::vector<cudaEvent_t>();
    g_event_pool->push_back(r.a);
    g_event_pool->push_back(r.b);
  }
  g_recs->clear();
  int n = (int)agg.size();
  for (int i = 0; i < n && i < max_out; ++i) out[i] = agg[i];
  return n;
}

long long rest_launch_count(int reset) {
  long long v = g_launches;
  if (reset) g_launches = 0;
  return v;
}

rest_status rest_workspace_size(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                                const rest_enc_layer* layers, int n_layers, const rest_requests* reqs, int K,
                                size_t* bytes) {
  if (!bytes) return REST_ERR_INVALID_ARG;
  try {
    Plan p;
    rest_status st = make_plan(p, dt, heads, batch, layers, n_layers, n_layers, reqs, K,
                               n_layers > 0 || !reqs);
    if (st != REST_OK) return st;
    *bytes = p.L.total;
    return REST_OK;
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

rest_status rest_rotation_table(const rest_heads* heads, const rest_batch* batch, const int64_t* ts,
                                int64_t* idx_out, float* cos_out, float* sin_out, void* ws, size_t ws_bytes,
                                int32_t* dev_err, void* stream) {
  try {
    Plan p;
    rest_status st = make_plan(p, REST_F32, heads, batch, nullptr, 0, 0, nullptr, 1, true);
    if (st != REST_OK) return st;
    if ((cos_out == nullptr) != (sin_out == nullptr)) return REST_ERR_INVALID_ARG;
    if (p.T > 0 && !ts) return REST_ERR_INVALID_ARG;
    if (!ws || ws_bytes < p.L.total) return REST_ERR_WORKSPACE;
    if (p.T == 0) return REST_OK;
    if ((st = check_device()) != REST_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    p.err = dev_err;
    if ((st = upload_meta(p, ws, s)) != REST_OK) return st;
    TableParams tp = table_params(heads);
    REST_KLAUNCH(s, "rotation_table", 0, 8.0 * p.T + 4.0 * p.T * heads->d,
                 launch_rotation_table(ts, at<int32_t>(ws, p.L.cu), batch->n_users, (int)p.T, tp, idx_out, cos_out,
                                       sin_out, dev_err, s));
    return REST_OK;
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

rest_status rest_encoder_attn(rest_dtype dt, const rest_heads* heads, const rest_batch* batch, const void* x,
                              const int64_t* ts, const rest_enc_layer* layers, int n_layers, int l_switch,
                              void* h_out, void* ws, size_t ws_bytes, int32_t* dev_err, void* stream) {
  try {
    Plan p;
    rest_status st = make_plan(p, dt, heads, batch, layers, n_layers, l_switch, nullptr, 1, true);
    if (st != REST_OK) return st;
    if (p.T > 0 && (!x || !ts || !h_out || !aligned16(x) || !aligned16(ts) || !aligned16(h_out)))
      return REST_ERR_INVALID_ARG;
    if (!ws || ws_bytes < p.L.total || !aligned16(ws)) return REST_ERR_WORKSPACE;
    if (p.T == 0) return REST_OK;
    if ((st = check_device()) != REST_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    p.err = dev_err;
    if ((st = upload_meta(p, ws, s)) != REST_OK) return st;
    return run_encoder(p, x, ts, layers, n_layers, l_switch, h_out, ws, dev_err, s);
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

rest_status rest_append_workspace_size(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                                       const rest_enc_layer* layers, int n_layers, size_t* bytes) {
  if (!bytes) return REST_ERR_INVALID_ARG;
  try {
    Plan p;
    rest_status st = make_plan(p, dt, heads, batch, layers, n_layers, n_layers, nullptr, 1, true, nullptr, true);
    if (st != REST_OK) return st;
    *bytes = p.L.total;
    return REST_OK;
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

rest_status rest_encoder_append(rest_dtype dt, const rest_heads* heads, const rest_batch* batch, const void* x,
                                const int64_t* ts, const rest_enc_layer* layers, int n_layers, int l_switch,
                                const rest_kv_cache* cache, void* h_out, void* ws, size_t ws_bytes,
                                int32_t* dev_err, void* stream) {
  try {
    if (!cache) return REST_ERR_INVALID_ARG;
    Plan p;
    rest_status st = make_plan(p, dt, heads, batch, layers, n_layers, l_switch, nullptr, 1, true, cache, true);
    if (st != REST_OK) return st;
    if (p.T > 0 && (!x || !ts || !h_out || !aligned16(x) || !aligned16(ts) || !aligned16(h_out)))
      return REST_ERR_INVALID_ARG;
    if (!ws || ws_bytes < p.L.total || !aligned16(ws)) return REST_ERR_WORKSPACE;
    if (p.T == 0) return REST_OK;
    if ((st = check_device()) != REST_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    p.err = dev_err;
    if ((st = upload_meta(p, ws, s)) != REST_OK) return st;
    return run_encoder(p, x, ts, layers, n_layers, l_switch, h_out, ws, dev_err, s, cache);
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

rest_status rest_selftest_wait_timeout(int n_ctas, long long limit_cycles, int32_t* dev_err, void* stream) {
  if (n_ctas < 1 || n_ctas > 1024 || limit_cycles < 1000000LL || limit_cycles > 4000000000LL || !dev_err)
    return REST_ERR_INVALID_ARG;
  rest_status st = check_device();
  if (st != REST_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(dev_err, 0, sizeof(int32_t), s) != cudaSuccess) return REST_ERR_CUDA;
  REST_KLAUNCH(s, "selftest_wait_timeout", 0, 0, launch_wait_timeout(n_ctas, limit_cycles, dev_err, s));
  return REST_OK;
}

rest_status rest_attn_workspace_size(rest_dtype dt, const rest_heads* heads, const rest_batch* batch, size_t* bytes) {
  if (!bytes) return REST_ERR_INVALID_ARG;
  try {
    Plan p;
    rest_status st = make_plan(p, dt, heads, batch, nullptr, 0, 0, nullptr, 1, true, nullptr, false, true);
    if (st != REST_OK) return st;
    *bytes = p.L.total;
    return REST_OK;
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

rest_status rest_attn_forward(rest_dtype dt, const rest_heads* heads, const rest_batch* batch, const void* q,
                              const void* k, const void* v, void* o, void* o_lo, float* lse, void* ws,
                              size_t ws_bytes, int32_t* dev_err, void* stream) {
  try {
    Plan p;
    rest_status st = make_plan(p, dt, heads, batch, nullptr, 0, 0, nullptr, 1, true, nullptr, false, true);
    if (st != REST_OK) return st;
    if (p.T > 0 && (!q || !k || !v || !o || !lse || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
                    !aligned16(o) || !aligned16(lse) || !aligned16(o_lo) || (o_lo && dt != REST_BF16)))
      return REST_ERR_INVALID_ARG;
    if (!ws || ws_bytes < p.L.total || !aligned16(ws)) return REST_ERR_WORKSPACE;
    if (p.T == 0) return REST_OK;
    if ((st = check_device()) != REST_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    p.err = dev_err;
    if ((st = upload_meta(p, ws, s)) != REST_OK) return st;
    const bool bf = dt == REST_BF16;
    const int d = heads->d, hd = heads->head_dim, H = heads->n_heads;
    const size_t e = dt_size(dt);
    double pairs = 0;
    for (int u = 0; u < batch->n_users; ++u) {
      const double L = batch->cu_seqlens[u + 1] - batch->cu_seqlens[u];
      pairs += L * (L + 1) / 2;
    }
    EncAttnArgs ea;
    memset(&ea, 0, sizeof(ea));
    ea.q = q; ea.k = k; ea.v = v; ea.gate = nullptr; ea.out = o; ea.out_lo = o_lo; ea.lse = lse;
    ea.cu = at<int32_t>(ws, p.L.cu);
    ea.tiles = at<EncTile>(ws, p.L.enc_tiles); ea.n_tiles = p.L.n_enc_tiles;
    ea.sched = at<int>(ws, p.L.enc_sched);
    ea.n_cta = p.enc_sched.empty() ? 0 : std::min((int)p.enc_tiles.size() * H, SCHED_CTAS);
    ea.n_heads = H; ea.d = d;
    ea.scale_log2 = (float)(1.4426950408889634 / sqrt((double)hd));
    ea.rows = p.T;
    ea.key_rows = p.T;
    const double flops = 4.0 * d * pairs, bytes = (double)p.T * d * ((o_lo ? 5 : 4) * e) + 4.0 * p.T * H;
    if (bf && sm100_attn_supported(hd)) {
      REST_KLAUNCH(s, "attn_fwd", flops, bytes, launch_enc_attn_sm100(hd, ea, s, dev_err));
    } else {
      REST_KLAUNCH(s, "attn_fwd", flops, bytes, launch_enc_attn_simt(bf, hd, ea, s));
    }
    return REST_OK;
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

rest_status rest_attn_backward(rest_dtype dt, const rest_heads* heads, const rest_batch* batch, const void* q,
                               const void* k, const void* v, const void* o, const void* o_lo, const float* lse,
                               const void* d_o, float* dq, float* dk, float* dv, void* ws, size_t ws_bytes,
                               int32_t* dev_err, void* stream) {
  try {
    Plan p;
    rest_status st = make_plan(p, dt, heads, batch, nullptr, 0, 0, nullptr, 1, true, nullptr, false, true);
    if (st != REST_OK) return st;
    const void* ptrs[] = {q, k, v, o, lse, d_o, dq, dk, dv};
    if (p.T > 0) {
      for (const void* ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return REST_ERR_INVALID_ARG;
      if (!aligned16(o_lo) || (o_lo && dt != REST_BF16)) return REST_ERR_INVALID_ARG;
    }
    if (!ws || ws_bytes < p.L.total || !aligned16(ws)) return REST_ERR_WORKSPACE;
    if (p.T == 0) return REST_OK;
    if ((st = check_device()) != REST_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    p.err = dev_err;
    if ((st = upload_meta(p, ws, s)) != REST_OK) return st;
    const bool bf = dt == REST_BF16;
    const int d = heads->d, hd = heads->head_dim, H = heads->n_heads;
    const size_t e = dt_size(dt);
    double pairs = 0;
    for (int u = 0; u < batch->n_users; ++u) {
      const double L = batch->cu_seqlens[u + 1] - batch->cu_seqlens[u];
      pairs += L * (L + 1) / 2;
    }
    AttnBwdArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.o = o; a.o_lo = o_lo; a.d_o = d_o; a.lse = lse;
    a.delta = at<float>(ws, p.L.delta);
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.cu = at<int32_t>(ws, p.L.cu);
    a.tiles = at<EncTile>(ws, p.L.bwd_tiles); a.n_tiles = p.L.n_bwd_tiles;
    a.n_heads = H; a.d = d;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)hd));
    a.rows = p.T;
    // delta = rowsum(dO * O); then dq (S, dP and dS K per visible (query, key, head)) and dk, dv
    // (S, dP, P^T dO and dS^T q): 6 + 8 d_h-long products, against 5 in one fused pass
    const double td = (double)p.T * d;
    REST_KLAUNCH(s, "attn_bwd_delta", 0, td * (o_lo ? 3 : 2) * e + 4.0 * p.T * H,
                 launch_attn_bwd_simt(bf, hd, 0, a, s));
    if (bf && sm100_attn_supported(hd) && !p.bwd_sched.empty()) {
      // one pass: S^T, dP^T, dV, dK, dQ per (key block, query block); dq gathers by atomics
      if (cudaMemsetAsync(dq, 0, sizeof(float) * (size_t)p.T * d, s) != cudaSuccess) return REST_ERR_CUDA;
      a.sched = at<int>(ws, p.L.bwd_sched);
      a.n_cta = std::min((int)p.bwd_tiles.size() * H, SCHED_CTAS);
      // algorithmic bytes: q, k, v, dO in, dq, dk, dv out (fp32), lse and delta
      REST_KLAUNCH(s, "attn_bwd", 10.0 * d * pairs, td * (4 * e + 12) + 8.0 * p.T * H,
                   launch_attn_bwd_sm100(hd, a, s, dev_err));
    } else {
      REST_KLAUNCH(s, "attn_bwd_dq", 6.0 * d * pairs, td * (3 * e + 4), launch_attn_bwd_simt(bf, hd, 1, a, s));
      REST_KLAUNCH(s, "attn_bwd_dkdv", 8.0 * d * pairs, td * (4 * e + 8), launch_attn_bwd_simt(bf, hd, 2, a, s));
    }
    return REST_OK;
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

rest_status rest_cross_decode(rest_dtype dt, const rest_heads* heads, const rest_batch* batch, const void* h,
                              const rest_requests* reqs, const void* z, const rest_dec_params* dec, float* y_out,
                              void* ws, size_t ws_bytes, int32_t* dev_err, void* stream) {
  try {
    rest_status st = check_dec(dec);
    if (st != REST_OK) return st;
    if (!reqs) return REST_ERR_INVALID_ARG;
    Plan p;
    if ((st = make_plan(p, dt, heads, batch, nullptr, 0, 0, reqs, dec->K, false)) != REST_OK) return st;
    if (p.NK > 0 && (!h || !z || !y_out || !aligned16(h) || !aligned16(z) || !aligned16(y_out)))
      return REST_ERR_INVALID_ARG;
    if (!ws || ws_bytes < p.L.total || !aligned16(ws)) return REST_ERR_WORKSPACE;
    if (p.NK == 0) return REST_OK;
    if ((st = check_device()) != REST_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    p.err = dev_err;
    if ((st = upload_meta(p, ws, s)) != REST_OK) return st;
    return run_decoder(p, reqs, h, false, z, dec, y_out, ws, dev_err, s);
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

rest_status rest_rank_request(rest_dtype dt, const rest_heads* heads, const rest_batch* batch, const void* x,
                              const int64_t* ts, const rest_enc_layer* layers, int n_layers, int l_switch,
                              const rest_requests* reqs, const void* z, const rest_dec_params* dec, void* h_out,
                              float* y_out, void* ws, size_t ws_bytes, int32_t* dev_err, void* stream) {
  try {
    rest_status st = check_dec(dec);
    if (st != REST_OK) return st;
    if (!reqs) return REST_ERR_INVALID_ARG;
    Plan p;
    if ((st = make_plan(p, dt, heads, batch, layers, n_layers, l_switch, reqs, dec->K, true)) != REST_OK) return st;
    if (p.T > 0 && (!x || !ts || !h_out || !aligned16(x) || !aligned16(ts) || !aligned16(h_out)))
      return REST_ERR_INVALID_ARG;
    if (p.NK > 0 && (!z || !y_out || !aligned16(z) || !aligned16(y_out))) return REST_ERR_INVALID_ARG;
    if (!ws || ws_bytes < p.L.total || !aligned16(ws)) return REST_ERR_WORKSPACE;
    if (p.T == 0) return REST_OK;
    if ((st = check_device()) != REST_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    p.err = dev_err;
    if ((st = upload_meta(p, ws, s)) != REST_OK) return st;
    if ((st = run_encoder(p, x, ts, layers, n_layers, l_switch, h_out, ws, dev_err, s)) != REST_OK) return st;
    if (p.NK == 0) return REST_OK;
    return run_decoder(p, reqs, h_out, true, z, dec, y_out, ws, dev_err, s);
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

// ---------------------------------------------------------------- decoder block and score

// Workspace of the score head: the LN output u and the SwiGLU hidden state.
// The block has no residual scale to damp their rounding, so they do not enter
// its products as plain bf16. In bf16 with d a multiple of 128 and d_ff of 64
// (the tensor-core GEMMs' shapes) the products run in fp16 (kind::f16 with fp16
// operands): u and the hidden state in fp16, 8 times finer than bf16, and fp16
// copies of the token-specific weights made each call (exact within fp16's
// range). Otherwise (bf16) u = u + u_lo and hid = hid + hid_lo, each with a bf16
// low part, feed two passes of the products at fp32-level precision.
struct ScoreLayout {
  size_t u, u_lo, hid, hid_lo, w13, w2, total;
  bool f16;
};

static rest_status score_layout(rest_dtype dt, int d, int K, long long n, int d_ff, ScoreLayout* L) {
  if ((dt != REST_F32 && dt != REST_BF16) || d <= 0 || d > 1024 || d % 8 || K < 1 || K > 8 || n < 0 ||
      d_ff <= 0 || d_ff % 8)
    return REST_ERR_INVALID_ARG;
  const size_t e = dt_size(dt), rows = (size_t)n * K;
  const size_t ub = align_up(rows * d * e, 256), hb = align_up(rows * (size_t)d_ff * e, 256);
  L->f16 = dt == REST_BF16 && d % 128 == 0 && d_ff % 64 == 0;
  const bool lo = dt == REST_BF16 && !L->f16;
  L->u = 0;
  L->u_lo = ub;
  L->hid = L->u_lo + (lo ? ub : 0);
  L->hid_lo = L->hid + hb;
  L->w13 = L->hid_lo + (lo ? hb : 0);
  L->w2 = L->w13 + (L->f16 ? align_up((size_t)K * d * 2 * d_ff * 2, 256) : 0);
  L->total = L->w2 + (L->f16 ? align_up((size_t)K * d_ff * d * 2, 256) : 0);
  if (L->total == 0) L->total = 256;
  return REST_OK;
}

rest_status rest_score_workspace_size(rest_dtype dt, int d, int K, long long n_cands, int d_ff, size_t* bytes) {
  if (!bytes) return REST_ERR_INVALID_ARG;
  ScoreLayout L;
  rest_status st = score_layout(dt, d, K, n_cands, d_ff, &L);
  if (st == REST_OK) *bytes = L.total;
  return st;
}

rest_status rest_score_head(rest_dtype dt, int d, int K, long long n_cands, const void* z, const float* y,
                            const rest_score_params* sp, float* f_out, float* score_out, void* ws, size_t ws_bytes,
                            int32_t* dev_err, void* stream) {
  try {
    if (!sp) return REST_ERR_INVALID_ARG;
    ScoreLayout SL;
    rest_status st = score_layout(dt, d, K, n_cands, sp->d_ff, &SL);
    const size_t total = SL.total;
    if (st != REST_OK) return st;
    if (n_cands == 0) return REST_OK;
    if (!z || !y || !f_out || !score_out || !sp->w_ffn13 || !sp->w_ffn2 || !sp->ln_g || !sp->ln_b || !sp->w_s ||
        !aligned16(z) || !aligned16(y) || !aligned16(f_out) || !aligned16(sp->w_ffn13) || !aligned16(sp->w_ffn2))
      return REST_ERR_INVALID_ARG;
    if (!ws || ws_bytes < total || !aligned16(ws)) return REST_ERR_WORKSPACE;
    if ((st = check_device()) != REST_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (dev_err && cudaMemsetAsync(dev_err, 0, sizeof(int32_t), s) != cudaSuccess) return REST_ERR_CUDA;
    Plan p;
    p.dt = dt;
    p.err = dev_err;
    const bool bf = dt == REST_BF16;
    const bool f16 = SL.f16;  // the products in fp16
    const size_t e = dt_size(dt);
    const long long rows = n_cands * K;
    const int dff = sp->d_ff;
    char* u = at<char>(ws, SL.u);
    char* u_lo = bf && !f16 ? at<char>(ws, SL.u_lo) : nullptr;
    char* hid = at<char>(ws, SL.hid);
    char* hid_lo = bf && !f16 ? at<char>(ws, SL.hid_lo) : nullptr;
    const void* w13 = sp->w_ffn13;
    const void* w2 = sp->w_ffn2;
    if (f16) {  // fp16 copies of the token-specific weights
      w13 = at<void>(ws, SL.w13);
      w2 = at<void>(ws, SL.w2);
      REST_KLAUNCH(s, "score_w_f16", 0, 4.0 * K * d * 2 * dff,
                   launch_bf16_to_f16(sp->w_ffn13, at<void>(ws, SL.w13), (long long)K * d * 2 * dff, dev_err, s));
      REST_KLAUNCH(s, "score_w_f16", 0, 4.0 * K * dff * d,
                   launch_bf16_to_f16(sp->w_ffn2, at<void>(ws, SL.w2), (long long)K * dff * d, dev_err, s));
    }
    // a = z + y (the query token's residual, fp32 in f_out) and u = LN_k(a)
    REST_KLAUNCH(s, "score_ln", 0, (double)rows * d * (e + 4 + 4 + (f16 ? 2 : 2 * e)),
                 launch_score_ln(bf, z, y, f_out, u, u_lo, sp->ln_g, sp->ln_b, rows, d, K, s, f16, dev_err));
    // token type k: columns [k d, k d + d) of u and f_out and [k d_ff, k d_ff + d_ff) of the
    // hidden state (rows n K + k of the [n K, d] views), with that type's weights (eq. 8). The
    // tensor-core GEMM takes all token types in one grouped launch; otherwise one launch each.
    auto ffn13 = [&](int k) {
      GemmArgs a = gemm(u + e * (size_t)k * d, (long long)K * d,
                        (const char*)w13 + e * (size_t)k * d * 2 * dff, 2LL * dff, n_cands, 2 * dff, d,
                        EPI_SWIGLU, hid + e * (size_t)k * dff, (long long)K * dff);
      a.d = dff;
      a.f16 = f16;
      if (bf && !f16) {
        a.A2 = u_lo + e * (size_t)k * d;
        a.out1 = hid_lo + e * (size_t)k * dff;
      }
      return a;
    };
    auto ffn2 = [&](int k) {
      GemmArgs a = gemm(hid + e * (size_t)k * dff, (long long)K * dff,
                        (const char*)w2 + e * (size_t)k * dff * d, d, n_cands, d, dff, EPI_RESID,
                        f_out + (size_t)k * d, (long long)K * d);
      a.alpha = 1.0f;
      a.f16 = f16;
      if (bf && !f16) a.A2 = hid_lo + e * (size_t)k * dff;
      return a;
    };
    for (int stage = 0; stage < 2; ++stage) {
      const char* name = stage == 0 ? "gemm_score_ffn13" : "gemm_score_ffn2";
      GemmArgs all = stage == 0 ? ffn13(0) : ffn2(0);
      all.groups = K;
      // The down-projections of all token types run as one grouped launch (fewer
      // partial waves: 0.190 -> 0.165 ms for the ragged workload's three); the
      // SwiGLU up-projections only when one type's launch would leave SMs idle
      // (grouped they measured slower there, 0.278 -> 0.331 ms).
      const long long tiles = (n_cands + 255) / 256 * ((dff + 127) / 128);
      if (bf && K > 1 && (stage == 1 || tiles < 2 * SCHED_CTAS) && sm100_gemm_supported(all)) {
        if ((st = run_gemm(p, all, name, s)) != REST_OK) return st;
      } else {
        for (int k = 0; k < K; ++k)
          if ((st = run_gemm(p, stage == 0 ? ffn13(k) : ffn2(k), name, s)) != REST_OK) return st;
      }
    }
    REST_KLAUNCH(s, "score_readout", 2.0 * n_cands * d, (double)n_cands * d * 4,
                 launch_score_readout(f_out, sp->w_s, sp->b_s, score_out, n_cands, d, K, s));
    return REST_OK;
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}

}  // extern "C"

// ---------------------------------------------------------------- decoder without a caller workspace
//
// For callers that cannot allocate device memory (see rest.h): the decoder's
// scratch lives in a fixed array in the library's own device image instead of
// a caller-provided workspace. Every call on a device shares this one array.

namespace rest {

static __device__ __align__(256) unsigned char g_static_ws[REST_STATIC_WS_BYTES];

// Device address of g_static_ws in the current device's context. Host code may
// not use the symbol itself as an address. The lookup runs on every call: once
// the library's device image is loaded it costs little, and it also loads that
// image (with the array) on a device's first call, since the CUDA runtime loads
// modules lazily. An address cached across calls would go stale if the context
// were destroyed and re-created (cudaDeviceReset loads the image again).
static rest_status static_ws_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return REST_ERR_CUDA;
  }
  *out = p;
  return REST_OK;
}

}  // namespace rest

extern "C" size_t rest_static_ws_bytes(void) { return (size_t)REST_STATIC_WS_BYTES; }

extern "C" rest_status rest_cross_decode_static_ws(rest_dtype dt, const rest_heads* heads, const rest_batch* batch,
                                                   const void* h, const rest_requests* reqs, const void* z,
                                                   const rest_dec_params* dec, float* y_out, int32_t* dev_err,
                                                   void* stream) {
  try {
    rest_status st = check_dec(dec);
    if (st != REST_OK) return st;
    if (!reqs) return REST_ERR_INVALID_ARG;
    Plan p;
    if ((st = make_plan(p, dt, heads, batch, nullptr, 0, 0, reqs, dec->K, false)) != REST_OK) return st;
    if (p.NK > 0 && (!h || !z || !y_out || !aligned16(h) || !aligned16(z) || !aligned16(y_out)))
      return REST_ERR_INVALID_ARG;
    if (p.L.total > (size_t)REST_STATIC_WS_BYTES) return REST_ERR_WORKSPACE;  // batch too large for the array
    if ((st = check_device()) != REST_OK) return st;
    // Before the empty-batch return, so that a call with no candidates loads the
    // array on this device: the warm-up call that reserves it up front.
    void* ws = nullptr;
    if ((st = static_ws_address(&ws)) != REST_OK) return st;
    if (p.NK == 0) return REST_OK;
    cudaStream_t s = (cudaStream_t)stream;
    p.err = dev_err;
    // Nothing in the scratch needs to start at zero: the index/tile lists are
    // uploaded and q, g, o are written in full before they are read.
    if ((st = upload_meta(p, ws, s)) != REST_OK) return st;
    return run_decoder(p, reqs, h, false, z, dec, y_out, ws, dev_err, s);
  } catch (...) {
    return REST_ERR_INVALID_ARG;
  }
}
