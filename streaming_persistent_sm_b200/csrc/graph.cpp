// Host graph compiler for the persistent decode program.
//
// The compiler follows the pages' split of responsibilities: it starts from a
// fixed op list of the decoder (the tensor-level graph of "Why real-time
// inference wants a megakernel", "A concrete design"), splits every op into
// tiles sized to one worker's staging slot, derives tile-to-tile tensor
// edges (dropping the barrier edges between consecutive kernels and keeping
// the tile-to-tile tensor edges: "One Megakernel is Not Enough", Table I,
// cross-kernel readiness), dedups dependency counters by identical
// predecessor set, and emits the ticket order the device queue hands out.
// Dependency counters that let a consumer start once its own input chunk is
// ready follow "Persistent threads and megakernels", §6 (Hazy's Llama-1B
// megakernel); the down projection's K-chunks are that finer edge here.
#include "graph.h"

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstring>
#include <map>
#include <random>
#include <thread>
#include <unordered_map>

namespace wpk {

namespace {

uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

std::string fmt(const char* f, long long a = 0, long long b = 0, long long c = 0) {
  char buf[512];
  snprintf(buf, sizeof buf, f, a, b, c);
  return buf;
}

}  // namespace

std::string normalize_plan(const wpk_model_cfg& m, const wpk_plan_cfg& in, Plan* p, int* code) {
  *code = WPK_ERR_INVALID_ARG;
  if (m.n_layers <= 0 || m.hidden <= 0 || m.n_heads <= 0 || m.n_kv_heads <= 0 || m.head_dim <= 0 ||
      m.ffn <= 0 || m.vocab <= 0)
    return "model dimensions must be positive";
  if (m.n_heads % m.n_kv_heads) return "n_heads must be a multiple of n_kv_heads";
  if (m.n_heads / m.n_kv_heads > kMaxGroup) return "more than 8 query heads per kv head";
  {  // decode attention serves a kv group's heads in at most two head groups of <= 4
    const int grp = m.n_heads / m.n_kv_heads;
    if (grp > 4 && grp % 2) { *code = WPK_ERR_UNSUPPORTED; return "query heads per kv head must be 1-4, 6 or 8"; }
  }
  if (m.head_dim != 64) { *code = WPK_ERR_UNSUPPORTED; return "head_dim must be 64"; }
  if (m.hidden % 8 || m.ffn % 8) { *code = WPK_ERR_SHAPE; return "hidden and ffn must be multiples of 8"; }
  if (m.hidden > 2048 * 4) { *code = WPK_ERR_UNSUPPORTED; return "hidden > 8192"; }
  if (!(m.rms_eps >= 0.f) || !(m.rope_theta > 0.f)) return "bad rms_eps / rope_theta";
  if (in.max_batch <= 0 || in.max_context <= 0) return "max_batch and max_context must be positive";
  p->max_batch = in.max_batch;
  p->max_context = in.max_context;
  p->page_tokens = in.page_tokens ? in.page_tokens : 64;
  if (p->page_tokens % 8 || p->page_tokens > 256) return "page_tokens must be a multiple of 8, <= 256";
  p->workers_per_sm = in.workers_per_sm ? in.workers_per_sm : 1;
  p->n_workers = in.n_workers;
  if (p->n_workers < 0 || p->workers_per_sm < 0 || p->workers_per_sm > 4) return "bad worker count";
  p->mode = in.mode;
  if (p->mode != WPK_MEGAKERNEL && p->mode != WPK_PER_OP_GRAPH) return "bad mode";
  p->resident = in.resident;
  if (p->resident && p->mode != WPK_MEGAKERNEL) return "resident needs WPK_MEGAKERNEL";
  p->n_regions = in.n_regions ? in.n_regions : 1;
  if (p->n_regions < 1 || p->n_regions > 4) return "n_regions must be 1..4";
  if (p->resident && p->n_regions != 1) return "resident mode runs one region";
  for (int r = 0; r < 4; ++r) p->region_cut[r] = in.region_cut[r];
  if (p->n_regions > 1) {
    if (p->region_cut[0] != 0) return "region_cut[0] must be 0";
    for (int r = 1; r < p->n_regions; ++r)
      if (p->region_cut[r] <= p->region_cut[r - 1] || p->region_cut[r] > m.n_layers)
        return "region cuts must increase and be <= n_layers";
  }
  p->trace = in.trace;
  p->wait_timeout_ns = in.wait_timeout_ns ? in.wait_timeout_ns : 2000000000ull;
  p->lookahead = in.lookahead ? in.lookahead : 4;
  p->schedule = in.schedule;
  if (p->schedule != WPK_SCHED_QUEUE && p->schedule != WPK_SCHED_STATIC && p->schedule != WPK_SCHED_TEAMS)
    return "bad schedule";
  if (p->schedule == WPK_SCHED_TEAMS && (p->n_regions != 1 || p->resident || p->mode != WPK_MEGAKERNEL)) {
    *code = WPK_ERR_UNSUPPORTED;
    return "the team schedule runs one megakernel region launched per step";
  }
  if (p->lookahead < 1 || p->lookahead > kMaxQueue) return "lookahead must be 1..8";
  // activation staging: up to kMaxGemvBatch rows of the longest GEMV K (<= 2048)
  const int q_rows = m.n_heads * m.head_dim;
  const int kmax = std::max(std::max(m.hidden, q_rows), std::min(m.ffn, 2048));
  if (kmax > 2048) { *code = WPK_ERR_UNSUPPORTED; return "hidden and n_heads*head_dim must be <= 2048"; }
  const int kmax_pad = (kmax + 255) / 256 * 256;  // staged rows are padded to whole 256-column segments
  // the decode attention tiles use the same buffer: q, the current k/v, each
  // warp's per-head (m, l, o) and probabilities
  const int grp = m.n_heads / m.n_kv_heads;
  const int attn_need = (kMaxGroup * kHeadDim + 2 * kHeadDim + kWarps * grp * (2 + kHeadDim) + kWarps * 32 * grp) * 4;
  p->act_bytes = std::max(std::max(16384, attn_need), std::min(in.max_batch, kMaxGemvBatch) * kmax_pad * 4);
  p->act_bytes = (p->act_bytes + 1023) / 1024 * 1024;
  const int fixed = 4096 + 1024;  // partial outputs, tile queue, barriers
  const int budget = std::min(kMaxSmem, 233472 / p->workers_per_sm - 1024) - p->act_bytes - fixed;
  if (in.slot_bytes) {
    if (in.slot_bytes % kStageBytes || in.slot_bytes < kStageBytes || in.slot_bytes > kMaxStages * kStageBytes)
      return "slot_bytes must be a multiple of 16384, at most 13 stages";
    if (in.slot_bytes > budget) return "slot_bytes does not fit shared memory with this many workers per SM";
    p->slot_bytes = in.slot_bytes;
  } else {
    p->slot_bytes = std::min(12, budget / kStageBytes) * kStageBytes;
    if (p->slot_bytes < kStageBytes) return "no room for a staging slot";
  }
  // minimum weight bytes per tile: tensor-core decode tiles split along K are
  // faster with fewer, larger splits (64 KB measured best at batch 16 and 48)
  p->tile_bytes = in.tile_bytes ? in.tile_bytes
                                : ((in.decode == WPK_DECODE_MMA ||
                                    (in.decode == WPK_DECODE_AUTO && in.max_batch > kAutoGemvBatch))
                                       ? 65536
                                       : 32768);
  if (p->tile_bytes < 1024 || p->tile_bytes > 1 << 20) return "tile_bytes must be in [1K, 1M]";
  p->split_pages = in.split_pages;  // 0: chosen by compile_graph
  if (p->split_pages < 0) return "split_pages must be >= 0";
  if ((int64_t)p->page_tokens * m.head_dim * 2 * 2 > kStageBytes)
    return "a KV page (K and V rows) does not fit one 16 KB stage";
  p->per_op_slot = 0;  // set by compile_graph
  p->lm_rows = m.vocab;  // a two-stage backbone overrides it with its projection width
  {
    const int qr = m.n_heads * m.head_dim, kvr = m.n_kv_heads * m.head_dim;
    const bool mma_ok = (qr + 2 * kvr) % 128 == 0 && m.hidden % 128 == 0 && (2 * m.ffn) % 128 == 0 &&
                        m.hidden % 64 == 0 && qr % 128 == 0 && m.ffn % 64 == 0 && kvr % 128 == 0;
    if (in.decode == WPK_DECODE_AUTO)
      p->decode_mode = (in.max_batch > kAutoGemvBatch && in.max_batch <= kMaxMmaBatch && mma_ok) ? WPK_DECODE_MMA
                                                                                                : WPK_DECODE_GEMV;
    else if (in.decode == WPK_DECODE_MMA) {
      if (!mma_ok) { *code = WPK_ERR_UNSUPPORTED; return "shapes do not fit the tensor-core decode tiles"; }
      if (in.max_batch > kMaxMmaBatch) { *code = WPK_ERR_SHAPE; return "tensor-core decode takes at most 128 sequences"; }
      p->decode_mode = WPK_DECODE_MMA;
    } else if (in.decode == WPK_DECODE_GEMV)
      p->decode_mode = WPK_DECODE_GEMV;
    else
      return "bad decode mode";
    p->dec_n = p->dec_stage_bytes = p->dec_stages = p->dec_act_bytes = p->dec_cps = 0;
    if (p->decode_mode == WPK_DECODE_MMA) {
      // one ring stage = cps 16 KB weight chunks + their hi/lo activation
      // chunks of N tokens (N rows of 128 bytes each), each part one bulk copy
      // (an SM's copy engine completes only a few copies per microsecond, so
      // two chunks per stage when three or more stages still fit)
      p->dec_n = (in.max_batch + 15) / 16 * 16;
      // attention scratch: queries, one page of scores, the combine's (m, l) pairs
      const int max_pages = (in.max_context + p->page_tokens - 1) / p->page_tokens;
      const int need = std::max(attn_need, max_pages * kMaxGroup * 2 * 4);
      p->dec_act_bytes = std::max(16384, (need + 1023) / 1024 * 1024);
      const int room = kMaxSmem - fixed - 4096 - p->dec_act_bytes;  // 4 KB: the kernel's static shared memory
      int want = in.slot_bytes ? in.slot_bytes / kStageBytes : 12;
      const int one = kMmaChunkBytes + 2 * p->dec_n * 128;
      p->dec_cps = room / (2 * one) >= 3 ? 2 : 1;
      p->dec_stage_bytes = p->dec_cps * one;
      p->dec_stages = std::min(std::min(want, kMaxStages), room / p->dec_stage_bytes);
      if (p->dec_stages < 2) { *code = WPK_ERR_UNSUPPORTED; return "no room for the tensor-core decode ring"; }
    }
    if (in.prefill == WPK_PREFILL_AUTO)
      p->prefill_mode = mma_ok ? WPK_PREFILL_MMA : WPK_PREFILL_TOKENWISE;
    else if (in.prefill == WPK_PREFILL_MMA) {
      if (!mma_ok) { *code = WPK_ERR_UNSUPPORTED; return "shapes do not fit the tensor-core prefill tiles"; }
      p->prefill_mode = WPK_PREFILL_MMA;
    } else if (in.prefill == WPK_PREFILL_TOKENWISE)
      p->prefill_mode = WPK_PREFILL_TOKENWISE;
    else
      return "bad prefill mode";
  }
  *code = WPK_OK;
  return "";
}

// ---------------------------------------------------------------------------
// Dataflow edges: for each buffer keep, per element range, the last plain
// writer and the accumulators since then.  A read depends on the frontier
// (the accumulators if any, else the last writer); an accumulate depends on
// the last plain writer.  Write-after-read and write-after-write order is not
// added as edges; verify_graph proves every such pair is ordered by a path.
// ---------------------------------------------------------------------------
namespace {

struct Seg {
  int wgroup;                // group id of the current writers (-1 = single)
  std::vector<int> writers;  // last plain write (one tile, or one write group)
  std::vector<int> accs;     // accumulators since then
};

// Disjoint segments covering [0, size), keyed by their low end.
struct BufState {
  std::map<int64_t, Seg> segs;
  int64_t hi_;
  explicit BufState(int64_t size = 1) : hi_(size) { segs.emplace(0, Seg{-1, {}, {}}); }
  // make x a segment boundary
  void cut(int64_t x) {
    if (x <= 0 || x >= hi_) return;
    auto it = segs.upper_bound(x);
    --it;
    if (it->first == x) return;
    segs.emplace(x, it->second);
  }
  // first segment overlapping [lo, ...)
  std::map<int64_t, Seg>::iterator first(int64_t lo) {
    auto it = segs.upper_bound(lo);
    --it;
    return it;
  }
};

struct DataflowBuilder {
  std::vector<BufState> bufs;
  const std::vector<std::vector<int32_t>>* preds_of = nullptr;
  // memo of a read's frontier: (buf, lo, hi) -> preds, dropped when buf changes
  std::map<std::tuple<int, int64_t, int64_t>, std::vector<int>> memo;

  std::vector<int> frontier(int b, int64_t lo, int64_t hi) {
    auto key = std::make_tuple(b, lo, hi);
    auto mit = memo.find(key);
    if (mit != memo.end()) return mit->second;
    std::vector<int> out;
    BufState& B = bufs[b];
    for (auto it = B.first(lo); it != B.segs.end() && it->first < hi; ++it) {
      const auto& src = it->second.accs.empty() ? it->second.writers : it->second.accs;
      out.insert(out.end(), src.begin(), src.end());
    }
    std::sort(out.begin(), out.end());
    out.erase(std::unique(out.begin(), out.end()), out.end());
    memo[key] = out;
    return out;
  }
  void invalidate(int b) {
    for (auto it = memo.begin(); it != memo.end();) {
      if (std::get<0>(it->first) == b)
        it = memo.erase(it);
      else
        ++it;
    }
  }
  bool is_pred(int u, int w) const {
    const auto& P = (*preds_of)[w];
    return std::binary_search(P.begin(), P.end(), u);
  }
  // Exact "is u an ancestor of one of `preds`" for the few writers that
  // accumulations need ordering after: per watched writer, a descendant flag
  // per tile, extended as tiles are finished.
  std::unordered_map<int, std::vector<char>> desc;
  int n_done = 0;
  bool descends(int u, const std::vector<int>& preds) {
    auto it = desc.find(u);
    if (it == desc.end()) {
      std::vector<char> d(preds_of->size(), 0);
      for (int t = u + 1; t < n_done; ++t)
        for (int x : (*preds_of)[t])
          if (x == u || d[x]) {
            d[t] = 1;
            break;
          }
      it = desc.emplace(u, std::move(d)).first;
    }
    for (int x : preds)
      if (x == u || it->second[x]) return true;
    return false;
  }
  void finish(int t) {
    for (auto& kv : desc) {
      if (t <= kv.first) continue;
      for (int x : (*preds_of)[t])
        if (x == kv.first || kv.second[x]) {
          kv.second[t] = 1;
          break;
        }
    }
    n_done = t + 1;
  }
  void apply(int t, const std::vector<Access>& acc, std::vector<int>* preds) {
    std::vector<int> acc_deps;
    for (auto& a : acc) {
      if (a.kind == 0) {
        auto f = frontier(a.buf, a.lo, a.hi);
        preds->insert(preds->end(), f.begin(), f.end());
      } else if (a.kind == 2) {
        BufState& B = bufs[a.buf];
        for (auto it = B.first(a.lo); it != B.segs.end() && it->first < a.hi; ++it)
          acc_deps.insert(acc_deps.end(), it->second.writers.begin(), it->second.writers.end());
      }
    }
    std::sort(preds->begin(), preds->end());
    preds->erase(std::unique(preds->begin(), preds->end()), preds->end());
    // An accumulate must follow the write that initialised its range; skip the
    // edge when one of the tile's read predecessors already depends on it.
    std::sort(acc_deps.begin(), acc_deps.end());
    acc_deps.erase(std::unique(acc_deps.begin(), acc_deps.end()), acc_deps.end());
    for (int u : acc_deps) {
      bool implied = std::binary_search(preds->begin(), preds->end(), u);
      for (size_t i = 0; !implied && i < preds->size() && i < 4; ++i) implied = is_pred(u, (*preds)[i]);
      if (!implied && !preds->empty()) implied = descends(u, *preds);
      if (!implied) preds->push_back(u);
    }
    for (auto& a : acc) {
      if (a.kind == 0) continue;
      BufState& B = bufs[a.buf];
      B.cut(a.lo);
      B.cut(a.hi);
      for (auto it = B.first(a.lo); it != B.segs.end() && it->first < a.hi; ++it) {
        Seg& s = it->second;
        if (a.kind == 1) {
          if (a.group >= 0 && s.wgroup == a.group && s.accs.empty()) {
            s.writers.push_back(t);
          } else {
            s.writers.assign(1, t);
            s.wgroup = a.group;
            s.accs.clear();
          }
        } else {
          s.accs.push_back(t);
        }
      }
      invalidate(a.buf);
    }
    std::sort(preds->begin(), preds->end());
    preds->erase(std::unique(preds->begin(), preds->end()), preds->end());
    preds->erase(std::remove(preds->begin(), preds->end(), t), preds->end());
    finish(t);
  }
};

struct VecHash {
  size_t operator()(const std::vector<int>& v) const {
    size_t h = v.size() * 0x9E3779B97F4A7C15ull;
    for (int x : v) h ^= (size_t)x + 0x9E3779B97F4A7C15ull + (h << 6) + (h >> 2);
    return h;
  }
};

// Rows per GEMV tile for an op with `op_rows` rows of `row_bytes`: about
// 1/W of the op (W workers) so that every worker gets about one tile per op,
// at least tile_bytes, at most kMaxTileRows, a multiple of the rows per chunk
// stage.  Chunks stream through the staging ring; only when more than 8
// sequences force several passes over a tile's chunks must a tile fit the
// ring.
int rows_per_tile(int row_bytes, int op_rows, const Plan& p, int W) {
  int rpc = (kStageBytes / row_bytes) & ~1;
  if (rpc < 2) rpc = 2;
  int r = std::max(p.tile_bytes / row_bytes, (op_rows + W - 1) / std::max(1, W));
  r = (r + rpc - 1) / rpc * rpc;
  if (p.max_batch > kMaxGemvBatch) r = std::min(r, gemv_ring_chunks(p.slot_bytes) * rpc);
  r = std::min(r, kMaxTileRows / rpc * rpc);
  return std::max(r, 2);
}

// GEMV LM head tiles (fused final RMSNorm + logits + argmax): row ranges of
// the LM head in the weight image.
struct LmTile {
  uint64_t w_off;
  uint32_t w_bytes;
  int r0, n;
};
// Offsets are relative to the LM head's base (the launch's lm_head_off).
std::vector<LmTile> gemv_lm_tiles(const wpk_model_cfg& m, const Plan& p, int W, const Layout& L) {
  (void)L;
  std::vector<LmTile> out;
  const int h = m.hidden, rows = p.lm_rows;
  const int R = rows_per_tile(h * 2, rows, p, W);
  for (int r0 = 0; r0 < rows; r0 += R) {
    const int n = std::min(R, rows - r0);
    out.push_back({(uint64_t)r0 * h * 2, (uint32_t)n * h * 2, r0, n});
  }
  return out;
}

// K splits of a tensor-core op with `rb` blocks of 128 rows and `nkc` 64-column
// chunks: as many tiles as fit the workers in one round (rb x splits <= W, so
// that no worker runs two tiles of the op while another idles), none smaller
// than tile_bytes.
int mma_splits(int rb, int nkc, const Plan& p, int W) {
  const int want = std::max(1, W / rb);
  const int most = std::max(1, nkc * kMmaChunkBytes / std::max(p.tile_bytes, kMmaChunkBytes));
  return std::max(1, std::min(std::min(want, most), nkc));
}

// Batched decode program: every projection is a tensor-core tile of 128
// weight rows x (K range) x (the step's N tokens), swap-AB (the weights are
// the MMA's M operand, the tokens its N).  Projections followed by a
// nonlinearity (gate/up, LM head) take the whole K; the others are split
// along K so that every worker has a tile and sum into fp32 buffers.  The
// last split of each O / down row block turns its finished residual rows into
// the next RMSNorm's input image (x * g) and adds their x^2 to the per-token
// sums; consumers apply 1/rms per token column in their epilogue.
template <class Add>
void build_mma_decode_tiles(const wpk_model_cfg& m, const Plan& p, int W, CompiledGraph& g, Add& add,
                            std::vector<uint32_t>* layer_begin) {
  const int h = m.hidden, hd = m.head_dim, grp = m.n_heads / m.n_kv_heads;
  const int q_rows = m.n_heads * hd, kv_rows = m.n_kv_heads * hd, qkv_rows = q_rows + 2 * kv_rows;
  const uint32_t chunk = kMmaChunkBytes;
  const int nkc_h = h / 64, nkc_q = q_rows / 64, nkc_f = m.ffn / 64;
  const int s_qkv = mma_splits(qkv_rows / 128, nkc_h, p, W);
  g.o_splits = mma_splits(h / 128, nkc_q, p, W);
  g.down_splits = mma_splits(h / 128, nkc_f, p, W);
  auto krange = [](int nkc, int s, int i, int* c0, int* c1) {
    *c0 = (int)((int64_t)nkc * i / s);
    *c1 = (int)((int64_t)nkc * (i + 1) / s);
  };
  const Layout& L = g.lay;
  // x = E[tok] per 128-feature block, with the first RMSNorm's input image
  for (int fb = 0; fb < h / 128; ++fb)
    add(OP_EMBED, 0, 0, 0, fb, 0, 0, 0,
        {{BUF_XA, fb * 128, fb * 128 + 128, 1}, {BUF_DXN, fb * 128, fb * 128 + 128, 1}, {BUF_TOK, 0, 1, 0}});
  for (int l = 0; l < m.n_layers; ++l) {
    const LayerDev& d = L.layers[l];
    (*layer_begin)[l] = (uint32_t)g.tiles.size();
    for (int fb = 0; fb < qkv_rows / 128; ++fb)
      for (int i = 0; i < s_qkv; ++i) {
        int c0, c1;
        krange(nkc_h, s_qkv, i, &c0, &c1);
        add(OP_BQKV, l, d.mma_qkv + ((uint64_t)fb * nkc_h + c0) * chunk, (uint32_t)(c1 - c0) * chunk, fb, 0, c0 * 64,
            (c1 - c0) * 64, {{BUF_DXN, 0, h, 0}, {BUF_QKV, fb * 128, fb * 128 + 128, 2}});
      }
    const int attn_group = 1000 + l;
    for (int b = 0; b < p.max_batch; ++b)
      for (int gi = 0; gi < m.n_kv_heads; ++gi)
        for (int j = 0; j < g.n_splits; ++j)
          add(OP_ATTN, l, 0, 0, b, gi, j, 0,
              {{BUF_QKV, gi * grp * hd, (gi + 1) * grp * hd, 0},
               {BUF_QKV, q_rows + gi * hd, q_rows + (gi + 1) * hd, 0},
               {BUF_QKV, q_rows + kv_rows + gi * hd, q_rows + kv_rows + (gi + 1) * hd, 0},
               {BUF_ATTN, gi * grp * hd, (gi + 1) * grp * hd, 1, attn_group}});
    for (int fb = 0; fb < h / 128; ++fb)
      for (int i = 0; i < g.o_splits; ++i) {
        int c0, c1;
        krange(nkc_q, g.o_splits, i, &c0, &c1);
        add(OP_BO, l, d.mma_wo + ((uint64_t)fb * nkc_q + c0) * chunk, (uint32_t)(c1 - c0) * chunk, fb, 0, c0 * 64,
            (c1 - c0) * 64,
            {{BUF_ATTN, c0 * 64, c1 * 64, 0}, {BUF_XA, fb * 128, fb * 128 + 128, 2},
             {BUF_DXF, fb * 128, fb * 128 + 128, 1, 3000 + l}});
      }
    for (int fb = 0; fb < 2 * m.ffn / 128; ++fb)
      add(OP_BGU, l, d.mma_gu + (uint64_t)fb * nkc_h * chunk, (uint32_t)nkc_h * chunk, fb, 0, 0, h,
          {{BUF_DXF, 0, h, 0}, {BUF_H, fb * 64, fb * 64 + 64, 1}});
    for (int fb = 0; fb < h / 128; ++fb)
      for (int i = 0; i < g.down_splits; ++i) {
        int c0, c1;
        krange(nkc_f, g.down_splits, i, &c0, &c1);
        add(OP_BDOWN, l, d.mma_down + ((uint64_t)fb * nkc_f + c0) * chunk, (uint32_t)(c1 - c0) * chunk, fb, 0,
            c0 * 64, (c1 - c0) * 64,
            {{BUF_H, c0 * 64, c1 * 64, 0}, {BUF_XA, fb * 128, fb * 128 + 128, 2},
             {BUF_DXN, fb * 128, fb * 128 + 128, 1, 4000 + l}});
      }
  }
  (*layer_begin)[m.n_layers] = (uint32_t)g.tiles.size();
  for (int vb = 0; vb < L.vocab_blocks; ++vb) {  // offsets relative to the launch's lm_mma_off
    const int r0 = vb * 128, n = std::min(128, p.lm_rows - r0);
    add(OP_BLM, m.n_layers, (uint64_t)vb * nkc_h * chunk, (uint32_t)nkc_h * chunk, vb, 0, 0, h,
        {{BUF_DXN, 0, h, 0}, {BUF_LOGITS, r0, r0 + n, 1}, {BUF_BEST, 0, 1, 2}});
  }
  add(OP_FINAL, m.n_layers, 0, 0, 0, 0, 0, 0, {{BUF_BEST, 0, 1, 0}, {BUF_TOK, 0, 1, 1}});
}

// Team schedule ("Why real-time inference wants a megakernel", "A concrete
// design: one WPK update"): every op group (phase) goes to one team of
// workers - all W workers, a half, a quarter, ... or one worker (aligned
// blocks of floor(W / 2^j)) - the smallest team with at least as many workers
// as the op has tiles, and among those the team whose busiest worker has the
// least work so far; inside the team each tile goes to the least loaded
// worker.  Work is estimated as the bytes a tile stages (weights or KV pages)
// plus a fixed cost per tile.  Each worker's tiles form its stream, in ticket
// order, so an edge between two tiles of one stream is already kept by that
// order and is dropped; only edges between streams keep a counter.  Deadlock
// freedom holds as for the static streams: every remaining edge points to a
// smaller ticket, and the worker holding the smallest unfinished ticket has
// finished everything before it in its own stream.
void assign_teams(CompiledGraph* g, int W) {
  const size_t n = g->tiles.size();
  const double kTileCost = 32768.0;  // fixed cost of a tile, in staged-byte equivalents
  std::vector<double> load(W, 0.0);
  g->worker_of.assign(n, 0);
  for (const OpGroup& og : g->groups) {
    const int tiles = (int)(og.end - og.begin);
    int size = W;
    while (size > 1 && size / 2 >= tiles) size /= 2;
    const int n_teams = W / size;
    int best_team = 0;
    double best = 1e300;
    for (int k = 0; k < n_teams; ++k) {
      double mx = 0.0;
      for (int w = k * size; w < (k + 1) * size; ++w) mx = std::max(mx, load[w]);
      if (mx < best) {
        best = mx;
        best_team = k;
      }
    }
    for (uint32_t t = og.begin; t < og.end; ++t) {
      const Tile& T = g->tiles[t];
      double cost = kTileCost + (double)T.w_bytes;
      if (T.op == OP_ATTN) cost += (double)g->split_tokens * g->m.head_dim * 4;  // K and V bf16 rows
      int w0 = best_team * size, wb = w0;
      for (int w = w0; w < w0 + size; ++w)
        if (load[w] < load[wb]) wb = w;
      g->worker_of[t] = wb;
      load[wb] += cost;
    }
  }
  // streams in ticket order, and each tile's predecessor in its stream
  std::vector<std::vector<uint32_t>> per(W);
  for (size_t t = 0; t < n; ++t) per[g->worker_of[t]].push_back((uint32_t)t);
  g->stream_begin.assign(W + 1, 0);
  g->stream.clear();
  g->stream_prev.assign(n, -1);
  for (int w = 0; w < W; ++w) {
    g->stream_begin[w] = (uint32_t)g->stream.size();
    for (size_t i = 0; i < per[w].size(); ++i) {
      g->stream.push_back(per[w][i]);
      if (i) g->stream_prev[per[w][i]] = (int32_t)per[w][i - 1];
    }
  }
  g->stream_begin[W] = (uint32_t)g->stream.size();
}

// Team schedule counters: a worker signals once per op group it served, from
// its last tile of the group (the phase barrier of the pages' design); a tile
// waits for the workers that hold its predecessors in each predecessor group -
// itself included, so that every consumer of a group shares one counter -
// except when all of them are on its own worker, where its stream order
// already keeps the dependency.  Returns, per tile, the signalling tiles it
// waits for (sorted).
std::vector<std::vector<int>> team_waits(const CompiledGraph& g) {
  const size_t n = g.tiles.size();
  std::vector<int> group_of(n, 0);
  for (size_t gi = 0; gi < g.groups.size(); ++gi)
    for (uint32_t t = g.groups[gi].begin; t < g.groups[gi].end; ++t) group_of[t] = (int)gi;
  // last tile of (group, worker): scan in ticket order
  std::unordered_map<uint64_t, int> last;
  for (size_t t = 0; t < n; ++t) last[((uint64_t)group_of[t] << 32) | (uint32_t)g.worker_of[t]] = (int)t;
  std::vector<std::vector<int>> waits(n);
  for (size_t v = 0; v < n; ++v) {
    std::map<int, std::vector<int>> by_group;  // predecessor group -> workers holding v's predecessors there
    for (int u : g.preds[v]) by_group[group_of[u]].push_back(g.worker_of[u]);
    for (auto& kv : by_group) {
      auto& ws = kv.second;
      std::sort(ws.begin(), ws.end());
      ws.erase(std::unique(ws.begin(), ws.end()), ws.end());
      if (ws.size() == 1 && ws[0] == g.worker_of[v]) continue;  // kept by v's own stream
      for (int w : ws) {
        const int x = last[((uint64_t)kv.first << 32) | (uint32_t)w];
        if (x < (int)v) {
          waits[v].push_back(x);
        } else {  // the group reaches past v (an edge inside one op): keep the tile edges
          for (int u : g.preds[v])
            if (group_of[u] == kv.first && g.worker_of[u] == w) waits[v].push_back(u);
        }
      }
    }
    std::sort(waits[v].begin(), waits[v].end());
    waits[v].erase(std::unique(waits[v].begin(), waits[v].end()), waits[v].end());
  }
  return waits;
}

}  // namespace

std::string compile_graph(const wpk_model_cfg& m, const Plan& p, CompiledGraph* g, int* code, int W) {
  *code = WPK_ERR_SHAPE;
  g->m = m;
  g->plan = p;
  const int h = m.hidden, hd = m.head_dim, grp = m.n_heads / m.n_kv_heads;
  const int q_rows = m.n_heads * hd, kv_rows = m.n_kv_heads * hd, qkv_rows = q_rows + 2 * kv_rows;
  // down projection K chunks: at most 2048 columns each, multiple of 8
  int nch = (m.ffn + 2047) / 2048;
  while (m.ffn % nch || (m.ffn / nch) % 8) ++nch;
  const int kc = m.ffn / nch;
  // a GEMV chunk holds an even number of rows (RoPE and gate/up pairs): two
  // rows of every GEMV op must fit one 16 KB chunk
  if (h * 4 > kStageBytes || q_rows * 4 > kStageBytes || kc * 4 > kStageBytes)
    return "two weight rows do not fit one 16 KB chunk";

  // ---- weight image layout ----
  Layout& L = g->lay;
  uint64_t off = 0;
  auto take = [&](uint64_t bytes) {
    uint64_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.layers.resize(m.n_layers);
  for (int l = 0; l < m.n_layers; ++l) {
    LayerDev& d = L.layers[l];
    d.attn_norm = take((uint64_t)h * 4);
    d.ffn_norm = take((uint64_t)h * 4);
    d.qkv = take((uint64_t)qkv_rows * h * 2);
    d.wo = take((uint64_t)h * q_rows * 2);
    d.gu = take((uint64_t)2 * m.ffn * h * 2);
    d.down = take((uint64_t)h * m.ffn * 2);
  }
  L.final_norm = take((uint64_t)h * 4);
  L.embed = take((uint64_t)m.vocab * h * 2);
  L.lm_head = m.tied_embedding ? L.embed : take((uint64_t)p.lm_rows * h * 2);
  L.mma = p.prefill_mode == WPK_PREFILL_MMA || p.decode_mode == WPK_DECODE_MMA;
  for (int l = 0; l < m.n_layers; ++l) {
    LayerDev& d = L.layers[l];
    d.mma_qkv = d.mma_wo = d.mma_gu = d.mma_down = 0;
    if (!L.mma) continue;
    d.mma_qkv = take((uint64_t)qkv_rows * h * 2);
    d.mma_wo = take((uint64_t)h * q_rows * 2);
    d.mma_gu = take((uint64_t)2 * m.ffn * h * 2);
    d.mma_down = take((uint64_t)h * m.ffn * 2);
  }
  L.lm_mma = 0;
  L.vocab_blocks = 0;
  if (p.decode_mode == WPK_DECODE_MMA) {
    L.vocab_blocks = (p.lm_rows + 127) / 128;
    L.lm_mma = take((uint64_t)L.vocab_blocks * (h / 64) * kMmaChunkBytes);
  }
  L.total = off;
  L.down_kc = kc;
  L.n_down_chunks = nch;

  // ---- attention splits: KV pages per tile; by default about two attention
  // tiles per worker over the batch and kv heads ----
  g->W = W;
  g->max_blocks = (p.max_context + p.page_tokens - 1) / p.page_tokens;
  {
    int sp = p.split_pages;
    if (sp == 0) {
      // about two attention tiles per worker on CUDA cores; on the tensor-core
      // decode, whose ring stages also hold the preceding QKV tile's weights,
      // at most one per worker (a second tile's pages would be staged late:
      // 1572 against 1767 us per step at batch 16)
      const int pairs = p.max_batch * m.n_kv_heads;
      const int per = p.decode_mode == WPK_DECODE_MMA ? W : 2 * W;
      const int ns = std::max(1, std::min(g->max_blocks, (per + pairs / 2) / pairs));
      sp = (g->max_blocks + ns - 1) / ns;
    }
    g->plan.split_pages = sp;
    g->split_tokens = sp * p.page_tokens;
  }
  g->n_splits = (p.max_context + g->split_tokens - 1) / g->split_tokens;

  // ---- tiles in ticket order ----
  std::vector<Tile>& T = g->tiles;
  std::vector<std::vector<Access>>& A = g->access;
  T.clear();
  A.clear();
  g->groups.clear();
  int64_t wbytes = 0;
  auto add = [&](uint16_t op, int layer, uint64_t w_off, uint32_t w_bytes, int a0, int a1, int a2, int a3,
                 std::vector<Access> acc) {
    Tile t{};
    t.op = op;
    t.layer = (uint16_t)layer;
    t.wait_ctr = kNoCounter;
    t.w_off = w_off;
    t.w_bytes = w_bytes;
    t.a0 = a0; t.a1 = a1; t.a2 = a2; t.a3 = a3;
    wbytes += w_bytes;
    if (g->groups.empty() || g->groups.back().op != op || g->groups.back().layer != layer)
      g->groups.push_back({op, layer, (uint32_t)T.size(), (uint32_t)T.size()});
    T.push_back(t);
    A.push_back(std::move(acc));
    g->groups.back().end = (uint32_t)T.size();
  };
  std::vector<uint32_t> layer_begin(m.n_layers + 1, 0);

  if (p.decode_mode == WPK_DECODE_MMA) {
    build_mma_decode_tiles(m, p, W, *g, add, &layer_begin);
  } else {
  add(OP_EMBED, 0, 0, 0, 0, 0, 0, 0, {{BUF_XA, 0, h, 1}, {BUF_TOK, 0, 1, 0}});
  for (int l = 0; l < m.n_layers; ++l) {
    const LayerDev& d = L.layers[l];
    layer_begin[l] = (uint32_t)T.size();
    const int attn_group = 1000 + l;
    // fused RMSNorm + QKV + RoPE + KV write; tiles never straddle q/k/v sections
    {
      int R = rows_per_tile(h * 2, qkv_rows, p, W);
      int sec_lo[3] = {0, q_rows, q_rows + kv_rows}, sec_hi[3] = {q_rows, q_rows + kv_rows, qkv_rows};
      for (int s = 0; s < 3; ++s)
        for (int r0 = sec_lo[s]; r0 < sec_hi[s]; r0 += R) {
          int n = std::min(R, sec_hi[s] - r0);
          add(OP_QKV, l, d.qkv + (uint64_t)r0 * h * 2, (uint32_t)n * h * 2, r0, n, 0, h,
              {{BUF_XA, 0, h, 0}, {BUF_QKV, r0, r0 + n, 1}});
        }
    }
    // split-KV attention per (sequence, kv head, split)
    for (int b = 0; b < p.max_batch; ++b)
      for (int gi = 0; gi < m.n_kv_heads; ++gi)
        for (int j = 0; j < g->n_splits; ++j)
          add(OP_ATTN, l, 0, 0, b, gi, j, 0,
              {{BUF_QKV, gi * grp * hd, (gi + 1) * grp * hd, 0},
               {BUF_QKV, q_rows + gi * hd, q_rows + (gi + 1) * hd, 0},
               {BUF_QKV, q_rows + kv_rows + gi * hd, q_rows + kv_rows + (gi + 1) * hd, 0},
               {BUF_ATTN, gi * grp * hd, (gi + 1) * grp * hd, 1, attn_group}});
    // O projection + residual
    {
      int R = rows_per_tile(q_rows * 2, h, p, W);
      for (int r0 = 0; r0 < h; r0 += R) {
        int n = std::min(R, h - r0);
        add(OP_O, l, d.wo + (uint64_t)r0 * q_rows * 2, (uint32_t)n * q_rows * 2, r0, n, 0, q_rows,
            {{BUF_ATTN, 0, q_rows, 0}, {BUF_XB, r0, r0 + n, 1}, {BUF_XA, r0, r0 + n, 1}});
      }
    }
    // fused RMSNorm + gate/up + SwiGLU (physical rows: gate j at 2j, up j at 2j+1)
    {
      int R = rows_per_tile(h * 2, 2 * m.ffn, p, W);
      for (int r0 = 0; r0 < 2 * m.ffn; r0 += R) {
        int n = std::min(R, 2 * m.ffn - r0);
        add(OP_GU, l, d.gu + (uint64_t)r0 * h * 2, (uint32_t)n * h * 2, r0, n, 0, h,
            {{BUF_XB, 0, h, 0}, {BUF_H, r0 / 2, (r0 + n) / 2, 1}});
      }
    }
    // down projection, split along K into chunks (finer edges), accumulated into x
    {
      int R = rows_per_tile(kc * 2, h * nch, p, W);
      for (int c = 0; c < nch; ++c)
        for (int r0 = 0; r0 < h; r0 += R) {
          int n = std::min(R, h - r0);
          add(OP_DOWN, l, d.down + ((uint64_t)c * h + r0) * kc * 2, (uint32_t)n * kc * 2, r0, n, c * kc, kc,
              {{BUF_H, c * kc, (c + 1) * kc, 0}, {BUF_XA, r0, r0 + n, 2}});
        }
    }
  }
  layer_begin[m.n_layers] = (uint32_t)T.size();
  for (const LmTile& t : gemv_lm_tiles(m, p, W, L))
    add(OP_LMHEAD, m.n_layers, t.w_off, t.w_bytes, t.r0, t.n, 0, h,
        {{BUF_XA, 0, h, 0}, {BUF_LOGITS, t.r0, t.r0 + t.n, 1}, {BUF_BEST, 0, 1, 2}});
  add(OP_FINAL, m.n_layers, 0, 0, 0, 0, 0, 0, {{BUF_BEST, 0, 1, 0}, {BUF_TOK, 0, 1, 1}});
  }
  g->algo_weight_bytes = wbytes;
  // a per-op CTA holds one whole tile in its ring
  int max_chunks = 1;
  for (const Tile& t : T)
    if (t.op != OP_ATTN && t.w_bytes && t.op < OP_BQKV) {
      const int rpc = std::max(2, (kStageBytes / (t.a3 * 2)) & ~1);
      max_chunks = std::max(max_chunks, (t.a1 + rpc - 1) / rpc);
    }
  // a per-op CTA streams its tile through a ring no larger than a worker's
  // (an even chunk count: GEMV stages take two chunks)
  g->plan.per_op_slot = std::min((max_chunks + 1) / 2 * 2 * kStageBytes, p.slot_bytes);
  if (T.size() >= (1u << 31)) return "too many tiles";

  // ---- edges from dataflow ----
  DataflowBuilder df;
  int sizes[BUF_COUNT] = {h, h, qkv_rows, q_rows, m.ffn, p.lm_rows, 1, 1, 1, 1, 1, 1, 1, 1, h, h};
  for (int b = 0; b < BUF_COUNT; ++b) df.bufs.emplace_back(sizes[b]);
  g->preds.assign(T.size(), {});
  df.preds_of = &g->preds;
  g->n_edges = 0;
  for (size_t t = 0; t < T.size(); ++t) {
    df.apply((int)t, A[t], &g->preds[t]);
    g->n_edges += (int64_t)g->preds[t].size();
  }

  // ---- team schedule: teams per op, worker streams, same-stream edges dropped ----
  if (p.schedule == WPK_SCHED_TEAMS) assign_teams(g, W);

  // ---- counters: one per distinct predecessor set (the team schedule: per
  //      distinct set of signalling tiles, one per worker and group) ----
  std::vector<std::vector<int>> tw;
  if (p.schedule == WPK_SCHED_TEAMS) tw = team_waits(*g);
  std::unordered_map<std::vector<int>, uint32_t, VecHash> ctr_of;
  std::vector<std::vector<uint32_t>> sig_of(T.size());
  g->ctr_need.clear();
  for (size_t t = 0; t < T.size(); ++t) {
    const auto& P = tw.empty() ? g->preds[t] : tw[t];
    if (P.empty()) continue;
    auto it = ctr_of.find(P);
    uint32_t c;
    if (it == ctr_of.end()) {
      c = (uint32_t)g->ctr_need.size();
      ctr_of.emplace(P, c);
      g->ctr_need.push_back((uint32_t)P.size());
      for (int u : P) sig_of[u].push_back(c);
    } else {
      c = it->second;
    }
    T[t].wait_ctr = c;
    T[t].need = g->ctr_need[c];
  }
  g->sig.clear();
  for (size_t t = 0; t < T.size(); ++t) {
    T[t].sig_off = (uint32_t)g->sig.size();
    T[t].sig_cnt = (uint32_t)sig_of[t].size();
    g->sig.insert(g->sig.end(), sig_of[t].begin(), sig_of[t].end());
  }

  // ---- regions: contiguous ticket ranges starting at layer cuts ----
  g->region_begin.assign(1, 0);
  for (int r = 1; r < p.n_regions; ++r) g->region_begin.push_back(layer_begin[p.region_cut[r]]);
  g->region_begin.push_back((uint32_t)T.size());
  *code = WPK_OK;
  return "";
}

// ---------------------------------------------------------------------------
// Prefill program.  Token rows m = b*T + t (M = B*T) are processed in blocks of
// kTokBlock rows.  Per layer: RMSNorm of each block into a bf16 hi/lo image,
// tensor-core QKV tiles (RoPE, q to Q, k/v to the KV cache), causal attention
// tiles of 128 / group queries (the GQA group of one kv head: 128 rows), tensor-core O
// tiles (X += .), RMSNorm again, tensor-core gate/up tiles (SwiGLU into the h
// image) and down tiles (X += .).  Then the last position of every sequence is
// gathered and the decode program's LM head + argmax tiles produce the first
// token.  Buffers are modelled per token block so that edges follow blocks.
// ---------------------------------------------------------------------------
std::string compile_prefill_graph(const CompiledGraph& dec, int B, int T, CompiledGraph* g) {
  const wpk_model_cfg& m = dec.m;
  const Plan& p = dec.plan;
  if (!dec.lay.mma) return "the weight image has no tensor-core layout";
  g->m = m;
  g->plan = p;
  g->lay = dec.lay;
  g->split_tokens = dec.split_tokens;
  g->n_splits = dec.n_splits;
  g->max_blocks = dec.max_blocks;
  g->B = B;
  g->T = T;
  g->M = B * T;
  g->n_tb = (g->M + kTokBlock - 1) / kTokBlock;
  g->W = dec.W;
  const int h = m.hidden, hd = m.head_dim, grp = m.n_heads / m.n_kv_heads;
  const int q_rows = m.n_heads * hd, kv_rows = m.n_kv_heads * hd, qkv_rows = q_rows + 2 * kv_rows;
  const int nq = g->n_tb;
  const int64_t TB = kTokBlock;
  std::vector<Tile>& Tl = g->tiles;
  std::vector<std::vector<Access>>& A = g->access;
  Tl.clear();
  A.clear();
  g->groups.clear();
  int64_t wbytes = 0;
  auto add = [&](uint16_t op, int layer, uint64_t w_off, uint32_t w_bytes, int a0, int a1, int a2, int a3,
                 std::vector<Access> acc) {
    Tile t{};
    t.op = op;
    t.layer = (uint16_t)layer;
    t.wait_ctr = kNoCounter;
    t.w_off = w_off;
    t.w_bytes = w_bytes;
    t.a0 = a0; t.a1 = a1; t.a2 = a2; t.a3 = a3;
    wbytes += w_bytes;
    if (g->groups.empty() || g->groups.back().op != op || g->groups.back().layer != layer)
      g->groups.push_back({op, layer, (uint32_t)Tl.size(), (uint32_t)Tl.size()});
    Tl.push_back(t);
    A.push_back(std::move(acc));
    g->groups.back().end = (uint32_t)Tl.size();
  };
  // modelled intervals: block tb of a buffer with `width` features
  auto blk = [&](int buf, int width, int tb, int f0, int f1, int kind, int group = -1) {
    Access a;
    a.buf = buf;
    a.lo = (int64_t)tb * width * TB + (int64_t)f0 * TB;
    a.hi = (int64_t)tb * width * TB + (int64_t)f1 * TB;
    a.kind = kind;
    a.group = group;
    return a;
  };
  auto kvblk = [&](int layer, int tb, int f0, int f1, int kind) {  // per-layer KV, features [0, 2*kv_rows)
    Access a;
    a.buf = BUF_PKV;
    a.lo = ((int64_t)layer * nq + tb) * (2 * kv_rows) * TB + (int64_t)f0 * TB;
    a.hi = ((int64_t)layer * nq + tb) * (2 * kv_rows) * TB + (int64_t)f1 * TB;
    a.kind = kind;
    a.group = -1;
    return a;
  };
  std::vector<uint32_t> layer_begin(m.n_layers + 1, 0);
  // prefill attention: query blocks of qbt tokens (x group heads = 128 rows);
  // split along the keys when the tiles would leave workers idle
  // The split: the smallest whole number of pages (two at least, at most
  // kMaxKeySplits splits) whose tiles still run in one round of the workers,
  // so that the longest query blocks stop being the critical path (a split
  // into more tiles than workers measured slower: 256 against 208 us per
  // layer at batch 1).
  const int qbt = kTokBlock / grp;
  const int n_qb = (T + qbt - 1) / qbt;
  int KS = 0;
  for (int ks = 2 * p.page_tokens; ks < T && !KS; ks += p.page_tokens) {
    int64_t tiles = 0;
    bool fits = true;
    for (int qb = 0; qb < n_qb; ++qb) {
      const int t1 = std::min(T, (qb + 1) * qbt), n = (t1 + ks - 1) / ks;
      if (n > kMaxKeySplits) fits = false;
      tiles += n;
    }
    if (fits && tiles * B * m.n_kv_heads <= dec.W) KS = ks;
  }
  if (KS && (int64_t)B * m.n_kv_heads * n_qb >= dec.W) KS = 0;  // already a round or more without splits
  g->pattn_ks = KS;
  const int s_o = mma_splits(nq * (h / 128), q_rows / 64, p, dec.W);
  const int s_dn = mma_splits(nq * (h / 128), m.ffn / 64, p, dec.W);
  auto krange = [](int nkc, int s, int i, int* c0, int* c1) {
    *c0 = (int)((int64_t)nkc * i / s);
    *c1 = (int)((int64_t)nkc * (i + 1) / s);
  };
  for (int tb = 0; tb < nq; ++tb) add(OP_PEMBED, 0, 0, 0, tb, 0, 0, 0, {blk(BUF_PX, h, tb, 0, h, 1)});
  const uint32_t chunk = kMmaChunkBytes;
  for (int l = 0; l < m.n_layers; ++l) {
    const LayerDev& d = dec.lay.layers[l];
    layer_begin[l] = (uint32_t)Tl.size();
    // RMSNorm tiles of kNormRows rows; the tiles of one block form one write
    auto norms = [&](int which) {
      for (int tb = 0; tb < nq; ++tb)
        for (int r0 = 0; r0 < kTokBlock; r0 += kNormRows)
          add(OP_NORM, l, 0, 0, tb, which, r0, h,
              {blk(BUF_PX, h, tb, 0, h, 0), blk(BUF_PXN, h, tb, 0, h, 1, 100000 + (2 * l + which) * nq + tb)});
    };
    norms(0);
    // QKV: feature blocks of 128 rows; never straddle q/k/v (all multiples of 128)
    for (int tb = 0; tb < nq; ++tb)
      for (int fb = 0; fb < qkv_rows / 128; ++fb) {
        const int f0 = fb * 128;
        std::vector<Access> acc{blk(BUF_PXN, h, tb, 0, h, 0)};
        if (f0 < q_rows)
          acc.push_back(blk(BUF_PQ, q_rows, tb, f0, f0 + 128, 1));
        else
          acc.push_back(kvblk(l, tb, f0 - q_rows, f0 - q_rows + 128, 1));
        add(OP_MQKV, l, d.mma_qkv + (uint64_t)fb * (h / 64) * chunk, (uint32_t)(h / 64) * chunk, fb, tb, 0, h, acc);
      }
    // causal attention: (sequence, kv head, query block), split along the
    // keys into splits of KS keys when those tiles are fewer than the workers
    // (the last split to finish combines them)
    const int attn_group = 2000 + l;
    for (int b = 0; b < B; ++b)
      for (int gi = 0; gi < m.n_kv_heads; ++gi)
        for (int qb = 0; qb * qbt < T; ++qb) {
          const int t0 = qb * qbt, t1 = std::min(T, t0 + qbt);
          const int m0 = b * T + t0, m1 = b * T + t1;  // query rows
          const int n_ks = KS ? (t1 + KS - 1) / KS : 1;
          for (int ks = 0; ks < n_ks; ++ks) {
            const int k0 = ks * KS, k1 = KS ? std::min(t1, k0 + KS) : t1;  // keys [k0, k1)
            std::vector<Access> acc;
            for (int tb = m0 / kTokBlock; tb <= (m1 - 1) / kTokBlock; ++tb) {
              acc.push_back(blk(BUF_PQ, q_rows, tb, gi * grp * hd, (gi + 1) * grp * hd, 0));
              acc.push_back(blk(BUF_PATT, q_rows, tb, gi * grp * hd, (gi + 1) * grp * hd, 1, attn_group));
            }
            for (int tb = (b * T + k0) / kTokBlock; tb <= (b * T + k1 - 1) / kTokBlock; ++tb) {
              acc.push_back(kvblk(l, tb, gi * hd, (gi + 1) * hd, 0));                      // k of head gi
              acc.push_back(kvblk(l, tb, kv_rows + gi * hd, kv_rows + (gi + 1) * hd, 0));  // v of head gi
            }
            add(OP_PATTN, l, 0, 0, b, gi, qb, ks, acc);
          }
        }
    // O and down: split along K when the token blocks alone give too few tiles
    // for the workers; the splits add into X
    for (int tb = 0; tb < nq; ++tb)
      for (int fb = 0; fb < h / 128; ++fb)
        for (int i = 0; i < s_o; ++i) {
          int c0, c1;
          krange(q_rows / 64, s_o, i, &c0, &c1);
          add(OP_MO, l, d.mma_wo + ((uint64_t)fb * (q_rows / 64) + c0) * chunk, (uint32_t)(c1 - c0) * chunk, fb, tb,
              c0 * 64, (c1 - c0) * 64,
              {blk(BUF_PATT, q_rows, tb, c0 * 64, c1 * 64, 0), blk(BUF_PX, h, tb, fb * 128, fb * 128 + 128, 2)});
        }
    norms(1);
    for (int tb = 0; tb < nq; ++tb)
      for (int fb = 0; fb < 2 * m.ffn / 128; ++fb)
        add(OP_MGU, l, d.mma_gu + (uint64_t)fb * (h / 64) * chunk, (uint32_t)(h / 64) * chunk, fb, tb, 0, h,
            {blk(BUF_PXN, h, tb, 0, h, 0), blk(BUF_PH, m.ffn, tb, fb * 64, fb * 64 + 64, 1)});
    for (int tb = 0; tb < nq; ++tb)
      for (int fb = 0; fb < h / 128; ++fb)
        for (int i = 0; i < s_dn; ++i) {
          int c0, c1;
          krange(m.ffn / 64, s_dn, i, &c0, &c1);
          add(OP_MDOWN, l, d.mma_down + ((uint64_t)fb * (m.ffn / 64) + c0) * chunk, (uint32_t)(c1 - c0) * chunk, fb,
              tb, c0 * 64, (c1 - c0) * 64,
              {blk(BUF_PH, m.ffn, tb, c0 * 64, c1 * 64, 0), blk(BUF_PX, h, tb, fb * 128, fb * 128 + 128, 2)});
        }
  }
  layer_begin[m.n_layers] = (uint32_t)Tl.size();
  {
    std::vector<Access> acc{{BUF_XA, 0, h, 1, -1}};
    for (int b = 0; b < B; ++b) acc.push_back(blk(BUF_PX, h, (b * T + T - 1) / kTokBlock, 0, h, 0));
    add(OP_GATHER, m.n_layers, 0, 0, 0, 0, 0, 0, acc);
  }
  // LM head + argmax + publish: GEMV tiles over the gathered last positions
  for (const LmTile& t : gemv_lm_tiles(m, p, dec.W, dec.lay))
    add(OP_LMHEAD, m.n_layers, t.w_off, t.w_bytes, t.r0, t.n, 0, h,
        {{BUF_XA, 0, h, 0, -1}, {BUF_LOGITS, t.r0, t.r0 + t.n, 1, -1}, {BUF_BEST, 0, 1, 2, -1}});
  add(OP_FINAL, m.n_layers, 0, 0, 0, 0, 0, 0, {{BUF_BEST, 0, 1, 0, -1}, {BUF_TOK, 0, 1, 1, -1}});
  g->algo_weight_bytes = wbytes;
  if (Tl.size() >= (1u << 31)) return "too many tiles";

  DataflowBuilder df;
  const int64_t sizes[BUF_COUNT] = {h, h, qkv_rows, q_rows, m.ffn, p.lm_rows, 1, 1,
                                    (int64_t)nq * h * TB, (int64_t)nq * h * TB, (int64_t)nq * q_rows * TB,
                                    (int64_t)m.n_layers * nq * 2 * kv_rows * TB, (int64_t)nq * q_rows * TB,
                                    (int64_t)nq * m.ffn * TB, h, h};
  for (int b = 0; b < BUF_COUNT; ++b) df.bufs.emplace_back(sizes[b]);
  g->preds.assign(Tl.size(), {});
  df.preds_of = &g->preds;
  g->n_edges = 0;
  for (size_t t = 0; t < Tl.size(); ++t) {
    df.apply((int)t, A[t], &g->preds[t]);
    g->n_edges += (int64_t)g->preds[t].size();
  }
  std::unordered_map<std::vector<int>, uint32_t, VecHash> ctr_of;
  std::vector<std::vector<uint32_t>> sig_of(Tl.size());
  g->ctr_need.clear();
  for (size_t t = 0; t < Tl.size(); ++t) {
    const auto& P = g->preds[t];
    if (P.empty()) continue;
    auto it = ctr_of.find(P);
    uint32_t c;
    if (it == ctr_of.end()) {
      c = (uint32_t)g->ctr_need.size();
      ctr_of.emplace(P, c);
      g->ctr_need.push_back((uint32_t)P.size());
      for (int u : P) sig_of[u].push_back(c);
    } else {
      c = it->second;
    }
    Tl[t].wait_ctr = c;
    Tl[t].need = g->ctr_need[c];
  }
  g->sig.clear();
  for (size_t t = 0; t < Tl.size(); ++t) {
    Tl[t].sig_off = (uint32_t)g->sig.size();
    Tl[t].sig_cnt = (uint32_t)sig_of[t].size();
    g->sig.insert(g->sig.end(), sig_of[t].begin(), sig_of[t].end());
  }
  g->region_begin.assign(1, 0);
  for (int r = 1; r < p.n_regions; ++r) g->region_begin.push_back(layer_begin[p.region_cut[r]]);
  g->region_begin.push_back((uint32_t)Tl.size());
  g->plan.per_op_slot = dec.plan.per_op_slot;
  return "";
}

// ---------------------------------------------------------------------------
std::string verify_graph(const CompiledGraph& g) {
  const size_t n = g.tiles.size();
  if (n > 20000) return "graph too large for the quadratic verifier";
  // topological ticket order and counter consistency
  std::vector<std::vector<int>> signalers(g.ctr_need.size());
  for (size_t t = 0; t < n; ++t) {
    for (int u : g.preds[t])
      if (u >= (int)t) return fmt("edge %lld -> %lld goes backwards in ticket order", u, (long long)t);
    const Tile& T = g.tiles[t];
    for (uint32_t i = 0; i < T.sig_cnt; ++i) signalers[g.sig[T.sig_off + i]].push_back((int)t);
  }
  const bool teams = !g.worker_of.empty();
  for (size_t t = 0; t < n; ++t) {
    const Tile& T = g.tiles[t];
    if (teams) {
      // every predecessor is on the tile's own worker (stream order) or is
      // covered by a signaller of its counter: a tile of the predecessor's
      // worker and op group at or after it in ticket order
      const std::vector<int> none;
      const auto& S = T.wait_ctr == kNoCounter ? none : signalers[T.wait_ctr];
      if (T.wait_ctr != kNoCounter && T.need != S.size())
        return fmt("tile %lld need %lld != signal count", (long long)t, T.need);
      for (int u : g.preds[t]) {
        if (g.worker_of[u] == g.worker_of[t]) continue;
        bool covered = false;
        for (int x : S)
          if (x >= u && x < (int)t && g.worker_of[x] == g.worker_of[u] && g.tiles[x].op == g.tiles[u].op &&
              g.tiles[x].layer == g.tiles[u].layer)
            covered = true;
        if (!covered) return fmt("team schedule: edge %lld -> %lld is not signalled", u, (long long)t);
      }
      continue;
    }
    if (g.preds[t].empty()) {
      if (T.wait_ctr != kNoCounter) return fmt("tile %lld waits without predecessors", (long long)t);
      continue;
    }
    if (T.wait_ctr == kNoCounter) return fmt("tile %lld has predecessors but no counter", (long long)t);
    const auto& S = signalers[T.wait_ctr];
    if (S != g.preds[t]) return fmt("counter %lld of tile %lld: signalers != predecessors", T.wait_ctr, (long long)t);
    if (T.need != S.size()) return fmt("tile %lld need %lld != signal count", (long long)t, T.need);
  }
  // reachability bitsets
  const size_t W = (n + 63) / 64;
  std::vector<uint64_t> anc(n * W, 0);
  for (size_t t = 0; t < n; ++t) {
    uint64_t* a = &anc[t * W];
    auto add = [&](int u) {
      const uint64_t* b = &anc[(size_t)u * W];
      for (size_t i = 0; i < W; ++i) a[i] |= b[i];
      a[u / 64] |= 1ull << (u % 64);
    };
    for (int u : g.preds[t]) add(u);
    // team schedule: the tile before t in its worker's stream ran first
    if (!g.stream_prev.empty() && g.stream_prev[t] >= 0) add(g.stream_prev[t]);
  }
  auto reach = [&](int u, int v) { return (anc[(size_t)v * W + u / 64] >> (u % 64)) & 1; };
  // every conflicting access pair must be ordered by a path
  struct Acc { int t; int64_t lo, hi; int kind, group; };
  std::vector<std::vector<Acc>> per(BUF_COUNT);
  for (size_t t = 0; t < n; ++t)
    for (auto& a : g.access[t]) per[a.buf].push_back({(int)t, a.lo, a.hi, a.kind, a.group});
  for (int b = 0; b < BUF_COUNT; ++b) {
    const auto& v = per[b];
    for (size_t i = 0; i < v.size(); ++i)
      for (size_t j = i + 1; j < v.size(); ++j) {
        const Acc &x = v[i], &y = v[j];
        if (x.t == y.t) continue;
        if (x.hi <= y.lo || y.hi <= x.lo) continue;
        if (x.kind == 0 && y.kind == 0) continue;
        if (x.kind == 2 && y.kind == 2) continue;
        if (x.kind == 1 && y.kind == 1 && x.group >= 0 && x.group == y.group) continue;
        if (!reach(x.t, y.t))
          return fmt("unordered conflicting accesses: tile %lld and tile %lld (buffer %lld)", x.t, y.t, b);
      }
  }
  return "";
}

// ---------------------------------------------------------------------------
// Host threads standing in for workers: the same ticket queue, counter targets
// (need x epoch, counters never reset) and signals, with random delays.
int simulate_graph(const CompiledGraph& g, int n_threads, int n_epochs, uint64_t seed, int wait_ms,
                   int stuck_tile, int32_t* done_order, std::string* msg) {
  const uint64_t T = g.tiles.size();
  const uint64_t total = T * (uint64_t)n_epochs;
  std::vector<std::atomic<uint32_t>> ctr(g.ctr_need.size());
  for (auto& c : ctr) c.store(0);
  std::atomic<uint64_t> head{0}, done_idx{0};
  std::atomic<uint32_t> epochs_done{0};  // the doorbell: step e starts after step e-1 completed
  std::atomic<int> failed{0};
  std::atomic<uint64_t> fail_tile{0};
  const bool static_sched = g.plan.schedule == WPK_SCHED_STATIC;
  const bool teams = g.plan.schedule == WPK_SCHED_TEAMS && !g.stream.empty();
  if (teams && n_threads != (int)g.stream_begin.size() - 1) {
    *msg = "the team schedule simulates exactly its compiled workers";
    return WPK_ERR_INVALID_ARG;
  }
  auto worker = [&](int wid) {
    std::mt19937_64 rng(seed * 1000003ull + wid);
    for (uint64_t i = 0;; ++i) {
      if (failed.load()) return;
      uint64_t t;
      if (teams) {  // the worker's own stream, epoch after epoch
        const uint64_t len = g.stream_begin[wid + 1] - g.stream_begin[wid];
        if (len == 0 || i >= len * (uint64_t)n_epochs) return;
        t = (i / len) * T + g.stream[g.stream_begin[wid] + i % len];
      } else {
        t = static_sched ? wid + i * (uint64_t)n_threads : head.fetch_add(1);
      }
      if (t >= total) return;
      uint32_t e = (uint32_t)(t / T) + 1;
      const Tile& tile = g.tiles[t % T];
      {
        auto t0 = std::chrono::steady_clock::now();
        while (epochs_done.load(std::memory_order_acquire) + 1 < e) {
          if (failed.load()) return;
          std::this_thread::yield();
          if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(wait_ms)) {
            failed.store(1);
            fail_tile.store(t % T);
            return;
          }
        }
      }
      if (tile.wait_ctr != kNoCounter) {
        uint64_t target = (uint64_t)tile.need * e;
        auto t0 = std::chrono::steady_clock::now();
        while (ctr[tile.wait_ctr].load(std::memory_order_acquire) < target) {
          if (failed.load()) return;
          std::this_thread::yield();
          if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(wait_ms)) {
            failed.store(1);
            fail_tile.store(t % T);
            return;
          }
        }
      }
      if (rng() % 8 == 0) std::this_thread::sleep_for(std::chrono::microseconds(rng() % 50));
      uint64_t d = done_idx.fetch_add(1);
      if (done_order && d < total) done_order[d] = (int32_t)(t % T);
      if ((int64_t)(t % T) == stuck_tile) continue;
      for (uint32_t i = 0; i < tile.sig_cnt; ++i)
        ctr[g.sig[tile.sig_off + i]].fetch_add(1, std::memory_order_release);
      if (t % T == T - 1) epochs_done.fetch_add(1, std::memory_order_release);
    }
  };
  std::vector<std::thread> th;
  for (int i = 0; i < n_threads; ++i) th.emplace_back(worker, i);
  for (auto& x : th) x.join();
  if (failed.load()) {
    *msg = fmt("simulated worker timed out waiting before tile %lld", (long long)fail_tile.load());
    return WPK_ERR_TIMEOUT;
  }
  return WPK_OK;
}

// Tensor-core image of a [rows][K] bf16 matrix: blocks of 128 rows x 64
// columns (16 KB), block (r / 128, c / 64) at ((r / 128) * K / 64 + c / 64) *
// 16 KB, the 16-byte unit u of row r stored at unit u XOR (r % 8); rows past
// `rows` in the last block stay as the caller initialised them.
void arrange_mma_image(uint8_t* base, int K, int rows, const uint16_t* src) {
  const int nkc = K / 64;
  for (int r = 0; r < rows; ++r) {
    uint8_t* blk0 = base + (uint64_t)(r / 128) * nkc * kMmaChunkBytes;
    const int rr = r % 128;
    for (int c = 0; c < nkc; ++c)
      for (int u = 0; u < 8; ++u)
        memcpy(blk0 + (uint64_t)c * kMmaChunkBytes + rr * 128 + ((u ^ (rr & 7)) * 16),
               src + (uint64_t)r * K + c * 64 + u * 8, 16);
  }
}

// ---------------------------------------------------------------------------
// Weight image: fp32 norm gains; QKV rows permuted so that RoPE pair rows
// (i, i + d/2) of every q/k head sit next to each other; gate/up rows
// interleaved (gate j, up j); down projection stored K-chunk-major.
std::string arrange_weights(const CompiledGraph& g, const wpk_weights& w, uint8_t* img) {
  const wpk_model_cfg& m = g.m;
  const int h = m.hidden, hd = m.head_dim;
  const int q_rows = m.n_heads * hd, kv_rows = m.n_kv_heads * hd;
  // (a two-stage head has no token embedding, and its output heads live
  // outside this decoder's image: both pointers may then be NULL)
  if (!w.final_norm || !w.layers || (m.tied_embedding && !w.embed)) return "missing weight pointer";
  auto gain = [&](const uint16_t* src, uint64_t off) {
    float* dst = reinterpret_cast<float*>(img + off);
    for (int i = 0; i < h; ++i) {
      uint32_t u = (uint32_t)src[i] << 16;
      memcpy(&dst[i], &u, 4);
    }
  };
  auto row = [&](const uint16_t* src, uint64_t dst_off, int64_t dst_row, int64_t src_row, int cols) {
    memcpy(img + dst_off + (uint64_t)dst_row * cols * 2, src + (uint64_t)src_row * cols, (size_t)cols * 2);
  };
  auto rope_phys = [&](int logical) {  // within a head
    int i = logical % hd, head = logical / hd, half = hd / 2;
    return head * hd + (i < half ? 2 * i : 2 * (i - half) + 1);
  };
  std::vector<std::thread> th;
  std::string err;
  for (int l = 0; l < m.n_layers; ++l) {
    const wpk_layer_weights& W = w.layers[l];
    if (!W.attn_norm || !W.wq || !W.wk || !W.wv || !W.wo || !W.ffn_norm || !W.w_gate || !W.w_up || !W.w_down)
      return fmt("missing weight pointer in layer %lld", l);
  }
  // tensor-core image: block (r / 128, c / 64) of 128 rows x 64 columns, the
  // 16-byte unit u of row r stored at unit index u XOR (r % 8)
  auto mma_row = [&](uint64_t base, int K, int r, const uint16_t* src_row) {
    const int nkc = K / 64;
    uint8_t* blk0 = img + base + (uint64_t)(r / 128) * nkc * kMmaChunkBytes;
    const int rr = r % 128;
    for (int c = 0; c < nkc; ++c)
      for (int u = 0; u < 8; ++u)
        memcpy(blk0 + (uint64_t)c * kMmaChunkBytes + rr * 128 + ((u ^ (rr & 7)) * 16), src_row + c * 64 + u * 8, 16);
  };
  auto do_layer = [&](int l) {
    const wpk_layer_weights& W = w.layers[l];
    const LayerDev& d = g.lay.layers[l];
    if (g.lay.mma) {
      for (int r = 0; r < q_rows; ++r) mma_row(d.mma_qkv, h, rope_phys(r), W.wq + (uint64_t)r * h);
      for (int r = 0; r < kv_rows; ++r) mma_row(d.mma_qkv, h, q_rows + rope_phys(r), W.wk + (uint64_t)r * h);
      for (int r = 0; r < kv_rows; ++r) mma_row(d.mma_qkv, h, q_rows + kv_rows + r, W.wv + (uint64_t)r * h);
      for (int r = 0; r < h; ++r) mma_row(d.mma_wo, q_rows, r, W.wo + (uint64_t)r * q_rows);
      for (int j = 0; j < m.ffn; ++j) {
        mma_row(d.mma_gu, h, 2 * j, W.w_gate + (uint64_t)j * h);
        mma_row(d.mma_gu, h, 2 * j + 1, W.w_up + (uint64_t)j * h);
      }
      for (int r = 0; r < h; ++r) mma_row(d.mma_down, m.ffn, r, W.w_down + (uint64_t)r * m.ffn);
    }
    gain(W.attn_norm, d.attn_norm);
    gain(W.ffn_norm, d.ffn_norm);
    for (int r = 0; r < q_rows; ++r) row(W.wq, d.qkv, rope_phys(r), r, h);
    for (int r = 0; r < kv_rows; ++r) row(W.wk, d.qkv, q_rows + rope_phys(r), r, h);
    for (int r = 0; r < kv_rows; ++r) row(W.wv, d.qkv, q_rows + kv_rows + r, r, h);
    memcpy(img + d.wo, W.wo, (size_t)h * q_rows * 2);
    for (int j = 0; j < m.ffn; ++j) {
      row(W.w_gate, d.gu, 2 * j, j, h);
      row(W.w_up, d.gu, 2 * j + 1, j, h);
    }
    const int kc = g.lay.down_kc;
    uint16_t* dd = reinterpret_cast<uint16_t*>(img + d.down);
    for (int c = 0; c < g.lay.n_down_chunks; ++c)
      for (int r = 0; r < h; ++r)
        memcpy(dd + ((uint64_t)c * h + r) * kc, W.w_down + (uint64_t)r * m.ffn + (uint64_t)c * kc, (size_t)kc * 2);
  };
  // the LM head's tensor-core image (batched decode), in 16 row slices per task
  const uint16_t* lm_src = m.tied_embedding ? w.embed : w.lm_head;
  const int lm_tasks = (g.lay.lm_mma && lm_src) ? 16 : 0;
  auto do_lm = [&](int i) {
    const int rows = g.plan.lm_rows;
    const int r0 = (int)((int64_t)rows * i / lm_tasks), r1 = (int)((int64_t)rows * (i + 1) / lm_tasks);
    for (int r = r0; r < r1; ++r) mma_row(g.lay.lm_mma, h, r, lm_src + (uint64_t)r * h);
  };
  unsigned nt = std::max(1u, std::min(16u, std::thread::hardware_concurrency()));
  std::atomic<int> next{0};
  for (unsigned i = 0; i < nt; ++i)
    th.emplace_back([&] {
      for (int l; (l = next.fetch_add(1)) < m.n_layers + lm_tasks;) {
        if (l < m.n_layers)
          do_layer(l);
        else
          do_lm(l - m.n_layers);
      }
    });
  gain(w.final_norm, g.lay.final_norm);
  if (w.embed) memcpy(img + g.lay.embed, w.embed, (size_t)m.vocab * h * 2);
  if (!m.tied_embedding && w.lm_head) memcpy(img + g.lay.lm_head, w.lm_head, (size_t)g.plan.lm_rows * h * 2);
  for (auto& x : th) x.join();
  return "";
}

}  // namespace wpk
