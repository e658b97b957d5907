// Composition planner: predicts the time of one program (a decode step or a
// prefill) under a candidate composition - one persistent launch, 2-4
// persistent region launches, or conventional per-op launches - without
// running the candidate ("One Megakernel is Not Enough", abstract and plain-
// language summary: rank candidate compositions by simulating their tile and
// event graphs from existing measurements).
//
// The model follows that paper's Table I, one row at a time:
//   * cross-kernel readiness (tile graph): inside a persistent launch a tile
//     waits only for its tile-to-tile predecessors (the compiled edges), not
//     for whole preceding ops;
//   * weight prefetch (tile graph): every worker has `slots` staging slots; a
//     tile's weight load is issued as soon as a slot is free - while its
//     predecessors still run - and its compute still waits for them
//     (slots = 1 is the paper's one-slot rule);
//   * on-chip forwarding (node weights): already inside the measured tile
//     service times, whose tiles never store the forwarded tensors;
//   * fewer launches, internal synchronization (event graph): a dispatch
//     node of `dispatch_ns` before every launch, and `sync_ns` added to a
//     tile's ready time for each counter wait inside a persistent launch;
//   * smaller CTA budget (service table): a conventional launch of g CTAs on
//     n_sms SMs runs in ceil(g / n_sms) waves; a persistent region runs on
//     n_workers workers.
//
// Inputs are per-tile service times (ns): in practice the measured busy time
// of each tile in a traced persistent run, plus a load time per tile from its
// staged weight bytes and a per-worker bandwidth.
#include <algorithm>
#include <cmath>
#include <string>
#include <vector>

#include "graph.h"

namespace wpk {

namespace {

// One worker's pipeline state in a persistent launch.
struct WorkerState {
  double load_free = 0.0;          // when its loader can issue the next tile's copies
  double comp_free = 0.0;          // when its compute warps are free
  std::vector<double> slot_free;   // per staging slot: when the tile held there finished
  size_t next_slot = 0;
};

// First ticket of layer `l` (the first op group of that layer), or the end.
uint32_t layer_first_ticket(const CompiledGraph& g, int l) {
  for (const OpGroup& og : g.groups)
    if (og.layer >= l && og.op != OP_EMBED && og.op != OP_PEMBED) return og.begin;
  return (uint32_t)g.tiles.size();
}

}  // namespace

std::string predict_program(const CompiledGraph& g, const double* service_ns, const double* load_ns,
                            const PredictCfg& c, double* out_ns) {
  const size_t T = g.tiles.size();
  if (T == 0) return "empty program";
  if (c.n_workers <= 0 || c.n_sms <= 0 || c.slots <= 0) return "workers, SMs and slots must be positive";
  for (size_t t = 0; t < T; ++t)
    if (!(service_ns[t] >= 0.0) || !(load_ns[t] >= 0.0)) return "service and load times must be >= 0";
  std::vector<double> done(T, 0.0);
  double clock = 0.0;  // the stream: when the previous launch completed
  if (c.mode == WPK_PER_OP_GRAPH) {
    // conventional launches: one per op group, its tiles as CTAs over the SMs
    // in waves (the next CTA takes the SM that frees first); no prefetch
    // across tiles, no counters (stream order replaces them)
    for (const OpGroup& og : g.groups) {
      clock += c.dispatch_ns;
      std::vector<double> sm(std::min<size_t>((size_t)c.n_sms, og.end - og.begin), clock);
      double end = clock;
      for (uint32_t t = og.begin; t < og.end; ++t) {
        auto it = std::min_element(sm.begin(), sm.end());
        const double start = *it;
        const double fin = std::max(start + c.first_chunk_ns + service_ns[t], start + load_ns[t]);
        *it = fin;
        done[t] = fin;
        end = std::max(end, fin);
      }
      clock = end;
    }
    *out_ns = clock;
    return "";
  }
  if (c.mode != WPK_MEGAKERNEL) return "bad mode";
  // persistent launches over contiguous ticket ranges cut at layer boundaries
  const int R = std::max(1, c.n_regions);
  if (R > 4) return "at most 4 regions";
  std::vector<uint32_t> begin;
  begin.push_back(0);
  for (int r = 1; r < R; ++r) {
    if (c.region_cut[r] <= c.region_cut[r - 1] || c.region_cut[r] > g.m.n_layers) return "bad region cuts";
    begin.push_back(layer_first_ticket(g, c.region_cut[r]));
  }
  begin.push_back((uint32_t)T);
  for (int r = 0; r < R; ++r) {
    const uint32_t b = begin[r], e = begin[r + 1];
    clock += c.dispatch_ns;
    const double launch = clock;
    const int W = c.n_workers;
    std::vector<WorkerState> ws(W);
    for (auto& w : ws) {
      w.load_free = w.comp_free = launch;
      w.slot_free.assign(c.slots, launch);
    }
    // ticket -> worker: static streams (w, w + W, ...) or the queue (the
    // worker whose slot frees first claims the next ticket)
    double end = launch;
    for (uint32_t t = b; t < e; ++t) {
      int w;
      if (c.schedule == WPK_SCHED_TEAMS && !g.worker_of.empty()) {
        w = g.worker_of[t] % W;  // the compiled team streams
      } else if (c.schedule == WPK_SCHED_STATIC) {
        w = (int)((t - b) % (uint32_t)W);
      } else {
        w = 0;
        double best = 1e300;
        for (int i = 0; i < W; ++i) {
          const double f = std::max(ws[i].load_free, ws[i].slot_free[ws[i].next_slot]);
          if (f < best) {
            best = f;
            w = i;
          }
        }
      }
      WorkerState& S = ws[w];
      // weight load: as soon as the loader and a slot are free
      const double load_start = std::max(S.load_free, S.slot_free[S.next_slot]);
      const double load_end = load_start + load_ns[t];
      S.load_free = load_end;
      // ready: every predecessor done (earlier regions finished at launch)
      double ready = launch;
      bool waits = false;
      for (int32_t u : g.preds[t])
        if ((uint32_t)u >= b) {
          ready = std::max(ready, done[u]);
          waits = true;
        }
      if (waits) ready += c.sync_ns;
      const double start = std::max(std::max(ready, S.comp_free), load_start + c.first_chunk_ns);
      const double fin = std::max(start + service_ns[t], load_end);
      done[t] = fin;
      S.comp_free = fin;
      S.slot_free[S.next_slot] = fin;
      S.next_slot = (S.next_slot + 1) % S.slot_free.size();
      end = std::max(end, fin);
    }
    clock = end;
  }
  *out_ns = clock;
  return "";
}

}  // namespace wpk
