// Host graph compiler: turns a decoder shape + plan into the step program
// (tiles in ticket order, dependency counters, signal lists, regions) and the
// layout of the arranged weight image.
#pragma once
#include <string>
#include <vector>

#include "wpk_internal.h"

namespace wpk {

struct Plan {
  int max_batch, max_context, page_tokens, n_workers, workers_per_sm, mode, resident, n_regions;
  int region_cut[4];
  int trace;
  uint64_t wait_timeout_ns;
  int slot_bytes, tile_bytes, split_pages, lookahead, schedule;
  int act_bytes;        // activation staging per worker (fp32)
  int prefill_mode;     // 1 = tensor-core prefill program, 2 = token by token
  int per_op_slot;      // ring bytes of a per-op CTA (holds one whole tile)
  int decode_mode;      // WPK_DECODE_GEMV or WPK_DECODE_MMA (resolved)
  // batched decode program: MMA N (max_batch rounded up to 16), its ring
  // stage (16 KB of weights + hi/lo activation chunks), stages, scratch bytes
  int dec_n, dec_stage_bytes, dec_stages, dec_act_bytes;
  int dec_cps;          // K chunks per ring stage of the batched decode tiles (1 or 2)
  int lm_rows;          // rows of the output head (0 = vocab; the two-stage backbone's is its projection)
};

struct Layout {
  std::vector<LayerDev> layers;
  uint64_t final_norm = 0, embed = 0, lm_head = 0;
  uint64_t total = 0;
  int down_kc = 0, n_down_chunks = 0;
  bool mma = false;     // tensor-core image present
  uint64_t lm_mma = 0;  // tensor-core image of the LM head (batched decode only)
  int vocab_blocks = 0; // 128-row blocks of that image (last one zero-padded)
};

struct CompiledGraph {
  wpk_model_cfg m{};
  Plan plan{};
  Layout lay;
  std::vector<Tile> tiles;                    // ticket order
  std::vector<std::vector<Access>> access;    // per tile (for the verifier)
  std::vector<std::vector<int32_t>> preds;    // expanded tile edges
  std::vector<uint32_t> sig;                  // concatenated signal lists
  std::vector<uint32_t> ctr_need;             // per counter
  std::vector<OpGroup> groups;                // op groups in ticket order
  std::vector<uint32_t> region_begin;         // n_regions + 1 ticket boundaries
  int64_t n_edges = 0;
  int64_t algo_weight_bytes = 0;              // weight bytes a step reads
  int n_splits = 0, split_tokens = 0, max_blocks = 0;
  int B = 0, T = 0, M = 0, n_tb = 0;  // prefill programs
  int W = 0;                          // workers the tiles were sized for
  int o_splits = 0, down_splits = 0;  // batched decode: K splits of O and down
  int pattn_ks = 0;                   // prefill: keys per attention split (0 = none)
  // team schedule: each tile's worker, every worker's stream of tickets
  // (stream_begin[w] .. stream_begin[w + 1] in `stream`), and each tile's
  // predecessor in its worker's stream (-1 for the first), an implicit edge
  std::vector<int32_t> worker_of;
  std::vector<uint32_t> stream_begin, stream;
  std::vector<int32_t> stream_prev;
};

// Returns "" on success, else an error message; *code receives the WPK code.
std::string normalize_plan(const wpk_model_cfg& m, const wpk_plan_cfg& in, Plan* out, int* code);
// W: number of worker CTAs the program will run on (tiles are sized so each
// worker gets about one tile per op).
std::string compile_graph(const wpk_model_cfg& m, const Plan& p, CompiledGraph* g, int* code, int W);
// Prefill program for B sequences of T prompt tokens, over the decode graph's
// weight layout (which must include the tensor-core image).
std::string compile_prefill_graph(const CompiledGraph& dec, int B, int T, CompiledGraph* g);
std::string verify_graph(const CompiledGraph& g);
int simulate_graph(const CompiledGraph& g, int n_threads, int n_epochs, uint64_t seed, int wait_ms,
                   int stuck_tile, int32_t* done_order, std::string* msg);
// Composition planner (planner.cpp): predicted time of one run of program g
// under composition c from per-tile service and load times (ns).
using PredictCfg = wpk_predict_cfg;
std::string predict_program(const CompiledGraph& g, const double* service_ns, const double* load_ns,
                            const PredictCfg& c, double* out_ns);
// Arrange host bf16 weights into the image (host buffer of lay.total bytes).
std::string arrange_weights(const CompiledGraph& g, const wpk_weights& w, uint8_t* image);
// Tensor-core image of one [rows][K] bf16 matrix (see graph.cpp).
void arrange_mma_image(uint8_t* base, int K, int rows, const uint16_t* src);

}  // namespace wpk
