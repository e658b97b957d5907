// C ABI of the persistent decode library (declared in include/wpk.h).
//
// Host side of the runtime: device tables, launches per step (cooperative
// persistent grid per region, or per-op launches captured once into a CUDA
// Graph and replayed), prompt prefill, error word and trace access.
#include <map>
#include <mutex>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <thread>
#include <cstring>
#include <memory>
#include <string>
#include <vector>

#include "graph.h"

namespace wpk {
size_t worker_smem_bytes(int n_stages, int stage_bytes, int act_bytes);
const void* persistent_kernel_ptr(bool mma);  // decode on tensor cores (mma) or CUDA cores
const void* per_op_kernel_ptr(bool mma);
const void* prefill_kernel_ptr();
int cta_threads(const void* fn);
const void* prefill_op_kernel_ptr();
}  // namespace wpk

using namespace wpk;

struct GraphEntry {
  const void* key0;  // decode: out_tok; prefill: tokens
  const void* key1;  // decode: logits;  prefill: first_tok
  const void* key2;  // prefill: logits
  cudaGraph_t graph;
  cudaGraphExec_t exec;
};

// A prefill program compiled for (B, T), with its own device tables.
struct PrefillProgram {
  CompiledGraph g;
  uint8_t* d_base = nullptr;
  Tile* d_tiles = nullptr;
  uint32_t* d_sig = nullptr;
  uint32_t* d_ctr = nullptr;
  TraceRec* d_trace = nullptr;
  std::vector<GraphEntry> graphs;
};

struct wpk_handle {
  CompiledGraph g;
  int device = 0, n_sms = 0, n_workers = 0;
  size_t smem = 0, smem_per_op = 0;
  // library-owned device tables (one allocation)
  uint8_t* d_base = nullptr;
  Tile* d_tiles = nullptr;
  uint32_t* d_sig = nullptr;
  uint32_t* d_ctr = nullptr;
  uint32_t* d_head = nullptr;
  ErrWord* d_err = nullptr;
  TraceRec* d_trace = nullptr;
  uint32_t* d_evclock = nullptr;
  LayerDev* d_layers = nullptr;
  float2* d_rope = nullptr;
  int32_t* d_block_table = nullptr;
  uint32_t* d_arrive = nullptr;
  uint32_t* d_rb_arrive = nullptr;  // batched decode: split arrivals per O / down row block
  ResDev* d_res = nullptr;          // resident grid: device copy of the doorbell
  unsigned long long* d_best = nullptr;
  int32_t* d_seqlen = nullptr;
  int32_t* d_tok_fb = nullptr;
  int32_t* d_active = nullptr;
  int32_t* d_slot_active = nullptr;  // [max_batch] slot mask (nonzero = stepped)
  uint32_t* d_pattn_arrive = nullptr;  // prefill key-split attention: arrivals per tile
  uint32_t* d_stream_begin = nullptr;  // team schedule: worker streams
  uint32_t* d_stream = nullptr;
  // fixed-cohort serving (wpk_prefill_slots): every slot of the plan is
  // stepped, the mask says which are live; host mirrors of each slot's cached
  // tokens and mask
  bool cohort = false;
  std::vector<int> slot_len;
  std::vector<char> slot_on;
  int32_t cohort_batch = 0;          // stable source of an asynchronous copy
  int prefill_slot0 = 0;             // first slot of the prefill being launched
  int32_t* h_err_code = nullptr;  // pinned mirror of d_err->code
  // caller-owned buffers
  uint8_t* weights = nullptr;
  uint16_t* kv = nullptr;
  uint8_t* scratch = nullptr;
  size_t kv_bytes = 0, scratch_bytes = 0;
  // the part of the scratch a GEMV decode step touches (its buffers are laid
  // out first; prefill and tensor-core regions follow)
  size_t decode_scratch_bytes = 0;
  size_t off_xa = 0, off_xb = 0, off_q = 0, off_attn = 0, off_h = 0, off_part = 0;
  // batched decode program: residual (feature-major), q/k/v sums, x^2 sums,
  // hi/lo images of x*g_attn, x*g_ffn, the attention output and h
  size_t off_xt = 0, off_acc = 0, off_ss = 0, off_dimg[4] = {};
  int64_t n_blocks = 0;
  bool loaded = false, prefilled = false, poisoned = false, has_device = false;
  int batch = 0, ctx = 0;
  std::vector<GraphEntry> graphs;
  cudaStream_t capture_stream = nullptr;
  std::string err;
  // prefill programs and their scratch (offsets in the caller's scratch)
  std::vector<std::unique_ptr<PrefillProgram>> prefills;
  size_t off_px = 0, off_pq = 0, off_xn = 0, off_att = 0, off_hi = 0, off_ppart = 0;
  int64_t prefill_max_tokens = 0;
  int prefill_stages = 0;
  int prefill_cps = 1;  // K chunks per prefill ring stage
  size_t smem_prefill = 0;
  // program the inspection calls refer to (nullptr = the decode program)
  PrefillProgram* selected = nullptr;
  // resident grid: control block in mapped host memory, its own stream
  ResCtl* res_ctl = nullptr;      // host view
  ResCtl* res_ctl_dev = nullptr;  // device view
  cudaStream_t res_stream = nullptr;
  bool res_live = false;
  uint32_t res_epoch = 0;         // last step rung on the live grid
  std::chrono::steady_clock::time_point res_last;
  // per-launch step I/O overrides (the two-stage composition)
  struct IO {
    bool set = false;
    int n_in = 1, in_rows = 0, logits_stride = 0, out_stride = 1;
    uint64_t in_off[kMaxInTables] = {};
    const float* in_vec = nullptr;
    uint64_t lm_head_off = 0, lm_mma_off = 0;
  } io;
  // two-stage model: the head decoder and the tables outside both decoders
  wpk_handle* head = nullptr;
  int n_cb = 0, cb_vocab = 0;
  uint64_t head_base = 0, weights_total = 0;  // head image offset; whole image
  std::vector<uint64_t> frame_embed_off, head_embed_off, out_head_off, out_head_mma_off;
  size_t off_p = 0, off_codes = 0;  // scratch: projection output [B][head hidden], last codes [B][K]
  // chunked two-stage frame: this handle is chunk 0's backbone; `chunks` holds
  // the (backbone + head) pairs of chunks 1.., all over this handle's weights
  std::vector<wpk_handle*> chunks;
  int chunk_rows = 0;                   // sequences per chunk
  cudaStream_t head_stream = nullptr;   // the heads' stream
  // a chunk pair's programs run beside another persistent launch: a
  // cooperative launch may then be refused, so they launch as plain grids
  // (backbone + head workers fit the SMs together, one CTA per SM)
  bool plain_launch = false;
  int per_sm = 0, per_sm_prefill = 0;  // co-resident workers an SM holds (decode, prefill programs)
  std::vector<cudaEvent_t> chunk_ev;    // [0] fork, [1] join, [2 + c] backbone of chunk c done
};

namespace {

thread_local std::string g_build_error;  // message of the last failed wpk_build_graph

int fail(wpk_handle* h, int code, const std::string& msg) {
  if (h) h->err = msg;
  return code;
}

#define CUDA_TRY(h, call)                                                                  \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess)                                                                 \
      return fail(h, WPK_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

size_t a256(size_t x) { return (x + 255) / 256 * 256; }

int check_live(wpk_handle* h) {
  if (!h) return WPK_ERR_INVALID_ARG;
  if (!h->has_device) {
    h->err = "no CUDA device: host-only handle";
    return WPK_ERR_CUDA;
  }
  auto dev_err = [](const wpk_handle* x) {
    return x && x->h_err_code && *(volatile int32_t*)x->h_err_code != 0;
  };
  bool any = dev_err(h) || dev_err(h->head);
  for (const wpk_handle* c : h->chunks) any = any || dev_err(c) || dev_err(c->head);
  if (!h->poisoned && any) {
    h->poisoned = true;
    h->err = "device program reported an error (see wpk_get_error_info)";
  }
  if (h->poisoned) return WPK_ERR_POISONED;
  return WPK_OK;
}

// Tensor-core accumulators: a tile's buffer holds up to 4 accumulators of 2N
// columns; a worker holds two buffers within the 512 TMEM columns of an SM
// (one worker CTA per SM when its buffers take all 512).
void set_mma_geometry(KParams* P) {
  const int w = 2 * P->mma_n;
  P->mma_acc = std::max(1, std::min(4, 256 / w));
  P->mma_buf_cols = w * P->mma_acc;
  int cols = 32;
  while (cols < 2 * P->mma_buf_cols) cols <<= 1;
  P->tmem_cols = cols;
}

KParams make_params(const wpk_handle* h) {
  const CompiledGraph& g = h->g;
  const wpk_model_cfg& m = g.m;
  KParams P{};
  P.n_layers = m.n_layers;
  P.hidden = m.hidden;
  P.n_heads = m.n_heads;
  P.n_kv = m.n_kv_heads;
  P.head_dim = m.head_dim;
  P.ffn = m.ffn;
  P.vocab = m.vocab;
  P.group = m.n_heads / m.n_kv_heads;
  P.q_rows = m.n_heads * m.head_dim;
  P.kv_rows = m.n_kv_heads * m.head_dim;
  P.qkv_rows = P.q_rows + 2 * P.kv_rows;
  P.down_kc = g.lay.down_kc;
  P.n_down_chunks = g.lay.n_down_chunks;
  P.eps = m.rms_eps;
  P.max_batch = g.plan.max_batch;
  P.max_context = g.plan.max_context;
  P.page_tokens = g.plan.page_tokens;
  P.max_blocks = g.max_blocks;
  P.split_tokens = g.split_tokens;
  P.n_splits = g.n_splits;
  P.gemv_cps = gemv_chunks_per_stage(g.plan.slot_bytes);
  P.stage_bytes = P.gemv_cps * kStageBytes;
  P.n_stages = g.plan.slot_bytes / P.stage_bytes;
  P.lookahead = g.plan.lookahead;
  P.act_bytes = g.plan.act_bytes;
  P.timeout_ns = g.plan.wait_timeout_ns;
  P.trace = g.plan.trace;
  P.weights = h->weights;
  P.layers = h->d_layers;
  P.final_norm_off = g.lay.final_norm;
  P.embed_off = g.lay.embed;
  P.lm_head_off = g.lay.lm_head;
  P.lm_rows = g.plan.lm_rows;
  P.logits_stride = g.plan.lm_rows;
  P.out_stride = 1;
  P.n_in = 1;
  P.in_rows = m.vocab;
  P.in_table_off[0] = g.lay.embed;
  P.in_vec = nullptr;
  P.kv = h->kv;
  P.n_blocks = h->n_blocks;
  P.block_table = h->d_block_table;
  P.rope = h->d_rope;
  P.xa = reinterpret_cast<float*>(h->scratch + h->off_xa);
  P.xb = reinterpret_cast<float*>(h->scratch + h->off_xb);
  P.qbuf = reinterpret_cast<float*>(h->scratch + h->off_q);
  P.attn = reinterpret_cast<float*>(h->scratch + h->off_attn);
  P.hbuf = reinterpret_cast<float*>(h->scratch + h->off_h);
  P.part = reinterpret_cast<float*>(h->scratch + h->off_part);
  P.arrive = h->d_arrive;
  P.best = h->d_best;
  P.seqlen = h->d_seqlen;
  P.tok_fb = h->d_tok_fb;
  P.active_batch = h->d_active;
  P.slot_active = h->d_slot_active;
  P.slot0 = 0;
  P.tiles = h->d_tiles;
  P.sig = h->d_sig;
  P.ctr = h->d_ctr;
  P.head = h->d_head;
  P.err = h->d_err;
  P.trace_buf = h->d_trace;
  P.evclock = h->d_evclock;
  P.in_tok_stride = 1;
  P.epoch = 1;
  P.idle_ns = std::max<uint64_t>(200000000ull, 20 * g.plan.wait_timeout_ns);
  // the team schedule's streams belong to the decode program; any other
  // program of the handle (the prefill) runs the static streams
  P.static_sched = g.plan.schedule == WPK_SCHED_STATIC || g.plan.schedule == WPK_SCHED_TEAMS;
  P.team_sched = g.plan.schedule == WPK_SCHED_TEAMS;
  P.stream_begin = h->d_stream_begin;
  P.stream = h->d_stream;
  P.mma_n = kTokBlock;
  P.act_chunk = kMmaChunkBytes;
  P.img_stride = kMmaChunkBytes;
  P.mma_cps = 1;
  if (g.plan.decode_mode == WPK_DECODE_MMA) {
    P.dec_mma = 1;
    P.uses_tmem = 1;
    P.mma_n = g.plan.dec_n;
    P.act_chunk = g.plan.dec_n * 128;
    P.img_stride = 2 * P.act_chunk;  // hi and lo rows of a chunk adjacent
    P.mma_cps = g.plan.dec_cps;
    P.stage_bytes = g.plan.dec_stage_bytes;
    P.n_stages = g.plan.dec_stages;
    P.gemv_cps = 1;
    P.act_bytes = g.plan.dec_act_bytes;
    P.o_splits = g.o_splits;
    P.down_splits = g.down_splits;
    P.xt = reinterpret_cast<float*>(h->scratch + h->off_xt);
    P.acc = reinterpret_cast<float*>(h->scratch + h->off_acc);
    P.ss = reinterpret_cast<float*>(h->scratch + h->off_ss);
    for (int i = 0; i < 2; ++i) {  // lo rows follow the hi rows of each chunk
      P.xn_img[i] = h->scratch + h->off_dimg[0] + i * P.act_chunk;
      P.xf_img[i] = h->scratch + h->off_dimg[1] + i * P.act_chunk;
      P.att_img[i] = h->scratch + h->off_dimg[2] + i * P.act_chunk;
      P.h_img[i] = h->scratch + h->off_dimg[3] + i * P.act_chunk;
    }
    P.rb_arrive = h->d_rb_arrive;
    P.lm_mma_off = g.lay.lm_mma;
  }
  set_mma_geometry(&P);
  if (h->io.set) {
    P.n_in = h->io.n_in;
    P.in_rows = h->io.in_rows;
    for (int k = 0; k < kMaxInTables; ++k) P.in_table_off[k] = h->io.in_off[k];
    P.in_vec = h->io.in_vec;
    P.lm_head_off = h->io.lm_head_off;
    if (P.dec_mma) P.lm_mma_off = h->io.lm_mma_off;
    P.logits_stride = h->io.logits_stride;
    P.out_stride = h->io.out_stride;
  }
  return P;
}

void scratch_layout(wpk_handle* h) {
  const CompiledGraph& g = h->g;
  const wpk_model_cfg& m = g.m;
  const size_t B = g.plan.max_batch, q_rows = (size_t)m.n_heads * m.head_dim;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = a256(off + bytes); return o; };
  h->off_xa = take(B * m.hidden * 4);
  h->off_xb = take(B * m.hidden * 4);
  h->off_q = take(B * q_rows * 4);
  h->off_attn = take(B * q_rows * 4);
  h->off_h = take(B * m.ffn * 4);
  h->off_part = take(B * m.n_kv_heads * g.n_splits * (m.n_heads / m.n_kv_heads) * (2 + m.head_dim) * 4);
  h->decode_scratch_bytes = off;
  if (g.plan.prefill_mode == WPK_PREFILL_MMA) {
    // prefill of up to max_batch prompts of max_context tokens, in blocks of 128
    const size_t M = (size_t)g.plan.max_batch * g.plan.max_context;
    const size_t n_tb = (M + kTokBlock - 1) / kTokBlock;
    h->prefill_max_tokens = (int64_t)M;
    h->off_px = take(M * m.hidden * 4);
    h->off_pq = take(M * q_rows * 4);
    // activation images [token block][K / 64][hi, lo][128 rows x 128 B]: the
    // hi and lo halves of a chunk adjacent, so one bulk copy stages both
    h->off_xn = take(n_tb * (m.hidden / 64) * 2 * kMmaChunkBytes);
    h->off_att = take(n_tb * (q_rows / 64) * 2 * kMmaChunkBytes);
    h->off_hi = take(n_tb * (m.ffn / 64) * 2 * kMmaChunkBytes);
    // key-split attention partials: fewer (sequence, kv head, query block)
    // tiles than workers, each with up to kMaxKeySplits splits of 128 rows
    const int Wk = g.W > 0 ? g.W : 148;
    h->off_ppart = take((size_t)Wk * kMaxKeySplits * 128 * (2 + kHeadDim) * 4);
  }
  if (g.plan.decode_mode == WPK_DECODE_MMA) {
    const size_t N = g.plan.dec_n, chunk = N * 128;
    const size_t qkv_rows = q_rows + 2 * (size_t)m.n_kv_heads * m.head_dim;
    h->off_xt = take((size_t)m.hidden * N * 4);
    h->off_acc = take(qkv_rows * N * 4);
    h->off_ss = take((2 * (size_t)m.n_layers + 1) * N * 4);
    const size_t widths[4] = {(size_t)m.hidden, (size_t)m.hidden, q_rows, (size_t)m.ffn};
    for (int t = 0; t < 4; ++t) h->off_dimg[t] = take(widths[t] / 64 * 2 * chunk);  // [K/64][hi, lo][chunk]
  }
  h->scratch_bytes = off;
  h->n_blocks = (int64_t)B * g.max_blocks;
  h->kv_bytes = (size_t)m.n_layers * h->n_blocks * 2 * m.n_kv_heads * g.plan.page_tokens * m.head_dim * 2;
}

// A worker grid: cooperative, so that all its CTAs are co-resident, unless
// the handle runs beside another persistent grid (plain_launch).
cudaError_t launch_grid(const wpk_handle* h, const void* fn, void** args, size_t smem, cudaStream_t s) {
  if (h->plain_launch) return cudaLaunchKernel(fn, dim3(h->n_workers), dim3(cta_threads(fn)), args, smem, s);
  return cudaLaunchCooperativeKernel(fn, dim3(h->n_workers), dim3(cta_threads(fn)), args, smem, s);
}

int launch_megakernel(wpk_handle* h, const KParams& base, cudaStream_t s) {
  const CompiledGraph& g = h->g;
  CUDA_TRY(h, cudaMemsetAsync(h->d_ctr, 0, std::max<size_t>(1, g.ctr_need.size()) * 4, s));
  CUDA_TRY(h, cudaMemsetAsync(h->d_head, 0, 4 * 4, s));
  for (int r = 0; r + 1 < (int)g.region_begin.size(); ++r) {
    KParams P = base;
    P.t_begin = g.region_begin[r];
    P.t_end = g.region_begin[r + 1];
    P.region = r;
    void* args[] = {&P};
    CUDA_TRY(h, launch_grid(h, persistent_kernel_ptr(h->g.plan.decode_mode == WPK_DECODE_MMA), args, h->smem, s));
  }
  return WPK_OK;
}

int capture_per_op(wpk_handle* h, int32_t* out_tok, float* logits, GraphEntry* out) {
  const CompiledGraph& g = h->g;
  if (!h->capture_stream) CUDA_TRY(h, cudaStreamCreateWithFlags(&h->capture_stream, cudaStreamNonBlocking));
  KParams base = make_params(h);
  base.in_tok = nullptr;
  base.out_tok = out_tok;
  base.logits = logits;
  CUDA_TRY(h, cudaStreamBeginCapture(h->capture_stream, cudaStreamCaptureModeThreadLocal));
  for (const OpGroup& og : g.groups) {
    KParams P = base;
    P.t_begin = og.begin;
    P.t_end = og.end;
    P.per_op = 1;
    if (!P.dec_mma) {
      P.gemv_cps = gemv_chunks_per_stage(g.plan.per_op_slot);
      P.stage_bytes = P.gemv_cps * kStageBytes;
      P.n_stages = g.plan.per_op_slot / P.stage_bytes;
    }
    void* args[] = {&P};
    cudaError_t e = cudaLaunchKernel(per_op_kernel_ptr(h->g.plan.decode_mode == WPK_DECODE_MMA), dim3(og.end - og.begin), dim3(cta_threads(per_op_kernel_ptr(h->g.plan.decode_mode == WPK_DECODE_MMA))), args,
                                     h->smem_per_op, h->capture_stream);
    if (e != cudaSuccess) {
      cudaGraph_t junk = nullptr;
      cudaStreamEndCapture(h->capture_stream, &junk);
      if (junk) cudaGraphDestroy(junk);
      return fail(h, WPK_ERR_CUDA, std::string("per-op capture: ") + cudaGetErrorString(e));
    }
  }
  out->key0 = out_tok;
  out->key1 = logits;
  out->key2 = nullptr;
  CUDA_TRY(h, cudaStreamEndCapture(h->capture_stream, &out->graph));
  CUDA_TRY(h, cudaGraphInstantiate(&out->exec, out->graph, 0));
  return WPK_OK;
}

// ------------------------------------------------------------- resident grid
// Stops a live resident grid (doorbell = shutdown) and waits for it to return.
int res_shutdown(wpk_handle* h) {
  if (!h->res_live) return WPK_OK;
  h->res_ctl->db = kResShutdown;
  std::atomic_thread_fence(std::memory_order_seq_cst);
  h->res_live = false;
  CUDA_TRY(h, cudaStreamSynchronize(h->res_stream));
  if (h->res_ctl->err && h->h_err_code) *h->h_err_code = h->res_ctl->err;
  return WPK_OK;
}

int res_launch(wpk_handle* h) {
  const CompiledGraph& g = h->g;
  CUDA_TRY(h, cudaMemsetAsync(h->d_ctr, 0, std::max<size_t>(1, g.ctr_need.size()) * 4, h->res_stream));
  CUDA_TRY(h, cudaMemsetAsync(h->d_head, 0, 4 * 4, h->res_stream));
  CUDA_TRY(h, cudaMemsetAsync(h->d_res, 0, sizeof(ResDev), h->res_stream));
  ResCtl* c = h->res_ctl;
  c->db = 0;
  c->ack = 0;
  c->err = 0;
  c->t_done_ns = 0;
  std::atomic_thread_fence(std::memory_order_seq_cst);
  KParams P = make_params(h);
  P.resident = 1;
  P.ctl = h->res_ctl_dev;
  P.rdev = h->d_res;
  P.t_begin = 0;
  P.t_end = (uint32_t)g.tiles.size();
  P.region = 0;
  void* args[] = {&P};
  CUDA_TRY(h, cudaLaunchCooperativeKernel(persistent_kernel_ptr(h->g.plan.decode_mode == WPK_DECODE_MMA), dim3(h->n_workers), dim3(cta_threads(persistent_kernel_ptr(h->g.plan.decode_mode == WPK_DECODE_MMA))), args,
                                          h->smem, h->res_stream));
  h->res_live = true;
  h->res_epoch = 0;
  h->res_last = std::chrono::steady_clock::now();
  return WPK_OK;
}

// One step on the resident grid: the step's inputs must be complete on stream
// `s`; returns once the grid has acknowledged the step.
int res_step(wpk_handle* h, const int32_t* in_tok, int stride, int32_t* out_tok, float* logits, cudaStream_t s) {
  const uint64_t idle_ns = std::max<uint64_t>(200000000ull, 20 * h->g.plan.wait_timeout_ns);
  const auto now = std::chrono::steady_clock::now();
  // never ring a grid that may be about to leave on its idle limit, and start
  // a fresh grid before 32-bit tickets could wrap
  const uint32_t max_steps = (uint32_t)((1u << 31) / std::max<size_t>(1, h->g.tiles.size()));
  if (h->res_live && (cudaStreamQuery(h->res_stream) != cudaErrorNotReady || h->res_epoch >= max_steps ||
                      (uint64_t)std::chrono::duration_cast<std::chrono::nanoseconds>(now - h->res_last).count() >
                          idle_ns / 2)) {
    int rc = res_shutdown(h);
    if (rc) return rc;
  }
  cudaGetLastError();
  CUDA_TRY(h, cudaStreamSynchronize(s));  // the step's inputs
  if (!h->res_live) {
    int rc = res_launch(h);
    if (rc) return rc;
  }
  ResCtl* c = h->res_ctl;
  c->in_tok = (uint64_t)(uintptr_t)in_tok;
  c->in_stride = stride;
  c->out_tok = (uint64_t)(uintptr_t)out_tok;
  c->logits = (uint64_t)(uintptr_t)logits;
  std::atomic_thread_fence(std::memory_order_seq_cst);
  const uint32_t e = ++h->res_epoch;
  c->db = e;
  const auto t0 = std::chrono::steady_clock::now();
  const uint64_t limit = 2 * h->g.plan.wait_timeout_ns + 1000000000ull;
  for (uint64_t it = 0; c->ack < e; ++it) {
    if (c->err) {
      *h->h_err_code = c->err;
      h->poisoned = true;
      res_shutdown(h);
      return fail(h, WPK_ERR_POISONED, "device program reported an error (see wpk_get_error_info)");
    }
    if ((it & 1023) == 1023) {
      const uint64_t el =
          std::chrono::duration_cast<std::chrono::nanoseconds>(std::chrono::steady_clock::now() - t0).count();
      if (el > limit || cudaStreamQuery(h->res_stream) != cudaErrorNotReady) {
        if (c->ack >= e) break;
        h->poisoned = true;
        res_shutdown(h);
        return fail(h, WPK_ERR_TIMEOUT, "resident grid did not acknowledge the step");
      }
      std::this_thread::yield();
    }
  }
  std::atomic_thread_fence(std::memory_order_seq_cst);
  h->res_last = std::chrono::steady_clock::now();
  h->ctx += 1;
  return WPK_OK;
}

int step_impl(wpk_handle* h, const int32_t* in_tok, int stride, int32_t* out_tok, float* logits, cudaStream_t s) {
  if (h->g.plan.resident) return res_step(h, in_tok, stride, out_tok, logits, s);
  if (h->g.plan.mode == WPK_MEGAKERNEL) {
    KParams P = make_params(h);
    P.in_tok = in_tok;
    P.in_tok_stride = stride;
    P.out_tok = out_tok;
    P.logits = logits;
    int rc = launch_megakernel(h, P, s);
    if (rc) return rc;
  } else {
    if (in_tok)
      CUDA_TRY(h, cudaMemcpy2DAsync(h->d_tok_fb, 4, in_tok, (size_t)stride * 4, 4, h->batch,
                                    cudaMemcpyDeviceToDevice, s));
    GraphEntry* ge = nullptr;
    for (auto& e : h->graphs)
      if (e.key0 == out_tok && e.key1 == logits) ge = &e;
    if (!ge) {
      GraphEntry e{};
      int rc = capture_per_op(h, out_tok, logits, &e);
      if (rc) return rc;
      h->graphs.push_back(e);
      ge = &h->graphs.back();
    }
    CUDA_TRY(h, cudaGraphLaunch(ge->exec, s));
  }
  CUDA_TRY(h, cudaMemcpyAsync(h->h_err_code, &h->d_err->code, 4, cudaMemcpyDeviceToHost, s));
  CUDA_TRY(h, cudaGetLastError());
  h->ctx += 1;
  return WPK_OK;
}


// ------------------------------------------------------------ prefill program
int get_prefill_program(wpk_handle* h, int B, int T, PrefillProgram** out) {
  for (auto& p : h->prefills)
    if (p->g.B == B && p->g.T == T) {
      *out = p.get();
      return WPK_OK;
    }
  auto prog = std::make_unique<PrefillProgram>();
  std::string msg = compile_prefill_graph(h->g, B, T, &prog->g);
  if (!msg.empty()) return fail(h, WPK_ERR_UNSUPPORTED, msg);
  if (h->has_device) {
    const CompiledGraph& g = prog->g;
    const size_t n_tiles = g.tiles.size(), n_ctr = std::max<size_t>(1, g.ctr_need.size());
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = a256(off + bytes); return o; };
    const size_t o_tiles = take(n_tiles * sizeof(Tile)), o_sig = take(std::max<size_t>(1, g.sig.size()) * 4),
                 o_ctr = take(n_ctr * 4), o_trace = take(n_tiles * sizeof(TraceRec));
    CUDA_TRY(h, cudaMalloc(&prog->d_base, off));
    CUDA_TRY(h, cudaMemset(prog->d_base, 0, off));
    prog->d_tiles = reinterpret_cast<Tile*>(prog->d_base + o_tiles);
    prog->d_sig = reinterpret_cast<uint32_t*>(prog->d_base + o_sig);
    prog->d_ctr = reinterpret_cast<uint32_t*>(prog->d_base + o_ctr);
    prog->d_trace = reinterpret_cast<TraceRec*>(prog->d_base + o_trace);
    CUDA_TRY(h, cudaMemcpy(prog->d_tiles, g.tiles.data(), n_tiles * sizeof(Tile), cudaMemcpyHostToDevice));
    if (!g.sig.empty())
      CUDA_TRY(h, cudaMemcpy(prog->d_sig, g.sig.data(), g.sig.size() * 4, cudaMemcpyHostToDevice));
  }
  *out = prog.get();
  h->prefills.push_back(std::move(prog));
  return WPK_OK;
}

KParams prefill_params(const wpk_handle* h, const PrefillProgram* prog, const int32_t* tokens, int32_t* first_tok,
                       float* logits) {
  KParams P = make_params(h);
  const CompiledGraph& g = prog->g;
  P.tiles = prog->d_tiles;
  P.sig = prog->d_sig;
  P.ctr = prog->d_ctr;
  P.trace_buf = prog->d_trace;
  P.stage_bytes = h->prefill_cps * 3 * kMmaChunkBytes;
  P.n_stages = h->prefill_stages;
  P.gemv_cps = 1;
  P.uses_tmem = 1;
  // the prefill program's own geometry (its LM head tiles are GEMV tiles)
  P.dec_mma = 0;
  P.act_bytes = g.plan.act_bytes;
  P.mma_n = kTokBlock;
  P.act_chunk = kMmaChunkBytes;
  P.img_stride = 2 * kMmaChunkBytes;  // hi and lo halves of a chunk adjacent
  P.mma_cps = h->prefill_cps;
  set_mma_geometry(&P);
  P.M = g.M;
  P.T = g.T;
  P.n_tb = g.n_tb;
  P.pattn_ks = g.pattn_ks;
  P.ppart = reinterpret_cast<float*>(h->scratch + h->off_ppart);
  P.pattn_arrive = h->d_pattn_arrive;
  P.ptok = tokens;
  P.px = reinterpret_cast<float*>(h->scratch + h->off_px);
  P.pq = reinterpret_cast<float*>(h->scratch + h->off_pq);
  for (int i = 0; i < 2; ++i) {
    P.xn_img[i] = h->scratch + h->off_xn + i * kMmaChunkBytes;
    P.att_img[i] = h->scratch + h->off_att + i * kMmaChunkBytes;
    P.h_img[i] = h->scratch + h->off_hi + i * kMmaChunkBytes;
  }
  P.in_tok = nullptr;
  P.out_tok = first_tok;
  P.logits = logits;
  P.slot0 = h->prefill_slot0;
  P.team_sched = 0;  // the prefill program runs the static streams
  return P;
}

int launch_prefill(wpk_handle* h, PrefillProgram* prog, const int32_t* tokens, int32_t* first_tok, float* logits,
                   cudaStream_t s) {
  const CompiledGraph& g = prog->g;
  const KParams base = prefill_params(h, prog, tokens, first_tok, logits);
  if (g.plan.mode == WPK_MEGAKERNEL) {
    CUDA_TRY(h, cudaMemsetAsync(prog->d_ctr, 0, std::max<size_t>(1, g.ctr_need.size()) * 4, s));
    CUDA_TRY(h, cudaMemsetAsync(h->d_head, 0, 4 * 4, s));
    for (int r = 0; r + 1 < (int)g.region_begin.size(); ++r) {
      KParams P = base;
      P.t_begin = g.region_begin[r];
      P.t_end = g.region_begin[r + 1];
      P.region = r;
      void* args[] = {&P};
      CUDA_TRY(h, launch_grid(h, prefill_kernel_ptr(), args, h->smem_prefill, s));
    }
    return WPK_OK;
  }
  GraphEntry* ge = nullptr;
  for (auto& e : prog->graphs)
    if (e.key0 == tokens && e.key1 == first_tok && e.key2 == logits) ge = &e;
  if (!ge) {
    if (!h->capture_stream) CUDA_TRY(h, cudaStreamCreateWithFlags(&h->capture_stream, cudaStreamNonBlocking));
    GraphEntry e{tokens, first_tok, logits, nullptr, nullptr};
    CUDA_TRY(h, cudaStreamBeginCapture(h->capture_stream, cudaStreamCaptureModeThreadLocal));
    for (const OpGroup& og : g.groups) {
      KParams P = base;
      P.t_begin = og.begin;
      P.t_end = og.end;
      P.per_op = 1;
      void* args[] = {&P};
      cudaError_t err = cudaLaunchKernel(prefill_op_kernel_ptr(), dim3(og.end - og.begin), dim3(kCtaThreadsTc), args,
                                         h->smem_prefill, h->capture_stream);
      if (err != cudaSuccess) {
        cudaGraph_t junk = nullptr;
        cudaStreamEndCapture(h->capture_stream, &junk);
        if (junk) cudaGraphDestroy(junk);
        return fail(h, WPK_ERR_CUDA, std::string("per-op prefill capture: ") + cudaGetErrorString(err));
      }
    }
    CUDA_TRY(h, cudaStreamEndCapture(h->capture_stream, &e.graph));
    CUDA_TRY(h, cudaGraphInstantiate(&e.exec, e.graph, 0));
    prog->graphs.push_back(e);
    ge = &prog->graphs.back();
  }
  CUDA_TRY(h, cudaGraphLaunch(ge->exec, s));
  return WPK_OK;
}

const CompiledGraph& selected_graph(const wpk_handle* h) { return h->selected ? h->selected->g : h->g; }

}  // namespace

extern "C" {

// The dynamic shared memory limit is an attribute of the kernel function,
// shared by every handle of the process: it only ever rises, to the largest
// worker any handle on this device launches.
static cudaError_t raise_smem_limit(const void* fn, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, size_t> limit;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  size_t& cur = limit[{dev, fn}];
  if (bytes <= cur) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) cur = bytes;
  return e;
}

static int setup_device(wpk_handle* h) {
  CompiledGraph& g = h->g;
  const Plan& p = g.plan;
  const wpk_model_cfg* model = &g.m;
  CUDA_TRY(h, cudaGetDevice(&h->device));
  CUDA_TRY(h, cudaDeviceGetAttribute(&h->n_sms, cudaDevAttrMultiProcessorCount, h->device));
  if (p.decode_mode == WPK_DECODE_MMA) {
    h->smem = worker_smem_bytes(p.dec_stages, p.dec_stage_bytes, p.dec_act_bytes);
    h->smem_per_op = h->smem;
  } else {
    h->smem = worker_smem_bytes(p.slot_bytes / kStageBytes, kStageBytes, p.act_bytes);
    h->smem_per_op = worker_smem_bytes(p.per_op_slot / kStageBytes, kStageBytes, p.act_bytes);
  }
  if (h->smem > (size_t)kMaxSmem || h->smem_per_op > (size_t)kMaxSmem)
    return fail(h, WPK_ERR_UNSUPPORTED, "staging slot and activations exceed shared memory");
  if (p.prefill_mode == WPK_PREFILL_MMA) {
    // the kernel's static shared memory counts against the same per-CTA limit
    cudaFuncAttributes fa{};
    CUDA_TRY(h, cudaFuncGetAttributes(&fa, prefill_kernel_ptr()));
    const size_t fixed = worker_smem_bytes(0, 0, p.act_bytes) + fa.sharedSizeBytes;
    if (fixed >= (size_t)kMaxSmem) return fail(h, WPK_ERR_UNSUPPORTED, "no room for the prefill staging ring");
    // a stage holds cps K chunks of weights (16 KB each) and their 128
    // tokens' hi and lo rows (32 KB each): two chunks per stage when two such
    // stages fit, since a worker completes about one stage per half
    // microsecond whatever its size
    const size_t room = (size_t)kMaxSmem - fixed;
    h->prefill_cps = room / (2 * 3 * kMmaChunkBytes) >= 2 ? 2 : 1;
    const size_t stage = (size_t)h->prefill_cps * 3 * kMmaChunkBytes;
    h->prefill_stages = (int)std::min<size_t>(kMaxStages, room / stage);
    if (h->prefill_stages < 2) return fail(h, WPK_ERR_UNSUPPORTED, "no room for the prefill staging ring");
    h->smem_prefill = worker_smem_bytes(h->prefill_stages, (int)stage, p.act_bytes);
  }
  const size_t smem_max = h->smem;
  CUDA_TRY(h, raise_smem_limit(persistent_kernel_ptr(h->g.plan.decode_mode == WPK_DECODE_MMA), smem_max));
  CUDA_TRY(h, raise_smem_limit(per_op_kernel_ptr(h->g.plan.decode_mode == WPK_DECODE_MMA), h->smem_per_op));
  if (h->smem_prefill) {
    CUDA_TRY(h, raise_smem_limit(prefill_kernel_ptr(), h->smem_prefill));
    CUDA_TRY(h, raise_smem_limit(prefill_op_kernel_ptr(), h->smem_prefill));
    int per_sm_p = 0;
    CUDA_TRY(h, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm_p, prefill_kernel_ptr(), kCtaThreadsTc,
                                                              h->smem_prefill));
    if (per_sm_p < 1) return fail(h, WPK_ERR_UNSUPPORTED, "the prefill worker does not fit an SM");
  }
  int per_sm = 0;
  CUDA_TRY(h, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, persistent_kernel_ptr(h->g.plan.decode_mode == WPK_DECODE_MMA), cta_threads(persistent_kernel_ptr(h->g.plan.decode_mode == WPK_DECODE_MMA)), smem_max));
  h->per_sm = per_sm;
  {
    // tcgen05.alloc waits until the SM has free TMEM columns: workers that
    // share an SM must fit its 512 columns together
    KParams probe{};
    probe.mma_n = p.decode_mode == WPK_DECODE_MMA ? p.dec_n : kTokBlock;
    set_mma_geometry(&probe);
    if (p.decode_mode == WPK_DECODE_MMA && per_sm * probe.tmem_cols > 512)
      return fail(h, WPK_ERR_UNSUPPORTED, "co-resident decode workers would not fit the SM's tensor memory");
    if (h->smem_prefill) {
      KParams pp{};
      pp.mma_n = kTokBlock;
      set_mma_geometry(&pp);
      int per_sm_p = 0;
      CUDA_TRY(h, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm_p, prefill_kernel_ptr(), kCtaThreadsTc,
                                                                h->smem_prefill));
      h->per_sm_prefill = per_sm_p;
      if (per_sm_p * pp.tmem_cols > 512)
        return fail(h, WPK_ERR_UNSUPPORTED, "co-resident prefill workers would not fit the SM's tensor memory");
    }
  }
  h->n_workers = p.n_workers ? p.n_workers : h->n_sms * p.workers_per_sm;
  if (per_sm < 1 || h->n_workers > per_sm * h->n_sms)
    return fail(h, WPK_ERR_UNSUPPORTED, "the worker grid cannot be co-resident with this slot size");

  // one allocation for the small tables
  const size_t n_tiles = g.tiles.size(), n_ctr = std::max<size_t>(1, g.ctr_need.size());
  const size_t B = p.max_batch, hd2 = model->head_dim / 2;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = a256(off + bytes); return o; };
  const size_t o_tiles = take(n_tiles * sizeof(Tile)), o_sig = take(std::max<size_t>(1, g.sig.size()) * 4),
               o_ctr = take(n_ctr * 4), o_head = take(4 * 4), o_err = take(sizeof(ErrWord)),
               o_trace = take(n_tiles * sizeof(TraceRec)), o_ev = take(4),
               o_layers = take(g.lay.layers.size() * sizeof(LayerDev)),
               o_rope = take((size_t)p.max_context * hd2 * sizeof(float2)),
               o_bt = take(B * g.max_blocks * 4), o_arr = take(B * model->n_kv_heads * 4), o_best = take(B * 8),
               o_seq = take(B * 4), o_fb = take(B * 4), o_act = take(4), o_slot = take(B * 4),
               o_sb = take((g.stream_begin.size() + 1) * 4), o_st = take((g.stream.size() + 1) * 4),
               o_pa = take((size_t)std::max(1, g.W) * 4),
               o_rb = take((size_t)model->n_layers * 2 * (model->hidden / 128 + 1) * 4),
               o_res = take(sizeof(ResDev));
  CUDA_TRY(h, cudaMalloc(&h->d_base, off));
  CUDA_TRY(h, cudaMemset(h->d_base, 0, off));
  h->d_tiles = reinterpret_cast<Tile*>(h->d_base + o_tiles);
  h->d_sig = reinterpret_cast<uint32_t*>(h->d_base + o_sig);
  h->d_ctr = reinterpret_cast<uint32_t*>(h->d_base + o_ctr);
  h->d_head = reinterpret_cast<uint32_t*>(h->d_base + o_head);
  h->d_err = reinterpret_cast<ErrWord*>(h->d_base + o_err);
  h->d_trace = reinterpret_cast<TraceRec*>(h->d_base + o_trace);
  h->d_evclock = reinterpret_cast<uint32_t*>(h->d_base + o_ev);
  h->d_layers = reinterpret_cast<LayerDev*>(h->d_base + o_layers);
  h->d_rope = reinterpret_cast<float2*>(h->d_base + o_rope);
  h->d_block_table = reinterpret_cast<int32_t*>(h->d_base + o_bt);
  h->d_arrive = reinterpret_cast<uint32_t*>(h->d_base + o_arr);
  h->d_best = reinterpret_cast<unsigned long long*>(h->d_base + o_best);
  h->d_seqlen = reinterpret_cast<int32_t*>(h->d_base + o_seq);
  h->d_tok_fb = reinterpret_cast<int32_t*>(h->d_base + o_fb);
  h->d_active = reinterpret_cast<int32_t*>(h->d_base + o_act);
  h->d_slot_active = reinterpret_cast<int32_t*>(h->d_base + o_slot);
  h->d_pattn_arrive = reinterpret_cast<uint32_t*>(h->d_base + o_pa);
  h->d_stream_begin = reinterpret_cast<uint32_t*>(h->d_base + o_sb);
  h->d_stream = reinterpret_cast<uint32_t*>(h->d_base + o_st);
  if (!g.stream.empty()) {
    CUDA_TRY(h, cudaMemcpy(h->d_stream_begin, g.stream_begin.data(), g.stream_begin.size() * 4,
                           cudaMemcpyHostToDevice));
    CUDA_TRY(h, cudaMemcpy(h->d_stream, g.stream.data(), g.stream.size() * 4, cudaMemcpyHostToDevice));
  }
  h->d_rb_arrive = reinterpret_cast<uint32_t*>(h->d_base + o_rb);
  h->d_res = reinterpret_cast<ResDev*>(h->d_base + o_res);
  CUDA_TRY(h, cudaMemcpy(h->d_tiles, g.tiles.data(), n_tiles * sizeof(Tile), cudaMemcpyHostToDevice));
  if (!g.sig.empty()) CUDA_TRY(h, cudaMemcpy(h->d_sig, g.sig.data(), g.sig.size() * 4, cudaMemcpyHostToDevice));
  CUDA_TRY(h, cudaMemcpy(h->d_layers, g.lay.layers.data(), g.lay.layers.size() * sizeof(LayerDev),
                         cudaMemcpyHostToDevice));
  // RoPE (cos, sin) table: angle = pos * theta^(-2i/d), evaluated in double
  std::vector<float2> rope((size_t)p.max_context * hd2);
  for (int pos = 0; pos < p.max_context; ++pos)
    for (size_t i = 0; i < hd2; ++i) {
      const double inv = std::pow((double)model->rope_theta, -2.0 * (double)i / (double)model->head_dim);
      const double a = (double)pos * inv;
      rope[(size_t)pos * hd2 + i] = make_float2((float)std::cos(a), (float)std::sin(a));
    }
  CUDA_TRY(h, cudaMemcpy(h->d_rope, rope.data(), rope.size() * sizeof(float2), cudaMemcpyHostToDevice));
  std::vector<int32_t> bt(B * g.max_blocks);
  for (size_t i = 0; i < bt.size(); ++i) bt[i] = (int32_t)i;
  CUDA_TRY(h, cudaMemcpy(h->d_block_table, bt.data(), bt.size() * 4, cudaMemcpyHostToDevice));
  CUDA_TRY(h, cudaHostAlloc(&h->h_err_code, 4, cudaHostAllocDefault));
  *h->h_err_code = 0;
  if (p.resident) {
    CUDA_TRY(h, cudaHostAlloc(&h->res_ctl, sizeof(ResCtl), cudaHostAllocMapped));
    memset((void*)h->res_ctl, 0, sizeof(ResCtl));
    CUDA_TRY(h, cudaHostGetDevicePointer((void**)&h->res_ctl_dev, (void*)h->res_ctl, 0));
    CUDA_TRY(h, cudaStreamCreateWithFlags(&h->res_stream, cudaStreamNonBlocking));
  }
  h->has_device = true;
  return WPK_OK;
}

static int build_two_stage(const wpk_model_cfg* model, const wpk_plan_cfg* plan, wpk_handle** out);

// SMs of the current device (148, a B200's count, when there is no device).
static int device_sms() {
  int n_dev = 0, sms = 148;
  if (cudaGetDeviceCount(&n_dev) == cudaSuccess && n_dev > 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  cudaGetLastError();
  return sms;
}

// One decoder; lm_rows > 0 replaces its output head's row count.
static int build_decoder(const wpk_model_cfg* model, const wpk_plan_cfg* plan, int lm_rows, wpk_handle** out) {
  *out = nullptr;
  auto* h = new wpk_handle();
  int code = 0;
  Plan p;
  std::string msg = normalize_plan(*model, *plan, &p, &code);
  if (lm_rows > 0) p.lm_rows = lm_rows;
  // worker count the tiles are sized for: the plan's, else #SMs x workers per SM
  const int W = p.n_workers ? p.n_workers : device_sms() * p.workers_per_sm;
  if (msg.empty()) msg = compile_graph(*model, p, &h->g, &code, W);
  if (!msg.empty()) {
    g_build_error = msg;
    delete h;
    return code;
  }
  scratch_layout(h);
  // Without a CUDA device the handle is host-only: the compiled tables can be
  // inspected, verified and simulated; device calls return WPK_ERR_CUDA.
  int n_dev = 0;
  if (cudaGetDeviceCount(&n_dev) != cudaSuccess || n_dev == 0) {
    cudaGetLastError();
    h->n_workers = p.n_workers;
    h->err = "no CUDA device: host-only handle";
    *out = h;
    return WPK_OK;
  }
  int rc = setup_device(h);
  if (rc) {
    g_build_error = h->err;
    if (h->d_base) cudaFree(h->d_base);
    delete h;
    return rc;
  }
  *out = h;
  return WPK_OK;
}

int wpk_build_graph(const wpk_model_cfg* model, const wpk_plan_cfg* plan, wpk_handle** out) {
  if (!model || !plan || !out) return WPK_ERR_INVALID_ARG;
  *out = nullptr;
  if (model->n_codebooks < 0) {
    g_build_error = "n_codebooks must be >= 0";
    return WPK_ERR_INVALID_ARG;
  }
  if (plan->frame_chunks < 0 || plan->frame_chunks > 8 || plan->head_workers < 0) {
    g_build_error = "frame_chunks must be 0..8 and head_workers >= 0";
    return WPK_ERR_INVALID_ARG;
  }
  if (model->n_codebooks > 0) return build_two_stage(model, plan, out);
  if (plan->frame_chunks > 1 || plan->head_workers) {
    g_build_error = "frame_chunks and head_workers apply to the two-stage model only";
    return WPK_ERR_INVALID_ARG;
  }
  return build_decoder(model, plan, 0, out);
}

// Two-stage model: a backbone decoder whose output head is the projection into
// the head's width, and a head decoder (its own handle, tables and program)
// whose input and output tables change from one head step to the next.  Both
// images, the frame / head-input / output tables and the tensor-core images of
// the output tables share one weight buffer; KV and scratch likewise.
// One backbone + head pair: the backbone for `plan`, the head for `head_plan`
// (its batch and worker count; the head's cache holds one frame).
static int build_pair(const wpk_model_cfg* model, const wpk_plan_cfg* plan, const wpk_plan_cfg* head_plan,
                      wpk_handle** out) {
  const int K = model->n_codebooks, V = model->codebook_vocab;
  wpk_model_cfg mb = *model;  // backbone: output head = projection (untied)
  mb.n_codebooks = 0;
  mb.codebook_vocab = 0;
  mb.head = nullptr;
  mb.tied_embedding = 0;
  wpk_model_cfg mh = *model->head;  // head: input and output tables have V rows
  mh.vocab = V;
  mh.tied_embedding = 0;
  mh.n_codebooks = 0;
  mh.codebook_vocab = 0;
  mh.head = nullptr;
  wpk_plan_cfg ph = *head_plan;  // the head's cache holds one frame
  ph.max_context = K;
  ph.page_tokens = (K + 7) / 8 * 8;
  ph.n_regions = 1;
  ph.prefill = WPK_PREFILL_TOKENWISE;
  wpk_handle* h = nullptr;
  int rc = build_decoder(&mb, plan, mh.hidden, &h);
  if (rc) return rc;
  wpk_handle* hh = nullptr;
  rc = build_decoder(&mh, &ph, 0, &hh);
  if (rc) {
    wpk_destroy(h);
    return rc;
  }
  h->head = hh;
  h->n_cb = K;
  h->cb_vocab = V;
  // combined weight image: backbone, head, then the per-codebook tables
  uint64_t off = a256(h->g.lay.total);
  h->head_base = off;
  off = a256(off + hh->g.lay.total);
  auto take = [&](uint64_t bytes) { uint64_t o = off; off = a256(off + bytes); return o; };
  const uint64_t vb = (uint64_t)(V + 127) / 128;
  for (int k = 0; k < K; ++k) h->frame_embed_off.push_back(take((uint64_t)V * mb.hidden * 2));
  for (int k = 0; k < K; ++k) h->head_embed_off.push_back(k ? take((uint64_t)V * mh.hidden * 2) : 0);
  for (int k = 0; k < K; ++k) h->out_head_off.push_back(take((uint64_t)V * mh.hidden * 2));
  for (int k = 0; k < K; ++k)
    h->out_head_mma_off.push_back(hh->g.plan.decode_mode == WPK_DECODE_MMA
                                      ? take(vb * (mh.hidden / 64) * kMmaChunkBytes)
                                      : 0);
  h->weights_total = off;
  // scratch: the projection output and the last frame's codes, then the head's
  const size_t B = plan->max_batch;
  size_t so = h->scratch_bytes;
  h->off_p = so;
  so = a256(so + B * mh.hidden * 4);
  h->off_codes = so;
  so = a256(so + B * K * 4);
  h->scratch_bytes = so;
  *out = h;
  return WPK_OK;
}

static int build_two_stage(const wpk_model_cfg* model, const wpk_plan_cfg* plan, wpk_handle** out) {
  const int K = model->n_codebooks, V = model->codebook_vocab;
  if (!model->head || K > kMaxInTables || V <= 0) {
    g_build_error = "two-stage model: needs a head shape, n_codebooks <= 16 and codebook_vocab > 0";
    return WPK_ERR_INVALID_ARG;
  }
  if (plan->mode != WPK_MEGAKERNEL || plan->resident) {
    g_build_error = "two-stage model: runs in WPK_MEGAKERNEL mode without a resident grid";
    return WPK_ERR_UNSUPPORTED;
  }
  const int C = plan->frame_chunks;
  if (C <= 1) {
    if (plan->head_workers) {
      g_build_error = "head_workers needs frame_chunks >= 2";
      return WPK_ERR_INVALID_ARG;
    }
    return build_pair(model, plan, plan, out);
  }
  // chunked frame: C pairs of ceil(B / C) sequences; backbones and heads on
  // disjoint worker counts that together fill the grid
  if (C > plan->max_batch) {
    g_build_error = "frame_chunks exceeds max_batch";
    return WPK_ERR_INVALID_ARG;
  }
  const int W = plan->n_workers ? plan->n_workers : device_sms() * std::max(1, plan->workers_per_sm);
  const int Wh = plan->head_workers ? plan->head_workers : W / 2;
  if (Wh < 1 || Wh >= W) {
    g_build_error = "head_workers must leave the backbones at least one worker";
    return WPK_ERR_INVALID_ARG;
  }
  wpk_plan_cfg pb = *plan;
  pb.max_batch = (plan->max_batch + C - 1) / C;
  pb.n_workers = W - Wh;
  pb.frame_chunks = 0;
  pb.head_workers = 0;
  wpk_plan_cfg ph = pb;
  ph.n_workers = Wh;
  std::vector<wpk_handle*> pairs;
  for (int c = 0; c < C; ++c) {
    wpk_handle* x = nullptr;
    const int rc = build_pair(model, &pb, &ph, &x);
    if (rc) {
      for (wpk_handle* y : pairs) wpk_destroy(y);
      return rc;
    }
    pairs.push_back(x);
  }
  // Grids of different programs share SMs only if an SM holds more than one
  // worker; tensor-memory programs then could wait on each other's columns
  for (wpk_handle* x : pairs)
    for (wpk_handle* y : {x, x->head})
      if (y->has_device && (y->per_sm > 1 || y->per_sm_prefill > 1) && y->g.lay.mma) {
        for (wpk_handle* z : pairs) wpk_destroy(z);
        g_build_error = "chunked frames with tensor-core programs need one worker per SM";
        return WPK_ERR_UNSUPPORTED;
      }
  for (wpk_handle* x : pairs) x->plain_launch = x->head->plain_launch = true;
  wpk_handle* h = pairs[0];
  h->chunks.assign(pairs.begin() + 1, pairs.end());
  h->chunk_rows = pb.max_batch;
  *out = h;
  return WPK_OK;
}

int wpk_workspace_size(const wpk_handle* h, size_t* weight_bytes, size_t* kv_bytes, size_t* scratch_bytes) {
  if (!h) return WPK_ERR_INVALID_ARG;
  if (h->head) {  // every pair's KV and scratch, one after another
    size_t kv = 0, sc = 0;
    for (int c = 0; c <= (int)h->chunks.size(); ++c) {
      const wpk_handle* x = c ? h->chunks[c - 1] : h;
      kv += x->kv_bytes + x->head->kv_bytes;
      sc += x->scratch_bytes + x->head->scratch_bytes;
    }
    if (weight_bytes) *weight_bytes = h->weights_total;
    if (kv_bytes) *kv_bytes = kv;
    if (scratch_bytes) *scratch_bytes = sc;
    return WPK_OK;
  }
  if (weight_bytes) *weight_bytes = h->g.lay.total;
  if (kv_bytes) *kv_bytes = h->kv_bytes;
  if (scratch_bytes) *scratch_bytes = h->scratch_bytes;
  return WPK_OK;
}

// Two-stage weights: the backbone (output head = projection), the head, and
// the per-codebook tables, arranged into one image.
static int load_two_stage(wpk_handle* h, const wpk_weights* w, void* dev_weights, void* dev_kv, void* dev_scratch,
                          void* stream) {
  wpk_handle* hh = h->head;
  const int K = h->n_cb, V = h->cb_vocab;
  if (!w->proj || !w->frame_embed || !w->head_embed || !w->out_head || !w->head_layers || !w->head_final_norm)
    return fail(h, WPK_ERR_INVALID_ARG, "two-stage model: missing table pointers");
  for (int k = 0; k < K; ++k)
    if (!w->frame_embed[k] || !w->out_head[k] || (k > 0 && !w->head_embed[k]))
      return fail(h, WPK_ERR_INVALID_ARG, "two-stage model: missing per-codebook table");
  std::vector<uint8_t> img(h->weights_total, 0);
  wpk_weights wb{};
  wb.embed = w->embed;
  wb.final_norm = w->final_norm;
  wb.lm_head = w->proj;
  wb.layers = w->layers;
  if (!wb.embed) return fail(h, WPK_ERR_INVALID_ARG, "missing token embedding");
  std::string msg = arrange_weights(h->g, wb, img.data());
  if (!msg.empty()) return fail(h, WPK_ERR_INVALID_ARG, msg);
  wpk_weights wh{};
  wh.final_norm = w->head_final_norm;
  wh.layers = w->head_layers;
  msg = arrange_weights(hh->g, wh, img.data() + h->head_base);
  if (!msg.empty()) return fail(h, WPK_ERR_INVALID_ARG, msg);
  const int hb = h->g.m.hidden, hd = hh->g.m.hidden;
  for (int k = 0; k < K; ++k) {
    memcpy(img.data() + h->frame_embed_off[k], w->frame_embed[k], (size_t)V * hb * 2);
    if (k) memcpy(img.data() + h->head_embed_off[k], w->head_embed[k], (size_t)V * hd * 2);
    memcpy(img.data() + h->out_head_off[k], w->out_head[k], (size_t)V * hd * 2);
    if (h->out_head_mma_off[k]) arrange_mma_image(img.data() + h->out_head_mma_off[k], hd, V, w->out_head[k]);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUDA_TRY(h, cudaMemcpyAsync(dev_weights, img.data(), img.size(), cudaMemcpyHostToDevice, s));
  CUDA_TRY(h, cudaStreamSynchronize(s));
  // every pair reads the one image; KV and scratch are laid out pair by pair
  uint8_t* kv = static_cast<uint8_t*>(dev_kv);
  uint8_t* sc = static_cast<uint8_t*>(dev_scratch);
  for (int c = 0; c <= (int)h->chunks.size(); ++c) {
    wpk_handle* x = c ? h->chunks[c - 1] : h;
    wpk_handle* xh = x->head;
    x->weights = static_cast<uint8_t*>(dev_weights);
    xh->weights = x->weights + x->head_base;
    x->kv = reinterpret_cast<uint16_t*>(kv);
    kv += x->kv_bytes;
    xh->kv = reinterpret_cast<uint16_t*>(kv);
    kv += xh->kv_bytes;
    x->scratch = sc;
    sc += x->scratch_bytes;
    xh->scratch = sc;
    sc += xh->scratch_bytes;
    x->loaded = xh->loaded = true;
    x->prefilled = xh->prefilled = false;
    x->graphs.clear();
    xh->graphs.clear();
  }
  return WPK_OK;
}

int wpk_load_weights(wpk_handle* h, const wpk_weights* w, void* dev_weights, void* dev_kv, void* dev_scratch,
                     void* stream) {
  int rc = check_live(h);
  if (rc) return rc;
  rc = res_shutdown(h);
  if (rc) return rc;
  if (!w || !dev_weights || !dev_kv || !dev_scratch)
    return fail(h, WPK_ERR_INVALID_ARG, "null weights or device buffer");
  if (((uintptr_t)dev_weights | (uintptr_t)dev_kv | (uintptr_t)dev_scratch) & 255)
    return fail(h, WPK_ERR_INVALID_ARG, "device buffers must be 256-byte aligned");
  if (h->head) return load_two_stage(h, w, dev_weights, dev_kv, dev_scratch, stream);
  std::vector<uint8_t> img(h->g.lay.total, 0);
  std::string msg = arrange_weights(h->g, *w, img.data());
  if (!msg.empty()) return fail(h, WPK_ERR_INVALID_ARG, msg);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUDA_TRY(h, cudaMemcpyAsync(dev_weights, img.data(), img.size(), cudaMemcpyHostToDevice, s));
  CUDA_TRY(h, cudaStreamSynchronize(s));
  h->weights = static_cast<uint8_t*>(dev_weights);
  h->kv = static_cast<uint16_t*>(dev_kv);
  h->scratch = static_cast<uint8_t*>(dev_scratch);
  h->loaded = true;
  h->prefilled = false;
  h->graphs.clear();  // captured pointers may have changed
  return WPK_OK;
}

int wpk_set_block_table(wpk_handle* h, const int32_t* table) {
  int rc = check_live(h);
  if (rc) return rc;
  if (!table) return fail(h, WPK_ERR_INVALID_ARG, "null table");
  if (!h->chunks.empty()) return fail(h, WPK_ERR_UNSUPPORTED, "a chunked two-stage frame keeps its own block tables");
  const size_t n = (size_t)h->g.plan.max_batch * h->g.max_blocks;
  std::vector<char> seen(n, 0);
  for (size_t i = 0; i < n; ++i) {
    if (table[i] < 0 || (size_t)table[i] >= n || seen[table[i]])
      return fail(h, WPK_ERR_INVALID_ARG, "block table must be a permutation of page ids");
    seen[table[i]] = 1;
  }
  CUDA_TRY(h, cudaMemcpy(h->d_block_table, table, n * 4, cudaMemcpyHostToDevice));
  return WPK_OK;
}

static int prefill_impl(wpk_handle* h, const int32_t* tokens_dev, int batch, int prompt_len, int32_t* first_tok_dev,
                        float* logits_dev, void* stream);

// State the step programs keep between steps, cleared for a new batch of
// sequences: argmax keys, split arrivals and (tensor-core decode) the fp32
// sums and per-token x^2 sums, which the program itself returns to zero.
static int reset_step_state(wpk_handle* h, cudaStream_t s) {
  const size_t B = h->g.plan.max_batch;
  CUDA_TRY(h, cudaMemsetAsync(h->d_seqlen, 0, B * 4, s));
  // every slot live (bytes 0x01: a nonzero word); a new batch leaves the cohort mode
  CUDA_TRY(h, cudaMemsetAsync(h->d_slot_active, 1, B * 4, s));
  h->cohort = false;
  CUDA_TRY(h, cudaMemsetAsync(h->d_best, 0, B * 8, s));
  CUDA_TRY(h, cudaMemsetAsync(h->d_arrive, 0, B * h->g.m.n_kv_heads * 4, s));
  if (h->g.plan.decode_mode == WPK_DECODE_MMA) {
    const wpk_model_cfg& m = h->g.m;
    const size_t N = h->g.plan.dec_n;
    const size_t qkv_rows = (size_t)(m.n_heads + 2 * m.n_kv_heads) * m.head_dim;
    CUDA_TRY(h, cudaMemsetAsync(h->scratch + h->off_acc, 0, qkv_rows * N * 4, s));
    CUDA_TRY(h, cudaMemsetAsync(h->scratch + h->off_ss, 0, (2 * (size_t)m.n_layers + 1) * N * 4, s));
    CUDA_TRY(h, cudaMemsetAsync(h->d_rb_arrive, 0, (size_t)m.n_layers * 2 * (m.hidden / 128 + 1) * 4, s));
  }
  return WPK_OK;
}
static int head_frame(wpk_handle* h, int32_t* codes_out, float* logits, cudaStream_t s);

// Chunked two-stage frame: the pair of chunk c, and the stream and events
// that let each head overlap the next chunk's backbone.
static wpk_handle* pair_of(wpk_handle* h, int c) { return c ? h->chunks[c - 1] : h; }

static int chunk_streams(wpk_handle* h) {
  if (h->head_stream) return WPK_OK;
  CUDA_TRY(h, cudaStreamCreateWithFlags(&h->head_stream, cudaStreamNonBlocking));
  const int n = 2 + 1 + (int)h->chunks.size();
  for (int i = 0; i < n; ++i) {
    cudaEvent_t e;
    CUDA_TRY(h, cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    h->chunk_ev.push_back(e);
  }
  return WPK_OK;
}

// The heads' stream starts after what the caller's stream holds so far.
static int chunk_fork(wpk_handle* h, cudaStream_t s) {
  CUDA_TRY(h, cudaEventRecord(h->chunk_ev[0], s));
  CUDA_TRY(h, cudaStreamWaitEvent(h->head_stream, h->chunk_ev[0], 0));
  return WPK_OK;
}

// The caller's stream continues after every head; taken on error paths too.
static int chunk_join(wpk_handle* h, cudaStream_t s, int rc) {
  const cudaError_t e1 = cudaEventRecord(h->chunk_ev[1], h->head_stream);
  const cudaError_t e2 = cudaStreamWaitEvent(s, h->chunk_ev[1], 0);
  if (!rc && (e1 != cudaSuccess || e2 != cudaSuccess)) return fail(h, WPK_ERR_CUDA, "stream join failed");
  return rc;
}

// Head c may start once the caller's stream has finished chunk c's backbone.
static int chunk_handoff(wpk_handle* h, int c, cudaStream_t s) {
  CUDA_TRY(h, cudaEventRecord(h->chunk_ev[2 + c], s));
  CUDA_TRY(h, cudaStreamWaitEvent(h->head_stream, h->chunk_ev[2 + c], 0));
  return WPK_OK;
}

static int chunked_prefill(wpk_handle* h, const int32_t* tokens_dev, int batch, int prompt_len,
                           int32_t* first_tok_dev, float* logits_dev, cudaStream_t s) {
  if (!tokens_dev || batch <= 0 || prompt_len <= 0) return fail(h, WPK_ERR_INVALID_ARG, "bad prefill arguments");
  const int C = 1 + (int)h->chunks.size(), bc = h->chunk_rows, K = h->n_cb, V = h->cb_vocab;
  if (batch > bc * C) return fail(h, WPK_ERR_SHAPE, "batch or prompt exceeds the plan");
  int rc = chunk_streams(h);
  if (rc) return rc;
  // every head's batch is set before any launch, so nothing below waits on a head
  std::vector<int32_t> n(C);
  for (int c = 0; c < C; ++c) {
    wpk_handle* x = pair_of(h, c);
    n[c] = std::max(0, std::min(bc, batch - c * bc));
    x->batch = n[c];
    x->prefilled = false;
    if (!n[c]) continue;
    rc = reset_step_state(x->head, s);
    if (rc) return rc;
    CUDA_TRY(h, cudaMemcpyAsync(x->head->d_active, &n[c], 4, cudaMemcpyHostToDevice, s));
  }
  CUDA_TRY(h, cudaStreamSynchronize(s));  // `n` lives on this stack frame
  rc = chunk_fork(h, s);
  if (rc) return rc;
  for (int c = 0; c < C && !rc && n[c]; ++c) {
    wpk_handle* x = pair_of(h, c);
    const size_t r0 = (size_t)c * bc;
    int32_t* codes = reinterpret_cast<int32_t*>(x->scratch + x->off_codes);
    rc = prefill_impl(x, tokens_dev + r0 * prompt_len, n[c], prompt_len, codes,
                      reinterpret_cast<float*>(x->scratch + x->off_p), s);
    if (!rc) rc = chunk_handoff(h, c, s);
    if (rc) break;
    x->head->batch = n[c];
    x->head->prefilled = true;
    int32_t* out = first_tok_dev ? first_tok_dev + r0 * K : codes;
    rc = head_frame(x, out, logits_dev ? logits_dev + r0 * K * V : nullptr, h->head_stream);
    if (!rc && first_tok_dev &&
        cudaMemcpyAsync(codes, out, (size_t)n[c] * K * 4, cudaMemcpyDeviceToDevice, h->head_stream) != cudaSuccess)
      rc = fail(h, WPK_ERR_CUDA, "copying a chunk's codes failed");
    else if (x != h && rc)
      h->err = x->err;
  }
  return chunk_join(h, s, rc);
}

int wpk_prefill(wpk_handle* h, const int32_t* tokens_dev, int batch, int prompt_len, int32_t* first_tok_dev,
                float* logits_dev, void* stream) {
  if (!h || !h->head) return prefill_impl(h, tokens_dev, batch, prompt_len, first_tok_dev, logits_dev, stream);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!h->chunks.empty()) {
    int rc = check_live(h);
    if (rc) return rc;
    return chunked_prefill(h, tokens_dev, batch, prompt_len, first_tok_dev, logits_dev, s);
  }
  // two-stage: the prompt through the backbone, whose output head yields the
  // projection p at the last position; then the head's first frame
  int32_t* codes = reinterpret_cast<int32_t*>(h->scratch + h->off_codes);
  float* p = reinterpret_cast<float*>(h->scratch + h->off_p);
  int rc = prefill_impl(h, tokens_dev, batch, prompt_len, codes, p, stream);
  if (rc) return rc;
  wpk_handle* hh = h->head;
  rc = reset_step_state(hh, s);
  if (rc) return rc;
  CUDA_TRY(h, cudaMemcpyAsync(hh->d_active, &batch, 4, cudaMemcpyHostToDevice, s));
  CUDA_TRY(h, cudaStreamSynchronize(s));  // `batch` lives on this stack frame
  hh->batch = batch;
  hh->prefilled = true;
  rc = head_frame(h, first_tok_dev ? first_tok_dev : codes, logits_dev, s);
  if (rc) return rc;
  if (first_tok_dev)
    CUDA_TRY(h, cudaMemcpyAsync(codes, first_tok_dev, (size_t)batch * h->n_cb * 4, cudaMemcpyDeviceToDevice, s));
  return WPK_OK;
}

static int prefill_impl(wpk_handle* h, const int32_t* tokens_dev, int batch, int prompt_len, int32_t* first_tok_dev,
                        float* logits_dev, void* stream) {
  int rc = check_live(h);
  if (rc) return rc;
  rc = res_shutdown(h);
  if (rc) return rc;
  if (!h->loaded) return fail(h, WPK_ERR_NOT_LOADED, "weights not loaded");
  if (!tokens_dev || batch <= 0 || prompt_len <= 0) return fail(h, WPK_ERR_INVALID_ARG, "bad prefill arguments");
  if (batch > h->g.plan.max_batch || prompt_len > h->g.plan.max_context)
    return fail(h, WPK_ERR_SHAPE, "batch or prompt exceeds the plan");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = reset_step_state(h, s);
  if (rc) return rc;
  CUDA_TRY(h, cudaMemcpyAsync(h->d_active, &batch, 4, cudaMemcpyHostToDevice, s));
  CUDA_TRY(h, cudaStreamSynchronize(s));  // `batch` lives on this stack frame
  h->batch = batch;
  h->ctx = 0;
  if (h->g.plan.prefill_mode == WPK_PREFILL_MMA) {
    if ((int64_t)batch * prompt_len > h->prefill_max_tokens)
      return fail(h, WPK_ERR_SHAPE, "prompt tokens exceed the prefill scratch");
    PrefillProgram* prog = nullptr;
    rc = get_prefill_program(h, batch, prompt_len, &prog);
    if (rc) return rc;
    // positions count up from 0; the final tile advances them to prompt_len
    std::vector<int32_t> pos(h->g.plan.max_batch, prompt_len - 1);
    CUDA_TRY(h, cudaMemcpyAsync(h->d_seqlen, pos.data(), pos.size() * 4, cudaMemcpyHostToDevice, s));
    CUDA_TRY(h, cudaStreamSynchronize(s));  // `pos` lives on this stack frame
    rc = launch_prefill(h, prog, tokens_dev, first_tok_dev, logits_dev, s);
    if (rc) return rc;
    CUDA_TRY(h, cudaMemcpyAsync(h->h_err_code, &h->d_err->code, 4, cudaMemcpyDeviceToHost, s));
    CUDA_TRY(h, cudaGetLastError());
    h->ctx = prompt_len;
    h->prefilled = true;
    return WPK_OK;
  }
  // The prompt runs through the decode program one position at a time.
  for (int t = 0; t < prompt_len; ++t) {
    const bool last = (t + 1 == prompt_len);
    rc = step_impl(h, tokens_dev + t, prompt_len, last ? first_tok_dev : nullptr, last ? logits_dev : nullptr, s);
    if (rc) return rc;
  }
  h->prefilled = true;
  return WPK_OK;
}

// The backbone step of a two-stage frame: input sum_k frame_embed_k[c_k] of
// the codes at in_codes ([batch][K]); output p through the projection.
static int backbone_step(wpk_handle* h, const int32_t* in_codes, cudaStream_t s) {
  const int K = h->n_cb;
  h->io = wpk_handle::IO{};
  h->io.set = true;
  h->io.n_in = K;
  h->io.in_rows = h->cb_vocab;
  for (int k = 0; k < K; ++k) h->io.in_off[k] = h->frame_embed_off[k];
  h->io.lm_head_off = h->g.lay.lm_head;
  h->io.lm_mma_off = h->g.lay.lm_mma;
  h->io.logits_stride = h->g.plan.lm_rows;
  h->io.out_stride = 1;
  const int rc = step_impl(h, in_codes, K, nullptr, reinterpret_cast<float*>(h->scratch + h->off_p), s);
  h->io.set = false;
  return rc;
}

static int chunked_frame(wpk_handle* h, const int32_t* in_tok_dev, int32_t* out_tok_dev, float* logits_dev,
                         cudaStream_t s) {
  const int C = 1 + (int)h->chunks.size(), bc = h->chunk_rows, K = h->n_cb, V = h->cb_vocab;
  int rc = chunk_fork(h, s);
  if (rc) return rc;
  for (int c = 0; c < C && !rc; ++c) {
    wpk_handle* x = pair_of(h, c);
    if (!x->batch) break;
    const size_t r0 = (size_t)c * bc;
    int32_t* codes = reinterpret_cast<int32_t*>(x->scratch + x->off_codes);
    rc = backbone_step(x, in_tok_dev ? in_tok_dev + r0 * K : codes, s);
    if (!rc) rc = chunk_handoff(h, c, s);
    if (rc) {
      if (x != h) h->err = x->err;
      break;
    }
    int32_t* out = out_tok_dev ? out_tok_dev + r0 * K : codes;
    rc = head_frame(x, out, logits_dev ? logits_dev + r0 * K * V : nullptr, h->head_stream);
    if (!rc && out_tok_dev &&
        cudaMemcpyAsync(codes, out, (size_t)x->batch * K * 4, cudaMemcpyDeviceToDevice, h->head_stream) != cudaSuccess)
      rc = fail(h, WPK_ERR_CUDA, "copying a chunk's codes failed");
    else if (x != h && rc)
      h->err = x->err;
  }
  return chunk_join(h, s, rc);
}

// Fixed-cohort serving: refuse a step that would take a live slot past the
// context limit; after a step, the live slots hold one more token.
static int cohort_check(wpk_handle* h) {
  if (!h->cohort) return WPK_OK;
  for (size_t b = 0; b < h->slot_on.size(); ++b)
    if (h->slot_on[b] && h->slot_len[b] >= h->g.plan.max_context)
      return fail(h, WPK_ERR_SHAPE, "slot " + std::to_string(b) + " reached the context limit");
  return WPK_OK;
}
static void cohort_advance(wpk_handle* h) {
  if (!h->cohort) return;
  int mx = 0;
  for (size_t b = 0; b < h->slot_on.size(); ++b) {
    if (h->slot_on[b]) ++h->slot_len[b];
    if (h->slot_on[b]) mx = std::max(mx, h->slot_len[b]);
  }
  h->ctx = mx;
}

int wpk_set_active_slots(wpk_handle* h, const int32_t* active, int n) {
  int rc = check_live(h);
  if (rc) return rc;
  if (!active || n <= 0 || n > h->g.plan.max_batch) return fail(h, WPK_ERR_INVALID_ARG, "bad slot mask");
  if (h->head) return fail(h, WPK_ERR_UNSUPPORTED, "slot masks are for a single decoder");
  if (!h->cohort) return fail(h, WPK_ERR_NOT_LOADED, "no slot was filled with wpk_prefill_slots");
  for (int b = 0; b < n; ++b)
    if (active[b] && h->slot_len[b] == 0)
      return fail(h, WPK_ERR_INVALID_ARG, "slot " + std::to_string(b) + " holds no prefilled sequence");
  rc = res_shutdown(h);
  if (rc) return rc;
  std::vector<int32_t> m(n);
  for (int b = 0; b < n; ++b) {
    m[b] = active[b] ? 1 : 0;
    h->slot_on[b] = (char)(active[b] != 0);
  }
  CUDA_TRY(h, cudaDeviceSynchronize());  // no step of this handle is in flight
  CUDA_TRY(h, cudaMemcpy(h->d_slot_active, m.data(), (size_t)n * 4, cudaMemcpyHostToDevice));
  int mx = 0;
  for (size_t b = 0; b < h->slot_on.size(); ++b)
    if (h->slot_on[b]) mx = std::max(mx, h->slot_len[b]);
  h->ctx = mx;
  return WPK_OK;
}

int wpk_prefill_slots(wpk_handle* h, const int32_t* tokens_dev, int slot0, int batch, int prompt_len,
                      int32_t* first_tok_dev, float* logits_dev, void* stream) {
  int rc = check_live(h);
  if (rc) return rc;
  if (h->head) return fail(h, WPK_ERR_UNSUPPORTED, "slot prefill is for a single decoder");
  if (h->g.plan.prefill_mode != WPK_PREFILL_MMA)
    return fail(h, WPK_ERR_UNSUPPORTED, "slot prefill needs the tensor-core prefill program");
  if (!h->loaded) return fail(h, WPK_ERR_NOT_LOADED, "weights not loaded");
  const int B = h->g.plan.max_batch;
  if (!tokens_dev || batch <= 0 || prompt_len <= 0 || slot0 < 0)
    return fail(h, WPK_ERR_INVALID_ARG, "bad slot prefill arguments");
  if (slot0 + batch > B || prompt_len > h->g.plan.max_context)
    return fail(h, WPK_ERR_SHAPE, "slots or prompt exceed the plan");
  if ((int64_t)batch * prompt_len > h->prefill_max_tokens)
    return fail(h, WPK_ERR_SHAPE, "prompt tokens exceed the prefill scratch");
  rc = res_shutdown(h);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PrefillProgram* prog = nullptr;
  rc = get_prefill_program(h, batch, prompt_len, &prog);
  if (rc) return rc;
  if (!h->cohort) {  // entering the cohort mode: every slot empty and idle
    rc = reset_step_state(h, s);
    if (rc) return rc;
    CUDA_TRY(h, cudaMemsetAsync(h->d_slot_active, 0, (size_t)B * 4, s));
    h->cohort = true;
    h->slot_len.assign(B, 0);
    h->slot_on.assign(B, 0);
  }
  // the new slots: positions count up from 0 (the final tile advances them
  // to prompt_len), live from now on; the prefill runs `batch` sequences
  std::vector<int32_t> pos(batch, prompt_len - 1), on(batch, 1);
  CUDA_TRY(h, cudaMemcpyAsync(h->d_seqlen + slot0, pos.data(), (size_t)batch * 4, cudaMemcpyHostToDevice, s));
  CUDA_TRY(h, cudaMemcpyAsync(h->d_slot_active + slot0, on.data(), (size_t)batch * 4, cudaMemcpyHostToDevice, s));
  CUDA_TRY(h, cudaMemcpyAsync(h->d_active, &batch, 4, cudaMemcpyHostToDevice, s));
  CUDA_TRY(h, cudaStreamSynchronize(s));  // the sources live on this stack frame
  h->prefill_slot0 = slot0;
  rc = launch_prefill(h, prog, tokens_dev, first_tok_dev, logits_dev, s);
  h->prefill_slot0 = 0;
  if (rc) return rc;
  // the decode steps run every slot of the cohort
  h->cohort_batch = B;
  CUDA_TRY(h, cudaMemcpyAsync(h->d_active, &h->cohort_batch, 4, cudaMemcpyHostToDevice, s));
  CUDA_TRY(h, cudaMemcpyAsync(h->h_err_code, &h->d_err->code, 4, cudaMemcpyDeviceToHost, s));
  CUDA_TRY(h, cudaGetLastError());
  for (int b = 0; b < batch; ++b) {
    h->slot_len[slot0 + b] = prompt_len;
    h->slot_on[slot0 + b] = 1;
  }
  h->batch = B;
  h->ctx = 0;
  for (int b = 0; b < B; ++b)
    if (h->slot_on[b]) h->ctx = std::max(h->ctx, h->slot_len[b]);
  h->prefilled = true;
  return WPK_OK;
}

int wpk_step(wpk_handle* h, const int32_t* in_tok_dev, int32_t* out_tok_dev, float* logits_dev, void* stream) {
  int rc = check_live(h);
  if (rc) return rc;
  if (!h->loaded || !h->prefilled) return fail(h, WPK_ERR_NOT_LOADED, "weights or prefill missing");
  if (!h->cohort && h->ctx >= h->g.plan.max_context) return fail(h, WPK_ERR_SHAPE, "context limit reached");
  rc = cohort_check(h);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!h->head) {
    rc = step_impl(h, in_tok_dev, 1, out_tok_dev, logits_dev, s);
    if (!rc) cohort_advance(h);
    return rc;
  }
  if (!h->chunks.empty()) return chunked_frame(h, in_tok_dev, out_tok_dev, logits_dev, s);
  // two-stage frame: backbone step on sum_k frame_embed_k[c_k] -> p, then the head
  int32_t* codes = reinterpret_cast<int32_t*>(h->scratch + h->off_codes);
  rc = backbone_step(h, in_tok_dev ? in_tok_dev : codes, s);
  if (rc) return rc;
  rc = head_frame(h, out_tok_dev ? out_tok_dev : codes, logits_dev, s);
  if (rc) return rc;
  if (out_tok_dev)
    CUDA_TRY(h, cudaMemcpyAsync(codes, out_tok_dev, (size_t)h->batch * h->n_cb * 4, cudaMemcpyDeviceToDevice, s));
  return WPK_OK;
}

// The head's K steps of one frame: step k reads p (k = 0) or head_embed_k of
// code k-1, writes code k (and its logits) through output table k; the head's
// positions restart at 0.
static int head_frame(wpk_handle* h, int32_t* codes_out, float* logits, cudaStream_t s) {
  wpk_handle* hh = h->head;
  const int K = h->n_cb, V = h->cb_vocab;
  CUDA_TRY(h, cudaMemsetAsync(hh->d_seqlen, 0, (size_t)hh->g.plan.max_batch * 4, s));
  hh->ctx = 0;
  int rc = WPK_OK;
  for (int k = 0; k < K && !rc; ++k) {
    hh->io = wpk_handle::IO{};
    hh->io.set = true;
    if (k == 0) {
      hh->io.n_in = 0;
      hh->io.in_vec = reinterpret_cast<const float*>(h->scratch + h->off_p);
    } else {
      hh->io.n_in = 1;
      hh->io.in_off[0] = h->head_embed_off[k] - h->head_base;
    }
    hh->io.in_rows = V;
    hh->io.lm_head_off = h->out_head_off[k] - h->head_base;
    hh->io.lm_mma_off = h->out_head_mma_off[k] ? h->out_head_mma_off[k] - h->head_base : 0;
    hh->io.logits_stride = K * V;
    hh->io.out_stride = K;
    rc = step_impl(hh, k ? codes_out + (k - 1) : nullptr, K, codes_out + k, logits ? logits + (size_t)k * V : nullptr,
                   s);
  }
  hh->io.set = false;
  if (rc) {
    h->err = "head: " + hh->err;
    return rc;
  }
  if (*hh->h_err_code && !*h->h_err_code) *h->h_err_code = *hh->h_err_code;
  return WPK_OK;
}

int wpk_graph_stats_get(const wpk_handle* h, wpk_graph_stats* st) {
  if (!h || !st) return WPK_ERR_INVALID_ARG;
  memset(st, 0, sizeof *st);
  const CompiledGraph& g = selected_graph(h);
  st->n_tiles = (int64_t)g.tiles.size();
  st->n_counters = (int64_t)g.ctr_need.size();
  st->n_edges = g.n_edges;
  st->n_signals = (int64_t)g.sig.size();
  st->n_ops = (int64_t)g.groups.size();
  st->n_workers = h->n_workers;
  st->weight_bytes = g.algo_weight_bytes;
  st->n_regions = (int64_t)g.region_begin.size() - 1;
  for (size_t i = 0; i < g.region_begin.size() && i < 5; ++i) st->region_begin[i] = g.region_begin[i];
  return WPK_OK;
}

int wpk_get_edges(const wpk_handle* h, int32_t* pairs, int64_t max_pairs, int64_t* n_pairs) {
  if (!h || !n_pairs) return WPK_ERR_INVALID_ARG;
  int64_t k = 0;
  const CompiledGraph& g = selected_graph(h);
  for (size_t v = 0; v < g.preds.size(); ++v)
    for (int u : g.preds[v]) {
      if (pairs && k < max_pairs) {
        pairs[2 * k] = u;
        pairs[2 * k + 1] = (int32_t)v;
      }
      ++k;
    }
  *n_pairs = k;
  return WPK_OK;
}

int wpk_get_tile_ops(const wpk_handle* h, int32_t* ops, int64_t n) {
  if (!h || !ops) return WPK_ERR_INVALID_ARG;
  const CompiledGraph& g = selected_graph(h);
  if (n < (int64_t)g.tiles.size()) return WPK_ERR_INVALID_ARG;
  for (size_t i = 0; i < g.tiles.size(); ++i) ops[i] = g.tiles[i].op;
  return WPK_OK;
}

int wpk_get_tile_bytes(const wpk_handle* h, int64_t* bytes, int64_t n) {
  if (!h || !bytes) return WPK_ERR_INVALID_ARG;
  const CompiledGraph& g = selected_graph(h);
  if (n < (int64_t)g.tiles.size()) return WPK_ERR_INVALID_ARG;
  for (size_t i = 0; i < g.tiles.size(); ++i) bytes[i] = g.tiles[i].w_bytes;
  return WPK_OK;
}

int wpk_select_program(wpk_handle* h, int batch, int prompt_len) {
  if (!h) return WPK_ERR_INVALID_ARG;
  if (batch == 0) {
    h->selected = nullptr;
    return WPK_OK;
  }
  if (h->g.plan.prefill_mode != WPK_PREFILL_MMA)
    return fail(h, WPK_ERR_UNSUPPORTED, "the plan prefills token by token through the decode program");
  if (batch < 0 || prompt_len <= 0 || batch > h->g.plan.max_batch || prompt_len > h->g.plan.max_context)
    return fail(h, WPK_ERR_SHAPE, "batch or prompt exceeds the plan");
  PrefillProgram* prog = nullptr;
  int rc = get_prefill_program(h, batch, prompt_len, &prog);
  if (rc) return rc;
  h->selected = prog;
  return WPK_OK;
}

int wpk_verify_graph(const wpk_handle* h) {
  if (!h) return WPK_ERR_INVALID_ARG;
  std::string msg = verify_graph(selected_graph(h));
  if (!msg.empty()) {
    const_cast<wpk_handle*>(h)->err = msg;
    return WPK_ERR_SHAPE;
  }
  return WPK_OK;
}

int wpk_simulate(const wpk_handle* h, int n_threads, int n_epochs, uint64_t seed, int wait_ms, int stuck_tile,
                 int32_t* done_order) {
  if (!h || n_threads <= 0 || n_epochs <= 0 || wait_ms <= 0) return WPK_ERR_INVALID_ARG;
  std::string msg;
  int rc = simulate_graph(selected_graph(h), n_threads, n_epochs, seed, wait_ms, stuck_tile, done_order, &msg);
  if (rc) const_cast<wpk_handle*>(h)->err = msg;
  return rc;
}

int wpk_predict(const wpk_handle* h, const double* service_ns, const double* load_ns, const wpk_predict_cfg* cfg,
                double* out_ns) {
  if (!h || !service_ns || !load_ns || !cfg || !out_ns) return WPK_ERR_INVALID_ARG;
  std::string msg = predict_program(selected_graph(h), service_ns, load_ns, *cfg, out_ns);
  if (!msg.empty()) {
    const_cast<wpk_handle*>(h)->err = msg;
    return WPK_ERR_INVALID_ARG;
  }
  return WPK_OK;
}

int wpk_get_trace(wpk_handle* h, void* host_buf, size_t bytes) {
  if (!h || !host_buf) return WPK_ERR_INVALID_ARG;
  if (!h->has_device) return fail(h, WPK_ERR_CUDA, "no CUDA device");
  int rc = res_shutdown(h);
  if (rc) return rc;
  const CompiledGraph& g = selected_graph(h);
  const size_t need = g.tiles.size() * sizeof(TraceRec);
  if (bytes < need) return fail(h, WPK_ERR_INVALID_ARG, "trace buffer too small");
  if (!h->g.plan.trace) return fail(h, WPK_ERR_UNSUPPORTED, "plan was built without trace");
  CUDA_TRY(h, cudaDeviceSynchronize());
  CUDA_TRY(h, cudaMemcpy(host_buf, h->selected ? h->selected->d_trace : h->d_trace, need, cudaMemcpyDeviceToHost));
  return WPK_OK;
}

int wpk_get_error_info(wpk_handle* h, wpk_error_info* info) {
  if (!h || !info) return WPK_ERR_INVALID_ARG;
  if (!h->has_device) return fail(h, WPK_ERR_CUDA, "no CUDA device");
  int rc = res_shutdown(h);
  if (rc) return rc;
  CUDA_TRY(h, cudaDeviceSynchronize());
  // the first error among this program and (two-stage) the head and chunk pairs
  std::vector<const wpk_handle*> progs{h, h->head};
  for (const wpk_handle* c : h->chunks) {
    progs.push_back(c);
    progs.push_back(c->head);
  }
  ErrWord e{};
  for (const wpk_handle* x : progs) {
    if (!x || !x->d_err) continue;
    CUDA_TRY(h, cudaMemcpy(&e, x->d_err, sizeof e, cudaMemcpyDeviceToHost));
    if (e.code) break;
  }
  info->code = e.code;
  info->tile = e.tile;
  info->counter = e.counter;
  info->epoch = e.epoch;
  info->observed = e.observed;
  info->target = e.target;
  if (e.code) h->poisoned = true;
  return WPK_OK;
}

const char* wpk_last_error(const wpk_handle* h) { return h ? h->err.c_str() : g_build_error.c_str(); }

int wpk_destroy(wpk_handle* h) {
  if (!h) return WPK_ERR_INVALID_ARG;
  if (h->head) {
    wpk_destroy(h->head);
    h->head = nullptr;
  }
  for (wpk_handle* c : h->chunks) wpk_destroy(c);
  h->chunks.clear();
  if (h->head_stream) {
    cudaStreamSynchronize(h->head_stream);
    cudaStreamDestroy(h->head_stream);
  }
  for (cudaEvent_t e : h->chunk_ev) cudaEventDestroy(e);
  if (h->has_device) {
    res_shutdown(h);
    cudaDeviceSynchronize();
  }
  if (h->res_stream) cudaStreamDestroy(h->res_stream);
  if (h->res_ctl) cudaFreeHost((void*)h->res_ctl);
  for (auto& e : h->graphs) {
    if (e.exec) cudaGraphExecDestroy(e.exec);
    if (e.graph) cudaGraphDestroy(e.graph);
  }
  for (auto& p : h->prefills) {
    for (auto& e : p->graphs) {
      if (e.exec) cudaGraphExecDestroy(e.exec);
      if (e.graph) cudaGraphDestroy(e.graph);
    }
    if (p->d_base) cudaFree(p->d_base);
  }
  if (h->capture_stream) cudaStreamDestroy(h->capture_stream);
  if (h->d_base) cudaFree(h->d_base);
  if (h->h_err_code) cudaFreeHost(h->h_err_code);
  delete h;
  return WPK_OK;
}

// Step with a different scratch buffer (used by wpk_step_noalloc).  The
// megakernel reads the scratch address at every launch, so swapping it for one
// call changes nothing else; the per-op mode bakes addresses into a captured
// graph (and instantiating one may allocate), so it is not offered there.
int wpk_internal_step_scratch(wpk_handle* h, void* scratch, size_t scratch_bytes, const int32_t* in_tok_dev,
                              int32_t* out_tok_dev, float* logits_dev, void* stream) {
  int rc = check_live(h);
  if (rc) return rc;
  if (h->g.plan.mode != WPK_MEGAKERNEL)
    return fail(h, WPK_ERR_UNSUPPORTED, "wpk_step_noalloc needs the megakernel mode");
  if (h->head)
    return fail(h, WPK_ERR_UNSUPPORTED, "wpk_step_noalloc runs a single decoder, not the two-stage model");
  if (h->g.plan.resident)
    return fail(h, WPK_ERR_UNSUPPORTED, "wpk_step_noalloc needs a launch per step (the resident grid keeps its "
                                        "scratch pointer for its lifetime)");
  if (h->g.plan.decode_mode == WPK_DECODE_MMA)
    return fail(h, WPK_ERR_UNSUPPORTED, "wpk_step_noalloc needs the GEMV decode program (the tensor-core "
                                        "decode program keeps sums in its scratch between steps)");
  // only the decode step's part of the scratch moves into the static array;
  // the prefill program keeps the caller's buffer
  if (h->decode_scratch_bytes > scratch_bytes)
    return fail(h, WPK_ERR_SHAPE, "the decode step needs " + std::to_string(h->decode_scratch_bytes) +
                                      " scratch bytes, more than the " + std::to_string(scratch_bytes) +
                                      " bytes of the static scratch array");
  if (!h->loaded || !h->prefilled) return fail(h, WPK_ERR_NOT_LOADED, "weights or prefill missing");
  int dev = -1;
  CUDA_TRY(h, cudaGetDevice(&dev));
  if (dev != h->device) return fail(h, WPK_ERR_INVALID_ARG, "current device is not the handle's device");
  if (!h->cohort && h->ctx >= h->g.plan.max_context) return fail(h, WPK_ERR_SHAPE, "context limit reached");
  rc = cohort_check(h);
  if (rc) return rc;
  uint8_t* saved = h->scratch;
  h->scratch = static_cast<uint8_t*>(scratch);
  rc = step_impl(h, in_tok_dev, 1, out_tok_dev, logits_dev, static_cast<cudaStream_t>(stream));
  h->scratch = saved;
  if (!rc) cohort_advance(h);
  return rc;
}

int wpk_debug_break_counter(wpk_handle* h, int counter) {
  if (!h || counter < 0 || counter >= (int)h->g.ctr_need.size()) return WPK_ERR_INVALID_ARG;
  if (h->has_device && res_shutdown(h)) return WPK_ERR_CUDA;
  for (auto& t : h->g.tiles)
    if (t.wait_ctr == (uint32_t)counter) t.need += 1;
  if (!h->has_device) return WPK_OK;
  CUDA_TRY(h, cudaMemcpy(h->d_tiles, h->g.tiles.data(), h->g.tiles.size() * sizeof(Tile), cudaMemcpyHostToDevice));
  return WPK_OK;
}

}  // extern "C"
