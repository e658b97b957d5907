// Internal tables shared by the host graph compiler (graph.cpp), the C ABI
// (capi.cu) and the persistent kernel (runtime.cu).
#pragma once
#include <stddef.h>
#include <stdint.h>

#include "../../include/wpk.h"

namespace wpk {

constexpr uint32_t kNoCounter = 0xFFFFFFFFu;
constexpr int kThreads = 256;          // consumer (compute) threads per worker CTA
constexpr int kWarps = kThreads / 32;
constexpr int kCtaThreadsGemv = kThreads + 32;  // + the producer warp
constexpr int kCtaThreadsTc = kThreads + 64;    // + the producer warp + the tensor-core issuer warp
constexpr int kStageBytes = 16384;     // one chunk stage of the staging ring
constexpr int kMaxStages = 13;         // ring stages per worker
// GEMV chunks (kStageBytes each) per ring stage of a staging slot of `slot`
// bytes: two per stage, one copy each, when the slot holds two (a worker
// issues and completes about one stage per half microsecond whatever its
// size, so 16 KB stages cap a worker near 30 GB/s), and the chunks the slot
// holds at once in whole stages.
inline int gemv_chunks_per_stage(int slot) { return slot >= 2 * kStageBytes ? 2 : 1; }
inline int gemv_ring_chunks(int slot) {
  const int c = gemv_chunks_per_stage(slot);
  return slot / (c * kStageBytes) * c;
}
constexpr int kMaxQueue = 8;           // tiles a worker may hold (lookahead)
constexpr int kMaxGemvBatch = 8;       // token rows per GEMV pass
// largest batch the automatic choice decodes on CUDA cores (B200, 1B shape:
// the GEMV step at 4 sequences matches the tensor-core step, at 8 it takes
// twice as long)
constexpr int kAutoGemvBatch = 4;
constexpr int kMaxTileRows = 128;      // rows per GEMV tile (partial-output buffer)
constexpr int kMaxGroup = 8;           // q heads per kv head handled by one attention tile
constexpr int kHeadDim = 64;           // the head dimension the attention tiles are written for
constexpr int kMaxSmem = 232448;       // dynamic shared memory per CTA on sm_100

// Op codes of the tiles.  One "op group" = the tiles of one op of one layer.
enum Op : uint16_t {
  OP_EMBED = 0,    // x = E[tok]
  OP_QKV = 1,      // fused RMSNorm + [q;k;v] = W a + RoPE + KV-cache write
  OP_ATTN = 2,     // split-KV GQA decode attention + last-arriver combine
  OP_O = 3,        // x_mid = x + Wo attn  (also re-initialises x for down)
  OP_GU = 4,       // fused RMSNorm + gate/up + SwiGLU
  OP_DOWN = 5,     // x += Wd h  (split-K, accumulated)
  OP_LMHEAD = 6,   // fused final RMSNorm + logits + packed argmax
  OP_FINAL = 7,    // publish tokens, reset argmax, advance positions
  // prefill program (token blocks of kTokBlock rows; tensor-core tiles)
  OP_PEMBED = 8,   // X[block] = E[prompt tokens]
  OP_NORM = 9,     // RMSNorm of X[block] -> bf16 hi/lo activation image
  OP_MQKV = 10,    // [q;k;v] = W . a on tensor cores, RoPE, q -> Q, k/v -> KV cache
  OP_MO = 11,      // X += Wo . attn on tensor cores
  OP_MGU = 12,     // gate/up on tensor cores, SwiGLU -> hi/lo image of h
  OP_MDOWN = 13,   // X += Wd . h on tensor cores
  OP_PATTN = 14,   // causal GQA attention of one query block (tensor cores)
  OP_GATHER = 15,  // xa[b] = X[last prompt position of b]
  // batched decode program (the step's tokens are the MMA N dimension)
  OP_BQKV = 16,    // [q;k;v] partial over a K range on tensor cores, RoPE, summed into acc
  OP_BO = 17,      // x += Wo . attn over a K range; last split -> RMSNorm input image
  OP_BGU = 18,     // gate/up on tensor cores, SwiGLU -> hi/lo image of h
  OP_BDOWN = 19,   // x += Wd . h over a K range; last split -> RMSNorm input image
  OP_BLM = 20,     // logits on tensor cores + packed argmax
  OP_COUNT = 21
};

constexpr int kTokBlock = 128;   // tokens per tensor-core tile (the MMA N)
constexpr int kNormRows = 16;    // token rows per prefill RMSNorm tile
constexpr int kMaxKeySplits = 8; // key splits of one prefill attention tile, at most
constexpr int kMaxMmaBatch = 128;  // sequences of a batched decode step (MMA N <= 128)
constexpr int kMaxInTables = 16;   // input tables a step's input may sum over
constexpr int kMmaChunkBytes = 128 * 128;  // 128 rows x 64 bf16, one K chunk

// One tile of the step program, in ticket order.  48 bytes.
struct alignas(16) Tile {
  uint16_t op;
  uint16_t layer;
  uint32_t wait_ctr;   // counter to wait on, or kNoCounter
  uint32_t need;       // signals that counter receives per step
  uint32_t sig_off;    // first entry of this tile's signal list
  uint32_t sig_cnt;    // counters it increments when done
  uint32_t w_bytes;    // bytes staged into the worker's slot before the wait
  uint64_t w_off;      // byte offset of those bytes in the weight image
  int32_t a0, a1, a2, a3;  // op arguments (see runtime.cu)
};
static_assert(sizeof(Tile) == 48, "Tile layout");

// Device-side offsets of one layer's tensors in the weight image (bytes).
struct LayerDev {
  uint64_t attn_norm;   // fp32 [hidden]
  uint64_t ffn_norm;    // fp32 [hidden]
  uint64_t qkv;         // bf16 [qkv_rows][hidden], RoPE pairs adjacent
  uint64_t wo;          // bf16 [hidden][q_rows]
  uint64_t gu;          // bf16 [2*ffn][hidden], gate/up rows interleaved
  uint64_t down;        // bf16 [n_kchunks][hidden][kc]
  // tensor-core image: [rows/128][K/64] blocks of 128 rows x 64 columns, each
  // 16 KB block stored with the 128-byte swizzle (0 when not built)
  uint64_t mma_qkv, mma_wo, mma_gu, mma_down;
};

struct TraceRec {
  uint32_t tile;
  uint16_t worker;
  uint16_t op;
  uint32_t ev_issue, ev_start, ev_done, epoch;
  uint64_t t_claim_ns, t_issued_ns, t_start_ns, t_data_ns, t_end_ns;
};
static_assert(sizeof(TraceRec) == sizeof(wpk_trace_rec), "trace layout");

// Resident grid control block in mapped (pinned) host memory: the host rings
// the doorbell with the step number (steps count from 1 per grid launch) after
// writing the step's I/O pointers; the last tile of a step stores its number
// in `ack` after a system-scope fence.
constexpr uint32_t kResShutdown = 0xFFFFFFFFu;
struct ResCtl {
  volatile uint32_t db;        // host: last step requested, or kResShutdown
  volatile uint32_t ack;       // device: last step completed
  volatile int32_t err;        // device: copy of the error word's code
  volatile int32_t in_stride;  // step input: token stride
  volatile uint64_t in_tok, out_tok, logits;  // step I/O device pointers (0 = none)
  volatile uint64_t t_done_ns; // device %globaltimer when the last step completed
};

// Device-memory copy of the doorbell and step I/O: worker 0 alone polls the
// mapped control block and publishes each step here (release), so the other
// workers poll L2 instead of host memory.
struct ResDev {
  uint32_t db;
  int32_t in_stride;
  uint64_t in_tok, out_tok, logits;
};

struct ErrWord {
  int32_t code;
  uint32_t tile, counter, epoch, observed, target;
};

// Everything a kernel launch needs.  Passed by value.
struct KParams {
  // model shape
  int n_layers, hidden, n_heads, n_kv, head_dim, ffn, vocab, group;
  int q_rows, kv_rows, qkv_rows, down_kc, n_down_chunks;
  float eps;
  // plan
  int max_batch, max_context, page_tokens, max_blocks, split_tokens, n_splits;
  int n_stages, lookahead, act_bytes;
  uint64_t timeout_ns;
  int trace;
  // device buffers (weights image and KV are caller-owned)
  const uint8_t* weights;
  const LayerDev* layers;
  uint64_t final_norm_off;   // fp32 [hidden]
  uint64_t embed_off;        // bf16 [vocab][hidden]
  uint64_t lm_head_off;      // bf16 [vocab][hidden]
  uint16_t* kv;              // bf16 [n_layers][n_blocks][2][n_kv][page][head_dim]
  int64_t n_blocks;
  const int32_t* block_table;  // [max_batch][max_blocks]
  const float2* rope;          // (cos, sin) [max_context][head_dim/2]
  // scratch (caller-owned)
  float* xa;       // [max_batch][hidden]   residual stream
  float* xb;       // [max_batch][hidden]   residual after attention (read by FFN)
  float* qbuf;     // [max_batch][q_rows]   roped queries
  float* attn;     // [max_batch][q_rows]   attention output
  float* hbuf;     // [max_batch][ffn]      SwiGLU output
  float* part;     // [max_batch][n_kv][n_splits][group][2 + head_dim] partials
  // library-owned state
  uint32_t* arrive;          // [max_batch][n_kv] split arrivals
  unsigned long long* best;  // [max_batch] packed argmax keys
  int32_t* seqlen;           // [max_batch] tokens already in the cache
  int32_t* tok_fb;           // [max_batch] last greedy tokens
  int32_t* active_batch;     // [1]
  // fixed-cohort serving: slot b of the decode programs is stepped only when
  // slot_active[b] != 0; an inactive slot gets a neutral input (code 0, RoPE
  // position 0), writes nothing to its KV cache, keeps its position and last
  // token, and outputs -1.  The prefill program writes sequence b's cache and
  // state into slot slot0 + b.
  const int32_t* slot_active;  // [max_batch]
  int slot0;
  const Tile* tiles;
  const uint32_t* sig;
  uint32_t* ctr;
  uint32_t* head;            // queue heads, one per region
  ErrWord* err;
  TraceRec* trace_buf;
  uint32_t* evclock;
  // per-step I/O
  const int32_t* in_tok;     // NULL = tok_fb
  int in_tok_stride;
  int32_t* out_tok;          // may be NULL
  float* logits;             // may be NULL
  // launch
  uint32_t t_begin, t_end;   // ticket range of this launch
  uint32_t epoch;            // counter target multiplier (>= 1)
  int region;
  int per_op;                // 1: one tile per CTA, no queue, no counters
  int static_sched;          // 1: worker w takes tickets w, w + W, ... (no queue)
  int team_sched;            // 1: worker w walks stream[stream_begin[w] .. stream_begin[w + 1])
  const uint32_t* stream_begin;  // [W + 1]
  const uint32_t* stream;        // tickets of every worker's stream
  int resident;              // 1: tickets run on across steps (epoch = ticket / tiles + 1)
  uint64_t idle_ns;          // resident: how long a worker waits for the next step
  ResCtl* ctl;               // resident: control block (device view of mapped memory)
  ResDev* rdev;              // resident: its device-memory copy
  int stage_bytes;           // bytes per staging-ring stage
  // GEMV chunks per stage: a GEMV tile's rows are cut into chunks of
  // stage_bytes / gemv_cps bytes (one warp each), gemv_cps consecutive
  // chunks staged with one copy; the stage's empty barrier takes gemv_cps
  // arrivals in the GEMV decode program (1 elsewhere)
  int gemv_cps;
  int uses_tmem;             // the program has tensor-core tiles
  // prefill program (token rows m = b * T + t, M = B * T, blocks of 128)
  int M, T, n_tb;
  const int32_t* ptok;       // prompt tokens [M]
  float* px;                 // [M][hidden] residual stream
  float* pq;                 // [M][q_rows] roped queries
  uint8_t* xn_img[2];        // hi/lo image of the normalised activations [n_tb][hidden/64][16 KB]
  uint8_t* att_img[2];       // hi/lo image of the attention output     [n_tb][q_rows/64][16 KB]
  uint8_t* h_img[2];         // hi/lo image of the SwiGLU output        [n_tb][ffn/64][16 KB]
  // prefill attention split along keys (small batches, where the (sequence,
  // kv head, query block) tiles are fewer than the workers): keys per split
  // (0 = no split), the splits' partial (m, l, o) per query row, and an
  // arrival counter per (sequence, kv head, query block)
  int pattn_ks;
  float* ppart;              // [tiles][kMaxKeySplits][128 rows][2 + head_dim]
  uint32_t* pattn_arrive;    // [workers]
  // tensor-core operand geometry: the MMA N (tokens per tile) and the bytes of
  // one 64-column activation chunk (N rows of 128 bytes, 128-byte swizzle)
  int mma_n, act_chunk;
  // bytes between two consecutive 64-column chunks of an activation image
  // (batched decode: 2 act_chunk, the hi and the lo rows of a chunk adjacent;
  // prefill: the hi and lo images are separate, one chunk apart), and the K
  // chunks a tensor-core tile stages per ring stage (1 or 2)
  int img_stride, mma_cps;
  // accumulators a tile rotates its K-steps over (2 mma_n TMEM columns each),
  // the columns of one tile's accumulator buffer (2 mma_n mma_acc; a worker
  // holds two, so that one tile's epilogue overlaps the next tile's MMAs) and
  // the TMEM columns a worker allocates (a power of two >= 2 mma_buf_cols)
  int mma_acc, mma_buf_cols, tmem_cols;
  // batched decode program (dec_mma = 1).  Token n of the step is MMA column n;
  // columns >= the active batch hold zeros.  Images are [K/64][act_chunk].
  int dec_mma;
  int o_splits, down_splits;  // K splits of the O and down projections
  float* xt;                  // [hidden][mma_n] residual stream, feature-major
  float* acc;                 // [qkv_rows][mma_n] q/k/v sums (zero between uses)
  float* ss;                  // [2 n_layers + 1][mma_n] sums of x^2 per RMSNorm
  uint8_t* xf_img[2];         // hi/lo image of x * g_ffn (xn_img holds x * g_attn / g_final)
  uint32_t* rb_arrive;        // [n_layers][2][hidden/128] split-K arrivals per row block
  uint64_t lm_mma_off;        // tensor-core image of the LM head [lm_rows/128][hidden/64][16 KB]
  // output head and step I/O layout: LM head tiles hold offsets relative to
  // lm_head_off / lm_mma_off, so one program can switch output tables per launch
  int lm_rows;                // rows of the output head (= vocab for a plain decoder)
  int logits_stride;          // floats between two sequences' logits
  int out_stride;             // int32s between two sequences' output tokens
  // step input: x = sum over n_in tables of table_k[code_k] (codes at
  // in_tok[b * stride + k], below in_rows), or the vector in_vec[b][hidden]
  // when n_in == 0
  int n_in, in_rows;
  uint64_t in_table_off[kMaxInTables];
  const float* in_vec;
};

// Host-side compiled graph.
struct Access {
  int buf;
  int64_t lo, hi;
  int kind;        // 0 = read, 1 = write, 2 = accumulate (commutes with itself)
  int group = -1;  // writes with the same group id (>= 0) form one logical write
};

enum Buf {
  BUF_XA = 0, BUF_XB, BUF_QKV, BUF_ATTN, BUF_H, BUF_LOGITS, BUF_BEST, BUF_TOK,
  // prefill buffers, modelled per token block (index = block * width * 128 + feature * 128 + row)
  BUF_PX, BUF_PXN, BUF_PQ, BUF_PKV, BUF_PATT, BUF_PH,
  // batched decode: the RMSNorm input images (x * g_attn or g_final; x * g_ffn)
  BUF_DXN, BUF_DXF,
  BUF_COUNT
};

struct OpGroup {
  int op, layer;
  uint32_t begin, end;  // ticket range
};

}  // namespace wpk
