/*
 * wpk.h - C ABI of the persistent decode/prefill library for one B200 (sm_100a).
 *
 * The library runs one recurring decoder update - a Llama-style decode step,
 * and the prompt prefill that yields the first token - as a persistent GPU
 * program instead of a sequence of kernel launches.  Resident workers (one or
 * more CTAs per SM) pull tiles from a device-side ticket queue; a host-built
 * tile graph with per-tile dependency counters replaces the barriers between
 * ops ("One Megakernel is Not Enough", Table I: cross-kernel readiness); each
 * tile's weight load is issued into its worker's staging slot before its
 * predecessors finish (Table I: weight prefetch); tensors consumed inside one
 * tile are not stored and reloaded (Table I: on-chip forwarding).  The same
 * tiles can also run as 1-4 region launches or as per-op launches captured in
 * a CUDA Graph, so compositions can be compared ("One Megakernel is Not
 * Enough", abstract and Fig. 3; "Persistent threads and megakernels", §7).
 *
 * Conventions for every entry point:
 *   - Return value: WPK_OK (0) or a negative WPK_ERR_* code.  Nothing aborts,
 *     traps or exits the process.  wpk_last_error() gives a message.
 *   - Pointers named *_dev are CUDA device pointers; everything else is host.
 *   - `stream` arguments are cudaStream_t values passed as void* (NULL = the
 *     legacy default stream).
 *   - A handle is not thread-safe: use it from one host thread at a time.
 *   - Ownership: the caller allocates and owns the three large device buffers
 *     sized by wpk_workspace_size (weights, KV pages, scratch) and keeps them
 *     alive until wpk_destroy.  The library owns the handle, its host tables
 *     and small device tables (tiles, counters, queue heads, trace, error word).
 *   - After WPK_ERR_TIMEOUT the handle is poisoned: every call but
 *     wpk_last_error / wpk_get_error_info / wpk_get_trace / wpk_destroy returns
 *     WPK_ERR_POISONED.
 */
#ifndef WPK_H_
#define WPK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ codes */
enum {
  WPK_OK = 0,
  WPK_ERR_INVALID_ARG = -1,  /* bad pointer, size or enum value            */
  WPK_ERR_CUDA = -2,         /* a CUDA runtime call failed                  */
  WPK_ERR_TIMEOUT = -3,      /* a device or host wait gave up (stall)       */
  WPK_ERR_NOT_LOADED = -4,   /* weights / prefill missing                   */
  WPK_ERR_SHAPE = -5,        /* shape outside what the plan was built for   */
  WPK_ERR_UNSUPPORTED = -6,  /* valid request this build does not implement */
  WPK_ERR_POISONED = -7      /* handle unusable after a timeout             */
};

enum { WPK_MEGAKERNEL = 0, WPK_PER_OP_GRAPH = 1 };
enum { WPK_SCHED_QUEUE = 0, WPK_SCHED_STATIC = 1, WPK_SCHED_TEAMS = 2 };
enum { WPK_PREFILL_AUTO = 0, WPK_PREFILL_MMA = 1, WPK_PREFILL_TOKENWISE = 2 };
enum { WPK_DECODE_AUTO = 0, WPK_DECODE_GEMV = 1, WPK_DECODE_MMA = 2 };

/* --------------------------------------------------------------- configs */
/* Decoder shape.  Weights are bf16, matmul weights stored [out][in].
 *
 * Two-stage streaming model ("Why real-time inference wants a megakernel":
 * a backbone step followed by a short sequence of dependent head steps per
 * frame; "One Megakernel is Not Enough", Table I, the two-stage TTS rows):
 * set n_codebooks > 0 and `head` to the head decoder's shape.  The decoder
 * described by the other fields is then the backbone; per frame and sequence
 *   p = W_proj . RMSNorm(backbone state)          (the backbone's output head)
 *   head step k (0..n_codebooks-1) reads p (k = 0) or head_embed_k[c_(k-1)],
 *   c_k = argmax(out_head_k . RMSNorm(head state)), the head's cache restarting
 *   every frame; the next backbone input is sum_k frame_embed_k[c_k].
 * wpk_prefill / wpk_step then produce codes [B][n_codebooks] per frame (and
 * logits [B][n_codebooks][codebook_vocab] when asked); the step's input is
 * the previous frame's codes.  Two-stage handles run in WPK_MEGAKERNEL mode,
 * without a resident grid. */
typedef struct wpk_model_cfg {
  int n_layers, hidden, n_heads, n_kv_heads, head_dim, ffn, vocab;
  float rms_eps, rope_theta;
  int tied_embedding;   /* 1: the LM head is the token embedding */
  int n_codebooks;      /* two-stage model: codebooks per frame (<= 16), else 0      */
  int codebook_vocab;   /* two-stage model: codes per codebook                      */
  const struct wpk_model_cfg *head;  /* two-stage model: the head decoder (its vocab,
                                        n_codebooks and head fields are ignored) */
} wpk_model_cfg;

/* Execution plan: the operating point the program is compiled for ("Why
 * real-time inference wants a megakernel", section "The cohort is known":
 * a model, a device, a session capacity and a context limit).  Zero fields
 * take the defaults noted. */
typedef struct wpk_plan_cfg {
  int max_batch;        /* sequences per step (session capacity)               */
  int max_context;      /* tokens per sequence, prompt included                */
  int page_tokens;      /* KV page size in tokens (0 = 64)                     */
  int n_workers;        /* resident worker CTAs (0 = #SMs x workers_per_sm)    */
  int workers_per_sm;   /* 0 = 1                                               */
  int mode;             /* WPK_MEGAKERNEL or WPK_PER_OP_GRAPH                  */
  int resident;         /* megakernel only: 1 = the grid stays alive across
                           steps and is driven by a host doorbell              */
  int n_regions;        /* megakernel only: 1..4 launches per step (0 = 1)     */
  int region_cut[4];    /* first layer of each region; region_cut[0] = 0; a cut
                           equal to n_layers puts the LM head in its own region */
  int trace;            /* 1 = record the per-tile device trace                */
  uint64_t wait_timeout_ns; /* bound on every device wait (0 = 2 s)            */
  int slot_bytes;       /* staging slot per worker, used as a ring of 16 KB
                           chunk stages (0 = 12 stages, 192 KB, or what fits) */
  int tile_bytes;       /* minimum weight bytes per tile; tiles are sized to give
                           each worker about one tile per op (0 = 32768, or
                           65536 for tensor-core decode tiles)                 */
  int split_pages;      /* KV pages per attention tile (split); 0 = chosen so that
                           a step has about two attention tiles per worker     */
  int lookahead;        /* tiles a worker may claim and stage ahead of the one
                           it computes (0 = 4); 1 = a tile's weights are staged
                           only after the previous tile of that worker is done */
  int schedule;         /* WPK_SCHED_QUEUE (0): tickets from one atomic device
                           queue; WPK_SCHED_STATIC: worker w takes tickets
                           w, w + W, w + 2W, ... (W workers), no atomics;
                           WPK_SCHED_TEAMS: every op of the step is given a
                           team of workers (all, a half, a quarter, ... one),
                           the least loaded one, and each worker walks its own
                           compiled stream of tiles; an edge between two tiles
                           of one worker's stream needs no counter (decode
                           program, one region, launch per step; the prefill
                           program runs the static streams)                  */
  int prefill;          /* WPK_PREFILL_AUTO (0): the tensor-core prefill program
                           when the shapes allow, else token by token;
                           WPK_PREFILL_MMA; WPK_PREFILL_TOKENWISE (the prompt
                           runs through the decode program one position at a
                           time)                                                */
  int decode;           /* WPK_DECODE_AUTO (0): tensor-core decode tiles when
                           max_batch > 4 and the shapes allow, else CUDA-core
                           GEMV tiles; WPK_DECODE_GEMV; WPK_DECODE_MMA (the
                           step's sequences are the MMA N dimension, so
                           max_batch <= 128)                                    */
  int frame_chunks;     /* two-stage model only.  0 or 1: a frame is the backbone
                           step, then the head steps, each on all workers.
                           C >= 2 (C <= max_batch, C <= 8): the sequences split
                           into C chunks of ceil(max_batch / C), each with its
                           own backbone and head programs over one shared weight
                           image.  Per frame, the backbones run chunk after chunk
                           on the caller's stream and the heads on a second
                           stream, as separate persistent launches on disjoint
                           worker sets; the head of chunk c starts as soon as the
                           backbone has finished chunk c, overlapping the
                           backbone of chunk c + 1 ("One Megakernel is Not
                           Enough", Table I, producer-consumer overlap).  The
                           call returns with the caller's stream ordered after
                           the whole frame.  wpk_set_block_table is not
                           supported then; the inspection calls (stats,
                           edges, trace, program selection) see chunk 0's
                           backbone program.                                    */
  int head_workers;     /* frame_chunks >= 2: worker CTAs of the head programs
                           (0 = half of the workers); the backbones take the
                           rest of n_workers (0 = #SMs x workers_per_sm)        */
} wpk_plan_cfg;

/* Host weights: bf16 bit patterns, row-major [out][in]. */
typedef struct wpk_layer_weights {
  const uint16_t *attn_norm;   /* [hidden]                     */
  const uint16_t *wq;          /* [n_heads*head_dim][hidden]   */
  const uint16_t *wk;          /* [n_kv_heads*head_dim][hidden]*/
  const uint16_t *wv;          /* [n_kv_heads*head_dim][hidden]*/
  const uint16_t *wo;          /* [hidden][n_heads*head_dim]   */
  const uint16_t *ffn_norm;    /* [hidden]                     */
  const uint16_t *w_gate;      /* [ffn][hidden]                */
  const uint16_t *w_up;        /* [ffn][hidden]                */
  const uint16_t *w_down;      /* [hidden][ffn]                */
} wpk_layer_weights;

typedef struct wpk_weights {
  const uint16_t *embed;             /* [vocab][hidden]                      */
  const uint16_t *final_norm;        /* [hidden]                             */
  const uint16_t *lm_head;           /* [vocab][hidden]; NULL when tied      */
  const wpk_layer_weights *layers;   /* [n_layers]                           */
  /* two-stage model only (NULL otherwise); K = n_codebooks, V = codebook_vocab */
  const uint16_t *proj;                   /* [head.hidden][hidden]                 */
  const uint16_t *const *frame_embed;     /* K tables [V][hidden]                  */
  const uint16_t *const *head_embed;      /* K tables [V][head.hidden]; entry 0 unused */
  const uint16_t *const *out_head;        /* K tables [V][head.hidden]             */
  const wpk_layer_weights *head_layers;   /* [head.n_layers]                       */
  const uint16_t *head_final_norm;        /* [head.hidden]                         */
} wpk_weights;

typedef struct wpk_handle wpk_handle;

/* Counts describing a compiled graph (for tests and reports). */
typedef struct wpk_graph_stats {
  int64_t n_tiles;          /* tiles per decode step (one epoch)              */
  int64_t n_counters;       /* dependency counters after dedup                */
  int64_t n_edges;          /* tile-to-tile edges before counter dedup        */
  int64_t n_signals;        /* counter increments per step                    */
  int64_t n_ops;            /* op groups (= launches per step in per-op mode) */
  int64_t n_workers;        /* worker CTAs of the persistent grid             */
  int64_t weight_bytes;     /* algorithmic weight bytes read per step         */
  int64_t region_begin[5];  /* ticket boundaries of the regions               */
  int64_t n_regions;
} wpk_graph_stats;

/* One trace record per tile of the last traced step (wpk_plan_cfg.trace).
 * Times are %globaltimer nanoseconds; event-clock values come from one global
 * counter, so they order events across workers exactly. */
typedef struct wpk_trace_rec {
  uint32_t tile;         /* tile index (= ticket within the step)              */
  uint16_t worker;       /* worker CTA that ran it                             */
  uint16_t op;           /* op code                                            */
  uint32_t ev_issue;     /* event clock when its staging copies were issued    */
  uint32_t ev_start;     /* event clock after its dependency wait succeeded    */
  uint32_t ev_done;      /* event clock after its body, before it signalled    */
  uint32_t epoch;        /* step epoch it belongs to                           */
  uint64_t t_claim_ns;   /* producer took the ticket                           */
  uint64_t t_issued_ns;  /* producer had issued all its staging copies         */
  uint64_t t_start_ns;   /* compute warps passed the dependency wait           */
  uint64_t t_data_ns;    /* the last staged chunk had landed and been consumed */
  uint64_t t_end_ns;     /* body and epilogue done                             */
} wpk_trace_rec;

/* The first device error recorded by the program. */
typedef struct wpk_error_info {
  int32_t code;         /* WPK_ERR_* or 0                                      */
  uint32_t tile;        /* tile that failed                                    */
  uint32_t counter;     /* counter it waited on (0xFFFFFFFF if none)           */
  uint32_t epoch;
  uint32_t observed;    /* counter value seen when it gave up                  */
  uint32_t target;      /* value it waited for                                 */
} wpk_error_info;

/* ----------------------------------------------------------- entry points */

/* Compile the tile graph for a model and plan (host only; also allocates the
 * library's small device tables on the current device).  Splits every op into
 * tiles sized to the staging slot, derives tile-to-tile tensor edges, dedups
 * counters by predecessor set, emits the ticket order and region cuts
 * ("Why real-time inference wants a megakernel", "A concrete design": the
 * compiled program is worker assignment, ordering, synchronization and the
 * memory plan).  *out receives the handle.  Errors: INVALID_ARG, SHAPE,
 * UNSUPPORTED, CUDA. */
int wpk_build_graph(const wpk_model_cfg *model, const wpk_plan_cfg *plan, wpk_handle **out);

/* Bytes the caller must allocate (device memory, 256-byte aligned) for the
 * arranged weights, the paged KV cache and the activation scratch. */
int wpk_workspace_size(const wpk_handle *h, size_t *weight_bytes, size_t *kv_bytes,
                       size_t *scratch_bytes);

/* Arrange the host bf16 weights into tile-contiguous blocks (each tile's
 * weights become one contiguous bulk copy) and copy them to dev_weights; bind
 * the KV and scratch buffers.  Synchronous with respect to the host buffers
 * (they may be freed on return); the device copy is ordered on `stream`. */
int wpk_load_weights(wpk_handle *h, const wpk_weights *w, void *dev_weights, void *dev_kv,
                     void *dev_scratch, void *stream);

/* Replace the KV block table (host array [max_batch][max_blocks] of page ids,
 * each < max_batch*max_blocks and distinct).  Results do not depend on it. */
int wpk_set_block_table(wpk_handle *h, const int32_t *table);

/* Prompt prefill: tokens_dev [batch][prompt_len] (int32, row-major) fills the
 * KV cache from position 0, resets the step epoch, and writes the first
 * greedy token per sequence to first_tok_dev [batch] and, if logits_dev is
 * not NULL, the fp32 logits at the last prompt position to logits_dev
 * [batch][vocab].  Stream-ordered on `stream`.  batch <= max_batch,
 * prompt_len + decode steps <= max_context. */
int wpk_prefill(wpk_handle *h, const int32_t *tokens_dev, int batch, int prompt_len,
                int32_t *first_tok_dev, float *logits_dev, void *stream);

/* One decode step for the active batch: consumes in_tok_dev [batch] (NULL =
 * feed back the last greedy tokens), writes the greedy tokens to out_tok_dev
 * [batch] (may be NULL) and the fp32 logits to logits_dev [batch][vocab] (may
 * be NULL).  Stream-ordered in launch modes; in resident mode it rings the
 * grid's doorbell and returns when the device publishes completion (or
 * WPK_ERR_TIMEOUT). */
int wpk_step(wpk_handle *h, const int32_t *in_tok_dev, int32_t *out_tok_dev, float *logits_dev,
             void *stream);

/* Choose the program the inspection calls below (stats, edges, tile ops,
 * verifier, simulator, trace) refer to: batch 0 selects the decode program;
 * otherwise the prefill program for `batch` prompts of `prompt_len` tokens,
 * compiled on first use (host work only).  WPK_ERR_UNSUPPORTED when the plan
 * prefills token by token. */
int wpk_select_program(wpk_handle *h, int batch, int prompt_len);

/* Graph facts; *st is filled. */
int wpk_graph_stats_get(const wpk_handle *h, wpk_graph_stats *st);

/* Tile-to-tile edges of one step as (producer, consumer) pairs: writes up to
 * max_pairs pairs into pairs[2*i], pairs[2*i+1]; *n_pairs gets the total. */
int wpk_get_edges(const wpk_handle *h, int32_t *pairs, int64_t max_pairs, int64_t *n_pairs);

/* Op code of every tile in ticket order (int32 [n_tiles]). */
int wpk_get_tile_ops(const wpk_handle *h, int32_t *ops, int64_t n);

/* Weight bytes each tile stages into its worker's slot before its
 * dependency wait (int64 [n_tiles], ticket order; 0 for tiles that stage no
 * weights), for the selected program. */
int wpk_get_tile_bytes(const wpk_handle *h, int64_t *bytes, int64_t n);

/* Check the compiled graph on the host: the ticket order is topological,
 * every read-after-write, write-after-read and write-after-write pair of
 * accesses to the same tensor range is ordered by a path of edges (commuting
 * accumulations excepted), and every counter's target equals its signal count.
 * Returns WPK_OK or WPK_ERR_SHAPE with the first violation in
 * wpk_last_error.  Cost is quadratic in tiles: meant for small configs. */
int wpk_verify_graph(const wpk_handle *h);

/* Run the compiled ticket queue on `n_threads` host threads standing in for
 * workers (same atomic ticket claim, counter targets and signals, random
 * delays from `seed`) for `n_epochs` steps.  Writes the order in which tiles
 * finished (int32 [n_epochs*n_tiles]) to done_order if not NULL.  A thread
 * whose wait exceeds wait_ms returns WPK_ERR_TIMEOUT.  `stuck_tile` >= 0 makes
 * that tile never signal (fault injection on the host). */
int wpk_simulate(const wpk_handle *h, int n_threads, int n_epochs, uint64_t seed, int wait_ms,
                 int stuck_tile, int32_t *done_order);

/* A candidate composition for wpk_predict ("One Megakernel is Not Enough",
 * Table I: the feature rows it models and how). */
typedef struct wpk_predict_cfg {
  int mode;              /* WPK_MEGAKERNEL (persistent launches) or
                            WPK_PER_OP_GRAPH (one conventional launch per op) */
  int n_regions;         /* megakernel: persistent launches, 1..4 */
  int region_cut[4];     /* first layer of each region (region_cut[0] = 0) */
  int n_workers;         /* persistent workers of each launch (the CTA budget) */
  int n_sms;             /* SMs a conventional launch spreads its CTAs over */
  int schedule;          /* WPK_SCHED_QUEUE or WPK_SCHED_STATIC */
  int slots;             /* staging slots per worker: a tile's weight load is
                            issued when one is free, before its predecessors
                            are done (1 = one staging slot per worker) */
  double dispatch_ns;    /* cost of a launch: a dispatch node before each */
  double sync_ns;        /* added to a tile's ready time when it waits on a
                            counter inside a persistent launch */
  double first_chunk_ns; /* from a load's issue to its first bytes landing */
} wpk_predict_cfg;

/* Predict the time (ns) of one run of the selected program (the decode step,
 * or the prefill program chosen with wpk_select_program) under composition
 * `cfg`, by list-scheduling its tile graph (the compiled tile-to-tile edges)
 * on the composition's workers and launches.  service_ns[t] is tile t's busy
 * time once its weights are staged and its inputs ready; load_ns[t] the time
 * to stage its weights (both double [n_tiles], host memory).  Host-only; it
 * runs nothing on the GPU.  WPK_ERR_INVALID_ARG for a bad configuration. */
int wpk_predict(const wpk_handle *h, const double *service_ns, const double *load_ns, const wpk_predict_cfg *cfg,
                double *out_ns);

/* Copy the last traced step's records (n_tiles wpk_trace_rec) to host_buf.
 * Synchronizes the device. */
int wpk_get_trace(wpk_handle *h, void *host_buf, size_t bytes);

/* First device error (code 0 if none).  Synchronizes the device. */
int wpk_get_error_info(wpk_handle *h, wpk_error_info *info);

/* Human-readable message for the last failing call on this handle; with
 * h == NULL, the message of this thread's last failed wpk_build_graph. */
const char *wpk_last_error(const wpk_handle *h);

/* Stop the resident grid (if any), release library-owned tables, free h. */
int wpk_destroy(wpk_handle *h);

/* Fixed-cohort serving ("Why real-time inference wants a megakernel", "The
 * cohort is known": compile for a session capacity, keep separate state per
 * slot, step the live sessions together and mask the idle ones so that
 * arrivals do not change the execution shape).
 *
 * wpk_prefill_slots prefills `batch` new sequences (tokens_dev [batch][T],
 * device) into slots [slot0, slot0 + batch) of the plan, leaving every other
 * slot's cache, position and last token as they were; the new slots become
 * live.  The first call after a plain wpk_prefill (or on a fresh handle)
 * enters the cohort mode: all slots start empty and idle.  From then on each
 * wpk_step steps every slot of the plan (max_batch): a live slot as usual, an
 * idle slot with a neutral input (code 0, RoPE position 0) that writes
 * nothing to its cache, keeps its position and last token, and outputs -1 in
 * out_tok_dev.  Slots keep their own context lengths; a step that would take
 * a live slot past max_context fails with WPK_ERR_SHAPE.  first_tok_dev gets
 * [batch] tokens and logits_dev (or NULL) [batch][vocab].  Needs the
 * tensor-core prefill program (WPK_ERR_UNSUPPORTED otherwise) and a single
 * decoder.  Stream-ordered; synchronizes `stream` once before the launch. */
int wpk_prefill_slots(wpk_handle *h, const int32_t *tokens_dev, int slot0, int batch, int prompt_len,
                      int32_t *first_tok_dev, float *logits_dev, void *stream);

/* Cohort mode: set the live mask of slots [0, n) from active[n] (host, nonzero
 * = live).  A slot that holds no prefilled sequence cannot be made live
 * (WPK_ERR_INVALID_ARG).  Synchronizes the device (call it between steps). */
int wpk_set_active_slots(wpk_handle *h, const int32_t *active, int n);

/* One decode step like wpk_step (megakernel mode only), for callers that
 * cannot allocate device memory when they step the model: a host application
 * that owns the whole device pool and gives plugins no allocator, or a
 * real-time loop that must never enter an allocator.  It allocates nothing
 * (no cudaMalloc/cudaFree, no allocating library call): the activation
 * scratch comes from a static 8 MiB device array inside the library instead
 * of the buffer bound by wpk_load_weights.  The paper has no counterpart;
 * this entry point exists for those callers only.
 *   - Every GPU that loads the library holds the 8 MiB until process exit.
 *   - The limit applies to the decode step's part of the scratch (the GEMV
 *     decode buffers; about 6.9 MiB for the 1B shape at batch 48 and a
 *     624-token context); the prefill program keeps using the caller's
 *     buffer.  A larger decode scratch gets WPK_ERR_SHAPE.
 *   - WPK_ERR_UNSUPPORTED for: the per-op graph mode (its captured graph
 *     holds the scratch address), the resident grid (it keeps its scratch
 *     pointer for its lifetime), the tensor-core decode program (it keeps
 *     sums in its scratch between steps) and the two-stage model.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is cached per device: do not
 *     use this entry point across a device reset.
 *   - All calls share the one array and it keeps the last call's contents;
 *     no part of it needs to start at zero (each step writes every scratch
 *     value before reading it).  Calls that overlap on the GPU, from any
 *     handle or stream, race on it.
 * Inputs, outputs and errors are those of wpk_step. */
int wpk_step_noalloc(wpk_handle *h, const int32_t *in_tok_dev, int32_t *out_tok_dev, float *logits_dev,
                     void *stream);

/* Check of the tensor-core tile (tests): D[128][N] = A . (B1 + B2)^T with fp32
 * accumulation, computed by one CTA through the same path as the program's
 * tensor-core tiles.  Operands are device "images" of 16-bit values (bf16 if
 * `bf16`, else fp16): for each 64-column K chunk c, A's 128 rows x 128 bytes
 * and B's N rows x 128 bytes, each row's eight 16-byte units stored at unit
 * index (u XOR row % 8) (the 128-byte swizzle).  b2_img_dev may be NULL.
 * d_dev receives fp32 [128][N] row-major.  N is a multiple of 16 in
 * [16, 256].  Synchronous on `stream`; WPK_ERR_TIMEOUT if a bounded wait gave
 * up. */
int wpk_debug_gemm(const void *a_img_dev, const void *b1_img_dev, const void *b2_img_dev, float *d_dev,
                   int n_chunks, int N, int bf16, void *stream);

/* Test hook: make counter `counter` need one more signal than it can ever get
 * (an unsatisfiable dependency), so the next step's device wait must time out
 * and return WPK_ERR_TIMEOUT.  Host-side fault injection; no GPU fault. */
int wpk_debug_break_counter(wpk_handle *h, int counter);

#ifdef __cplusplus
}
#endif
#endif /* WPK_H_ */
