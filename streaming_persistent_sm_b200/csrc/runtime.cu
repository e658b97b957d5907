// Persistent decode program for sm_100a: the worker and the tile bodies.
//
// A worker is one CTA: a producer warp and eight consumer (compute) warps.
//   producer: takes tickets from the device queue (one atomic per tile), and
//     for each tile streams its staging data - weight rows, or the KV pages of
//     an attention split - into the worker's staging slot, a ring of 16 KB
//     chunk stages, with bulk copies.  It does this before the tile's
//     predecessors are done ("One Megakernel is Not Enough", Table I, weight
//     prefetch: a staged tile's weight load is queued while its predecessors
//     still run; its compute still waits for them).  It may hold up to
//     `lookahead` tiles; lookahead 1 stages a tile only once the worker's
//     previous tile has finished.
//   consumers: take the worker's tiles in ticket order, wait (acquire,
//     bounded by %globaltimer) until the tile's counter holds need x epoch,
//     compute each chunk as it lands, release the stage, and after the
//     epilogue release-increment the counters of the tile's consumers ("Why
//     real-time inference wants a megakernel", "What the megakernel changes":
//     wait for dependencies, run, signal consumers).
// Tensors consumed inside a tile (normalised activations, pre-RoPE q/k,
// gate/up) are never stored ("One Megakernel is Not Enough", Table I, on-chip
// forwarding); the normalised activation a worker staged for one tile is kept
// for its next tile of the same op.
//
// Deadlock freedom: tickets follow a topological order, each worker computes
// its tiles in ticket order and streams their data in that order, so the
// worker holding the smallest unfinished ticket can always run it; the grid
// is co-resident (cooperative launch).  Every wait is bounded: on timeout a
// worker records {code, tile, counter, epoch, observed, target} in the error
// word, the other workers see it and stop, and each waits (bounded) for its
// own copies in flight before returning.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mma.cuh"
#include "ptx.cuh"
#include "wpk_internal.h"

namespace wpk {

namespace {

constexpr int kOutFloats = kMaxTileRows * kMaxGemvBatch;  // GEMV partial outputs [row][8]
constexpr int kSigQueue = 8;                               // finished tiles awaiting their signals
constexpr uint32_t kSigStop = 0xFFFFFFFFu;
constexpr int kNoAct = -1;

// the current step's I/O pointers (from the launch, or per step from the
// resident control block), set by compute thread 0 before each tile
__shared__ const int32_t* s_in_tok;
__shared__ int s_in_stride;
__shared__ int32_t* s_out_tok;
__shared__ float* s_logits;
__shared__ uint32_t s_io_epoch;

struct TQEntry {  // producer -> consumers, one per tile held by the worker
  Tile tile;
  uint32_t ticket;
  int32_t valid;
  int32_t n_chunks;
  int32_t rows_per_chunk;
  uint32_t ev_issue;  // event clock when its first copy was issued (trace)
  uint32_t epoch;     // step the tile belongs to (counter targets are need x epoch)
  uint64_t t_claim, t_issued;  // trace timestamps
};

struct Shared {
  uint8_t* ring;
  float* act;
  float* out;
  TQEntry* tq;
  uint64_t* full;    // [n_stages]
  uint64_t* empty;   // [n_stages]
  uint64_t* tq_full;   // [kMaxQueue]
  uint64_t* tq_empty;  // [kMaxQueue]
  uint64_t* acc;       // tensor-core accumulator ready
  uint64_t* sig_full;  // [kSigQueue] consumers -> signaller
  uint64_t* sig_empty; // [kSigQueue] signaller -> consumers
  uint2* sig_req;      // [kSigQueue] (sig_off, sig_cnt) of a finished tile
};

__device__ __forceinline__ Shared carve(uint8_t* base, const KParams& P) {
  Shared s;
  s.ring = base;
  uint8_t* p = base + (size_t)P.n_stages * P.stage_bytes;
  s.act = reinterpret_cast<float*>(p);
  p += P.act_bytes;
  s.out = reinterpret_cast<float*>(p);
  p += kOutFloats * 4;
  s.tq = reinterpret_cast<TQEntry*>(p);
  p += kMaxQueue * sizeof(TQEntry);
  s.full = reinterpret_cast<uint64_t*>(p);
  s.empty = s.full + kMaxStages;
  s.tq_full = s.empty + kMaxStages;
  s.tq_empty = s.tq_full + kMaxQueue;
  s.acc = s.tq_empty + kMaxQueue;
  s.sig_full = s.acc + 1;
  s.sig_empty = s.sig_full + kSigQueue;
  s.sig_req = reinterpret_cast<uint2*>(s.sig_empty + kSigQueue);
  return s;
}

// Consumer-only barrier (named barrier 1, the eight compute warps).
__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ bool cbar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(n) : "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ void unpack8(const uint4 w, float* f) {
  f[0] = __uint_as_float(w.x << 16);
  f[1] = __uint_as_float(w.x & 0xFFFF0000u);
  f[2] = __uint_as_float(w.y << 16);
  f[3] = __uint_as_float(w.y & 0xFFFF0000u);
  f[4] = __uint_as_float(w.z << 16);
  f[5] = __uint_as_float(w.z & 0xFFFF0000u);
  f[6] = __uint_as_float(w.w << 16);
  f[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

__device__ __forceinline__ uint16_t f2bf(float x) {
  __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&b);
}

__device__ __forceinline__ float bf2f(uint16_t u) { return __uint_as_float((uint32_t)u << 16); }

__device__ void record_error(const KParams& P, int code, uint32_t tile, uint32_t ctr, uint32_t obs,
                             uint32_t target) {
  if (atomicCAS(&P.err->code, 0, code) == 0) {
    P.err->tile = tile;
    P.err->counter = ctr;
    P.err->epoch = P.epoch;
    P.err->observed = obs;
    P.err->target = target;
    __threadfence();
    if (P.resident) {
      P.ctl->err = code;
      __threadfence_system();
    }
  }
}

// Bounded wait on an mbarrier phase.  `abort` (shared) ends the wait early.
// `slack` multiplies the bound: the producer's and signaller's waits only
// idle behind the compute warps, so they give up later than any wait of the
// compute warps and the error word names the wait that actually stalled.
__device__ bool wait_phase(const KParams& P, uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t tile,
                           uint32_t slack = 1) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  // waits that only idle behind other warps (slack > 1) also idle while a
  // resident grid waits for its next step
  const uint64_t bound = (P.resident && slack > 1) ? max(P.timeout_ns * slack, 2 * P.idle_ns) : P.timeout_ns * slack;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > bound) {
        record_error(P, WPK_ERR_TIMEOUT, tile, kNoCounter, 0, 0);
        *abort = 1;
        return false;
      }
    }
  }
}

// Bounded wait until a shared counter written by other warps of this CTA
// reaches `target`.
__device__ bool wait_count(const KParams& P, volatile uint32_t* v, uint32_t target, volatile int* abort,
                           uint32_t tile) {
  if (*v >= target) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (*v >= target) return true;
    if ((it & 31) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > 4 * P.timeout_ns) {
        record_error(P, WPK_ERR_TIMEOUT, tile, kNoCounter, target, *v);
        *abort = 1;
        return false;
      }
    }
  }
}

// KV cache element (layer, block, kv head g, sel = 0 for K / 1 for V, row):
// the K page and the V page of one (block, head) are adjacent, so a page is
// staged with one bulk copy.
__device__ __forceinline__ size_t kv_index(const KParams& P, int layer, int block, int sel, int g, int row) {
  return ((((size_t)layer * P.n_blocks + block) * P.n_kv + g) * 2 + sel) * P.page_tokens * P.head_dim +
         (size_t)row * P.head_dim;
}

__device__ __forceinline__ int active_batch(const KParams& P) { return *P.active_batch; }
__device__ __forceinline__ bool slot_on(const KParams& P, int b) { return P.slot_active[b] != 0; }

struct AttnSpan {
  int b, g, j, pos, t0, t1;  // tokens [t0, t1) of sequence b, current position pos
};

// KV pages a decode attention tile stages per ring stage (a tensor-core decode
// stage holds two 64-token pages).
__device__ __forceinline__ int attn_pps(const KParams& P) {
  return max(1, P.stage_bytes / (2 * P.page_tokens * P.head_dim * 2));
}

__device__ __forceinline__ AttnSpan attn_span(const KParams& P, const Tile& T) {
  AttnSpan s;
  s.b = T.a0;
  s.g = T.a1;
  s.j = T.a2;
  s.pos = P.seqlen[s.b];
  s.t0 = s.j * P.split_tokens;
  s.t1 = min(s.t0 + P.split_tokens, s.pos + 1);
  return s;
}

// ---------------------------------------------------------------------------
// Producer side: how a tile's staging data is cut into chunks, and the copies.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool is_mma_op(int op) {
  return (op >= OP_MQKV && op <= OP_MDOWN) || (op >= OP_BQKV && op <= OP_BLM);
}

// Prefill attention: queries [t0, t1) of sequence b read keys [0, t1).
__device__ __forceinline__ void pattn_span(const KParams& P, const Tile& T, int* t0, int* t1) {
  const int qb_tokens = kTokBlock / P.group;
  *t0 = T.a2 * qb_tokens;
  *t1 = min(P.T, *t0 + qb_tokens);
}
// Its keys [k0, k1): split a3 of pattn_ks keys, or all keys up to t1.
__device__ __forceinline__ void pattn_keys(const KParams& P, const Tile& T, int t1, int* k0, int* k1) {
  *k0 = P.pattn_ks ? T.a3 * P.pattn_ks : 0;
  *k1 = P.pattn_ks ? min(t1, *k0 + P.pattn_ks) : t1;
}

__device__ __forceinline__ void tile_chunks(const KParams& P, const Tile& T, int* n_chunks, int* rpc) {
  *rpc = 0;
  *n_chunks = 0;
  if (is_mma_op(T.op)) {  // ring stages: units of mma_cps K chunks
    *n_chunks = (T.a3 / 64 + P.mma_cps - 1) / P.mma_cps;
    return;
  }
  if (T.op == OP_PATTN) {
    int t0, t1, k0, k1;
    pattn_span(P, T, &t0, &t1);
    pattn_keys(P, T, t1, &k0, &k1);
    *n_chunks = (k1 - 1) / P.page_tokens - k0 / P.page_tokens + 1;
    return;
  }
  if (T.op == OP_ATTN) {  // attn_pps KV pages per ring stage
    if (T.a0 >= active_batch(P) || !slot_on(P, T.a0)) return;
    const AttnSpan s = attn_span(P, T);
    const int pages = s.t1 > s.t0 ? (s.t1 - 1) / P.page_tokens - s.t0 / P.page_tokens + 1 : 0;
    *n_chunks = (pages + attn_pps(P) - 1) / attn_pps(P);
    return;
  }
  if (T.w_bytes == 0) return;
  int r = P.stage_bytes / P.gemv_cps / (T.a3 * 2);
  r &= ~1;  // even: RoPE and gate/up row pairs never straddle a chunk
  *rpc = r < 2 ? 2 : r;
  // ring stages of gemv_cps chunks each
  *n_chunks = ((T.a1 + *rpc - 1) / *rpc + P.gemv_cps - 1) / P.gemv_cps;
}

// Source image (hi or lo) of a tensor-core tile's activations: the tile covers
// the K range [a2, a2 + a3) of token block a1 (the batched decode program has
// one token block); a token block's image holds the op's whole K.
__device__ __forceinline__ const uint8_t* mma_act_src(const KParams& P, const Tile& T, int part) {
  const uint8_t* const* img;
  int k_full;  // the op's whole K: a token block's image holds k_full / 64 chunks
  switch (T.op) {
    case OP_MO: case OP_BO: img = P.att_img; k_full = P.q_rows; break;
    case OP_MDOWN: case OP_BDOWN: img = P.h_img; k_full = P.ffn; break;
    case OP_BGU: img = P.xf_img; k_full = P.hidden; break;
    default: img = P.xn_img; k_full = P.hidden; break;
  }
  return img[part] + ((size_t)T.a1 * (k_full / 64) + T.a2 / 64) * P.img_stride;
}

// A tensor-core tile stages its K chunks in units of mma_cps consecutive
// chunks, one ring stage each: [the units' weight blocks, 16 KB each][their
// activation chunks, hi then lo rows of each].  Units are walked rotated by
// the tile's row block, so that tiles running at the same time copy different
// activation chunks (every tile of an op reads the same activation image).
// The sum over K is the same; only the fp32 summation order differs.
struct MmaUnit {
  int c0, nc;  // first K chunk of the unit, chunks in it
};
__device__ __forceinline__ MmaUnit mma_unit(const KParams& P, const Tile& T, int u) {
  const int nch = T.a3 / 64, cps = P.mma_cps;
  const int nu = (nch + cps - 1) / cps;
  const int rot = nu > 1 ? (int)((uint32_t)T.a0 % (uint32_t)nu) : 0;
  const int ur = u + rot >= nu ? u + rot - nu : u + rot;
  MmaUnit m;
  m.c0 = ur * cps;
  m.nc = min(cps, nch - m.c0);
  return m;
}

// Tensor-core unit u: arm the barrier with all its bytes and copy its weight
// blocks (the activation chunks follow in issue_mma_act).
__device__ void issue_mma_w(const KParams& P, const Tile& T, int u, uint8_t* dst, uint64_t* bar) {
  const MmaUnit m = mma_unit(P, T, u);
  mbar_arrive_expect_tx(bar, (uint32_t)m.nc * ((uint32_t)kMmaChunkBytes + 2u * (uint32_t)P.act_chunk));
  const uint64_t base = (T.op == OP_BLM) ? P.lm_mma_off : 0;  // LM tiles are relative to the launch's head
  bulk_g2s(dst, P.weights + base + T.w_off + (size_t)m.c0 * kMmaChunkBytes, (uint32_t)m.nc * kMmaChunkBytes, bar);
}
__device__ void issue_mma_act(const KParams& P, const Tile& T, int u, uint8_t* dst, uint64_t* bar) {
  const MmaUnit m = mma_unit(P, T, u);
  const uint32_t a = (uint32_t)P.act_chunk;
  uint8_t* act = dst + (size_t)P.mma_cps * kMmaChunkBytes;
  if (P.img_stride == 2 * P.act_chunk) {  // hi and lo rows adjacent: the unit's chunks in one copy
    bulk_g2s(act, mma_act_src(P, T, 0) + (size_t)m.c0 * P.img_stride, (uint32_t)m.nc * 2u * a, bar);
  } else {  // separate hi and lo images (one chunk per unit)
    bulk_g2s(act, mma_act_src(P, T, 0) + (size_t)m.c0 * P.img_stride, a, bar);
    bulk_g2s(act + a, mma_act_src(P, T, 1) + (size_t)m.c0 * P.img_stride, a, bar);
  }
}

// The KV pages an attention tile stages: whole pages (a page's K rows, then
// its V rows at page * head_dim), one copy each, pps per ring stage; prefill
// attention: pages of sequence a0, kv head a1 over the tile's keys, one per
// stage; decode: the split's pages, packed into the stages.  Computed once per
// tile by the producer.
struct PageWalk {
  const int32_t* row;  // the sequence's block-table row
  int first, n_pages, pps, g;
};
__device__ PageWalk page_walk(const KParams& P, const Tile& T) {
  PageWalk w;
  if (T.op == OP_PATTN) {
    int t0, t1, k0, k1;
    pattn_span(P, T, &t0, &t1);
    pattn_keys(P, T, t1, &k0, &k1);
    w.row = P.block_table + (size_t)(P.slot0 + T.a0) * P.max_blocks;
    w.first = k0 / P.page_tokens;
    w.n_pages = (k1 - 1) / P.page_tokens - w.first + 1;
    w.pps = 1;
    w.g = T.a1;
  } else {
    const AttnSpan sp = attn_span(P, T);
    w.row = P.block_table + (size_t)sp.b * P.max_blocks;
    w.first = sp.t0 / P.page_tokens;
    w.n_pages = sp.t1 > sp.t0 ? (sp.t1 - 1) / P.page_tokens + 1 - w.first : 0;
    w.pps = attn_pps(P);
    w.g = sp.g;
  }
  return w;
}

// Block ids of the first kPagePrefetch pages of stage k, loaded together (the
// producer loads them before it waits for the stage: one dependent L2 round
// trip per page took a b16 attention tile's four stages 14 us to issue).
constexpr int kPagePrefetch = 8;
__device__ __forceinline__ void page_blocks(const PageWalk& w, int k, int* blk) {
  const int p0 = w.first + k * w.pps, n = min(w.pps, w.n_pages - k * w.pps);
#pragma unroll
  for (int j = 0; j < kPagePrefetch; ++j) blk[j] = j < n ? __ldcg(w.row + p0 + j) : 0;
}

// Copies of stage k of an attention tile into `dst`; arms `bar` with their
// bytes.  blk holds the stage's first block ids (page_blocks).
__device__ void issue_pages(const KParams& P, const Tile& T, const PageWalk& w, int k, const int* blk, uint8_t* dst,
                            uint64_t* bar) {
  const uint32_t bytes = 2u * (uint32_t)P.page_tokens * (uint32_t)P.head_dim * 2u;
  const int p0 = w.first + k * w.pps, n = min(w.pps, w.n_pages - k * w.pps);
  mbar_arrive_expect_tx(bar, (uint32_t)n * bytes);
#pragma unroll
  for (int j = 0; j < kPagePrefetch; ++j)
    if (j < n) bulk_g2s(dst + (size_t)j * bytes, P.kv + kv_index(P, T.layer, blk[j], 0, w.g, 0), bytes, bar);
  for (int j = kPagePrefetch; j < n; ++j)
    bulk_g2s(dst + (size_t)j * bytes, P.kv + kv_index(P, T.layer, __ldcg(w.row + p0 + j), 0, w.g, 0), bytes, bar);
}

// Copies of GEMV stage k of tile T into `dst`; arms `bar` with their bytes.
__device__ void issue_chunk(const KParams& P, const Tile& T, int k, int rpc, uint8_t* dst, uint64_t* bar) {
  // GEMV stage k: chunks k gemv_cps .. (consecutive rows), one copy
  const size_t row_bytes = (size_t)T.a3 * 2;
  const int r0 = k * P.gemv_cps * rpc;
  const uint32_t bytes = (uint32_t)(min(P.gemv_cps * rpc, T.a1 - r0) * row_bytes);
  const uint64_t base = (T.op == OP_LMHEAD) ? P.lm_head_off : 0;  // LM tiles are relative to the launch's head
  mbar_arrive_expect_tx(bar, bytes);
  bulk_g2s(dst, P.weights + base + T.w_off + r0 * row_bytes, bytes, bar);
}

// ---------------------------------------------------------------------------
// GEMV (CUDA cores).  A work item is one row (or one part of a row's 256-column
// segments when a chunk has fewer rows than warps): each lane reads 16
// contiguous weight bytes per segment (a warp reads 512 contiguous bytes),
// accumulates across its segments in registers and reduces once.
// Activations are staged lane-permuted - element k = 256*seg + 8*lane + 4*h + e
// lives at 256*seg + 128*h + 4*lane + e - so each float4 read of a warp is 512
// contiguous bytes (no bank conflicts).  Per token the staged row is padded to
// whole segments (act_stride floats).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int act_stride(int K) { return (K + 255) & ~255; }

__device__ __forceinline__ int act_pos(int k) {
  return (k & ~255) | (((k >> 2) & 1) << 7) | (((k >> 3) & 31) << 2) | (k & 3);
}

// Stage bg rows of K floats (row stride `stride`) into act, lane-permuted;
// optionally RMS-normalise each row and multiply by `gain` (then K is the whole
// row).
__device__ void stage_act(const float* src, int stride, int K, int bg, const float* gain, float eps, float* act) {
  __shared__ float red[kWarps][kMaxGemvBatch];
  __shared__ float scale_s[kMaxGemvBatch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Kp = act_stride(K);
  for (int b = 0; b < bg; ++b) {
    float ss = 0.f;
    for (int k = threadIdx.x * 4; k < K; k += kThreads * 4) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(src + (size_t)b * stride + k));
      *reinterpret_cast<float4*>(act + b * Kp + act_pos(k)) = v;
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    if (gain) {
      ss = warp_sum(ss);
      if (lane == 0) red[warp][b] = ss;
    }
  }
  if (gain) {
    cbar();
    if (threadIdx.x < bg) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) tot += red[w][threadIdx.x];
      scale_s[threadIdx.x] = 1.0f / sqrtf(tot / (float)K + eps);
    }
    cbar();
    for (int b = 0; b < bg; ++b) {
      const float sc = scale_s[b];
      for (int k = threadIdx.x * 4; k < K; k += kThreads * 4) {
        float4* a = reinterpret_cast<float4*>(act + b * Kp + act_pos(k));
        const float4 gg = __ldg(reinterpret_cast<const float4*>(gain + k));
        float4 v = *a;
        v.x *= sc * gg.x;
        v.y *= sc * gg.y;
        v.z *= sc * gg.z;
        v.w *= sc * gg.w;
        *a = v;
      }
    }
  }
  cbar();
}

__device__ void epilogue(const KParams& P, const Tile& T, const float* out, int b0, int bg) {
  const int r0 = T.a0, R = T.a1, hd = P.head_dim, half = hd / 2;
  constexpr int S = kMaxGemvBatch;
  switch (T.op) {
    case OP_QKV: {
      for (int idx = threadIdx.x; idx < (R / 2) * bg; idx += kThreads) {
        const int pr = idx % (R / 2), b = idx / (R / 2), bi = b0 + b;
        const int r = r0 + 2 * pr;
        const float y0 = out[(2 * pr) * S + b], y1 = out[(2 * pr + 1) * S + b];
        const bool on = slot_on(P, bi);
        const int pos = on ? P.seqlen[bi] : 0;
        if (r < P.q_rows + P.kv_rows) {
          const bool is_q = r < P.q_rows;
          const int rr = is_q ? r : r - P.q_rows;
          const int head = rr / hd, i = (rr % hd) / 2;
          const float2 cs = P.rope[(size_t)pos * half + i];
          const float o0 = y0 * cs.x - y1 * cs.y;
          const float o1 = y1 * cs.x + y0 * cs.y;
          if (is_q) {
            float* q = P.qbuf + (size_t)bi * P.q_rows + head * hd;
            q[i] = o0;
            q[i + half] = o1;
          } else if (on) {
            const int blk = P.block_table[bi * P.max_blocks + pos / P.page_tokens];
            uint16_t* k = P.kv + kv_index(P, T.layer, blk, 0, head, pos % P.page_tokens);
            k[i] = f2bf(o0);
            k[i + half] = f2bf(o1);
          }
        } else if (on) {
          const int rr = r - P.q_rows - P.kv_rows;
          const int head = rr / hd, d = rr % hd;
          const int blk = P.block_table[bi * P.max_blocks + pos / P.page_tokens];
          uint16_t* v = P.kv + kv_index(P, T.layer, blk, 1, head, pos % P.page_tokens);
          v[d] = f2bf(y0);
          v[d + 1] = f2bf(y1);
        }
      }
      break;
    }
    case OP_O: {
      for (int idx = threadIdx.x; idx < R * bg; idx += kThreads) {
        const int rr = idx % R, b = idx / R, bi = b0 + b;
        const size_t o = (size_t)bi * P.hidden + r0 + rr;
        const float x = __ldcg(P.xa + o) + out[rr * S + b];
        P.xb[o] = x;
        P.xa[o] = x;
      }
      break;
    }
    case OP_GU: {
      for (int idx = threadIdx.x; idx < (R / 2) * bg; idx += kThreads) {
        const int pr = idx % (R / 2), b = idx / (R / 2), bi = b0 + b;
        const float g = out[(2 * pr) * S + b], u = out[(2 * pr + 1) * S + b];
        P.hbuf[(size_t)bi * P.ffn + r0 / 2 + pr] = g / (1.0f + expf(-g)) * u;
      }
      break;
    }
    case OP_DOWN: {
      for (int idx = threadIdx.x; idx < R * bg; idx += kThreads) {
        const int rr = idx % R, b = idx / R, bi = b0 + b;
        atomicAdd(P.xa + (size_t)bi * P.hidden + r0 + rr, out[rr * S + b]);
      }
      break;
    }
    case OP_LMHEAD: {
      if (s_logits)
        for (int idx = threadIdx.x; idx < R * bg; idx += kThreads) {
          const int rr = idx % R, b = idx / R, bi = b0 + b;
          s_logits[(size_t)bi * P.logits_stride + r0 + rr] = out[rr * S + b];
        }
      const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
      if (warp < bg) {
        float bv = -INFINITY;
        int bidx = 0x7FFFFFFF;
        for (int rr = lane; rr < R; rr += 32) {
          const float v = out[rr * S + warp];
          if (v > bv) { bv = v; bidx = r0 + rr; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
          if (ov > bv || (ov == bv && oi < bidx)) { bv = ov; bidx = oi; }
        }
        if (lane == 0) {
          const uint32_t fb = __float_as_uint(bv);
          const uint32_t ord = (fb & 0x80000000u) ? ~fb : (fb | 0x80000000u);
          const unsigned long long key = ((unsigned long long)ord << 32) | (0xFFFFFFFFu - (uint32_t)bidx);
          atomicMax(P.best + b0 + warp, key);
        }
      }
      break;
    }
    default:
      break;
  }
}

__device__ bool wait_counter(const KParams& P, const Tile& T, uint32_t tile, uint32_t epoch, volatile int* abort);

// Resident grid: bounded wait until the host has rung the doorbell for step
// `epoch`.  False ends the worker: shutdown, an error elsewhere, or no step for
// idle_ns (an idle grid exits; the host launches a new one for the next step).
// Worker 0 polls the mapped control block and publishes each step (its I/O
// pointers, then the step number with release semantics) in device memory;
// the other workers poll that copy.  `seen` caches the last step observed.
__device__ bool wait_doorbell(const KParams& P, uint32_t epoch, volatile int* abort, uint32_t* seen) {
  if (epoch <= *seen) return true;
  const uint64_t t0 = globaltimer();
  if (blockIdx.x == 0) {
    // worker 0 publishes every step it sees, also steps it holds no ticket of
    for (;;) {
      const uint32_t db = P.ctl->db;
      const bool quit = db == kResShutdown || *abort || ld_volatile_s32(&P.err->code) != 0 ||
                        globaltimer() - t0 > P.idle_ns;
      if (quit) {
        __threadfence();
        st_release_u32(&P.rdev->db, kResShutdown);
        return false;
      }
      if (db > *seen) {
        __threadfence_system();  // the host wrote the pointers before the step number
        P.rdev->in_tok = P.ctl->in_tok;
        P.rdev->in_stride = P.ctl->in_stride;
        P.rdev->out_tok = P.ctl->out_tok;
        P.rdev->logits = P.ctl->logits;
        __threadfence();
        st_release_u32(&P.rdev->db, db);
        *seen = db;
      }
      if (db >= epoch) return true;
      __nanosleep(256);
    }
  }
  for (uint32_t it = 1;; ++it) {
    const uint32_t db = ld_acquire_u32(&P.rdev->db);
    if (db == kResShutdown) return false;
    if (db >= epoch) {
      *seen = db;
      return true;
    }
    if ((it & 15) == 0) {
      if (*abort || ld_volatile_s32(&P.err->code) != 0) return false;
      if (globaltimer() - t0 > 2 * P.idle_ns + P.timeout_ns) return false;
    }
    __nanosleep(128);
  }
}

// Consumer-side chunk cursor: chunk c lives in stage c % n_stages and is the
// (c / n_stages)-th use of that stage.
struct Cursor {
  uint32_t c;
};

struct ConsumerState {
  int act_key;      // (op, layer, k0) of the staged activation, or kNoAct
  uint32_t last_ctr;    // counter known satisfied in this launch ...
  uint32_t last_epoch;  // ... for this step
  uint32_t acc_phase;  // parity of the accumulator barrier (prefill attention)
  uint32_t act_epoch;  // step the staged activation belongs to
  uint32_t n_mma;      // tensor-core tiles taken (accumulator buffer n_mma % 2)
};

__shared__ uint32_t s_tmem;  // TMEM base address (tensor-core programs)
// Tensor-core tiles: the issuer warp fills accumulator buffer b (s_accf[b]
// completes when the tile's MMAs have), the consumers empty it after the
// epilogue (s_acce[b]); s_mma_fin covers every MMA issued before TMEM is freed.
__shared__ uint64_t s_accf[2], s_acce[2], s_mma_fin;
// tiles (queue positions) the consumers have finished
__shared__ volatile uint32_t s_cons_tiles;

__shared__ uint64_t s_t_data;  // trace: when the tile's last chunk had landed
// GEMV: per stage, 1 + the global index of the last chunk a warp saw land there
__shared__ volatile uint32_t s_seen[kMaxStages];

__device__ __forceinline__ int act_key_of(const Tile& T) { return (int)T.op | ((int)T.layer << 4) | (T.a2 << 12); }

// One staged chunk of a GEMV tile (rows [0, rows) of the chunk, rows <= 4 at
// a time share each activation load), computed by one warp.  The row's dot
// product stays in the warp: one shuffle reduction per row, plain stores.
template <int BG>
__device__ __forceinline__ void gemv_chunk(const uint8_t* chunk, int K, int rows, int row_base, const float* act,
                                           float* out, int bg) {
  const int lane = threadIdx.x & 31;
  const int segs = (K + 255) >> 8;
  const int Kp = act_stride(K);
  const size_t row_bytes = (size_t)K * 2;
  constexpr int RG = (BG <= 2) ? 4 : 2;  // rows per pass
  for (int r0 = 0; r0 < rows; r0 += RG) {
    const int nr = min(RG, rows - r0);
    float acc[RG][BG];
#pragma unroll
    for (int i = 0; i < RG; ++i)
#pragma unroll
      for (int b = 0; b < BG; ++b) acc[i][b] = 0.f;
#pragma unroll 2
    for (int seg = 0; seg < segs; ++seg) {  // two segments in flight: the stage is held for less time
      const int k = seg * 256 + lane * 8;
      if (k >= K) continue;
      float f[RG][8];
#pragma unroll
      for (int i = 0; i < RG; ++i)
        unpack8(*reinterpret_cast<const uint4*>(chunk + (size_t)(r0 + min(i, nr - 1)) * row_bytes + (size_t)k * 2),
                f[i]);
      const float* ap = act + seg * 256 + lane * 4;
#pragma unroll
      for (int b = 0; b < BG; ++b) {
        if (BG > 4 && b >= bg) break;
        const float4 a0 = *reinterpret_cast<const float4*>(ap + b * Kp);
        const float4 a1 = *reinterpret_cast<const float4*>(ap + b * Kp + 128);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int i = 0; i < RG; ++i)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[i][b] = fmaf(f[i][e], av[e], acc[i][b]);
      }
    }
#pragma unroll
    for (int i = 0; i < RG; ++i)
#pragma unroll
      for (int b = 0; b < BG; ++b) {
        if (BG > 4 && b >= bg) break;
        const float v = warp_sum(acc[i][b]);
        if (lane == 0 && i < nr) out[(row_base + r0 + i) * kMaxGemvBatch + b] = v;
      }
  }
}

// Bounded wait (one warp) until the GEMV warp that owns stage st's previous
// use has seen that use land: s_seen[st] >= target.
__device__ bool wait_seen(const KParams& P, int st, uint32_t target, volatile int* abort, uint32_t tile) {
  if (s_seen[st] >= target) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (s_seen[st] >= target) return true;
    if ((it & 15) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > P.timeout_ns) {
        if ((threadIdx.x & 31) == 0) record_error(P, WPK_ERR_TIMEOUT, tile, kNoCounter, s_seen[st], target);
        return false;
      }
    }
  }
}

// GEMV tile body.  Chunk k of the tile belongs to warp k % 8: the warp waits
// for that stage only, computes its rows and hands the stage back at once, so
// a tile of any size streams through the ring and no block barrier is taken
// per chunk.  Returns false on a wait failure.
template <int CPS>
__device__ bool body_gemv_t(const KParams& P, const Tile& T, const Shared& S, Cursor& cur, int n_chunks, int rpc,
                            ConsumerState& cs, volatile int* abort) {
  const int K = T.a3, R = T.a1;
  const int nb = active_batch(P);
  const LayerDev* L = P.layers + (T.op == OP_LMHEAD ? 0 : T.layer);
  const float* gain = nullptr;
  const float* src = nullptr;
  int stride = 0;
  switch (T.op) {
    case OP_QKV: gain = reinterpret_cast<const float*>(P.weights + L->attn_norm); src = P.xa; stride = P.hidden; break;
    case OP_O: src = P.attn; stride = P.q_rows; break;
    case OP_GU: gain = reinterpret_cast<const float*>(P.weights + L->ffn_norm); src = P.xb; stride = P.hidden; break;
    case OP_DOWN: src = P.hbuf + T.a2; stride = P.ffn; break;
    case OP_LMHEAD: gain = reinterpret_cast<const float*>(P.weights + P.final_norm_off); src = P.xa; stride = P.hidden; break;
  }
  int bgmax = P.act_bytes / (act_stride(K) * 4);
  if (bgmax > kMaxGemvBatch) bgmax = kMaxGemvBatch;
  // chunks, CPS (= gemv_cps, a constant: the per-chunk divisions by a
  // run-time value cost the b1 step 16 us) per stage
  constexpr int cps = CPS;
  const int n_real = (R + rpc - 1) / rpc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  bool ok = true;
  for (int b0 = 0; b0 < nb || (nb == 0 && b0 == 0); b0 += bgmax) {
    const int bg = max(0, min(bgmax, nb - b0));
    const bool last_group = b0 + bgmax >= nb;
    if (bg > 0) {
      const int key = (b0 == 0 && last_group) ? act_key_of(T) : kNoAct;
      if (key == kNoAct || cs.act_key != key) {
        stage_act(src + (size_t)b0 * stride, stride, K, bg, gain, P.eps, S.act);
        cs.act_key = key;
      }
    }
    for (int k = warp; k < n_real; k += kWarps) {
      const int u = k / cps;  // the tile's stage holding chunk k
      const uint32_t c = cur.c + u;
      const int st = c % P.n_stages;
      // the stage is waited for on the first token group only
      if (b0 == 0) {
        // A parity wait only tells the current phase from the one before it.
        // When the stage's previous use (c - n_stages) is this tile's too,
        // another warp owns it and may not have seen it land yet: wait for
        // that first, so that the parity wait below cannot be satisfied by
        // the phase before the previous one.
        if (u >= P.n_stages && !wait_seen(P, st, c - P.n_stages + 1, abort, T.a0)) {
          ok = false;
          break;
        }
        if (!wait_phase(P, &S.full[st], (c / P.n_stages) & 1u, abort, T.a0)) {
          ok = false;
          break;
        }
        __syncwarp();
        if (lane == 0) s_seen[st] = c + 1;
      }
      const uint8_t* chunk = S.ring + (size_t)st * P.stage_bytes + (size_t)(k % cps) * rpc * K * 2;
      const int r0 = k * rpc, rows = min(rpc, R - r0);
      switch (bg) {
        case 0: break;
        case 1: gemv_chunk<1>(chunk, K, rows, r0, S.act, S.out, bg); break;
        case 2: gemv_chunk<2>(chunk, K, rows, r0, S.act, S.out, bg); break;
        case 3: gemv_chunk<3>(chunk, K, rows, r0, S.act, S.out, bg); break;
        case 4: gemv_chunk<4>(chunk, K, rows, r0, S.act, S.out, bg); break;
        default: gemv_chunk<8>(chunk, K, rows, r0, S.act, S.out, bg); break;
      }
      if (last_group) {
        // the stage takes gemv_cps arrivals: the last chunk of a short stage
        // arrives for the chunks it lacks
        const int in_stage = min(cps, n_real - u * cps);
        __syncwarp();
        if (lane == 0) mbar_arrive_n(&S.empty[st], (k % cps == in_stage - 1) ? (uint32_t)(cps - in_stage + 1) : 1u);
      }
    }
    if (!cbar_and(ok)) return false;
    if (P.trace && threadIdx.x == 0 && b0 == 0) s_t_data = globaltimer();
    if (bg > 0) epilogue(P, T, S.out, b0, bg);
    cbar();
    if (nb == 0) break;
  }
  cur.c += n_chunks;
  return true;
}

__device__ bool body_gemv(const KParams& P, const Tile& T, const Shared& S, Cursor& cur, int n_chunks, int rpc,
                          ConsumerState& cs, volatile int* abort) {
  return P.gemv_cps == 2 ? body_gemv_t<2>(P, T, S, cur, n_chunks, rpc, cs, abort)
                         : body_gemv_t<1>(P, T, S, cur, n_chunks, rpc, cs, abort);
}

// ---------------------------------------------------------------------------
// Split-KV GQA decode attention.  The tile (b, g, j) handles the `group`
// query heads of kv head g over the tokens of split j of sequence b, one KV
// page per staged chunk with an online softmax across the pages; it writes a
// partial (m, l, o) and the last split to arrive combines all partials of
// (b, g) ("Persistent threads and megakernels", §6: split long histories into
// chunks, combine partial attention in a reduction signalled through global
// memory).  A single split writes its result directly.
//
// Batched decode program: the current token's q, k and v are still fp32 sums
// (acc, feature-major); the tile whose split holds the current position rounds
// k and v to bf16, writes them to the KV cache and clears their sums, and the
// tile that writes the result clears the q sums.  The result goes to the hi/lo
// attention image that the O projection's tensor-core tiles read.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void attn_result(const KParams& P, int b, int f, float v) {
  if (P.dec_mma) {
    const size_t off = (size_t)(f >> 6) * P.img_stride + sw128_offset(b, f & 63);
    const __nv_bfloat16 hb = __float2bfloat16_rn(v);
    *reinterpret_cast<__nv_bfloat16*>(P.att_img[0] + off) = hb;
    *reinterpret_cast<__nv_bfloat16*>(P.att_img[1] + off) = __float2bfloat16_rn(v - __bfloat162float(hb));
    P.acc[(size_t)f * P.mma_n + b] = 0.f;  // q sums start from zero next step
  } else {
    P.attn[(size_t)b * P.q_rows + f] = v;
  }
}

// Scores and P.V of one 32-token block of a staged KV page for all GRP query
// heads of the kv group, by one warp: lane t scores token t against every head
// (its K row is read once), then lane l accumulates head dims 2l, 2l+1 of every
// head over the block's tokens (each V row is read once, the probabilities come
// from a per-warp shared array).  `skip` is the block row holding the stale
// copy of the current token (its score is left out and its V row is read as
// zero); `cnt` rows of the block are valid.
template <int GRP>
__device__ __forceinline__ void attn_block(const uint8_t* krows, const uint8_t* vrows, int cnt, int skip,
                                           const float* q_perm, float scale, float* p_w, float (&m)[GRP],
                                           float (&l)[GRP], float (&o0)[GRP], float (&o1)[GRP]) {
  const int lane = threadIdx.x & 31;
  const bool valid = lane < cnt && lane != skip;
  float sc[GRP];
#pragma unroll
  for (int h = 0; h < GRP; ++h) sc[h] = 0.f;
  if (valid) {
    const uint4* kr = reinterpret_cast<const uint4*>(krows + (size_t)lane * kHeadDim * 2);
#pragma unroll
    for (int u = 0; u < kHeadDim / 8; ++u) {
      const int uu = (u + lane) & (kHeadDim / 8 - 1);  // rotated: neighbouring lanes, other banks
      float kf[8];
      unpack8(kr[uu], kf);
#pragma unroll
      for (int h = 0; h < GRP; ++h) {
        // q is stored [head][half][unit][4]: the 8 lanes of a phase read 8
        // consecutive 16-byte units (no bank conflict)
        const float4 qa = *reinterpret_cast<const float4*>(q_perm + h * kHeadDim + 4 * uu);
        const float4 qb = *reinterpret_cast<const float4*>(q_perm + h * kHeadDim + 32 + 4 * uu);
        sc[h] = fmaf(qa.x, kf[0], fmaf(qa.y, kf[1], fmaf(qa.z, kf[2], fmaf(qa.w, kf[3], sc[h]))));
        sc[h] = fmaf(qb.x, kf[4], fmaf(qb.y, kf[5], fmaf(qb.z, kf[6], fmaf(qb.w, kf[7], sc[h]))));
      }
    }
  }
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    const float s_h = valid ? sc[h] * scale : -INFINITY;
    const float m_new = fmaxf(m[h], warp_max(s_h));
    float pp = 0.f, corr = 1.f;
    if (m_new != -INFINITY) {  // warp-uniform
      corr = expf(m[h] - m_new);
      pp = valid ? expf(s_h - m_new) : 0.f;
      m[h] = m_new;
    }
    l[h] = l[h] * corr + warp_sum(pp);
    o0[h] *= corr;
    o1[h] *= corr;
    p_w[lane * GRP + h] = pp;
  }
  __syncwarp();
  const uint32_t* vrow = reinterpret_cast<const uint32_t*>(vrows) + lane;
  for (int j = 0; j < cnt; ++j) {
    const uint32_t vv = (j == skip) ? 0u : vrow[(size_t)j * (kHeadDim / 2)];
    const float v0 = __uint_as_float(vv << 16), v1 = __uint_as_float(vv & 0xFFFF0000u);
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float pj = p_w[j * GRP + h];  // same address in every lane: a broadcast
      o0[h] = fmaf(pj, v0, o0[h]);
      o1[h] = fmaf(pj, v1, o1[h]);
    }
  }
  __syncwarp();
}

// The page loop of a decode attention tile.  The group's query heads are cut
// into head groups of GRP heads (one head group when the kv group has at most
// four heads, two otherwise), each served by `wpg` warps: warp w attends with
// heads [head0, head0 + GRP) over the tile's 32-token blocks wi, wi + wpg, ...
// (wi = w mod wpg); its per-head state (m, l, o) goes to st_s[w][h] for the
// merge.
template <int GRP>
__device__ bool attn_pages(const KParams& P, const AttnSpan& s, const Shared& Sh, Cursor& cur, int n_chunks,
                           volatile int* abort, const float* q_perm, const float* kv_cur, float* st_s, float* p_s,
                           uint32_t* page_rel, bool has_cur, int wpg) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wi = warp % wpg, head0 = (warp / wpg) * GRP;
  q_perm += head0 * kHeadDim;
  const int page = P.page_tokens, hd = kHeadDim;
  const float scale = 1.0f / sqrtf((float)hd);
  float m[GRP], l[GRP], o0[GRP], o1[GRP];
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
    o0[h] = 0.f;
    o1[h] = 0.f;
  }
  float* p_w = p_s + warp * 32 * GRP;
  bool ok = true;
  const int pps = attn_pps(P);
  const int page_bytes = 2 * page * hd * 2;
  for (int k = 0; k < n_chunks; ++k) {  // ring stage k: pages k * pps .. of the split
    const uint32_t c = cur.c + k;
    const int st = c % P.n_stages;
    // every warp waits for every stage, also one without a block for it: a
    // parity wait only tells a phase from the one before it, so no warp may
    // run a whole ring ahead of a stage it has not seen land
    if (ok && !wait_phase(P, &Sh.full[st], (c / P.n_stages) & 1u, abort, 0xFFFFFFFFu)) ok = false;
    if (P.trace && threadIdx.x == 0 && k + 1 == n_chunks) s_t_data = globaltimer();  // the last page landed
    for (int j = 0; j < pps && ok; ++j) {
      const int pg = k * pps + j;  // page of the split
      const int p0 = (s.t0 / page + pg) * page;
      if (p0 >= s.t1) break;
      const int n = min(page, s.t1 - p0);
      const int nblk = (n + 31) / 32;
      // blocks are numbered across the tile's pages so that every warp gets work
      const int first = (pg * ((page + 31) / 32)) % wpg;
      const int mine = (wi - first + wpg) % wpg;  // this warp's first block in the page
      const uint8_t* stage = Sh.ring + (size_t)st * P.stage_bytes + (size_t)j * page_bytes;
      for (int b = mine; b < nblk; b += wpg) {
        const int cnt = min(32, n - b * 32);
        // the staged copy of the current token's row is stale (it was copied
        // before this step wrote it): leave it out, read zeros for its V
        const int rel = s.pos - p0 - b * 32;
        const int skip = (rel >= 0 && rel < 32) ? rel : -1;
        attn_block<GRP>(stage + (size_t)b * 32 * hd * 2, stage + (size_t)page * hd * 2 + (size_t)b * 32 * hd * 2,
                        cnt, skip, q_perm, scale, p_w, m, l, o0, o1);
      }
    }
    // the last warp to finish with the page hands the stage back
    __syncwarp();
    if (lane == 0) {
      const uint32_t r = atomicAdd(&page_rel[st], 1u) + 1u;
      if (r == (uint32_t)kWarps * (uint32_t)(k / P.n_stages + 1)) mbar_arrive_n(&Sh.empty[st], (uint32_t)P.gemv_cps);
    }
  }
  cur.c += n_chunks;
  if (has_cur && wi == 0) {  // the current token, read from where this step wrote it
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const int u0 = (2 * lane) >> 3, e0 = (2 * lane) & 7;  // dims 2 lane, 2 lane + 1 in the permuted q
      const float* qh = q_perm + h * hd;
      const float qd0 = qh[(e0 >> 2) * 32 + 4 * u0 + (e0 & 3)], qd1 = qh[(e0 >> 2) * 32 + 4 * u0 + (e0 & 3) + 1];
      const float sc = warp_sum(qd0 * kv_cur[2 * lane] + qd1 * kv_cur[2 * lane + 1]) * scale;
      const float m_new = fmaxf(m[h], sc);
      const float corr = expf(m[h] - m_new), pp = expf(sc - m_new);
      l[h] = l[h] * corr + pp;
      o0[h] = o0[h] * corr + pp * kv_cur[hd + 2 * lane];
      o1[h] = o1[h] * corr + pp * kv_cur[hd + 2 * lane + 1];
      m[h] = m_new;
    }
  }
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    float* mine = st_s + (warp * GRP + h) * (2 + kHeadDim);
    mine[2 + 2 * lane] = o0[h];
    mine[3 + 2 * lane] = o1[h];
    if (lane == 0) {
      mine[0] = m[h];
      mine[1] = l[h];
    }
  }
  return ok;
}

__device__ bool body_attn(const KParams& P, const Tile& T, const Shared& Sh, Cursor& cur, int n_chunks,
                          volatile int* abort) {
  if (T.a0 >= active_batch(P)) return true;
  if (!slot_on(P, T.a0)) {
    // an inactive slot attends to nothing; the tensor-core decode still
    // returns its q/k/v sums to zero for the next step (split 0 does it)
    if (P.dec_mma && T.a2 == 0) {
      const int nq = P.group * P.head_dim, hd = P.head_dim;
      for (int i = threadIdx.x; i < nq + 2 * hd; i += kThreads) {
        const int f = i < nq ? T.a1 * nq + i
                             : P.q_rows + ((i - nq) / hd) * P.kv_rows + T.a1 * hd + (i - nq) % hd;
        P.acc[(size_t)f * P.mma_n + T.a0] = 0.f;
      }
    }
    return true;
  }
  __shared__ int s_last;
  __shared__ uint32_t s_page_rel[kMaxStages];  // warps done with a stage, this tile
  const AttnSpan s = attn_span(P, T);
  const int hd = P.head_dim, grp = P.group, page = P.page_tokens;
  const int nq = grp * hd;
  float* part = P.part + ((((size_t)s.b * P.n_kv + s.g) * P.n_splits + s.j) * grp) * (2 + hd);
  // shared scratch (the activation buffer): q permuted per head as
  // [half][unit][4], the current token's k and v, each warp's per-head
  // (m, l, o), each warp's probabilities [32][grp]
  float* q_perm = Sh.act;                          // [grp][hd]
  float* kv_cur = q_perm + kMaxGroup * hd;         // [2][hd]
  float* st_s = kv_cur + 2 * kHeadDim;             // [kWarps][grp][2 + hd]
  float* p_s = st_s + kWarps * grp * (2 + kHeadDim);  // [kWarps][32][grp]
  const bool has_cur = s.pos >= s.t0 && s.pos < s.t1;
  (void)page;
  for (int i = threadIdx.x; i < nq; i += kThreads) {
    const float v = P.dec_mma ? __ldcg(P.acc + (size_t)(s.g * nq + i) * P.mma_n + s.b)
                              : __ldcg(P.qbuf + (size_t)s.b * P.q_rows + (size_t)s.g * nq + i);
    const int h = i / hd, d = i % hd, u = d >> 3, e = d & 7;
    q_perm[h * hd + (e >> 2) * 32 + 4 * u + (e & 3)] = v;
  }
  // the current token's k and v were produced this step, after its page was
  // copied: read them directly (tensor-core decode: round the fp32 sums to the
  // cache's bf16 here, store them and clear the sums)
  if (has_cur && threadIdx.x < 2 * hd) {
    const int sel = threadIdx.x / hd, d = threadIdx.x % hd;
    const int blk = P.block_table[s.b * P.max_blocks + s.pos / page];
    uint16_t* dst = P.kv + kv_index(P, T.layer, blk, sel, s.g, s.pos % page) + d;
    uint16_t v;
    if (P.dec_mma) {
      float* a = P.acc + (size_t)(P.q_rows + sel * P.kv_rows + s.g * hd + d) * P.mma_n + s.b;
      v = f2bf(__ldcg(a));
      *a = 0.f;
      *dst = v;
    } else {
      v = __ldcg(dst);
    }
    kv_cur[sel * kHeadDim + d] = bf2f(v);
  }
  if (threadIdx.x < kMaxStages) s_page_rel[threadIdx.x] = 0;
  cbar();
  // Head groups: the kv group's heads are split into n_hg groups of hg heads
  // (hg <= 4), each served by wpg = 8 / n_hg warps over the tile's 32-token
  // blocks.  A long tile reads every K/V row once for all heads (one group);
  // a tile of few blocks splits the heads so that all eight warps have work.
  const int pages = s.t1 > s.t0 ? (s.t1 - 1) / page - s.t0 / page + 1 : 0;  // the split's pages
  const int nb_tot = pages * ((page + 31) / 32);
  int n_hg = 8;
  while (n_hg > 1 && (grp % n_hg || n_hg * nb_tot > kWarps)) n_hg >>= 1;
  while (grp / n_hg > 4 || grp % n_hg) n_hg <<= 1;  // at most four heads per group
  const int hg = grp / n_hg;
  const int wpg = kWarps / n_hg;
  bool ok;
  switch (hg) {
    case 1: ok = attn_pages<1>(P, s, Sh, cur, n_chunks, abort, q_perm, kv_cur, st_s, p_s, s_page_rel, has_cur, wpg); break;
    case 2: ok = attn_pages<2>(P, s, Sh, cur, n_chunks, abort, q_perm, kv_cur, st_s, p_s, s_page_rel, has_cur, wpg); break;
    case 3: ok = attn_pages<3>(P, s, Sh, cur, n_chunks, abort, q_perm, kv_cur, st_s, p_s, s_page_rel, has_cur, wpg); break;
    default: ok = attn_pages<4>(P, s, Sh, cur, n_chunks, abort, q_perm, kv_cur, st_s, p_s, s_page_rel, has_cur, wpg); break;
  }
  if (!cbar_and(ok)) return false;
  // merge the warps of each head; one split: the result directly, else the
  // split's partial (m, l, o) for the combine
  for (int i = threadIdx.x; i < nq; i += kThreads) {
    const int hh = i / hd, d = i % hd;
    const int w0 = (hh / hg) * wpg, hl = hh % hg;  // the warps serving head hh, its slot in their state
    float M = -INFINITY;
    for (int q = w0; q < w0 + wpg; ++q) M = fmaxf(M, st_s[(q * hg + hl) * (2 + kHeadDim)]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY)
      for (int q = w0; q < w0 + wpg; ++q) {
        const float* w = st_s + (q * hg + hl) * (2 + kHeadDim);
        const float f = expf(w[0] - M);
        L = fmaf(w[1], f, L);
        O = fmaf(w[2 + d], f, O);
      }
    if (P.n_splits == 1) {
      attn_result(P, s.b, s.g * nq + i, O / L);
    } else {
      float* pr = part + (size_t)hh * (2 + hd);
      pr[2 + d] = O;
      if (d == 0) {
        pr[0] = M;  // -inf with l = 0 for a split past the current position
        pr[1] = L;
      }
    }
  }
  if (P.n_splits == 1) return true;
  cbar();
  uint32_t* arr = P.arrive + (size_t)s.b * P.n_kv + s.g;
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(arr, 1u);
    s_last = (old == (uint32_t)P.n_splits - 1u);
    __threadfence();
  }
  cbar();
  if (s_last) {
    const float* base = P.part + (((size_t)s.b * P.n_kv + s.g) * P.n_splits) * grp * (2 + hd);
    // (m, l) of every split and head into shared memory in one parallel step
    float* ml = Sh.act;  // [n_splits][grp][2]
    for (int i = threadIdx.x; i < P.n_splits * grp; i += kThreads) {
      const float2 v = __ldcg(reinterpret_cast<const float2*>(base + (size_t)i * (2 + hd)));
      ml[2 * i] = v.x;
      ml[2 * i + 1] = v.y;
    }
    cbar();
    for (int idx = threadIdx.x; idx < nq; idx += kThreads) {
      const int hh = idx / hd, d = idx % hd;
      float M = -INFINITY;
      for (int j = 0; j < P.n_splits; ++j) M = fmaxf(M, ml[2 * (j * grp + hh)]);
      float L = 0.f, O = 0.f;
#pragma unroll 8
      for (int j = 0; j < P.n_splits; ++j) {
        const float w = expf(ml[2 * (j * grp + hh)] - M);
        L = fmaf(ml[2 * (j * grp + hh) + 1], w, L);
        O = fmaf(__ldcg(base + ((size_t)j * grp + hh) * (2 + hd) + 2 + d), w, O);
      }
      attn_result(P, s.b, s.g * nq + idx, O / L);
    }
    if (threadIdx.x == 0) *arr = 0u;
  }
  return true;
}

// ---------------------------------------------------------------------------
// Prefill bodies.  Token row m = b*T + t; block tb holds rows [128 tb, 128 tb + 128).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16x2(float lo_elem, float hi_elem) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ bool body_pembed(const KParams& P, const Tile& T) {
  const uint16_t* E = reinterpret_cast<const uint16_t*>(P.weights + P.embed_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = P.hidden / 8;
  for (int n = warp; n < kTokBlock; n += kWarps) {
    const int m = T.a0 * kTokBlock + n;
    if (m >= P.M) break;
    int tok = P.ptok[m];
    if (tok < 0 || tok >= P.vocab) {
      if (lane == 0) record_error(P, WPK_ERR_INVALID_ARG, (uint32_t)m, kNoCounter, (uint32_t)tok, (uint32_t)P.vocab);
      tok = 0;
    }
    const uint4* row = reinterpret_cast<const uint4*>(E + (size_t)tok * P.hidden);
    float4* x = reinterpret_cast<float4*>(P.px + (size_t)m * P.hidden);
    for (int u = lane; u < units; u += 32) {
      float f[8];
      unpack8(__ldg(row + u), f);
      x[2 * u] = make_float4(f[0], f[1], f[2], f[3]);
      x[2 * u + 1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
  return true;
}

__device__ bool body_gather(const KParams& P) {
  const int nb = active_batch(P);
  for (int b = 0; b < nb; ++b) {
    const float4* src = reinterpret_cast<const float4*>(P.px + ((size_t)b * P.T + P.T - 1) * P.hidden);
    float4* dst = reinterpret_cast<float4*>(P.xa + (size_t)b * P.hidden);
    for (int k = threadIdx.x; k < P.hidden / 4; k += kThreads) dst[k] = __ldcg(src + k);
  }
  return true;
}

// RMSNorm of a token block into the hi/lo bf16 image (rows past M become zero).
__device__ bool body_norm(const KParams& P, const Tile& T) {
  const LayerDev* L = P.layers + T.layer;
  const float* gain = reinterpret_cast<const float*>(P.weights + (T.a1 == 0 ? L->attn_norm : L->ffn_norm));
  const int h = P.hidden, units = h / 8, nkc = h / 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tb = T.a0;
  uint8_t* hi = P.xn_img[0] + (size_t)tb * nkc * P.img_stride;
  uint8_t* lo = P.xn_img[1] + (size_t)tb * nkc * P.img_stride;
  constexpr int kMaxUnits = 2048 / 8 / 32;
  for (int n = T.a2 + warp; n < T.a2 + kNormRows; n += kWarps) {  // the tile's rows of the block
    const int m = tb * kTokBlock + n;
    const bool valid = m < P.M;
    float xr[kMaxUnits][8];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxUnits; ++i) {
      const int u = lane + 32 * i;
      if (u < units && valid) {
        const float4* xs = reinterpret_cast<const float4*>(P.px + (size_t)m * h + 8 * u);
        const float4 a = __ldcg(xs), b = __ldcg(xs + 1);
        xr[i][0] = a.x; xr[i][1] = a.y; xr[i][2] = a.z; xr[i][3] = a.w;
        xr[i][4] = b.x; xr[i][5] = b.y; xr[i][6] = b.z; xr[i][7] = b.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) xr[i][e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += xr[i][e] * xr[i][e];
    }
    ss = warp_sum(ss);
    const float rs = valid ? 1.0f / sqrtf(ss / (float)h + P.eps) : 0.f;
#pragma unroll
    for (int i = 0; i < kMaxUnits; ++i) {
      const int u = lane + 32 * i;
      if (u >= units) continue;
      const int k = 8 * u;
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(gain + k));
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(gain + k + 4));
      const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      uint32_t ph[4], pl[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float a0 = xr[i][e] * rs * gg[e], a1 = xr[i][e + 1] * rs * gg[e + 1];
        const __nv_bfloat162 hv = __floats2bfloat162_rn(a0, a1);
        const float r0 = a0 - __bfloat162float(hv.x), r1 = a1 - __bfloat162float(hv.y);
        ph[e / 2] = *reinterpret_cast<const uint32_t*>(&hv);
        pl[e / 2] = pack_bf16x2(r0, r1);
      }
      const size_t off = (size_t)(k / 64) * P.img_stride + sw128_offset(n, k % 64);
      *reinterpret_cast<uint4*>(hi + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
      *reinterpret_cast<uint4*>(lo + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
    }
  }
  return true;
}

// Batched decode: 1/rms of each token column for the RMSNorm a tile consumes,
// and the tile's best (value, index) key per token of the LM head.
__shared__ float s_rn[kMaxMmaBatch];
__shared__ unsigned long long s_best[kMaxMmaBatch];
// Per token column of a tensor-core QKV tile, filled once per tile: the RoPE
// position (batched decode: the sequence's position, 0 for an idle or absent
// column; prefill: the token's position, -1 past the prompt tokens), and
// (prefill) the element index of the token's row in its KV page for kv head 0's
// K (the other heads and V follow at fixed offsets).  The prefill table shares
// its storage with s_best, which only the batched decode's LM head uses.
__shared__ int s_col_pos[kMaxMmaBatch];
#define s_col_kv s_best

// Adds the 16 token columns n0..n0+15 (those below nb) of one feature row to a
// feature-major fp32 buffer row `dst` (16-byte aligned at column n0).
template <int CW>
__device__ __forceinline__ void red_add_cols(float* dst, const float* o, int n0, int nb) {
#pragma unroll
  for (int j = 0; j < CW; j += 4) {
    if (n0 + j + 4 <= nb) {
      red_add_v4_f32(dst + j, o[j], o[j + 1], o[j + 2], o[j + 3]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (n0 + j + e < nb) atomicAdd(dst + j + e, o[j + e]);
    }
  }
}

__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
  const uint32_t fb = __float_as_uint(v);
  const uint32_t ord = (fb & 0x80000000u) ? ~fb : (fb | 0x80000000u);
  return ((unsigned long long)ord << 32) | (0xFFFFFFFFu - (uint32_t)idx);
}

// Tensor-core tile epilogue for CW token columns n0..n0+CW-1 of feature row fl
// (CW = 8 for the batched decode, whose few columns are split finer so that all
// eight warps share the work; 16 for the prefill).
// Gate/up epilogue output: the even lanes of a warp hold h of its 16
// features (lane / 2) for tokens n0 .. n0 + CW.  The values go through the
// warp's shared scratch ([hi, lo][CW tokens][16 features] bf16) so that the
// image takes 16-byte stores of 8 consecutive features of one token.
template <int CW>
__device__ __forceinline__ void store_h_units(uint8_t* hi, uint8_t* lo, int col0, int n0, const float* hv,
                                              uint16_t* scratch) {
  const int lane = threadIdx.x & 31;
  if ((lane & 1) == 0) {
    const int m = lane >> 1;
#pragma unroll
    for (int i = 0; i < CW; ++i) {
      const __nv_bfloat16 hb = __float2bfloat16_rn(hv[i]);
      const __nv_bfloat16 lb = __float2bfloat16_rn(hv[i] - __bfloat162float(hb));
      scratch[i * 16 + m] = *reinterpret_cast<const uint16_t*>(&hb);
      scratch[(CW + i) * 16 + m] = *reinterpret_cast<const uint16_t*>(&lb);
    }
  }
  __syncwarp();
#pragma unroll
  for (int u = lane; u < 4 * CW; u += 32) {  // (hi or lo, token, feature half)
    const int part = u / (2 * CW), rem = u % (2 * CW), i = rem >> 1, fh = rem & 1;
    const uint4 x = *reinterpret_cast<const uint4*>(scratch + (part * CW + i) * 16 + 8 * fh);
    *reinterpret_cast<uint4*>((part ? lo : hi) + sw128_offset(n0 + i, col0 + 8 * fh)) = x;
  }
  __syncwarp();
}

template <int CW>
__device__ void mma_epilogue(const KParams& P, const Tile& T, int fl, int n0, const float* v, uint16_t* scratch) {
  const int f = T.a0 * 128 + fl;
  const int tb = T.a1;
  const int lane = threadIdx.x & 31;
  const int hd = P.head_dim, half = hd / 2;
  switch (T.op) {
    case OP_BQKV: {
      // 128-row blocks never straddle q / k / v; q and k rows hold RoPE pairs
      // (i, i + hd/2) next to each other (even lane: i, odd lane: i + hd/2)
      const int nb = active_batch(P);
      const bool is_q = f < P.q_rows, is_v = f >= P.q_rows + P.kv_rows;
      const int sec0 = is_q ? 0 : (is_v ? P.q_rows + P.kv_rows : P.q_rows);
      const int head = (f - sec0) / hd, within = (f - sec0) % hd;
      const bool even = (lane & 1) == 0;
      const int pi = within / 2;
      const int dim = is_v ? within : (even ? pi : pi + half);
      float o[CW];
      float2 rp[CW];  // the columns' RoPE factors, loaded before any store
#pragma unroll
      for (int i = 0; i < CW; ++i)
        rp[i] = is_v ? make_float2(1.f, 0.f) : __ldg(P.rope + (size_t)s_col_pos[n0 + i] * half + pi);
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const float y = v[i] * s_rn[n0 + i];
        const float partner = __shfl_xor_sync(0xffffffffu, y, 1);
        if (is_v) {
          o[i] = y;
        } else {
          const float2 cs = rp[i];
          const float y0 = even ? y : partner, y1 = even ? partner : y;
          o[i] = even ? (y0 * cs.x - y1 * cs.y) : (y1 * cs.x + y0 * cs.y);
        }
      }
      red_add_cols<CW>(P.acc + (size_t)(sec0 + head * hd + dim) * P.mma_n + n0, o, n0, nb);
      break;
    }
    case OP_BO:
    case OP_BDOWN:
      red_add_cols<CW>(P.xt + (size_t)f * P.mma_n + n0, v, n0, active_batch(P));
      break;
    case OP_BGU: {
      const int nb = active_batch(P);
      // h features 64 a0 + fl / 2; the warp's 16 start at column (fl - lane) / 2
      uint8_t* hi = P.h_img[0] + (size_t)T.a0 * P.img_stride;
      uint8_t* lo = P.h_img[1] + (size_t)T.a0 * P.img_stride;
      float hv[CW];
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const float g = v[i] * s_rn[n0 + i];
        const float up = __shfl_xor_sync(0xffffffffu, g, 1);
        hv[i] = (n0 + i < nb) ? g / (1.0f + expf(-g)) * up : 0.f;  // even lanes: gate, odd: up
      }
      store_h_units<CW>(hi, lo, (fl - lane) / 2, n0, hv, scratch);
      break;
    }
    case OP_BLM: {
      const int nb = active_batch(P);
      const bool valid = f < P.lm_rows;
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const int n = n0 + i;
        const float val = v[i] * s_rn[n];
        if (s_logits && valid && n < nb) s_logits[(size_t)n * P.logits_stride + f] = val;
        unsigned long long key = valid ? argmax_key(val, f) : 0ull;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
          key = other > key ? other : key;
        }
        if (lane == 0 && n < nb) atomicMax(&s_best[n], key);
      }
      break;
    }
    case OP_MQKV: {
      // per-token position and KV row base come from the tile's table
      // (s_col_pos / s_col_kv, filled once per tile before the epilogue)
      const bool is_v = f >= P.q_rows + P.kv_rows;
      const bool is_q = f < P.q_rows;
      const int sec = is_q ? f : (is_v ? f - P.q_rows - P.kv_rows : f - P.q_rows);
      const int head = sec / hd, within = sec % hd;
      const size_t kv_off = (size_t)(head * 2 + (is_v ? 1 : 0)) * P.page_tokens * hd;  // (head, K or V) in a page row
      const int pi = within / 2;
      const bool even = (lane & 1) == 0;
      const int dim = is_v ? within : (even ? pi : pi + half);
      // every column's RoPE factors first: loaded after the stores below,
      // which may alias them as far as the compiler knows, they would make
      // one round trip each
      float2 rp[CW];
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const int t = s_col_pos[n0 + i];
        rp[i] = (is_v || t < 0) ? make_float2(1.f, 0.f) : __ldg(P.rope + (size_t)t * half + pi);
      }
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const float partner = __shfl_xor_sync(0xffffffffu, v[i], 1);
        const int n = n0 + i;
        const int t = s_col_pos[n];
        if (t < 0) continue;  // a row past the prompt tokens
        if (is_v) {
          P.kv[s_col_kv[n] + kv_off + dim] = f2bf(v[i]);
          continue;
        }
        const float2 cs = rp[i];
        const float y0 = even ? v[i] : partner, y1 = even ? partner : v[i];
        const float o = even ? (y0 * cs.x - y1 * cs.y) : (y1 * cs.x + y0 * cs.y);
        if (is_q)
          P.pq[(size_t)(tb * kTokBlock + n) * P.q_rows + head * hd + dim] = o;
        else
          P.kv[s_col_kv[n] + kv_off + dim] = f2bf(o);
      }
      break;
    }
    case OP_MO:
    case OP_MDOWN: {  // K splits of one row block add into X
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const int m = tb * kTokBlock + n0 + i;
        if (m < P.M) atomicAdd(P.px + (size_t)m * P.hidden + f, v[i]);
      }
      break;
    }
    case OP_MGU: {
      // the warp's 16 h features start at j0 (a multiple of 16: one chunk)
      const int j0 = (f - lane) / 2, c = j0 / 64, nkc = P.ffn / 64;
      uint8_t* hi = P.h_img[0] + ((size_t)tb * nkc + c) * P.img_stride;
      uint8_t* lo = P.h_img[1] + ((size_t)tb * nkc + c) * P.img_stride;
      float hv[CW];
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const float up = __shfl_xor_sync(0xffffffffu, v[i], 1);
        const float g = v[i];
        hv[i] = (tb * kTokBlock + n0 + i < P.M) ? g / (1.0f + expf(-g)) * up : 0.f;  // even lanes: gate, odd: up
      }
      store_h_units<CW>(hi, lo, j0 % 64, n0, hv, scratch);
      break;
    }
    default:
      break;
  }
}

// Batched decode, after an O or down tile: the last of the K splits of its
// 128-row block to finish holds the block's final residual rows.  It writes
// them, times the gain of the RMSNorm that reads them next (this layer's FFN
// norm after O; the next layer's attention norm, or the final norm, after
// down), into that norm's hi/lo input image and adds their squares to the
// per-token sums of x^2 (the consumers scale by 1/rms per token).  Splits
// arrive on a counter per row block (release/acquire through fences, as the
// attention combine).  Columns past the active batch get zeros.
__device__ void rowblock_done(const KParams& P, const Tile& T) {
  __shared__ int s_last_rb;
  __shared__ float s_sq[kMaxMmaBatch];
  const bool down = T.op == OP_BDOWN;
  const int splits = down ? P.down_splits : P.o_splits;
  const int N = P.mma_n, nb = active_batch(P);
  if (threadIdx.x < N) s_sq[threadIdx.x] = 0.f;
  if (threadIdx.x == 0) {
    uint32_t* a = P.rb_arrive + ((size_t)T.layer * 2 + (down ? 1 : 0)) * (P.hidden / 128) + T.a0;
    __threadfence();
    const uint32_t old = atomicAdd(a, 1u);
    s_last_rb = old == (uint32_t)splits - 1u;
    if (s_last_rb) *a = 0u;
    __threadfence();
  }
  cbar();
  if (!s_last_rb) return;
  const int nidx = down ? 2 * T.layer + 2 : 2 * T.layer + 1;
  const uint64_t goff = !down ? P.layers[T.layer].ffn_norm
                              : (T.layer + 1 < P.n_layers ? P.layers[T.layer + 1].attn_norm : P.final_norm_off);
  const float* gain = reinterpret_cast<const float*>(P.weights + goff);
  uint8_t* const* img = down ? P.xn_img : P.xf_img;
  for (int u = threadIdx.x; u < 16 * N; u += kThreads) {  // (8 features, token n) per step
    const int j = u / N, n = u % N;
    const int f0 = T.a0 * 128 + 8 * j;
    float x[8];
    float sq = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      x[e] = n < nb ? __ldcg(P.xt + (size_t)(f0 + e) * N + n) : 0.f;
      sq = fmaf(x[e], x[e], sq);
    }
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(gain + f0));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(gain + f0 + 4));
    const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    uint32_t ph[4], pl[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float a0 = x[e] * gg[e], a1 = x[e + 1] * gg[e + 1];
      const __nv_bfloat162 hv = __floats2bfloat162_rn(a0, a1);
      ph[e / 2] = *reinterpret_cast<const uint32_t*>(&hv);
      pl[e / 2] = pack_bf16x2(a0 - __bfloat162float(hv.x), a1 - __bfloat162float(hv.y));
    }
    const size_t off = (size_t)(f0 / 64) * P.img_stride + sw128_offset(n, f0 % 64);
    *reinterpret_cast<uint4*>(img[0] + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
    *reinterpret_cast<uint4*>(img[1] + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
    if (n < nb) atomicAdd(&s_sq[n], sq);
  }
  cbar();
  if (threadIdx.x < nb) atomicAdd(P.ss + (size_t)nidx * N + threadIdx.x, s_sq[threadIdx.x]);
}

// Issues the MMAs of one tensor-core tile (D[128 features][128 tokens] =
// W . (a_hi + a_lo)^T over its K chunks) into the accumulator buffer at TMEM
// column `tmem`, committing each stage back to the producer as its MMAs
// complete.  The hi and lo activation rows sit back to back in the stage, so
// one MMA with N' = 2N covers both: columns [0, N) get W . hi, [N, 2N) W . lo.
// Successive K-steps rotate over the buffer's NA accumulators (2N columns
// each), so that small-N MMAs do not wait on one another.  Run by the issuer
// warp's lane 0; `c` is the tile's first chunk.
__device__ bool issue_tile_mmas(const KParams& P, const Tile& T, const Shared& S, uint32_t c, int n_chunks,
                                uint32_t tmem, volatile int* abort, uint32_t tile) {
  const int N = P.mma_n, NA = P.mma_acc;
  const uint32_t idesc = idesc_f16(128, 2 * N, true);
  uint32_t mi = 0;  // MMAs issued for this tile
  for (int k = 0; k < n_chunks; ++k, ++c) {  // one unit of K chunks per stage
    const int st = c % P.n_stages;
    if (!wait_phase(P, &S.full[st], (c / P.n_stages) & 1u, abort, tile)) return false;
    tc_fence_after();
    const uint32_t base = smem_u32(S.ring + (size_t)st * P.stage_bytes);
    const uint32_t act = base + (uint32_t)P.mma_cps * kMmaChunkBytes;
    const int nc = mma_unit(P, T, k).nc;
    for (int j = 0; j < nc; ++j) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk, ++mi) {
        const int a = (int)(mi % (uint32_t)NA);
        umma_f16(tmem + (uint32_t)(a * 2 * N), sdesc_k_sw128(base + j * kMmaChunkBytes + kk * 32),
                 sdesc_k_sw128(act + j * 2 * P.act_chunk + kk * 32), idesc, mi >= (uint32_t)NA ? 1u : 0u);
      }
    }
    umma_commit(&S.empty[st]);
  }
  return true;
}

// Tensor-core tile, consumer side: the issuer warp has issued (or is issuing)
// the tile's MMAs into accumulator buffer n_mma % 2; the compute warps build
// the epilogue's tables meanwhile, wait for the accumulators, read TMEM and
// hand the buffer back.
__device__ bool body_mma(const KParams& P, const Tile& T, const Shared& S, Cursor& cur, int n_chunks,
                         ConsumerState& cs, volatile int* abort, uint32_t tile) {
  const int N = P.mma_n, NA = P.mma_acc;
  const int buf = (int)(cs.n_mma & 1u);
  const uint32_t use = cs.n_mma >> 1;
  const uint32_t tmem = s_tmem + (uint32_t)(buf * P.mma_buf_cols);
  // QKV tiles: the per-column position / KV-row table
  if (T.op == OP_BQKV || T.op == OP_MQKV) {
    const int n = (int)threadIdx.x;
    if (n >= 0 && n < N) {
      if (T.op == OP_BQKV) {
        s_col_pos[n] = (n < active_batch(P) && slot_on(P, n)) ? P.seqlen[n] : 0;
      } else {
        const int m = T.a1 * kTokBlock + n;
        if (m < P.M) {
          const int b = P.slot0 + m / P.T, t = m % P.T;
          const int blk = P.block_table[b * P.max_blocks + t / P.page_tokens];
          s_col_pos[n] = t;
          s_col_kv[n] = kv_index(P, T.layer, blk, 0, 0, t % P.page_tokens);
        } else {
          s_col_pos[n] = -1;
        }
      }
    }
  }
  // batched decode: 1/rms per token column of the RMSNorm this tile consumes
  // (its x^2 sums are complete: the tile's counter covers every contribution)
  if (T.op == OP_BQKV || T.op == OP_BGU || T.op == OP_BLM) {
    const int idx = T.op == OP_BQKV ? 2 * T.layer : (T.op == OP_BGU ? 2 * T.layer + 1 : 2 * P.n_layers);
    if (threadIdx.x < N)
      s_rn[threadIdx.x] = 1.0f / sqrtf(__ldcg(P.ss + (size_t)idx * N + threadIdx.x) / (float)P.hidden + P.eps);
    if (threadIdx.x < N) s_best[threadIdx.x] = 0ull;
  }
  cbar();
  bool ok = true;
  // (slack: the wait covers the tile's whole mainloop)
  if (!wait_phase(P, &s_accf[buf], use & 1u, abort, tile, 4)) ok = false;
  if (P.trace && threadIdx.x == 0) s_t_data = globaltimer();  // the accumulators are complete
  ++cs.n_mma;
  cur.c += n_chunks;
  if (!cbar_and(ok)) return false;
  tc_fence_after();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3, half = warp >> 2;
  const int fl = 32 * q + lane;
  // the warp's shared scratch for the gate/up output (the activation buffer:
  // no other tile body uses it while this one runs)
  uint16_t* scratch = reinterpret_cast<uint16_t*>(S.act) + warp * (2 * 16 * 16);
  if (P.dec_mma) {
    for (int cg = half; cg < N / 8; cg += 2) {  // 8-column groups alternate between the two warp halves
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
      const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(8 * cg);
      for (int a = 0; a < NA; ++a)  // hi and lo parts of every accumulator
        tmem_add8x2(lane_base + (uint32_t)(a * 2 * N), lane_base + (uint32_t)(a * 2 * N + N), v);
      mma_epilogue<8>(P, T, fl, 8 * cg, v, scratch);
    }
  } else {
    for (int cg = half; cg < N / 16; cg += 2) {  // 16-column groups alternate between the two warp halves
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.f;
      const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(16 * cg);
      for (int a = 0; a < NA; ++a)  // hi and lo parts of every accumulator
        tmem_add16x2(lane_base + (uint32_t)(a * 2 * N), lane_base + (uint32_t)(a * 2 * N + N), v);
      mma_epilogue<16>(P, T, fl, 16 * cg, v, scratch);
    }
  }
  tc_fence_before();
  cbar();
  if (threadIdx.x == 0) mbar_arrive(&s_acce[buf]);  // the buffer's TMEM has been read
  if (T.op == OP_BO || T.op == OP_BDOWN) {
    rowblock_done(P, T);
  } else if (T.op == OP_BLM) {
    const int nb = active_batch(P);
    if (threadIdx.x < nb && s_best[threadIdx.x]) atomicMax(P.best + threadIdx.x, s_best[threadIdx.x]);
  }
  return true;
}

// Causal GQA attention for the queries [t0, t1) of sequence b and the query
// heads of kv head g, on the tensor cores.  The tile's 128 rows (query qi and
// head hh at row qi * group + hh) are the MMA's M and TMEM lanes 0-127; warps
// w and w + 4 share TMEM lanes 32 (w % 4) ..: each thread owns one row and one
// half of its keys and of its output dims.  Per staged KV page of 64 keys:
//   1. all warps build, in the stage, the page's K rows and its V transposed
//      ([dim][key]) as K-major operands with the 128-byte swizzle;
//   2. S = (Q_hi + Q_lo) K^T on the tensor cores, Q (scaled by log2(e) /
//      sqrt(d), so that the softmax runs in base 2) split into bf16 hi and lo
//      halves held in TMEM;
//   3. each row's online softmax over S (causal mask key <= query), the two
//      halves exchanging their maxima and sums through shared memory; the
//      probabilities split into bf16 hi and lo, written to TMEM;
//   4. O_page = (P_hi + P_lo) V^T on the tensor cores, added into the row's
//      fp32 output registers.
// The hi/lo splits keep q and p to about 16 significant bits; K and V are
// the cache's bf16 values; every product accumulates in fp32.  A query block
// split along the keys (pattn_ks) writes each split's (m, l, o) partial and
// the last split to finish combines them, as the decode attention does.
namespace pattn {
constexpr uint32_t kS = 0, kO = 64, kQh = 128, kQl = 160, kPh = 192, kPl = 224;  // TMEM columns
constexpr int kKRows = 16384, kVt = 24576;  // stage offsets of the swizzled K rows and V transposed
constexpr float kQScale = 0.125f * 1.44269504088896341f;  // log2(e) / sqrt(64)
}

__device__ bool body_pattn(const KParams& P, const Tile& T, const Shared& S, Cursor& cur, int n_chunks,
                           ConsumerState& cs, volatile int* abort, uint32_t tile) {
  const int b = T.a0, g = T.a1, grp = P.group, hd = P.head_dim;
  int t0, t1, k_first, k_end;
  pattn_span(P, T, &t0, &t1);
  pattn_keys(P, T, t1, &k_first, &k_end);
  k_first = k_first / P.page_tokens * P.page_tokens;  // splits start on a page
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hw = warp >> 2;                // key half (S columns) and dim half (O columns)
  const int r = 32 * (warp & 3) + lane;    // the row: TMEM lane
  const int qi = r / grp, hh = r % grp;
  const int t = t0 + qi;
  const bool valid = t < t1;
  const int m = b * P.T + (valid ? t : t0);
  const int head = g * grp + hh;
  const uint32_t tmem = s_tmem;
  const uint32_t lane_addr = ((uint32_t)(32 * (warp & 3)) << 16);
  // the two halves' row maxima and sums: red[max or sum][key half][row], in
  // the activation buffer (the program's GEMV tiles restage it)
  float(*red)[2][128] = reinterpret_cast<float(*)[2][128]>(S.act);
  // Q row -> TMEM (hi, lo): dims [32 hw, 32 hw + 32), all loads first
  {
    const float4* qs = reinterpret_cast<const float4*>(P.pq + (size_t)m * P.q_rows + head * hd + 32 * hw);
    float4 q4[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) q4[e] = __ldcg(qs + e);
#pragma unroll
    for (int c = 0; c < 2; ++c) {  // 16 dims = 8 columns per store
      uint32_t hi[8], lo[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 x = q4[4 * c + e];
        const float qv[4] = {x.x * pattn::kQScale, x.y * pattn::kQScale, x.z * pattn::kQScale, x.w * pattn::kQScale};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const __nv_bfloat162 hv = __floats2bfloat162_rn(qv[2 * h2], qv[2 * h2 + 1]);
          hi[2 * e + h2] = *reinterpret_cast<const uint32_t*>(&hv);
          lo[2 * e + h2] = pack_bf16x2(qv[2 * h2] - __bfloat162float(hv.x), qv[2 * h2 + 1] - __bfloat162float(hv.y));
        }
      }
      tmem_st8(tmem + lane_addr + pattn::kQh + 16 * hw + 8 * c, hi);
      tmem_st8(tmem + lane_addr + pattn::kQl + 16 * hw + 8 * c, lo);
    }
    tmem_st_wait();
  }
  float o[32];  // output dims [32 hw, 32 hw + 32) of the row
#pragma unroll
  for (int d = 0; d < 32; ++d) o[d] = 0.f;
  float mrun = -INFINITY, lrun = 0.f;  // base-2 running max and sum (identical in both halves)
  const uint32_t idesc = idesc_f16(128, 64, true);
  bool ok = true;
  for (int k = 0; k < n_chunks; ++k) {
    const int st = cur.c % P.n_stages;
    if (!wait_phase(P, &S.full[st], (cur.c / P.n_stages) & 1u, abort, tile)) ok = false;
    if (!cbar_and(ok)) return false;
    uint8_t* stage = S.ring + (size_t)st * P.stage_bytes;
    const int kp = k_first + k * P.page_tokens;  // first key of this page
    const int rows = min(P.page_tokens, k_end - kp);
    // 1. swizzled K rows (unit u of row j at u ^ (j & 7)) and V transposed
    {
      const uint4* kr = reinterpret_cast<const uint4*>(stage);
      for (int i = threadIdx.x; i < 64 * 8; i += kThreads) {
        const int j = i >> 3, u = i & 7;
        const uint4 v = j < rows ? kr[i] : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(stage + pattn::kKRows + j * 128 + ((u ^ (j & 7)) << 4)) = v;
      }
      const uint16_t* vr = reinterpret_cast<const uint16_t*>(stage + (size_t)P.page_tokens * hd * 2);
      for (int i = threadIdx.x; i < 64 * 8; i += kThreads) {  // (dim d, keys 8 ku .. 8 ku + 7)
        const int d = i & 63, ku = i >> 6;  // a warp reads 32 adjacent dims of one key row
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j0 = 8 * ku + 2 * e;
          const uint32_t x0 = j0 < rows ? vr[j0 * 64 + d] : 0u, x1 = j0 + 1 < rows ? vr[(j0 + 1) * 64 + d] : 0u;
          w[e] = x0 | (x1 << 16);
        }
        *reinterpret_cast<uint4*>(stage + pattn::kVt + d * 128 + ((ku ^ (d & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    fence_proxy_async_smem();  // the MMAs read these generic-proxy writes
    tc_fence_before();
    cbar();
    tc_fence_after();
    // 2. S = Q K^T
    if (threadIdx.x == 0) {
      const uint32_t kb = smem_u32(stage + pattn::kKRows);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        umma_f16_ta(tmem + pattn::kS, tmem + pattn::kQh + 8 * kk, sdesc_k_sw128(kb + kk * 32), idesc, kk > 0);
        umma_f16_ta(tmem + pattn::kS, tmem + pattn::kQl + 8 * kk, sdesc_k_sw128(kb + kk * 32), idesc, 1u);
      }
      umma_commit(S.acc);
    }
    if (!wait_phase(P, S.acc, cs.acc_phase, abort, tile)) ok = false;
    cs.acc_phase ^= 1u;
    if (!cbar_and(ok)) return false;
    tc_fence_after();
    // 3. online softmax of the row over the page's keys [32 hw, 32 hw + 32)
    float sv[32];
    tmem_ld16x2(tmem + lane_addr + pattn::kS + 32 * hw, sv);
    float mx = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) {
      const int j = 32 * hw + jj;
      const bool live = valid && j < rows && kp + j <= t;
      sv[jj] = live ? sv[jj] : -INFINITY;
      mx = fmaxf(mx, sv[jj]);
    }
    red[0][hw][r] = mx;
    cbar();
    const float mnew = fmaxf(mrun, fmaxf(mx, red[0][hw ^ 1][r]));
    // (a row with no live key yet keeps m = -inf, its p = 0 and corr = 1)
    const float corr = mnew == -INFINITY ? 1.f : (mrun == -INFINITY ? 0.f : exp2f(mrun - mnew));
    float psum = 0.f;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t hi[8], lo[8];
#pragma unroll
      for (int jj = 0; jj < 16; jj += 2) {
        const float p0 = sv[16 * c + jj] == -INFINITY ? 0.f : exp2f(sv[16 * c + jj] - mnew);
        const float p1 = sv[16 * c + jj + 1] == -INFINITY ? 0.f : exp2f(sv[16 * c + jj + 1] - mnew);
        psum += p0 + p1;
        const __nv_bfloat162 hv = __floats2bfloat162_rn(p0, p1);
        hi[jj / 2] = *reinterpret_cast<const uint32_t*>(&hv);
        lo[jj / 2] = pack_bf16x2(p0 - __bfloat162float(hv.x), p1 - __bfloat162float(hv.y));
      }
      tmem_st8(tmem + lane_addr + pattn::kPh + 16 * hw + 8 * c, hi);
      tmem_st8(tmem + lane_addr + pattn::kPl + 16 * hw + 8 * c, lo);
    }
    red[1][hw][r] = psum;
    tmem_st_wait();
    tc_fence_before();
    cbar();
    tc_fence_after();
    lrun = lrun * corr + (psum + red[1][hw ^ 1][r]);
    mrun = mnew;
    // 4. O_page = P V^T
    if (threadIdx.x == 0) {
      const uint32_t vb = smem_u32(stage + pattn::kVt);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        umma_f16_ta(tmem + pattn::kO, tmem + pattn::kPh + 8 * kk, sdesc_k_sw128(vb + kk * 32), idesc, kk > 0);
        umma_f16_ta(tmem + pattn::kO, tmem + pattn::kPl + 8 * kk, sdesc_k_sw128(vb + kk * 32), idesc, 1u);
      }
      umma_commit(S.acc);
    }
    if (!wait_phase(P, S.acc, cs.acc_phase, abort, tile)) ok = false;
    cs.acc_phase ^= 1u;
    if (!cbar_and(ok)) return false;
    tc_fence_after();
    {
      float ov[32];
      tmem_ld16x2(tmem + lane_addr + pattn::kO + 32 * hw, ov);
#pragma unroll
      for (int d = 0; d < 32; ++d) o[d] = fmaf(o[d], corr, ov[d]);
    }
    // the stage and the TMEM operands are free again: hand the stage back
    tc_fence_before();
    cbar();
    if (threadIdx.x == 0) mbar_arrive(&S.empty[st]);
    ++cur.c;
  }
  const int n_ks = P.pattn_ks ? (t1 + P.pattn_ks - 1) / P.pattn_ks : 1;
  if (n_ks > 1) {
    // a key split: store this split's (m, l, o) of every row; the last split
    // of the (sequence, kv head, query block) to arrive combines them
    const int n_qb = (P.T + kTokBlock / grp - 1) / (kTokBlock / grp);
    const int idx = (b * P.n_kv + g) * n_qb + T.a2;
    float* base = P.ppart + (size_t)idx * kMaxKeySplits * 128 * (2 + kHeadDim);
    float* mine = base + ((size_t)T.a3 * 128 + r) * (2 + kHeadDim);
#pragma unroll
    for (int d = 0; d < 32; d += 2)  // records are 66 floats: 8-byte aligned
      *reinterpret_cast<float2*>(mine + 2 + 32 * hw + d) = make_float2(o[d], o[d + 1]);
    if (hw == 0) {
      mine[0] = mrun;  // -inf with l = 0 when no key of the split is at or before the query
      mine[1] = lrun;
    }
    __shared__ int s_last_split;
    cbar();
    if (threadIdx.x == 0) {
      __threadfence();
      const uint32_t old = atomicAdd(P.pattn_arrive + idx, 1u);
      s_last_split = old == (uint32_t)n_ks - 1u;
      if (s_last_split) P.pattn_arrive[idx] = 0u;
      __threadfence();
    }
    cbar();
    if (!s_last_split) return true;
    float M = -INFINITY;
    for (int j = 0; j < n_ks; ++j) M = fmaxf(M, __ldcg(base + ((size_t)j * 128 + r) * (2 + kHeadDim)));
    lrun = 0.f;
#pragma unroll
    for (int d = 0; d < 32; ++d) o[d] = 0.f;
    for (int j = 0; j < n_ks; ++j) {
      const float* w = base + ((size_t)j * 128 + r) * (2 + kHeadDim);
      const float f = M == -INFINITY ? 0.f : exp2f(__ldcg(w) - M);
      lrun = fmaf(__ldcg(w + 1), f, lrun);
#pragma unroll
      for (int d = 0; d < 32; d += 2) {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(w + 2 + 32 * hw + d));
        o[d] = fmaf(x.x, f, o[d]);
        o[d + 1] = fmaf(x.y, f, o[d + 1]);
      }
    }
  }
  if (valid) {
    const float inv = 1.0f / lrun;
    const int tb = m / kTokBlock, n = m % kTokBlock, nkc = P.q_rows / 64;
    const size_t blk = ((size_t)tb * nkc + head) * P.img_stride;  // 64-column chunk == one head
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t ph[4], pl[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float a0 = o[8 * u + e] * inv, a1 = o[8 * u + e + 1] * inv;
        const __nv_bfloat162 hv = __floats2bfloat162_rn(a0, a1);
        ph[e / 2] = *reinterpret_cast<const uint32_t*>(&hv);
        pl[e / 2] = pack_bf16x2(a0 - __bfloat162float(hv.x), a1 - __bfloat162float(hv.y));
      }
      const uint32_t off = sw128_offset(n, 32 * hw + 8 * u);
      *reinterpret_cast<uint4*>(P.att_img[0] + blk + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
      *reinterpret_cast<uint4*>(P.att_img[1] + blk + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
    }
  }
  return true;
}

// x[b] = the step's input of sequence b: the sum over n_in tables of
// table_k[code_k] (code_k at input row b, column k; the last greedy token when
// no input is given), or the vector in_vec[b] when n_in == 0.
__device__ bool step_codes(const KParams& P, int b, int* codes) {
  if (threadIdx.x < P.n_in) {
    int tok = s_in_tok ? s_in_tok[(size_t)b * s_in_stride + threadIdx.x] : P.tok_fb[b];
    if (!slot_on(P, b)) tok = 0;  // an inactive slot gets a neutral input
    if (tok < 0 || tok >= P.in_rows) {
      record_error(P, WPK_ERR_INVALID_ARG, (uint32_t)b, kNoCounter, (uint32_t)tok, (uint32_t)P.in_rows);
      tok = 0;
    }
    codes[threadIdx.x] = tok;
  }
  return true;
}

__device__ bool body_embed(const KParams& P) {
  __shared__ int s_code[kMaxInTables];
  const int nb = active_batch(P);
  for (int b = 0; b < nb; ++b) {
    step_codes(P, b, s_code);
    cbar();
    float* x = P.xa + (size_t)b * P.hidden;
    for (int k = threadIdx.x; k < P.hidden / 8; k += kThreads) {
      float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (P.n_in == 0) {
        const float4* v = reinterpret_cast<const float4*>(P.in_vec + (size_t)b * P.hidden) + 2 * k;
        const float4 a = __ldcg(v), c = __ldcg(v + 1);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = c.x; f[5] = c.y; f[6] = c.z; f[7] = c.w;
      }
      for (int t = 0; t < P.n_in; ++t) {
        const uint4* row = reinterpret_cast<const uint4*>(P.weights + P.in_table_off[t]) + (size_t)s_code[t] * (P.hidden / 8);
        float e[8];
        unpack8(__ldg(row + k), e);
#pragma unroll
        for (int q = 0; q < 8; ++q) f[q] += e[q];
      }
      reinterpret_cast<float4*>(x)[2 * k] = make_float4(f[0], f[1], f[2], f[3]);
      reinterpret_cast<float4*>(x)[2 * k + 1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    cbar();
  }
  return true;
}

// Batched decode: x = E[tok] for the 128 features of block a0, feature-major,
// with the first RMSNorm's input image (x * g) and the x^2 sums.
__device__ bool body_embed_mma(const KParams& P, const Tile& T, int* codes /* [mma_n][n_in], shared */) {
  __shared__ float s_sq2[kMaxMmaBatch];
  const int N = P.mma_n, nb = active_batch(P);
  for (int i = threadIdx.x; i < N * P.n_in; i += kThreads) {
    const int n = i / P.n_in, t = i % P.n_in;
    int tok = 0;
    if (n < nb) {
      tok = s_in_tok ? s_in_tok[(size_t)n * s_in_stride + t] : P.tok_fb[n];
      if (!slot_on(P, n)) tok = 0;  // an inactive slot gets a neutral input
      if (tok < 0 || tok >= P.in_rows) {
        record_error(P, WPK_ERR_INVALID_ARG, (uint32_t)n, kNoCounter, (uint32_t)tok, (uint32_t)P.in_rows);
        tok = 0;
      }
    }
    codes[i] = tok;
  }
  if (threadIdx.x < N) s_sq2[threadIdx.x] = 0.f;
  cbar();
  const float* gain = reinterpret_cast<const float*>(P.weights + P.layers[0].attn_norm);
  for (int u = threadIdx.x; u < 16 * N; u += kThreads) {
    const int j = u / N, n = u % N;
    const int f0 = T.a0 * 128 + 8 * j;
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (n < nb) {
      if (P.n_in == 0) {
        const float4* v = reinterpret_cast<const float4*>(P.in_vec + (size_t)n * P.hidden + f0);
        const float4 a = __ldcg(v), c = __ldcg(v + 1);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = c.x; x[5] = c.y; x[6] = c.z; x[7] = c.w;
      }
      for (int t = 0; t < P.n_in; ++t) {
        const uint16_t* E = reinterpret_cast<const uint16_t*>(P.weights + P.in_table_off[t]);
        float e[8];
        unpack8(__ldg(reinterpret_cast<const uint4*>(E + (size_t)codes[n * P.n_in + t] * P.hidden + f0)), e);
#pragma unroll
        for (int q = 0; q < 8; ++q) x[q] += e[q];
      }
    }
    float sq = 0.f;
    uint32_t ph[4], pl[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      sq = fmaf(x[e], x[e], fmaf(x[e + 1], x[e + 1], sq));
      const float a0 = x[e] * gain[f0 + e], a1 = x[e + 1] * gain[f0 + e + 1];
      const __nv_bfloat162 hv = __floats2bfloat162_rn(a0, a1);
      ph[e / 2] = *reinterpret_cast<const uint32_t*>(&hv);
      pl[e / 2] = pack_bf16x2(a0 - __bfloat162float(hv.x), a1 - __bfloat162float(hv.y));
    }
    if (n < nb) {
#pragma unroll
      for (int e = 0; e < 8; ++e) P.xt[(size_t)(f0 + e) * N + n] = x[e];
      atomicAdd(&s_sq2[n], sq);
    }
    const size_t off = (size_t)(f0 / 64) * P.img_stride + sw128_offset(n, f0 % 64);
    *reinterpret_cast<uint4*>(P.xn_img[0] + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
    *reinterpret_cast<uint4*>(P.xn_img[1] + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
  }
  cbar();
  if (threadIdx.x < nb) atomicAdd(P.ss + threadIdx.x, s_sq2[threadIdx.x]);
  return true;
}

__device__ bool body_final(const KParams& P, uint32_t epoch) {
  const int nb = active_batch(P);
  if (P.dec_mma)  // the x^2 sums start from zero next step
    for (int i = threadIdx.x; i < (2 * P.n_layers + 1) * P.mma_n; i += kThreads) P.ss[i] = 0.f;
  for (int b = threadIdx.x; b < nb; b += kThreads) {
    const unsigned long long key = P.best[b];
    const int32_t idx = (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
    const int sb = P.slot0 + b;  // the prefill program's sequence b fills slot slot0 + b
    const bool on = slot_on(P, sb);
    if (s_out_tok) s_out_tok[(size_t)b * P.out_stride] = on ? idx : -1;
    if (on) {
      P.tok_fb[sb] = idx;
      P.seqlen[sb] += 1;
    }
    P.best[b] = 0ull;
  }
  if (P.resident) {  // the step is complete: tell the host
    cbar();
    if (threadIdx.x == 0) {
      __threadfence_system();
      P.ctl->t_done_ns = globaltimer();
      __threadfence_system();
      P.ctl->ack = epoch;
    }
  }
  return true;
}

// Thread 0 of the consumers: bounded acquire-wait until the tile's counter
// reaches need x epoch.
__device__ bool wait_counter(const KParams& P, const Tile& T, uint32_t tile, uint32_t epoch, volatile int* abort) {
  if (T.wait_ctr == kNoCounter) return true;
  const uint32_t target = T.need * epoch;
  const uint32_t* ctr = P.ctr + T.wait_ctr;
  uint32_t v = ld_acquire_u32(ctr);
  if ((int32_t)(v - target) >= 0) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    v = ld_acquire_u32(ctr);
    if ((int32_t)(v - target) >= 0) return true;
    if ((it & 15) == 0) {
      if (*abort || ld_volatile_s32(&P.err->code) != 0) return false;
      if (globaltimer() - t0 > P.timeout_ns) {
        record_error(P, WPK_ERR_TIMEOUT, tile, T.wait_ctr, v, target);
        return false;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// The worker: producer warp (warp 8) + consumer warps (0..7).
// ---------------------------------------------------------------------------
// Program kinds: each kernel carries only the tile bodies its program uses, so
// that the compiler sizes registers for that program alone.
constexpr int kProgGemv = 0;     // decode on CUDA cores (GEMV tiles)
constexpr int kProgMma = 1;      // batched decode on tensor cores
constexpr int kProgPrefill = 2;  // prefill (tensor-core tiles, causal attention, GEMV LM head)

template <int kProg>
__device__ void worker(const KParams& P, uint8_t* smem_raw) {
  // the 128-byte-swizzled tensor-core operands need 1024-byte aligned stages
  if (P.uses_tmem && (smem_u32(smem_raw) & 1023u)) {
    if (threadIdx.x == 0) record_error(P, WPK_ERR_UNSUPPORTED, 0xFFFFFFFFu, kNoCounter, smem_u32(smem_raw), 1024u);
    return;
  }
  const Shared S = carve(smem_raw, P);
  __shared__ volatile int s_abort;
  __shared__ uint32_t s_prod_chunks;  // chunks the producer issued
  __shared__ uint32_t s_cons_chunks;  // chunks the consumers finished
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < P.n_stages; ++i) {
      mbar_init(&S.full[i], 1);
      mbar_init(&S.empty[i], (uint32_t)P.gemv_cps);
    }
    for (int i = 0; i < kMaxQueue; ++i) {
      mbar_init(&S.tq_full[i], 1);
      // released by the consumers, and in tensor-core programs by the issuer
      mbar_init(&S.tq_empty[i], kProg == kProgGemv ? 1 : 2);
    }
    mbar_init(S.acc, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_accf[i], 1);
      mbar_init(&s_acce[i], 1);
    }
    mbar_init(&s_mma_fin, 1);
    s_cons_tiles = 0;
    for (int i = 0; i < kSigQueue; ++i) {
      mbar_init(&S.sig_full[i], 1);
      mbar_init(&S.sig_empty[i], 1);
    }
    fence_mbar_init();
    for (int i = 0; i < kMaxStages; ++i) s_seen[i] = 0;
    s_io_epoch = 0;
    s_abort = 0;
    s_prod_chunks = 0;
    s_cons_chunks = 0;
  }
  if (P.uses_tmem && warp == 0) {
    tmem_alloc(&s_tmem, (uint32_t)P.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == kWarps && (threadIdx.x & 31) == 1) {
    // ----------------------------------------------------------- signaller
    // Release-increments the counters of finished tiles, so that no compute
    // warp stalls on the release fence.  The compute warps' writes reach it
    // through the CTA barrier and the mbarrier hand-off (release/acquire at
    // CTA scope); its gpu-scope release covers them.
    if (!P.per_op)
      for (uint32_t j = 0;; ++j) {
        const int slot = j % kSigQueue;
        if (!wait_phase(P, &S.sig_full[slot], (j / kSigQueue) & 1u, &s_abort, 0xFFFFFFFFu, 4)) break;
        const uint2 req = S.sig_req[slot];
        if (req.y == kSigStop) break;
        for (uint32_t k = 0; k < req.y; ++k) red_release_add_u32(P.ctr + P.sig[req.x + k], 1u);
        mbar_arrive(&S.sig_empty[slot]);
      }
  } else if (warp == kWarps) {
    // ------------------------------------------------------------ producer
    if ((threadIdx.x & 31) == 0) {
      uint32_t c = 0;  // chunks issued
      uint32_t db_seen = 0;  // resident: last step the doorbell showed
      const int Q = P.per_op ? 1 : P.lookahead;
      for (uint32_t i = 0;; ++i) {
        const int slot = i % Q;
        if (i >= (uint32_t)Q && !wait_phase(P, &S.tq_empty[slot], ((i / Q) - 1) & 1u, &s_abort, 0xFFFFFFFFu, 4))
          break;
        uint32_t t;
        if (P.per_op)
          t = (i == 0) ? P.t_begin + blockIdx.x : P.t_end;
        else if (P.team_sched) {  // the worker's compiled stream
          const uint32_t b0 = P.stream_begin[blockIdx.x], len = P.stream_begin[blockIdx.x + 1] - b0;
          t = i < len ? P.stream[b0 + i] : P.t_end;
        } else if (P.static_sched)
          t = P.t_begin + blockIdx.x + i * gridDim.x;  // worker w: tickets w, w + W, ...
        else
          t = P.t_begin + atomicAdd(&P.head[P.region], 1u);
        const uint64_t t_claim = P.trace ? globaltimer() : 0;
        TQEntry& e = S.tq[slot];
        uint32_t epoch = P.epoch;
        if (P.resident) {
          // tickets run on across steps; nothing of a step is copied before
          // the host has asked for it (the previous step is then complete)
          const uint32_t n_tiles = P.t_end - P.t_begin;
          epoch = t / n_tiles + 1;
          t = P.t_begin + t % n_tiles;
          if (!wait_doorbell(P, epoch, &s_abort, &db_seen)) {
            e.valid = 0;
            mbar_arrive(&S.tq_full[slot]);
            break;
          }
          fence_proxy_async_global();
        } else if (t >= P.t_end) {
          e.valid = 0;
          mbar_arrive(&S.tq_full[slot]);
          break;
        }
        e.tile = P.tiles[t];
        e.ticket = t;
        e.epoch = epoch;
        e.valid = 1;
        int nch, rpc;
        tile_chunks(P, e.tile, &nch, &rpc);
        e.n_chunks = nch;
        e.rows_per_chunk = rpc;
        e.ev_issue = P.trace ? atomicAdd(P.evclock, 1u) : 0u;
        e.t_claim = t_claim;
        e.t_issued = 0;
        const Tile T = e.tile;
        mbar_arrive(&S.tq_full[slot]);
        bool stop = false;
        auto stage_ptr = [&](uint32_t cc) { return S.ring + (size_t)(cc % P.n_stages) * P.stage_bytes; };
        auto free_stage = [&](uint32_t cc) {
          const uint32_t use = cc / P.n_stages;
          if (use >= 1 && !wait_phase(P, &S.empty[cc % P.n_stages], (use - 1) & 1u, &s_abort, t, 4)) return false;
          fence_proxy_async_smem();
          return true;
        };
        if (is_mma_op(T.op)) {
          // Weights of the first stages are staged before the dependency wait;
          // the activations are produced inside this program, so they are
          // copied only after the tile's counter is satisfied.
          const int pre = min(nch, P.n_stages);
          const uint32_t c0 = c;
          for (int k = 0; k < pre && !stop; ++k, ++c) {
            if (!free_stage(c)) { stop = true; break; }
            issue_mma_w(P, T, k, stage_ptr(c), &S.full[c % P.n_stages]);
          }
          // (per-op launches get their order from the stream; no counters run)
          if (!stop && !P.per_op && !wait_counter(P, T, t, e.epoch, &s_abort)) stop = true;
          if (!stop) {
            fence_proxy_async_global();
            for (int k = 0; k < pre; ++k) issue_mma_act(P, T, k, stage_ptr(c0 + k), &S.full[(c0 + k) % P.n_stages]);
          }
          for (int k = pre; k < nch && !stop; ++k, ++c) {
            if (!free_stage(c)) { stop = true; break; }
            issue_mma_w(P, T, k, stage_ptr(c), &S.full[c % P.n_stages]);
            issue_mma_act(P, T, k, stage_ptr(c), &S.full[c % P.n_stages]);
          }
        } else {
          if (T.op == OP_PATTN) {  // its KV pages are written inside this program
            if (!P.per_op && !wait_counter(P, T, t, e.epoch, &s_abort)) stop = true;
            else fence_proxy_async_global();
          }
          if (T.op == OP_ATTN || T.op == OP_PATTN) {
            const PageWalk w = page_walk(P, T);
            for (int k = 0; k < nch && !stop; ++k, ++c) {
              int blk[kPagePrefetch];
              page_blocks(w, k, blk);
              if (!free_stage(c)) { stop = true; break; }
              issue_pages(P, T, w, k, blk, stage_ptr(c), &S.full[c % P.n_stages]);
            }
          } else {
            for (int k = 0; k < nch && !stop; ++k, ++c) {
              if (!free_stage(c)) { stop = true; break; }
              issue_chunk(P, T, k, rpc, stage_ptr(c), &S.full[c % P.n_stages]);
            }
          }
        }
        // the entry is still owned by the consumers until they release it;
        // this plain store is only read for the trace record
        if (P.trace) *(volatile uint64_t*)&e.t_issued = globaltimer();
        s_prod_chunks = c;
        if (stop) break;
      }
    }
  } else if (warp == kWarps + 1) {
    // ------------------------------------------------- tensor-core issuer
    // Walks the tile queue in the consumers' order and issues each
    // tensor-core tile's MMAs into one of two TMEM accumulator buffers, so
    // the consumers' epilogue of one tile overlaps the next tile's mainloop.
    if constexpr (kProg != kProgGemv) {
      if ((threadIdx.x & 31) == 0) {
        const int Q = P.per_op ? 1 : P.lookahead;
        uint32_t c = 0;       // the consumers' chunk cursor, mirrored
        uint32_t n_mma = 0;   // tensor-core tiles issued
        uint32_t other = 0;   // 1 + queue position of the last other tile that takes chunks
        bool issued = false;
        for (uint32_t i = 0;; ++i) {
          const int slot = i % Q;
          if (!wait_phase(P, &S.tq_full[slot], (i / Q) & 1u, &s_abort, 0xFFFFFFFFu, 2)) break;
          const TQEntry& e = S.tq[slot];
          const bool valid = e.valid != 0;
          const Tile T = e.tile;
          const uint32_t t = e.ticket;
          const int nch = e.n_chunks;
          mbar_arrive(&S.tq_empty[slot]);  // the issuer's share of the slot's release
          if (!valid) break;
          if (!is_mma_op(T.op)) {
            c += nch;
            // (prefill attention also issues its own MMAs into TMEM)
            if (nch > 0 || T.op == OP_PATTN) other = i + 1;
            continue;
          }
          // The consumers take the chunks of other tiles.  A parity wait
          // only tells a phase from the one before it, so every earlier
          // chunk must have landed before this tile's stages are waited for.
          if (other && !wait_count(P, &s_cons_tiles, other, &s_abort, t)) break;
          const int b = (int)(n_mma & 1u);
          const uint32_t use = n_mma >> 1;
          // the buffer's previous tile has been read out
          if (use >= 1 && !wait_phase(P, &s_acce[b], (use - 1) & 1u, &s_abort, t, 4)) break;
          tc_fence_after();
          issued = true;
          if (!issue_tile_mmas(P, T, S, c, nch, s_tmem + (uint32_t)(b * P.mma_buf_cols), &s_abort, t)) break;
          umma_commit(&s_accf[b]);
          c += nch;
          ++n_mma;
        }
        if (issued) {
          // every MMA issued has completed before TMEM is released (bounded)
          umma_commit(&s_mma_fin);
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&s_mma_fin, 0u))
            if (globaltimer() - t0 > P.timeout_ns) {
              record_error(P, WPK_ERR_TIMEOUT, 0xFFFFFFFDu, kNoCounter, n_mma, 0);
              break;
            }
        }
      }
    }
  } else {
    // ----------------------------------------------------------- consumers
    Cursor cur{0};
    ConsumerState cs{kNoAct, kNoCounter, 0u, 0u, 0u, 0u};
    uint32_t n_sig = 0;  // requests pushed to the signaller (thread 0)
    const int Q = P.per_op ? 1 : P.lookahead;
    __shared__ int s_fail;
    for (uint32_t i = 0;; ++i) {
      const int slot = i % Q;
      if (!wait_phase(P, &S.tq_full[slot], (i / Q) & 1u, &s_abort, 0xFFFFFFFFu, 2)) break;
      const TQEntry& e = S.tq[slot];
      if (!e.valid) break;
      const Tile T = e.tile;
      const uint32_t t = e.ticket;
      const int n_chunks = e.n_chunks, rpc = e.rows_per_chunk;
      if (e.epoch != cs.act_epoch) {  // a staged activation never outlives its step
        cs.act_key = kNoAct;
        cs.act_epoch = e.epoch;
      }
      uint32_t ev_start = 0;
      uint64_t t_start = 0;
      if (threadIdx.x == 0) {
        s_t_data = 0;
        if (e.epoch != s_io_epoch) {  // this step's I/O pointers
          if (P.resident) {  // published by worker 0 before the step number
            s_in_tok = reinterpret_cast<const int32_t*>(__ldcg(&P.rdev->in_tok));
            s_in_stride = __ldcg(&P.rdev->in_stride);
            s_out_tok = reinterpret_cast<int32_t*>(__ldcg(&P.rdev->out_tok));
            s_logits = reinterpret_cast<float*>(__ldcg(&P.rdev->logits));
          } else {
            s_in_tok = P.in_tok;
            s_in_stride = P.in_tok_stride;
            s_out_tok = P.out_tok;
            s_logits = P.logits;
          }
          s_io_epoch = e.epoch;
        }
        bool ok = true;
        if (!P.per_op && (T.wait_ctr != cs.last_ctr || e.epoch != cs.last_epoch)) {
          ok = wait_counter(P, T, t, e.epoch, &s_abort);
          if (ok) {
            cs.last_ctr = T.wait_ctr;
            cs.last_epoch = e.epoch;
          }
        } else if (s_abort) {
          ok = false;
        }
        s_fail = ok ? 0 : 1;
        if (P.trace) {
          t_start = globaltimer();
          if (ok) ev_start = atomicAdd(P.evclock, 1u);
        }
      }
      cbar();
      bool ok = !s_fail;
      if (ok) {
        bool known = true;  // the op belongs to this kernel's program
        switch (T.op) {
          case OP_EMBED:
            if constexpr (kProg == kProgMma)
              ok = body_embed_mma(P, T, reinterpret_cast<int*>(S.act));
            else
              ok = body_embed(P);
            break;
          case OP_ATTN:
            if constexpr (kProg != kProgPrefill) ok = body_attn(P, T, S, cur, n_chunks, &s_abort);
            else known = false;
            break;
          case OP_FINAL: ok = body_final(P, e.epoch); break;
          case OP_PEMBED:
          case OP_GATHER:
          case OP_NORM:
          case OP_PATTN:
          case OP_MQKV:
          case OP_MO:
          case OP_MGU:
          case OP_MDOWN:
            if constexpr (kProg == kProgPrefill) {
              if (T.op == OP_PEMBED) ok = body_pembed(P, T);
              else if (T.op == OP_GATHER) ok = body_gather(P);
              else if (T.op == OP_NORM) ok = body_norm(P, T);
              else if (T.op == OP_PATTN) ok = body_pattn(P, T, S, cur, n_chunks, cs, &s_abort, t);
              else ok = body_mma(P, T, S, cur, n_chunks, cs, &s_abort, t);
            } else {
              known = false;
            }
            break;
          case OP_BQKV:
          case OP_BO:
          case OP_BGU:
          case OP_BDOWN:
          case OP_BLM:
            if constexpr (kProg == kProgMma) ok = body_mma(P, T, S, cur, n_chunks, cs, &s_abort, t);
            else known = false;
            break;
          default:  // GEMV tiles (decode ops, and the prefill's LM head)
            if constexpr (kProg == kProgPrefill)  // (one chunk per stage there)
              ok = body_gemv_t<1>(P, T, S, cur, n_chunks, rpc, cs, &s_abort);
            else if constexpr (kProg != kProgMma)
              ok = body_gemv(P, T, S, cur, n_chunks, rpc, cs, &s_abort);
            else known = false;
            break;
        }
        if (!known) {
          if (threadIdx.x == 0) record_error(P, WPK_ERR_UNSUPPORTED, t, kNoCounter, T.op, (uint32_t)kProg);
          ok = false;
        }
        // attention and tensor-core tiles use the activation buffer as
        // scratch; the gather rewrites the LM head's input
        if (T.op == OP_ATTN || T.op == OP_PATTN || T.op == OP_GATHER || is_mma_op(T.op)) cs.act_key = kNoAct;
      }
      ok = cbar_and(ok);
      if (!ok) {
        if (threadIdx.x == 0) s_abort = 1;
        break;
      }
      if (threadIdx.x == 0) {
        if (P.trace && !P.per_op) {
          TraceRec r;
          r.tile = t;
          r.worker = (uint16_t)blockIdx.x;
          r.op = T.op;
          r.ev_issue = e.ev_issue;
          r.ev_start = ev_start;
          r.ev_done = atomicAdd(P.evclock, 1u);
          r.epoch = e.epoch;
          r.t_claim_ns = e.t_claim;
          r.t_issued_ns = *(volatile uint64_t*)&e.t_issued;
          r.t_start_ns = t_start;
          r.t_data_ns = s_t_data ? s_t_data : t_start;
          r.t_end_ns = globaltimer();
          P.trace_buf[t] = r;
        }
        if (!P.per_op && T.sig_cnt) {
          const int ss = n_sig % kSigQueue;
          if (n_sig >= (uint32_t)kSigQueue &&
              !wait_phase(P, &S.sig_empty[ss], ((n_sig / kSigQueue) - 1) & 1u, &s_abort, t)) {
            s_fail = 1;
          } else {
            S.sig_req[ss] = make_uint2(T.sig_off, T.sig_cnt);
            mbar_arrive(&S.sig_full[ss]);
            ++n_sig;
          }
        }
        s_cons_tiles = i + 1;
        mbar_arrive(&S.tq_empty[slot]);
      }
    }
    if (threadIdx.x == 0) {
      s_cons_chunks = cur.c;
      if (!P.per_op) {  // stop the signaller after the requests already queued
        const int ss = n_sig % kSigQueue;
        if (n_sig < (uint32_t)kSigQueue ||
            wait_phase(P, &S.sig_empty[ss], ((n_sig / kSigQueue) - 1) & 1u, &s_abort, 0xFFFFFFFFu)) {
          S.sig_req[ss] = make_uint2(0u, kSigStop);
          mbar_arrive(&S.sig_full[ss]);
        }
      }
    }
  }
  __syncthreads();
  // Drain: wait (bounded) for chunks issued but never consumed.  Every copy
  // reads a valid global range, so it lands; the bound is a guard only.  If it
  // ever runs out, the error word says so (the handle is then poisoned) before
  // the CTA leaves with that copy still counted as in flight.
  if (threadIdx.x == 0) {
    for (uint32_t c = s_cons_chunks; c < s_prod_chunks; ++c) {
      const int s = c % P.n_stages;
      const uint32_t par = (c / P.n_stages) & 1u;
      const uint64_t t0 = globaltimer();
      bool landed = true;
      while (!mbar_try_wait(&S.full[s], par))
        if (globaltimer() - t0 > P.timeout_ns) {
          landed = false;
          break;
        }
      if (!landed) {
        record_error(P, WPK_ERR_TIMEOUT, 0xFFFFFFFEu, kNoCounter, c, s_prod_chunks);
        break;
      }
    }
  }
  if (P.uses_tmem) {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(s_tmem, (uint32_t)P.tmem_cols);
  }
}

}  // namespace

// Decode on CUDA cores: the persistent worker grid (one cooperative launch per
// region per step, or one for many steps when resident).
__global__ void __launch_bounds__(kCtaThreadsGemv, 1) wpk_persistent_kernel(const KParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  worker<kProgGemv>(P, smem_raw);
}

// Per-op launch: one CTA per tile of one op group; stream order replaces the
// counters.  Used for the CUDA-Graph comparator.
__global__ void __launch_bounds__(kCtaThreadsGemv, 1) wpk_per_op_kernel(const KParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  worker<kProgGemv>(P, smem_raw);
}

// Batched decode on tensor cores: the same two launch forms.
__global__ void __launch_bounds__(kCtaThreadsTc, 1) wpk_persistent_mma_kernel(const KParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  worker<kProgMma>(P, smem_raw);
}
__global__ void __launch_bounds__(kCtaThreadsTc, 1) wpk_per_op_mma_kernel(const KParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  worker<kProgMma>(P, smem_raw);
}

// The prefill program.
__global__ void __launch_bounds__(kCtaThreadsTc, 1) wpk_prefill_kernel(const KParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  worker<kProgPrefill>(P, smem_raw);
}
__global__ void __launch_bounds__(kCtaThreadsTc, 1) wpk_prefill_op_kernel(const KParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  worker<kProgPrefill>(P, smem_raw);
}

size_t worker_smem_bytes(int n_stages, int stage_bytes, int act_bytes) {
  return (size_t)n_stages * stage_bytes + act_bytes + kOutFloats * 4 + kMaxQueue * sizeof(TQEntry) +
         (2 * kMaxStages + 2 * kMaxQueue + 1 + 2 * kSigQueue) * 8 + kSigQueue * sizeof(uint2);
}

const void* persistent_kernel_ptr(bool mma) {
  return mma ? reinterpret_cast<const void*>(&wpk_persistent_mma_kernel)
             : reinterpret_cast<const void*>(&wpk_persistent_kernel);
}
const void* per_op_kernel_ptr(bool mma) {
  return mma ? reinterpret_cast<const void*>(&wpk_per_op_mma_kernel) : reinterpret_cast<const void*>(&wpk_per_op_kernel);
}
const void* prefill_kernel_ptr() { return reinterpret_cast<const void*>(&wpk_prefill_kernel); }
int cta_threads(const void* fn) {
  return (fn == reinterpret_cast<const void*>(&wpk_persistent_kernel) ||
          fn == reinterpret_cast<const void*>(&wpk_per_op_kernel))
             ? kCtaThreadsGemv
             : kCtaThreadsTc;
}
const void* prefill_op_kernel_ptr() { return reinterpret_cast<const void*>(&wpk_prefill_op_kernel); }

}  // namespace wpk
