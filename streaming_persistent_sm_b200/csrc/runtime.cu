// Persistent decode program for sm_100a: the worker loop and the tile bodies.
//
// Worker loop ("Why real-time inference wants a megakernel", "What the
// megakernel changes": wait for dependencies, run, signal consumers):
//   1. take the next ticket from the device queue (one atomic per tile; the
//      ticket after it is claimed while the current tile runs),
//   2. issue the tile's staging copy (weights, or the KV pages of an attention
//      split) into the worker's one staging slot - before waiting, so the load
//      overlaps the predecessors ("One Megakernel is Not Enough", Table I,
//      weight prefetch: one staging slot per worker, the load is queued while
//      predecessors run, compute still waits for them),
//   3. wait (acquire, bounded by %globaltimer) until the tile's counter holds
//      need x epoch,
//   4. run the body; tensors consumed inside the body (normalised activations,
//      pre-RoPE q/k, gate/up) are never stored (Table I, on-chip forwarding),
//   5. release-increment the counters of its consumers.
// Tickets are handed out in a topological order and every resident worker
// holds at most two, so the smallest unfinished ticket can always run: the
// program cannot deadlock while all workers are co-resident (cooperative
// launch guarantees that).
//
// Every wait is bounded: on timeout the worker records {code, tile, counter,
// epoch, observed, target} in the error word, waits (bounded) for its own
// copies in flight and returns; other workers see the error word and stop.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "wpk_internal.h"

namespace wpk {

namespace {

constexpr int kOutFloats = 1024;  // GEMV partial outputs [row][4]

struct Ctx {
  uint8_t* slot;
  float* act;
  float* out;
  uint64_t* bars;
};

__device__ __forceinline__ Ctx carve(uint8_t* base, int slot_bytes) {
  Ctx c;
  c.slot = base;
  c.act = reinterpret_cast<float*>(base + slot_bytes);
  c.out = c.act + kActBytes / 4;
  c.bars = reinterpret_cast<uint64_t*>(c.out + kOutFloats);
  return c;
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
  }
}

// Bounded wait for a staging barrier; every thread calls it.
__device__ bool wait_bar(const KParams& P, uint64_t* bar, uint32_t parity, uint32_t tile) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31) == 0 && globaltimer() - t0 > P.timeout_ns) {
      record_error(P, WPK_ERR_TIMEOUT, tile, kNoCounter, 0, 0);
      return false;
    }
  }
}

__device__ __forceinline__ size_t kv_index(const KParams& P, int layer, int block, int sel, int g, int row) {
  return ((((size_t)layer * P.n_blocks + block) * 2 + sel) * P.n_kv + g) * P.page_tokens * P.head_dim +
         (size_t)row * P.head_dim;
}

__device__ __forceinline__ int active_batch(const KParams& P) { return *P.active_batch; }

// ---------------------------------------------------------------------------
// Staging: which barriers a tile arms, and the copies (thread 0 only).
// ---------------------------------------------------------------------------
struct AttnSpan {
  int b, g, j, pos, t0, t1;  // tokens [t0, t1) of sequence b, current position pos
};

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

__device__ __forceinline__ int gemv_rows_per_chunk(const KParams& P, int K) {
  int r = P.chunk_bytes / (K * 2);
  return r < 1 ? 1 : r;
}

// Mask of chunk barriers this tile uses (identical on every thread).
__device__ __forceinline__ uint32_t staging_mask(const KParams& P, const Tile& T) {
  if (T.op == OP_ATTN) {
    if (T.a0 >= active_batch(P)) return 0;
    AttnSpan s = attn_span(P, T);
    return s.t1 > s.t0 ? 1u : 0u;
  }
  if (T.w_bytes == 0) return 0;
  const int rpc = gemv_rows_per_chunk(P, T.a3);
  const int n = (T.a1 + rpc - 1) / rpc;
  return (n >= 32) ? 0xFFFFFFFFu : ((1u << n) - 1u);
}

__device__ void issue_staging(const KParams& P, const Tile& T, const Ctx& c) {
  if (T.op == OP_ATTN) {
    if (T.a0 >= active_batch(P)) return;
    AttnSpan s = attn_span(P, T);
    if (s.t1 <= s.t0) return;
    const int page = P.page_tokens, hd = P.head_dim;
    const int p0 = s.t0 / page, p1 = (s.t1 - 1) / page;
    uint32_t total = 0;
    for (int p = p0; p <= p1; ++p) total += 2u * (uint32_t)(min(page, s.t1 - p * page)) * hd * 2;
    mbar_arrive_expect_tx(&c.bars[0], total);
    const uint32_t vbase = (uint32_t)P.split_tokens * hd * 2;
    for (int p = p0; p <= p1; ++p) {
      const int rows = min(page, s.t1 - p * page);
      const int blk = P.block_table[s.b * P.max_blocks + p];
      const uint32_t bytes = (uint32_t)rows * hd * 2;
      const uint32_t dst = (uint32_t)(p - p0) * page * hd * 2;
      bulk_g2s(c.slot + dst, P.kv + kv_index(P, T.layer, blk, 0, s.g, 0), bytes, &c.bars[0]);
      bulk_g2s(c.slot + vbase + dst, P.kv + kv_index(P, T.layer, blk, 1, s.g, 0), bytes, &c.bars[0]);
    }
    return;
  }
  if (T.w_bytes == 0) return;
  const int row_bytes = T.a3 * 2;
  const int rpc = gemv_rows_per_chunk(P, T.a3);
  const uint8_t* src = P.weights + T.w_off;
  for (int r0 = 0, ci = 0; r0 < T.a1; r0 += rpc, ++ci) {
    const uint32_t bytes = (uint32_t)min(rpc, T.a1 - r0) * row_bytes;
    mbar_arrive_expect_tx(&c.bars[ci], bytes);
    bulk_g2s(c.slot + (size_t)r0 * row_bytes, src + (size_t)r0 * row_bytes, bytes, &c.bars[ci]);
  }
}

// ---------------------------------------------------------------------------
// GEMV bodies (CUDA cores).  Weights: the tile's rows, row-major, in the slot.
// Activations: fp32 [bg][K] staged in shared memory (RMSNorm fused when the
// op consumes a normalised residual).  Work item = (row, 256-column segment);
// lanes read 16 contiguous bytes each, so a warp reads 512 contiguous bytes.
// ---------------------------------------------------------------------------
template <int BG>
__device__ __forceinline__ void gemv_items(const uint8_t* slot, int K, int row_lo, int row_hi, const float* act,
                                           float* out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int segs = (K + 255) >> 8;
  const int n_items = (row_hi - row_lo) * segs;
  const size_t row_bytes = (size_t)K * 2;
  for (int it = warp; it < n_items; it += kWarps) {
    const int row = row_lo + it / segs;
    const int k = (it % segs) * 256 + lane * 8;
    float acc[BG];
#pragma unroll
    for (int b = 0; b < BG; ++b) acc[b] = 0.f;
    if (k < K) {
      const uint4 w = *reinterpret_cast<const uint4*>(slot + row * row_bytes + (size_t)k * 2);
      float wf[8];
      unpack8(w, wf);
#pragma unroll
      for (int b = 0; b < BG; ++b) {
        const float4 a0 = *reinterpret_cast<const float4*>(act + b * K + k);
        const float4 a1 = *reinterpret_cast<const float4*>(act + b * K + k + 4);
        float s = wf[0] * a0.x;
        s = fmaf(wf[1], a0.y, s);
        s = fmaf(wf[2], a0.z, s);
        s = fmaf(wf[3], a0.w, s);
        s = fmaf(wf[4], a1.x, s);
        s = fmaf(wf[5], a1.y, s);
        s = fmaf(wf[6], a1.z, s);
        s = fmaf(wf[7], a1.w, s);
        acc[b] = s;
      }
    }
#pragma unroll
    for (int b = 0; b < BG; ++b) acc[b] = warp_sum(acc[b]);
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < BG; ++b) atomicAdd(&out[row * 4 + b], acc[b]);
    }
  }
}

// Copy bg rows of K floats (stride `stride`) into act; optionally RMS-normalise
// each row and multiply by `gain` (which must cover the whole row: K = hidden).
__device__ void stage_act(const float* src, int stride, int K, int bg, const float* gain, float eps, float* act) {
  __shared__ float red[kWarps][4];
  float ss[4] = {0.f, 0.f, 0.f, 0.f};
  for (int b = 0; b < bg; ++b) {
    for (int k = threadIdx.x * 4; k < K; k += kThreads * 4) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(src + (size_t)b * stride + k));
      *reinterpret_cast<float4*>(act + b * K + k) = v;
      ss[b] += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
  }
  if (gain) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int b = 0; b < bg; ++b) {
      float v = warp_sum(ss[b]);
      if (lane == 0) red[warp][b] = v;
    }
    __syncthreads();
    float scale[4];
    for (int b = 0; b < bg; ++b) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) tot += red[w][b];
      scale[b] = 1.0f / sqrtf(tot / (float)K + eps);
    }
    for (int b = 0; b < bg; ++b)
      for (int k = threadIdx.x * 4; k < K; k += kThreads * 4) {
        float4* a = reinterpret_cast<float4*>(act + b * K + k);
        const float4 gg = __ldg(reinterpret_cast<const float4*>(gain + k));
        float4 v = *a;
        v.x *= scale[b] * gg.x;
        v.y *= scale[b] * gg.y;
        v.z *= scale[b] * gg.z;
        v.w *= scale[b] * gg.w;
        *a = v;
      }
  }
  __syncthreads();
}

__device__ void epilogue(const KParams& P, const Tile& T, const float* out, int b0, int bg) {
  const int r0 = T.a0, R = T.a1, hd = P.head_dim, half = hd / 2;
  switch (T.op) {
    case OP_QKV: {
      for (int idx = threadIdx.x; idx < (R / 2) * bg; idx += kThreads) {
        const int pr = idx % (R / 2), b = idx / (R / 2), bi = b0 + b;
        const int r = r0 + 2 * pr;
        const float y0 = out[(2 * pr) * 4 + b], y1 = out[(2 * pr + 1) * 4 + b];
        const int pos = P.seqlen[bi];
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
          } else {
            const int blk = P.block_table[bi * P.max_blocks + pos / P.page_tokens];
            uint16_t* k = P.kv + kv_index(P, T.layer, blk, 0, head, pos % P.page_tokens);
            k[i] = f2bf(o0);
            k[i + half] = f2bf(o1);
          }
        } else {
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
        const float x = __ldcg(P.xa + o) + out[rr * 4 + b];
        P.xb[o] = x;
        P.xa[o] = x;
      }
      break;
    }
    case OP_GU: {
      for (int idx = threadIdx.x; idx < (R / 2) * bg; idx += kThreads) {
        const int pr = idx % (R / 2), b = idx / (R / 2), bi = b0 + b;
        const float g = out[(2 * pr) * 4 + b], u = out[(2 * pr + 1) * 4 + b];
        P.hbuf[(size_t)bi * P.ffn + r0 / 2 + pr] = g / (1.0f + expf(-g)) * u;
      }
      break;
    }
    case OP_DOWN: {
      for (int idx = threadIdx.x; idx < R * bg; idx += kThreads) {
        const int rr = idx % R, b = idx / R, bi = b0 + b;
        atomicAdd(P.xa + (size_t)bi * P.hidden + r0 + rr, out[rr * 4 + b]);
      }
      break;
    }
    case OP_LMHEAD: {
      if (P.logits)
        for (int idx = threadIdx.x; idx < R * bg; idx += kThreads) {
          const int rr = idx % R, b = idx / R, bi = b0 + b;
          P.logits[(size_t)bi * P.vocab + r0 + rr] = out[rr * 4 + b];
        }
      const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
      if (warp < bg) {
        float bv = -INFINITY;
        int bidx = 0x7FFFFFFF;
        for (int rr = lane; rr < R; rr += 32) {
          const float v = out[rr * 4 + warp];
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

template <int BG>
__device__ void gemv_group(const KParams& P, const Tile& T, const Ctx& c, int b0, bool first, uint32_t phase,
                           bool* ok) {
  const int K = T.a3, R = T.a1;
  const int rpc = gemv_rows_per_chunk(P, K);
  for (int i = threadIdx.x; i < R * 4; i += kThreads) c.out[i] = 0.f;
  __syncthreads();
  for (int r0 = 0, ci = 0; r0 < R; r0 += rpc, ++ci) {
    if (first && !wait_bar(P, &c.bars[ci], (phase >> ci) & 1u, T.a0)) *ok = false;
    if (!__syncthreads_and(*ok)) {
      *ok = false;
      return;
    }
    gemv_items<BG>(c.slot, K, r0, min(R, r0 + rpc), c.act, c.out);
  }
  __syncthreads();
}

__device__ bool body_gemv(const KParams& P, const Tile& T, const Ctx& c, uint32_t phase) {
  const int K = T.a3;
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
  int bgmax = kActBytes / (K * 4);
  if (bgmax > 4) bgmax = 4;
  bool ok = true;
  for (int b0 = 0; b0 < nb; b0 += bgmax) {
    const int bg = min(bgmax, nb - b0);
    stage_act(src + (size_t)b0 * stride, stride, K, bg, gain, P.eps, c.act);
    const bool first = (b0 == 0);
    switch (bg) {
      case 1: gemv_group<1>(P, T, c, b0, first, phase, &ok); break;
      case 2: gemv_group<2>(P, T, c, b0, first, phase, &ok); break;
      case 3: gemv_group<3>(P, T, c, b0, first, phase, &ok); break;
      default: gemv_group<4>(P, T, c, b0, first, phase, &ok); break;
    }
    if (!ok) return false;
    epilogue(P, T, c.out, b0, bg);
    __syncthreads();
  }
  if (nb == 0) {  // nothing to compute, but the staged chunks must still land
    const int rpc = gemv_rows_per_chunk(P, K);
    for (int r0 = 0, ci = 0; r0 < T.a1; r0 += rpc, ++ci)
      if (!wait_bar(P, &c.bars[ci], (phase >> ci) & 1u, T.a0)) ok = false;
    ok = __syncthreads_and(ok);
  }
  return ok;
}

// ---------------------------------------------------------------------------
// Split-KV GQA decode attention.  The tile (b, g, j) handles the `group` query
// heads of kv head g over tokens [j*S, (j+1)*S) of sequence b, writes an
// online-softmax partial (m, l, o), and the last split to arrive combines all
// partials of (b, g) ("Persistent threads and megakernels", §6: split long
// histories into chunks, then combine partial attention with a reduction
// signalled through global memory).
// ---------------------------------------------------------------------------
__device__ bool body_attn(const KParams& P, const Tile& T, const Ctx& c, uint32_t phase) {
  if (T.a0 >= active_batch(P)) return true;
  __shared__ int s_last;
  __shared__ float s_m[kMaxGroup], s_l[kMaxGroup];
  const AttnSpan s = attn_span(P, T);
  const int hd = P.head_dim, grp = P.group, S = P.split_tokens;
  const int n = s.t1 - s.t0;
  float* part = P.part + ((((size_t)s.b * P.n_kv + s.g) * P.n_splits + s.j) * grp) * (2 + hd);
  const uint16_t* Ks = reinterpret_cast<const uint16_t*>(c.slot);
  const uint16_t* Vs = reinterpret_cast<const uint16_t*>(c.slot + (size_t)S * hd * 2);
  float* q_s = c.act;                 // [grp][hd]
  float* p_s = c.act + kMaxGroup * hd;  // [grp][S]
  if (n > 0) {
    bool ok = wait_bar(P, &c.bars[0], phase & 1u, 0xFFFFFFFFu);
    if (!__syncthreads_and(ok)) return false;
    // the current token's row was written this step, after the copy was issued
    if (s.pos >= s.t0 && s.pos < s.t1) {
      const int blk = P.block_table[s.b * P.max_blocks + s.pos / P.page_tokens];
      const int row = s.pos - s.t0;
      const int lanes = hd * 2 / 16;  // 16-byte pieces per row
      if (threadIdx.x < 2 * lanes) {
        const int sel = threadIdx.x / lanes, piece = threadIdx.x % lanes;
        const uint4* src = reinterpret_cast<const uint4*>(
            P.kv + kv_index(P, T.layer, blk, sel, s.g, s.pos % P.page_tokens));
        uint8_t* dst = c.slot + (size_t)sel * S * hd * 2 + (size_t)row * hd * 2;
        reinterpret_cast<uint4*>(dst)[piece] = __ldcg(src + piece);
      }
    }
    for (int i = threadIdx.x; i < grp * hd; i += kThreads)
      q_s[i] = __ldcg(P.qbuf + (size_t)s.b * P.q_rows + (size_t)s.g * grp * hd + i);
    __syncthreads();
    const float scale = 1.0f / sqrtf((float)hd);
    const int words = hd / 2;
    for (int idx = threadIdx.x; idx < grp * n; idx += kThreads) {
      const int hh = idx / n, t = idx % n;
      const uint32_t* kr = reinterpret_cast<const uint32_t*>(Ks + (size_t)t * hd);
      const float* qr = q_s + hh * hd;
      float acc = 0.f;
      for (int w = 0; w < words; ++w) {
        const int ww = (w + t) & (words - 1);
        const uint32_t kk = kr[ww];
        acc = fmaf(qr[2 * ww], __uint_as_float(kk << 16), acc);
        acc = fmaf(qr[2 * ww + 1], __uint_as_float(kk & 0xFFFF0000u), acc);
      }
      p_s[hh * S + t] = acc * scale;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < grp) {
      float m = -INFINITY;
      for (int t = lane; t < n; t += 32) m = fmaxf(m, p_s[warp * S + t]);
      m = warp_max(m);
      float l = 0.f;
      for (int t = lane; t < n; t += 32) {
        const float e = expf(p_s[warp * S + t] - m);
        p_s[warp * S + t] = e;
        l += e;
      }
      l = warp_sum(l);
      if (lane == 0) { s_m[warp] = m; s_l[warp] = l; }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < grp * hd; idx += kThreads) {
      const int hh = idx / hd, d = idx % hd;
      float o = 0.f;
      for (int t = 0; t < n; ++t) o = fmaf(p_s[hh * S + t], bf2f(Vs[(size_t)t * hd + d]), o);
      float* pr = part + (size_t)hh * (2 + hd);
      pr[2 + d] = o;
      if (d == 0) { pr[0] = s_m[hh]; pr[1] = s_l[hh]; }
    }
  } else {
    for (int idx = threadIdx.x; idx < grp * (2 + hd); idx += kThreads) {
      const int k = idx % (2 + hd);
      part[idx] = (k == 0) ? -INFINITY : 0.f;
    }
  }
  __syncthreads();
  uint32_t* arr = P.arrive + (size_t)s.b * P.n_kv + s.g;
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(arr, 1u);
    s_last = (old == (uint32_t)P.n_splits - 1u);
    __threadfence();
  }
  __syncthreads();
  if (s_last) {
    const float* base = P.part + (((size_t)s.b * P.n_kv + s.g) * P.n_splits) * grp * (2 + hd);
    for (int idx = threadIdx.x; idx < grp * hd; idx += kThreads) {
      const int hh = idx / hd, d = idx % hd;
      float M = -INFINITY;
      for (int j = 0; j < P.n_splits; ++j) M = fmaxf(M, __ldcg(base + ((size_t)j * grp + hh) * (2 + hd)));
      float L = 0.f, O = 0.f;
      for (int j = 0; j < P.n_splits; ++j) {
        const float* pr = base + ((size_t)j * grp + hh) * (2 + hd);
        const float w = expf(__ldcg(pr) - M);
        L = fmaf(__ldcg(pr + 1), w, L);
        O = fmaf(__ldcg(pr + 2 + d), w, O);
      }
      P.attn[(size_t)s.b * P.q_rows + ((size_t)s.g * grp + hh) * hd + d] = O / L;
    }
    if (threadIdx.x == 0) *arr = 0u;
  }
  return true;
}

__device__ bool body_embed(const KParams& P, const Tile& T) {
  const int nb = active_batch(P);
  const uint16_t* E = reinterpret_cast<const uint16_t*>(P.weights + P.embed_off);
  for (int b = 0; b < nb; ++b) {
    int tok = P.in_tok ? P.in_tok[(size_t)b * P.in_tok_stride] : P.tok_fb[b];
    if (tok < 0 || tok >= P.vocab) {
      if (threadIdx.x == 0) record_error(P, WPK_ERR_INVALID_ARG, 0, kNoCounter, (uint32_t)tok, (uint32_t)P.vocab);
      tok = 0;
    }
    const uint4* row = reinterpret_cast<const uint4*>(E + (size_t)tok * P.hidden);
    float* x = P.xa + (size_t)b * P.hidden;
    for (int k = threadIdx.x; k < P.hidden / 8; k += kThreads) {
      float f[8];
      unpack8(__ldg(row + k), f);
      reinterpret_cast<float4*>(x)[2 * k] = make_float4(f[0], f[1], f[2], f[3]);
      reinterpret_cast<float4*>(x)[2 * k + 1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
  return true;
}

__device__ bool body_final(const KParams& P) {
  const int nb = active_batch(P);
  for (int b = threadIdx.x; b < nb; b += kThreads) {
    const unsigned long long key = P.best[b];
    const int32_t idx = (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
    if (P.out_tok) P.out_tok[b] = idx;
    P.tok_fb[b] = idx;
    P.best[b] = 0ull;
    P.seqlen[b] += 1;
  }
  return true;
}

__device__ __forceinline__ bool run_body(const KParams& P, const Tile& T, const Ctx& c, uint32_t phase) {
  switch (T.op) {
    case OP_EMBED: return body_embed(P, T);
    case OP_ATTN: return body_attn(P, T, c, phase);
    case OP_FINAL: return body_final(P);
    default: return body_gemv(P, T, c, phase);
  }
}

__device__ void drain(const KParams& P, const Ctx& c, uint32_t used, uint32_t phase) {
  if (threadIdx.x != 0) return;
  for (int i = 0; i < kMaxChunks; ++i)
    if ((used >> i) & 1u) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&c.bars[i], (phase >> i) & 1u))
        if (globaltimer() - t0 > P.timeout_ns) break;
    }
}

// Thread 0: bounded acquire-wait until the tile's counter reaches need x epoch.
__device__ bool wait_counter(const KParams& P, const Tile& T, uint32_t tile) {
  if (ld_volatile_s32(&P.err->code) != 0) return false;
  if (T.wait_ctr == kNoCounter) return true;
  const uint32_t target = T.need * P.epoch;
  const uint32_t* ctr = P.ctr + T.wait_ctr;
  uint32_t v = ld_acquire_u32(ctr);
  if ((int32_t)(v - target) >= 0) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    v = ld_acquire_u32(ctr);
    if ((int32_t)(v - target) >= 0) return true;
    if ((it & 15) == 0) {
      if (ld_volatile_s32(&P.err->code) != 0) return false;
      if (globaltimer() - t0 > P.timeout_ns) {
        record_error(P, WPK_ERR_TIMEOUT, tile, T.wait_ctr, v, target);
        return false;
      }
    }
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// The persistent worker grid (one launch per region per step).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 2) wpk_persistent_kernel(const KParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const Ctx c = carve(smem_raw, P.slot_bytes);
  __shared__ uint32_t s_tk[2];
  __shared__ int s_fail;
  __shared__ uint32_t s_ev_issue;
  __shared__ uint64_t s_t_start;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxChunks; ++i) mbar_init(&c.bars[i], 1);
    fence_mbar_init();
    s_tk[0] = P.t_begin + atomicAdd(&P.head[P.region], 1u);
  }
  __syncthreads();
  uint32_t phase = 0;
  for (;;) {
    const uint32_t t = s_tk[0];
    if (t >= P.t_end) break;
    const Tile T = P.tiles[t];
    const uint32_t used = staging_mask(P, T);
    if (threadIdx.x == 0) {
      fence_proxy_async_smem();
      issue_staging(P, T, c);
      if (P.trace) s_ev_issue = atomicAdd(P.evclock, 1u);
      s_tk[1] = P.t_begin + atomicAdd(&P.head[P.region], 1u);  // claim the next ticket early
      s_fail = wait_counter(P, T, t) ? 0 : 1;
      if (P.trace) s_t_start = globaltimer();
    }
    __syncthreads();
    uint32_t ev_start = 0;
    if (P.trace && threadIdx.x == 0 && !s_fail) ev_start = atomicAdd(P.evclock, 1u);
    bool ok = !s_fail;
    if (ok) ok = run_body(P, T, c, phase);
    ok = __syncthreads_and(ok);
    if (!ok) {
      drain(P, c, used, phase);
      break;
    }
    phase ^= used;
    if (threadIdx.x == 0) {
      if (P.trace) {
        TraceRec r;
        r.tile = t;
        r.worker = (uint16_t)blockIdx.x;
        r.op = T.op;
        r.ev_issue = s_ev_issue;
        r.ev_start = ev_start;
        r.ev_done = atomicAdd(P.evclock, 1u);
        r.epoch = P.epoch;
        r.t_start_ns = s_t_start;
        r.t_end_ns = globaltimer();
        P.trace_buf[t] = r;
      }
      __threadfence();
      for (uint32_t i = 0; i < T.sig_cnt; ++i) red_release_add_u32(P.ctr + P.sig[T.sig_off + i], 1u);
      s_tk[0] = s_tk[1];
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Per-op launch: one CTA per tile of one op group; stream order replaces the
// counters.  Used for the CUDA-Graph comparator.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 2) wpk_per_op_kernel(const KParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const Ctx c = carve(smem_raw, P.slot_bytes);
  const uint32_t t = P.t_begin + blockIdx.x;
  if (t >= P.t_end) return;
  const Tile T = P.tiles[t];
  const uint32_t used = staging_mask(P, T);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxChunks; ++i) mbar_init(&c.bars[i], 1);
    fence_mbar_init();
    issue_staging(P, T, c);
  }
  __syncthreads();
  bool ok = ld_volatile_s32(&P.err->code) == 0;
  ok = __syncthreads_and(ok);
  if (ok) ok = run_body(P, T, c, 0u);
  ok = __syncthreads_and(ok);
  if (!ok) drain(P, c, used, 0u);
}

size_t worker_smem_bytes(int slot_bytes) {
  return (size_t)slot_bytes + kActBytes + kOutFloats * 4 + kMaxChunks * 8;
}

const void* persistent_kernel_ptr() { return reinterpret_cast<const void*>(&wpk_persistent_kernel); }
const void* per_op_kernel_ptr() { return reinterpret_cast<const void*>(&wpk_per_op_kernel); }

}  // namespace wpk
