// Tensor-core tile core shared by the program bodies and the GEMM check:
// D[128 x N] (+)= A[128 x K] * B[N x K]^T with A and B K-major in shared
// memory (128-byte swizzle), fp32 accumulation in TMEM.
//
// Operands arrive as "images": for every 64-wide K chunk, A is one contiguous
// 16 KB block (128 rows x 128 bytes, swizzled) and B is N x 128 bytes, so each
// chunk is one bulk copy per operand (no tensor maps).  A second B image (the
// low half of a hi/lo split activation) can be accumulated with the same A.
#pragma once
#include "ptx.cuh"
#include "wpk_internal.h"

namespace wpk {

constexpr int kMmaChunkK = 64;                 // K elements per chunk (one 128-byte row)
constexpr int kMmaABytes = 128 * 128;          // A bytes per chunk


struct MmaRing {
  uint8_t* base;      // stage s at base + s * stage_bytes (1024-aligned)
  int stage_bytes;
  int stages;
  uint64_t* full;     // [stages]
  uint64_t* empty;    // [stages]
  uint64_t* done;     // accumulator ready
  uint32_t full_phase, empty_phase, done_phase;  // parity bits (uniform across threads)
};

struct MmaJob {
  const uint8_t* a;   // A image: chunk c at a + c * kMmaABytes
  const uint8_t* b;   // B image: chunk c at b + c * b_chunk_bytes
  const uint8_t* b2;  // optional second B image (same layout), or nullptr
  int b_chunk_bytes;  // N * 128
  int n_chunks;
  int N;              // multiple of 16, <= 256
  bool bf16;
};

// Thread 0 only: stream all chunks through the ring and issue the MMAs.  The
// loads for the first `stages` chunks are issued before anything waits.
// Returns false on a bounded-wait timeout.  *pend receives the stages whose
// last "empty" completion was not consumed; after R.done has been waited,
// mma_retire() flips their parities (those MMAs are then certainly done).
__device__ inline bool mma_run_issuer(MmaRing& R, const MmaJob& J, uint32_t d_tmem, uint64_t timeout_ns,
                                      uint32_t* pend_out) {
  uint32_t pend = 0;
  const uint32_t idesc = idesc_f16(128, J.N, J.bf16);
  const int nb = J.b2 ? 2 : 1;
  const uint32_t stage_tx = kMmaABytes + nb * J.b_chunk_bytes;
  auto load = [&](int c) {
    const int s = c % R.stages;
    uint8_t* st = R.base + (size_t)s * R.stage_bytes;
    mbar_arrive_expect_tx(&R.full[s], stage_tx);
    bulk_g2s(st, J.a + (size_t)c * kMmaABytes, kMmaABytes, &R.full[s]);
    bulk_g2s(st + kMmaABytes, J.b + (size_t)c * J.b_chunk_bytes, J.b_chunk_bytes, &R.full[s]);
    if (J.b2) bulk_g2s(st + kMmaABytes + J.b_chunk_bytes, J.b2 + (size_t)c * J.b_chunk_bytes, J.b_chunk_bytes,
                       &R.full[s]);
  };
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
      if (mbar_try_wait(bar, parity)) return true;
      if ((it & 31) == 0 && globaltimer() - t0 > timeout_ns) return false;
    }
  };
  const int pre = J.n_chunks < R.stages ? J.n_chunks : R.stages;
  fence_proxy_async_smem();
  for (int c = 0; c < pre; ++c) load(c);
  for (int c = 0; c < J.n_chunks; ++c) {
    const int s = c % R.stages;
    if (!wait(&R.full[s], (R.full_phase >> s) & 1u)) return false;
    R.full_phase ^= 1u << s;
    tc_fence_after();
    const uint32_t st = smem_u32(R.base + (size_t)s * R.stage_bytes);
#pragma unroll
    for (int kk = 0; kk < kMmaChunkK / 16; ++kk) {
      const uint64_t ad = sdesc_k_sw128(st + kk * 32);
      for (int p = 0; p < nb; ++p) {
        const uint64_t bd = sdesc_k_sw128(st + kMmaABytes + p * J.b_chunk_bytes + kk * 32);
        umma_f16(d_tmem, ad, bd, idesc, (c | kk | p) != 0);
      }
    }
    umma_commit(&R.empty[s]);
    pend |= 1u << s;
    // refill the stage consumed by the previous chunk once its MMAs are done
    if (c >= 1) {
      const int pc = c - 1, ps = pc % R.stages;
      if (pc + R.stages < J.n_chunks) {
        if (!wait(&R.empty[ps], (R.empty_phase >> ps) & 1u)) {
          *pend_out = pend;
          return false;
        }
        R.empty_phase ^= 1u << ps;
        pend &= ~(1u << ps);
        load(pc + R.stages);
      }
    }
  }
  umma_commit(R.done);
  *pend_out = pend;
  return true;
}

__device__ __forceinline__ void mma_retire(MmaRing& R, uint32_t pend) { R.empty_phase ^= pend; }

}  // namespace wpk
