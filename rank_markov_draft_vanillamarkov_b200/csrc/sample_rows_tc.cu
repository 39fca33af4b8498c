// Left-to-right block sampling on the sm_100a tensor cores, batch rows on the
// MMA's M side (VanillaMarkov.sample_block_tokens and _sample_tokens of the
// vendored markov_head.py). For k = 0 .. M-1 and every block b:
//
//     c_k[b, v] = round_bf16( U[b, k, v] + sum_j W1[x_{k-1}[b], j] * W2[v, j] )
//     x_k[b]    = argmax_v c_k[b, v]                    (greedy)
//              or argmax_v c_k[b, v] / T + g(b, k, v)   (Gumbel-max, Philox noise)
//
// with x_{-1} = first_prev, in one cooperative persistent launch for all M
// steps. CTA c owns a contiguous range of vocabulary ids (whole 64-id spans,
// so that no TMA box of logits crosses into a neighbour's range), cut into
// chunks of up to 256 ids.
//
// Why this layout. A tcgen05.mma's time grows far more slowly than its N (on
// this part about 130 cycles at N = 32, the batch, and about 230 at N = 256),
// so the ids go on N, 256 at a time, and the batch on M:
// D[lane][id] = X[lane] . W2[id]^T with A = X = W1[x_{k-1}] rows in shared
// memory and B = a W2 chunk. M is 128, so the batch (padded to BP = 32 or 64
// rows) is repeated REP = 128 / BP times down the lanes; each repeat serves a
// different part of the chunk's columns, so that all four TMEM lane quarters
// (one per epilogue warp quarter) carry useful rows.
//
// Why the epilogue warps keep off global memory. A tcgen05.wait::ld, and a
// proxy fence, also wait for the thread's global accesses still in flight:
// a few dozen cycles alone, a thousand and more behind outstanding loads or
// behind reductions that 148 CTAs aim at the same keys. So the epilogue
// threads issue no global stores or reductions and no loads that are still
// in flight at a tensor-memory load: a loader warp brings each chunk's U into
// shared memory (boxes of 64 ids x B rows, 128-byte swizzle) through a ring
// of stages, the epilogue adds the bias and rounds in place, and the same
// warp stores the stage back to the corrected-logit tensor; the per-row
// maxima leave through shared memory and warp 3 merges them into the global
// keys. U does not depend on the chain, so its loads run ahead of the MMAs
// (and L2 prefetches one step ahead of them). The one global read the
// epilogue makes is X's rows at the start of a step, and those loads have
// landed (their values are stored to shared memory) before any tensor-memory
// load.
//
// W2 stays on chip: the CTA's chunks are loaded into shared memory once; when
// they do not all fit, the rest stream from L2 through a two-slot ring every
// step, ordered so that their loads hide behind the resident chunks' MMAs and
// the grid barrier.
//
// Per step: warp 3 waits at the grid barrier (bounded) and decodes x_{k-1}
// from the global keys; the epilogue warps gather X (each distinct 16-byte
// piece of the rows W1[x_{k-1}] loaded once per CTA and stored into every
// repeat of its row in the swizzled operand layout); the MMA
// warp runs the chunks into two alternating 256-column accumulators, one
// chunk ahead of the epilogue; the epilogue rounds and selects and leaves its
// per-row maxima in shared memory; warp 3 merges them into the global keys
// (one red.max per row) and arrives at the barrier with one release-add.
//
// Warp roles (640 threads): 0 W2 loader and ring producer; 1 TMEM owner and
// MMA issuer; 2 U loader and corrected-logit storer; 3 key merge, grid
// barrier, key decode and U prefetch; 4-19 X gather and epilogue (warp
// 4 + 4e + q reads TMEM lane quarter q).
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace dspark {
namespace {

constexpr int kChunk = 256;                      // ids per chunk (MMA N at most)
constexpr int kSpan = 64;                        // ids per logit box; CTA ranges are whole spans
constexpr int kBoxesPerChunk = kChunk / kSpan;
constexpr int kGroup = 16;                       // ids per epilogue piece (one tcgen05.ld x16)
constexpr int kMaxStages = 3;                    // logit stages in shared memory
constexpr int kMaxRowsBatch = 64;                // batch rows the stages hold
constexpr int kEpiWarps = 16;
constexpr int kEpiPerQuarter = kEpiWarps / 4;    // E
constexpr int kThreads = 128 + kEpiWarps * 32;
constexpr uint32_t kTmemCols = 512;              // two 256-column accumulators
constexpr uint32_t kXAtomBytes = 128 * 128;      // 128 rows x 64 bf16
constexpr uint32_t kFullBlockBytes = kChunk * 128;  // 256 ids x 64 bf16
constexpr int kMaxChunks = 8;
constexpr size_t kSmemLimit = 232448;

struct __align__(64) RowsMaps {
  CUtensorMap w2;     // [vocab, rank] bf16, box 64 x 256, 128B swizzle
  CUtensorMap w2_16;  // same tensor, box 64 x 16 (the last, partial chunk)
  CUtensorMap u;      // base logits [B, M, V] as (v, k, b), box 64 x 1 x B, 128B swizzle
  CUtensorMap out;    // corrected logits, the same layout
};

struct RowsParams {
  const __nv_bfloat16* base;  // [B, M, V] (L2 prefetch)
  const int64_t* first_prev;
  const __nv_bfloat16* w1;    // [V, r]
  int64_t* tokens;
  unsigned long long* keys;   // [M, B] step maxima
  uint32_t* barrier;
  uint32_t* status;
  int64_t vocab;
  int32_t batch, bp, steps, ka;
  int32_t spans;         // 64-id spans of the vocabulary
  int32_t resident_full; // full chunks a CTA keeps in shared memory (the rest stream)
  uint32_t w2_bytes;     // shared memory reserved for resident W2 blocks
  int32_t ring;          // 1 when the streaming ring exists
  int32_t stages;        // logit stages (2 or 3)
  float temperature;
  PhiloxRoundKeys round_keys;
  uint64_t wait_limit_ns;
  uint32_t debug_flags;
};

struct RowsTail {
  uint64_t w2_full;
  uint64_t ring_full[2], ring_empty[2];
  uint64_t xid_ready, x_full, merge_ready;
  uint64_t u_full[kMaxStages], tile_ready[kMaxStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  int32_t xid[128];
  uint32_t tmem_base;
  int abort_flag;
};

// The CTA's vocabulary range and its chunks: ids [v0, v1), chunk j starts at
// v0 + 256 j; all chunks but the last are full.
struct Range {
  int64_t v0, v1;
  int nchunks, nfull;
  __device__ int width(int j) const {
    const int64_t w = ((v1 - v0 + 15) & ~15ll) - (int64_t)kChunk * j;
    return w < kChunk ? (int)w : kChunk;  // MMA N: a multiple of 16
  }
  __device__ int boxes(int j) const { return (width(j) + kSpan - 1) / kSpan; }
};

// CTA c owns spans [S c / G, S (c + 1) / G); only the last range can end
// inside a span (at the vocabulary's end), where the boxes' extra ids fall
// outside the tensor: zeros on load, dropped on store.
__device__ __forceinline__ Range cta_range(const RowsParams& p) {
  Range r;
  const int64_t s0 = (int64_t)p.spans * blockIdx.x / gridDim.x;
  const int64_t s1 = (int64_t)p.spans * (blockIdx.x + 1) / gridDim.x;
  r.v0 = s0 * kSpan;
  r.v1 = s1 * kSpan < p.vocab ? s1 * kSpan : p.vocab;
  // Chunks are counted on the length rounded up to 16 ids (the last range
  // can end 8 ids short of a group; those W2 rows read as zero).
  const int64_t n16 = (r.v1 - r.v0 + 15) & ~15ll;
  r.nchunks = (int)((n16 + kChunk - 1) / kChunk);
  r.nfull = (int)(n16 / kChunk);
  return r;
}

// Per-step chunk order: the first streamed chunk (its blocks were prefetched
// into the ring during the previous step), then the resident chunks (the
// remaining streamed blocks load behind their MMAs), then the other streamed
// chunks. Chunks [0, res) are resident, [res, nfull) stream, and a partial
// last chunk is always resident.
__device__ __forceinline__ int resident_full_of(const Range& r, const RowsParams& p) {
  return r.nfull < p.resident_full ? r.nfull : p.resident_full;
}

// The chunk at position i of the step's order (i < r.nchunks).
__device__ __forceinline__ int chunk_at(int i, const Range& r, int res) {
  if (res < r.nfull) {  // streaming: the first streamed chunk leads
    if (i == 0) return res;
    i -= 1;
  }
  if (i < res) return i;
  i -= res;
  if (r.nchunks > r.nfull) {  // the partial chunk
    if (i == 0) return r.nfull;
    i -= 1;
  }
  return res + 1 + i;
}

// Shared-memory offset of resident block (chunk j, atom a) inside the W2 area:
// full chunks first (ka atoms of 32 KB each), then the partial chunk.
__device__ __forceinline__ uint32_t resident_offset(int j, int a, const Range& r, int res, int ka) {
  if (j < r.nfull) return (uint32_t)(j * ka + a) * kFullBlockBytes;
  const uint32_t pw = (uint32_t)r.width(j);
  return (uint32_t)res * ka * kFullBlockBytes + (uint32_t)a * pw * 128u;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_max_gpu(unsigned long long* p, unsigned long long v) {
  asm volatile("red.relaxed.gpu.global.max.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void red_add_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_gpu(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// A warp-uniform bounded wait: lane 0 waits, the warp follows its verdict, and
// the other lanes then observe the (already completed) phase themselves.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, int lane) {
  bool ok = lane == 0 ? mbar_wait(bar, parity, ctl) : true;
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok && lane != 0) mbar_wait(bar, parity, ctl);
  return ok;
}

__device__ __forceinline__ bool grid_wait(const uint32_t* counter, uint32_t target, const WaitCtl& ctl, int lane) {
  bool ok = true;
  if (lane == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(counter) < target) {
      if (*ctl.abort_flag) {
        ok = false;
        break;
      }
      if (globaltimer_ns() - t0 > ctl.limit_ns) {
        *ctl.abort_flag = 1;
        atomicOr(ctl.status, DSPARK_STATUS_TIMEOUT);
        ok = false;
        break;
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  return ok;
}

// Order-preserving bits of a bf16 value held in the high half of `w` (the low
// half is ignored): the sign bit set for non-negative values, every bit
// flipped for negative ones; the low 16 bits of the result are zero.
__device__ __forceinline__ uint32_t ordered_hi16(uint32_t w) {
  return (w ^ ((uint32_t)((int32_t)w >> 31) | 0x80000000u)) & 0xFFFF0000u;
}

// Order-preserving bits of an fp32 score (see the tile sampler): +0 first
// turns -0 into +0 and any NaN into the canonical positive NaN.
__device__ __forceinline__ uint32_t ordered_bits(float x) {
  const uint32_t b = __float_as_uint(x + 0.0f);
  return b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
}

// Corrected logits of two ids as one bf16x2 word: U (two bf16 in `u2`) plus
// the fp32 bias, rounded once. Adding +0 makes a -0 sum +0 and keeps NaN the
// canonical positive NaN, so the selection keys need no further care.
__device__ __forceinline__ uint32_t add_round2(uint32_t u2, uint32_t a_lo, uint32_t a_hi) {
  const float lo = __uint_as_float(u2 << 16) + __uint_as_float(a_lo) + 0.0f;
  const float hi = __uint_as_float(u2 & 0xFFFF0000u) + __uint_as_float(a_hi) + 0.0f;
  __nv_bfloat162 o = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&o);
}

template <int KA, bool GREEDY>
__global__ void __launch_bounds__(kThreads, 1)
    tc_sample_rows_kernel(const __grid_constant__ RowsMaps maps, const RowsParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t box_bytes = (uint32_t)p.bp * 128u;               // one box: BP rows of 64 ids
  const uint32_t stage_bytes = kBoxesPerChunk * box_bytes;        // one chunk of logits
  uint8_t* w2_smem = smem;                                        // resident W2 blocks
  uint8_t* ring_smem = w2_smem + p.w2_bytes;                      // 2 x 32 KB when streaming
  uint8_t* x_smem = ring_smem + (p.ring ? 2 * kFullBlockBytes : 0u);  // KA atoms of 16 KB
  uint8_t* u_smem = x_smem + KA * kXAtomBytes;                    // p.stages logit stages
  unsigned long long* red = reinterpret_cast<unsigned long long*>(u_smem + (uint32_t)p.stages * stage_bytes);
  RowsTail* sh = reinterpret_cast<RowsTail*>(red + 128);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int M = p.steps;
  const int B = p.batch;
  const int BP = p.bp;
  const int NS = p.stages;
  const Range rg = cta_range(p);
  const int res = resident_full_of(rg, p);
  const int nc = rg.nchunks;
  const bool has_partial = rg.nchunks > rg.nfull;

  if (threadIdx.x == 0) {
    mbar_init(&sh->w2_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh->ring_full[i], 1);
      mbar_init(&sh->ring_empty[i], 1);
      mbar_init(&sh->acc_full[i], 1);
      mbar_init(&sh->acc_empty[i], kEpiWarps);
    }
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(&sh->u_full[i], 1);                // the chunk's logits have landed
      mbar_init(&sh->tile_ready[i], kEpiWarps);    // the epilogue has rewritten the stage
    }
    mbar_init(&sh->xid_ready, 1);                  // the step's previous tokens are in xid
    mbar_init(&sh->x_full, kEpiWarps);             // the epilogue warps have gathered X
    mbar_init(&sh->merge_ready, kEpiWarps);        // the step's maxima are in red[]
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < 128; i += blockDim.x) red[i] = 0ull;
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = sh->tmem_base;
  const WaitCtl ctl{&sh->abort_flag, p.status, p.wait_limit_ns};
  volatile int never = 0;
  const WaitCtl drain_ctl{&never, p.status, p.wait_limit_ns};

  if (warp == 0) {
    // ------------------------- resident W2, then the streaming ring ----
    if (lane == 0) {
      prefetch_tensormap(&maps.w2);
      prefetch_tensormap(&maps.w2_16);
      const uint64_t pol = policy_evict_last();
      const uint32_t pw = has_partial ? (uint32_t)rg.width(rg.nfull) : 0u;
      const uint32_t bytes = (uint32_t)res * KA * kFullBlockBytes + (uint32_t)KA * pw * 128u;
      if (bytes) {
        mbar_arrive_expect_tx(&sh->w2_full, bytes);
        for (int j = 0; j < res; ++j)
          for (int a = 0; a < KA; ++a)
            tma_load_2d(w2_smem + resident_offset(j, a, rg, res, KA), &maps.w2, &sh->w2_full, a * 64,
                        (int32_t)(rg.v0 + (int64_t)kChunk * j), pol);
        if (has_partial)
          for (int a = 0; a < KA; ++a)
            for (uint32_t r = 0; r < pw; r += 16)
              tma_load_2d(w2_smem + resident_offset(rg.nfull, a, rg, res, KA) + r * 128u, &maps.w2_16,
                          &sh->w2_full, a * 64, (int32_t)(rg.v0 + (int64_t)kChunk * rg.nfull + r), pol);
      }
      // Streamed chunks, every step, in the MMA order.
      int64_t gs = 0;
      bool ok = true;
      for (int k = 0; k < M && ok; ++k)
        for (int i = 0; i < nc && ok; ++i) {
          const int j = chunk_at(i, rg, res);
          if (j < res || j >= rg.nfull) continue;
          for (int a = 0; a < KA; ++a, ++gs) {
            const int s = (int)(gs & 1);
            if (!mbar_wait(&sh->ring_empty[s], ((uint32_t)(gs >> 1) & 1u) ^ 1u, ctl)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&sh->ring_full[s], kFullBlockBytes);
            tma_load_2d(ring_smem + s * kFullBlockBytes, &maps.w2, &sh->ring_full[s], a * 64,
                        (int32_t)(rg.v0 + (int64_t)kChunk * j), pol);
          }
        }
      for (int64_t j = (gs > 2 ? gs - 2 : 0); j < gs; ++j)
        mbar_wait(&sh->ring_full[j & 1], (uint32_t)(j >> 1) & 1u, drain_ctl);
      if (bytes) mbar_wait(&sh->w2_full, 0, drain_ctl);
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      const uint64_t x_desc = sw128_kmajor_desc(smem_u32(x_smem));
      const uint32_t w2_base = smem_u32(w2_smem);
      const uint32_t ring_base = smem_u32(ring_smem);
      bool ok = !(res > 0 || has_partial) || mbar_wait(&sh->w2_full, 0, ctl);
      int64_t t = 0, gs = 0;
      for (int k = 0; k < M && ok; ++k) {
        if (!mbar_wait(&sh->x_full, (uint32_t)k & 1u, ctl)) break;
        tc_fence_after_sync();
        for (int i = 0; i < nc && ok; ++i, ++t) {
          const int j = chunk_at(i, rg, res);
          const int buf = (int)(t & 1);
          // The buffer's previous chunk (t - 2) has been read into registers,
          // so this chunk's MMAs run while the epilogue works on chunk t - 1.
          if (t > 1 && !mbar_wait(&sh->acc_empty[buf], (uint32_t)((t - 2) >> 1) & 1u, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)rg.width(j));
          const uint32_t d_tmem = tmem_base + (uint32_t)(buf * kChunk);
          const bool streamed = j >= res && j < rg.nfull;
          for (int a = 0; a < KA; ++a) {
            uint32_t b_addr;
            int s = 0;
            if (streamed) {
              s = (int)(gs & 1);
              if (!mbar_wait(&sh->ring_full[s], (uint32_t)(gs >> 1) & 1u, ctl)) {
                ok = false;
                break;
              }
              tc_fence_after_sync();
              b_addr = ring_base + (uint32_t)s * kFullBlockBytes;
            } else {
              b_addr = w2_base + resident_offset(j, a, rg, res, KA);
            }
            const uint64_t b_desc = sw128_kmajor_desc(b_addr);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(d_tmem, desc_advance(x_desc, (uint32_t)a * kXAtomBytes + kk * 32),
                           desc_advance(b_desc, kk * 32), idesc, (a | kk) != 0);
            if (streamed) {
              umma_commit(&sh->ring_empty[s]);
              ++gs;
            }
          }
          if (ok) umma_commit(&sh->acc_full[buf]);
        }
      }
      umma_commit(&sh->drain);
      mbar_wait(&sh->drain, 0, drain_ctl);
    }
  } else if (warp == 2) {
    // ----------------------- logits in and out through the stages ----
    // Chunk t (step t / nc, position t % nc) uses stage t % NS. Its boxes
    // load once the stage's previous chunk has been stored (the store has
    // read the stage), so the loads run up to NS chunks ahead of the
    // epilogue, across step boundaries.
    if (lane == 0) {
      prefetch_tensormap(&maps.u);
      prefetch_tensormap(&maps.out);
      const uint64_t pol = policy_evict_first();
      const int64_t T = (int64_t)M * nc;
      const uint32_t box_tx = (uint32_t)B * 128u;
      auto chunk_x = [&](int64_t t, int& k, int& nb) {
        k = (int)(t / nc);
        const int j = chunk_at((int)(t % nc), rg, res);
        nb = rg.boxes(j);
        return (int32_t)(rg.v0 + (int64_t)kChunk * j);
      };
      auto load = [&](int64_t t) {
        int k, nb;
        const int32_t x = chunk_x(t, k, nb);
        const int s = (int)(t % NS);
        mbar_arrive_expect_tx(&sh->u_full[s], (uint32_t)nb * box_tx);
        for (int bx = 0; bx < nb; ++bx)
          tma_load_3d(u_smem + (uint32_t)s * stage_bytes + (uint32_t)bx * box_bytes, &maps.u, &sh->u_full[s],
                      x + bx * kSpan, k, 0, pol);
      };
      int64_t issued = 0;
      for (; issued < T && issued < NS; ++issued) load(issued);
      for (int64_t t = 0; t < T; ++t) {
        const int s = (int)(t % NS);
        if (!mbar_wait(&sh->tile_ready[s], (uint32_t)(t / NS) & 1u, ctl)) break;
        int k, nb;
        const int32_t x = chunk_x(t, k, nb);
        for (int bx = 0; bx < nb; ++bx)
          tma_store_3d(&maps.out, u_smem + (uint32_t)s * stage_bytes + (uint32_t)bx * box_bytes, x + bx * kSpan, k,
                       0);
        bulk_commit_group();
        if (issued < T) {
          bulk_wait_group_read<0>();  // the stage may be refilled once the store has read it
          load(issued);
          ++issued;
        }
      }
      bulk_wait_group<0>();
      // On an abort, the loads still in flight land before the CTA exits.
      for (int64_t t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        mbar_wait(&sh->u_full[t % NS], (uint32_t)(t / NS) & 1u, drain_ctl);
    }
  } else if (warp == 3) {
    // ---------- key merge, grid barrier, previous tokens, U prefetch ----
    // U of step k is prefetched into L2 (bulk prefetch of each row's range)
    // one step ahead: it does not depend on the chain.
    const uint32_t row_bytes = (uint32_t)((rg.v1 - rg.v0) * 2);
    auto prefetch_u = [&](int k) {
      for (int b = lane; b < B && row_bytes; b += 32)
        bulk_prefetch_l2(p.base + ((int64_t)b * M + k) * p.vocab + rg.v0, row_bytes);
    };
    // This CTA's step-k maxima (left in red[] by the epilogue) into the global
    // keys, one red.max per row, then the CTA's arrival: the release-add is
    // cumulative over the lanes' reductions, which __syncwarp orders before
    // it. Each candidate's W1 row then goes into L2, in case it wins (after
    // the arrival, so that the release does not wait for the prefetches).
    auto merge = [&](int k) -> bool {
      if (!warp_wait(&sh->merge_ready, (uint32_t)k & 1u, ctl, lane)) return false;
      unsigned long long* part = p.keys + (size_t)k * B;
      unsigned long long key0 = 0ull, key1 = 0ull;  // rows lane and lane + 32 (B <= 64)
      if (lane < B) {
        key0 = red[lane];
        red[lane] = 0ull;
        if (key0) red_max_gpu(part + lane, key0);
      }
      if (lane + 32 < B) {
        key1 = red[lane + 32];
        red[lane + 32] = 0ull;
        if (key1) red_max_gpu(part + lane + 32, key1);
      }
      __syncwarp();
      if (lane == 0) {
        const bool skip = (p.debug_flags & DSPARK_DEBUG_SKIP_BARRIER_ARRIVAL) && blockIdx.x == 0 && k == 0;
        if (!skip) red_add_release_gpu(p.barrier, 1u);
      }
      __syncwarp();
      if (k + 1 < M) {
        if (key0) bulk_prefetch_l2(p.w1 + (size_t)key_token(key0) * (size_t)(KA * 64), (uint32_t)KA * 128u);
        if (key1) bulk_prefetch_l2(p.w1 + (size_t)key_token(key1) * (size_t)(KA * 64), (uint32_t)KA * 128u);
      }
      return true;
    };
    prefetch_u(0);
    for (int k = 0; k < M; ++k) {
      if (k > 0) {
        if (!merge(k - 1)) break;
        // Every CTA has merged its step k-1 maxima once the counter reaches k * G.
        if (!grid_wait(p.barrier, (uint32_t)k * (uint32_t)G, ctl, lane)) break;
      }
      bool bad = false;
      for (int b = lane; b < BP; b += 32) {
        int32_t row = (int32_t)p.vocab;  // outside W1: the gather writes zeros
        if (b < B) {
          const int64_t id =
              k == 0 ? p.first_prev[b] : (int64_t)key_token(ld_relaxed_gpu(&p.keys[(size_t)(k - 1) * B + b]));
          if (k > 0 && blockIdx.x == 0) p.tokens[(size_t)b * M + (k - 1)] = id;
          if (id < 0 || id >= p.vocab)
            bad = true;
          else
            row = (int32_t)id;
        }
        sh->xid[b] = row;
      }
      if (bad) report_status(p.status, DSPARK_STATUS_TOKEN_RANGE);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->xid_ready);
      __syncwarp();
      // The next step's U goes into L2 once X has landed, out of the window
      // where the epilogue warps wait for W1 rows.
      if (k + 1 < M && warp_wait(&sh->x_full, (uint32_t)k & 1u, ctl, lane)) prefetch_u(k + 1);
      if (k == M - 1 && merge(M - 1) && blockIdx.x == 0) {
        // The last step's tokens, once every CTA has merged its maxima.
        if (grid_wait(p.barrier, (uint32_t)M * (uint32_t)G, ctl, lane))
          for (int b = lane; b < B; b += 32)
            p.tokens[(size_t)b * M + (M - 1)] = (int64_t)key_token(ld_relaxed_gpu(&p.keys[(size_t)(M - 1) * B + b]));
      }
    }
  } else if (warp >= 4) {
    // -------------------------------------------------- epilogue ----
    const int ew = warp - 4;
    const int q = ew & 3;             // TMEM lane quarter
    const int e = ew >> 2;            // which of the quarter's warps
    const int L = 32 * q + lane;      // accumulator lane = operand row
    const int b = L % BP;             // batch row
    const int rep = 128 / BP;
    const int slot = (L / BP) * kEpiPerQuarter + e;
    const int nslots = rep * kEpiPerQuarter;
    const bool row_ok = b < B;
    const uint32_t lane_base = tmem_base + ((uint32_t)(32 * q) << 16);
    const float inv_t = GREEDY ? 0.0f : 1.0f / p.temperature;
    // Row b of a box sits at b * 128 bytes; its 16-byte piece c at (c ^ (b & 7)) * 16.
    const uint32_t row_smem = (uint32_t)b * 128u;
    const uint32_t swz = (uint32_t)(b & 7);
    int64_t t = 0;
    bool ok = true;
    for (int k = 0; k < M && ok; ++k) {
      // X for this step: row L of the operand is W1[x_{k-1}[L % BP]], in the
      // 128-byte swizzle layout (16-byte chunk j of row L at chunk j ^ (L & 7)
      // of its atom). Each distinct 16-byte piece is loaded once per CTA (a
      // warp reads whole rows, so every W1 line is one request; all CTAs read
      // the same rows at once) and stored into every repeat of its row (BP is
      // a multiple of 8, so the repeats share the swizzle). The previous
      // step's MMAs are complete: warp 3 publishes xid only after every
      // epilogue warp has finished the previous step.
      if (!warp_wait(&sh->xid_ready, (uint32_t)k & 1u, ctl, lane)) {
        ok = false;
        break;
      }
      {
        constexpr int kPieces = 8 * KA;  // 16-byte pieces of a W1 row
        const int te = ew * 32 + lane;
        for (int i = te; i < BP * kPieces; i += kEpiWarps * 32) {
          const int row = i / kPieces, c = i % kPieces;
          const int32_t id = sh->xid[row];
          const uint4 val = id < p.vocab
                                ? ld_nc_v4(reinterpret_cast<const uint4*>(p.w1 + (size_t)id * (KA * 64)) + c)
                                : make_uint4(0u, 0u, 0u, 0u);
          uint8_t* dst = x_smem + (uint32_t)(c >> 3) * kXAtomBytes + (uint32_t)row * 128u +
                         (uint32_t)(((c & 7) ^ (row & 7)) << 4);
          for (int r = 0; r < rep; ++r) *reinterpret_cast<uint4*>(dst + (uint32_t)(r * BP) * 128u) = val;
        }
        fence_proxy_async_smem();  // read by the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->x_full);
      }
      uint32_t best = 0u;      // greedy: (ordered bf16 bits, 0xFFFF - local id); temperature: ordered score
      uint32_t best_lid = 0u;  // temperature: the CTA-local id of `best`
      for (int i = 0; i < nc; ++i, ++t) {
        const int j = chunk_at(i, rg, res);
        const int buf = (int)(t & 1);
        const int s = (int)(t % NS);
        const int ngroups = rg.width(j) / kGroup;
        const int64_t c0 = rg.v0 + (int64_t)kChunk * j;
        uint8_t* stage = u_smem + (uint32_t)s * stage_bytes;
        if (!warp_wait(&sh->u_full[s], (uint32_t)(t / NS) & 1u, ctl, lane) ||
            !warp_wait(&sh->acc_full[buf], (uint32_t)(t >> 1) & 1u, ctl, lane)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        // The accumulator goes back to the MMA warp right after this warp's
        // last tensor-memory load of the chunk (at once if it has none).
        if (slot >= ngroups) {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->acc_empty[buf]);
        }
        for (int g = slot; g < ngroups; g += nslots) {
          const int64_t v = c0 + (int64_t)kGroup * g;  // first id of the piece
          const bool full = v + kGroup <= p.vocab;     // else only the first 8 ids exist
          uint32_t d[16];
          __syncwarp();  // tcgen05.ld is warp-aligned
          tmem_ld_32x32b_x16(lane_base + (uint32_t)(buf * kChunk + kGroup * g), d);
          tmem_ld_wait();
          if (g + nslots >= ngroups) {
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->acc_empty[buf]);
          }
          if (!row_ok) continue;
          uint8_t* rowp = stage + (uint32_t)(g >> 2) * box_bytes + row_smem;
          const uint32_t pc = (uint32_t)(g & 3) * 2u;
          uint4* p0 = reinterpret_cast<uint4*>(rowp + ((pc ^ swz) << 4));
          uint4* p1 = reinterpret_cast<uint4*>(rowp + (((pc + 1u) ^ swz) << 4));
          const uint4 u0 = *p0, u1 = *p1;
          uint32_t c[8];
          c[0] = add_round2(u0.x, d[0], d[1]);
          c[1] = add_round2(u0.y, d[2], d[3]);
          c[2] = add_round2(u0.z, d[4], d[5]);
          c[3] = add_round2(u0.w, d[6], d[7]);
          c[4] = add_round2(u1.x, d[8], d[9]);
          c[5] = add_round2(u1.y, d[10], d[11]);
          c[6] = add_round2(u1.z, d[12], d[13]);
          c[7] = add_round2(u1.w, d[14], d[15]);
          *p0 = make_uint4(c[0], c[1], c[2], c[3]);
          *p1 = make_uint4(c[4], c[5], c[6], c[7]);
          const int nid = full ? 16 : 8;
          const uint32_t lid0 = (uint32_t)(v - rg.v0);
          if constexpr (GREEDY) {
            const uint32_t low0 = 0xFFFFu - lid0;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
              if (2 * m >= nid) break;
              const uint32_t klo = ordered_hi16(c[m] << 16) + (low0 - 2 * m);
              const uint32_t khi = ordered_hi16(c[m]) + (low0 - 2 * m - 1);
              best = max(best, max(klo, khi));
            }
          } else {
#pragma unroll
            for (int m4 = 0; m4 < 4; ++m4) {
              if (4 * m4 >= nid) break;
              const uint32_t vq = (uint32_t)(v + 4 * m4);
              const Philox4 r = philox4x32_10(vq >> 2, (uint32_t)k, (uint32_t)b, 0u, p.round_keys);
              const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
              for (int i4 = 0; i4 < 4; ++i4) {
                const uint32_t cw = c[2 * m4 + (i4 >> 1)];
                const float cv = __uint_as_float((i4 & 1) ? (cw & 0xFFFF0000u) : (cw << 16));
                const uint32_t o = ordered_bits(cv * inv_t + gumbel_from_word(w4[i4]));
                if (o > best) {
                  best = o;
                  best_lid = lid0 + 4 * m4 + i4;
                }
              }
            }
          }
        }
        // The stage goes to the storer: the rewritten logits are made visible
        // to the async proxy first.
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->tile_ready[s]);
      }
      if (!ok) break;
      // This CTA's maximum per row, through one shared 64-bit atomic per
      // thread (orderable score, complement of the id); warp 3 takes it on.
      if (row_ok) {
        unsigned long long key;
        if constexpr (GREEDY) {
          const uint32_t vid = (uint32_t)rg.v0 + (0xFFFFu - (best & 0xFFFFu));
          key = best ? ((unsigned long long)(best >> 16) << 32) | (unsigned long long)(0xFFFFFFFFu - vid) : 0ull;
        } else {
          const uint32_t vid = (uint32_t)rg.v0 + best_lid;
          key = best ? ((unsigned long long)best << 32) | (unsigned long long)(0xFFFFFFFFu - vid) : 0ull;
        }
        if (key) atomicMax(&red[b], key);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->merge_ready);
    }
  }

  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

struct RowsPlan {
  int bp, resident_full, ring, stages;
  uint32_t w2_bytes;
  size_t smem;
  bool ok;
};

// The shared-memory plan for `stages` logit stages: resident W2 chunks, the
// streaming ring when they do not all fit, X, the stages and the tail.
RowsPlan rows_plan_stages(int64_t batch, int64_t vocab, int32_t rank, int grid, int stages) {
  RowsPlan c{};
  if (batch < 1 || batch > kMaxRowsBatch || rank % 64 != 0 || rank < 64 || rank > 256 || vocab % 8 != 0 ||
      grid < 1 || stages < 2 || stages > kMaxStages)
    return c;
  c.bp = batch <= 32 ? 32 : 64;
  c.stages = stages;
  const int ka = rank / 64;
  const int64_t spans = (vocab + kSpan - 1) / kSpan;
  if (grid > spans) return c;
  // Every CTA's range as the kernel cuts it: the most chunks, the most full
  // chunks and the widest partial chunk over all of them.
  int64_t nmax = 0;
  int64_t part_w = 0;
  for (int g = 0; g < grid; ++g) {
    const int64_t v0 = spans * g / grid * kSpan;
    const int64_t e = spans * (g + 1) / grid * kSpan;
    const int64_t v1 = e < vocab ? e : vocab;
    if (v1 <= v0) return c;
    const int64_t n16 = (v1 - v0 + 15) & ~15ll;
    nmax = n16 > nmax ? n16 : nmax;
    part_w = n16 % kChunk > part_w ? n16 % kChunk : part_w;
  }
  if (nmax > 65535 || (nmax + kChunk - 1) / kChunk > kMaxChunks) return c;
  const int nfull = (int)(nmax / kChunk);
  const uint32_t full_bytes = (uint32_t)ka * kFullBlockBytes;
  const uint32_t part_bytes = (uint32_t)ka * (uint32_t)part_w * 128u;
  const size_t stage_bytes = (size_t)kBoxesPerChunk * c.bp * 128;
  const size_t fixed = 1024 + (size_t)ka * kXAtomBytes + (size_t)stages * stage_bytes + 128 * 8 + sizeof(RowsTail) + 64;
  if (fixed >= kSmemLimit) return c;
  const size_t budget = kSmemLimit - fixed;
  const size_t ring_bytes = 2 * (size_t)kFullBlockBytes;
  if ((size_t)nfull * full_bytes + part_bytes <= budget) {
    c.resident_full = nfull;
    c.ring = 0;
  } else {
    if (budget < ring_bytes + part_bytes) return c;
    c.resident_full = (int)((budget - ring_bytes - part_bytes) / full_bytes);
    c.ring = 1;
  }
  // Every CTA keeps min(its full chunks, resident_full) full chunks and its
  // partial chunk, which fit in this area.
  c.w2_bytes = (uint32_t)c.resident_full * full_bytes + part_bytes;
  c.smem = fixed + c.w2_bytes + (c.ring ? ring_bytes : 0);
  c.ok = c.smem <= kSmemLimit;
  return c;
}

// Three stages where they cost no resident W2 chunk, else two.
RowsPlan rows_plan(int64_t batch, int64_t vocab, int32_t rank, int grid) {
  const RowsPlan two = rows_plan_stages(batch, vocab, rank, grid, 2);
  const RowsPlan three = rows_plan_stages(batch, vocab, rank, grid, 3);
  if (three.ok && (!two.ok || (three.resident_full >= two.resident_full && three.ring <= two.ring))) return three;
  return two;
}

template <int KA, bool GREEDY>
cudaError_t launch_rows_ka(const TcSampleArgs& a, const RowsPlan& c, int grid, cudaStream_t stream) {
  RowsMaps maps;
  const uint64_t wdim[2] = {(uint64_t)a.rank, (uint64_t)a.vocab};
  const uint64_t wstr[1] = {(uint64_t)a.rank * 2};
  const uint32_t box[2] = {64, (uint32_t)kChunk};
  const uint32_t box16[2] = {64, 16};
  const uint64_t udim[3] = {(uint64_t)a.vocab, (uint64_t)a.steps, (uint64_t)a.batch};
  const uint64_t ustr[2] = {(uint64_t)a.vocab * 2, (uint64_t)a.vocab * 2 * (uint64_t)a.steps};
  const uint32_t ubox[3] = {(uint32_t)kSpan, 1u, (uint32_t)a.batch};
  if (!encode_tensor_map(&maps.w2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w2, wdim, wstr, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&maps.w2_16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w2, wdim, wstr, box16,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&maps.u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.base, udim, ustr, ubox,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&maps.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.corrected, udim, ustr, ubox,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  RowsParams p{};
  p.base = static_cast<const __nv_bfloat16*>(a.base);
  p.first_prev = a.first_prev;
  p.w1 = static_cast<const __nv_bfloat16*>(a.w1);
  p.tokens = a.tokens;
  p.keys = a.keys;
  p.barrier = a.barrier;
  p.status = a.status;
  p.vocab = a.vocab;
  p.batch = (int32_t)a.batch;
  p.bp = c.bp;
  p.steps = (int32_t)a.steps;
  p.ka = KA;
  p.spans = (int32_t)((a.vocab + kSpan - 1) / kSpan);
  p.resident_full = c.resident_full;
  p.w2_bytes = c.w2_bytes;
  p.ring = c.ring;
  p.stages = c.stages;
  p.temperature = a.temperature;
  p.round_keys = round_keys_for(a.seed);
  p.wait_limit_ns = a.wait_limit_ns;
  p.debug_flags = a.debug_flags;

  cudaError_t e = cudaFuncSetAttribute(tc_sample_rows_kernel<KA, GREEDY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)c.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, tc_sample_rows_kernel<KA, GREEDY>, maps, p);
  note_launch();
  return e;
}

template <bool GREEDY>
cudaError_t launch_rows_mode(const TcSampleArgs& a, const RowsPlan& c, int grid, cudaStream_t s) {
  switch (a.rank / 64) {
    case 1: return launch_rows_ka<1, GREEDY>(a, c, grid, s);
    case 2: return launch_rows_ka<2, GREEDY>(a, c, grid, s);
    case 3: return launch_rows_ka<3, GREEDY>(a, c, grid, s);
    case 4: return launch_rows_ka<4, GREEDY>(a, c, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

int rows_grid(int64_t vocab, int num_sms) {
  const int64_t spans = (vocab + kSpan - 1) / kSpan;
  return (int)(spans < num_sms ? spans : num_sms);
}

}  // namespace

bool tc_sample_rows_supported(int64_t batch, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype,
                              int num_sms) {
  if (logits_dtype != DSPARK_DTYPE_BF16 || weight_dtype != DSPARK_DTYPE_BF16) return false;
  if (vocab < 16 || vocab >= (1ll << 31) - kChunk || num_sms < 1) return false;
  return rows_plan(batch, vocab, rank, rows_grid(vocab, num_sms)).ok;
}

cudaError_t launch_tc_sample_rows(const TcSampleArgs& a, int num_sms, cudaStream_t s) {
  const int grid = rows_grid(a.vocab, num_sms);
  const RowsPlan c = rows_plan(a.batch, a.vocab, a.rank, grid);
  if (!c.ok) return cudaErrorInvalidValue;
  return a.greedy ? launch_rows_mode<true>(a, c, grid, s) : launch_rows_mode<false>(a, c, grid, s);
}

}  // namespace dspark
