// Left-to-right block sampling on the sm_100a tensor cores
// (VanillaMarkov.sample_block_tokens and _sample_tokens of the vendored
// markov_head.py). For k = 0 .. M-1 and every block b:
//
//     c_k[b, v] = round_bf16( U[b, k, v] + sum_j W1[x_{k-1}[b], j] * W2[v, j] )
//     x_k[b]    = argmax_v c_k[b, v]                    (greedy)
//              or argmax_v c_k[b, v] / T + g(b, k, v)   (Gumbel-max, Philox noise)
//
// with x_{-1} = first_prev. One launch covers all M steps. The grid is one
// CTA per SM (cooperative launch, so all CTAs are resident); CTA c owns a
// contiguous run of 128-id vocabulary tiles.
//
// W2 stays on chip for the whole launch. Each CTA loads its slice of W2 once:
// as many tiles as fit into shared memory (by TMA, 128-byte swizzle), the rest
// into tensor memory (tcgen05.st), where they serve as the A operand of the
// MMA directly. Across 148 SMs that holds a 33 MB W2, so the M steps read it
// from HBM once and never again.
//
// Per step each CTA
//   - gathers X = W1[x_{k-1}] ([B_pad x r], TMA tile::gather4 row gathers);
//   - computes bias^T = W2_tile[128 x r] . X^T[r x B_pad] per vocabulary tile
//     on tcgen05 (swap-AB: M = 128 ids, N = B padded to 16, K = r);
//   - adds U (TMA-staged [B x 128] tiles, prefetched across step boundaries
//     since U does not depend on the chain), rounds to bf16, stores c_k, and
//     keeps the packed (score, id) maximum per b;
//   - merges its maxima into a per-(k, b) 64-bit key with atomicMax, then
//     passes a grid barrier (bounded wait) after which every CTA decodes x_k.
//
// Warp roles (640 threads): 0 W2 loader, then the tile store warp; 1 MMA
// issuer and TMEM owner; 2 U producer; 3 W1 gather and grid barrier; 4-19 up
// to four epilogue groups of four warps that take tiles round-robin (one TMEM
// accumulator each; thread = vocabulary id). Several groups in flight hide the
// latency of the per-element work and even out the tile counts per step.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace dspark {
namespace {

constexpr int kBV = 128;                           // vocabulary ids per tile (MMA M)
constexpr int kAtomK = 64;                         // bf16 elements per 128-byte swizzle row
constexpr int kW2AtomBytes = 128 * 128;            // one 128-id x 64-element W2 atom
constexpr int kMaxGroups = 4;                      // epilogue groups
constexpr int kThreads = 128 + kMaxGroups * 128;   // four single-role warps + the groups
constexpr int kMaxStages = 12;
constexpr int kMaxBatch = 256;
constexpr int kMaxTiles = 24;                      // vocabulary tiles per CTA
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmemLimit = 232448;              // dynamic shared memory per block on sm_100

__host__ __device__ constexpr size_t align8(size_t x) { return (x + 7) & ~size_t(7); }

struct __align__(64) SampleMaps {
  CUtensorMap w2;   // [vocab, rank] bf16, box 64 x 128, 128B swizzle
  CUtensorMap w1;   // [vocab, rank] bf16, box 64 x 1 (row gathers), 128B swizzle
  CUtensorMap u;    // [batch, steps, vocab] bf16, box 128 x 1 x batch
  CUtensorMap out;  // same geometry as u
};

struct SampleParams {
  const int64_t* first_prev;
  const __nv_bfloat16* w1;
  const __nv_bfloat16* w2;
  int64_t* tokens;
  unsigned long long* keys;
  uint32_t* barrier;
  uint32_t* status;
  int32_t batch, batch_pad, steps, rank;
  int64_t vocab;
  int32_t vocab_tiles;
  int32_t smem_tiles;  // W2 tiles a CTA keeps in shared memory; the rest go to TMEM
  int32_t u_slots;
  uint32_t u_slot_bytes, x_bytes;  // x_bytes: one step's gathered operand
  float temperature;
  PhiloxRoundKeys round_keys;  // of the launch's seed
  uint64_t wait_limit_ns;
  uint32_t debug_flags;
  int32_t groups;  // epilogue groups in use (<= kMaxGroups)
};

struct SampleTail {
  uint64_t w2_full, w2t_full;
  uint64_t u_full[kMaxStages], u_empty[kMaxStages], tile_ready[kMaxStages];
  uint64_t x_full, x_empty;
  uint64_t acc_full[kMaxGroups], acc_empty[kMaxGroups];
  uint64_t drain;
  int32_t xid[kMaxBatch];
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool barrier_and(bool v, uint32_t id, uint32_t n) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return out != 0;
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

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p) : "memory");
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

// Order-preserving bits of an fp32 value computed by this kernel's own
// arithmetic, as an unsigned integer: the sign bit is set for non-negative
// values and every bit is flipped for negative ones. Adding +0 first makes -0
// into +0 (the two compare equal), and turns any NaN into the canonical
// positive NaN of the GPU's floating-point unit, which orders above +inf
// (NaN counts as the largest value). Two ALU operations besides the add.
__device__ __forceinline__ uint32_t ordered_bits(float x) {
  const uint32_t b = __float_as_uint(x + 0.0f);
  return b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
}

// Greedy key of a bf16 corrected logit: its order-preserving bits in the high
// half and `low` = 0xFFFF - (CTA-local vocabulary index) in the low half, so
// that the maximum is the largest value and, among equal values, the lowest
// id. The low half of a bf16 value widened to fp32 is zero, except for the
// canonical NaN, whose low half the mask clears (so equal NaNs tie too).
__device__ __forceinline__ uint32_t greedy_key(uint32_t bf16_bits, uint32_t low) {
  return (ordered_bits(__uint_as_float(bf16_bits << 16)) & 0xFFFF0000u) | low;
}

// Lane 0 waits (bounded) until the grid-barrier counter reaches `target`; the
// warp follows its verdict.
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
      __nanosleep(32);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  return ok;
}

// GREEDY selects at compile time: the greedy instance carries no noise code.
template <int KA, bool GREEDY>
__global__ void __launch_bounds__(kThreads, 1)
    tc_sample_kernel(const __grid_constant__ SampleMaps maps, const SampleParams p) {
  using Key = typename std::conditional<GREEDY, uint32_t, unsigned long long>::type;
  constexpr int kTileCols = KA * 32;  // TMEM columns of one W2 tile (two bf16 per column)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* w2_smem = smem;                                              // smem_tiles x KA atoms
  uint8_t* x_smem = w2_smem + (size_t)p.smem_tiles * KA * kW2AtomBytes;  // one step's X
  uint8_t* u_smem = x_smem + (size_t)p.x_bytes;                         // u_slots x u_slot_bytes
  Key* red = reinterpret_cast<Key*>(u_smem + (size_t)p.u_slots * p.u_slot_bytes);  // [group][quarter][b]
  SampleTail* sh = reinterpret_cast<SampleTail*>(
      u_smem + (size_t)p.u_slots * p.u_slot_bytes + align8((size_t)kMaxGroups * 4 * p.batch_pad * sizeof(Key)));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int t_begin = (int)((int64_t)p.vocab_tiles * blockIdx.x / G);
  const int t_end = (int)((int64_t)p.vocab_tiles * (blockIdx.x + 1) / G);
  const int nt = t_end - t_begin;
  const int n_smem = nt < p.smem_tiles ? nt : p.smem_tiles;  // tiles [0, n_smem) in smem, the rest in TMEM
  const int M = p.steps;
  const int B = p.batch;
  const int BB = p.batch_pad;
  const int NG = p.groups;
  const int64_t items = (int64_t)M * nt;
  const uint32_t atom_x = (uint32_t)BB * 128u;  // bytes of one X atom
  const uint32_t acc_cols = (uint32_t)(NG * BB);

  if (threadIdx.x == 0) {
    mbar_init(&sh->w2_full, 1);
    mbar_init(&sh->w2t_full, 4);
    for (int i = 0; i < p.u_slots; ++i) {
      mbar_init(&sh->u_full[i], 1);
      mbar_init(&sh->u_empty[i], 1);
      mbar_init(&sh->tile_ready[i], 4);  // the four warps of the tile's epilogue group
    }
    mbar_init(&sh->x_full, 1);
    mbar_init(&sh->x_empty, 1);
    for (int i = 0; i < kMaxGroups; ++i) {
      mbar_init(&sh->acc_full[i], 1);
      mbar_init(&sh->acc_empty[i], 4);
    }
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  __syncwarp();  // warp 0 diverged around the barrier set-up
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = sh->tmem_base;
  const WaitCtl ctl{&sh->abort_flag, p.status, p.wait_limit_ns};
  volatile int never = 0;
  const WaitCtl drain_ctl{&never, p.status, p.wait_limit_ns};

  if (warp == 0) {
    // ------------------------- W2 into shared memory, then store warp ----
    if (lane == 0) {
      if (n_smem > 0) {
        prefetch_tensormap(&maps.w2);
        const uint64_t pol = policy_evict_first();
        mbar_arrive_expect_tx(&sh->w2_full, (uint32_t)(n_smem * KA * kW2AtomBytes));
        for (int tt = 0; tt < n_smem; ++tt)
#pragma unroll
          for (int ka = 0; ka < KA; ++ka)
            tma_load_2d(w2_smem + (size_t)(tt * KA + ka) * kW2AtomBytes, &maps.w2, &sh->w2_full, ka * kAtomK,
                        (t_begin + tt) * kBV, pol);
      }
      // TMA-store each finished tile of corrected logits and hand its U slot
      // back to the producer once the store has read it; one store in flight.
      int prev_s = -1;
      for (int64_t i = 0; i < items; ++i) {
        const int k = (int)(i / nt);
        const int t = t_begin + (int)(i % nt);
        const int s = (int)(i % p.u_slots);
        if (!mbar_wait(&sh->tile_ready[s], (uint32_t)(i / p.u_slots) & 1u, ctl)) break;
        tma_store_3d(&maps.out, u_smem + (size_t)s * p.u_slot_bytes, t * kBV, k, 0);
        bulk_commit_group();
        if (prev_s >= 0) {
          bulk_wait_group_read<1>();
          mbar_arrive(&sh->u_empty[prev_s]);
        }
        prev_s = s;
      }
      bulk_wait_group<0>();
      if (n_smem > 0) mbar_wait(&sh->w2_full, 0, drain_ctl);  // the W2 copies are done before exit
    }
  } else if (warp == 2) {
    // ------------------------------------------------ U producer ----
    if (lane == 0) {
      prefetch_tensormap(&maps.u);
      prefetch_tensormap(&maps.out);
      const uint64_t pol_stream = policy_evict_first();
      int64_t i = 0;
      for (; i < items; ++i) {
        const int k = (int)(i / nt);
        const int t = t_begin + (int)(i % nt);
        const int s = (int)(i % p.u_slots);
        if (!mbar_wait(&sh->u_empty[s], ((uint32_t)(i / p.u_slots) & 1u) ^ 1u, ctl)) break;
        mbar_arrive_expect_tx(&sh->u_full[s], (uint32_t)B * kBV * 2u);  // the box, not the padded slot
        tma_load_3d(u_smem + (size_t)s * p.u_slot_bytes, &maps.u, &sh->u_full[s], t * kBV, k, 0, pol_stream);
      }
      for (int64_t j = (i > p.u_slots ? i - p.u_slots : 0); j < i; ++j)
        mbar_wait(&sh->u_full[j % p.u_slots], (uint32_t)(j / p.u_slots) & 1u, drain_ctl);
    }
  } else if (warp == 3) {
    // ------------------------------------ W1 gather + grid barrier ----
    const uint64_t pol_w1 = policy_evict_last();
    if (lane == 0) prefetch_tensormap(&maps.w1);
    // One X buffer suffices: step k+1's rows are gathered only after the grid
    // barrier, i.e. after every MMA of step k has completed.
    for (int k = 0; k < M; ++k) {
      const uint32_t xe_par = ((uint32_t)k & 1u) ^ 1u;
      // Lane 0 decides and the warp follows, so the lanes never split around
      // the warp-wide shuffles below.
      bool xe_ok = lane == 0 ? mbar_wait(&sh->x_empty, xe_par, ctl) : true;
      xe_ok = __shfl_sync(0xffffffffu, xe_ok ? 1 : 0, 0) != 0;
      if (!xe_ok) break;
      if (lane != 0) mbar_wait(&sh->x_empty, xe_par, ctl);  // already complete
      // Every CTA has merged its step k-1 maxima once the counter reaches k * G.
      if (k > 0 && !grid_wait(p.barrier, (uint32_t)k * (uint32_t)G, ctl, lane)) break;
      bool bad = false;
      // Row of W1 for each batch column; padding columns and invalid ids use
      // row `vocab`, outside the tensor, which the gather reads as zeros.
      for (int b = lane; b < BB; b += 32) {
        int32_t row = (int32_t)p.vocab;
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
      // The operand arrives through the async proxy (TMA row gathers into the
      // 128-byte-swizzle K-major layout), so no proxy fence is needed before
      // the MMA reads it: x_full completes on the transferred byte count.
      if (lane == 0) mbar_arrive_expect_tx(&sh->x_full, p.x_bytes);
      __syncwarp();
      const int quads = BB / 4;
      for (int i = lane; i < quads * KA; i += 32) {
        const int j = i % quads, ka = i / quads;
        tma_gather4(x_smem + ka * atom_x + j * 4 * 128, &maps.w1, &sh->x_full, ka * kAtomK, sh->xid[4 * j],
                    sh->xid[4 * j + 1], sh->xid[4 * j + 2], sh->xid[4 * j + 3], pol_w1);
      }
      __syncwarp();
      if (k == M - 1 && blockIdx.x == 0) {
        // The last step's tokens, once every CTA has merged its maxima.
        if (grid_wait(p.barrier, (uint32_t)M * (uint32_t)G, ctl, lane))
          for (int b = lane; b < B; b += 32)
            p.tokens[(size_t)b * M + (M - 1)] = (int64_t)key_token(ld_relaxed_gpu(&p.keys[(size_t)(M - 1) * B + b]));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBV, (uint32_t)BB);
      // Descriptors are built once; each K-step only advances the start address.
      const uint64_t w2_desc = sw128_kmajor_desc(smem_u32(w2_smem));
      const uint64_t x_desc = sw128_kmajor_desc(smem_u32(x_smem));
      bool ok = (n_smem == 0 || mbar_wait(&sh->w2_full, 0, ctl)) && (nt == n_smem || mbar_wait(&sh->w2t_full, 0, ctl));
      for (int k = 0; k < M && ok; ++k) {
        if (!mbar_wait(&sh->x_full, (uint32_t)k & 1u, ctl)) break;
        for (int tt = 0; tt < nt; ++tt) {
          const int64_t i = (int64_t)k * nt + tt;
          const int abuf = (int)(i % NG);
          if (!mbar_wait(&sh->acc_empty[abuf], ((uint32_t)(i / NG) & 1u) ^ 1u, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * BB);
          if (tt < n_smem) {
            const uint64_t a0 = desc_advance(w2_desc, (uint32_t)(tt * KA) * kW2AtomBytes);
#pragma unroll
            for (int kk = 0; kk < KA * kAtomK / 16; ++kk)
              umma_bf16_ss(d_tmem, desc_advance(a0, (kk >> 2) * kW2AtomBytes + (kk & 3) * 32),
                           desc_advance(x_desc, (kk >> 2) * atom_x + (kk & 3) * 32), idesc, kk != 0);
          } else {
            const uint32_t a_tmem = tmem_base + acc_cols + (uint32_t)((tt - n_smem) * kTileCols);
#pragma unroll
            for (int kk = 0; kk < KA * kAtomK / 16; ++kk)
              umma_bf16_ts(d_tmem, a_tmem + kk * 8, desc_advance(x_desc, (kk >> 2) * atom_x + (kk & 3) * 32), idesc,
                           kk != 0);
          }
          umma_commit(&sh->acc_full[abuf]);
        }
        if (ok) umma_commit(&sh->x_empty);
      }
      umma_commit(&sh->drain);
      mbar_wait(&sh->drain, 0, drain_ctl);
    }
  } else if ((warp - 4) / 4 < NG) {
    // -------------------------------------------------- epilogue ----
    // Group g takes the tiles whose item index k * nt + tt is g modulo the
    // group count, with TMEM accumulator g. Thread (quarter q, lane) owns
    // vocabulary id 32q + lane of the tile (its TMEM lane) and every batch
    // column b.
    const int g = (warp - 4) >> 2;
    const int te = threadIdx.x - 128;            // 0..NG*128-1 across the groups
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const uint32_t allbar = 1;  // all epilogue warps (named barrier 0 is __syncthreads)
    const uint32_t all_n = (uint32_t)NG * 128u;
    const int chunks = (B + 15) >> 4;  // 16 batch columns per chunk
    Key* my_red = red + (size_t)(g * 4 + q) * BB;
    const uint32_t vbase = (uint32_t)t_begin * kBV;
    const float inv_t = GREEDY ? 0.0f : 1.0f / p.temperature;

    if (g == 0 && nt > n_smem) {
      // W2 tiles beyond the shared-memory share go to TMEM once: thread `row`
      // writes W2[v] (rank bf16, two per column) into its own lane.
      const uint32_t lane_base = tmem_base + ((uint32_t)(32 * q) << 16) + acc_cols;
      for (int j = 0; j < nt - n_smem; ++j) {
        const int64_t v = (int64_t)(t_begin + n_smem + j) * kBV + row;
        const uint4* src = reinterpret_cast<const uint4*>(p.w2 + (v < p.vocab ? v : 0) * p.rank);
#pragma unroll
        for (int c = 0; c < KA; ++c) {
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint4 x = v < p.vocab ? ld_nc_v4(src + c * 8 + i) : make_uint4(0u, 0u, 0u, 0u);
            w[4 * i + 0] = x.x;
            w[4 * i + 1] = x.y;
            w[4 * i + 2] = x.z;
            w[4 * i + 3] = x.w;
          }
          __syncwarp();
          tmem_st_32x32b_x32(lane_base + (uint32_t)(j * kTileCols + c * 32), w);
        }
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->w2t_full);
      __syncwarp();
    }

    bool ok = true;
    for (int k = 0; k < M; ++k) {
      for (int b = lane; b < BB; b += 32) my_red[b] = 0;
      const int first = (g - (int)(((int64_t)k * nt) % NG) + NG) % NG;
      for (int tt = first; tt < nt && ok; tt += NG) {
        const int64_t i = (int64_t)k * nt + tt;
        const int s = (int)(i % p.u_slots);
        const uint32_t acc_par = (uint32_t)(i / NG) & 1u;
        const uint32_t u_par = (uint32_t)(i / p.u_slots) & 1u;
        if (!warp_wait(&sh->acc_full[g], acc_par, ctl, lane) || !warp_wait(&sh->u_full[s], u_par, ctl, lane)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const int t = t_begin + tt;
        const uint32_t v = (uint32_t)(t * kBV + row);
        const bool valid = (int64_t)v < p.vocab;
        __nv_bfloat16* slot = reinterpret_cast<__nv_bfloat16*>(u_smem + (size_t)s * p.u_slot_bytes) + row;
        const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(g * BB);
        // A chunk is 16 batch columns. Full chunks of a tile whose ids are all
        // in the vocabulary need no per-element validity selects.
        const bool tile_valid = (int64_t)(t + 1) * kBV <= p.vocab;
        const uint32_t low = 0xFFFFu - (v - vbase);      // greedy key's low half
        const uint32_t vwarp = (uint32_t)(t * kBV + 32 * q);  // id of lane 0
        auto chunk = [&](int ch, auto full_tag) {
          constexpr bool FULL = decltype(full_tag)::value;
          uint32_t d[16];
          tmem_ld_32x32b_x16(tb + 16 * ch, d);
          tmem_ld_wait();
          const int nb = FULL ? 16 : (B - 16 * ch < 16 ? B - 16 * ch : 16);  // batch columns of this chunk
          __nv_bfloat16* col = slot + (size_t)(16 * ch) * kBV;
          Key* red_ch = my_red + 16 * ch;
          // All loads first, then the arithmetic, then all stores: the loads
          // of one thread are independent, so they overlap instead of each
          // waiting out the shared-memory latency of the previous element.
          __nv_bfloat16 c[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) c[j] = (FULL || j < nb) ? col[j * kBV] : __float2bfloat16_rn(0.0f);
#pragma unroll
          for (int j = 0; j < 16; ++j) c[j] = __float2bfloat16_rn(__bfloat162float(c[j]) + __uint_as_float(d[j]));
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (FULL || j < nb) col[j * kBV] = c[j];
          // Per column: the warp's maximum key (one redux each, with no
          // branch between them); lane j keeps column j's, and each lane
          // merges its column into this warp's running maxima with one
          // shared-memory atomic.
          if constexpr (GREEDY) {
            uint32_t mine = 0u;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (!FULL && j >= nb) break;  // uniform
              uint32_t kj = greedy_key(__bfloat16_as_ushort(c[j]), low);
              if (!FULL) kj = valid ? kj : 0u;
              const uint32_t m = __reduce_max_sync(0xffffffffu, kj);
              mine = lane == j ? m : mine;
            }
            if (lane < nb) atomicMax(&red_ch[lane], mine);
          } else {
            // One Philox call (counter v>>2, k, b, 0) serves the four ids of a
            // lane quad. Lane i of the quad computes the calls of columns
            // 4jj + i; a 4 x 4 transpose inside the quad then hands each lane
            // the word of its own id (v & 3) for all four columns.
            const uint32_t qi = (uint32_t)lane & 3u;
            uint32_t o[16];  // order-preserving bits of each column's score (0: no candidate)
#pragma unroll
            for (int j = 0; j < 16; ++j) o[j] = 0u;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              if (!FULL && 4 * jj >= nb) break;  // uniform: no batch column left in this chunk
              const Philox4 r = philox4x32_10(v >> 2, (uint32_t)k, (uint32_t)(16 * ch + 4 * jj) + qi, 0u,
                                              p.round_keys);
              uint32_t a0 = r.x, a1 = r.y, a2 = r.z, a3 = r.w;
              {  // exchange across lane bit 0
                const bool odd = (qi & 1u) != 0;
                const uint32_t s0 = odd ? a0 : a1, s1 = odd ? a2 : a3;
                const uint32_t r0 = __shfl_xor_sync(0xffffffffu, s0, 1), r1 = __shfl_xor_sync(0xffffffffu, s1, 1);
                if (odd) { a0 = r0; a2 = r1; } else { a1 = r0; a3 = r1; }
              }
              {  // exchange across lane bit 1
                const bool hi = (qi & 2u) != 0;
                const uint32_t s0 = hi ? a0 : a2, s1 = hi ? a1 : a3;
                const uint32_t r0 = __shfl_xor_sync(0xffffffffu, s0, 2), r1 = __shfl_xor_sync(0xffffffffu, s1, 2);
                if (hi) { a0 = r0; a1 = r1; } else { a2 = r0; a3 = r1; }
              }
              const uint32_t wv[4] = {a0, a1, a2, a3};  // words of columns 4jj + 0..3 for this lane's id
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int j = 4 * jj + i;
                const float score = __bfloat162float(c[j]) * inv_t + gumbel_from_word(wv[i]);
                o[j] = ordered_bits(score);
                if (!FULL) o[j] = (j < nb && valid) ? o[j] : 0u;
              }
            }
            // Per column: the largest score bits (one redux) and the lowest
            // lane (lowest id) holding them (a ballot); lane j keeps column j's
            // pair and forms one 64-bit key.
            uint32_t mo = 0u, mw = 0u;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (!FULL && j >= nb) break;  // uniform
              const uint32_t m = __reduce_max_sync(0xffffffffu, o[j]);
              const uint32_t w = (uint32_t)(__ffs(__ballot_sync(0xffffffffu, o[j] == m)) - 1);
              mo = lane == j ? m : mo;
              mw = lane == j ? w : mw;
            }
            const Key mine = mo ? ((Key)mo << 32) | (Key)(0xffffffffu - (vwarp + mw)) : (Key)0;
            if (lane < nb && mine > red_ch[lane]) red_ch[lane] = mine;
          }
        };
#pragma unroll 1
        for (int ch = 0; ch < chunks; ++ch) {
          if (tile_valid && B - 16 * ch >= 16)
            chunk(ch, std::true_type{});
          else
            chunk(ch, std::false_type{});
        }
        __syncwarp();
        tc_fence_before_sync();
        fence_proxy_async_smem();  // this thread's stores become visible to the TMA store
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sh->acc_empty[g]);
          mbar_arrive(&sh->tile_ready[s]);
        }
        __syncwarp();
      }
      // The groups agree to go on (an abort anywhere ends every step here).
      if (!barrier_and(ok, allbar, all_n)) break;
      // Merge the partial maxima of each b, then this CTA's into the global
      // keys (64-bit: orderable score, complement of the global id). The
      // arrival below is a release by one thread after the CTA barrier, so
      // it is cumulative over every thread's reduction ordered before it; a
      // fence per thread would wait for each contended reduction in turn.
      // The W1 row of this CTA's candidate goes into L2 after the arrival
      // (a release also waits for the thread's earlier prefetches): if it
      // wins, the next step's gather finds it there.
      unsigned long long cand = 0ull;  // this thread's row candidate (B <= all_n rows)
      for (int b = te; b < B; b += (int)all_n) {
        Key m = 0;
        for (int r = 0; r < NG * 4; ++r) m = red[(size_t)r * BB + b] > m ? red[(size_t)r * BB + b] : m;
        unsigned long long gk;
        if constexpr (GREEDY) {
          const uint32_t vid = vbase + (0xFFFFu - (m & 0xFFFFu));
          gk = m ? ((unsigned long long)(m >> 16) << 32) | (unsigned long long)(0xFFFFFFFFu - vid) : 0ull;
        } else {
          gk = m;
        }
        if (gk) red_max_gpu(&p.keys[(size_t)k * B + b], gk);
        cand = gk;
      }
      named_barrier_sync(allbar, all_n);
      if (te == 0) {
        const bool skip = (p.debug_flags & DSPARK_DEBUG_SKIP_BARRIER_ARRIVAL) && blockIdx.x == 0 && k == 0;
        if (!skip) red_add_release_gpu(p.barrier, 1u);
      }
      if (cand && k + 1 < M) prefetch_l2(p.w1 + (size_t)key_token(cand) * p.rank);
    }
  }

  // Single-lane roles and lane-0 branches leave warps diverged; bar.sync is
  // warp-aligned, so every warp reconverges first.
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

struct SampleConfig {
  int smem_tiles, u_slots, groups;
  uint32_t u_slot_bytes, x_bytes;
  size_t smem_bytes;
  bool ok;
};

size_t align1024(size_t x) { return (x + 1023) & ~size_t(1023); }

int batch_pad_of(int64_t batch) { return (int)(((batch + 15) / 16) * 16); }

// Shared memory: [W2 tiles][X][U ring][partial maxima][tail]; tensor memory:
// [accumulators: groups x batch_pad][W2 tiles that did not fit in smem].
// Prefer four epilogue groups, then more U slots, and give the rest of shared
// memory to W2; the remaining tiles must fit in tensor memory.
SampleConfig plan(int ka, int batch, int batch_pad, int tiles_per_cta) {
  SampleConfig c{};
  c.u_slot_bytes = (uint32_t)align1024((size_t)batch * kBV * 2);
  c.x_bytes = (uint32_t)((size_t)ka * batch_pad * 128);
  const size_t tile_bytes = (size_t)ka * kW2AtomBytes;
  const size_t fixed =
      1024 + (size_t)c.x_bytes + align8((size_t)kMaxGroups * 4 * batch_pad * 8) + sizeof(SampleTail) + 64;
  if (tiles_per_cta > kMaxTiles || fixed > kSmemLimit) return c;
  for (int groups = kMaxGroups; groups >= 1; groups >>= 1) {
    for (int u = 8; u >= 2; --u) {
      const size_t used = fixed + (size_t)u * c.u_slot_bytes;
      if (used > kSmemLimit) continue;
      int smem_tiles = (int)((kSmemLimit - used) / tile_bytes);
      if (smem_tiles > tiles_per_cta) smem_tiles = tiles_per_cta;
      const int tmem_tiles = tiles_per_cta - smem_tiles;
      if ((uint32_t)(groups * batch_pad + tmem_tiles * ka * 32) > kTmemCols) continue;
      c.smem_tiles = smem_tiles;
      c.u_slots = u;
      c.groups = groups;
      c.smem_bytes = used + (size_t)smem_tiles * tile_bytes;
      c.ok = true;
      return c;
    }
  }
  return c;
}

template <int KA, bool GREEDY>
cudaError_t launch_ka(const TcSampleArgs& a, int num_sms, cudaStream_t stream) {
  const int BB = batch_pad_of(a.batch);
  const int tiles = (int)((a.vocab + kBV - 1) / kBV);
  const int grid = tiles < num_sms ? tiles : num_sms;
  const SampleConfig c = plan(KA, (int)a.batch, BB, (tiles + grid - 1) / grid);
  if (!c.ok) return cudaErrorInvalidValue;
  SampleMaps maps;
  const uint32_t wbox[2] = {64, 128};
  const uint64_t wdim[2] = {(uint64_t)a.rank, (uint64_t)a.vocab};
  const uint64_t wstr[1] = {(uint64_t)a.rank * 2};
  if (!encode_tensor_map(&maps.w2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w2, wdim, wstr, wbox,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const uint32_t rbox[2] = {64, 1};
  if (!encode_tensor_map(&maps.w1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w1, wdim, wstr, rbox,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const uint64_t udim[3] = {(uint64_t)a.vocab, (uint64_t)a.steps, (uint64_t)a.batch};
  const uint64_t ustr[2] = {(uint64_t)a.vocab * 2, (uint64_t)a.vocab * 2 * (uint64_t)a.steps};
  const uint32_t ubox[3] = {(uint32_t)kBV, 1u, (uint32_t)a.batch};
  if (!encode_tensor_map(&maps.u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.base, udim, ustr, ubox,
                         CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tensor_map(&maps.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.corrected, udim, ustr, ubox,
                         CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;

  SampleParams p{};
  p.first_prev = a.first_prev;
  p.w1 = static_cast<const __nv_bfloat16*>(a.w1);
  p.w2 = static_cast<const __nv_bfloat16*>(a.w2);
  p.tokens = a.tokens;
  p.keys = a.keys;
  p.barrier = a.barrier;
  p.status = a.status;
  p.batch = (int32_t)a.batch;
  p.batch_pad = BB;
  p.steps = (int32_t)a.steps;
  p.rank = a.rank;
  p.vocab = a.vocab;
  p.vocab_tiles = tiles;
  p.smem_tiles = c.smem_tiles;
  p.u_slots = c.u_slots;
  p.u_slot_bytes = c.u_slot_bytes;
  p.x_bytes = c.x_bytes;
  p.temperature = a.temperature;
  p.round_keys = round_keys_for(a.seed);
  p.wait_limit_ns = a.wait_limit_ns;
  p.debug_flags = a.debug_flags;
  p.groups = c.groups;

  cudaError_t e = cudaFuncSetAttribute(tc_sample_kernel<KA, GREEDY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)c.smem_bytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = c.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, tc_sample_kernel<KA, GREEDY>, maps, p);
  note_launch();
  return e;
}

template <bool GREEDY>
cudaError_t launch_mode(const TcSampleArgs& a, int num_sms, cudaStream_t s) {
  switch (a.rank / 64) {
    case 1: return launch_ka<1, GREEDY>(a, num_sms, s);
    case 2: return launch_ka<2, GREEDY>(a, num_sms, s);
    case 3: return launch_ka<3, GREEDY>(a, num_sms, s);
    case 4: return launch_ka<4, GREEDY>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

namespace {

bool tile_sample_supported(int64_t batch, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype,
                           int num_sms) {
  if (logits_dtype != DSPARK_DTYPE_BF16 || weight_dtype != DSPARK_DTYPE_BF16) return false;
  if (vocab % 8 != 0 || rank % 64 != 0 || rank < 64 || rank > 256) return false;
  if (batch < 1 || batch > kMaxBatch) return false;
  if (vocab >= (1ll << 31) - kBV || num_sms < 1) return false;
  const int64_t tiles = (vocab + kBV - 1) / kBV;
  const int64_t grid = tiles < num_sms ? tiles : num_sms;
  const int64_t per_cta = (tiles + grid - 1) / grid;
  // The greedy key keeps a CTA-local vocabulary index in 16 bits, and W2 must
  // fit on chip (shared plus tensor memory) for the whole launch.
  if (per_cta * kBV > 65536) return false;
  return plan(rank / 64, (int)batch, batch_pad_of(batch), (int)per_cta).ok;
}

}  // namespace

bool tc_sample_supported(int64_t batch, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype,
                         int num_sms) {
  return tc_sample_rows_supported(batch, vocab, rank, logits_dtype, weight_dtype, num_sms) ||
         tile_sample_supported(batch, vocab, rank, logits_dtype, weight_dtype, num_sms);
}

// This file's tile kernel (vocabulary ids on the MMA's M side, batch up to
// 256) or the row-layout kernel (batch up to 64). Unforced, temperature
// sampling takes the row layout and greedy decoding the tile layout: on the
// V = 129280 .. 151936 shapes the row layout's epilogue spreads the Philox
// and Gumbel arithmetic over all its threads and wins, while the greedy
// chain is shorter in the tile layout.
cudaError_t launch_tc_sample(const TcSampleArgs& a, int num_sms, cudaStream_t s, int layout, int* variant) {
  const bool rows_ok = tc_sample_rows_supported(a.batch, a.vocab, a.rank, DSPARK_DTYPE_BF16, DSPARK_DTYPE_BF16, num_sms);
  const bool tile_ok = tile_sample_supported(a.batch, a.vocab, a.rank, DSPARK_DTYPE_BF16, DSPARK_DTYPE_BF16, num_sms);
  const bool want_rows = layout == kSampleRows || (layout == kSampleAuto && !a.greedy);
  if (rows_ok && (want_rows || !tile_ok)) {
    *variant |= DSPARK_VARIANT_SAMPLE_ROWS;
    return launch_tc_sample_rows(a, num_sms, s);
  }
  return a.greedy ? launch_mode<true>(a, num_sms, s) : launch_mode<false>(a, num_sms, s);
}

}  // namespace dspark
