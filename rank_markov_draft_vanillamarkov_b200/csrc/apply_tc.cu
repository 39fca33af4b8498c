// Teacher-forced corrected logits on the sm_100a tensor cores
// (VanillaMarkov.apply_block_logits of the vendored markov_head.py):
//
//     out[i, v] = round_bf16( U[i, v] + sum_j W1[prev_i, j] * W2[v, j] )
//
// One persistent CTA per SM walks a contiguous run of 128-row x 128-id output
// tiles ("units"). The gathered rows W1[prev] (the MMA's A operand, [128 rows
// x rank]) live in tensor memory, loaded with tcgen05.st by four gather
// warps. When every row tile fits there (at rank 128 up to 512 rows) they stay
// for the whole launch and the units go vocab-tile major: all row tiles of one
// vocab tile, then the next, so each W2 tile [128 ids x rank] is loaded by TMA
// once and stays in shared memory while the CTA walks that tile's rows.
// Otherwise A is double-buffered and the units go row-tile major, so that a
// row tile is gathered once per CTA and the W2 tiles stream from L2 through a
// ring of atoms; where the grid allows, the CTAs of all row tiles sweep the
// vocabulary in lockstep so that each W2 tile leaves DRAM about once (see
// unit_coords). Shared memory holds only W2 and a deep ring of U tiles, which
// is what keeps enough HBM reads in flight.
//
// Warp roles (512 threads):
//   warp 0       TMA producer: W2 tiles (vocab-tile major) and U tiles (two 64-id boxes of 128
//                rows each, 128-byte swizzle) into rings.
//   warp 1       owns tensor memory (512 columns); lane 0 issues
//                tcgen05.mma.kind::f16 with A in TMEM and B = the W2 tile in
//                shared memory (M = 128, N = 128, K = 16 per instruction).
//   warp 2       row-tile major only: each unit's W2 tile, one 128-id x 64-rank
//                atom at a time, into a ring of atoms.
//   warps 4-7    gather W1[prev] rows into TMEM (warp w owns lanes 32*(w%4)).
//   warps 8-11   epilogue group 0, warps 12-15 group 1: tcgen05.ld of the
//                fp32 accumulator (thread = row; the two accumulators
//                alternate between units), add the U tile in place in shared
//                memory, round to bf16, TMA-store the tile. Vocab-tile major:
//                group g takes the units of parity g; row-tile major: both
//                take every unit, group g ids [64 g, 64 g + 64).
//
// Tensor memory: columns [0,128) and [128,256) are the two accumulators,
// [256,512) holds A (rank/2 columns per 128-row tile; two bf16 per column).
//
// Every wait is bounded (WaitCtl); a wait that runs out sets the TIMEOUT bit
// of the status word and the CTA winds down without faulting.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace dspark {
namespace {

constexpr int kBM = 128;              // rows per unit (MMA M)
constexpr int kBN = 128;              // vocabulary ids per unit (MMA N)
constexpr int kAtomK = 64;            // bf16 elements in one 128-byte swizzle row
constexpr int kAtomBytes = 128 * 128; // one 128-row x 64-element W2 atom / one U box (128-byte rows)
// A U stage holds one unit, 128 rows x 128 ids: two boxes of 64 bf16 ids, or
// four boxes of 32 fp32 ids (every box row is 128 bytes).
__host__ __device__ constexpr int u_stage_bytes(bool f32) { return (f32 ? 4 : 2) * kAtomBytes; }
constexpr int kThreads = 512;
constexpr int kTmemCols = 512;
constexpr int kAccCols = 2 * kBN;     // accumulators occupy [0, 256)
constexpr int kMaxStages = 8;
constexpr int kMaxResidentTiles = 8;
constexpr int kMaxW2Slots = 8;
constexpr size_t kSmemLimit = 232448;

struct __align__(64) ApplyMaps {
  CUtensorMap u;    // [rows, vocab] bf16, box 64 x 128, 128B swizzle
  CUtensorMap out;  // same geometry as u
  CUtensorMap w2;   // [vocab, rank] bf16, box 64 x 128, 128B swizzle
};

struct ApplyParams {
  const int64_t* ids;
  const __nv_bfloat16* w1;
  int64_t rows, vocab;
  int32_t rank;
  int32_t row_tiles, vocab_tiles;
  int32_t w2_slots, u_stages;  // W2 blocks in the ring (a whole tile each, or one atom when row-major)
  int32_t resident;  // all row tiles of A stay in tensor memory
  int32_t row_major; // units walk the vocabulary tiles of one row tile, then the next
  int32_t lock_q;    // >0 (row-tile major only): CTA c takes row tile c / lock_q and vocabulary tiles
                     // c % lock_q, c % lock_q + lock_q, ...: every row tile sweeps the vocabulary in step
  uint32_t* status;
  uint64_t wait_limit_ns;
};

struct SharedTail {
  uint64_t w2_full[kMaxW2Slots], w2_empty[kMaxW2Slots];
  uint64_t a_full[kMaxResidentTiles], a_empty[2];
  uint64_t u_full[kMaxStages], u_empty[kMaxStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
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

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t add_round_pair(uint32_t u2, uint32_t acc_lo, uint32_t acc_hi) {
  __nv_bfloat162 u = *reinterpret_cast<__nv_bfloat162*>(&u2);
  const float2 f = __bfloat1622float2(u);
  __nv_bfloat162 o = __floats2bfloat162_rn(f.x + __uint_as_float(acc_lo), f.y + __uint_as_float(acc_hi));
  return *reinterpret_cast<uint32_t*>(&o);
}

// A warp-uniform bounded wait: lane 0 waits, the warp follows its verdict, and
// the other lanes then observe the (already completed) phase themselves.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, int lane) {
  bool ok = lane == 0 ? mbar_wait(bar, parity, ctl) : true;
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok && lane != 0) mbar_wait(bar, parity, ctl);
  return ok;
}

// Unit u's row tile m and vocabulary tile n. Vocab-tile major (all row tiles
// of a vocabulary tile, then the next) shares each W2 tile between row tiles;
// row-tile major shares each A tile between vocabulary tiles, which is what
// counts when A does not stay in tensor memory and must be gathered again
// whenever the row tile changes.
//
// Lockstep (row-tile major with lock_q CTAs per row tile): the i-th unit of
// CTA c is (row tile c / lock_q, vocabulary tile c % lock_q + i lock_q), so
// at any moment every row tile's CTAs work on the same few vocabulary tiles
// and each streamed W2 tile comes from DRAM about once, then from L2. With
// contiguous unit ranges the row tiles reached a W2 tile at times far apart
// and it was read from DRAM several times over (264 MB extra at 2560 rows).
__device__ __forceinline__ void unit_coords(const ApplyParams& p, int64_t u, int32_t& n, int32_t& m) {
  if (p.lock_q > 0) {
    m = (int32_t)(blockIdx.x / p.lock_q);
    n = (int32_t)(blockIdx.x % p.lock_q + u * p.lock_q);
  } else if (p.row_major) {
    m = (int32_t)(u / p.vocab_tiles);
    n = (int32_t)(u % p.vocab_tiles);
  } else {
    n = (int32_t)(u / p.row_tiles);
    m = (int32_t)(u % p.row_tiles);
  }
}

// One 128-row tile of A into tensor memory: thread `row` loads W1[prev] (rank
// bf16 = rank/2 32-bit words) and stores it to its own TMEM lane, columns
// [col, col + rank/2), eight words per 16-byte load.
template <int KA>
__device__ __forceinline__ void gather_tile_to_tmem(const ApplyParams& p, int m, int row, uint32_t taddr) {
  const int64_t grow = (int64_t)m * kBM + row;
  int64_t id = -1;
  if (grow < p.rows) {
    id = p.ids[grow];
    if (id < 0 || id >= p.vocab) {
      report_status(p.status, DSPARK_STATUS_TOKEN_RANGE);
      id = -1;
    }
  }
  __syncwarp();  // tcgen05.st below is warp-aligned
  const uint4* src = reinterpret_cast<const uint4*>(p.w1 + (id < 0 ? 0 : id) * p.rank);
#pragma unroll
  for (int c = 0; c < KA; ++c) {  // 64 bf16 = 32 words = 8 loads per chunk
    uint32_t w[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 x = id >= 0 ? ld_nc_v4(src + c * 8 + i) : make_uint4(0u, 0u, 0u, 0u);
      w[4 * i + 0] = x.x;
      w[4 * i + 1] = x.y;
      w[4 * i + 2] = x.z;
      w[4 * i + 3] = x.w;
    }
    tmem_st_32x32b_x32(taddr + c * 32, w);
  }
  tmem_st_wait();
}

// HAS_BASE false: no U (the bias alone, rounded once): the producer loads no
// U tile and the epilogue adds zero, using the stage only to assemble the
// output tile for its TMA store. F32: fp32 logits (U and out); the bias is
// added in fp32, which is the one rounding.
template <int KA, bool HAS_BASE, bool F32>
__global__ void __launch_bounds__(kThreads, 1)
    tc_apply_kernel(const __grid_constant__ ApplyMaps maps, const ApplyParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* w2_smem = smem;  // w2_slots blocks of KA atoms (vocab-tile major) or of one atom (row-tile major)
  constexpr int kUStageBytes = u_stage_bytes(F32);
  constexpr int kBoxIds = F32 ? 32 : 64;  // ids per 128-byte box row
  const int w2_block_atoms = p.row_major ? 1 : KA;
  uint8_t* u_smem = w2_smem + (size_t)p.w2_slots * w2_block_atoms * kAtomBytes;  // u_stages x kUStageBytes
  SharedTail* sh = reinterpret_cast<SharedTail*>(u_smem + (size_t)p.u_stages * kUStageBytes);

  constexpr int kACols = KA * 32;  // TMEM columns of one A tile
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t units = (int64_t)p.row_tiles * p.vocab_tiles;
  // Lockstep: this CTA's units are numbered 0 .. count - 1 (see unit_coords).
  const int64_t u_begin = p.lock_q > 0 ? 0 : units * blockIdx.x / gridDim.x;
  const int64_t u_end = p.lock_q > 0 ? (p.vocab_tiles - (int64_t)(blockIdx.x % p.lock_q) + p.lock_q - 1) / p.lock_q
                                     : units * (blockIdx.x + 1) / gridDim.x;
  const int MT = p.row_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxW2Slots; ++i) {
      mbar_init(&sh->w2_full[i], 1);
      mbar_init(&sh->w2_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh->a_empty[i], 1);
      mbar_init(&sh->acc_full[i], 1);
      mbar_init(&sh->acc_empty[i], p.row_major ? 8 : 4);  // the warps that read it
    }
    for (int i = 0; i < kMaxResidentTiles; ++i) mbar_init(&sh->a_full[i], 4);  // one arrival per gather warp
    for (int i = 0; i < p.u_stages; ++i) {
      mbar_init(&sh->u_full[i], 1);
      mbar_init(&sh->u_empty[i], p.row_major ? 2 : 1);  // the groups that store from it
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
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      prefetch_tensormap(&maps.u);
      prefetch_tensormap(&maps.w2);
      prefetch_tensormap(&maps.out);
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int64_t cur_n = -1;
      uint32_t w2_loads = 0;
      uint32_t fills[kMaxStages];
      for (int i = 0; i < kMaxStages; ++i) fills[i] = 0;
      int64_t it = 0;
      for (int64_t u = u_begin; u < u_end; ++u, ++it) {
        int32_t n, m;
        unit_coords(p, u, n, m);
        if (!p.row_major && n != cur_n) {  // (row-tile major: warp 2 streams W2)
          const int ws = (int)(w2_loads % p.w2_slots);
          if (!mbar_wait(&sh->w2_empty[ws], ((w2_loads / p.w2_slots) & 1u) ^ 1u, ctl)) break;
          mbar_arrive_expect_tx(&sh->w2_full[ws], KA * kAtomBytes);
#pragma unroll
          for (int ka = 0; ka < KA; ++ka)
            tma_load_2d(w2_smem + (ws * KA + ka) * kAtomBytes, &maps.w2, &sh->w2_full[ws], ka * kAtomK, n * kBN,
                        pol_keep);
          ++w2_loads;
          cur_n = n;
        }
        const int s = (int)(it % p.u_stages);
        if (!mbar_wait(&sh->u_empty[s], ((uint32_t)(it / p.u_stages) & 1u) ^ 1u, ctl)) break;
        if constexpr (HAS_BASE) {
          mbar_arrive_expect_tx(&sh->u_full[s], kUStageBytes);
          uint8_t* st = u_smem + s * kUStageBytes;
#pragma unroll
          for (int bx = 0; bx < kUStageBytes / kAtomBytes; ++bx)
            tma_load_2d(st + bx * kAtomBytes, &maps.u, &sh->u_full[s], n * kBN + bx * kBoxIds, m * kBM, pol_stream);
        } else {
          mbar_arrive(&sh->u_full[s]);  // the stage is free for the epilogue
        }
        ++fills[s];
      }
      // Wait (bounded, even after an abort) for every copy this thread
      // started before the CTA may exit.
      for (int s = 0; s < p.u_stages; ++s)
        if (fills[s]) mbar_wait(&sh->u_full[s], (fills[s] - 1) & 1u, drain_ctl);
      for (uint32_t j = (w2_loads > (uint32_t)p.w2_slots ? w2_loads - p.w2_slots : 0); j < w2_loads; ++j)
        mbar_wait(&sh->w2_full[j % p.w2_slots], (j / p.w2_slots) & 1u, drain_ctl);
    }
  } else if (warp == 2) {
    // ------------------------- W2 ring producer (row-tile major) ----
    // A new W2 tile every unit, atom by atom through the ring, so the next
    // unit's atoms load as soon as this unit's MMAs release theirs, whatever
    // the U ring is waiting for.
    if (lane == 0 && p.row_major) {
      const uint64_t pol_keep = policy_evict_last();
      uint32_t w2_loads = 0;
      bool ok = true;
      for (int64_t u = u_begin; u < u_end && ok; ++u) {
        int32_t n, m;
        unit_coords(p, u, n, m);
        for (int ka = 0; ka < KA; ++ka, ++w2_loads) {
          const int ws = (int)(w2_loads % p.w2_slots);
          ok = mbar_wait(&sh->w2_empty[ws], ((w2_loads / p.w2_slots) & 1u) ^ 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(&sh->w2_full[ws], kAtomBytes);
          tma_load_2d(w2_smem + ws * kAtomBytes, &maps.w2, &sh->w2_full[ws], ka * kAtomK, n * kBN, pol_keep);
        }
      }
      for (uint32_t j = (w2_loads > (uint32_t)p.w2_slots ? w2_loads - p.w2_slots : 0); j < w2_loads; ++j)
        mbar_wait(&sh->w2_full[j % p.w2_slots], (j / p.w2_slots) & 1u, drain_ctl);
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      const uint32_t w2_addr = smem_u32(w2_smem);
      int64_t cur_n = -1;
      uint32_t w2_uses = 0;
      int ws = 0;
      int64_t it = 0;
      int32_t cur_m = -1;
      uint32_t a_seq = 0;  // row tiles gathered so far (double-buffered A)
      for (int64_t u = u_begin; u < u_end; ++u, ++it) {
        int32_t n, m;
        unit_coords(p, u, n, m);
        if (m != cur_m) {
          ++a_seq;
          cur_m = m;
        }
        if (!p.row_major && n != cur_n) {
          ws = (int)(w2_uses % p.w2_slots);
          if (!mbar_wait(&sh->w2_full[ws], (w2_uses / p.w2_slots) & 1u, ctl)) break;
          ++w2_uses;
          cur_n = n;
        }
        const int abuf = (int)(it & 1);
        if (!mbar_wait(&sh->acc_empty[abuf], ((uint32_t)(it >> 1) & 1u) ^ 1u, ctl)) break;
        const int aslot = p.resident ? m : (int)((a_seq - 1) & 1u);
        const uint32_t apar = p.resident ? 0u : ((a_seq - 1) >> 1) & 1u;
        if (!mbar_wait(&sh->a_full[aslot], apar, ctl)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * kBN);
        const uint32_t a_tmem = tmem_base + (uint32_t)(kAccCols + aslot * kACols);
        if (p.row_major) {
          bool ok = true;
          for (int ka = 0; ka < KA; ++ka, ++w2_uses) {
            const int wr = (int)(w2_uses % p.w2_slots);
            if (!mbar_wait(&sh->w2_full[wr], (w2_uses / p.w2_slots) & 1u, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint64_t bd0 = sw128_kmajor_desc(w2_addr + wr * kAtomBytes);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              umma_bf16_ts(d_tmem, a_tmem + (ka * 4 + k4) * 8, desc_advance(bd0, k4 * 32), idesc, (ka | k4) != 0);
            umma_commit(&sh->w2_empty[wr]);
          }
          if (!ok) break;
        } else {
#pragma unroll
          for (int kk = 0; kk < KA * kAtomK / 16; ++kk) {
            const uint64_t bd = sw128_kmajor_desc(w2_addr + (ws * KA + (kk >> 2)) * kAtomBytes + (kk & 3) * 32);
            umma_bf16_ts(d_tmem, a_tmem + kk * 8, bd, idesc, kk != 0);
          }
        }
        umma_commit(&sh->acc_full[abuf]);
        int32_t next_n = -1, next_m = -1;
        if (u + 1 < u_end) unit_coords(p, u + 1, next_n, next_m);
        if (!p.resident && next_m != m) umma_commit(&sh->a_empty[aslot]);
        if (!p.row_major && next_n != n) umma_commit(&sh->w2_empty[ws]);
      }
      // All MMAs issued by this thread are complete once `drain` flips.
      umma_commit(&sh->drain);
      mbar_wait(&sh->drain, 0, drain_ctl);
    }
  } else if (warp >= 4 && warp < 8) {
    // --------------------------------------- W1 gather into TMEM -------
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(32 * q) << 16);
    if (p.resident) {
      // Every row tile, starting with the one this CTA's first unit needs.
      int32_t n0 = 0, m0 = 0;
      if (u_begin < u_end) unit_coords(p, u_begin, n0, m0);
      for (int i = 0; i < MT; ++i) {
        const int m = (m0 + i) % MT;
        gather_tile_to_tmem<KA>(p, m, row, lane_base + kAccCols + m * kACols);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->a_full[m]);
      }
    } else {
      // A new tile whenever the row tile changes, into the free buffer.
      int32_t cur_m = -1;
      uint32_t a_seq = 0;
      for (int64_t u = u_begin; u < u_end; ++u) {
        int32_t n, m;
        unit_coords(p, u, n, m);
        if (m == cur_m) continue;
        cur_m = m;
        const int aslot = (int)(a_seq & 1u);
        if (!warp_wait(&sh->a_empty[aslot], ((a_seq >> 1) & 1u) ^ 1u, ctl, lane)) break;
        tc_fence_after_sync();
        gather_tile_to_tmem<KA>(p, m, row, lane_base + kAccCols + aslot * kACols);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->a_full[aslot]);
        ++a_seq;
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------- epilogue -------
    // Vocab-tile major: group g takes the units of parity g whole (the two
    // groups' per-unit waits and stores overlap). Row-tile major: both groups
    // take every unit, group g its ids [64 g, 64 g + 64), and the accumulator
    // goes back to the MMA warp right after the tensor-memory loads (there,
    // each unit waits for a freshly streamed W2 tile, and this halves the
    // time an accumulator is held).
    const bool split = p.row_major != 0;
    const int g = (warp - 8) >> 2;               // group
    const int et = threadIdx.x - 256 - 128 * g;  // 0..127 within the group
    const int q = warp & 3;                      // TMEM lane quarter this warp may access
    const int row = 32 * q + lane;
    const uint32_t bar_id = 1 + g;
    const int h0 = split ? g : 0, h1 = split ? g + 1 : 2;  // 64-id halves of the unit this group adds
    constexpr int kHalfBoxes = kUStageBytes / kAtomBytes / 2;
    const int64_t step = split ? 1 : 2;
    int64_t it = split ? 0 : g;
    for (int64_t u = u_begin + it; u < u_end; u += step, it += step) {
      int32_t n, m;
      unit_coords(p, u, n, m);
      const int s = (int)(it % p.u_stages);
      const int abuf = (int)(it & 1);
      const uint32_t acc_par = (uint32_t)(it >> 1) & 1u;
      const uint32_t u_par = (uint32_t)(it / p.u_stages) & 1u;
      bool ok = true;
      if (et == 0) ok = mbar_wait(&sh->acc_full[abuf], acc_par, ctl) && mbar_wait(&sh->u_full[s], u_par, ctl);
      __syncwarp();
      if (!barrier_and(ok, bar_id, 128)) break;
      if (et != 0) {
        mbar_wait(&sh->acc_full[abuf], acc_par, ctl);
        mbar_wait(&sh->u_full[s], u_par, ctl);
      }
      __syncwarp();  // tcgen05.ld below is warp-aligned
      tc_fence_after_sync();
      uint8_t* st = u_smem + s * kUStageBytes;
      const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(abuf * kBN);
      // A lane quarter that holds only rows past the end (the ragged last row
      // tile) has nothing to add: its rows are not stored.
      const bool live = (int64_t)m * kBM + 32 * q < p.rows;
      for (int h = h0; h < h1; ++h) {
        uint32_t acc[64];
        if (live) {
          tmem_ld_32x32b_x32(tbase + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&acc[0]));
          tmem_ld_32x32b_x32(tbase + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&acc[32]));
          tmem_ld_wait();
        }
        if (split) {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->acc_empty[abuf]);
        }
        if (!live) continue;
        if constexpr (F32) {
          // The half's 64 ids are boxes 2h and 2h+1, 32 fp32 each: chunk c
          // of a box row holds ids 4c .. 4c+3.
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            uint8_t* box = st + (2 * h + sub) * kAtomBytes + row * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float4* ptr = reinterpret_cast<float4*>(box + ((c ^ (row & 7)) << 4));
              float4 x = HAS_BASE ? *ptr : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              const uint32_t* a4 = &acc[sub * 32 + c * 4];
              x.x += __uint_as_float(a4[0]);
              x.y += __uint_as_float(a4[1]);
              x.z += __uint_as_float(a4[2]);
              x.w += __uint_as_float(a4[3]);
              *ptr = x;
            }
          }
        } else {
          uint8_t* box = st + h * kAtomBytes + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4* ptr = reinterpret_cast<uint4*>(box + ((c ^ (row & 7)) << 4));
            uint4 x = HAS_BASE ? *ptr : make_uint4(0u, 0u, 0u, 0u);
            x.x = add_round_pair(x.x, acc[c * 8 + 0], acc[c * 8 + 1]);
            x.y = add_round_pair(x.y, acc[c * 8 + 2], acc[c * 8 + 3]);
            x.z = add_round_pair(x.z, acc[c * 8 + 4], acc[c * 8 + 5]);
            x.w = add_round_pair(x.w, acc[c * 8 + 6], acc[c * 8 + 7]);
            *ptr = x;
          }
        }
      }
      if (!split) {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->acc_empty[abuf]);
      }
      __syncwarp();
      fence_proxy_async_smem();
      named_barrier_sync(bar_id, 128);
      if (et == 0) {
        for (int bx = h0 * kHalfBoxes; bx < h1 * kHalfBoxes; ++bx)
          tma_store_2d(&maps.out, st + bx * kAtomBytes, n * kBN + bx * kBoxIds, m * kBM);
        bulk_commit_group();
        bulk_wait_group_read<0>();  // the stage may be refilled once its stores have read it
        mbar_arrive(&sh->u_empty[s]);
      }
      __syncwarp();
    }
    if (et == 0) bulk_wait_group<0>();
  }

  // Single-lane roles and lane-0 branches leave warps diverged; bar.sync is
  // warp-aligned, so every warp reconverges first.
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

struct ApplyConfig {
  int w2_slots, u_stages, resident, row_major;
  size_t smem_bytes;
};

ApplyConfig plan(int ka, int row_tiles, bool f32) {
  const int kUStageBytes = u_stage_bytes(f32);
  ApplyConfig c{};
  c.resident = (row_tiles <= kMaxResidentTiles && row_tiles * ka * 32 <= kTmemCols - kAccCols) ? 1 : 0;
  const size_t fixed = 1024 + sizeof(SharedTail) + 64;
  auto stages_for = [&](int slots) {
    const int st = (int)((kSmemLimit - fixed - (size_t)slots * ka * kAtomBytes) / kUStageBytes);
    return st > kMaxStages ? kMaxStages : st;
  };
  // Row-tile major streams W2 through a ring of single atoms: four U stages
  // (three where four leave no room for two atoms) and the rest of shared
  // memory for the ring. On 2560 rows at rank 256 that split (six atoms)
  // measured 309 us, against 313 us with three stages and eight atoms and
  // 328 us with five stages and four atoms: the next tile's W2 atoms need
  // to be in flight while the current tile's are still in use.
  int ring_stages = 4;
  while (ring_stages > 3 && fixed + (size_t)ring_stages * kUStageBytes + 2 * (size_t)kAtomBytes > kSmemLimit)
    --ring_stages;
  int ring = (int)((kSmemLimit - fixed - (size_t)ring_stages * kUStageBytes) / kAtomBytes);
  if (ring > kMaxW2Slots) ring = kMaxW2Slots;
  if (!c.resident && ring >= 2 && fixed + (size_t)ring_stages * kUStageBytes + (size_t)ring * kAtomBytes <= kSmemLimit) {
    c.row_major = 1;
    c.w2_slots = ring;
    c.u_stages = ring_stages;
    c.smem_bytes = fixed + (size_t)ring * kAtomBytes + (size_t)c.u_stages * kUStageBytes;
    return c;
  }
  // Vocab-tile major: two W2 slots hide the reload at a vocab-tile change,
  // which comes every row_tiles units; with many row tiles, or where two
  // slots leave fewer than three U stages, one slot leaves room for more U.
  c.row_major = 0;
  c.w2_slots = (row_tiles < 8 && stages_for(2) >= 3) ? 2 : 1;
  c.u_stages = stages_for(c.w2_slots);
  c.smem_bytes = fixed + (size_t)c.w2_slots * ka * kAtomBytes + (size_t)c.u_stages * kUStageBytes;
  return c;
}

template <int KA>
cudaError_t launch_ka(const TcApplyArgs& a, int num_sms, cudaStream_t stream) {
  ApplyMaps maps;
  const bool f32 = a.logits_f32 != 0;
  const CUtensorMapDataType ldt = f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t ldim[2] = {(uint64_t)a.vocab, (uint64_t)a.rows};
  const uint64_t lstr[1] = {(uint64_t)a.vocab * (f32 ? 4 : 2)};
  const uint32_t ubox[2] = {f32 ? 32u : 64u, 128};  // 128-byte rows
  const uint32_t lbox[2] = {64, 128};
  const bool has_base = a.base != nullptr;
  // Without a base the U map is never read; it is encoded on `out` to stay valid.
  if (!encode_tensor_map(&maps.u, ldt, 2, has_base ? a.base : a.out, ldim, lstr, ubox, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&maps.out, ldt, 2, a.out, ldim, lstr, ubox, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const uint64_t wdim[2] = {(uint64_t)a.rank, (uint64_t)a.vocab};
  const uint64_t wstr[1] = {(uint64_t)a.rank * 2};
  if (!encode_tensor_map(&maps.w2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w2, wdim, wstr, lbox,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  ApplyParams p{};
  p.ids = a.ids;
  p.w1 = static_cast<const __nv_bfloat16*>(a.w1);
  p.rows = a.rows;
  p.vocab = a.vocab;
  p.rank = a.rank;
  p.row_tiles = (int32_t)((a.rows + kBM - 1) / kBM);
  p.vocab_tiles = (int32_t)((a.vocab + kBN - 1) / kBN);
  const ApplyConfig c = plan(KA, p.row_tiles, f32);
  p.w2_slots = c.w2_slots;
  p.u_stages = c.u_stages;
  p.resident = c.resident;
  p.row_major = c.row_major;
  // Lockstep when its grid (row tiles x CTAs per row tile) still fills at
  // least 90 % of the SMs: 2560 rows (20 row tiles) run on 140 CTAs, and
  // that measured 319 us against 358 us with contiguous unit ranges on 148.
  p.lock_q = 0;
  if (c.row_major && p.row_tiles <= num_sms) {
    int q = num_sms / p.row_tiles;
    if (q > p.vocab_tiles) q = p.vocab_tiles;
    if ((int64_t)p.row_tiles * q * 10 >= (int64_t)num_sms * 9) p.lock_q = q;
  }
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;

  auto kernel = f32 ? (has_base ? tc_apply_kernel<KA, true, true> : tc_apply_kernel<KA, false, true>)
                    : (has_base ? tc_apply_kernel<KA, true, false> : tc_apply_kernel<KA, false, false>);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)c.smem_bytes);
  if (e != cudaSuccess) return e;
  const int64_t units = (int64_t)p.row_tiles * p.vocab_tiles;
  const int grid = p.lock_q > 0 ? p.row_tiles * p.lock_q : (int)(units < num_sms ? units : num_sms);
  kernel<<<grid, kThreads, c.smem_bytes, stream>>>(maps, p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool tc_apply_supported(int64_t rows, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype) {
  // bf16 weights; logits bf16 or fp32 (fp32 logits with a bf16 head).
  if (weight_dtype != DSPARK_DTYPE_BF16) return false;
  if (logits_dtype != DSPARK_DTYPE_BF16 && logits_dtype != DSPARK_DTYPE_FP32) return false;
  if (vocab % 8 != 0 || rank % 64 != 0 || rank < 64 || rank > 256) return false;
  const int64_t row_tiles = (rows + kBM - 1) / kBM;
  const int64_t vocab_tiles = (vocab + kBN - 1) / kBN;
  // TMA coordinates are signed 32-bit.
  return row_tiles * kBM < (1ll << 31) && vocab_tiles * kBN < (1ll << 31);
}

cudaError_t launch_tc_apply(const TcApplyArgs& a, int num_sms, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  switch (a.rank / 64) {
    case 1: return launch_ka<1>(a, num_sms, s);
    case 2: return launch_ka<2>(a, num_sms, s);
    case 3: return launch_ka<3>(a, num_sms, s);
    case 4: return launch_ka<4>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dspark
