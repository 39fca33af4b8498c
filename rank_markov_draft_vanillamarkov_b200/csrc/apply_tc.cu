// Teacher-forced corrected logits on the sm_100a tensor cores
// (VanillaMarkov.apply_block_logits of the vendored markov_head.py):
//
//     out[i, v] = round_bf16( U[i, v] + sum_j W1[prev_i, j] * W2[v, j] )
//
// One persistent CTA per SM walks a contiguous run of 128 x 128 output tiles,
// ordered vocab-tile major (all row tiles of one vocab tile, then the next), so
// the W2 tile [128 ids x rank] is loaded once per vocab tile and stays in
// shared memory while the CTA walks the row tiles.
//
// Warp roles (256 threads):
//   warp 0      TMA producer: W2 tiles and U tiles (two 64-column boxes of
//               128 rows, 128-byte swizzle) into a ring of stages.
//   warp 1      owns tensor memory; lane 0 issues tcgen05.mma
//               (M = 128 rows, N = 128 ids, K = 16 per instruction) into one
//               of two TMEM accumulators.
//   warps 2-3   gather W1[prev] rows (the A operand) into shared memory in the
//               128-byte swizzle layout. When all row tiles fit, they are
//               gathered once and stay resident.
//   warps 4-7   epilogue: tcgen05.ld the fp32 accumulator (thread = row),
//               add the U tile in place in shared memory, round to bf16, and
//               TMA-store the tile to `out`.
//
// Every wait is bounded (WaitCtl); a wait that runs out sets the TIMEOUT bit
// of the status word and the CTA winds down without faulting.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace dspark {
namespace {

constexpr int kBM = 128;              // rows per tile (MMA M)
constexpr int kBN = 128;              // vocabulary ids per tile (MMA N)
constexpr int kAtomK = 64;            // bf16 elements in one 128-byte swizzle row
constexpr int kAtomBytes = 128 * 128; // one 128-row x 64-element operand atom
constexpr int kUStageBytes = 2 * kAtomBytes;  // 128 rows x 128 ids of bf16
constexpr int kThreads = 256;
constexpr int kSlotBudget = 14;       // 16 KB slots that fit next to the barriers
constexpr int kTmemCols = 2 * kBN;    // two accumulators
constexpr int kMaxStages = 16;

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
  int32_t a_slots, u_stages;
  int32_t resident;  // all row tiles of A stay in shared memory
  uint32_t* status;
  uint64_t wait_limit_ns;
};

struct SharedTail {
  uint64_t w2_full, w2_empty, drain;
  uint64_t a_full[kMaxStages], a_empty[kMaxStages];
  uint64_t u_full[kMaxStages], u_empty[kMaxStages];
  uint64_t acc_full[2], acc_empty[2];
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
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t add_round_pair(uint32_t u2, uint32_t acc_lo, uint32_t acc_hi) {
  __nv_bfloat162 u = *reinterpret_cast<__nv_bfloat162*>(&u2);
  const float2 f = __bfloat1622float2(u);
  __nv_bfloat162 o = __floats2bfloat162_rn(f.x + __uint_as_float(acc_lo), f.y + __uint_as_float(acc_hi));
  return *reinterpret_cast<uint32_t*>(&o);
}

template <int KA>
__global__ void __launch_bounds__(kThreads, 1)
    tc_apply_kernel(const __grid_constant__ ApplyMaps maps, const ApplyParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* w2_smem = smem;
  uint8_t* a_smem = w2_smem + KA * kAtomBytes;
  uint8_t* u_smem = a_smem + p.a_slots * kAtomBytes;
  SharedTail* sh = reinterpret_cast<SharedTail*>(u_smem + p.u_stages * kUStageBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t units = (int64_t)p.row_tiles * p.vocab_tiles;
  const int64_t u_begin = units * blockIdx.x / gridDim.x;
  const int64_t u_end = units * (blockIdx.x + 1) / gridDim.x;
  const int MT = p.row_tiles;

  if (threadIdx.x == 0) {
    mbar_init(&sh->w2_full, 1);
    mbar_init(&sh->w2_empty, 1);
    mbar_init(&sh->drain, 1);
    for (int i = 0; i < p.a_slots; ++i) {
      mbar_init(&sh->a_full[i], 64);
      mbar_init(&sh->a_empty[i], 1);
    }
    for (int i = 0; i < p.u_stages; ++i) {
      mbar_init(&sh->u_full[i], 1);
      mbar_init(&sh->u_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh->acc_full[i], 1);
      mbar_init(&sh->acc_empty[i], 4);
    }
    sh->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = sh->tmem_base;
  const WaitCtl ctl{&sh->abort_flag, p.status, p.wait_limit_ns};

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
        const int32_t n = (int32_t)(u / MT), m = (int32_t)(u % MT);
        const int s = (int)(it % p.u_stages);
        if (!mbar_wait(&sh->u_empty[s], ((uint32_t)(it / p.u_stages) & 1u) ^ 1u, ctl)) break;
        mbar_arrive_expect_tx(&sh->u_full[s], kUStageBytes);
        uint8_t* st = u_smem + s * kUStageBytes;
        tma_load_2d(st, &maps.u, &sh->u_full[s], n * kBN, m * kBM, pol_stream);
        tma_load_2d(st + kAtomBytes, &maps.u, &sh->u_full[s], n * kBN + 64, m * kBM, pol_stream);
        ++fills[s];
        if (n != cur_n) {
          if (w2_loads > 0 && !mbar_wait(&sh->w2_empty, (w2_loads - 1) & 1u, ctl)) break;
          mbar_arrive_expect_tx(&sh->w2_full, KA * kAtomBytes);
#pragma unroll
          for (int ka = 0; ka < KA; ++ka)
            tma_load_2d(w2_smem + ka * kAtomBytes, &maps.w2, &sh->w2_full, ka * kAtomK, n * kBN, pol_keep);
          ++w2_loads;
          cur_n = n;
        }
      }
      // Wait (bounded, even after an abort) for every copy this thread
      // started before the CTA may exit.
      volatile int never = 0;
      const WaitCtl drain_ctl{&never, p.status, p.wait_limit_ns};
      for (int s = 0; s < p.u_stages; ++s)
        if (fills[s]) mbar_wait(&sh->u_full[s], (fills[s] - 1) & 1u, drain_ctl);
      if (w2_loads) mbar_wait(&sh->w2_full, (w2_loads - 1) & 1u, drain_ctl);
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      const uint32_t w2_addr = smem_u32(w2_smem);
      const uint32_t a_addr = smem_u32(a_smem);
      int64_t cur_n = -1;
      uint32_t w2_waits = 0;
      int64_t a_it = 0;
      int64_t it = 0;
      bool ok = true;
      for (int64_t u = u_begin; u < u_end && ok; ++u, ++it) {
        const int32_t n = (int32_t)(u / MT), m = (int32_t)(u % MT);
        if (n != cur_n) {
          if (!mbar_wait(&sh->w2_full, w2_waits & 1u, ctl)) break;
          ++w2_waits;
          cur_n = n;
        }
        const int abuf = (int)(it & 1);
        if (!mbar_wait(&sh->acc_empty[abuf], ((uint32_t)(it >> 1) & 1u) ^ 1u, ctl)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * kBN);
#pragma unroll
        for (int ka = 0; ka < KA; ++ka) {
          int slot;
          uint32_t parity;
          if (p.resident) {
            slot = m * KA + ka;
            parity = 0;
          } else {
            slot = (int)(a_it % p.a_slots);
            parity = (uint32_t)(a_it / p.a_slots) & 1u;
          }
          if (!mbar_wait(&sh->a_full[slot], parity, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < kAtomK / 16; ++kk) {
            const uint64_t ad = sw128_kmajor_desc(a_addr + slot * kAtomBytes + kk * 32);
            const uint64_t bd = sw128_kmajor_desc(w2_addr + ka * kAtomBytes + kk * 32);
            umma_bf16_ss(d_tmem, ad, bd, idesc, (ka | kk) != 0);
          }
          if (!p.resident) {
            umma_commit(&sh->a_empty[slot]);
            ++a_it;
          }
        }
        if (!ok) break;
        umma_commit(&sh->acc_full[abuf]);
        const int64_t next_n = (u + 1 < u_end) ? (u + 1) / MT : -1;
        if (next_n != n) umma_commit(&sh->w2_empty);
      }
      // All MMAs issued by this thread are complete once `drain` flips.
      umma_commit(&sh->drain);
      volatile int never = 0;
      const WaitCtl drain_ctl{&never, p.status, p.wait_limit_ns};
      mbar_wait(&sh->drain, 0, drain_ctl);
    }
  } else if (warp < 4) {
    // ------------------------------------------------ W1 gather -------
    const int gt = threadIdx.x - 64;  // 0..63
    const int rank = p.rank;
    auto gather = [&](int m, int ka, int slot) {
      uint8_t* dst = a_smem + slot * kAtomBytes;
      uint4 vals[16];
      bool bad = false;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int q = gt + 64 * i;
        const int row = q >> 3, j = q & 7;
        const int64_t grow = (int64_t)m * kBM + row;
        vals[i] = make_uint4(0u, 0u, 0u, 0u);
        if (grow < p.rows) {
          const int64_t id = p.ids[grow];
          if (id >= 0 && id < p.vocab)
            vals[i] = ld_nc_v4(p.w1 + id * rank + ka * kAtomK + j * 8);
          else
            bad = true;
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int q = gt + 64 * i;
        const int row = q >> 3, j = q & 7;
        *reinterpret_cast<uint4*>(dst + row * 128 + ((j ^ (row & 7)) << 4)) = vals[i];
      }
      if (bad) report_status(p.status, DSPARK_STATUS_TOKEN_RANGE);
      fence_proxy_async_smem();
      mbar_arrive(&sh->a_full[slot]);
    };
    if (p.resident) {
      for (int m = 0; m < MT; ++m)
        for (int ka = 0; ka < KA; ++ka) gather(m, ka, m * KA + ka);
    } else {
      int64_t a_it = 0;
      bool ok = true;
      for (int64_t u = u_begin; u < u_end && ok; ++u) {
        const int m = (int)(u % MT);
        for (int ka = 0; ka < KA; ++ka, ++a_it) {
          const int slot = (int)(a_it % p.a_slots);
          if (!mbar_wait(&sh->a_empty[slot], ((uint32_t)(a_it / p.a_slots) & 1u) ^ 1u, ctl)) {
            ok = false;
            break;
          }
          gather(m, ka, slot);
        }
      }
    }
  } else {
    // ------------------------------------------------- epilogue -------
    const int et = threadIdx.x - 128;  // = TMEM lane = row within the tile
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int row = et;
    int64_t it = 0;
    int prev_s = -1;
    for (int64_t u = u_begin; u < u_end; ++u, ++it) {
      const int32_t n = (int32_t)(u / MT), m = (int32_t)(u % MT);
      const int s = (int)(it % p.u_stages);
      const int abuf = (int)(it & 1);
      const uint32_t acc_par = (uint32_t)(it >> 1) & 1u;
      const uint32_t u_par = (uint32_t)(it / p.u_stages) & 1u;
      bool ok = true;
      if (et == 0) ok = mbar_wait(&sh->acc_full[abuf], acc_par, ctl) && mbar_wait(&sh->u_full[s], u_par, ctl);
      if (!barrier_and(ok, 1, 128)) break;
      if (et != 0) {
        mbar_wait(&sh->acc_full[abuf], acc_par, ctl);
        mbar_wait(&sh->u_full[s], u_par, ctl);
      }
      tc_fence_after_sync();
      uint8_t* st = u_smem + s * kUStageBytes;
      const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(abuf * kBN);
#pragma unroll 2
      for (int c = 0; c < kBN / 16; ++c) {
        uint32_t acc[16];
        tmem_ld_32x32b_x16(tbase + c * 16, acc);
        tmem_ld_wait();
        const int box = c >> 2;
        const int j0 = (c & 3) * 2;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4* ptr = reinterpret_cast<uint4*>(st + box * kAtomBytes + row * 128 + (((j0 + h) ^ (row & 7)) << 4));
          uint4 x = *ptr;
          x.x = add_round_pair(x.x, acc[h * 8 + 0], acc[h * 8 + 1]);
          x.y = add_round_pair(x.y, acc[h * 8 + 2], acc[h * 8 + 3]);
          x.z = add_round_pair(x.z, acc[h * 8 + 4], acc[h * 8 + 5]);
          x.w = add_round_pair(x.w, acc[h * 8 + 6], acc[h * 8 + 7]);
          *ptr = x;
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->acc_empty[abuf]);
      fence_proxy_async_smem();
      named_barrier_sync(1, 128);
      if (et == 0) {
        tma_store_2d(&maps.out, st, n * kBN, m * kBM);
        tma_store_2d(&maps.out, st + kAtomBytes, n * kBN + 64, m * kBM);
        bulk_commit_group();
        if (prev_s >= 0) {
          bulk_wait_group_read<1>();
          mbar_arrive(&sh->u_empty[prev_s]);
        }
        prev_s = s;
      }
    }
    if (et == 0) bulk_wait_group<0>();
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

struct ApplyConfig {
  int a_slots, u_stages, resident;
  size_t smem_bytes;
};

ApplyConfig plan(int ka, int row_tiles) {
  ApplyConfig c{};
  const int free_slots = kSlotBudget - ka;
  if (row_tiles * ka + 2 * 3 <= free_slots) {
    c.resident = 1;
    c.a_slots = row_tiles * ka;
    c.u_stages = (free_slots - c.a_slots) / 2;
    if (c.u_stages > 4) c.u_stages = 4;
  } else {
    c.resident = 0;
    c.u_stages = 3;
    c.a_slots = free_slots - 2 * c.u_stages;
    if (c.a_slots > kMaxStages) c.a_slots = kMaxStages;
  }
  c.smem_bytes = 1024 + (size_t)(ka + c.a_slots) * kAtomBytes + (size_t)c.u_stages * kUStageBytes + sizeof(SharedTail);
  return c;
}

template <int KA>
cudaError_t launch_ka(const TcApplyArgs& a, int num_sms, cudaStream_t stream) {
  ApplyMaps maps;
  const uint64_t ldim[2] = {(uint64_t)a.vocab, (uint64_t)a.rows};
  const uint64_t lstr[1] = {(uint64_t)a.vocab * 2};
  const uint32_t lbox[2] = {64, 128};
  if (!encode_tensor_map(&maps.u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.base, ldim, lstr, lbox,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&maps.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.out, ldim, lstr, lbox,
                         CU_TENSOR_MAP_SWIZZLE_128B))
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
  const ApplyConfig c = plan(KA, p.row_tiles);
  p.a_slots = c.a_slots;
  p.u_stages = c.u_stages;
  p.resident = c.resident;
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;

  cudaError_t e = cudaFuncSetAttribute(tc_apply_kernel<KA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)c.smem_bytes);
  if (e != cudaSuccess) return e;
  const int64_t units = (int64_t)p.row_tiles * p.vocab_tiles;
  const int grid = (int)(units < num_sms ? units : num_sms);
  tc_apply_kernel<KA><<<grid, kThreads, c.smem_bytes, stream>>>(maps, p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool tc_apply_supported(int64_t rows, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype) {
  if (logits_dtype != DSPARK_DTYPE_BF16 || weight_dtype != DSPARK_DTYPE_BF16) return false;
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
