// Teacher-forced corrected logits on the sm_100a tensor cores, 256 ids per
// MMA (VanillaMarkov.apply_block_logits of the vendored markov_head.py):
//
//     out[i, v] = round_bf16( U[i, v] + sum_j W1[prev_i, j] * W2[v, j] )
//
// This kernel takes units of 128 rows x 256 ids: half the MMA instructions of
// the 128-id kernel (apply_tc.cu), and half the W1 row gathers where the rows'
// W1 rows cannot stay in tensor memory for the whole launch (many row tiles
// at rank 256). It is an opt-in variant: on every workload measured here it
// is slower than the 128-id kernel, whose per-unit stages move U by TMA.
//
// Persistent CTAs walk contiguous runs of units, id-tile major (all row tiles
// of one id tile, then the next), so a W2 tile [256 ids x rank] is loaded
// once per id tile. The gathered rows W1[prev] are the MMA's A operand in
// tensor memory (TS form): resident for the launch when every row tile fits
// beside the accumulator, else double-buffered and gathered for the next unit
// while the current unit's MMAs run.
//
// Warp roles (640 threads):
//   warp 0      TMA producer: W2 tiles (rank/64 boxes of 64 x 256,
//               128-byte swizzle).
//   warp 1      tensor-memory owner and MMA issuer (M = 128, N = 256, K = 16,
//               A from tensor memory, B = the W2 tile in shared memory).
//   warps 4-19  epilogue and gather. Warp 4 + 4e + q owns TMEM lane quarter q
//               (rows 32q..32q+31) and ids [64e, 64e + 64) of the unit. Each
//               thread loads its row's 64 U values (128 bytes) straight from
//               global memory before the unit's MMAs finish, reads its 64
//               accumulator columns in two tcgen05.ld halves (handing the
//               accumulator back after the second), adds, rounds once and
//               stores the 128 bytes with streaming stores. The same warp
//               gathers columns [e r/4, (e+1) r/4) of its rows' W1 rows with
//               tcgen05.st. Shared memory holds only W2 tiles, so it can keep
//               two or three of them.
//
// Tensor memory: the accumulator in columns [0, 256), A in [256, 512) (rank/2
// columns per row tile). Every wait is bounded.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace dspark {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kAtomK = 64;
constexpr uint32_t kW2AtomBytes = kBN * 128;  // 256 ids x 64 bf16
constexpr int kEpiWarps = 16;
constexpr int kThreads = 128 + kEpiWarps * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = kBN;
constexpr int kMaxW2Slots = 3;
constexpr int kMaxResident = 8;
constexpr size_t kSmemLimit = 232448;

struct __align__(64) WideMaps {
  CUtensorMap w2;  // [vocab, rank] bf16, box 64 x 256, 128B swizzle
};

struct WideParams {
  const __nv_bfloat16* base;  // [rows, vocab]
  __nv_bfloat16* out;         // [rows, vocab]
  const int64_t* ids;
  const __nv_bfloat16* w1;
  int64_t rows, vocab;
  int32_t rank;
  int32_t row_tiles, id_tiles;
  int32_t w2_slots;
  int32_t resident;
  uint32_t* status;
  uint64_t wait_limit_ns;
};

struct WideTail {
  uint64_t w2_full[kMaxW2Slots], w2_empty[kMaxW2Slots];
  uint64_t a_full[kMaxResident], a_empty[2];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ uint32_t add_round_pair(uint32_t u2, uint32_t acc_lo, uint32_t acc_hi) {
  const float lo = __uint_as_float(u2 << 16) + __uint_as_float(acc_lo);
  const float hi = __uint_as_float(u2 & 0xFFFF0000u) + __uint_as_float(acc_hi);
  __nv_bfloat162 o = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&o);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, int lane) {
  bool ok = lane == 0 ? mbar_wait(bar, parity, ctl) : true;
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok && lane != 0) mbar_wait(bar, parity, ctl);
  return ok;
}

// This warp's share of one 128-row tile of A into tensor memory: thread `lane`
// of quarter q loads columns [e * KA * 8, (e + 1) * KA * 8) (32-bit words, two
// bf16 each) of W1[prev] for row 32q + lane and stores them to its own lane.
template <int KA>
__device__ __forceinline__ void gather_share(const WideParams& p, int m, int q, int e, int lane, uint32_t taddr) {
  const int64_t grow = (int64_t)m * kBM + 32 * q + lane;
  int64_t id = -1;
  if (grow < p.rows) {
    id = p.ids[grow];
    if (id < 0 || id >= p.vocab) {
      report_status(p.status, DSPARK_STATUS_TOKEN_RANGE);
      id = -1;
    }
  }
  // KA * 8 words per share = KA * 32 bytes = KA * 2 loads of 16 bytes.
  const uint4* src = reinterpret_cast<const uint4*>(p.w1 + (id < 0 ? 0 : id) * p.rank) + e * KA * 2;
#pragma unroll
  for (int c = 0; c < KA; ++c) {
    const uint4 x0 = id >= 0 ? ld_nc_v4(src + 2 * c) : make_uint4(0u, 0u, 0u, 0u);
    const uint4 x1 = id >= 0 ? ld_nc_v4(src + 2 * c + 1) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    __syncwarp();  // tcgen05.st is warp-aligned
    tmem_st_32x32b_x8(taddr + (uint32_t)(e * KA * 8 + c * 8), w);
  }
  tmem_st_wait();
}

template <int KA>
__global__ void __launch_bounds__(kThreads, 1)
    tc_apply_wide_kernel(const __grid_constant__ WideMaps maps, const WideParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* w2_smem = smem;  // w2_slots x KA atoms
  WideTail* sh = reinterpret_cast<WideTail*>(w2_smem + (size_t)p.w2_slots * KA * kW2AtomBytes);

  constexpr uint32_t kACols = KA * 32;  // TMEM columns of one A tile
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t units = (int64_t)p.row_tiles * p.id_tiles;
  const int64_t u_begin = units * blockIdx.x / gridDim.x;
  const int64_t u_end = units * (blockIdx.x + 1) / gridDim.x;
  const int MT = p.row_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxW2Slots; ++i) {
      mbar_init(&sh->w2_full[i], 1);
      mbar_init(&sh->w2_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&sh->a_empty[i], 1);
    for (int i = 0; i < kMaxResident; ++i) mbar_init(&sh->a_full[i], kEpiWarps);
    mbar_init(&sh->acc_full, 1);
    mbar_init(&sh->acc_empty, kEpiWarps);
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_barrier_init();
  }
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
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      prefetch_tensormap(&maps.w2);
      const uint64_t pol_keep = policy_evict_last();
      int64_t cur_n = -1;
      uint32_t w2_loads = 0;
      for (int64_t u = u_begin; u < u_end; ++u) {
        const int32_t n = (int32_t)(u / MT);
        if (n == cur_n) continue;
        const int ws = (int)(w2_loads % p.w2_slots);
        if (!mbar_wait(&sh->w2_empty[ws], ((w2_loads / p.w2_slots) & 1u) ^ 1u, ctl)) break;
        mbar_arrive_expect_tx(&sh->w2_full[ws], KA * kW2AtomBytes);
#pragma unroll
        for (int ka = 0; ka < KA; ++ka)
          tma_load_2d(w2_smem + (size_t)(ws * KA + ka) * kW2AtomBytes, &maps.w2, &sh->w2_full[ws], ka * kAtomK,
                      n * kBN, pol_keep);
        ++w2_loads;
        cur_n = n;
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
      for (int64_t u = u_begin; u < u_end; ++u, ++it) {
        const int32_t n = (int32_t)(u / MT), m = (int32_t)(u % MT);
        if (n != cur_n) {
          ws = (int)(w2_uses % p.w2_slots);
          if (!mbar_wait(&sh->w2_full[ws], (w2_uses / p.w2_slots) & 1u, ctl)) break;
          ++w2_uses;
          cur_n = n;
        }
        if (!mbar_wait(&sh->acc_empty, ((uint32_t)it & 1u) ^ 1u, ctl)) break;
        const int aslot = p.resident ? m : (int)(it & 1);
        const uint32_t apar = p.resident ? 0u : (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(&sh->a_full[aslot], apar, ctl)) break;
        tc_fence_after_sync();
        const uint32_t a_tmem = tmem_base + kAccCols + (uint32_t)aslot * kACols;
#pragma unroll
        for (int kk = 0; kk < KA * kAtomK / 16; ++kk) {
          const uint64_t bd =
              sw128_kmajor_desc(w2_addr + (uint32_t)(ws * KA + (kk >> 2)) * kW2AtomBytes + (kk & 3) * 32);
          umma_bf16_ts(tmem_base, a_tmem + kk * 8, bd, idesc, kk != 0);
        }
        umma_commit(&sh->acc_full);
        if (!p.resident) umma_commit(&sh->a_empty[aslot]);
        const int64_t next_n = (u + 1 < u_end) ? (u + 1) / MT : -1;
        if (next_n != n) umma_commit(&sh->w2_empty[ws]);
      }
      umma_commit(&sh->drain);
      mbar_wait(&sh->drain, 0, drain_ctl);
    }
  } else if (warp >= 4) {
    // ---------------------------------------- gather and epilogue -----
    const int ew = warp - 4;
    const int q = ew & 3;     // TMEM lane quarter: rows 32q .. 32q + 31
    const int e = ew >> 2;    // ids [64e, 64e + 64) of the unit; W1 columns [e r/4, (e+1) r/4)
    const uint32_t lane_base = tmem_base + ((uint32_t)(32 * q) << 16);
    bool ok = true;
    // A for the first unit (or every row tile, when resident).
    if (u_begin < u_end) {
      if (p.resident) {
        for (int m = 0; m < MT; ++m) {
          gather_share<KA>(p, m, q, e, lane, lane_base + kAccCols + (uint32_t)m * kACols);
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->a_full[m]);
        }
      } else {
        gather_share<KA>(p, (int)(u_begin % MT), q, e, lane, lane_base + kAccCols);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->a_full[0]);
      }
    }
    // U rows of a unit into L2 ahead of their loads: warps of e = 0 prefetch
    // one 512-byte row range each (a row's 256 ids).
    auto prefetch_unit = [&](int64_t uu) {
      if (e != 0 || uu >= u_end) return;
      const int64_t r = (uu % MT) * kBM + 32 * q + lane;
      const int64_t i0 = (uu / MT) * kBN;
      if (r < p.rows) {
        const int64_t nid = p.vocab - i0 < kBN ? p.vocab - i0 : kBN;
        bulk_prefetch_l2(p.base + r * p.vocab + i0, (uint32_t)(nid * 2));
      }
    };
    prefetch_unit(u_begin);
    prefetch_unit(u_begin + 1);
    int64_t it = 0;
    for (int64_t u = u_begin; u < u_end && ok; ++u, ++it) {
      const int32_t n = (int32_t)(u / MT), m = (int32_t)(u % MT);
      prefetch_unit(u + 2);
      const int64_t grow = (int64_t)m * kBM + 32 * q + lane;
      const int64_t v0 = (int64_t)n * kBN + 64 * e;  // this thread's first id
      // Ids of this thread's eight 8-id chunks that exist (vocab is a
      // multiple of 8, so a chunk is wholly in or out).
      const int64_t left = p.vocab - v0;
      const int nchunk = grow < p.rows ? (left >= 64 ? 8 : (left > 0 ? (int)(left / 8) : 0)) : 0;
      // U of this unit, issued before its MMAs are awaited.
      uint4 uv[8];
      const __nv_bfloat16* src = p.base + grow * p.vocab + v0;
#pragma unroll
      for (int c = 0; c < 8; ++c) uv[c] = c < nchunk ? ld_stream_v4(src + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
      if (!p.resident && u + 1 < u_end) {
        // The next unit's rows into the other slot, once the MMAs of the unit
        // before this one have read it; the current unit's MMAs run meanwhile.
        const int ns = (int)((it + 1) & 1);
        if (!warp_wait(&sh->a_empty[ns], ((uint32_t)((it + 1) >> 1) & 1u) ^ 1u, ctl, lane)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        gather_share<KA>(p, (int)((u + 1) % MT), q, e, lane, lane_base + kAccCols + (uint32_t)ns * kACols);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->a_full[ns]);
      }
      if (!warp_wait(&sh->acc_full, (uint32_t)it & 1u, ctl, lane)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      __nv_bfloat16* dst = p.out + grow * p.vocab + v0;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t acc[32];
        __syncwarp();  // tcgen05.ld is warp-aligned
        tmem_ld_32x32b_x32(lane_base + (uint32_t)(64 * e + 32 * half), acc);
        tmem_ld_wait();
        if (half == 1) {
          // Every accumulator column of this warp is in registers.
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->acc_empty);
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = 4 * half + cc;
          if (c < nchunk) {
            const uint4 x = uv[c];
            const uint32_t* a8 = &acc[8 * cc];
            st_stream_v4(dst + 8 * c, make_uint4(add_round_pair(x.x, a8[0], a8[1]), add_round_pair(x.y, a8[2], a8[3]),
                                                 add_round_pair(x.z, a8[4], a8[5]),
                                                 add_round_pair(x.w, a8[6], a8[7])));
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

struct WidePlan {
  int w2_slots, resident;
  size_t smem;
  bool ok;
};

WidePlan wide_plan(int ka, int row_tiles) {
  WidePlan c{};
  const uint32_t a_cols = (uint32_t)ka * 32;
  c.resident = (row_tiles <= kMaxResident && (uint32_t)row_tiles * a_cols <= kTmemCols - kAccCols) ? 1 : 0;
  const size_t fixed = 1024 + sizeof(WideTail) + 64;
  const size_t w2_tile = (size_t)ka * kW2AtomBytes;
  // As many W2 slots as fit (up to three): the next id tile's W2 loads while
  // the current one is in use.
  int slots = (int)((kSmemLimit - fixed) / w2_tile);
  if (slots > kMaxW2Slots) slots = kMaxW2Slots;
  if (slots < 1) return c;
  c.w2_slots = slots;
  c.smem = fixed + (size_t)slots * w2_tile;
  c.ok = true;
  return c;
}

template <int KA>
cudaError_t launch_wide_ka(const TcApplyArgs& a, int num_sms, cudaStream_t stream) {
  WideMaps maps;
  const uint64_t wdim[2] = {(uint64_t)a.rank, (uint64_t)a.vocab};
  const uint64_t wstr[1] = {(uint64_t)a.rank * 2};
  const uint32_t wbox[2] = {64, (uint32_t)kBN};
  if (!encode_tensor_map(&maps.w2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w2, wdim, wstr, wbox,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  WideParams p{};
  p.base = static_cast<const __nv_bfloat16*>(a.base);
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.ids = a.ids;
  p.w1 = static_cast<const __nv_bfloat16*>(a.w1);
  p.rows = a.rows;
  p.vocab = a.vocab;
  p.rank = a.rank;
  p.row_tiles = (int32_t)((a.rows + kBM - 1) / kBM);
  p.id_tiles = (int32_t)((a.vocab + kBN - 1) / kBN);
  const WidePlan c = wide_plan(KA, p.row_tiles);
  if (!c.ok) return cudaErrorInvalidValue;
  p.w2_slots = c.w2_slots;
  p.resident = c.resident;
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;
  cudaError_t e =
      cudaFuncSetAttribute(tc_apply_wide_kernel<KA>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)c.smem);
  if (e != cudaSuccess) return e;
  const int64_t units = (int64_t)p.row_tiles * p.id_tiles;
  const int grid = (int)(units < num_sms ? units : num_sms);
  tc_apply_wide_kernel<KA><<<grid, kThreads, c.smem, stream>>>(maps, p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool tc_apply_wide_supported(int64_t rows, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype,
                             bool has_base) {
  if (!has_base || logits_dtype != DSPARK_DTYPE_BF16 || weight_dtype != DSPARK_DTYPE_BF16) return false;
  if (vocab % 8 != 0 || rank % 64 != 0 || rank < 64 || rank > 256) return false;
  const int64_t row_tiles = (rows + kBM - 1) / kBM;
  if (row_tiles * kBM >= (1ll << 31) || vocab + kBN >= (1ll << 31)) return false;
  return wide_plan(rank / 64, (int)(row_tiles < (1 << 30) ? row_tiles : (1 << 30))).ok;
}

cudaError_t launch_tc_apply_wide(const TcApplyArgs& a, int num_sms, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  switch (a.rank / 64) {
    case 1: return launch_wide_ka<1>(a, num_sms, s);
    case 2: return launch_wide_ka<2>(a, num_sms, s);
    case 3: return launch_wide_ka<3>(a, num_sms, s);
    case 4: return launch_wide_ka<4>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dspark
