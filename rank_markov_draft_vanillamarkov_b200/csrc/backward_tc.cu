// Gradients of the teacher-forced corrected logits on the sm_100a tensor cores
// (the training-time use of VanillaMarkov.apply_block_logits in the vendored
// markov_head.py). With G = dL/d(out) [rows, vocab] and A = W1[prev] [rows, rank]
// the gathered rows:
//
//     dW2[v, j] = sum_i G[i, v] * A[i, j]                        (DW1 = false)
//     dW1[x, j] = sum_{i : prev_i = x} sum_v G[i, v] * W2[v, j]  (DW1 = true)
//
// with NA = rank / 64 column blocks of 64.
//
// Both contract over a dimension that is the outer (strided) one of an operand
// in memory, so those operands enter the MMA MN-major: a TMA box with 128-byte
// rows of 64 consecutive M (or N) elements, one row per K index, in the
// 128-byte swizzle (instruction descriptor bits 15/16 select MN-major A/B).
// The same swizzled bytes read K-major are the other GEMM's view of G.
//
// dW2 instance: one unit = 128 vocabulary ids (M) x rank (N), K = rows in
// stages of 64. Per stage the producer warp loads two 64-id boxes of G (the
// A operand, MN-major) and gathers the stage's 64 W1 rows with tile::gather4
// (the B operand, MN-major; invalid ids and rows past the end read row
// `vocab`, outside the tensor, i.e. zeros). When all rows' W1 rows fit in
// shared memory beside three stages, they are gathered once per CTA instead
// (RES), and a stage carries only the G boxes. The epilogue writes the fp32 tile
// through up to four swizzled 32-column staging boxes with TMA stores, or TMA
// reduce-adds when accumulating.
//
// dW1 instance: split-K over the vocabulary. One unit = 128 rows (M) x rank
// (N) over one vocabulary range; per 64-id stage, one 128-row box of G (A,
// K-major) and rank/64 boxes of W2 [64 ids x 64 columns] (B, MN-major). The
// epilogue adds each row's partial sum into dW1[prev_i] with vector atomics
// (rows with an invalid id add nothing).
//
// Warp roles (192 threads): warp 0 producer, warp 1 owns tensor memory and
// issues the MMAs from lane 0, warps 2-5 epilogue (warp w reads TMEM lanes
// 32*(w%4)). Two fp32 accumulators of rank columns each. Every wait is
// bounded (WaitCtl).
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace dspark {
namespace {

constexpr int kBM = 128;         // MMA M: ids (dW2) or rows (dW1) per unit
constexpr int kKc = 64;          // K per stage: rows (dW2) or ids (dW1)
constexpr int kThreads = 192;
constexpr int kMaxStages = 8;
constexpr uint32_t kBlockBytes = kKc * 128;  // one 64-element-wide box of kKc 128-byte rows
constexpr uint32_t kOutBoxBytes = 128 * 128; // dW2 staging: 128 ids x 32 fp32
constexpr size_t kSmemLimit = 232448;
constexpr int32_t kRidCacheRows = 8192;     // dW2: rows whose W1 coordinates stay in shared memory

__host__ __device__ constexpr uint32_t a_bytes_of(bool dw1) { return dw1 ? kBM * 128u : 2u * kBlockBytes; }
__host__ __device__ constexpr uint32_t stage_bytes_of(int na, bool dw1) { return a_bytes_of(dw1) + na * kBlockBytes; }
// dW2 staging boxes (128 ids x 32 fp32 each): one per 32-column chunk, at most four.
__host__ __device__ constexpr int out_boxes_of(int na) { return 2 * na < 4 ? 2 * na : 4; }
__host__ __device__ constexpr uint32_t tmem_cols_of(int na) {
  return 2 * na * 64 <= 128 ? 128u : 2 * na * 64 <= 256 ? 256u : 512u;
}

// Shared-memory descriptor of an MN-major bf16 operand in the 128-byte swizzle
// layout: 64 consecutive M (or N) elements per 128-byte row, one row per K
// index, 8-row groups 1024 bytes apart along K (stride byte offset), and
// `mn_stride` bytes from one 64-element block of M (or N) to the next
// (leading byte offset). Version 1, base offset 0, layout 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t mn_stride) {
  return (uint64_t)((smem_addr & 0x3FFFFu) >> 4) | ((uint64_t)((mn_stride >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
constexpr uint32_t kAMnMajor = 1u << 15, kBMnMajor = 1u << 16;

__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void red_add_v4(float* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(__uint_as_float(a)),
               "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
               : "memory");
}

__device__ __forceinline__ bool barrier_and(bool v, uint32_t id, uint32_t n) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return out != 0;
}

// Lane 0 waits (bounded), the warp follows its verdict.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, int lane) {
  bool ok = lane == 0 ? mbar_wait(bar, parity, ctl) : true;
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok && lane != 0) mbar_wait(bar, parity, ctl);
  return ok;
}

struct __align__(64) BwdMaps {
  CUtensorMap g;    // G [rows, vocab] bf16; box 64 ids x 64 rows (dW2) or 64 ids x 128 rows (dW1)
  CUtensorMap w;    // W1 rows, box 64 x 1, for gather4 (dW2); W2, box 64 x 64 (dW1)
  CUtensorMap dw2;  // dW2 [vocab, rank] fp32, box 32 x 128 (dW2 kernel only)
};

struct BwdParams {
  const int64_t* ids;
  float* dw1;
  int64_t rows, vocab;
  int32_t rank;
  int32_t row_tiles;  // dW1: 128-row tiles
  int32_t splits;     // dW1: vocabulary ranges per row tile
  int32_t chunks;     // dW1: 64-id chunks of the vocabulary
  int32_t units;      // dW2: 128-id tiles; dW1: row_tiles * splits
  int32_t k_stages;   // dW2: 64-row stages of one unit
  int32_t stages;     // ring depth
  int32_t accumulate;
  int32_t keep_g;     // dW2: the dW1 kernel reads G next (ask L2 to keep it)
  int32_t rid_cached; // dW2: rows (rounded up to 64) whose W1 coordinates are cached in
                      // shared memory once per CTA; 0 = read per stage
  uint32_t* status;
  uint64_t wait_limit_ns;
};

struct BwdShared {
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t w1_full;  // dW2 with resident W1 rows: the one-time gather
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int32_t rid[kKc];  // W1 row coordinates of the stage being gathered
};

// Row coordinate in W1 for row r of G: its prev id, or `vocab` (outside the
// tensor, read as zeros) past the last row or for an invalid id.
__device__ __forceinline__ int32_t w1_row_of(const BwdParams& p, int64_t r) {
  if (r >= p.rows) return (int32_t)p.vocab;
  const int64_t id = p.ids[r];
  if (id < 0 || id >= p.vocab) {
    report_status(p.status, DSPARK_STATUS_TOKEN_RANGE);
    return (int32_t)p.vocab;
  }
  return (int32_t)id;
}

// Unit u of the dW1 kernel: row tile m, vocabulary chunks [c0, c1).
__device__ __forceinline__ void dw1_unit(const BwdParams& p, int64_t u, int32_t& m, int32_t& c0, int32_t& c1) {
  m = (int32_t)(u % p.row_tiles);
  const int64_t s = u / p.row_tiles;
  c0 = (int32_t)((int64_t)p.chunks * s / p.splits);
  c1 = (int32_t)((int64_t)p.chunks * (s + 1) / p.splits);
}

// RES (dW2 only): the W1 rows of all rows are gathered once per CTA into a
// resident MN-major B operand (rank/64 blocks of rid_cached 128-byte rows),
// and a stage carries only the two G boxes.
template <int NA, bool DW1, bool RES>
__global__ void __launch_bounds__(kThreads, 1) tc_backward_kernel(const __grid_constant__ BwdMaps maps, const BwdParams p) {
  static_assert(!(DW1 && RES), "resident W1 rows are a dW2 layout");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kN = NA * 64;
  constexpr uint32_t kABytes = a_bytes_of(DW1);
  constexpr uint32_t kStageBytes = RES ? kABytes : stage_bytes_of(NA, DW1);
  constexpr uint32_t kTmemCols = tmem_cols_of(NA);
  uint8_t* stage_smem = smem;
  uint8_t* w1_res = smem + (size_t)p.stages * kStageBytes;  // RES: NA blocks of rid_cached rows
  const uint32_t res_block = RES ? (uint32_t)p.rid_cached * 128u : 0u;
  uint8_t* out_smem = w1_res + (size_t)NA * res_block;  // dW2: staging boxes
  BwdShared* sh = reinterpret_cast<BwdShared*>(out_smem + (DW1 ? 0 : out_boxes_of(NA) * kOutBoxBytes));
  int32_t* rid_all = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(sh) + sizeof(BwdShared));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t u_begin = (int64_t)p.units * blockIdx.x / gridDim.x;
  const int64_t u_end = (int64_t)p.units * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&sh->full[i], 1);
      mbar_init(&sh->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh->acc_full[i], 1);
      mbar_init(&sh->acc_empty[i], 4);  // one arrival per epilogue warp
    }
    mbar_init(&sh->w1_full, 1);
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
      prefetch_tensormap(&maps.g);
      prefetch_tensormap(&maps.w);
    }
    // When both gradients are wanted G is read twice: the dW2 pass (run
    // first) asks L2 to keep it, and the dW1 pass reads it as evict-first.
    const uint64_t pol_g = (!DW1 && p.keep_g) ? policy_evict_last() : policy_evict_first();
    const uint64_t pol_w = policy_evict_last();
    if constexpr (!DW1) {
      // Every unit walks the same rows: their W1 coordinates are read once,
      // eight loads in flight per lane, and padded with `vocab` to a whole stage.
      for (int32_t r0 = 0; r0 < p.rid_cached; r0 += 32 * 8) {
        int64_t idv[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int64_t r = (int64_t)r0 + 32 * t + lane;
          idv[t] = r < p.rows ? p.ids[r] : 0;
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int32_t r = r0 + 32 * t + lane;
          if (r < p.rid_cached) {
            int32_t c = (int32_t)p.vocab;
            if (r < p.rows) {
              if (idv[t] >= 0 && idv[t] < p.vocab)
                c = (int32_t)idv[t];
              else
                report_status(p.status, DSPARK_STATUS_TOKEN_RANGE);
            }
            rid_all[r] = c;
          }
        }
      }
      __syncwarp();
      if constexpr (RES) {
        const int quads = p.rid_cached / 4;
        if (lane == 0) mbar_arrive_expect_tx(&sh->w1_full, (uint32_t)NA * res_block);
        __syncwarp();
        for (int i = lane; i < NA * quads; i += 32) {
          const int c = i / quads, j = i % quads;
          tma_gather4(w1_res + (size_t)c * res_block + j * 512, &maps.w, &sh->w1_full, c * 64, rid_all[4 * j],
                      rid_all[4 * j + 1], rid_all[4 * j + 2], rid_all[4 * j + 3], pol_w);
        }
        __syncwarp();
      }
    }
    uint32_t it = 0;
    bool ok = true;
    for (int64_t u = u_begin; u < u_end && ok; ++u) {
      int32_t m = 0, c0 = 0, c1 = p.k_stages;
      if constexpr (DW1) dw1_unit(p, u, m, c0, c1);
      for (int32_t kc = c0; kc < c1; ++kc, ++it) {
        const int s = (int)(it % (uint32_t)p.stages);
        if (!warp_wait(&sh->empty[s], ((it / (uint32_t)p.stages) & 1u) ^ 1u, ctl, lane)) {
          ok = false;
          break;
        }
        uint8_t* st = stage_smem + (size_t)s * kStageBytes;
        if constexpr (DW1) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&sh->full[s], kStageBytes);
            tma_load_2d(st, &maps.g, &sh->full[s], kc * kKc, m * kBM, pol_g);
#pragma unroll
            for (int c = 0; c < NA; ++c)
              tma_load_2d(st + kABytes + c * kBlockBytes, &maps.w, &sh->full[s], c * 64, kc * kKc, pol_w);
          }
        } else {
          const int32_t v0 = (int32_t)u * kBM;
          const int64_t r0 = (int64_t)kc * kKc;
          if constexpr (RES) {
            if (lane == 0) {
              mbar_arrive_expect_tx(&sh->full[s], kStageBytes);
              tma_load_2d(st, &maps.g, &sh->full[s], v0, (int32_t)r0, pol_g);
              tma_load_2d(st + kBlockBytes, &maps.g, &sh->full[s], v0 + 64, (int32_t)r0, pol_g);
            }
            __syncwarp();
            continue;
          }
          const int32_t* rsrc = rid_all + r0;
          if (!p.rid_cached) {
            sh->rid[lane] = w1_row_of(p, r0 + lane);
            sh->rid[32 + lane] = w1_row_of(p, r0 + 32 + lane);
            rsrc = sh->rid;
          }
          if (lane == 0) {
            mbar_arrive_expect_tx(&sh->full[s], kStageBytes);
            tma_load_2d(st, &maps.g, &sh->full[s], v0, (int32_t)r0, pol_g);
            tma_load_2d(st + kBlockBytes, &maps.g, &sh->full[s], v0 + 64, (int32_t)r0, pol_g);
          }
          __syncwarp();
          for (int i = lane; i < NA * (kKc / 4); i += 32) {
            const int c = i / (kKc / 4), j = i % (kKc / 4);
            tma_gather4(st + kABytes + c * kBlockBytes + j * 512, &maps.w, &sh->full[s], c * 64, rsrc[4 * j],
                        rsrc[4 * j + 1], rsrc[4 * j + 2], rsrc[4 * j + 3], pol_w);
          }
          __syncwarp();  // sh->rid is rewritten for the next stage
        }
      }
    }
    // Wait (bounded, even after an abort) for the copies this warp started.
    if (lane == 0) {
      const uint32_t S = (uint32_t)p.stages;
      for (uint32_t j = it > S ? it - S : 0; j < it; ++j) mbar_wait(&sh->full[j % S], (j / S) & 1u, drain_ctl);
      if (RES) mbar_wait(&sh->w1_full, 0, drain_ctl);
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kN) | kBMnMajor | (DW1 ? 0u : kAMnMajor);
      const uint32_t stage_addr = smem_u32(stage_smem);
      const uint32_t res_addr = smem_u32(w1_res);
      uint32_t it = 0;
      int64_t ui = 0;
      bool ok = !RES || mbar_wait(&sh->w1_full, 0, ctl);
      for (int64_t u = u_begin; u < u_end && ok; ++u, ++ui) {
        int32_t m = 0, c0 = 0, c1 = p.k_stages;
        if constexpr (DW1) dw1_unit(p, u, m, c0, c1);
        const int abuf = (int)(ui & 1);
        if (!mbar_wait(&sh->acc_empty[abuf], ((uint32_t)(ui >> 1) & 1u) ^ 1u, ctl)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * kN);
        for (int32_t kc = c0; kc < c1; ++kc, ++it) {
          const int s = (int)(it % (uint32_t)p.stages);
          if (!mbar_wait(&sh->full[s], (it / (uint32_t)p.stages) & 1u, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = stage_addr + (uint32_t)s * kStageBytes;
          // B: this stage's rows of the resident block, or the stage's own gather.
          const uint32_t b_addr = RES ? res_addr + (uint32_t)kc * kBlockBytes : a_addr + kABytes;
          const uint32_t b_stride = RES ? res_block : kBlockBytes;
#pragma unroll
          for (int kk = 0; kk < kKc / 16; ++kk) {
            // K = 16 per instruction: 32 bytes along a K-major row, or two
            // 8-row groups (2048 bytes) of an MN-major block.
            const uint64_t ad = DW1 ? sw128_kmajor_desc(a_addr + kk * 32)
                                    : sw128_mnmajor_desc(a_addr + kk * 2048, kBlockBytes);
            const uint64_t bd = sw128_mnmajor_desc(b_addr + kk * 2048, b_stride);
            umma_bf16_ss(d_tmem, ad, bd, idesc, (kc != c0 || kk != 0) ? 1u : 0u);
          }
          umma_commit(&sh->empty[s]);
        }
        if (ok) umma_commit(&sh->acc_full[abuf]);
      }
      umma_commit(&sh->drain);
      mbar_wait(&sh->drain, 0, drain_ctl);
    }
  } else {
    // ------------------------------------------------- epilogue -------
    const int et = threadIdx.x - 64;  // 0..127
    const int q = warp & 3;           // TMEM lane quarter of this warp
    const int row = 32 * q + lane;    // M index within the unit
    const uint32_t bar_id = 1;
    int64_t ui = 0;
    for (int64_t u = u_begin; u < u_end; ++u, ++ui) {
      const int abuf = (int)(ui & 1);
      const uint32_t par = (uint32_t)(ui >> 1) & 1u;
      bool ok = et == 0 ? mbar_wait(&sh->acc_full[abuf], par, ctl) : true;
      __syncwarp();
      if (!barrier_and(ok, bar_id, 128)) break;
      if (et != 0) mbar_wait(&sh->acc_full[abuf], par, ctl);  // already complete
      __syncwarp();
      tc_fence_after_sync();
      const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(abuf * kN);
      float* dst = nullptr;
      bool leader = false;
      uint32_t others = 0;  // lanes whose sums this lane adds in before its atomics
      uint32_t rounds = 0;
      if constexpr (DW1) {
        int32_t m, c0, c1;
        dw1_unit(p, u, m, c0, c1);
        const int64_t r = (int64_t)m * kBM + row;
        int64_t id = -1;
        if (r < p.rows) {
          id = p.ids[r];
          if (id >= 0 && id < p.vocab)
            dst = p.dw1 + id * p.rank;
          else
            id = -1, report_status(p.status, DSPARK_STATUS_TOKEN_RANGE);
        }
        // Rows of this warp with the same id are summed first (Zipf ids
        // repeat), so one atomic per id and warp reaches L2: the lowest lane of
        // each group pulls its peers' sums, one peer per round.
        const uint32_t peers = __match_any_sync(0xffffffffu, (unsigned long long)id);
        leader = (uint32_t)(__ffs(peers) - 1) == (uint32_t)lane;
        others = leader ? (peers & ~(1u << lane)) : 0u;
        rounds = __reduce_max_sync(0xffffffffu, (uint32_t)__popc(others));
#pragma unroll 1
        for (int c = 0; c < kN / 32; ++c) {
          uint32_t acc[32];
          tmem_ld_32x32b_x32(tb + c * 32, acc);
          tmem_ld_wait();
          if (c == kN / 32 - 1) {
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->acc_empty[abuf]);
          }
          uint32_t rest = others;
          for (uint32_t k = 0; k < rounds; ++k) {
            const int src = rest ? __ffs(rest) - 1 : lane;
            rest &= rest - 1u;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float x = __shfl_sync(0xffffffffu, __uint_as_float(acc[e]), src);
              if (src != lane) acc[e] = __float_as_uint(__uint_as_float(acc[e]) + x);
            }
          }
          if (leader && dst) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
              red_add_v4(dst + c * 32 + 4 * k, acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3]);
          }
        }
      } else {
        // Up to four 32-column chunks at a time: all are read from TMEM first
        // (the accumulator is released as soon as the last group is in
        // registers), staged in their own swizzled boxes and stored together.
        constexpr int kChunks = kN / 32;
        constexpr int kBoxes = out_boxes_of(NA);
#pragma unroll
        for (int h = 0; h < kChunks; h += kBoxes) {
          uint32_t acc[kBoxes][32];
#pragma unroll
          for (int cc = 0; cc < kBoxes; ++cc)
            if (h + cc < kChunks) tmem_ld_32x32b_x32(tb + (h + cc) * 32, acc[cc]);
          tmem_ld_wait();
          if (h + kBoxes >= kChunks) {
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->acc_empty[abuf]);
          }
          // The boxes are free once the stores issued from them have read them.
          if (et == 0) bulk_wait_group_read<0>();
          named_barrier_sync(bar_id, 128);
#pragma unroll
          for (int cc = 0; cc < kBoxes; ++cc) {
            if (h + cc < kChunks) {
              uint8_t* box = out_smem + cc * kOutBoxBytes + row * 128;
#pragma unroll
              for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4*>(box + ((k ^ (row & 7)) << 4)) =
                    make_uint4(acc[cc][4 * k], acc[cc][4 * k + 1], acc[cc][4 * k + 2], acc[cc][4 * k + 3]);
            }
          }
          fence_proxy_async_smem();
          named_barrier_sync(bar_id, 128);
          if (et == 0) {
#pragma unroll
            for (int cc = 0; cc < kBoxes; ++cc) {
              if (h + cc < kChunks) {
                const uint8_t* box = out_smem + cc * kOutBoxBytes;
                if (p.accumulate)
                  tma_reduce_add_2d(&maps.dw2, box, (h + cc) * 32, (int32_t)u * kBM);
                else
                  tma_store_2d(&maps.dw2, box, (h + cc) * 32, (int32_t)u * kBM);
              }
            }
            bulk_commit_group();
          }
        }
      }
    }
    if (!DW1 && et == 0) bulk_wait_group<0>();
  }

  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// Shared memory outside the stage ring: alignment slack, barriers, the cached
// W1 coordinates of `rid_cached` rows, the dW2 output boxes and, with RES, the
// resident block of those rows' W1 rows (NA 128-byte rows per row).
size_t fixed_smem_bytes(int na, bool dw1, bool res, int64_t rid_cached) {
  return 1024 + sizeof(BwdShared) + (size_t)rid_cached * 4 + 64 + (dw1 ? 0 : (size_t)out_boxes_of(na) * kOutBoxBytes) +
         (res ? (size_t)na * (size_t)rid_cached * 128 : 0);
}

// The rows whose W1 coordinates dW2 caches in shared memory (all of them, rounded
// up to a whole stage, when there are at most kRidCacheRows; else none).
int64_t rid_cached_of(int64_t rows) { return rows <= kRidCacheRows ? (rows + kKc - 1) / kKc * kKc : 0; }

template <int NA, bool DW1, bool RES>
cudaError_t launch_one(const BackwardArgs& a, int num_sms, uint64_t wait_limit_ns, cudaStream_t stream) {
  BwdMaps maps;
  const uint64_t gdim[2] = {(uint64_t)a.vocab, (uint64_t)a.rows};
  const uint64_t gstr[1] = {(uint64_t)a.vocab * 2};
  const uint32_t gbox[2] = {64, DW1 ? (uint32_t)kBM : (uint32_t)kKc};
  const uint64_t wdim[2] = {(uint64_t)a.rank, (uint64_t)a.vocab};
  const uint64_t wstr[1] = {(uint64_t)a.rank * 2};
  const uint32_t wbox[2] = {64, DW1 ? (uint32_t)kKc : 1u};
  if (!encode_tensor_map(&maps.g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.grad_out, gdim, gstr, gbox,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&maps.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DW1 ? a.w2 : a.w1, wdim, wstr, wbox,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!DW1) {
    const uint64_t odim[2] = {(uint64_t)a.rank, (uint64_t)a.vocab};
    const uint64_t ostr[1] = {(uint64_t)a.rank * 4};
    const uint32_t obox[2] = {32, (uint32_t)kBM};
    if (!encode_tensor_map(&maps.dw2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a.grad_w2, odim, ostr, obox,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    maps.dw2 = maps.w;  // unused
  }

  BwdParams p{};
  p.ids = a.ids;
  p.dw1 = a.grad_w1;
  p.rows = a.rows;
  p.vocab = a.vocab;
  p.rank = a.rank;
  p.accumulate = a.accumulate;
  p.keep_g = (!DW1 && a.grad_w1 != nullptr) ? 1 : 0;
  p.status = a.status;
  p.wait_limit_ns = wait_limit_ns;
  if (DW1) {
    p.row_tiles = (int32_t)((a.rows + kBM - 1) / kBM);
    p.chunks = (int32_t)((a.vocab + kKc - 1) / kKc);
    int32_t splits = num_sms / p.row_tiles;
    if (splits < 1) splits = 1;
    if (splits > p.chunks) splits = p.chunks;
    p.splits = splits;
    p.units = p.row_tiles * splits;
  } else {
    p.units = (int32_t)((a.vocab + kBM - 1) / kBM);
    p.k_stages = (int32_t)((a.rows + kKc - 1) / kKc);
    p.rid_cached = (int32_t)rid_cached_of(a.rows);
  }
  const size_t stage_bytes = RES ? a_bytes_of(false) : stage_bytes_of(NA, DW1);
  const size_t fixed = fixed_smem_bytes(NA, DW1, RES, p.rid_cached);
  if (fixed + 2 * stage_bytes > kSmemLimit) return cudaErrorInvalidValue;
  int stages = (int)((kSmemLimit - fixed) / stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  p.stages = stages;
  const size_t smem = fixed + (size_t)stages * stage_bytes;

  auto kernel = tc_backward_kernel<NA, DW1, RES>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = p.units < num_sms ? p.units : num_sms;
  kernel<<<grid, kThreads, smem, stream>>>(maps, p);
  note_launch();
  return cudaGetLastError();
}

template <int NA>
cudaError_t launch_na(const BackwardArgs& a, int num_sms, uint64_t wait_limit_ns, cudaStream_t s, int* variant) {
  cudaError_t e = cudaSuccess;
  if (a.grad_w2) {
    // Resident W1 rows when they fit beside at least three G stages.
    const int64_t rid = rid_cached_of(a.rows);
    const bool res = rid > 0 && fixed_smem_bytes(NA, false, true, rid) + 3 * (size_t)a_bytes_of(false) <= kSmemLimit;
    if (res) *variant |= DSPARK_VARIANT_BWD_RESIDENT_W1;
    e = res ? launch_one<NA, false, true>(a, num_sms, wait_limit_ns, s)
            : launch_one<NA, false, false>(a, num_sms, wait_limit_ns, s);
  }
  if (e == cudaSuccess && a.grad_w1) e = launch_one<NA, true, false>(a, num_sms, wait_limit_ns, s);
  return e;
}

}  // namespace

bool tc_backward_supported(int64_t rows, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype) {
  if (logits_dtype != DSPARK_DTYPE_BF16 || weight_dtype != DSPARK_DTYPE_BF16) return false;
  if (vocab % 8 != 0 || rank % 64 != 0 || rank < 64 || rank > 256) return false;
  // TMA coordinates are signed 32-bit; row and vocabulary tiles overhang by < 128.
  return rows + kBM < (1ll << 31) && vocab + kBM < (1ll << 31);
}

cudaError_t launch_tc_backward(const BackwardArgs& a, int num_sms, uint64_t wait_limit_ns, cudaStream_t s,
                               int* variant) {
  if (a.rows == 0) return cudaSuccess;
  switch (a.rank / 64) {
    case 1: return launch_na<1>(a, num_sms, wait_limit_ns, s, variant);
    case 2: return launch_na<2>(a, num_sms, wait_limit_ns, s, variant);
    case 3: return launch_na<3>(a, num_sms, wait_limit_ns, s, variant);
    case 4: return launch_na<4>(a, num_sms, wait_limit_ns, s, variant);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dspark
