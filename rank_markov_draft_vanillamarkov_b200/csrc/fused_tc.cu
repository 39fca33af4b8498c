// Corrected logits with the base logits produced in the same pass, on the
// sm_100a tensor cores:
//
//     out[i, v] = round( sum_{j<d} h[i, j] * Wlm[v, j] + sum_{j<r} W1[x_i, j] * W2[v, j] )
//
// The first sum is the backbone's base logit U = lm_head(hidden) (module
// docstring of markov_head.py; the frozen vocabulary head of
// DeepseekV41DSparkModel.compute_logits, weight [vocab, hidden], FP32
// result); the second is the VanillaMarkov transition bias of the row's
// previous token. Both are one GEMM over the concatenated K axis,
// [h | W1[x]] . [Wlm | W2]^T, accumulated in fp32 in tensor memory and
// rounded once, so U never reaches HBM.
//
// Persistent CTAs take units (row tile m of 128 rows, id tile n of 256 ids)
// round-robin in id-tile-major order: the row tiles of one id tile run at the
// same time on neighbouring CTAs, so the LM-head rows they all read come from
// HBM once and from L2 for the others. Per unit the K loop streams 64-wide
// blocks through a ring of shared-memory stages: ceil(d / 64) blocks of
// (h, Wlm) by TMA, then ceil(r / 64) blocks of (W1[x], W2), the W1 rows by
// tile::gather4 row gathers. Columns past d or r read as zeros.
//
// Warp roles (256 threads): 0 TMA producer; 1 tensor-memory owner and MMA
// issuer (tcgen05.mma kind::f16, M = 128 rows, N = 256 ids, K = 16, both
// operands K-major in shared memory, 128-byte swizzle); 4-7 epilogue: warp
// 4 + q reads accumulator lanes 32q..32q+31 (one row per thread), rounds and
// stores the row's 256 values with streaming 16-byte stores. Tensor memory
// holds two 256-column fp32 accumulators, so the epilogue of one unit overlaps
// the MMAs of the next. The widest N takes the fewest MMA instructions per id:
// on this part a narrow MMA costs far more per column than a wide one.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace dspark {
namespace {

constexpr int kBM = 128;                    // rows per unit (MMA M)
constexpr int kBN = 256;                    // ids per unit (MMA N)
constexpr int kBK = 64;                     // K per stage: one 128-byte swizzle row of bf16
constexpr uint32_t kABytes = kBM * 128;     // 16 KB
constexpr uint32_t kBBytes = kBN * 128;     // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr int kMaxStages = 4;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmemLimit = 232448;

struct __align__(64) FusedMaps {
  CUtensorMap h;   // [rows, d] bf16, box 64 x 128
  CUtensorMap lm;  // [vocab, d] bf16, box 64 x 256
  CUtensorMap w1;  // [vocab, rank] bf16, box 64 x 1 (row gathers)
  CUtensorMap w2;  // [vocab, rank] bf16, box 64 x 256
};

struct FusedParams {
  const int64_t* ids;
  void* out;
  int64_t rows, vocab;
  int32_t row_tiles, id_tiles;
  int32_t kb_h, kb_r;  // K blocks from the hidden dimension and from the rank
  int32_t stages;
  uint32_t* status;
  uint64_t wait_limit_ns;
};

struct FusedTail {
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  int32_t xid[kBM];
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void st_cs_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.cs.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
  __nv_bfloat162 o = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
  return *reinterpret_cast<uint32_t*>(&o);
}

template <bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    tc_fused_kernel(const __grid_constant__ FusedMaps maps, const FusedParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FusedTail* sh = reinterpret_cast<FusedTail*>(smem + (size_t)p.stages * kStageBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t units = (int64_t)p.row_tiles * p.id_tiles;
  const int MT = p.row_tiles;
  const int KB = p.kb_h + p.kb_r;
  const int S = p.stages;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&sh->full[i], 1);
      mbar_init(&sh->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh->acc_full[i], 1);
      mbar_init(&sh->acc_empty[i], 4);  // one arrival per epilogue warp
    }
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
      prefetch_tensormap(&maps.h);
      prefetch_tensormap(&maps.lm);
      prefetch_tensormap(&maps.w1);
      prefetch_tensormap(&maps.w2);
    }
    const uint64_t pol_keep = policy_evict_last();  // hidden rows and W1/W2: reused by many units
    int64_t g = 0;  // stage fills so far
    bool ok = true;
    for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int32_t n = (int32_t)(u / MT), m = (int32_t)(u % MT);
      if (p.kb_r > 0) {
        // The unit's previous tokens, four per lane; rows past the end and
        // invalid ids gather row `vocab`, outside the tensor, i.e. zeros.
        bool bad = false;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int64_t row = (int64_t)m * kBM + 4 * lane + j;
          int32_t x = (int32_t)p.vocab;
          if (row < p.rows) {
            const int64_t id = p.ids[row];
            if (id < 0 || id >= p.vocab)
              bad = true;
            else
              x = (int32_t)id;
          }
          sh->xid[4 * lane + j] = x;
        }
        if (bad) report_status(p.status, DSPARK_STATUS_TOKEN_RANGE);
      }
      __syncwarp();
      for (int kb = 0; kb < KB; ++kb, ++g) {
        const int s = (int)(g % S);
        const uint32_t e_par = ((uint32_t)(g / S) & 1u) ^ 1u;
        bool e_ok = lane == 0 ? mbar_wait(&sh->empty[s], e_par, ctl) : true;
        e_ok = __shfl_sync(0xffffffffu, e_ok ? 1 : 0, 0) != 0;
        if (!e_ok) {
          ok = false;
          break;
        }
        if (lane != 0) mbar_wait(&sh->empty[s], e_par, ctl);  // already complete
        uint8_t* a_s = smem + (size_t)s * kStageBytes;
        uint8_t* b_s = a_s + kABytes;
        if (lane == 0) mbar_arrive_expect_tx(&sh->full[s], kStageBytes);
        __syncwarp();
        if (kb < p.kb_h) {
          if (lane == 0) {
            tma_load_2d(a_s, &maps.h, &sh->full[s], kb * kBK, m * kBM, pol_keep);
            tma_load_2d_nohint(b_s, &maps.lm, &sh->full[s], kb * kBK, n * kBN);
          }
        } else {
          const int kr = (kb - p.kb_h) * kBK;
          if (lane == 0) tma_load_2d(b_s, &maps.w2, &sh->full[s], kr, n * kBN, pol_keep);
          tma_gather4(a_s + lane * 4 * 128, &maps.w1, &sh->full[s], kr, sh->xid[4 * lane], sh->xid[4 * lane + 1],
                      sh->xid[4 * lane + 2], sh->xid[4 * lane + 3], pol_keep);
        }
        __syncwarp();
      }
    }
    // Every copy this warp started has landed before the CTA may exit.
    if (lane == 0)
      for (int64_t j = (g > S ? g - S : 0); j < g; ++j) mbar_wait(&sh->full[j % S], (uint32_t)(j / S) & 1u, drain_ctl);
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      const uint64_t a0 = sw128_kmajor_desc(smem_u32(smem));
      const uint64_t b0 = sw128_kmajor_desc(smem_u32(smem + kABytes));
      int64_t g = 0;
      int64_t it = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x, ++it) {
        const int abuf = (int)(it & 1);
        if (!mbar_wait(&sh->acc_empty[abuf], ((uint32_t)(it >> 1) & 1u) ^ 1u, ctl)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * kBN);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = (int)(g % S);
          if (!mbar_wait(&sh->full[s], (uint32_t)(g / S) & 1u, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t off = (uint32_t)s * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16_ss(d_tmem, desc_advance(a0, off + kk * 32), desc_advance(b0, off + kk * 32), idesc,
                         (kb | kk) != 0);
          umma_commit(&sh->empty[s]);  // the stage is free once these MMAs have read it
        }
        if (ok) umma_commit(&sh->acc_full[abuf]);
      }
      umma_commit(&sh->drain);
      mbar_wait(&sh->drain, 0, drain_ctl);
    }
  } else if (warp >= 4) {
    // --------------------------------------------------- epilogue -----
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(32 * q) << 16);
    int64_t it = 0;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
      const int32_t n = (int32_t)(u / MT), m = (int32_t)(u % MT);
      const int abuf = (int)(it & 1);
      bool ok = lane == 0 ? mbar_wait(&sh->acc_full[abuf], (uint32_t)(it >> 1) & 1u, ctl) : true;
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      if (lane != 0) mbar_wait(&sh->acc_full[abuf], (uint32_t)(it >> 1) & 1u, ctl);  // already complete
      tc_fence_after_sync();
      const int64_t grow = (int64_t)m * kBM + row;
      const bool row_ok = grow < p.rows;
      const int64_t id0 = (int64_t)n * kBN;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        __syncwarp();  // tcgen05.ld is warp-aligned
        tmem_ld_32x32b_x32(lane_base + (uint32_t)(abuf * kBN + 32 * c), v);
        tmem_ld_wait();
        if (c == kBN / 32 - 1) {
          // The accumulator is in registers: hand it back to the MMA warp.
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->acc_empty[abuf]);
        }
        const int64_t ids = id0 + 32 * c;  // a multiple of 32; vocab is a multiple of 8
        if (!row_ok) continue;  // the warp reconverges at the __syncwarp above
        if constexpr (OUT_F32) {
          float* dst = static_cast<float*>(p.out) + grow * p.vocab + ids;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (ids + 4 * k < p.vocab) st_cs_v4(dst + 4 * k, v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        } else {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + grow * p.vocab + ids;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (ids + 8 * k < p.vocab)
              st_cs_v4(dst + 8 * k, pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                       pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
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

template <bool OUT_F32>
cudaError_t launch_out(const TcFusedArgs& a, int num_sms, cudaStream_t stream) {
  FusedMaps maps;
  const uint64_t hdim[2] = {(uint64_t)a.hidden_dim, (uint64_t)a.rows};
  const uint64_t hstr[1] = {(uint64_t)a.hidden_dim * 2};
  const uint32_t hbox[2] = {(uint32_t)kBK, (uint32_t)kBM};
  const uint64_t ldim[2] = {(uint64_t)a.hidden_dim, (uint64_t)a.vocab};
  const uint32_t nbox[2] = {(uint32_t)kBK, (uint32_t)kBN};
  const uint64_t wdim[2] = {(uint64_t)a.rank, (uint64_t)a.vocab};
  const uint64_t wstr[1] = {(uint64_t)a.rank * 2};
  const uint32_t gbox[2] = {(uint32_t)kBK, 1u};
  if (!encode_tensor_map(&maps.h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.hidden, hdim, hstr, hbox,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&maps.lm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.lm_head, ldim, hstr, nbox,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&maps.w1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w1, wdim, wstr, gbox,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&maps.w2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w2, wdim, wstr, nbox,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  FusedParams p{};
  p.ids = a.ids;
  p.out = a.out;
  p.rows = a.rows;
  p.vocab = a.vocab;
  p.row_tiles = (int32_t)((a.rows + kBM - 1) / kBM);
  p.id_tiles = (int32_t)((a.vocab + kBN - 1) / kBN);
  p.kb_h = (int32_t)((a.hidden_dim + kBK - 1) / kBK);
  p.kb_r = (int32_t)((a.rank + kBK - 1) / kBK);
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;
  const size_t tail = sizeof(FusedTail) + 64;
  int stages = (int)((kSmemLimit - 1024 - tail) / kStageBytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  p.stages = stages;
  const size_t smem = 1024 + (size_t)stages * kStageBytes + tail;

  auto kernel = tc_fused_kernel<OUT_F32>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t units = (int64_t)p.row_tiles * p.id_tiles;
  const int grid = (int)(units < num_sms ? units : num_sms);
  kernel<<<grid, kThreads, smem, stream>>>(maps, p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool tc_fused_supported(int64_t rows, int64_t hidden_dim, int64_t vocab, int32_t rank, int out_dtype,
                        int weight_dtype) {
  if (weight_dtype != DSPARK_DTYPE_BF16) return false;
  if (out_dtype != DSPARK_DTYPE_BF16 && out_dtype != DSPARK_DTYPE_FP32) return false;
  // 16-byte row strides for TMA; whole 16-byte output vectors per row.
  if (hidden_dim < 8 || hidden_dim % 8 != 0 || rank < 8 || rank % 8 != 0 || vocab % 8 != 0) return false;
  if (rank > 4096 || hidden_dim > (1 << 20)) return false;
  // TMA coordinates are signed 32-bit.
  return rows + kBM < (1ll << 31) && vocab + kBN < (1ll << 31);
}

cudaError_t launch_tc_fused(const TcFusedArgs& a, int num_sms, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  return a.out_f32 ? launch_out<true>(a, num_sms, s) : launch_out<false>(a, num_sms, s);
}

}  // namespace dspark
