// Generic (CUDA-core) kernels of the Markov head: any vocabulary size, any
// rank, fp32 or bf16 logits and weights. They serve the fp32 workloads and
// the shapes the tensor-core kernels do not take (vocab not a multiple of 8,
// rank not a multiple of 64, batch above 256 in the sampler).
//
// apply:  one CTA per (row, 1024-wide vocab slice). The CTA stages the row's
//         latent W1[prev] in shared memory; each thread forms the fp32 dot
//         product with W2[v, :] for four ids, adds U and rounds once.
// select: one CTA per batch row; every thread scans a strided part of the
//         corrected row keeping the largest packed (score, -id) key, then the
//         CTA reduces the keys.
#include "common.cuh"
#include "kernels.h"

namespace dspark {

namespace {

constexpr int kApplyThreads = 256;
constexpr int kApplyIdsPerThread = 4;
constexpr int kApplySlice = kApplyThreads * kApplyIdsPerThread;
constexpr int kSelectThreads = 512;

template <typename TL, typename TW>
__global__ void __launch_bounds__(kApplyThreads) generic_apply_kernel(GenericApplyArgs a) {
  extern __shared__ float latent[];
  const int64_t row = blockIdx.x;
  const int64_t id = a.ids[row * a.ld_id];
  const bool valid = id >= 0 && id < a.vocab;
  if (!valid && threadIdx.x == 0 && blockIdx.y == 0) report_status(a.status, DSPARK_STATUS_TOKEN_RANGE);
  const TW* w1 = static_cast<const TW*>(a.w1);
  const TW* w2 = static_cast<const TW*>(a.w2);
  for (int j = threadIdx.x; j < a.rank; j += blockDim.x) latent[j] = valid ? to_f32(w1[id * a.rank + j]) : 0.0f;
  __syncthreads();
  // A null base means U = 0: the output is the bias alone.
  const TL* in = a.base ? static_cast<const TL*>(a.base) + row * a.ld_in : nullptr;
  TL* out = static_cast<TL*>(a.out) + row * a.ld_out;
  const int64_t v0 = (int64_t)blockIdx.y * kApplySlice + threadIdx.x;
#pragma unroll
  for (int i = 0; i < kApplyIdsPerThread; ++i) {
    const int64_t v = v0 + (int64_t)i * kApplyThreads;
    if (v >= a.vocab) break;
    const TW* wrow = w2 + v * a.rank;
    float acc = 0.0f;
    for (int j = 0; j < a.rank; ++j) acc = fmaf(latent[j], to_f32(wrow[j]), acc);
    out[v] = from_f32<TL>((in ? to_f32(in[v]) : 0.0f) + acc);
  }
}

__device__ __forceinline__ unsigned long long max_u64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

template <typename TL>
__global__ void __launch_bounds__(kSelectThreads) generic_select_kernel(GenericSelectArgs a) {
  __shared__ unsigned long long warp_best[kSelectThreads / 32];
  const int64_t b = blockIdx.x;
  const TL* row = static_cast<const TL*>(a.corrected) + b * a.ld_row;
  unsigned long long best = 0ull;
  for (int64_t v = threadIdx.x; v < a.vocab; v += blockDim.x) {
    float s = to_f32(row[v]);
    if (!a.greedy) s = s / a.temperature + noise_for(a.seed, (uint32_t)b, a.step, (uint32_t)v);
    best = max_u64(best, pack_key(s, (uint32_t)v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = max_u64(best, __shfl_xor_sync(0xffffffffu, best, o));
  if ((threadIdx.x & 31) == 0) warp_best[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x < 32) {
    best = threadIdx.x < kSelectThreads / 32 ? warp_best[threadIdx.x] : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = max_u64(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (threadIdx.x == 0) a.tokens[b * a.ld_tok] = (int64_t)key_token(best);
  }
}

template <typename TL, typename TW>
cudaError_t launch_apply_t(const GenericApplyArgs& a, cudaStream_t stream) {
  const int64_t slices = (a.vocab + kApplySlice - 1) / kApplySlice;
  if (slices > 65535) return cudaErrorInvalidConfiguration;
  const size_t smem = (size_t)a.rank * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(generic_apply_kernel<TL, TW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  // Rows go on grid.x (up to 2^31 - 1); chunk anyway to keep offsets simple.
  const int64_t kMaxRows = 1ll << 30;
  for (int64_t r0 = 0; r0 < a.rows; r0 += kMaxRows) {
    GenericApplyArgs c = a;
    c.rows = a.rows - r0 < kMaxRows ? a.rows - r0 : kMaxRows;
    c.base = a.base ? static_cast<const char*>(a.base) + r0 * a.ld_in * (int64_t)sizeof(TL) : nullptr;
    c.out = static_cast<char*>(a.out) + r0 * a.ld_out * (int64_t)sizeof(TL);
    c.ids = a.ids + r0 * a.ld_id;
    dim3 grid((unsigned)c.rows, (unsigned)slices);
    generic_apply_kernel<TL, TW><<<grid, kApplyThreads, smem, stream>>>(c);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_generic_apply(const GenericApplyArgs& a, int logits_dtype, int weight_dtype, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  if (logits_dtype == DSPARK_DTYPE_FP32 && weight_dtype == DSPARK_DTYPE_FP32) return launch_apply_t<float, float>(a, s);
  if (logits_dtype == DSPARK_DTYPE_BF16 && weight_dtype == DSPARK_DTYPE_BF16)
    return launch_apply_t<__nv_bfloat16, __nv_bfloat16>(a, s);
  if (logits_dtype == DSPARK_DTYPE_FP32 && weight_dtype == DSPARK_DTYPE_BF16)
    return launch_apply_t<float, __nv_bfloat16>(a, s);
  return launch_apply_t<__nv_bfloat16, float>(a, s);
}

namespace {
// Embedding rows W1[ids[i]] into out[i, :] (exact copies); an out-of-range id
// gives a zero row and sets DSPARK_STATUS_TOKEN_RANGE.
template <typename TW>
__global__ void gather_rows_kernel(const int64_t* __restrict__ ids, const TW* __restrict__ w1, TW* __restrict__ out,
                                   int64_t rows, int64_t vocab, int32_t rank, uint32_t* status) {
  for (int64_t i = blockIdx.x; i < rows; i += gridDim.x) {
    const int64_t id = ids[i];
    const bool valid = id >= 0 && id < vocab;
    if (!valid && threadIdx.x == 0) report_status(status, DSPARK_STATUS_TOKEN_RANGE);
    for (int j = threadIdx.x; j < rank; j += blockDim.x)
      out[i * rank + j] = valid ? w1[id * rank + j] : from_f32<TW>(0.0f);
  }
}

// Test hook: the Gumbel variate every sampler kernel draws for each word.
__global__ void gumbel_probe_kernel(const uint32_t* __restrict__ words, float* __restrict__ out, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = gumbel_from_word(words[i]);
}
}  // namespace

namespace {
// Register-tiled fp32 contractions on CUDA cores: 256 threads, operand tiles
// of 32 along the summed dimension staged in shared memory as fp32.
constexpr int kBwdK = 32;       // summed-dimension tile
constexpr int kBwdSlice = 2048;  // vocabulary ids per dW1 block (split of the sum over V)

// dW1: G = dOut . W2 for 64 rows x 128 rank columns over one vocabulary
// slice; each thread owns 4 rows x 8 columns; the partial sums are added at
// the rows' ids (the embedding lookup's backward) with atomics.
template <typename TL, typename TW>
__global__ void __launch_bounds__(256) backward_dw1_kernel(BackwardArgs a) {
  __shared__ float sa[kBwdK][64 + 1];  // dOut^T tile [k][row]; the pad spreads the transposed stores over banks
  __shared__ __align__(16) float sb[kBwdK][128];  // W2 tile [k][column]
  const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
  const int64_t m0 = (int64_t)blockIdx.x * 64, n0 = (int64_t)blockIdx.z * 128;
  const int64_t k0 = (int64_t)blockIdx.y * kBwdSlice;
  const int64_t k1 = k0 + kBwdSlice < a.vocab ? k0 + kBwdSlice : a.vocab;
  const TL* g = static_cast<const TL*>(a.grad_out);
  const TW* w2 = static_cast<const TW*>(a.w2);
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  for (int64_t kk = k0; kk < k1; kk += kBwdK) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {  // 64 rows x 32 ids, consecutive threads along the ids
      const int e = tid + 256 * q, row = e >> 5, kx = e & 31;
      const int64_t gr = m0 + row, gk = kk + kx;
      sa[kx][row] = (gr < a.rows && gk < k1) ? to_f32(g[gr * a.vocab + gk]) : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {  // 32 ids x 128 columns, consecutive threads along the columns
      const int e = tid + 256 * q, kx = e >> 7, c = e & 127;
      const int64_t gk = kk + kx, gc = n0 + c;
      sb[kx][c] = (gk < k1 && gc < a.rank) ? to_f32(w2[gk * a.rank + gc]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kBwdK; ++k) {
      float av[4], bv[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = sa[k][tr * 4 + i];
      const float4 b0 = *reinterpret_cast<const float4*>(&sb[k][tc * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&sb[k][tc * 8 + 4]);
      bv[0] = b0.x; bv[1] = b0.y; bv[2] = b0.z; bv[3] = b0.w;
      bv[4] = b1.x; bv[5] = b1.y; bv[6] = b1.z; bv[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t gr = m0 + tr * 4 + i;
    if (gr >= a.rows) break;
    const int64_t id = a.ids[gr];
    if (id < 0 || id >= a.vocab) {
      if (blockIdx.y == 0 && blockIdx.z == 0 && tc == 0) report_status(a.status, DSPARK_STATUS_TOKEN_RANGE);
      continue;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t gc = n0 + tc * 8 + j;
      if (gc < a.rank) atomicAdd(&a.grad_w1[id * a.rank + gc], acc[i][j]);
    }
  }
}

// dW2 = dOut^T . W1[x] for 128 ids x 128 rank columns; each thread owns
// 8 ids x 8 columns and sums over all rows, 32 at a time.
template <typename TL, typename TW>
__global__ void __launch_bounds__(256) backward_dw2_kernel(BackwardArgs a) {
  __shared__ __align__(16) float sd[kBwdK][128];  // dOut tile [row][id]
  __shared__ __align__(16) float se[kBwdK][128];  // embedding tile [row][column]
  const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
  const int64_t v0 = (int64_t)blockIdx.x * 128, n0 = (int64_t)blockIdx.y * 128;
  const TL* g = static_cast<const TL*>(a.grad_out);
  const TW* w1 = static_cast<const TW*>(a.w1);
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  for (int64_t i0 = 0; i0 < a.rows; i0 += kBwdK) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = tid + 256 * q, k = e >> 7, c = e & 127;
      const int64_t gi = i0 + k, gv = v0 + c, gc = n0 + c;
      sd[k][c] = (gi < a.rows && gv < a.vocab) ? to_f32(g[gi * a.vocab + gv]) : 0.0f;
      float x = 0.0f;
      if (gi < a.rows && gc < a.rank) {
        const int64_t id = a.ids[gi];
        if (id >= 0 && id < a.vocab)
          x = to_f32(w1[id * a.rank + gc]);
        else if (blockIdx.x == 0 && blockIdx.y == 0 && c == 0)
          report_status(a.status, DSPARK_STATUS_TOKEN_RANGE);
      }
      se[k][c] = x;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < kBwdK; ++k) {
      const float4 d0 = *reinterpret_cast<const float4*>(&sd[k][tr * 8]);
      const float4 d1 = *reinterpret_cast<const float4*>(&sd[k][tr * 8 + 4]);
      const float4 e0 = *reinterpret_cast<const float4*>(&se[k][tc * 8]);
      const float4 e1 = *reinterpret_cast<const float4*>(&se[k][tc * 8 + 4]);
      const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
      const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(dv[i], ev[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t gv = v0 + tr * 8 + i;
    if (gv >= a.vocab) break;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t gc = n0 + tc * 8 + j;
      if (gc >= a.rank) break;
      float* dst = &a.grad_w2[gv * a.rank + gc];
      *dst = a.accumulate ? *dst + acc[i][j] : acc[i][j];
    }
  }
}

template <typename TL, typename TW>
cudaError_t launch_backward_t(const BackwardArgs& a, cudaStream_t s) {
  const int64_t ntiles = (a.rank + 127) / 128;
  if (a.grad_w1 && a.rows > 0) {
    const int64_t mtiles = (a.rows + 63) / 64, slices = (a.vocab + kBwdSlice - 1) / kBwdSlice;
    if (mtiles > 0x7fffffffll || slices > 65535 || ntiles > 65535) return cudaErrorInvalidConfiguration;
    backward_dw1_kernel<TL, TW><<<dim3((unsigned)mtiles, (unsigned)slices, (unsigned)ntiles), 256, 0, s>>>(a);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.grad_w2) {
    const int64_t vtiles = (a.vocab + 127) / 128;
    if (vtiles > 0x7fffffffll || ntiles > 65535) return cudaErrorInvalidConfiguration;
    backward_dw2_kernel<TL, TW><<<dim3((unsigned)vtiles, (unsigned)ntiles), 256, 0, s>>>(a);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}
}  // namespace

cudaError_t launch_backward(const BackwardArgs& a, int logits_dtype, int weight_dtype, cudaStream_t s) {
  if (logits_dtype == DSPARK_DTYPE_FP32 && weight_dtype == DSPARK_DTYPE_FP32) return launch_backward_t<float, float>(a, s);
  if (logits_dtype == DSPARK_DTYPE_BF16 && weight_dtype == DSPARK_DTYPE_BF16)
    return launch_backward_t<__nv_bfloat16, __nv_bfloat16>(a, s);
  if (logits_dtype == DSPARK_DTYPE_FP32 && weight_dtype == DSPARK_DTYPE_BF16)
    return launch_backward_t<float, __nv_bfloat16>(a, s);
  return launch_backward_t<__nv_bfloat16, float>(a, s);
}

cudaError_t launch_gather_rows(const int64_t* ids, const void* w1, void* out, int64_t rows, int64_t vocab,
                               int32_t rank, int weight_dtype, uint32_t* status, int num_sms, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int grid = (int)(rows < 16ll * num_sms ? rows : 16ll * num_sms);
  const int threads = rank < 256 ? ((rank + 31) / 32) * 32 : 256;
  if (weight_dtype == DSPARK_DTYPE_FP32)
    gather_rows_kernel<float><<<grid, threads, 0, s>>>(ids, static_cast<const float*>(w1), static_cast<float*>(out),
                                                        rows, vocab, rank, status);
  else
    gather_rows_kernel<__nv_bfloat16><<<grid, threads, 0, s>>>(ids, static_cast<const __nv_bfloat16*>(w1),
                                                                static_cast<__nv_bfloat16*>(out), rows, vocab, rank,
                                                                status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_gumbel_probe(const uint32_t* words, float* out, int64_t n, int num_sms, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  const int grid = (int)(blocks < 8ll * num_sms ? blocks : 8ll * num_sms);
  gumbel_probe_kernel<<<grid, 256, 0, s>>>(words, out, n);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_generic_select(const GenericSelectArgs& a, int logits_dtype, cudaStream_t s) {
  if (a.batch == 0) return cudaSuccess;
  if (a.batch > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  if (logits_dtype == DSPARK_DTYPE_FP32)
    generic_select_kernel<float><<<(unsigned)a.batch, kSelectThreads, 0, s>>>(a);
  else
    generic_select_kernel<__nv_bfloat16><<<(unsigned)a.batch, kSelectThreads, 0, s>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace dspark
