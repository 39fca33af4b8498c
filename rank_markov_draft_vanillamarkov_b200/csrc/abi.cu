// The C ABI (include/dspark_markov.h): argument checks, per-device state,
// kernel selection and launches. Nothing here allocates or synchronises on the
// hot path except the one-time per-device workspace (and its growth for a
// larger sampler call).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/dspark_markov.h"
#include "kernels.h"

namespace dspark {

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // about two seconds

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  uint32_t* status = nullptr;               // 1 word
  unsigned char* workspace = nullptr;       // sampler keys + barrier counter
  size_t workspace_bytes = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
std::atomic<int64_t> g_launches{0};
std::atomic<int32_t> g_algo{DSPARK_ALGO_AUTO};
std::atomic<uint32_t> g_debug_flags{0};
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};
thread_local int32_t t_last_algo = 0;
thread_local int32_t t_last_variant = 0;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

void load_encoder() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
}

// Per-device state of the current device, created on first use.
DeviceState* device_state(int* err) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = DSPARK_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaMalloc(&d.status, sizeof(uint32_t)) != cudaSuccess || cudaMemset(d.status, 0, sizeof(uint32_t)) != cudaSuccess) {
      *err = DSPARK_ERR_CUDA;
      return nullptr;
    }
    d.ready = true;
  }
  return &d;
}

// Workspace of at least `bytes`, grown (never shrunk) on demand.
unsigned char* workspace(DeviceState* d, size_t bytes) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (d->workspace_bytes < bytes) {
    if (d->workspace) {
      cudaDeviceSynchronize();
      cudaFree(d->workspace);
      d->workspace = nullptr;
      d->workspace_bytes = 0;
    }
    size_t cap = 4096;
    while (cap < bytes) cap <<= 1;
    if (cudaMalloc(&d->workspace, cap) != cudaSuccess) return nullptr;
    d->workspace_bytes = cap;
  }
  return d->workspace;
}

// The sampler layout the debug flags force, if any (rows wins over tile).
int sample_layout() {
  const uint32_t f = g_debug_flags.load();
  if (f & DSPARK_DEBUG_SAMPLE_ROWS) return kSampleRows;
  if (f & DSPARK_DEBUG_SAMPLE_TILE) return kSampleTile;
  return kSampleAuto;
}

// ---------------------------------------------------------------------------
// Fixed scratch of dspark_markov_sample_block_noalloc, for callers that cannot
// allocate device memory during the call. It lives in this module's static
// device memory, so it exists from module load on and nothing is allocated.
// Layout: status word at 0, grid-barrier counter at 256, then
// DSPARK_NOALLOC_MAX_KEYS packed step maxima.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocStatusOff = 0;
constexpr size_t kNoAllocCounterOff = 256;
constexpr size_t kNoAllocKeysOff = 512;
constexpr size_t kNoAllocBytes = kNoAllocKeysOff + (size_t)DSPARK_NOALLOC_MAX_KEYS * sizeof(unsigned long long);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

struct NoAllocState {
  bool ready = false;
  int num_sms = 0;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
};

NoAllocState g_noalloc[kMaxDevices];

// Set-up of the current device, done once by its first call: the SM count and
// the scratch's device address. Neither call allocates.
int noalloc_state(NoAllocState** out, bool* fresh) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSPARK_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  NoAllocState& n = g_noalloc[dev];
  if (!n.ready) {
    void* ptr = nullptr;
    if (cudaDeviceGetAttribute(&n.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return DSPARK_ERR_CUDA;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return DSPARK_ERR_CUDA;
    n.scratch = static_cast<unsigned char*>(ptr);
    n.ready = true;
    *fresh = true;
  }
  *out = &n;
  return DSPARK_OK;
}

// The scratch of the current device when its set-up has run, else null.
unsigned char* noalloc_scratch_if_ready() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  return g_noalloc[dev].ready ? g_noalloc[dev].scratch : nullptr;
}

bool dtype_ok(int32_t t) { return t == DSPARK_DTYPE_FP32 || t == DSPARK_DTYPE_BF16; }

int cuda_code(cudaError_t e) { return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA; }

}  // namespace

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, load_encoder);
  if (!g_encode) return false;
  cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  const CUresult r = g_encode(map, dtype, rank, const_cast<void*>(base), reinterpret_cast<const cuuint64_t*>(dims),
                              reinterpret_cast<const cuuint64_t*>(strides_bytes),
                              reinterpret_cast<const cuuint32_t*>(box), elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace dspark

using namespace dspark;

extern "C" {

int dspark_markov_apply_block_logits(const void* base_logits, void* out, const int64_t* prev_token_ids, int64_t rows,
                                     int64_t vocab, const void* w1, const void* w2, int32_t rank, int32_t logits_dtype,
                                     int32_t weight_dtype, void* stream) {
  t_last_algo = 0;
  t_last_variant = 0;
  if (rows < 0 || vocab <= 0 || rank <= 0 || !dtype_ok(logits_dtype) || !dtype_ok(weight_dtype))
    return DSPARK_ERR_INVALID_ARG;
  if (rows == 0) return DSPARK_OK;
  if (!base_logits || !out || !prev_token_ids || !w1 || !w2) return DSPARK_ERR_INVALID_ARG;
  int err = DSPARK_OK;
  DeviceState* d = device_state(&err);
  if (!d) return err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int32_t algo = g_algo.load();
  const bool tc_ok = tc_apply_supported(rows, vocab, rank, logits_dtype, weight_dtype) &&
                     (reinterpret_cast<uintptr_t>(base_logits) % 16 == 0) && (reinterpret_cast<uintptr_t>(out) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(w2) % 16 == 0) && (reinterpret_cast<uintptr_t>(w1) % 16 == 0);
  if (algo == DSPARK_ALGO_TENSOR_CORE && !tc_ok) return DSPARK_ERR_UNSUPPORTED;
  if (tc_ok && algo != DSPARK_ALGO_GENERIC) {
    TcApplyArgs a{base_logits, out, prev_token_ids, rows, vocab, w1, w2, rank, d->status, g_wait_limit_ns.load(),
                  logits_dtype == DSPARK_DTYPE_FP32 ? 1 : 0};
    t_last_algo = 2;
    // The 256-id kernel on request (in-place calls keep the 128-id one).
    const bool wide = (g_debug_flags.load() & DSPARK_DEBUG_APPLY_WIDE) != 0 && out != base_logits;
    if (wide && tc_apply_wide_supported(rows, vocab, rank, logits_dtype, weight_dtype, true)) {
      t_last_variant = DSPARK_VARIANT_APPLY_WIDE;
      return cuda_code(launch_tc_apply_wide(a, d->num_sms, s));
    }
    return cuda_code(launch_tc_apply(a, d->num_sms, s));
  }
  GenericApplyArgs a{base_logits, out, prev_token_ids, rows, vocab, vocab, vocab, 1, w1, w2, rank, d->status};
  t_last_algo = 1;
  return cuda_code(launch_generic_apply(a, logits_dtype, weight_dtype, s));
}

int dspark_markov_apply_block_logits_backward(const void* grad_out, const int64_t* prev_token_ids, int64_t rows,
                                              int64_t vocab, const void* w1, const void* w2, int32_t rank,
                                              float* grad_w1, float* grad_w2, int32_t accumulate,
                                              int32_t logits_dtype, int32_t weight_dtype, void* stream) {
  t_last_algo = 0;
  t_last_variant = 0;
  if (rows < 0 || vocab <= 0 || rank <= 0 || !dtype_ok(logits_dtype) || !dtype_ok(weight_dtype))
    return DSPARK_ERR_INVALID_ARG;
  if (!grad_w1 && !grad_w2) return DSPARK_OK;  // nothing wanted
  if (rows > 0 && (!grad_out || !prev_token_ids || !w1 || !w2)) return DSPARK_ERR_INVALID_ARG;
  if (rank > 1024) return DSPARK_ERR_UNSUPPORTED;
  int err = DSPARK_OK;
  DeviceState* d = device_state(&err);
  if (!d) return err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)vocab * (size_t)rank * sizeof(float);
  if (!accumulate) {  // the gradients start from zero (dW2 is overwritten in full)
    if (grad_w1 && cudaMemsetAsync(grad_w1, 0, bytes, s) != cudaSuccess) return DSPARK_ERR_CUDA;
    if (grad_w2 && rows == 0 && cudaMemsetAsync(grad_w2, 0, bytes, s) != cudaSuccess) return DSPARK_ERR_CUDA;
  }
  if (rows == 0) return DSPARK_OK;
  BackwardArgs a{grad_out, prev_token_ids, rows, vocab, w1, w2, rank, grad_w1, grad_w2, accumulate, d->status};
  const int32_t algo = g_algo.load();
  const auto aligned = [](const void* q) { return reinterpret_cast<uintptr_t>(q) % 16 == 0; };
  const bool tc_ok = tc_backward_supported(rows, vocab, rank, logits_dtype, weight_dtype) && aligned(grad_out) &&
                     aligned(w1) && aligned(w2) && aligned(grad_w1) && aligned(grad_w2);
  if (algo == DSPARK_ALGO_TENSOR_CORE && !tc_ok) return DSPARK_ERR_UNSUPPORTED;
  if (tc_ok && algo != DSPARK_ALGO_GENERIC) {
    t_last_algo = 2;
    int variant = 0;
    const cudaError_t e = launch_tc_backward(a, d->num_sms, g_wait_limit_ns.load(), s, &variant);
    t_last_variant = variant;
    return cuda_code(e);
  }
  t_last_algo = 1;
  return cuda_code(launch_backward(a, logits_dtype, weight_dtype, s));
}

int dspark_markov_transition_logits(const int64_t* token_ids, int64_t rows, int64_t vocab, const void* w1,
                                    const void* w2, int32_t rank, void* transition_out, void* embeddings_out,
                                    int32_t weight_dtype, void* stream) {
  t_last_algo = 0;
  t_last_variant = 0;
  if (rows < 0 || vocab <= 0 || rank <= 0 || !dtype_ok(weight_dtype)) return DSPARK_ERR_INVALID_ARG;
  if (rows == 0) return DSPARK_OK;
  if (!token_ids || !w1 || !w2 || !transition_out) return DSPARK_ERR_INVALID_ARG;
  int err = DSPARK_OK;
  DeviceState* d = device_state(&err);
  if (!d) return err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int32_t algo = g_algo.load();
  const bool tc_ok = tc_apply_supported(rows, vocab, rank, weight_dtype, weight_dtype) &&
                     (reinterpret_cast<uintptr_t>(transition_out) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(w2) % 16 == 0) && (reinterpret_cast<uintptr_t>(w1) % 16 == 0);
  if (algo == DSPARK_ALGO_TENSOR_CORE && !tc_ok) return DSPARK_ERR_UNSUPPORTED;
  cudaError_t e;
  if (tc_ok && algo != DSPARK_ALGO_GENERIC) {
    TcApplyArgs a{nullptr, transition_out, token_ids, rows, vocab, w1, w2, rank, d->status, g_wait_limit_ns.load(),
                  0};
    t_last_algo = 2;
    e = launch_tc_apply(a, d->num_sms, s);
  } else {
    GenericApplyArgs a{nullptr, transition_out, token_ids, rows, vocab, vocab, vocab, 1, w1, w2, rank, d->status};
    t_last_algo = 1;
    e = launch_generic_apply(a, weight_dtype, weight_dtype, s);
  }
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (embeddings_out)
    e = launch_gather_rows(token_ids, w1, embeddings_out, rows, vocab, rank, weight_dtype, d->status, d->num_sms, s);
  return cuda_code(e);
}

int dspark_markov_fused_lm_head_logits(const void* hidden, const int64_t* prev_token_ids, int64_t rows,
                                       int64_t hidden_dim, int64_t vocab, const void* lm_head, const void* w1,
                                       const void* w2, int32_t rank, void* out, int32_t out_dtype,
                                       int32_t weight_dtype, void* stream) {
  t_last_algo = 0;
  t_last_variant = 0;
  if (rows < 0 || hidden_dim <= 0 || vocab <= 0 || rank <= 0 || !dtype_ok(out_dtype) || !dtype_ok(weight_dtype))
    return DSPARK_ERR_INVALID_ARG;
  if (rows == 0) return DSPARK_OK;
  if (!hidden || !prev_token_ids || !lm_head || !w1 || !w2 || !out) return DSPARK_ERR_INVALID_ARG;
  const auto aligned = [](const void* q) { return reinterpret_cast<uintptr_t>(q) % 16 == 0; };
  if (!tc_fused_supported(rows, hidden_dim, vocab, rank, out_dtype, weight_dtype) || !aligned(hidden) ||
      !aligned(lm_head) || !aligned(w1) || !aligned(w2) || !aligned(out))
    return DSPARK_ERR_UNSUPPORTED;
  int err = DSPARK_OK;
  DeviceState* d = device_state(&err);
  if (!d) return err;
  TcFusedArgs a{};
  a.hidden = hidden;
  a.lm_head = lm_head;
  a.ids = prev_token_ids;
  a.w1 = w1;
  a.w2 = w2;
  a.out = out;
  a.rows = rows;
  a.hidden_dim = hidden_dim;
  a.vocab = vocab;
  a.rank = rank;
  a.out_f32 = out_dtype == DSPARK_DTYPE_FP32 ? 1 : 0;
  a.status = d->status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  t_last_algo = 2;
  return cuda_code(launch_tc_fused(a, d->num_sms, static_cast<cudaStream_t>(stream)));
}

int dspark_markov_sample_block(const void* base_logits, const int64_t* first_prev_token_ids, int64_t batch,
                               int64_t proposal_len, int64_t vocab, const void* w1, const void* w2, int32_t rank,
                               float temperature, uint64_t seed, int64_t* sampled_tokens, void* corrected_logits,
                               int32_t logits_dtype, int32_t weight_dtype, void* stream) {
  t_last_algo = 0;
  t_last_variant = 0;
  if (batch < 0 || proposal_len < 0 || vocab <= 0 || rank <= 0 || !dtype_ok(logits_dtype) ||
      !dtype_ok(weight_dtype) || std::isnan(temperature))
    return DSPARK_ERR_INVALID_ARG;
  if (batch == 0 || proposal_len == 0) return DSPARK_OK;
  if (!base_logits || !first_prev_token_ids || !w1 || !w2 || !sampled_tokens || !corrected_logits)
    return DSPARK_ERR_INVALID_ARG;
  if (vocab > 0xfffffffell || proposal_len > 0x7fffffffll || batch > 0x7fffffffll) return DSPARK_ERR_UNSUPPORTED;
  const size_t lsize = logits_dtype == DSPARK_DTYPE_BF16 ? 2 : 4;
  {
    // The corrected logits are written while base logits are still being read.
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(base_logits), c0 = reinterpret_cast<uintptr_t>(corrected_logits);
    const uintptr_t n = (uintptr_t)(batch * proposal_len * vocab) * lsize;
    if (a0 < c0 + n && c0 < a0 + n) return DSPARK_ERR_INVALID_ARG;
  }
  int err = DSPARK_OK;
  DeviceState* d = device_state(&err);
  if (!d) return err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool greedy = !(temperature >= 1e-5f);
  const int32_t algo = g_algo.load();
  const bool tc_ok = tc_sample_supported(batch, vocab, rank, logits_dtype, weight_dtype, d->num_sms) &&
                     (reinterpret_cast<uintptr_t>(base_logits) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(corrected_logits) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(w2) % 16 == 0) && (reinterpret_cast<uintptr_t>(w1) % 16 == 0);
  if (algo == DSPARK_ALGO_TENSOR_CORE && !tc_ok) return DSPARK_ERR_UNSUPPORTED;
  if (tc_ok && algo != DSPARK_ALGO_GENERIC) {
    const size_t keys_bytes = (size_t)batch * (size_t)proposal_len * sizeof(unsigned long long);
    unsigned char* ws = workspace(d, keys_bytes + 256);
    if (!ws) return DSPARK_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, keys_bytes + 256, s) != cudaSuccess) return DSPARK_ERR_CUDA;
    TcSampleArgs a{};
    a.base = base_logits;
    a.first_prev = first_prev_token_ids;
    a.batch = batch;
    a.steps = proposal_len;
    a.vocab = vocab;
    a.w1 = w1;
    a.w2 = w2;
    a.rank = rank;
    a.temperature = temperature;
    a.greedy = greedy ? 1 : 0;
    a.seed = seed;
    a.tokens = sampled_tokens;
    a.corrected = corrected_logits;
    a.keys = reinterpret_cast<unsigned long long*>(ws);
    a.barrier = reinterpret_cast<uint32_t*>(ws + keys_bytes);
    a.status = d->status;
    a.wait_limit_ns = g_wait_limit_ns.load();
    a.debug_flags = g_debug_flags.load();
    t_last_algo = 2;
    int variant = 0;
    const cudaError_t e = launch_tc_sample(a, d->num_sms, s, sample_layout(), &variant);
    t_last_variant = variant;
    return cuda_code(e);
  }
  // Generic path: one correction launch and one selection launch per step.
  t_last_algo = 1;
  for (int64_t k = 0; k < proposal_len; ++k) {
    GenericApplyArgs a{};
    a.base = static_cast<const char*>(base_logits) + (size_t)k * vocab * lsize;
    a.out = static_cast<char*>(corrected_logits) + (size_t)k * vocab * lsize;
    a.ids = k == 0 ? first_prev_token_ids : sampled_tokens + (k - 1);
    a.rows = batch;
    a.vocab = vocab;
    a.ld_in = proposal_len * vocab;
    a.ld_out = proposal_len * vocab;
    a.ld_id = k == 0 ? 1 : proposal_len;
    a.w1 = w1;
    a.w2 = w2;
    a.rank = rank;
    a.status = d->status;
    cudaError_t e = launch_generic_apply(a, logits_dtype, weight_dtype, s);
    if (e != cudaSuccess) return DSPARK_ERR_CUDA;
    GenericSelectArgs sel{};
    sel.corrected = a.out;
    sel.ld_row = proposal_len * vocab;
    sel.batch = batch;
    sel.vocab = vocab;
    sel.tokens = sampled_tokens + k;
    sel.ld_tok = proposal_len;
    sel.temperature = temperature;
    sel.greedy = greedy ? 1 : 0;
    sel.seed = seed;
    sel.step = (uint32_t)k;
    e = launch_generic_select(sel, logits_dtype, s);
    if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  }
  return DSPARK_OK;
}

int dspark_markov_sample_block_noalloc(const void* base_logits, const int64_t* first_prev_token_ids, int64_t batch,
                                       int64_t proposal_len, int64_t vocab, const void* w1, const void* w2,
                                       int32_t rank, float temperature, uint64_t seed, int64_t* sampled_tokens,
                                       void* corrected_logits, int32_t logits_dtype, int32_t weight_dtype,
                                       void* stream) {
  t_last_algo = 0;
  t_last_variant = 0;
  if (batch < 0 || proposal_len < 0 || vocab <= 0 || rank <= 0 || !dtype_ok(logits_dtype) ||
      !dtype_ok(weight_dtype) || std::isnan(temperature))
    return DSPARK_ERR_INVALID_ARG;
  if (batch == 0 || proposal_len == 0) return DSPARK_OK;
  if (!base_logits || !first_prev_token_ids || !w1 || !w2 || !sampled_tokens || !corrected_logits)
    return DSPARK_ERR_INVALID_ARG;
  if (batch * proposal_len > DSPARK_NOALLOC_MAX_KEYS) return DSPARK_ERR_UNSUPPORTED;
  {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(base_logits), c0 = reinterpret_cast<uintptr_t>(corrected_logits);
    const uintptr_t n = (uintptr_t)(batch * proposal_len * vocab) * (logits_dtype == DSPARK_DTYPE_BF16 ? 2 : 4);
    if (a0 < c0 + n && c0 < a0 + n) return DSPARK_ERR_INVALID_ARG;
  }
  NoAllocState* st = nullptr;
  bool fresh = false;
  const int err = noalloc_state(&st, &fresh);
  if (err != DSPARK_OK) return err;
  const bool tc_ok = tc_sample_supported(batch, vocab, rank, logits_dtype, weight_dtype, st->num_sms) &&
                     (reinterpret_cast<uintptr_t>(base_logits) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(corrected_logits) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(w2) % 16 == 0) && (reinterpret_cast<uintptr_t>(w1) % 16 == 0);
  if (!tc_ok) return DSPARK_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (fresh && cudaMemsetAsync(st->scratch + kNoAllocStatusOff, 0, sizeof(uint32_t), s) != cudaSuccess)
    return DSPARK_ERR_CUDA;
  // The barrier counter and the step maxima start at zero; the status word
  // keeps its bits until dspark_markov_get_status reads it.
  const size_t keys_bytes = (size_t)batch * (size_t)proposal_len * sizeof(unsigned long long);
  if (cudaMemsetAsync(st->scratch + kNoAllocCounterOff, 0, kNoAllocKeysOff - kNoAllocCounterOff + keys_bytes, s) !=
      cudaSuccess)
    return DSPARK_ERR_CUDA;
  TcSampleArgs a{};
  a.base = base_logits;
  a.first_prev = first_prev_token_ids;
  a.batch = batch;
  a.steps = proposal_len;
  a.vocab = vocab;
  a.w1 = w1;
  a.w2 = w2;
  a.rank = rank;
  a.temperature = temperature;
  a.greedy = !(temperature >= 1e-5f) ? 1 : 0;
  a.seed = seed;
  a.tokens = sampled_tokens;
  a.corrected = corrected_logits;
  a.keys = reinterpret_cast<unsigned long long*>(st->scratch + kNoAllocKeysOff);
  a.barrier = reinterpret_cast<uint32_t*>(st->scratch + kNoAllocCounterOff);
  a.status = reinterpret_cast<uint32_t*>(st->scratch + kNoAllocStatusOff);
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.debug_flags = g_debug_flags.load();
  t_last_algo = 2;
  int variant = 0;
  const cudaError_t e = launch_tc_sample(a, st->num_sms, s, sample_layout(), &variant);
  t_last_variant = variant;
  return cuda_code(e);
}

int dspark_markov_get_status(void* stream, int32_t* status_out) {
  if (!status_out) return DSPARK_ERR_INVALID_ARG;
  int err = DSPARK_OK;
  DeviceState* d = device_state(&err);
  if (!d) return err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSPARK_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, d->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return DSPARK_ERR_CUDA;
  if (cudaMemset(d->status, 0, sizeof(uint32_t)) != cudaSuccess) return DSPARK_ERR_CUDA;
  if (unsigned char* sc = noalloc_scratch_if_ready()) {
    // The no-allocation sampler reports into its own scratch's status word.
    uint32_t w = 0;
    if (cudaMemcpy(&w, sc + kNoAllocStatusOff, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(sc + kNoAllocStatusOff, 0, sizeof(uint32_t)) != cudaSuccess)
      return DSPARK_ERR_CUDA;
    v |= w;
  }
  *status_out = (int32_t)v;
  return DSPARK_OK;
}

const char* dspark_markov_strerror(int code) {
  switch (code) {
    case DSPARK_OK: return "ok";
    case DSPARK_ERR_INVALID_ARG: return "invalid argument";
    case DSPARK_ERR_UNSUPPORTED: return "unsupported dtype or shape";
    case DSPARK_ERR_CUDA: return "CUDA error";
    default: return "unknown error";
  }
}

int32_t dspark_markov_set_algo(int32_t algo) {
  if (algo != DSPARK_ALGO_AUTO && algo != DSPARK_ALGO_GENERIC && algo != DSPARK_ALGO_TENSOR_CORE) return -1;
  return g_algo.exchange(algo);
}

int64_t dspark_markov_launch_count(void) { return g_launches.load(); }

int dspark_markov_set_debug(uint32_t flags, uint64_t wait_limit_ns) {
  g_debug_flags.store(flags);
  g_wait_limit_ns.store(wait_limit_ns ? wait_limit_ns : kDefaultWaitLimitNs);
  return DSPARK_OK;
}

int32_t dspark_markov_last_algo(void) { return t_last_algo; }

int32_t dspark_markov_last_variant(void) { return t_last_variant; }

int dspark_markov_debug_gumbel(const uint32_t* words, float* out, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!words || !out))) return DSPARK_ERR_INVALID_ARG;
  if (n == 0) return DSPARK_OK;
  int err = DSPARK_OK;
  DeviceState* d = device_state(&err);
  if (!d) return err;
  return cuda_code(launch_gumbel_probe(words, out, n, d->num_sms, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
