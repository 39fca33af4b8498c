// Internal interface between the C-ABI layer (abi.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dspark {

// Counts kernel launches made by this library (dspark_markov_launch_count).
void note_launch();

// ---------------------------------------------------------------- generic --
struct GenericApplyArgs {
  const void* base;      // row i at base + i * ld_in elements
  void* out;             // row i at out + i * ld_out elements
  const int64_t* ids;    // prev id of row i at ids[i * ld_id]
  int64_t rows, vocab;
  int64_t ld_in, ld_out, ld_id;
  const void* w1;
  const void* w2;
  int32_t rank;
  uint32_t* status;
};

struct GenericSelectArgs {
  const void* corrected;  // row b at corrected + b * ld_row elements
  int64_t ld_row;
  int64_t batch, vocab;
  int64_t* tokens;  // token of row b at tokens[b * ld_tok]
  int64_t ld_tok;
  float temperature;
  int32_t greedy;
  uint64_t seed;
  uint32_t step;
};

cudaError_t launch_generic_apply(const GenericApplyArgs& a, int logits_dtype, int weight_dtype, cudaStream_t s);
cudaError_t launch_generic_select(const GenericSelectArgs& a, int logits_dtype, cudaStream_t s);
// Gradients of the teacher-forced apply (fp32, accumulated into or written).
struct BackwardArgs {
  const void* grad_out;  // [rows, vocab] logits dtype
  const int64_t* ids;    // [rows]
  int64_t rows, vocab;
  const void* w1;
  const void* w2;
  int32_t rank;
  float* grad_w1;  // [vocab, rank] or null
  float* grad_w2;  // [vocab, rank] or null
  int32_t accumulate;
  uint32_t* status;
};
cudaError_t launch_backward(const BackwardArgs& a, int logits_dtype, int weight_dtype, cudaStream_t s);

cudaError_t launch_gather_rows(const int64_t* ids, const void* w1, void* out, int64_t rows, int64_t vocab,
                               int32_t rank, int weight_dtype, uint32_t* status, int num_sms, cudaStream_t s);
cudaError_t launch_gumbel_probe(const uint32_t* words, float* out, int64_t n, int num_sms, cudaStream_t s);

// ----------------------------------------------------------- tensor core --
// Teacher-forced apply on tcgen05: bf16 logits, bf16 weights,
// vocab % 8 == 0, rank in {64, 128, 192, 256}.
struct TcApplyArgs {
  const void* base;
  void* out;
  const int64_t* ids;
  int64_t rows, vocab;
  const void* w1;
  const void* w2;
  int32_t rank;
  uint32_t* status;
  uint64_t wait_limit_ns;
  int32_t logits_f32;  // base/out are fp32 (else bf16); the weights are bf16
};
bool tc_apply_supported(int64_t rows, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype);
cudaError_t launch_tc_apply(const TcApplyArgs& a, int num_sms, cudaStream_t s);
// The same apply with 256-id units (apply_wide_tc.cu): bf16 logits with a
// base, bf16 weights, rank in {64, 128, 192, 256}.
bool tc_apply_wide_supported(int64_t rows, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype,
                             bool has_base);
cudaError_t launch_tc_apply_wide(const TcApplyArgs& a, int num_sms, cudaStream_t s);

// Persistent left-to-right sampler on tcgen05: bf16 logits, bf16 weights,
// vocab % 8 == 0, rank in {64, 128, 192, 256}, batch <= 256 (and within the
// shared-memory plan), at most 512 vocabulary tiles per CTA.
struct TcSampleArgs {
  const void* base;
  const int64_t* first_prev;
  int64_t batch, steps, vocab;
  const void* w1;
  const void* w2;
  int32_t rank;
  float temperature;
  int32_t greedy;
  uint64_t seed;
  int64_t* tokens;
  void* corrected;
  unsigned long long* keys;  // [steps, batch] workspace, zeroed by the launcher
  uint32_t* barrier;         // grid-barrier counter, zeroed by the launcher
  uint32_t* status;
  uint64_t wait_limit_ns;
  uint32_t debug_flags;
};
bool tc_sample_supported(int64_t batch, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype,
                         int num_sms);
// Sampler layout request: the measured-faster layout for the mode (row layout
// for temperature sampling, tile layout for greedy decoding), or one forced.
enum SampleLayout { kSampleAuto = 0, kSampleRows = 1, kSampleTile = 2 };
// The tile-layout or the row-layout kernel as `layout` asks, each only where
// it fits (else the other); sets DSPARK_VARIANT_SAMPLE_ROWS in *variant when
// the row-layout kernel runs.
cudaError_t launch_tc_sample(const TcSampleArgs& a, int num_sms, cudaStream_t s, int layout, int* variant);
// The row-layout sampler (sample_rows_tc.cu): batch on the MMA's M side,
// batch <= 64.
bool tc_sample_rows_supported(int64_t batch, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype,
                              int num_sms);
cudaError_t launch_tc_sample_rows(const TcSampleArgs& a, int num_sms, cudaStream_t s);

// Backward of the teacher-forced apply on tcgen05: bf16 gradient and bf16
// weights, vocab % 8 == 0, rank in {64, 128, 192, 256}, every pointer 16-byte
// aligned. grad_w1 must already hold its starting value (zero, or the sum to
// add to); grad_w2 is written, or added to when accumulate is set.
bool tc_backward_supported(int64_t rows, int64_t vocab, int32_t rank, int logits_dtype, int weight_dtype);
// Sets DSPARK_VARIANT_* bits in *variant for the kernel variants it launches.
cudaError_t launch_tc_backward(const BackwardArgs& a, int num_sms, uint64_t wait_limit_ns, cudaStream_t s,
                               int* variant);

// The fused producer on tcgen05: out = round(hidden . lm_head^T + W1[x] . W2^T),
// bf16 operands, fp32 accumulation, fp32 or bf16 output; hidden_dim, rank
// and vocab multiples of 8, every pointer 16-byte aligned.
struct TcFusedArgs {
  const void* hidden;   // [rows, hidden_dim]
  const void* lm_head;  // [vocab, hidden_dim]
  const int64_t* ids;   // [rows]
  const void* w1;       // [vocab, rank]
  const void* w2;       // [vocab, rank]
  void* out;            // [rows, vocab]
  int64_t rows, hidden_dim, vocab;
  int32_t rank;
  int32_t out_f32;
  uint32_t* status;
  uint64_t wait_limit_ns;
};
bool tc_fused_supported(int64_t rows, int64_t hidden_dim, int64_t vocab, int32_t rank, int out_dtype,
                        int weight_dtype);
cudaError_t launch_tc_fused(const TcFusedArgs& a, int num_sms, cudaStream_t s);

// Encodes a tiled TMA descriptor through the driver entry point.
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle);

}  // namespace dspark
