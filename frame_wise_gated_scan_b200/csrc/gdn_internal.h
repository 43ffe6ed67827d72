// Internal interface between the C-ABI layer (gdn_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// One scan request after validation. Arrays as documented in include/gdn.h.
struct Problem {
  const void* q;
  const void* k;
  const void* v;
  const float* gamma;
  const float* beta;
  const float* state_in;   // may be null (M_0 = 0)
  float* state_out;        // may be null
  void* out;
  int B, H, T, S, D;
  float key_scale;         // 1/sqrt(D*S), rounded once from double
  bool delta;              // delta-rule correction on (false: GDN_FLAG_NO_DELTA, R = V)
  cudaStream_t stream;
};

// CUDA-core kernels (gdn_simt.cu).
cudaError_t launch_simt_f32(const Problem& p);
cudaError_t launch_simt_bf16(const Problem& p);

// tcgen05 kernel (gdn_tc.cu).
// Returns the CTAs per head the tensor-core kernel would use for these sizes,
// or 0 if it does not take them.
int tc_ctas_per_head(int B, int H, int T, int S, int D);
cudaError_t launch_tc_bf16(const Problem& p, int ctas_per_head);
// The same kernel with its scratch taken from a fixed device array instead of
// stream-ordered allocations (gdn_frame_scan_noalloc). Needs B * H <=
// GDN_NOALLOC_MAX_HEADS; calls that overlap on the GPU race on the array.
cudaError_t launch_tc_bf16_noalloc(const Problem& p, int ctas_per_head);
// Reads and clears the device status word of the tensor-core kernel.
cudaError_t tc_read_status(unsigned int* status);

}  // namespace gdn
