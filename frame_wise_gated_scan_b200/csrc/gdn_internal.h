// Internal interface between the C-ABI layer (gdn_api.cu) and the kernels.
#pragma once

#include <cuda.h>
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

// tcgen05 kernel for D = 128 (gdn_tc128.cu): a cluster of two CTAs per head,
// producer and reader. Returns 2 if it takes these sizes, else 0.
int tc128_ctas_per_head(int B, int H, int T, int S, int D);
cudaError_t launch_tc128_bf16(const Problem& p);

// Row-split single-frame kernel (gdn_step.cu): T = 1, D = 64, a cluster of
// CTAs per head sharing the frame's rows. Returns the CTAs per head for these
// sizes, or 0 if it does not take them.
struct RopeParams;
int step_ctas_per_head(int B, int H, int T, int S, int D);
// rope: null, or the 3D RoPE to apply to Q and K in shared memory first.
cudaError_t launch_step_bf16(const Problem& p, int ctas_per_head, const RopeParams* rope = nullptr);
// Frame queue of the persistent streaming launch (gdn_frame_stream).
struct StreamQueue {
  const unsigned long long* posted;   // host-mapped, device view
  unsigned long long* done;           // host-mapped, device view
  unsigned int* queue_words;          // device [ring + 2], zero: relay (8 bytes), then a counter per slot
  int ring;
  unsigned long long idle_timeout_ns;
};
// 1 if the streaming kernel takes these sizes (D = 64, S <= 1536 and every
// head's cluster resident at once), else 0.
int stream_supported(int B, int H, int S, int D);
// p.q/k/v/out are rings [ring][B][H][S][D], p.gamma/beta rings [ring][B][H];
// p.T is unused.
cudaError_t launch_stream_bf16(const Problem& p, const StreamQueue& q, const RopeParams* rope);

// Causal temporal convolution (gdn_conv.cu), arrays as documented in include/gdn.h.
struct ConvProblem {
  const void* x;          // [B][T][S][C] bf16
  const float* w;         // [C][3]
  const float* bias;      // [C] or null
  const void* cache_in;   // [B][S][C] bf16 or null
  void* cache_out;        // [B][S][C] bf16 or null
  void* y;                // [B][T][S][C] bf16
  int B, T, S, C, F;
  cudaStream_t stream;
};
cudaError_t launch_tconv_bf16(const ConvProblem& p);

// 3D RoPE (gdn_rope.cu; the rotation itself is in gdn_rope.cuh).
void rope_params(RopeParams* rp, int D, int grid_w, int t0);
cudaError_t launch_rope_bf16(const void* x, void* y, int B, int H, int T, int S, int D, int grid_w,
                             int t0, cudaStream_t stream);

// Host helpers (gdn_host.cu).
// TMA map of a [frames][S][D] bf16 array as the 3-D tensor (D, S, frames),
// with 64-column (128-byte) x box_rows x 1 boxes and the 128-byte swizzle.
// Rows past S inside a frame read as zero and are not stored.
bool make_frame_map(CUtensorMap* m, const void* base, int D, int S, long long frames,
                    int box_rows);
// Device address of the status word on the current device (null on failure).
unsigned int* status_word();
// Reads and clears the device status word.
cudaError_t read_status(unsigned int* status);
// Bound of every device-side wait, in nanoseconds: 1 s. A build with
// GDN_DEBUG reads GDN_DEBUG_WAIT_NS instead, so tests can make waits run out.
unsigned long long wait_budget_ns();

}  // namespace gdn
