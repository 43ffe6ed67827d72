// Standalone 3D RoPE of a [B][H][T][S][D] bf16 array of queries or keys (the
// rotation and its layout are described in gdn_rope.cuh). HBM-bound: each
// thread reads one 16-byte chunk (4 pairs) of a token row and writes it back
// rotated; consecutive threads take consecutive chunks.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "gdn_internal.h"
#include "gdn_rope.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) gdn_rope_kernel(const uint4* x, uint4* y, long long chunks,
                                                            int T, int S, int D8,
                                                            const __grid_constant__ RopeParams rp) {
  for (long long idx = (long long)blockIdx.x * kThreads + threadIdx.x; idx < chunks;
       idx += (long long)gridDim.x * kThreads) {
    const int chunk = (int)(idx % D8);
    const long long row = idx / D8;
    const int r = (int)(row % S);
    const int t = (int)((row / S) % T);
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(x + idx));
    rope_chunk(rp, rp.t0 + t, r, chunk, v);
    y[idx] = v;
  }
}

}  // namespace

void rope_params(RopeParams* rp, int D, int grid_w, int t0) {
  const int dh = 2 * (D / 6);
  const int dt = D - 2 * dh;
  rp->nt = dt / 2;
  rp->nth = dt / 2 + dh / 2;
  rp->grid_w = grid_w;
  rp->t0 = t0;
  for (int i = 0; i < kRopeMaxPairs; ++i) {
    double f = 0.0;
    if (i < D / 2) {
      const int size = i < rp->nt ? dt : dh;
      const int local = i < rp->nt ? i : (i < rp->nth ? i - rp->nt : i - rp->nth);
      f = pow(10000.0, -2.0 * local / size);
    }
    rp->freq[i] = (float)f;
  }
}

cudaError_t launch_rope_bf16(const void* x, void* y, int B, int H, int T, int S, int D, int grid_w,
                             int t0, cudaStream_t stream) {
  RopeParams rp;
  rope_params(&rp, D, grid_w, t0);
  const long long chunks = (long long)B * H * T * S * (D / 8);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (chunks + kThreads - 1) / kThreads;
  const long long cap = (long long)sms * 32;
  if (blocks > cap) blocks = cap;
  gdn_rope_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(y), chunks, T, S, D / 8, rp);
  return cudaGetLastError();
}

}  // namespace gdn
