// Standalone 3D RoPE of a [B][H][T][S][D] bf16 array of queries or keys (the
// rotation and its layout are described in gdn_rope.cuh). HBM-bound: each
// thread reads 16-byte chunks (4 pairs) of token rows, four at a time, and
// writes them back rotated; consecutive threads take consecutive chunks.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "gdn_internal.h"
#include "gdn_rope.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 4;   // 16-byte chunks per thread and step

// One block per frame: cos/sin tables of the frame first (shared memory),
// then the frame's rows, four 16-byte chunks per thread and step. Frames whose
// tables would not fit take sincosf per pair instead.
__global__ void __launch_bounds__(kThreads) gdn_rope_kernel(const uint4* x, uint4* y, long long frames,
                                                            int T, int S, int D8,
                                                            const __grid_constant__ RopeParams rp) {
  __shared__ float tab[kRopeTabMaxFloats];
  const int nh = (S - 1) / rp.grid_w + 1;
  const bool use_tab = rope_tab_floats(rp, nh) <= kRopeTabMaxFloats;
  const long long chunks = (long long)S * D8;
  // Only the table's t section depends on the frame: the h and w sections are
  // built with the first frame, the t section again for every frame.
  bool built = false;
  for (long long f = blockIdx.x; f < frames; f += gridDim.x) {
    const int t = rp.t0 + (int)(f % T);
    if (use_tab) {
      if (!built) {
        rope_tab_build(rp, tab, t, 0, nh);
        built = true;
      } else {
        for (int e = threadIdx.x; e < rp.nt; e += kThreads) {
          float sn, cs;
          sincosf((float)t * rp.freq[e], &sn, &cs);
          tab[2 * e] = cs;
          tab[2 * e + 1] = sn;
        }
        __syncthreads();
      }
    }
    const uint4* xs = x + f * chunks;
    uint4* ys = y + f * chunks;
    // kBatch chunks per thread and step, their loads issued together so that
    // several are in flight; consecutive threads keep consecutive chunks.
    for (long long base = threadIdx.x; base < chunks; base += kBatch * kThreads) {
      uint4 v[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const long long idx = base + (long long)k * kThreads;
        if (idx < chunks)
          asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v[k].x), "=r"(v[k].y), "=r"(v[k].z), "=r"(v[k].w)
                       : "l"(xs + idx));
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const long long idx = base + (long long)k * kThreads;
        if (idx < chunks) {
          const int chunk = (int)(idx % D8);
          const int r = (int)(idx / D8);
          if (use_tab)
            rope_chunk_tab(rp, tab, 0, nh, r, chunk, v[k]);
          else
            rope_chunk(rp, t, r, chunk, v[k]);
          ys[idx] = v[k];
        }
      }
    }
    __syncthreads();   // the next frame's table may replace this one
  }
}

}  // namespace

void rope_params(RopeParams* rp, int D, int grid_w, int t0) {
  const int dh = 2 * (D / 6);
  const int dt = D - 2 * dh;
  rp->nt = dt / 2;
  rp->nth = dt / 2 + dh / 2;
  rp->np = D / 2;
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
  const long long frames = (long long)B * H * T;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = frames;
  const long long cap = (long long)sms * 16;
  if (blocks > cap) blocks = cap;
  gdn_rope_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(y), frames, T, S, D / 8, rp);
  return cudaGetLastError();
}

}  // namespace gdn
