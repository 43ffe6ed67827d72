// Causal temporal convolution with a carried last-frame cache, bf16 in and
// out, fp32 taps ("SANA-Video" ICLR 2026 oral transcript, shadowingenglish.com,
// the part on the causal FFN with temporal convolution).
//
// Per channel c, token s and frame t, with blocks of F frames counted from the
// call's first frame:
//     y[t] = w[c][0] x_prev + w[c][1] x[t] + w[c][2] x_next + bias[c]
// x_prev is x[t-1] (for t = 0 the cache handed in: the last frame of the
// previous call, zero without one); x_next is x[t+1] inside a block and zero
// for a block's last frame (the zero token between blocks). The cache handed
// on is x[T-1].
//
// The op moves each byte of x once in and each byte of y once out: HBM-bound,
// with no contraction, so it runs on CUDA cores with 16-byte accesses. Thread
// (column, segment) owns 8 channels of one token (one 16-byte vector per
// frame) over a run of frames, keeps the previous, current and next frame in
// registers, and keeps eight frames of loads in flight (a slot is reloaded as
// soon as its frame is used). Warps read and write
// 512 contiguous bytes per frame. Segments split long runs of frames across
// threads so that small S * C still fills the GPU; a segment reads the frame
// before it (or the cache) once.
#include <cuda_bf16.h>
#include <stdint.h>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kAhead = 8;   // frames loaded ahead of the one being written

__device__ __forceinline__ void unpack8(const uint4 r, float* f) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Streaming accesses: x and y are touched once, so they skip L1 and are
// evicted from L2 first.
__device__ __forceinline__ uint4 ld_stream(const uint4* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.L1::no_allocate.L2::cache_hint.v4.b32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ void st_stream(uint4* p, uint4 v, uint64_t pol) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(pol)
               : "memory");
}

__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__global__ void __launch_bounds__(kThreads, 2) gdn_tconv_kernel(
    const uint4* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias,
    const uint4* cache_in, uint4* cache_out, uint4* __restrict__ y, int T, int S, int C8, int F,
    int seg_frames, int nseg, long long cols) {
  const long long total = cols * nseg;
  const uint64_t pol = evict_first_policy();
  for (long long item = (long long)blockIdx.x * kThreads + threadIdx.x; item < total;
       item += (long long)gridDim.x * kThreads) {
    const long long col = item % cols;   // adjacent threads: adjacent channel vectors
    const int seg = (int)(item / cols);
    const int c8 = (int)(col % C8);
    const long long bs = col / C8;       // b * S + s
    const long long b = bs / S;
    const size_t fs = (size_t)S * C8;    // frame stride, in 16-byte vectors
    const uint4* xc = x + (size_t)b * T * fs + (size_t)(bs % S) * C8 + c8;
    uint4* yc = y + (size_t)b * T * fs + (size_t)(bs % S) * C8 + c8;
    const int t0 = seg * seg_frames;
    const int t1 = min(T, t0 + seg_frames);
    if (t0 >= t1) continue;

    float w0[8], w1[8], w2[8], bb[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = 8 * c8 + e;
      w0[e] = __ldg(w + 3 * c);
      w1[e] = __ldg(w + 3 * c + 1);
      w2[e] = __ldg(w + 3 * c + 2);
      bb[e] = bias ? __ldg(bias + c) : 0.f;
    }
    float prev[8];
    if (t0 > 0) {
      unpack8(ld_stream(xc + (size_t)(t0 - 1) * fs, pol), prev);
    } else if (cache_in) {
      unpack8(cache_in[bs * C8 + c8], prev);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) prev[e] = 0.f;
    }
    // Frame f is loaded when this segment needs it: f < t1 (written here) or
    // f == t1 (the next frame of the segment's last one), and f < T.
    auto load = [&](int f) -> uint4 {
      return (f < T && f <= t1) ? ld_stream(xc + (size_t)f * fs, pol) : make_uint4(0u, 0u, 0u, 0u);
    };
    // Rolling prefetch: on entry to each round, cur is frame t and ahead[u]
    // frame t+1+u. A slot is refilled, kAhead frames further on, as soon as
    // its frame is used, so about kAhead loads stay in flight.
    uint4 cur = load(t0);
    uint4 ahead[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) ahead[u] = load(t0 + 1 + u);
    uint4 last = cur;
    for (int t = t0; t < t1; t += kAhead) {
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        const int tt = t + u;
        if (tt < t1) {
          const uint4 raw = u == 0 ? cur : ahead[u - 1];
          const bool block_end = (tt + 1) % F == 0 || tt + 1 == T;
          float xc_[8], xn[8];
          unpack8(raw, xc_);
          unpack8(ahead[u], xn);
          if (u > 0) ahead[u - 1] = load(tt + kAhead);   // frame t + kAhead + u
          float o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float nx = block_end ? 0.f : xn[e];
            o[e] = fmaf(w2[e], nx, fmaf(w1[e], xc_[e], w0[e] * prev[e])) + bb[e];
            prev[e] = xc_[e];
          }
          st_stream(yc + (size_t)tt * fs,
                    make_uint4(pack2(o[0], o[1]), pack2(o[2], o[3]), pack2(o[4], o[5]),
                               pack2(o[6], o[7])),
                    pol);
          last = raw;
        }
      }
      cur = ahead[kAhead - 1];                           // frame t + kAhead
      ahead[kAhead - 1] = load(t + 2 * kAhead);          // frame t + kAhead + 1 + (kAhead - 1)
    }
    // The first segment hands the cache on: it is the thread that read
    // cache_in, so cache_in == cache_out is safe.
    if (cache_out && seg == 0)
      cache_out[bs * C8 + c8] = t1 == T ? last : ld_stream(xc + (size_t)(T - 1) * fs, pol);
  }
}

}  // namespace

cudaError_t launch_tconv_bf16(const ConvProblem& p) {
  const int C8 = p.C / 8;
  const long long cols = (long long)p.B * p.S * C8;
  // Enough (column, segment) items for about two waves of 2048 threads on
  // every SM; no segment shorter than 16 frames.
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = 2LL * sms * 2048;
  int nseg = (int)((want + cols - 1) / cols);
  nseg = nseg < 1 ? 1 : nseg;
  const int max_seg = (p.T + 15) / 16;
  if (nseg > max_seg) nseg = max_seg;
  const int seg_frames = (p.T + nseg - 1) / nseg;
  nseg = (p.T + seg_frames - 1) / seg_frames;
  const long long items = cols * nseg;
  long long blocks = (items + kThreads - 1) / kThreads;
  const long long cap = (long long)sms * 64;
  if (blocks > cap) blocks = cap;
  gdn_tconv_kernel<<<(unsigned)blocks, kThreads, 0, p.stream>>>(
      static_cast<const uint4*>(p.x), p.w, p.bias, static_cast<const uint4*>(p.cache_in),
      static_cast<uint4*>(p.cache_out), static_cast<uint4*>(p.y), p.T, p.S, C8, p.F, seg_frames,
      nseg, cols);
  return cudaGetLastError();
}

}  // namespace gdn
