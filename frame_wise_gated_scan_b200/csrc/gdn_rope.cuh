// 3D rotary position embedding (RoPE) of query and key rows, shared by the
// standalone rotation kernel and the kernels that rotate tiles on the fly
// ("SANA-Video" ICLR 2026 oral transcript, shadowingenglish.com: 3D RoPE for
// the linear attention).
//
// Layout (the reading of the talk this library takes): the head dimension D is
// cut into contiguous sections for the frame axis t, the grid-row axis h and
// the grid-column axis w, of D_h = D_w = 2 * floor(D / 6) dims each and
// D_t = D - D_h - D_w. Inside a section of D_a dims, dims (2i, 2i + 1) form
// pair i, turned counter-clockwise by p_a * 10000^(-2i / D_a), where p_a is the
// token's position on that axis: the frame's absolute index for t, and for
// token r of a frame on a grid W tokens wide, h = r / W and w = r % W.
//
// The angle is formed in fp32 (position times the pair's frequency, rounded
// once) and turned into cos and sin with sincosf; x' = x c - y s and
// y' = x s + y c in fp32, rounded to bf16 (nearest even).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace gdn {

constexpr int kRopeMaxPairs = 64;   // D <= 128

struct RopeParams {
  float freq[kRopeMaxPairs];   // frequency of pair i (i < D/2), from the host in double
  int nt;                      // pairs of the t section
  int nth;                     // pairs of the t and h sections together
  int np;                      // pairs in all (D / 2)
  int grid_w;                  // tokens per grid row
  int t0;                      // absolute index of the call's first frame
};

// cos/sin of every angle a block needs, in shared memory: the t section of
// one frame, the h section of grid rows [h0, h0 + nh), the w section of every
// grid column. Each entry is sincosf of the same fp32 angle the direct form
// uses, so lookups and direct evaluation agree bit for bit.
constexpr int kRopeTabMaxFloats = 2048;   // 8 KB

__device__ __forceinline__ int rope_tab_floats(const RopeParams& rp, int nh) {
  return 2 * (rp.nt + nh * (rp.nth - rp.nt) + rp.grid_w * (rp.np - rp.nth));
}

// All threads of the block call this (it ends with __syncthreads()).
__device__ __forceinline__ void rope_tab_build(const RopeParams& rp, float* tab, int t, int h0, int nh) {
  const int nhp = rp.nth - rp.nt, nwp = rp.np - rp.nth;
  const int n = rp.nt + nh * nhp + rp.grid_w * nwp;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    float pos;
    int i;
    if (e < rp.nt) {
      pos = (float)t;
      i = e;
    } else if (e < rp.nt + nh * nhp) {
      const int f = e - rp.nt;
      pos = (float)(h0 + f / nhp);
      i = rp.nt + f % nhp;
    } else {
      const int f = e - rp.nt - nh * nhp;
      pos = (float)(f / nwp);
      i = rp.nth + f % nwp;
    }
    float sn, cs;
    sincosf(pos * rp.freq[i], &sn, &cs);
    tab[2 * e] = cs;
    tab[2 * e + 1] = sn;
  }
  __syncthreads();
}

// Angles of the 4 pairs held by 16-byte chunk `chunk` (dims 8 chunk .. +7) of
// token `r` of frame `t` (absolute index).
__device__ __forceinline__ void rope_chunk(const RopeParams& rp, int t, int r, int chunk,
                                           uint4& v) {
  const float ph = (float)(r / rp.grid_w);
  const float pw = (float)(r % rp.grid_w);
  const float pt = (float)t;
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int i = 4 * chunk + e;
    const float pos = i < rp.nt ? pt : (i < rp.nth ? ph : pw);
    float s, c;
    sincosf(pos * rp.freq[i], &s, &c);
    const float x = __uint_as_float(w[e] << 16);
    const float y = __uint_as_float(w[e] & 0xffff0000u);
    const float xr = fmaf(x, c, -y * s);
    const float yr = fmaf(x, s, y * c);
    __nv_bfloat162 o = __floats2bfloat162_rn(xr, yr);
    w[e] = *reinterpret_cast<uint32_t*>(&o);
  }
  v = make_uint4(w[0], w[1], w[2], w[3]);
}

// The same rotation with cos/sin from a table built by rope_tab_build for this
// frame, grid rows from h0.
__device__ __forceinline__ void rope_chunk_tab(const RopeParams& rp, const float* tab, int h0, int nh,
                                               int r, int chunk, uint4& v) {
  const int nhp = rp.nth - rp.nt, nwp = rp.np - rp.nth;
  const int h = r / rp.grid_w - h0, wc = r % rp.grid_w;
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int i = 4 * chunk + e;
    const int idx = i < rp.nt ? i
                    : (i < rp.nth ? rp.nt + h * nhp + (i - rp.nt)
                                  : rp.nt + nh * nhp + wc * nwp + (i - rp.nth));
    const float c = tab[2 * idx], s = tab[2 * idx + 1];
    const float x = __uint_as_float(w[e] << 16);
    const float y = __uint_as_float(w[e] & 0xffff0000u);
    const float xr = fmaf(x, c, -y * s);
    const float yr = fmaf(x, s, y * c);
    __nv_bfloat162 o = __floats2bfloat162_rn(xr, yr);
    w[e] = *reinterpret_cast<uint32_t*>(&o);
  }
  v = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace gdn
