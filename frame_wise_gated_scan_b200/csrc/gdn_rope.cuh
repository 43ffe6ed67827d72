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
  int grid_w;                  // tokens per grid row
  int t0;                      // absolute index of the call's first frame
};

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

}  // namespace gdn
