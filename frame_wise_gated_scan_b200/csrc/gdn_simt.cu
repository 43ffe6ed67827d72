// CUDA-core (FFMA) kernels of the frame-wise GDN scan.
//
// They follow the update of "NVIDIA Apresenta SANA-WM ..." (acheiumaia.com.br),
// section "A Arquitetura", item "1. Atencao Linear Hibrida com Gated DeltaNet":
// per frame W = (sK)M, R = V - gamma W, M <- gamma M + beta (sK)^T R, O = Q M,
// in that order and in fp32. They serve the fp32-input calls and the bf16
// calls the tensor-core kernel does not take. Without the delta rule
// (GDN_FLAG_NO_DELTA) the residual is V itself and W is not formed.
//
// Decomposition: the value columns of M never mix (column j of W, R, the
// update and O only involves column j of M and V), so each CTA owns one
// block of CB = 16 state columns of one head and runs all T frames on it,
// keeping its D x 16 slice of the state in shared memory. Grid: (D/16, B*H).
// Per frame a CTA streams the frame twice in tiles of TS rows: pass A reads
// K and its V columns and accumulates the D x 16 block of K^T R in registers;
// pass B reads Q and writes its 16 columns of O.
#include <cuda_bf16.h>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kCB = 16;       // state columns per CTA
constexpr int kTS = 32;       // rows per tile
constexpr int kThreads = 256;

__device__ __forceinline__ float load_elt(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load_elt(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
__device__ __forceinline__ void store_elt(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_elt(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}

template <typename Elt, int D>
__global__ void __launch_bounds__(kThreads)
gdn_simt_kernel(const Elt* __restrict__ q, const Elt* __restrict__ k,
                const Elt* __restrict__ v, const float* __restrict__ gamma,
                const float* __restrict__ beta, const float* state_in, float* state_out,
                Elt* __restrict__ out, int T, int S, float s, bool delta) {
  constexpr int kAcc = D * kCB / kThreads;   // K^T R elements per thread
  static_assert(kAcc * kThreads == D * kCB, "D must be a multiple of 16");
  __shared__ float Ms[D][kCB];               // state columns [j0, j0+16)
  __shared__ float Xs[kTS][D + 1];           // scaled K tile (pass A) or Q tile (pass B)
  __shared__ float Vs[kTS][kCB];
  __shared__ float Rs[kTS][kCB];

  const int tid = threadIdx.x;
  const int j0 = blockIdx.x * kCB;
  const long long bh = blockIdx.y;
  const long long frame_elems = (long long)S * D;

  for (int e = tid; e < D * kCB; e += kThreads) {
    const int d = e / kCB, j = e % kCB;
    Ms[d][j] = state_in ? state_in[bh * D * D + (long long)d * D + j0 + j] : 0.f;
  }
  __syncthreads();

  for (int t = 0; t < T; ++t) {
    const long long base = (bh * T + t) * frame_elems;
    const float g = __ldg(gamma + bh * T + t);
    const float b = __ldg(beta + bh * T + t);
    float acc[kAcc];
#pragma unroll
    for (int i = 0; i < kAcc; ++i) acc[i] = 0.f;

    // Pass A: W = (sK) M, R = V - g W, acc += (sK)^T R, one tile of rows at a time.
    for (int r0 = 0; r0 < S; r0 += kTS) {
      for (int e = tid; e < kTS * D; e += kThreads) {
        const int r = e / D, d = e % D;
        Xs[r][d] = (r0 + r < S) ? s * load_elt(k + base + (long long)(r0 + r) * D + d) : 0.f;
      }
      for (int e = tid; e < kTS * kCB; e += kThreads) {
        const int r = e / kCB, j = e % kCB;
        Vs[r][j] = (r0 + r < S) ? load_elt(v + base + (long long)(r0 + r) * D + j0 + j) : 0.f;
      }
      __syncthreads();
      for (int e = tid; e < kTS * kCB; e += kThreads) {
        const int r = e / kCB, j = e % kCB;
        if (delta) {
          float w = 0.f;
#pragma unroll 8
          for (int d = 0; d < D; ++d) w = fmaf(Xs[r][d], Ms[d][j], w);
          Rs[r][j] = Vs[r][j] - g * w;
        } else {
          Rs[r][j] = Vs[r][j];
        }
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < kAcc; ++i) {
        const int e = tid + i * kThreads;
        const int d = e / kCB, j = e % kCB;
        float a = acc[i];
#pragma unroll 8
        for (int r = 0; r < kTS; ++r) a = fmaf(Xs[r][d], Rs[r][j], a);
        acc[i] = a;
      }
      __syncthreads();
    }

    // State update on the CTA's columns.
#pragma unroll
    for (int i = 0; i < kAcc; ++i) {
      const int e = tid + i * kThreads;
      const int d = e / kCB, j = e % kCB;
      Ms[d][j] = g * Ms[d][j] + b * acc[i];
    }
    __syncthreads();

    // Pass B: O = Q M_t on the CTA's columns.
    for (int r0 = 0; r0 < S; r0 += kTS) {
      for (int e = tid; e < kTS * D; e += kThreads) {
        const int r = e / D, d = e % D;
        Xs[r][d] = (r0 + r < S) ? load_elt(q + base + (long long)(r0 + r) * D + d) : 0.f;
      }
      __syncthreads();
      for (int e = tid; e < kTS * kCB; e += kThreads) {
        const int r = e / kCB, j = e % kCB;
        if (r0 + r < S) {
          float o = 0.f;
#pragma unroll 8
          for (int d = 0; d < D; ++d) o = fmaf(Xs[r][d], Ms[d][j], o);
          store_elt(out + base + (long long)(r0 + r) * D + j0 + j, o);
        }
      }
      __syncthreads();
    }
  }

  if (state_out) {
    for (int e = tid; e < D * kCB; e += kThreads) {
      const int d = e / kCB, j = e % kCB;
      state_out[bh * D * D + (long long)d * D + j0 + j] = Ms[d][j];
    }
  }
}

template <typename Elt>
cudaError_t launch(const Problem& p) {
  dim3 grid(p.D / kCB, p.B * p.H);
  const Elt* q = static_cast<const Elt*>(p.q);
  const Elt* k = static_cast<const Elt*>(p.k);
  const Elt* v = static_cast<const Elt*>(p.v);
  Elt* out = static_cast<Elt*>(p.out);
  switch (p.D) {
    case 32:
      gdn_simt_kernel<Elt, 32><<<grid, kThreads, 0, p.stream>>>(
          q, k, v, p.gamma, p.beta, p.state_in, p.state_out, out, p.T, p.S, p.key_scale, p.delta);
      break;
    case 64:
      gdn_simt_kernel<Elt, 64><<<grid, kThreads, 0, p.stream>>>(
          q, k, v, p.gamma, p.beta, p.state_in, p.state_out, out, p.T, p.S, p.key_scale, p.delta);
      break;
    case 128:
      gdn_simt_kernel<Elt, 128><<<grid, kThreads, 0, p.stream>>>(
          q, k, v, p.gamma, p.beta, p.state_in, p.state_out, out, p.T, p.S, p.key_scale, p.delta);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_f32(const Problem& p) { return launch<float>(p); }
cudaError_t launch_simt_bf16(const Problem& p) { return launch<__nv_bfloat16>(p); }

}  // namespace gdn
