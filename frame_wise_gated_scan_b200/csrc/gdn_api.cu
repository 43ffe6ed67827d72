// C-ABI entry points of libgdn (declared in include/gdn.h): argument checks,
// the key scale, kernel choice, launch.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "gdn.h"
#include "gdn_internal.h"
#include "gdn_rope.cuh"

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// [lo, hi) byte ranges overlap?
bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// Kernel override for debugging: GDN_IMPL=simt forces the CUDA-core kernel.
// Read once per process.
int forced_kernel() {
  static std::atomic<int> cached{-1};
  int v = cached.load(std::memory_order_relaxed);
  if (v < 0) {
    const char* e = getenv("GDN_IMPL");
    v = (e && strcmp(e, "simt") == 0) ? GDN_KERNEL_SIMT : 0;
    cached.store(v, std::memory_order_relaxed);
  }
  return v;
}

int check_sizes(int B, int H, int T, int S, int D) {
  if (B < 1 || H < 1 || T < 1 || S < 1) return GDN_ERR_SHAPE;
  if (D != 32 && D != 64 && D != 128) return GDN_ERR_UNSUPPORTED_D;
  const double elems = (double)B * H * T * S * D;
  if (elems > 9.0e18 / 4.0) return GDN_ERR_SHAPE;
  if ((long long)B * H > 0x7fffffffLL) return GDN_ERR_SHAPE;
  return GDN_OK;
}

int choose_kernel(int B, int H, int T, int S, int D, int* ctas) {
  const int f = forced_kernel();
  const int step = (f == GDN_KERNEL_SIMT) ? 0 : gdn::step_ctas_per_head(B, H, T, S, D);
  if (step > 0) {
    *ctas = step;
    return GDN_KERNEL_STEP;
  }
  const int tc128 = (f == GDN_KERNEL_SIMT) ? 0 : gdn::tc128_ctas_per_head(B, H, T, S, D);
  if (tc128 > 0) {
    *ctas = tc128;
    return GDN_KERNEL_TC;
  }
  const int tc = (f == GDN_KERNEL_SIMT) ? 0 : gdn::tc_ctas_per_head(B, H, T, S, D);
  if (tc > 0) {
    *ctas = tc;
    return GDN_KERNEL_TC;
  }
  *ctas = 1;
  return GDN_KERNEL_SIMT;
}

int run(const void* q, const void* k, const void* v, const float* gamma, const float* beta,
        const float* state_in, float* state_out, void* out, int B, int H, int T, int S, int D,
        void* stream, int elt_bytes, bool noalloc = false, unsigned int flags = 0,
        const gdn::RopeParams* rope = nullptr) {
  const int sz = check_sizes(B, H, T, S, D);
  if (sz != GDN_OK) return sz;
  if (flags & ~GDN_FLAG_NO_DELTA) return GDN_ERR_FLAGS;
  if (!q || !k || !v || !gamma || !beta || !out) return GDN_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(state_in, 16) || !aligned(state_out, 16) || !aligned(gamma, 4) ||
      !aligned(beta, 4))
    return GDN_ERR_ALIGN;
  const size_t n = (size_t)B * H * T * S * D * elt_bytes;
  const size_t ns = (size_t)B * H * D * D * sizeof(float);
  if (overlap(out, n, q, n) || overlap(out, n, k, n) || overlap(out, n, v, n) ||
      overlap(out, n, state_in, ns) || overlap(out, n, state_out, ns))
    return GDN_ERR_ALIAS;
  if (state_in && state_out && state_in != state_out && overlap(state_in, ns, state_out, ns))
    return GDN_ERR_ALIAS;
  int ctas = 1;
  const int kern = elt_bytes == 4 ? GDN_KERNEL_SIMT : choose_kernel(B, H, T, S, D, &ctas);
  if (rope && kern != GDN_KERNEL_STEP) return GDN_ERR_UNSUPPORTED;
  // The fixed scratch of the no-alloc call holds the transition-operand ring,
  // which only the D = 64 tensor-core kernel with more than one CTA per head uses.
  if (noalloc && kern == GDN_KERNEL_TC && D == 64 && ctas > 1 &&
      (long long)B * H > GDN_NOALLOC_MAX_HEADS)
    return GDN_ERR_SCRATCH;

  gdn::Problem p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.gamma = gamma;
  p.beta = beta;
  p.state_in = state_in;
  p.state_out = state_out;
  p.out = out;
  p.B = B;
  p.H = H;
  p.T = T;
  p.S = S;
  p.D = D;
  p.key_scale = (float)(1.0 / sqrt((double)D * (double)S));
  p.delta = (flags & GDN_FLAG_NO_DELTA) == 0;
  p.stream = static_cast<cudaStream_t>(stream);

  cudaError_t err;
  if (elt_bytes == 4) {
    err = gdn::launch_simt_f32(p);
  } else {
    if (kern == GDN_KERNEL_STEP)
      err = gdn::launch_step_bf16(p, ctas, rope);   // allocates nothing
    else if (kern != GDN_KERNEL_TC)
      err = gdn::launch_simt_bf16(p);   // allocates nothing either way
    else if (D == 128)
      err = gdn::launch_tc128_bf16(p);        // allocates nothing
    else
      err = noalloc ? gdn::launch_tc_bf16_noalloc(p, ctas) : gdn::launch_tc_bf16(p, ctas);
  }
  return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

extern "C" {

int gdn_frame_scan(const void* q, const void* k, const void* v, const float* gamma,
                   const float* beta, const float* state_in, float* state_out, void* out, int B,
                   int H, int T, int S, int D, void* stream) {
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, T, S, D, stream, 2);
}

int gdn_frame_scan_noalloc(const void* q, const void* k, const void* v, const float* gamma,
                           const float* beta, const float* state_in, float* state_out, void* out,
                           int B, int H, int T, int S, int D, void* stream) {
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, T, S, D, stream, 2, true);
}

int gdn_frame_step(const void* q, const void* k, const void* v, const float* gamma,
                   const float* beta, const float* state_in, float* state_out, void* out, int B,
                   int H, int S, int D, void* stream) {
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, 1, S, D, stream, 2);
}

int gdn_frame_step_rope(const void* q, const void* k, const void* v, const float* gamma,
                        const float* beta, const float* state_in, float* state_out, void* out,
                        int B, int H, int S, int D, int grid_w, int frame_index, unsigned int flags,
                        void* stream) {
  if (grid_w < 1 || frame_index < 0) return GDN_ERR_SHAPE;
  gdn::RopeParams rp;
  gdn::rope_params(&rp, 64, grid_w, frame_index);
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, 1, S, D, stream, 2, false, flags,
             &rp);
}

namespace {

// gdn_frame_stream and gdn_frame_stream_rope (rope: null, or the 3D RoPE of
// the first frame; frame n of the queue is turned as frame t0 + n).
int stream_impl(const void* q, const void* k, const void* v, const float* gamma,
                const float* beta, const float* state_in, float* state_out, void* out, int B,
                int H, int S, int D, int ring, const unsigned long long* posted,
                unsigned long long* done, unsigned int* queue_words,
                unsigned long long idle_timeout_ns, unsigned int flags, void* stream,
                const gdn::RopeParams* rope) {
  const int sz = check_sizes(B, H, 1, S, D);
  if (sz != GDN_OK) return sz;
  if (ring < 1 || (long long)ring * B * H > 0x7fffffffLL) return GDN_ERR_SHAPE;
  if (flags & ~GDN_FLAG_NO_DELTA) return GDN_ERR_FLAGS;
  if (!q || !k || !v || !gamma || !beta || !out || !posted || !done || !queue_words)
    return GDN_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(state_in, 16) || !aligned(state_out, 16) || !aligned(gamma, 4) ||
      !aligned(beta, 4) || !aligned(posted, 8) || !aligned(done, 8) || !aligned(queue_words, 8))
    return GDN_ERR_ALIGN;
  const size_t n = (size_t)ring * B * H * S * D * 2;
  const size_t ns = (size_t)B * H * D * D * sizeof(float);
  if (overlap(out, n, q, n) || overlap(out, n, k, n) || overlap(out, n, v, n) ||
      overlap(out, n, state_in, ns) || overlap(out, n, state_out, ns))
    return GDN_ERR_ALIAS;
  if (state_in && state_out && state_in != state_out && overlap(state_in, ns, state_out, ns))
    return GDN_ERR_ALIAS;
  if (!gdn::stream_supported(B, H, S, D)) return GDN_ERR_UNSUPPORTED;
  gdn::Problem p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.gamma = gamma;
  p.beta = beta;
  p.state_in = state_in;
  p.state_out = state_out;
  p.out = out;
  p.B = B;
  p.H = H;
  p.T = 1;
  p.S = S;
  p.D = D;
  p.key_scale = (float)(1.0 / sqrt((double)D * (double)S));
  p.delta = (flags & GDN_FLAG_NO_DELTA) == 0;
  p.stream = static_cast<cudaStream_t>(stream);
  gdn::StreamQueue qd;
  qd.posted = posted;
  qd.done = done;
  qd.queue_words = queue_words;
  qd.ring = ring;
  qd.idle_timeout_ns = idle_timeout_ns;
  return gdn::launch_stream_bf16(p, qd, rope) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

int gdn_frame_stream(const void* q, const void* k, const void* v, const float* gamma,
                     const float* beta, const float* state_in, float* state_out, void* out, int B,
                     int H, int S, int D, int ring, const unsigned long long* posted,
                     unsigned long long* done, unsigned int* queue_words,
                     unsigned long long idle_timeout_ns, unsigned int flags, void* stream) {
  return stream_impl(q, k, v, gamma, beta, state_in, state_out, out, B, H, S, D, ring, posted, done,
                     queue_words, idle_timeout_ns, flags, stream, nullptr);
}

int gdn_frame_stream_rope(const void* q, const void* k, const void* v, const float* gamma,
                          const float* beta, const float* state_in, float* state_out, void* out,
                          int B, int H, int S, int D, int ring, const unsigned long long* posted,
                          unsigned long long* done, unsigned int* queue_words,
                          unsigned long long idle_timeout_ns, int grid_w, int t0,
                          unsigned int flags, void* stream) {
  if (grid_w < 1 || t0 < 0) return GDN_ERR_SHAPE;
  gdn::RopeParams rp;
  gdn::rope_params(&rp, 64, grid_w, t0);
  return stream_impl(q, k, v, gamma, beta, state_in, state_out, out, B, H, S, D, ring, posted, done,
                     queue_words, idle_timeout_ns, flags, stream, &rp);
}

int gdn_frame_scan_f32(const float* q, const float* k, const float* v, const float* gamma,
                       const float* beta, const float* state_in, float* state_out, float* out,
                       int B, int H, int T, int S, int D, void* stream) {
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, T, S, D, stream, 4);
}

int gdn_frame_step_f32(const float* q, const float* k, const float* v, const float* gamma,
                       const float* beta, const float* state_in, float* state_out, float* out,
                       int B, int H, int S, int D, void* stream) {
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, 1, S, D, stream, 4);
}

int gdn_frame_scan_ex(const void* q, const void* k, const void* v, const float* gamma,
                      const float* beta, const float* state_in, float* state_out, void* out, int B,
                      int H, int T, int S, int D, unsigned int flags, void* stream) {
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, T, S, D, stream, 2, false, flags);
}

int gdn_frame_step_ex(const void* q, const void* k, const void* v, const float* gamma,
                      const float* beta, const float* state_in, float* state_out, void* out, int B,
                      int H, int S, int D, unsigned int flags, void* stream) {
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, 1, S, D, stream, 2, false, flags);
}

int gdn_frame_scan_f32_ex(const float* q, const float* k, const float* v, const float* gamma,
                          const float* beta, const float* state_in, float* state_out, float* out,
                          int B, int H, int T, int S, int D, unsigned int flags, void* stream) {
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, T, S, D, stream, 4, false, flags);
}

int gdn_frame_step_f32_ex(const float* q, const float* k, const float* v, const float* gamma,
                          const float* beta, const float* state_in, float* state_out, float* out,
                          int B, int H, int S, int D, unsigned int flags, void* stream) {
  return run(q, k, v, gamma, beta, state_in, state_out, out, B, H, 1, S, D, stream, 4, false, flags);
}

int gdn_temporal_conv(const void* x, const float* w, const float* bias, const void* cache_in,
                      void* cache_out, void* y, int B, int T, int S, int C, int frames_per_block,
                      void* stream) {
  if (B < 1 || T < 1 || S < 1 || C < 1 || frames_per_block < 1 || C % 8 != 0) return GDN_ERR_SHAPE;
  const double elems = (double)B * T * S * C;
  if (elems > 9.0e18 / 4.0) return GDN_ERR_SHAPE;
  if (!x || !w || !y) return GDN_ERR_NULL;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(cache_in, 16) || !aligned(cache_out, 16) ||
      !aligned(w, 4) || !aligned(bias, 4))
    return GDN_ERR_ALIGN;
  const size_t n = (size_t)B * T * S * C * 2;
  const size_t nc = (size_t)B * S * C * 2;
  if (overlap(y, n, x, n) || overlap(y, n, cache_in, nc) || overlap(y, n, cache_out, nc) ||
      overlap(cache_out, nc, x, n))
    return GDN_ERR_ALIAS;
  if (cache_in && cache_out && cache_in != cache_out && overlap(cache_in, nc, cache_out, nc))
    return GDN_ERR_ALIAS;
  gdn::ConvProblem p;
  p.x = x;
  p.w = w;
  p.bias = bias;
  p.cache_in = cache_in;
  p.cache_out = cache_out;
  p.y = y;
  p.B = B;
  p.T = T;
  p.S = S;
  p.C = C;
  p.F = frames_per_block;
  p.stream = static_cast<cudaStream_t>(stream);
  return gdn::launch_tconv_bf16(p) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_rope3d(const void* x, void* y, int B, int H, int T, int S, int D, int grid_w, int t0,
               void* stream) {
  const int sz = check_sizes(B, H, T, S, D);
  if (sz != GDN_OK) return sz;
  if (grid_w < 1 || t0 < 0 || (long long)t0 + T > 0x7fffffffLL) return GDN_ERR_SHAPE;
  if (!x || !y) return GDN_ERR_NULL;
  if (!aligned(x, 16) || !aligned(y, 16)) return GDN_ERR_ALIGN;
  const size_t n = (size_t)B * H * T * S * D * 2;
  if (x != y && overlap(x, n, y, n)) return GDN_ERR_ALIAS;
  return gdn::launch_rope_bf16(x, y, B, H, T, S, D, grid_w, t0, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? GDN_OK
             : GDN_ERR_CUDA;
}

int gdn_plan(int B, int H, int T, int S, int D, int* kernel, int* ctas_per_head) {
  const int sz = check_sizes(B, H, T, S, D);
  if (sz != GDN_OK) return sz;
  if (!kernel || !ctas_per_head) return GDN_ERR_NULL;
  *kernel = choose_kernel(B, H, T, S, D, ctas_per_head);
  return GDN_OK;
}

int gdn_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return GDN_ERR_CUDA;
  unsigned int st = 0;
  if (gdn::read_status(&st) != cudaSuccess) return GDN_ERR_CUDA;
  return st ? GDN_ERR_TIMEOUT : GDN_OK;
}

const char* gdn_status_string(int status) {
  switch (status) {
    case GDN_OK: return "ok";
    case GDN_ERR_NULL: return "a required pointer is NULL";
    case GDN_ERR_SHAPE: return "B, H, T and S must be >= 1 and the sizes must fit in 64 bits";
    case GDN_ERR_UNSUPPORTED_D: return "D must be 32, 64 or 128";
    case GDN_ERR_ALIGN: return "q, k, v, out and the states must be 16-byte aligned; gamma and beta 4-byte aligned";
    case GDN_ERR_CUDA: return "a CUDA call failed";
    case GDN_ERR_TIMEOUT: return "a device-side wait ran out; outputs of that call are incomplete";
    case GDN_ERR_ALIAS: return "out overlaps an input or a state buffer";
    case GDN_ERR_SCRATCH:
      return "B * H exceeds GDN_NOALLOC_MAX_HEADS (32), the fixed scratch of gdn_frame_scan_noalloc";
    case GDN_ERR_FLAGS: return "flags holds bits other than GDN_FLAG_NO_DELTA";
    case GDN_ERR_UNSUPPORTED:
      return "sizes the call's kernel does not take (gdn_frame_step_rope: D = 64, S <= 1408; "
             "gdn_frame_stream: the same, with every head's cluster resident at once)";
    default: return "unknown gdn_status";
  }
}

int gdn_version(void) {
  return GDN_VERSION_MAJOR * 10000 + GDN_VERSION_MINOR * 100 + GDN_VERSION_PATCH;
}

}  // extern "C"
