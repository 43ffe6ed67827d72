// Row-split single-frame kernel of the frame-wise Gated DeltaNet update, bf16
// inputs, D = 64: one frame per head (T = 1). This is the call of chunk-causal
// rollout, where frames arrive one at a time and each one's latency counts
// ("NVIDIA Apresenta SANA-WM ...", acheiumaia.com.br: the chunk-causal
// autoregressive generator for sequential rollout, and the GDN item of
// section "A Arquitetura").
//
// The update, with s = 1/sqrt(D*S), in the form the scan kernel also uses:
//     M' = gamma M + A' M + c,  A' = -gamma beta s^2 K^T K,  c = beta s K^T V,
//     O  = Q M'.
// A frame is only S x D per tensor, so one CTA per head leaves most SMs idle
// and streams its 450 KB alone. Here a thread-block cluster of P CTAs (P = 2
// or 4) shares each head, and CTA r owns rows [r*chunk, (r+1)*chunk):
//  1. one TMA burst loads its rows of K, V and Q (one box of up to 256 rows
//     per tensor, 128-byte swizzle) and the fp32 state M;
//  2. tcgen05: the partial K^T [K V] over its rows (M = 64, N = 128) into TMEM;
//  3. reduce-scatter over distributed shared memory: CTA q receives every
//     CTA's partial of state rows [q*64/P, (q+1)*64/P), by bulk copies that
//     complete on q's mbarrier;
//  4. CTA q sums them in a fixed order and updates its state rows with the
//     scan kernel's precision: the product A' M on the tensor cores with A'
//     and M rounded to bf16 and fp32 accumulation in TMEM (as M^T A'^T, so
//     that the 64 value columns are the MMA's rows), then gamma M and c added
//     in fp32. It writes those rows of the final state;
//  5. all-gather of M' in bf16 into every CTA of the cluster (bulk copies);
//  6. tcgen05: O = Q M' for its own rows, TMEM -> bf16 -> coalesced stores.
//
// Every wait is bounded. A wait that runs out records the role in the device
// status word and raises an abort flag in every CTA of the cluster; the
// remaining phases are skipped, every CTA drains the copies still in flight
// towards it, and the kernel returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdlib.h>

#include <atomic>

#include "gdn.h"
#include "gdn_internal.h"
#include "gdn_rope.cuh"
#include "gdn_wait.cuh"
#include "sm100_ptx.h"

namespace gdn {
namespace {

using namespace ptx;
using namespace wait;

constexpr int kD = 64;
constexpr int kThreads = 256;
constexpr int kBox = 32;                          // rows: a CTA's chunk is a multiple of this
constexpr int kRowsMax = 352;                     // rows of a frame per CTA
constexpr uint32_t kRegion = kRowsMax * kD * 2;   // 44 KB: one CTA's rows of K, V or Q
constexpr uint32_t kTmemCols = 256;

// Shared memory (from a 1 KB aligned base).
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kRegion;
constexpr uint32_t kOffQ = 2 * kRegion;
constexpr uint32_t kOffM0 = 3 * kRegion;          // M (fp32, 64 x 64), 16 KB
// Reduce-scatter slots, P x (64/P rows) x 256 B (fp32) for each half of the
// partial product: K^T K (A') and K^T V (c).
constexpr uint32_t kOffRedK = kOffM0 + 16384;
constexpr uint32_t kOffRedV = kOffRedK + 16384;
// M in bf16, two buffers of 64 rows x 128 B (128-byte swizzle) by frame parity:
// buffer n & 1 receives the all-gather of frame n's M' (the read-out's operand);
// the other one holds the M that frame n's row update multiplies (M' of frame
// n - 1, or the initial state rounded to bf16 at n = 0).
constexpr uint32_t kOffMg = kOffRedV + 16384;
constexpr uint32_t kMgBytes = 8192;
constexpr uint32_t kOffRope = kOffMg + 2 * kMgBytes;   // 3D RoPE cos/sin tables, 8 KB
constexpr uint32_t kOffMst = kOffRope + 4 * kRopeTabMaxFloats;   // own rows of M' in bf16, <= 4 KB
constexpr uint32_t kOffSendK = kOffMst + 4096;    // the K^T K half staged for its copies, 64 rows x 256 B
constexpr uint32_t kOffBar = kOffSendK + 16384;
enum { kBarKv, kBarQ, kBarMmaK, kBarMmaV, kBarRedK, kBarRedV, kBarU, kBarGather, kBarO, kBarDrain, kNumBars };
constexpr uint32_t kTmemU = 192;   // TMEM columns of the row update's accumulator (after the read-out's)
constexpr uint32_t kOffTmemPtr = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmemPtr + 16;
constexpr uint32_t kOffGo = kOffAbort + 4;         // streaming: the verdict of the wait for a frame
constexpr uint32_t kBytes = kOffAbort + 16;
constexpr uint32_t kSmemAlloc = kBytes + 1024;    // base alignment slack
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kRowsMax % 32 == 0 && kRowsMax <= 512, "at most two load boxes of 16-row multiples");
static_assert(kOffMg % 1024 == 0 && kOffQ % 1024 == 0 && kOffMst % 1024 == 0,
              "swizzled regions are 1 KB aligned");

// Regions reused once the partial product has read K (K region) and V (V region):
constexpr uint32_t kOffAt = kOffK + 16384;        // A' rows in bf16, 128-byte swizzle, <= 4 KB
static_assert(kOffAt % 1024 == 0, "swizzled operand is 1 KB aligned");
// (the own rows of M' have a region of their own: the all-gather copies read
// them while the next frame's loads may already fill the K region)
constexpr uint32_t kOffSendV = kOffV;             // the K^T V half staged, 64 rows x 256 B
// Output tiles (after the gather): tiles 0 and 1 in the V region, tile 2 at the
// start of the K region (free by then; its A' and c rows sit further on).

#ifdef GDN_TRACE
// Phase timeline (globaltimer ns) of the first kTraceHeads heads, per CTA of
// the cluster, for pipeline analysis builds only: [head][rank][event].
constexpr int kTraceHeads = 8, kTraceEvents = 24;
__device__ unsigned long long g_step_trace[kTraceHeads * 4 * kTraceEvents];
#define GDN_STEP_EV_AT(ev, frame_n)                                                              \
  do {                                                                                           \
    if (bh < kTraceHeads && (frame_n) == 0)                                                      \
      g_step_trace[(bh * 4 + (int)rank) * kTraceEvents + (ev)] = globaltimer_ns();               \
  } while (0)
#define GDN_STEP_EV(ev) GDN_STEP_EV_AT(ev, n)
// Streaming launch: [frame][rank][0: frame taken, 1: frame counted done], head 0.
constexpr int kTraceFrames = 64;
__device__ unsigned long long g_stream_trace[kTraceFrames * 4 * 2];
#define GDN_STREAM_EV(ev)                                                              \
  do {                                                                                 \
    if (bh == 0 && n < kTraceFrames)                                                   \
      g_stream_trace[(n * 4 + (int)rank) * 2 + (ev)] = globaltimer_ns();               \
  } while (0)
#else
#define GDN_STEP_EV_AT(ev, frame_n) \
  do {                              \
  } while (0)
#define GDN_STEP_EV(ev) \
  do {                  \
  } while (0)
#define GDN_STREAM_EV(ev) \
  do {                    \
  } while (0)
#endif

// Status bits (shared with the scan kernel's numbering scheme, high bits).
enum : uint32_t {
  kStLoad = 1u << 16, kStMma = 1u << 17, kStRed = 1u << 18, kStGather = 1u << 19,
  kStOut = 1u << 20, kStDrain = 1u << 21, kStConfig = 1u << 22, kStIdle = 1u << 23
};

__device__ __forceinline__ unsigned long long ld_acquire_sys_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_sys_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// tcgen05.ld of N consecutive 32-bit TMEM columns of the warp's 32 lanes
// (N = 8 or 16).
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld_cols<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t (&r)[16]) {
  tmem_ld16(taddr, r);
}

// Split cluster barrier: arrive once this thread's part in the exchanges is
// over, wait only before leaving. The arrive is relaxed: it publishes no data
// (every copy's landing is seen through an mbarrier, and raising the abort
// flag ends with a cluster-scope fence), so it does not wait for this
// thread's global stores to complete.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

struct StepParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  const float* gamma;
  const float* beta;
  const float* state_in;
  float* state_out;
  void* out;                       // [frames][S][64] bf16
  unsigned int* status;
  unsigned long long timeout_ns;   // bound of every wait
  int S;
  int chunk;      // rows per CTA (multiple of 32); CTA r owns [r*chunk, min(S, (r+1)*chunk))
  int lbox;       // rows per TMA load box of q, k and v (chunk / nlb, at most 256)
  int nlb;        // load boxes per tensor and CTA (1 or 2)
  float s;        // key scale 1/sqrt(D*S)
  float s2;       // its square
  float delta;    // 1: delta rule; 0: GDN_FLAG_NO_DELTA (A' = 0)
  int rope;       // 1: rotate Q and K by 3D RoPE in shared memory before use
  RopeParams rp;  // its layout; rp.t0 is the (first) frame's absolute index
  // frame queue (streaming launch only)
  const unsigned long long* posted;   // host-mapped: frames posted; bit 63 set: stop after them
  unsigned long long* done;           // host-mapped: frames every head has completed
  unsigned long long* relay;          // device: CTA 0's copy of `posted`, which every CTA polls
  unsigned int* frame_done;           // device [ring]: CTAs done with the frame in each slot (0 at start)
  int ring;                           // frame slots
  int heads;                          // B * H
  unsigned long long idle_ns;         // bound of the wait for the next frame
};

// Byte offset of 16-byte chunk `chunk` of row `row` in 128-byte rows with the
// 128-byte swizzle (the layout TMA writes and the tcgen05 descriptors read).
__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t chunk) {
  const uint32_t off = row * 128u + chunk * 16u;
  return off ^ (((off >> 7) & 7u) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// kStream = false: one frame (gdn_frame_step). kStream = true: a persistent
// launch that serves frames from a ring of slots as the host posts them (the
// frame queue of gdn_frame_stream), keeping the state on chip between frames.
template <int P, bool kStream>
__global__ void __launch_bounds__(kThreads, 1) gdn_step_kernel(const __grid_constant__ StepParams p) {
  constexpr int R = kD / P;   // state rows this CTA updates
  static_assert(R % 16 == 0, "a warp's 16 rows go to one CTA");
  extern __shared__ uint8_t smem_raw[];
  {
    // Wrong launch shape: record it and touch nothing (uniform over the cluster).
    uint32_t dsmem;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dsmem));
    if (blockDim.x != kThreads || blockDim.y != 1 || blockDim.z != 1 || dsmem < kSmemAlloc ||
        cluster_nctarank() != (uint32_t)P) {
      if (threadIdx.x == 0) atomicOr(p.status, kStConfig);
      return;
    }
  }
  const uint32_t sb = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int bh = blockIdx.x / P;
  const int r0 = (int)rank * p.chunk;
  const int r1 = min(p.S, r0 + p.chunk);
  const int nrows = max(0, r1 - r0);
  const int nbox = (nrows + kBox - 1) / kBox;
  const int nq = (nrows + 127) / 128;   // 128-row read-out tiles
  auto bar = [&](int i) -> uint32_t { return sb + kOffBar + 8u * i; };
  Ctl ctl{sb + kOffAbort, p.status, p.timeout_ns, P};
  if (threadIdx.x == 0) GDN_STEP_EV_AT(10, 0);   // kernel entry

  // The initial state arrives with the first frame's K and V (single frame:
  // one bulk copy counted on the same barrier) or is copied by the threads
  // (streaming launch, once).
  const bool state_bulk = !kStream && p.state_in != nullptr;
  // Issues the TMA loads of this CTA's rows of frame `frame` (thread 0).
  // A CTA with rows loads all of its chunk (rows past S read as zeros) in
  // p.nlb boxes per tensor: few TMA instructions, so the loads go out at once.
  // Q is needed only by the read-out: without RoPE (which turns Q and K
  // together) its loads go out once K and V have landed, so that K and V do
  // not share the memory bandwidth with it.
  const uint32_t tile_bytes = nbox > 0 ? (uint32_t)(p.nlb * p.lbox) * 128u : 0u;
  const bool q_later = !p.rope;
  auto issue_q = [&](int frame) {
    const uint64_t pol = policy_evict_first();   // read once
    mbar_arrive_expect_tx(bar(kBarQ), tile_bytes);
    for (int b = 0; b < p.nlb; ++b)
      tma_load_3d_hint(sb + kOffQ + (uint32_t)(b * p.lbox) * 128u, &p.tm_q, bar(kBarQ), 0,
                       r0 + b * p.lbox, frame, pol);
  };
  auto issue_loads = [&](int frame) {
    if (state_bulk) {
      mbar_arrive_expect_tx(bar(kBarKv), 2u * tile_bytes + kD * kD * 4u);
      bulk_load_global(sb + kOffM0, p.state_in + (size_t)bh * kD * kD, kD * kD * 4u, bar(kBarKv));
    } else if (nbox > 0) {
      mbar_arrive_expect_tx(bar(kBarKv), 2u * tile_bytes);
    }
    if (nbox > 0) {
      const uint64_t pol = policy_evict_first();   // read once
      for (int b = 0; b < p.nlb; ++b) {
        const uint32_t off = (uint32_t)(b * p.lbox) * 128u;
        tma_load_3d_hint(sb + kOffK + off, &p.tm_k, bar(kBarKv), 0, r0 + b * p.lbox, frame, pol);
        tma_load_3d_hint(sb + kOffV + off, &p.tm_v, bar(kBarKv), 0, r0 + b * p.lbox, frame, pol);
      }
      if (!q_later) issue_q(frame);
    }
  };
  // A single frame is launched with programmatic stream serialization: the
  // next launch on the stream may start as soon as every CTA of this one has
  // started, and does its setup while this one runs; each launch reads no
  // global memory before the grid ahead of it on the stream has completed
  // (griddepcontrol.wait), so whatever kernel precedes it, it sees its writes.
  if (!kStream) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 32) {   // the maps are launch parameters: fetch them ahead of the first copy
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    prefetch_tmap(&p.tm_q);
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(ctl.abort_addr), "r"(0u) : "memory");
    fence_mbar_init();
    GDN_STEP_EV_AT(16, 0);   // barriers initialised
  }
  if (!kStream) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) GDN_STEP_EV_AT(17, 0);   // the grid ahead has completed
    if (threadIdx.x == 0) issue_loads(bh);   // a single frame is known now: start its loads at once
  }
  if (threadIdx.x == 0) GDN_STEP_EV_AT(12, 0);   // loads issued
  // Generic pointer to the aligned shared memory, for plain loads and stores
  // the compiler may schedule.
  float* const smf = reinterpret_cast<float*>(smem_raw + (sb - smem_u32(smem_raw)));
  // The initial state, whole, in every CTA. A single frame takes it by the
  // bulk copy above, which lands before this CTA's partial product can go out,
  // so every CTA has read it before any CTA writes the final state (after all
  // partials are in): state_in == state_out is safe. Otherwise the threads
  // copy it here (or write zeros), before the first cluster barrier.
  if (!state_bulk) {
    constexpr int kPer = kD * kD / 4 / kThreads;   // float4 per thread
    float4 x[kPer];
    const float4* src = reinterpret_cast<const float4*>(p.state_in + (size_t)bh * kD * kD);
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      x[i] = p.state_in ? src[threadIdx.x + i * kThreads] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4* m0 = reinterpret_cast<float4*>(smf + kOffM0 / 4);
#pragma unroll
    for (int i = 0; i < kPer; ++i) m0[threadIdx.x + i * kThreads] = x[i];
  }
  if (warp == 0) {
    tmem_alloc(sb + kOffTmemPtr, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) GDN_STEP_EV_AT(13, 0);   // TMEM allocated, state in place
  cluster_sync();   // every CTA's barriers are initialised
  if (threadIdx.x == 0) GDN_STEP_EV_AT(11, 0);   // past the first cluster barrier
  const uint32_t tmem = ld_shared_u32(sb + kOffTmemPtr);
  bool issued_mma = false;
  int last = -1;          // the last frame started (its barrier phases may be in flight)
  bool loads_issued = false;
  bool q_issued = false;  // thread 0: the Q loads of the last frame started went out

  for (int n = 0;; ++n) {
    const uint32_t ph = (uint32_t)(n & 1);   // phase parity of every per-frame barrier
    if (threadIdx.x == 0) GDN_STEP_EV(0);
    int frame = bh;                          // index along the tensors' frame axis
    if (kStream) {
      // ------------------------------------------------------------ 0. next frame or stop
      // Only CTA 0 reads the host's counter (PCIe); it relays the value into
      // device memory, which every CTA polls in L2. Many CTAs reading host
      // memory at once would queue their reads behind each other.
      if (threadIdx.x == 0) {
        uint32_t go = 0;
        const uint64_t t0 = globaltimer_ns();
        while (true) {
          unsigned long long v = ld_acquire_gpu_u64(p.relay);
          if (blockIdx.x == 0) {
            const unsigned long long h = ld_acquire_sys_u64(p.posted);
            if (h != v) {
              st_release_gpu_u64(p.relay, h);
              v = h;
            }
          }
          if ((v & ~(1ull << 63)) > (unsigned long long)n) { go = 1; break; }
          if (v >> 63) break;                                   // stop after the posted frames
          if (aborted(ctl)) break;
          if (globaltimer_ns() - t0 > p.idle_ns) { raise_abort(ctl, kStIdle); break; }
          __nanosleep(64);
        }
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sb + kOffGo), "r"(go) : "memory");
        GDN_STREAM_EV(0);
      }
      __syncthreads();
      if (ld_shared_u32(sb + kOffGo) == 0 || aborted(ctl)) break;
      frame = (n % p.ring) * p.heads + bh;
    } else if (n > 0) {
      break;
    }
    last = n;
    // plain loads: in a frame queue the host refills slots between frames
    const float g = *reinterpret_cast<const volatile float*>(p.gamma + frame);
    const float be = *reinterpret_cast<const volatile float*>(p.beta + frame);

    // -------------------------------------------------------------- 1. loads of the frame
    // The exchange barriers are armed here. A peer's data for this frame can
    // only come after this CTA completed the previous frame's exchanges, so an
    // early bulk copy finds the barrier in this frame's phase (its byte count
    // runs ahead of the arming, which the barrier allows).
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(bar(kBarRedK), (uint32_t)(P * R * 256));
      mbar_arrive_expect_tx(bar(kBarRedV), (uint32_t)(P * R * 256));
      mbar_arrive_expect_tx(bar(kBarGather), (uint32_t)(kD * 128));
      if (kStream) issue_loads(frame);   // a single frame's loads went out in the prologue
      loads_issued = nbox > 0 || state_bulk;
      q_issued = nbox > 0 && !q_later;
    }

    // -------------------------------------------------------------- 1b. 3D RoPE (optional)
    // Q and K turned in place once they land, before any MMA reads them. The
    // swizzle only permutes whole 16-byte chunks of a row, and a chunk holds 4
    // whole pairs: physical chunk c of local row rho is logical chunk c ^ (rho & 7).
    if (p.rope && nbox > 0) {
      // cos/sin tables of this frame and of the grid rows this CTA's tiles
      // touch (zero-filled rows past S included), built while the tiles land
      const int hlo = r0 / p.rp.grid_w;
      const int nh = (r0 + nbox * kBox - 1) / p.rp.grid_w - hlo + 1;
      const bool tab = rope_tab_floats(p.rp, nh) <= kRopeTabMaxFloats;
      float* rtab = reinterpret_cast<float*>(smem_raw + (sb - smem_u32(smem_raw)) + kOffRope);
      if (tab) rope_tab_build(p.rp, rtab, p.rp.t0 + n, hlo, nh);
      const bool kv_ok = warp_wait(bar(kBarKv), ph, ctl, kStLoad);
      const bool q_ok = warp_wait(bar(kBarQ), ph, ctl, kStLoad);
      if (kv_ok && q_ok) {
        const int nchunks = nbox * kBox * 8;
        for (int e = threadIdx.x; e < 2 * nchunks; e += kThreads) {
          const int which = e / nchunks;             // 0: K, 1: Q
          const int ce = e - which * nchunks;
          const int rho = ce >> 3, cp = ce & 7;
          const uint32_t addr = sb + (which ? kOffQ : kOffK) + (uint32_t)rho * 128u + (uint32_t)cp * 16u;
          uint4 v = ld_shared_u4(addr);
          if (tab)
            rope_chunk_tab(p.rp, rtab, hlo, nh, r0 + rho, cp ^ (rho & 7), v);
          else
            rope_chunk(p.rp, p.rp.t0 + n, r0 + rho, cp ^ (rho & 7), v);
          st_shared_v4(addr, v);
        }
        fence_proxy_async_cta();   // rotated tiles visible to the tensor cores
      }
      __syncthreads();
    }

    // -------------------------------------------------------------- 2. partial K^T [K V]
    if (warp == 1 && lane == 0 && nbox > 0) {
      if (wait_bar(bar(kBarKv), ph, ctl, kStLoad)) {
        tc_fence_after();
        // A = K^T (M = 64 key dims, one 128-byte atom), B = K, then V (N = 64);
        // MN-major views of the row-major tiles; 16 rows per MMA. K^T K goes
        // first, into TMEM columns 0-63, and is committed on its own, so that
        // its exchange (and A') starts while K^T V (columns 64-127) still runs.
        constexpr uint32_t idesc = idesc_bf16(64, 64, 1, 1);
        for (int kk = 0; kk < 2 * nbox; ++kk) {
          const uint64_t a = smem_desc(sb + kOffK + kk * 2048, kRegion, 1024, 2);
          mma_bf16(tmem, a, a, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(kBarMmaK));
        for (int kk = 0; kk < 2 * nbox; ++kk) {
          const uint64_t a = smem_desc(sb + kOffK + kk * 2048, kRegion, 1024, 2);
          const uint64_t b = smem_desc(sb + kOffV + kk * 2048, kRegion, 1024, 2);
          mma_bf16(tmem + 64, a, b, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(kBarMmaV));
        issued_mma = true;
        GDN_STEP_EV(1);   // K and V landed, partial product issued
      }
    }
    // Q of the frame once K and V have landed (thread 0, which also drains it
    // on an abort).
    if (q_later && threadIdx.x == 0 && nbox > 0 && wait_bar(bar(kBarKv), ph, ctl, kStLoad)) {
      issue_q(frame);
      q_issued = true;
    }

    // -------------------------------------------------------------- 3. reduce-scatter
    // With M = 64 the accumulator row i (key dim) sits in TMEM lane 32(i/16) + i%16:
    // warp w (< 4) reads lanes 32w.., and its lanes 0-15 hold key rows 16w..16w+15,
    // columns 0-63 = K^T K, 64-127 = K^T V. For each half in turn, those 16 rows
    // (4 KB of fp32) go to the CTA that updates them, staged with chunk c of row
    // i at chunk c ^ (i & 7): K^T K in its own area, K^T V in the V region once
    // K^T V is done.
    if (warp < 4) {
      const int il = lane & 15;
      const uint32_t dst = (uint32_t)(warp * P / 4);
      const uint32_t slot_row = rank * R + (uint32_t)((warp * 16) % R);
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const bool ok = nbox == 0 || warp_wait(bar(h ? kBarMmaV : kBarMmaK), ph, ctl, kStMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t send = sb + (h ? kOffSendV : kOffSendK) + (uint32_t)warp * 16u * 256u;
        uint32_t v[64];
        if (nbox > 0) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r16[16];
            tmem_ld16(tmem + 64 * h + 16 * c + ((uint32_t)(warp * 32) << 16), r16);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[16 * c + e] = r16[e];
          }
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e) v[e] = 0u;
        }
        if (lane < 16) {
#pragma unroll
          for (int c = 0; c < 16; ++c)
            st_shared_v4(send + (uint32_t)il * 256u + (((uint32_t)c ^ (uint32_t)(il & 7)) << 4),
                         make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]));
        }
        tc_fence_before();
        fence_proxy_async_cta();   // staged rows visible to the bulk copy
        __syncwarp();
        if (lane == 0) {
          if (warp == 0 && h == 0) GDN_STEP_EV(2);   // K^T K half staged
          bulk_copy_to_cluster(mapa(sb + (h ? kOffRedV : kOffRedK) + slot_row * 256u, dst), send, 16u * 256u,
                               mapa(bar(h ? kBarRedV : kBarRedK), dst));
        }
      }
    }

    // The first frame's row update multiplies the state rounded to bf16 (later
    // frames take the gathered M' of the frame before). Warps 4-7 round it into
    // the other M buffer, in the operand layout, while warps 0-3 stage the
    // partials, once the bulk-copied state has landed.
    const uint32_t mg_in = sb + kOffMg + (ph ^ 1u) * kMgBytes;   // M of this frame's update
    const uint32_t mg_out = sb + kOffMg + ph * kMgBytes;         // M' of this frame (gathered)
    bool m0r_ok = true;
    if (n == 0 && warp >= 4) {
      if (state_bulk) m0r_ok = warp_wait(bar(kBarKv), 0, ctl, kStLoad);
      if (m0r_ok && !aborted(ctl)) {
        for (int e = threadIdx.x - 128; e < kD * kD / 2; e += kThreads - 128) {
          const int row = e >> 5, j = (e & 31) * 2;
          const float2 m = *reinterpret_cast<const float2*>(smf + kOffM0 / 4 + row * kD + j);
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(mg_in + swz128((uint32_t)row, (uint32_t)(j >> 3)) +
                                                    (uint32_t)(j & 7) * 2u),
                       "r"(pack_bf16x2(m.x, m.y))
                       : "memory");
        }
        fence_proxy_async_cta();   // visible to the tensor cores
      }
    }

    // -------------------------------------------------------------- 4. recurrence, own rows
    // A' first: it needs only the K^T K half, and its product with M runs
    // while the K^T V half is still on its way.
    bool red_ok = warp_wait(bar(kBarRedK), ph, ctl, kStRed) && m0r_ok;
    // the bulk-copied initial state has landed (a CTA without rows has not
    // waited on that barrier yet)
    if (state_bulk && n == 0 && warp < 4) red_ok = warp_wait(bar(kBarKv), 0, ctl, kStLoad) && red_ok;
    if (threadIdx.x == 0) GDN_STEP_EV(3);   // every K^T K partial received
    __syncthreads();   // also orders warps 0-3's view of the finished MMAs before the K region is reused
    if (red_ok && !aborted(ctl)) {
      // Sum of the P partials of K^T K (fixed order), one 16-byte chunk (4
      // columns) of a row at a time: A' = -gamma beta s^2 K^T K (0 without
      // delta), rounded to bf16 into the update's K-major operand.
      const float coef = -g * be * p.s2 * p.delta;
      for (int e = threadIdx.x; e < R * 16; e += kThreads) {
        const int il = e >> 4, cc = e & 15;
        const uint32_t phys = (uint32_t)((cc ^ (il & 7)) << 4);
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int src = 0; src < P; ++src) {
          const float4 x = ld_shared_f4(sb + kOffRedK + (uint32_t)(src * R + il) * 256u + phys);
          sum.x += x.x;
          sum.y += x.y;
          sum.z += x.z;
          sum.w += x.w;
        }
        const uint32_t addr = sb + kOffAt + swz128((uint32_t)il, (uint32_t)(cc >> 1)) + (uint32_t)(cc & 1) * 8u;
        asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr),
                     "r"(pack_bf16x2(coef * sum.x, coef * sum.y)), "r"(pack_bf16x2(coef * sum.z, coef * sum.w))
                     : "memory");
      }
      fence_proxy_async_cta();   // A' visible to the tensor cores
    }
    __syncthreads();
    if (threadIdx.x == 0) GDN_STEP_EV(14);   // A' ready
    // The product A' M on the tensor cores, transposed so that the 64 value
    // columns j are the MMA's rows: D = M^T A'^T (M = 64, N = R, K = 64), with
    // M (bf16, row-major [k][j]) as the MN-major A operand and the A' rows as
    // the K-major B operand; fp32 accumulation in TMEM. Row j of D sits in
    // TMEM lane 32 (j / 16) + j % 16.
    const bool upd_mma = p.delta != 0.f;
    if (warp == 1 && lane == 0 && upd_mma && red_ok && !aborted(ctl)) {
      tc_fence_after();
      constexpr uint32_t id_u = idesc_bf16(64, R, 1, 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t a = smem_desc(mg_in + kk * 2048, kMgBytes, 1024, 2);
        const uint64_t b = smem_desc(sb + kOffAt + kk * 32, 16, 1024, 2);
        mma_bf16(tmem + kTmemU, a, b, id_u, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar(kBarU));
      issued_mma = true;
    }
    {
      // M' = gamma M + A' M + c, with c = beta s K^T V summed here from the
      // second half's P partials (fixed order) in fp32.
      const bool v_ok = red_ok && warp_wait(bar(kBarRedV), ph, ctl, kStRed);
      const bool u_ok = v_ok && (!upd_mma || warp_wait(bar(kBarU), ph, ctl, kStMma));
      const bool go = __shfl_sync(0xffffffffu, (u_ok && !aborted(ctl)) ? 1 : 0, 0) != 0;
      if (go) {
        // Warp w reads lanes of TMEM subpartition w % 4: its lanes 0-15 hold
        // value columns j = 16 (w % 4) + lane; warps 0-3 take the CTA's rows
        // il < R / 2, warps 4-7 the rest.
        constexpr int H = R / 2;
        const int half = warp >> 2, sub = warp & 3;
        float acc[H];
        if (upd_mma) {
          tc_fence_after();
          uint32_t r[H];
          tmem_ld_cols<H>(tmem + kTmemU + (uint32_t)(half * H) + ((uint32_t)(sub * 32) << 16), r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < H; ++i) acc[i] = __uint_as_float(r[i]);
        } else {
#pragma unroll
          for (int i = 0; i < H; ++i) acc[i] = 0.f;
        }
        if (lane < 16) {
          const int j = sub * 16 + lane;
          const float cbs = be * p.s;
#pragma unroll
          for (int i = 0; i < H; ++i) {
            const int il = half * H + i;
            const int gi = (int)rank * R + il;
            const uint32_t col = (uint32_t)((((j >> 2) ^ (il & 7)) << 4) + (j & 3) * 4);
            float sum = 0.f;
#pragma unroll
            for (int src = 0; src < P; ++src)
              sum += ld_shared_f32(sb + kOffRedV + (uint32_t)(src * R + il) * 256u + col);
            const float m0 = smf[kOffM0 / 4 + gi * kD + j];
            const float m1 = fmaf(g, m0, acc[i]) + __fmul_rn(cbs, sum);   // c rounded on its own
            if (kStream) smf[kOffM0 / 4 + gi * kD + j] = m1;   // kept on chip
            if (!kStream && p.state_out) p.state_out[((size_t)bh * kD + gi) * kD + j] = m1;
            // bf16 copy of the row, in the swizzled layout of the read-out's operand
            st_shared_u16(sb + kOffMst + swz128((uint32_t)il, (uint32_t)(j >> 3)) + (uint32_t)(j & 7) * 2u,
                          __bfloat16_as_ushort(__float2bfloat16_rn(m1)));
          }
        }
        tc_fence_before();
      }
    }
    fence_proxy_async_cta();   // M' rows visible to the bulk copies
    __syncthreads();
    // -------------------------------------------------------------- 5. all-gather of M' (bf16)
    if (threadIdx.x == 0) GDN_STEP_EV(4);   // own rows of M' ready
    if (threadIdx.x == 0 && red_ok && !aborted(ctl)) {
      for (int d = 0; d < P; ++d)
        bulk_copy_to_cluster(mapa(mg_out + rank * (uint32_t)R * 128u, (uint32_t)d), sb + kOffMst,
                             (uint32_t)R * 128u, mapa(bar(kBarGather), (uint32_t)d));
    }

    // -------------------------------------------------------------- 6. read-out O = Q M'
    if (warp == 1 && lane == 0 && nq > 0) {
      if (wait_bar(bar(kBarGather), ph, ctl, kStGather) && wait_bar(bar(kBarQ), ph, ctl, kStLoad)) {
        tc_fence_after();
        GDN_STEP_EV(5);   // gathered M' and Q present
        constexpr uint32_t id_o = idesc_bf16(128, 64, 0, 1);   // Q K-major, M' MN-major
        for (int i = 0; i < nq; ++i) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = smem_desc(sb + kOffQ + i * 16384 + kk * 32, 16, 1024, 2);
            const uint64_t b = smem_desc(mg_out + kk * 2048, kMgBytes, 1024, 2);
            mma_bf16(tmem + 64 * i, a, b, id_o, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(bar(kBarO));
        issued_mma = true;
      }
    }
    // A CTA without rows of the frame issues no read-out, but peers still copy
    // M' into it: it sees those copies land before it may leave.
    if (!kStream && nq == 0 && threadIdx.x == 0 && red_ok && !aborted(ctl))
      wait_bar(bar(kBarGather), ph, ctl, kStGather);
    // Output tiles: warps 4g..4g+3 take tiles g, g + 2, ...; lane l of warp
    // quarter q holds tile row 32q + l.
    {
      const int grp = warp >> 2;
      const int qd = warp & 3;
      const bool ok = grp < nq && warp_wait(bar(kBarO), ph, ctl, kStOut);
      // A single frame: past this point the thread neither writes into a peer
      // nor waits on anything a peer sends (no wait is left that could raise
      // the abort flag in the cluster), and every copy into this CTA has been
      // seen to land (the partials by every thread, the gathered M' by warp 1,
      // or thread 0 above). It arrives on the closing cluster barrier now and
      // waits on it only before leaving, so the barrier's latency overlaps
      // the read-out.
      if (!kStream) cluster_arrive_relaxed();
      if (grp < nq && ok) {
        tc_fence_after();
        const uint64_t pol = policy_evict_first();   // written once
        uint4* const outp = reinterpret_cast<uint4*>(p.out);
        for (int i = grp; i < nq; i += 2) {
          uint32_t v[64];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r16[16];
            tmem_ld16(tmem + 64 * i + 16 * c + ((uint32_t)(qd * 32) << 16), r16);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[16 * c + e] = r16[e];
          }
          tmem_wait_ld();
          // Each warp stages its own 32 rows (bf16, swizzled against bank
          // conflicts) and reads them back with lane L on 16-byte chunk L % 8
          // of row 4u + L / 8, so that every store instruction writes four
          // whole 128-byte rows of out.
          const uint32_t tile = sb + (i < 2 ? kOffV + (uint32_t)i * 16384u : kOffK);
          const uint32_t row = (uint32_t)(qd * 32 + lane);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * c + 0]), __uint_as_float(v[8 * c + 1]));
            w.y = pack_bf16x2(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3]));
            w.z = pack_bf16x2(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5]));
            w.w = pack_bf16x2(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]));
            st_shared_v4(tile + swz128(row, (uint32_t)c), w);
          }
          __syncwarp();
          if (warp == 0 && lane == 0 && i == 0) GDN_STEP_EV(6);   // output tile staged
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t rr = (uint32_t)(qd * 32 + 4 * u + (lane >> 3));
            const int y = r0 + 128 * i + (int)rr;
            if (y < r1)
              st_global_v4_hint(outp + ((size_t)frame * p.S + y) * 8 + (lane & 7),
                                ld_shared_u4(tile + swz128(rr, (uint32_t)(lane & 7))), pol);
          }
        }
        tc_fence_before();
        if (kStream) __threadfence();   // the frame is done only once its rows are written
        if (warp == 0 && lane == 0) GDN_STEP_EV(7);   // stores issued
      }
    }
    if (!kStream) continue;

    // -------------------------------------------------------------- 7. frame done (stream)
    // The next frame's row update multiplies this frame's gathered M' (buffer
    // n & 1) in place: it has landed in this CTA before the frame counts as
    // done. The next frame's M' goes to the other buffer, and no peer can send
    // frame n + 2's M' into this one before this CTA's update of frame n + 1 is
    // complete (the peers first need its partial product of frame n + 2).
    warp_wait(bar(kBarGather), ph, ctl, kStGather);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0 && !aborted(ctl)) {
      // Every CTA of every head counts itself done with the slot; the last one
      // resets the count and tells the host.
      __threadfence();
      const unsigned int total = (unsigned int)(p.heads * P);
      const unsigned int slot = (unsigned int)(n % p.ring);
      GDN_STREAM_EV(1);
      if (atomicAdd(p.frame_done + slot, 1u) == total - 1u) {
        p.frame_done[slot] = 0u;
        __threadfence_system();
        st_release_sys_u64(p.done, (unsigned long long)(n + 1));
      }
    }
  }

  // ---------------------------------------------------------------- exit
  if (threadIdx.x == 0) GDN_STEP_EV_AT(8, 0);   // frame loop left
  if (kStream && p.state_out && !aborted(ctl)) {
    // this CTA's rows of the final state, fp32, kept on chip across the frames
    for (int e = threadIdx.x; e < R * kD; e += kThreads) {
      const int gi = (int)rank * R + e / kD;
      p.state_out[((size_t)bh * kD + gi) * kD + (e % kD)] =
          ld_shared_f32(sb + kOffM0 + (uint32_t)(gi * kD + e % kD) * 4u);
    }
  }
  if (warp == 1 && lane == 0 && issued_mma) {   // every MMA done before TMEM is freed
    mma_commit(bar(kBarDrain));
    drain_bar(bar(kBarDrain), 0, ctl, kStDrain);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) GDN_STEP_EV_AT(15, 0);   // MMAs drained
  // Normal path: every copy into each CTA has landed (each saw it land before
  // arriving). A single frame arrived on this barrier during its read-out.
  if (kStream)
    cluster_sync();
  else
    cluster_wait_acquire();
  if (aborted(ctl)) {
    // Same verdict in every CTA (the flag is raised in all of them before the
    // raising thread arrives on the barrier above). Let copies still in flight
    // land before any CTA of the cluster leaves: loads issued here, and bulk
    // copies from peers (all issued before that barrier), in the phase of the
    // last frame started.
    if (threadIdx.x == 0 && last >= 0) {
      const uint32_t ph = (uint32_t)(last & 1);
      if (loads_issued) {
        drain_bar(bar(kBarKv), ph, ctl, kStDrain);
        if (q_issued) drain_bar(bar(kBarQ), ph, ctl, kStDrain);
      }
      drain_bar(bar(kBarRedK), ph, ctl, kStDrain);
      drain_bar(bar(kBarRedV), ph, ctl, kStDrain);
      drain_bar(bar(kBarGather), ph, ctl, kStDrain);
    }
    __syncthreads();
    cluster_sync();
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) GDN_STEP_EV_AT(9, 0);   // end
}

// ------------------------------------------------------------------ host side

template <int P, bool kStream>
cudaError_t prepare() {
  static std::atomic<bool> done[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(reinterpret_cast<const void*>(&gdn_step_kernel<P, kStream>),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

int chunk_rows(int S, int P) {
  const int per = (S + P - 1) / P;
  return (per + kBox - 1) / kBox * kBox;
}

// attr holds 2 entries; the single-frame launch also allows programmatic
// stream serialization (see the kernel's prologue).
template <int P, bool kStream>
cudaLaunchConfig_t launch_config(long long heads, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)(heads * P), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = kStream ? 1 : 2;
  return cfg;
}

// Fills the parameters common to both modes; frames = the tensors' frame axis.
template <int P>
cudaError_t fill_params(StepParams* p, const Problem& pr, long long frames, const RopeParams* rope) {
  p->chunk = chunk_rows(pr.S, P);
  if (p->chunk > kRowsMax) return cudaErrorInvalidValue;
  // Load boxes: at most 256 rows (the TMA box limit), a multiple of 16 rows so
  // that each box starts on a 1 KB (swizzle period) boundary.
  p->nlb = (p->chunk + 255) / 256;
  p->lbox = p->chunk / p->nlb;
  if (!make_frame_map(&p->tm_q, pr.q, kD, pr.S, frames, p->lbox) ||
      !make_frame_map(&p->tm_k, pr.k, kD, pr.S, frames, p->lbox) ||
      !make_frame_map(&p->tm_v, pr.v, kD, pr.S, frames, p->lbox))
    return cudaErrorInvalidValue;
  p->status = status_word();
  if (!p->status) return cudaErrorInvalidDevice;
  p->gamma = pr.gamma;
  p->beta = pr.beta;
  p->state_in = pr.state_in;
  p->state_out = pr.state_out;
  p->out = pr.out;
  p->timeout_ns = wait_budget_ns();
  p->S = pr.S;
  p->s = pr.key_scale;
  p->s2 = (float)(1.0 / ((double)kD * (double)pr.S));
  p->delta = pr.delta ? 1.f : 0.f;
  p->rope = rope ? 1 : 0;
  if (rope) p->rp = *rope;
  else rope_params(&p->rp, kD, 1, 0);
  p->posted = nullptr;
  p->done = nullptr;
  p->relay = nullptr;
  p->frame_done = nullptr;
  p->ring = 1;
  p->heads = pr.B * pr.H;
  p->idle_ns = 0;
  return cudaSuccess;
}

template <int P>
cudaError_t launch_p(const Problem& pr, const RopeParams* rope) {
  cudaError_t e = prepare<P, false>();
  if (e != cudaSuccess) return e;
  StepParams p;
  e = fill_params<P>(&p, pr, (long long)pr.B * pr.H, rope);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = launch_config<P, false>((long long)pr.B * pr.H, pr.stream, attr);
  return cudaLaunchKernelEx(&cfg, gdn_step_kernel<P, false>, p);
}

// Clusters of the streaming kernel that can be resident at once (every head's
// cluster must be, since each waits for frames the others complete).
int stream_resident_clusters() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return -1;
  }
  const int known = cache[dev].load(std::memory_order_acquire);
  if (known != 0) return known - 2;
  int n = -1;
  if (prepare<4, true>() == cudaSuccess) {
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = launch_config<4, true>(64, nullptr, attr);
    if (cudaOccupancyMaxActiveClusters(&n, gdn_step_kernel<4, true>, &cfg) != cudaSuccess) n = -1;
  }
  cudaGetLastError();
  cache[dev].store(n + 2, std::memory_order_release);
  return n;
}

}  // namespace

int step_rows_max() { return kRowsMax; }

int step_ctas_per_head(int B, int H, int T, int S, int D) {
  if (D != kD || T != 1) return 0;
  const long long heads = (long long)B * H;
  if (heads * 4 > (1ll << 31) - 1) return 0;
  int P = 4;
  // Tuning override: GDN_STEP_CTAS=2|4 forces the cluster size; 0 turns this
  // kernel off (single frames then run on the scan kernels).
  if (const char* e = getenv("GDN_STEP_CTAS")) {
    const int v = atoi(e);
    if (e[0] == '0' && v == 0) return 0;
    if (v == 2 || v == 4) P = v;
  }
  if (chunk_rows(S, P) > kRowsMax) P = 4;
  if (chunk_rows(S, P) > kRowsMax) return 0;
  return P;
}

cudaError_t launch_step_bf16(const Problem& p, int ctas_per_head, const RopeParams* rope) {
  if (p.T != 1 || p.D != kD) return cudaErrorInvalidValue;
  switch (ctas_per_head) {
    case 2: return launch_p<2>(p, rope);
    case 4: return launch_p<4>(p, rope);
    default: return cudaErrorInvalidValue;
  }
}

int stream_supported(int B, int H, int S, int D) {
  if (D != kD || chunk_rows(S, 4) > kRowsMax) return 0;
  const int fit = stream_resident_clusters();
  const long long heads = (long long)B * H;
  return heads <= (fit >= 0 ? fit : 148 / 4) ? 1 : 0;
}

cudaError_t launch_stream_bf16(const Problem& pr, const StreamQueue& q, const RopeParams* rope) {
  cudaError_t e = prepare<4, true>();
  if (e != cudaSuccess) return e;
  StepParams p;
  e = fill_params<4>(&p, pr, (long long)q.ring * pr.B * pr.H, rope);
  if (e != cudaSuccess) return e;
  p.posted = q.posted;
  p.done = q.done;
  p.relay = reinterpret_cast<unsigned long long*>(q.queue_words);
  p.frame_done = q.queue_words + 2;
  p.ring = q.ring;
  p.idle_ns = q.idle_timeout_ns;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = launch_config<4, true>((long long)pr.B * pr.H, pr.stream, attr);
  return cudaLaunchKernelEx(&cfg, gdn_step_kernel<4, true>, p);
}

#ifdef GDN_TRACE
extern "C" __attribute__((visibility("default"))) int gdn_trace_stream_copy(void* dst, size_t bytes) {
  const size_t n = sizeof(g_stream_trace) < bytes ? sizeof(g_stream_trace) : bytes;
  return cudaMemcpyFromSymbol(dst, g_stream_trace, n) == cudaSuccess ? (int)n : -1;
}
extern "C" __attribute__((visibility("default"))) int gdn_trace_step_copy(void* dst, size_t bytes) {
  const size_t n = sizeof(g_step_trace) < bytes ? sizeof(g_step_trace) : bytes;
  return cudaMemcpyFromSymbol(dst, g_step_trace, n) == cudaSuccess ? (int)n : -1;
}
#endif

}  // namespace gdn
