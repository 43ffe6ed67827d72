// tcgen05 scan of the frame-wise Gated DeltaNet over every SM of the GPU,
// bf16 inputs, D = 64.
//
// The update ("NVIDIA Apresenta SANA-WM ...", acheiumaia.com.br, section
// "A Arquitetura", item "1. Atencao Linear Hibrida com Gated DeltaNet"), per
// head and frame t with s = 1/sqrt(D*S):
//     W = (sK) M,  R = V - gamma W,  M' = gamma M + beta (sK)^T R,  O = Q M',
// taken in the form M' = gamma M + A' M + c, A' = -gamma beta s^2 K^T K,
// c = beta s K^T V, with the arithmetic of the cluster kernel (gdn_tc.cu):
// A' and M enter their product as bf16, gamma M and c are added in fp32, the
// fp32 state stays in registers across all frames.
//
// What differs is where the work runs. The cluster kernel gives each head P
// CTAs that produce the head's transition operands (A', c) themselves; with
// 32 heads of 4 CTAs that leaves 20 of 148 SMs idle, and the head whose SMs
// stream slowest sets the time. Here one persistent CTA runs on every SM
// (a cooperative launch, so all are resident):
//  * head CTAs: P per head (P * heads <= SMs). Each runs the whole recurrence
//    of its head on its own copy of the state and reads out its block of
//    rows of every frame, as in the cluster kernel;
//  * every CTA, head CTAs included, produces transition operands: it claims
//    frames from per-head counters in global memory, streams their K and V
//    (TMA), forms [K V]^T K on the tensor cores and writes A' and c to a ring
//    in global memory (16 frames per head, kept in L2), published with a
//    release flag. A head CTA takes frames of its own head while there are
//    any; the other CTAs ("helpers") take frames of the head with the fewest
//    frames claimed, so spare SMs go where production lags. A producer claims
//    a frame only once every CTA of its head has loaded the frame 16 before
//    it (the ring slot is then free), so no ring wait can block on itself;
//  * helpers spend the shared memory of the head roles on K/V tiles in flight
//    (13 tile pairs instead of 5).
// The recurrence has no separate issuer: the last of the four recurrence warps
// to have written M_t issues the MMAs of frame t + 1 itself, which takes a
// cross-warp hand-off off the serial path.
//
// Every wait is bounded (1 s; a GDN_DEBUG build reads the bound of role waits
// from GDN_DEBUG_WAIT_NS). A wait that runs out records its role in the device
// status word and raises an abort flag in its CTA and in global memory; every
// other CTA sees the global flag within a bounded time, its roles stop
// waiting, in-flight copies and MMAs are drained, and the kernel returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdlib.h>

#include <atomic>

#include "gdn.h"
#include "gdn_internal.h"
#include "sm100_ptx.h"

namespace gdn {
namespace {

using namespace ptx;

constexpr uint64_t kDrainNs = 1000ull * 1000ull * 1000ull;     // 1 s per drain wait
constexpr int kThreads = 512;
constexpr int kD = 64;
constexpr int kTile = 128;                                      // Q / output rows per tile
constexpr uint32_t kTileBytes = kTile * kD * 2;                 // 16 KB
constexpr int kKvRows = 64;                                     // rows per K/V tile
constexpr uint32_t kKvTileBytes = kKvRows * kD * 2;             // 8 KB
constexpr int kRing = 16;                                       // frames per head in the ring
constexpr int kStoreRows = 16;                                  // rows per output store box
constexpr int kMaxP = 8;                                        // head CTAs per head

enum : uint32_t {
  kStKvLoad = 1u << 0, kStQLoad = 1u << 1, kStMma = 1u << 2, kStChain = 1u << 3,
  kStProd = 1u << 4, kStOut = 1u << 5, kStDrain = 1u << 6, kStMoEmpty = 1u << 7,
  kStRing = 1u << 9, kStConfig = 1u << 10, kStRoom = 1u << 11
};

struct L {
  static constexpr int NKV = 5;                      // K/V tile pairs in flight (head CTAs)
  static constexpr int NKV_HELP = 13;                // the same in helpers
  static constexpr int NKV_MAX = NKV_HELP;
  static constexpr int NQ = 4;                       // Q tiles in flight (also output staging)
  static constexpr int NAC = 2;                      // transition-operand slots
  static constexpr int NM = 4;                       // state operand buffers: M_t in t % NM
  static constexpr int NCLAIM = 16;                  // claimed jobs in flight
  static constexpr uint32_t KV_SLOT = 2 * kKvTileBytes;             // K tile, then V tile
  static constexpr uint32_t AP_BYTES = kD * kD * 2;                 // A' (bf16, K-major, swizzled)
  static constexpr uint32_t C_BYTES = kD * kD * 4;                  // c^T, fp32: row j = column j of c
  static constexpr uint32_t AC_BYTES = AP_BYTES + C_BYTES;          // one ring image, one bulk copy
  static constexpr uint32_t AC_SLOT = AC_BYTES;                     // a multiple of 1 KB
  // State operand: M in bf16, two MN-major blocks of 32 value columns
  // (64-byte rows, 64-byte swizzle, 8-row groups of 512 bytes).
  static constexpr uint32_t MB_RW = 64;
  static constexpr uint32_t MB_SBO = 8 * MB_RW;
  static constexpr uint32_t MB_BLOCK = kD * MB_RW;                  // 4 KB
  static constexpr uint32_t M_BUF = 2 * MB_BLOCK;                   // 8 KB

  static constexpr uint32_t OFF_KV = 0;
  static constexpr uint32_t OFF_Q = OFF_KV + NKV * KV_SLOT;
  static constexpr uint32_t OFF_AC = OFF_Q + NQ * kTileBytes;
  static constexpr uint32_t OFF_MCH = OFF_AC + NAC * AC_SLOT;      // [NM] M_t in buffer t % NM
  static constexpr uint32_t OFF_BAR = OFF_MCH + NM * M_BUF;
  // barrier indices (8 bytes each)
  static constexpr int B_KV_FULL = 0;
  static constexpr int B_KV_EMPTY = B_KV_FULL + NKV_MAX;
  static constexpr int B_Q_FULL = B_KV_EMPTY + NKV_MAX;
  static constexpr int B_Q_EMPTY = B_Q_FULL + NQ;
  static constexpr int B_AC_FULL = B_Q_EMPTY + NQ;      // [NAC] operands of the frame loaded
  static constexpr int B_AC_EMPTY = B_AC_FULL + NAC;    // [NAC] frame consumed (recurrence warps)
  static constexpr int B_GB_FULL = B_AC_EMPTY + NAC;
  static constexpr int B_GB_FREE = B_GB_FULL + 2;
  static constexpr int B_CHAIN_DONE = B_GB_FREE + 2;
  static constexpr int B_MCH_FULL = B_CHAIN_DONE + 1;   // [NM] M_t written (4 warps)
  static constexpr int B_MCH_FREE = B_MCH_FULL + NM;    // [NM] read-out MMAs of M_t done
  static constexpr int B_O_FULL = B_MCH_FREE + NM;
  static constexpr int B_O_FREE = B_O_FULL + 2;
  static constexpr int B_DRAIN = B_O_FREE + 2;          // [6] per MMA-issuing thread
  static constexpr int B_E1_STAGED = B_DRAIN + 6;       // [4] job's A'/c written (4 warps)
  static constexpr int B_PUB_DONE = B_E1_STAGED + 4;    // [4] job published to the ring
  static constexpr int B_STAGE = B_PUB_DONE + 4;        // [2] output tile staged (4 warps)
  static constexpr int B_CLAIM = B_STAGE + 2;           // [NCLAIM] job j known
  static constexpr int NBAR = B_CLAIM + NCLAIM;
  static constexpr uint32_t OFF_TMEM_PTR = OFF_BAR + 8 * NBAR;
  static constexpr uint32_t OFF_ABORT = OFF_TMEM_PTR + 4;
  static constexpr uint32_t OFF_CHAIN_CTR = OFF_ABORT + 16;   // recurrence warps done with a frame
  static constexpr uint32_t OFF_JOB_H = OFF_CHAIN_CTR + 16;   // [NCLAIM] s32: head of job j, -1 = done
  static constexpr uint32_t OFF_JOB_F = OFF_JOB_H + 4 * NCLAIM;   // [NCLAIM] s32: its frame
  static constexpr uint32_t BYTES = OFF_JOB_F + 4 * NCLAIM;
  static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;              // base alignment slack

  // TMEM columns (each region 128 lanes)
  static constexpr uint32_t T_GB = 0;        // 2 x 64: [G; (K^T V)^T] accumulators
  static constexpr uint32_t T_O = 128;       // 2 x 64: output tile accumulators
  static constexpr uint32_t T_CHAIN = 256;   // 32 columns; value columns 0-31 in lanes
                                             // 32q+0..15, columns 32-63 in lanes 32q+16..31
  static constexpr uint32_t TMEM_COLS = 512;
};

static_assert(L::SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(L::NKV_HELP * L::KV_SLOT <= L::OFF_BAR, "helper K/V slots fit below the barriers");
static_assert(L::AC_BYTES % 1024 == 0, "ring images keep the swizzle alignment");

struct WideParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_o;
  const float* gamma;
  const float* beta;
  const float* state_in;
  float* state_out;
  unsigned int* status;
  unsigned long long timeout_ns;     // bound of every role wait
  uint8_t* ring;                     // [heads][kRing][AC_BYTES]
  unsigned long long* ring_flag;     // [heads][kRing]: frame + 1 once published
  unsigned long long* ring_loaded;   // [heads][P]: frames loaded by each head CTA
  unsigned int* claim;               // [heads, rounded up to 4]: frames claimed per head
  unsigned int* started;             // [heads]: head CTAs that have read the initial state
  unsigned int* gabort;              // set by a CTA that gave up
  int heads;
  int P;            // head CTAs per head; CTAs from heads * P on are helpers
  int T;
  int S;
  int nkv;          // K/V tiles per frame (kKvRows rows each)
  int chunk;        // output rows per head CTA (multiple of 16); rank r owns [r*chunk, (r+1)*chunk)
  float s;     // key scale 1/sqrt(D*S)
  float s2;    // its square
  float delta; // 1: delta rule; 0: GDN_FLAG_NO_DELTA, so A' = 0 and M' = gamma M + c
};

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile whose rows are
// `row_bytes` long and grouped by 8 rows, with the matching swizzle (the
// layout TMA writes with CU_TENSOR_MAP_SWIZZLE_{32,64,128}B and the tcgen05
// descriptors read): bits [4, 4+b) of the offset are XORed with bits [7, 7+b).
__device__ __forceinline__ uint32_t swz_off(uint32_t row, uint32_t chunk, uint32_t row_bytes,
                                            int bits) {
  const uint32_t off = (row >> 3) * (8 * row_bytes) + (row & 7) * row_bytes + chunk * 16;
  return off ^ (((off >> 7) & ((1u << bits) - 1)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

__device__ __forceinline__ int ld_shared_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

struct Ctl {
  uint32_t abort_addr;    // local shared address of the CTA's abort flag
  unsigned int* status;
  unsigned int* gabort;   // grid-wide abort flag
  uint64_t timeout_ns;
};

__device__ __forceinline__ bool aborted(const Ctl& c) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(c.abort_addr) : "memory");
  return v != 0;
}

// The CTA's flag, or else the grid-wide one (copied into the CTA's flag).
__device__ __noinline__ bool aborted_any(const Ctl& c) {
  if (aborted(c)) return true;
  if (ld_volatile_u32(c.gabort) != 0) {
    asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(c.abort_addr), "r"(1u) : "memory");
    return true;
  }
  return false;
}

__device__ __noinline__ void raise_abort(const Ctl& c, uint32_t code) {
  atomicOr(c.status, code);
  asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(c.abort_addr), "r"(1u) : "memory");
  atomicExch(c.gabort, 1u);
}

// Bounded wait on a local mbarrier phase. False if the kernel is aborting or
// the wait ran out (then the abort is raised with `code`). The grid-wide flag
// is read every 64 tries.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& c,
                                         uint32_t code) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 63u) == 0 ? aborted_any(c) : aborted(c)) return false;
    if (globaltimer_ns() - t0 > c.timeout_ns) {
      raise_abort(c, code);
      return false;
    }
  }
}

// Bounded poll with a short sleep between tests, for the recurrence's
// latency-critical handoffs.
__device__ __forceinline__ bool poll_bar(uint32_t bar, uint32_t parity, const Ctl& c,
                                         uint32_t code) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    for (int k = 0; k < 32; ++k) {
      __nanosleep(20);
      if (mbar_test(bar, parity)) return true;
    }
    if ((i & 15u) == 0 ? aborted_any(c) : aborted(c)) return false;
    if (globaltimer_ns() - t0 > c.timeout_ns) {
      raise_abort(c, code);
      return false;
    }
  }
}

// Warp-uniform bounded wait: lane 0 waits, the verdict is broadcast, and on
// success every lane observes the completed phase itself (acquire).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Ctl& c,
                                          uint32_t code) {
  uint32_t ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, c, code) ? 1u : 0u;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) {
    for (int i = 0; i < 1024 && !mbar_try(bar, parity); ++i) {
    }
  }
  return ok != 0;
}

// Bounded wait that ignores the abort flags (drains copies and MMAs in flight).
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity, const Ctl& c) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainNs) {
      atomicOr(c.status, kStDrain);
      return;
    }
  }
}

// Bounded poll of a global counter written by another CTA (acquire).
__device__ __forceinline__ bool wait_global_ge(const unsigned long long* ptr,
                                               unsigned long long v, const Ctl& c,
                                               uint32_t code) {
  if (ld_acquire_gpu_u64(ptr) >= v) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (ld_acquire_gpu_u64(ptr) >= v) return true;
    if ((i & 15u) == 0 ? aborted_any(c) : aborted(c)) return false;
    if (globaltimer_ns() - t0 > c.timeout_ns) {
      raise_abort(c, code);
      return false;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) gdn_wide_kernel(const __grid_constant__ WideParams p) {
  constexpr int NAC = L::NAC;
  extern __shared__ uint8_t smem_raw[];
  {
    // A launch with the wrong block size or too little shared memory records
    // an error and touches nothing (every thread of every CTA returns here).
    uint32_t dsmem;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dsmem));
    if (blockDim.x != kThreads || blockDim.y != 1 || blockDim.z != 1 || dsmem < L::SMEM_ALLOC) {
      if (threadIdx.x == 0) atomicOr(p.status, kStConfig);
      return;
    }
  }
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;         // 1 KB aligned base
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int P = p.P;
  const bool helper = (int)blockIdx.x >= p.heads * P;
  const int bh = helper ? -1 : (int)blockIdx.x / P;    // own head (head CTAs)
  const int rank = helper ? 0 : (int)blockIdx.x % P;
  const int T = p.T;
  const int nkv = p.nkv;
  const int nslots = helper ? L::NKV_HELP : L::NKV;    // K/V tile pairs in flight

  auto bar = [&](int i) -> uint32_t { return sb + L::OFF_BAR + 8u * i; };
  auto kv_slot = [&](int i) -> uint32_t { return sb + L::OFF_KV + i * L::KV_SLOT; };
  auto q_slot = [&](int i) -> uint32_t { return sb + L::OFF_Q + i * kTileBytes; };
  auto ac_slot = [&](int i) -> uint32_t { return sb + L::OFF_AC + i * L::AC_SLOT; };
  auto mch = [&](int i) -> uint32_t { return sb + L::OFF_MCH + i * L::M_BUF; };
  auto job_h = [&](int j) -> uint32_t { return sb + L::OFF_JOB_H + 4u * (j % L::NCLAIM); };
  auto job_f = [&](int j) -> uint32_t { return sb + L::OFF_JOB_F + 4u * (j % L::NCLAIM); };
  // Output rows of a head CTA, in every frame, and its Q tiles.
  const int r0 = rank * p.chunk;
  const int r1 = helper ? r0 : min(p.S, r0 + p.chunk);
  const int nq = r1 > r0 ? (r1 - r0 + kTile - 1) / kTile : 0;
  const uint32_t tmem_ptr = sb + L::OFF_TMEM_PTR;
  Ctl ctl{sb + L::OFF_ABORT, p.status, p.gabort, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NKV_MAX; ++i) {
      mbar_init(bar(L::B_KV_FULL + i), 1);
      mbar_init(bar(L::B_KV_EMPTY + i), 1);
    }
    for (int i = 0; i < L::NQ; ++i) {
      mbar_init(bar(L::B_Q_FULL + i), 1);
      mbar_init(bar(L::B_Q_EMPTY + i), 1);
    }
    for (int i = 0; i < NAC; ++i) {
      mbar_init(bar(L::B_AC_FULL + i), 1);
      mbar_init(bar(L::B_AC_EMPTY + i), 4);         // the 4 recurrence warps
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::B_GB_FULL + i), 1);
      mbar_init(bar(L::B_GB_FREE + i), 4);
      mbar_init(bar(L::B_O_FULL + i), 1);
      mbar_init(bar(L::B_O_FREE + i), 4);
    }
    for (int i = 0; i < L::NM; ++i) {
      mbar_init(bar(L::B_MCH_FULL + i), 4);
      mbar_init(bar(L::B_MCH_FREE + i), 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar(L::B_E1_STAGED + i), 4);
      mbar_init(bar(L::B_PUB_DONE + i), 1);
    }
    mbar_init(bar(L::B_STAGE + 0), 4);
    mbar_init(bar(L::B_STAGE + 1), 4);
    mbar_init(bar(L::B_CHAIN_DONE), 1);
    for (int i = 0; i < 6; ++i) mbar_init(bar(L::B_DRAIN + i), 1);
    for (int i = 0; i < L::NCLAIM; ++i) mbar_init(bar(L::B_CLAIM + i), 1);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(ctl.abort_addr), "r"(0u) : "memory");
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(sb + L::OFF_CHAIN_CTR), "r"(0u) : "memory");
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    if (!helper) {
      prefetch_tmap(&p.tm_q);
      prefetch_tmap(&p.tm_o);
    }
  }
  if (warp == 2) {
    tmem_alloc(tmem_ptr, L::TMEM_COLS);
    tmem_relinquish();
  }
  // The recurrence warps read the initial state here. Rank 0 of the head
  // writes the final state only once every CTA of the head has counted itself
  // in `started` (after the barrier below), so state_in == state_out is safe.
  // Lane l of warp quarter q owns row 16q + (l % 16), value columns
  // 32 (l / 16) .. + 32.
  float m[32];
  if (!helper && warp >= 4 && warp < 8) {
    const int row = (warp & 3) * 16 + (lane & 15);
    const int col0 = 32 * (lane >> 4);
#pragma unroll
    for (int jj = 0; jj < 32; ++jj)
      m[jj] = p.state_in ? p.state_in[((size_t)bh * kD + row) * kD + col0 + jj] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (!helper && threadIdx.x == 0) red_release_gpu_add_u32(p.started + bh, 1u);
  uint32_t tmem;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(tmem_ptr) : "memory");

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ K/V loader and claims
    // A job is one frame of one head. Head CTAs claim frames of their own head
    // while it has any left; then, like the helpers from the start, they take
    // the head with the fewest frames claimed. Before a job's tiles are loaded
    // its ring slot must be free: every CTA of the head has loaded the frame
    // kRing before it. Each claim is made one job ahead and that job's tiles
    // are prefetched into L2. Inputs are read once: evict them first.
    const uint64_t stream_pol = policy_evict_first();
    bool own_done = helper;
    auto claim = [&]() -> int2 {
      if (!own_done) {
        const int f = (int)atomicAdd(p.claim + bh, 1u);
        if (f < T) return make_int2(bh, f);
        own_done = true;
      }
      // Each failed try leaves one more head with all frames claimed.
      for (int tries = 0; tries <= p.heads; ++tries) {
        int best = -1;
        unsigned int bv = 0xffffffffu;
        for (int h0 = 0; h0 < p.heads; h0 += 4) {
          const uint4 c4 = ld_volatile_v4_u32(p.claim + h0);
          const unsigned int cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (h0 + e < p.heads && cv[e] < (unsigned int)T && cv[e] < bv) {
              bv = cv[e];
              best = h0 + e;
            }
        }
        if (best < 0) break;                       // every frame of every head is claimed
        const int f = (int)atomicAdd(p.claim + best, 1u);
        if (f < T) return make_int2(best, f);
      }
      return make_int2(-1, -1);
    };
    auto prefetch_job = [&](int2 jb) {
      const int z = jb.x * T + jb.y;
      for (int i = 0; i < nkv; ++i) {
        tma_prefetch_3d(&p.tm_k, 0, i * kKvRows, z);
        tma_prefetch_3d(&p.tm_v, 0, i * kKvRows, z);
      }
    };
    int room_h = -1;                       // head whose CTAs' progress was last read,
    unsigned long long room_lo = 0;        // and the lowest of those readings
    int2 next = claim();
    if (next.x >= 0) prefetch_job(next);
    int it = 0;
    bool ok = true;
    for (int j = 0;; ++j) {
      int2 jb = next;
      if (jb.x >= 0 && jb.y >= kRing) {
        const unsigned long long need = (unsigned long long)(jb.y - kRing + 1);
        if (jb.x != room_h || room_lo < need) {
          unsigned long long lo = ~0ull;
          for (int q = 0; q < P && ok; ++q) {
            const unsigned long long* pl = p.ring_loaded + (size_t)jb.x * P + q;
            ok = wait_global_ge(pl, need, ctl, kStRoom);
            const unsigned long long v = ld_acquire_gpu_u64(pl);
            lo = v < lo ? v : lo;
          }
          room_h = jb.x;
          room_lo = lo;
        }
        if (!ok) jb = make_int2(-1, -1);   // abort: tell the other roles to stop
      }
      asm volatile("st.shared.s32 [%0], %1;" ::"r"(job_h(j)), "r"(jb.x) : "memory");
      asm volatile("st.shared.s32 [%0], %1;" ::"r"(job_f(j)), "r"(jb.y) : "memory");
      mbar_arrive(bar(L::B_CLAIM + j % L::NCLAIM));
      if (jb.x < 0) break;
      next = claim();
      if (next.x >= 0) prefetch_job(next);
      const int z = jb.x * T + jb.y;
      for (int i = 0; i < nkv; ++i, ++it) {
        const int slot = it % nslots;
        if (!wait_bar(bar(L::B_KV_EMPTY + slot), ((it / nslots) & 1) ^ 1, ctl, kStKvLoad)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(L::B_KV_FULL + slot), 2 * kKvTileBytes);
        tma_load_3d_hint(kv_slot(slot), &p.tm_k, bar(L::B_KV_FULL + slot), 0, i * kKvRows, z,
                         stream_pol);
        tma_load_3d_hint(kv_slot(slot) + kKvTileBytes, &p.tm_v, bar(L::B_KV_FULL + slot), 0,
                         i * kKvRows, z, stream_pol);
      }
      if (!ok) {
        // The other roles stop on the abort flag (their next wait fails).
        break;
      }
    }
    for (int k = it - 1; k >= 0 && k >= it - nslots; --k)
      drain_bar(bar(L::B_KV_FULL + k % nslots), (k / nslots) & 1, ctl);
  } else if (warp == 0 && lane == 16) {
    // ------------------------------------------------ publisher of this CTA's jobs
    for (int j = 0;; ++j) {
      if (!wait_bar(bar(L::B_CLAIM + j % L::NCLAIM), (j / L::NCLAIM) & 1, ctl, kStProd)) break;
      const int h = ld_shared_s32(job_h(j));
      const int f = ld_shared_s32(job_f(j));
      if (h < 0) break;
      if (!wait_bar(bar(L::B_E1_STAGED + (j & 3)), (j >> 2) & 1, ctl, kStProd)) break;
      __threadfence();
      fence_proxy_async_global();
      st_release_gpu_u64(p.ring_flag + (size_t)h * kRing + f % kRing, (unsigned long long)(f + 1));
      mbar_arrive(bar(L::B_PUB_DONE + (j & 3)));
    }
  } else if (warp == 1 && lane == 16) {
    // ------------------------------------------------ [K V]^T K MMA issuer (this CTA's jobs)
    constexpr uint32_t id_gb = idesc_bf16(128, 64, 1, 1);      // [K V]^T and K, both MN-major
    int kvit = 0;
    bool ok = true;
    for (int j = 0; ok; ++j) {
      if (!wait_bar(bar(L::B_CLAIM + j % L::NCLAIM), (j / L::NCLAIM) & 1, ctl, kStMma)) break;
      if (ld_shared_s32(job_h(j)) < 0) break;
      const int b = j & 1;
      if (!wait_bar(bar(L::B_GB_FREE + b), ((j >> 1) & 1) ^ 1, ctl, kStMma)) break;
      for (int i = 0; i < nkv; ++i, ++kvit) {
        const int slot = kvit % nslots;
        if (!wait_bar(bar(L::B_KV_FULL + slot), (kvit / nslots) & 1, ctl, kStMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kv = kv_slot(slot);
        const uint32_t dg = tmem + L::T_GB + 64 * b;
#pragma unroll
        for (int kk = 0; kk < kKvRows / 16; ++kk) {
          const uint64_t a = smem_desc(kv + kk * 2048, kKvTileBytes, 1024, 2);
          const uint64_t bd = smem_desc(kv + kk * 2048, kKvTileBytes, 1024, 2);
          mma_bf16(dg, a, bd, id_gb, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(L::B_KV_EMPTY + slot));
      }
      if (!ok) break;
      mma_commit(bar(L::B_GB_FULL + b));
    }
    mma_commit(bar(L::B_DRAIN + 0));
    drain_bar(bar(L::B_DRAIN + 0), 0, ctl);
  } else if (warp >= 8 && warp < 12) {
    // ------------------------------------------------ A' and c from [G; (K^T V)^T]
    const int qd = warp & 3;
    const int lrow = qd * 32 + lane;           // accumulator row = TMEM lane
    for (int j = 0;; ++j) {
      if (!warp_wait(bar(L::B_CLAIM + j % L::NCLAIM), (j / L::NCLAIM) & 1, ctl, kStProd)) break;
      const int h = ld_shared_s32(job_h(j));
      const int f = ld_shared_s32(job_f(j));
      if (h < 0) break;
      const int b = j & 1;
      const float g = __ldg(p.gamma + (size_t)h * T + f);
      const float be = __ldg(p.beta + (size_t)h * T + f);
      if (!warp_wait(bar(L::B_GB_FULL + b), (j >> 1) & 1, ctl, kStProd)) break;
      tc_fence_after();
      uint32_t v[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r16[16];
        tmem_ld16(tmem + L::T_GB + 64 * b + 16 * c + ((uint32_t)(qd * 32) << 16), r16);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[16 * c + e] = r16[e];
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::B_GB_FREE + b));
      // A' rows packed in place: chunk c (8 values) becomes 4 bf16x2 words in v[8c..8c+3].
      if (lrow < kD) {
        const float coef = -g * be * p.s2 * p.delta;   // A' = -gamma beta s^2 G (0 without delta)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = coef * __uint_as_float(v[8 * c + e]);
          v[8 * c + 0] = pack_bf16x2(x[0], x[1]);
          v[8 * c + 1] = pack_bf16x2(x[2], x[3]);
          v[8 * c + 2] = pack_bf16x2(x[4], x[5]);
          v[8 * c + 3] = pack_bf16x2(x[6], x[7]);
        }
      } else {
        const float coef = be * p.s;             // c = beta s K^T V
#pragma unroll
        for (int i = 0; i < kD; ++i) v[i] = __float_as_uint(coef * __uint_as_float(v[i]));
      }
      // The loader claimed this job only once its ring slot was free.
      uint8_t* img = p.ring + ((size_t)h * kRing + f % kRing) * L::AC_BYTES;
      const uint64_t ring_pol = policy_evict_last();
      if (lrow < kD) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t off = swz_off(lrow, c, 128, 3);
          st_global_v4_hint(img + off, make_uint4(v[8 * c], v[8 * c + 1], v[8 * c + 2], v[8 * c + 3]),
                            ring_pol);
        }
      } else {
        uint8_t* dst = img + L::AP_BYTES + (lrow - kD) * kD * 4;
#pragma unroll
        for (int i = 0; i < kD; i += 4)
          st_global_v4_hint(dst + i * 4, make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]), ring_pol);
      }
      __syncwarp();
      // The publisher must have published job j - 4 before its staging barrier is reused.
      if (j >= 4 && !warp_wait(bar(L::B_PUB_DONE + (j & 3)), ((j >> 2) - 1) & 1, ctl, kStProd))
        break;
      if (lane == 0) mbar_arrive(bar(L::B_E1_STAGED + (j & 3)));
    }
  } else if (helper) {
    // Helpers have no other role.
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ Q loader (this CTA's rows, every frame)
    const uint64_t stream_pol = policy_evict_first();
    for (int i = 0; i < nq; ++i) tma_prefetch_3d(&p.tm_q, 0, r0 + i * kTile, bh * T);
    int it = 0;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      if (t + 1 < T)
        for (int i = 0; i < nq; ++i) tma_prefetch_3d(&p.tm_q, 0, r0 + i * kTile, bh * T + t + 1);
      for (int i = 0; i < nq; ++i, ++it) {
        const int slot = it % L::NQ;
        if (!wait_bar(bar(L::B_Q_EMPTY + slot), ((it / L::NQ) & 1) ^ 1, ctl, kStQLoad)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(L::B_Q_FULL + slot), kTileBytes);
        tma_load_3d_hint(q_slot(slot), &p.tm_q, bar(L::B_Q_FULL + slot), 0, r0 + i * kTile, bh * T + t,
                         stream_pol);
      }
    }
    for (int k = it - 1; k >= 0 && k >= it - L::NQ; --k)
      drain_bar(bar(L::B_Q_FULL + k % L::NQ), (k / L::NQ) & 1, ctl);
  } else if (warp == 3 && lane == 16) {
    // ------------------------------------------------ read-out MMA issuer (this CTA's rows)
    constexpr uint32_t id_o = idesc_bf16(128, 64, 0, 1);       // Q K-major, M MN-major
    int qit = 0, on = 0;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int u = t % L::NM;
      if (!wait_bar(bar(L::B_MCH_FULL + u), (t / L::NM) & 1, ctl, kStMma)) break;
      for (int i = 0; i < nq; ++i, ++qit, ++on) {
        const int slot = qit % L::NQ;
        const int ob = on & 1;
        if (!wait_bar(bar(L::B_Q_FULL + slot), (qit / L::NQ) & 1, ctl, kStMma) ||
            !wait_bar(bar(L::B_O_FREE + ob), ((on >> 1) & 1) ^ 1, ctl, kStMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t qt = q_slot(slot);
        const uint32_t mo = mch(u);
        const uint32_t dO = tmem + L::T_O + 64 * ob;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = smem_desc(qt + kk * 32, 16, 1024, 2);
          const uint64_t bH = smem_desc(mo + kk * 2 * L::MB_SBO, L::MB_BLOCK, L::MB_SBO, 4);
          mma_bf16(dO, a, bH, id_o, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::B_O_FULL + ob));
      }
      if (ok) mma_commit(bar(L::B_MCH_FREE + u));   // M_t no longer read here
    }
    mma_commit(bar(L::B_DRAIN + 1));
    drain_bar(bar(L::B_DRAIN + 1), 0, ctl);
  } else if (warp == 3 && lane == 0) {
    // ------------------------------------------------ loader of the transition operands
    // Every frame of the head arrives through the ring, in frame order; the
    // bulk load completes the slot's "full" barrier itself.
    const uint64_t ring_pol = policy_evict_last();
    int t = 0;
    for (; t < T; ++t) {
      const int s = t % NAC;
      const size_t rs = (size_t)bh * kRing + t % kRing;
      if (!wait_global_ge(p.ring_flag + rs, (unsigned long long)(t + 1), ctl, kStRing)) break;
      if (!wait_bar(bar(L::B_AC_EMPTY + s), ((t / NAC) & 1) ^ 1, ctl, kStRing)) break;
      // Frame t - NAC has been consumed here, so its load (and every earlier one)
      // completed: ring slots up to it may be reused by their producers.
      if (t >= NAC)
        st_relaxed_gpu_u64(p.ring_loaded + (size_t)bh * P + rank, (unsigned long long)(t - NAC + 1));
      fence_proxy_async_global();
      mbar_arrive_expect_tx(bar(L::B_AC_FULL + s), L::AC_BYTES);
      bulk_load_global_hint(ac_slot(s), p.ring + rs * L::AC_BYTES, L::AC_BYTES, bar(L::B_AC_FULL + s),
                            ring_pol);
    }
    // The last frames' slots are no longer needed by anyone once loaded.
    for (int k = t - 1; k >= 0 && k >= t - NAC; --k)
      drain_bar(bar(L::B_AC_FULL + k % NAC), (k / NAC) & 1, ctl);
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------ recurrence (epilogue and issue)
    // The accumulator holds A' M for the 64 state rows: value columns 0-31 of
    // row 16q+i in TMEM lane 32q+i, columns 32-63 in lane 32q+16+i. So lane l
    // of warp quarter q owns row 16q+(l%16), columns 32*(l/16)..+32.
    const int qd = warp & 3;
    const int hf = lane >> 4;
    const int row = qd * 16 + (lane & 15);
    auto store_state = [&](uint32_t buf) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        st_shared_v4(buf + hf * L::MB_BLOCK + swz_off(row, c, L::MB_RW, 2), pack8(&m[8 * c]));
    };
    // MMAs A'_t M_{t-1}, issued by lane 0 of the last warp done with frame t - 1.
    bool issued = false;
    auto issue_chain = [&](int t) {
      constexpr uint32_t id_chain = idesc_bf16(64, 32, 0, 1);    // A' K-major, M half MN-major
      tc_fence_after();
      const uint32_t ac = ac_slot(t % NAC);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const uint32_t dt = tmem + L::T_CHAIN + ((uint32_t)h2 << 20);   // lane offset 16
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t aH = smem_desc(ac + kk * 32, 16, 1024, 2);
          const uint32_t mb = mch((t + L::NM - 1) % L::NM) + h2 * L::MB_BLOCK + kk * 2 * L::MB_SBO;
          const uint64_t bH = smem_desc(mb, L::MB_BLOCK, L::MB_SBO, 4);
          mma_bf16(dt, aH, bH, id_chain, kk > 0 ? 1u : 0u);
        }
      }
      mma_commit(bar(L::B_CHAIN_DONE));
      issued = true;
    };
    // Counts this warp done with the previous frame (its M rows written and
    // fenced, its accumulator reads complete); the fourth issues frame t.
    auto done_and_issue = [&](int t) -> bool {
      uint32_t ok = 1;
      if (lane == 0) {
        const uint32_t old = atom_add_acq_rel_shared(sb + L::OFF_CHAIN_CTR, 1u);
        if ((old & 3u) == 3u && t < T) {
          ok = wait_bar(bar(L::B_AC_FULL + t % NAC), (t / NAC) & 1, ctl, kStMma) ? 1u : 0u;
          if (ok) issue_chain(t);
        }
      }
      return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    store_state(mch(L::NM - 1));               // M_{-1} = M_0, read by the first MMA
    fence_proxy_async_cta();
    __syncwarp();
    bool ok = done_and_issue(0);
    const float* gam = p.gamma + (size_t)bh * T;
    float g_next = __ldg(gam);
    int t = 0;
    for (; t < T && ok; ++t) {
      const float g = g_next;
      if (t + 1 < T) g_next = __ldg(gam + t + 1);
      const int s = t % NAC;
      const bool acok = warp_wait(bar(L::B_AC_FULL + s), (t / NAC) & 1, ctl, kStChain);
      uint32_t cd = 0;
      if (acok && lane == 0) cd = poll_bar(bar(L::B_CHAIN_DONE), t & 1, ctl, kStChain) ? 1u : 0u;
      cd = __shfl_sync(0xffffffffu, cd, 0);
      if (cd) mbar_test(bar(L::B_CHAIN_DONE), t & 1);    // acquire for every lane
      // M_t goes to buffer t % NM, which held M_{t-NM}: its read-out MMAs must be done.
      if (!acok || !cd ||
          !warp_wait(bar(L::B_MCH_FREE + t % L::NM), ((t / L::NM) & 1) ^ 1, ctl, kStMoEmpty)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t d[32];
      {
        uint32_t a0[16], a1[16];
        tmem_ld16(tmem + L::T_CHAIN + ((uint32_t)(qd * 32) << 16), a0);
        tmem_ld16(tmem + L::T_CHAIN + 16 + ((uint32_t)(qd * 32) << 16), a1);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          d[e] = a0[e];
          d[16 + e] = a1[e];
        }
      }
      // c[row][32hf + jj] = c^T[32hf + jj][row]
      const uint32_t ccol = ac_slot(s) + L::AP_BYTES + ((32 * hf) * kD + row) * 4;
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        float cv;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(cv) : "r"(ccol + jj * kD * 4) : "memory");
        m[jj] = fmaf(g, m[jj], __uint_as_float(d[jj])) + cv;
      }
      store_state(mch(t % L::NM));
      tc_fence_before();
      fence_proxy_async_cta();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(L::B_AC_EMPTY + s));           // A'_t read by its MMA, c_t read here
        mbar_arrive(bar(L::B_MCH_FULL + t % L::NM));   // M_t ready for the read-out
      }
      ok = done_and_issue(t + 1);
    }
    if (lane == 0 && issued) {
      // MMAs this thread issued may still run if the loop stopped early.
      mma_commit(bar(L::B_DRAIN + 2 + qd));
      drain_bar(bar(L::B_DRAIN + 2 + qd), 0, ctl);
    }
    if (ok && t == T && p.state_out && rank == 0) {   // every CTA of the head holds the same state
      // Every CTA of the head has read the initial state (state_in may be state_out).
      uint32_t all = 1;
      if (lane == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu_u32(p.started + bh) < (unsigned int)P) {
          if (globaltimer_ns() - t0 > ctl.timeout_ns) {
            raise_abort(ctl, kStChain);
            all = 0;
            break;
          }
        }
      }
      if (__shfl_sync(0xffffffffu, all, 0)) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
          p.state_out[((size_t)bh * kD + row) * kD + 32 * hf + jj] = m[jj];
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------ output tiles: TMEM -> bf16 -> TMA store
    // Each tile is staged in the Q slot it was computed from (its MMA is done)
    // and written with bulk tensor stores of 16 rows, this CTA's rows only; the
    // slot goes back to the Q loader once the stores have read it.
    const int qd = warp & 3;
    const int lrow = qd * 32 + lane;           // tile row = TMEM lane
    const bool leader = (warp == 12 && lane == 0);
    const uint64_t out_pol = policy_evict_first();
    int n = 0;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      for (int i = 0; i < nq; ++i, ++n) {
        const int ob = n & 1;
        if (!warp_wait(bar(L::B_O_FULL + ob), (n >> 1) & 1, ctl, kStOut)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r16[16];
          tmem_ld16(tmem + L::T_O + 64 * ob + 16 * c + ((uint32_t)(qd * 32) << 16), r16);
#pragma unroll
          for (int e = 0; e < 16; ++e) v[16 * c + e] = r16[e];
        }
        tmem_wait_ld();
        tc_fence_before();
        const int slot = n % L::NQ;            // the Q tile this output came from
        const uint32_t tile = q_slot(slot);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * c + 0]), __uint_as_float(v[8 * c + 1]));
          w.y = pack_bf16x2(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3]));
          w.z = pack_bf16x2(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5]));
          w.w = pack_bf16x2(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]));
          st_shared_v4(tile + swz_off(lrow, c, 128, 3), w);
        }
        fence_proxy_async_cta();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(L::B_STAGE + (n & 1)));
          // Only now free the accumulator: tile n + 2 (same staging barrier) cannot
          // start before all four warps have staged tile n.
          mbar_arrive(bar(L::B_O_FREE + ob));
        }
        uint32_t stored = 1;
        if (leader) {
          stored = wait_bar(bar(L::B_STAGE + (n & 1)), (n >> 1) & 1, ctl, kStOut) ? 1u : 0u;
          if (stored) {
            const int y0 = r0 + i * kTile;
            const int y1 = min(r1, y0 + kTile);
            for (int y = y0; y < y1; y += kStoreRows)
              tma_store_3d_hint(&p.tm_o, tile + (uint32_t)(y - y0) * 128u, 0, y, bh * T + t, out_pol);
            bulk_commit();
            bulk_wait_read0();
            mbar_arrive(bar(L::B_Q_EMPTY + slot));
          }
        }
        if (!__shfl_sync(0xffffffffu, stored, 0)) {
          ok = false;
          break;
        }
      }
    }
    if (leader) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

// Raises the kernel's dynamic shared-memory limit, once per device.
cudaError_t prepare() {
  static std::atomic<bool> done[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(gdn_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)L::SMEM_ALLOC);
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

// CTAs of the kernel that can be resident at once on the current device (the
// grid of every launch), or -1 without a usable device. Cached per device.
int resident_ctas() {
  static std::atomic<int> cache[64];            // 0: not yet known; else the count + 2
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return -1;
  }
  const int known = cache[dev].load(std::memory_order_acquire);
  if (known != 0) return known - 2;
  int n = -1;
  int per_sm = 0, sms = 0, coop = 0;
  if (prepare() == cudaSuccess &&
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess && coop &&
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gdn_wide_kernel, kThreads,
                                                    L::SMEM_ALLOC) == cudaSuccess)
    n = per_sm * sms;
  cudaGetLastError();
  cache[dev].store(n + 2, std::memory_order_release);
  return n;
}

}  // namespace

int wide_ctas_per_head(int B, int H, int T, int S, int D) {
  if (D != kD || T < 2) return 0;
  const long long heads = (long long)B * H;
  if (heads * (long long)T >= (1ll << 31) || (long long)S * kD * 2 >= (1ll << 40)) return 0;
  {
    const char* e = getenv("GDN_WIDE");
    if (!e || atoi(e) == 0) return 0;
  }
  int grid = resident_ctas();
  if (grid < 0) grid = 148;              // planning without a device: a B200
  if (heads > grid) return 0;
  int P = (int)(grid / heads);
  if (P > 4) P = 4;
  // Tuning override: GDN_WIDE_P=1..8 (if the head CTAs fit).
  if (const char* e = getenv("GDN_WIDE_P")) {
    const int v = atoi(e);
    if (v >= 1 && v <= kMaxP && heads * v <= grid) P = v;
  }
  return P;
}

cudaError_t launch_wide_bf16(const Problem& pr, int P) {
  if (P < 1 || P > kMaxP) return cudaErrorInvalidValue;
  cudaError_t e = prepare();
  if (e != cudaSuccess) return e;
  const int grid = resident_ctas();
  const long long heads = (long long)pr.B * pr.H;
  if (grid <= 0 || heads * P > grid) return cudaErrorInvalidConfiguration;
  WideParams p;
  const long long frames = heads * pr.T;
  if (!make_frame_map(&p.tm_q, pr.q, kD, pr.S, frames, kTile) ||
      !make_frame_map(&p.tm_k, pr.k, kD, pr.S, frames, kKvRows) ||
      !make_frame_map(&p.tm_v, pr.v, kD, pr.S, frames, kKvRows) ||
      !make_frame_map(&p.tm_o, pr.out, kD, pr.S, frames, kStoreRows))
    return cudaErrorInvalidValue;
  unsigned int* status = status_word();
  if (!status) return cudaErrorInvalidDevice;
  p.gamma = pr.gamma;
  p.beta = pr.beta;
  p.state_in = pr.state_in;
  p.state_out = pr.state_out;
  p.status = status;
  p.timeout_ns = wait_budget_ns();
  p.heads = (int)heads;
  p.P = P;
  p.T = pr.T;
  p.S = pr.S;
  p.nkv = (pr.S + kKvRows - 1) / kKvRows;
  p.chunk = ((pr.S + P - 1) / P + 15) / 16 * 16;
  p.s = pr.key_scale;
  p.s2 = (float)(1.0 / ((double)kD * (double)pr.S));
  p.delta = pr.delta ? 1.f : 0.f;

  // Stream-ordered scratch, released right after the launch on the same
  // stream: the ring, then the control words (zeroed).
  const size_t ring_bytes = (size_t)heads * kRing * L::AC_BYTES;
  const size_t heads4 = ((size_t)heads + 3) / 4 * 4;
  const size_t flag_bytes = (size_t)heads * kRing * 8;
  const size_t loaded_bytes = ((size_t)heads * P * 8 + 15) / 16 * 16;   // keeps `claim` 16-byte aligned
  const size_t claim_bytes = heads4 * 4;
  const size_t started_bytes = heads4 * 4;
  const size_t ctrl_bytes = flag_bytes + loaded_bytes + claim_bytes + started_bytes + 16;
  void* scratch = nullptr;
  e = cudaMallocAsync(&scratch, ring_bytes + ctrl_bytes, pr.stream);
  if (e != cudaSuccess) return e;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  p.ring = base;
  uint8_t* ctrl = base + ring_bytes;
  p.ring_flag = reinterpret_cast<unsigned long long*>(ctrl);
  p.ring_loaded = reinterpret_cast<unsigned long long*>(ctrl + flag_bytes);
  p.claim = reinterpret_cast<unsigned int*>(ctrl + flag_bytes + loaded_bytes);
  p.started = reinterpret_cast<unsigned int*>(ctrl + flag_bytes + loaded_bytes + claim_bytes);
  p.gabort = reinterpret_cast<unsigned int*>(ctrl + flag_bytes + loaded_bytes + claim_bytes + started_bytes);
  e = cudaMemsetAsync(ctrl, 0, ctrl_bytes, pr.stream);
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;    // every CTA resident: they wait on each other
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = L::SMEM_ALLOC;
    cfg.stream = pr.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gdn_wide_kernel, p);
  }
  const cudaError_t ef = cudaFreeAsync(scratch, pr.stream);
  return e != cudaSuccess ? e : ef;
}

}  // namespace gdn
