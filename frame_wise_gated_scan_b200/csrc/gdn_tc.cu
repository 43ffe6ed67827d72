// tcgen05 kernel of the frame-wise Gated DeltaNet scan, bf16 inputs, D = 64.
//
// The update ("NVIDIA Apresenta SANA-WM ...", acheiumaia.com.br, section
// "A Arquitetura", item "1. Atencao Linear Hibrida com Gated DeltaNet"), per
// head and frame t with s = 1/sqrt(D*S):
//     W = (sK) M,  R = V - gamma W,  M' = gamma M + beta (sK)^T R,  O = Q M'.
// Since (sK)^T R = s K^T V - gamma s^2 (K^T K) M, the same update reads
//     M' = gamma M + A' M + c,   A' = -gamma beta s^2 G,  G = K^T K,  c = beta s K^T V.
// G and K^T V depend on the frame's keys and values only, not on the state,
// so the two S-long contractions that build them run ahead of the
// recurrence; the only work on the frame-to-frame critical path is the
// D x D x D product A' M. The read-out O = Q M' follows behind it.
//
// Work split. One thread-block cluster of P CTAs per head (P = 1, 2 or 4):
//  * production: the CTAs of a head claim frames from a counter in rank 0's
//    shared memory (so a faster SM produces more of them). For a claimed
//    frame a CTA streams K and V (TMA, 64-row tiles, 128-byte swizzle), forms
//    [G; (K^T V)^T] = [K V]^T K on the tensor cores, and turns it into A'
//    (bf16) and c^T (fp32);
//  * with P > 1 those operands go to a ring in global memory that stays in L2
//    (16 frames per head), published with a release flag; every CTA of the
//    head, the producer included, bulk-loads every frame from it in frame
//    order. With P = 1 they are written straight into shared memory;
//  * every CTA runs the whole recurrence: the fp32 state M stays in the
//    registers of four warps across all T frames (gamma M is added in exact
//    fp32), and its bf16 copy in shared memory is the operand of the next
//    frame's MMA A' M;
//  * CTA r reads out its own block of rows [r*chunk, (r+1)*chunk) of every
//    frame, O_t = Q_t M_t, from its own copy of M_t (four bf16 buffers, so the
//    read-out may trail the recurrence by up to four frames), and stores it
//    with TMA.
// Warp roles (512 threads): warp 0 K/V loader and frame claims (lane 0) and
// ring publisher (lane 16); warp 1 Q loader (lane 0) and [K V]^T K MMA issuer
// (lane 16); warp 2 recurrence MMA issuer (lane 0, and TMEM allocation); warp 3
// ring loader (lane 0) and read-out MMA issuer (lane 16); warps 4-7 recurrence
// epilogue; 8-11 A'/c epilogue; 12-15 output epilogue.
//
// Every wait is bounded (1 s; a GDN_DEBUG build reads the bound of role waits
// from GDN_DEBUG_WAIT_NS, drains keep 1 s). A wait that runs out sets the device
// status word and an abort flag in every CTA of the cluster; the other roles
// then stop, in-flight copies and MMAs are drained, and the kernel returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdlib.h>

#include <atomic>
#include <mutex>

#include "gdn.h"
#include "gdn_internal.h"
#include "sm100_ptx.h"

namespace gdn {

#ifdef GDN_TRACE
// Event timeline of head 0's cluster (globaltimer ns), for pipeline analysis
// builds only: [rank][event][frame or own-frame index].
constexpr int kTraceRanks = 4, kTraceEvents = 24, kTraceFrames = 1024;
__device__ unsigned long long g_trace[kTraceRanks * kTraceEvents * kTraceFrames];
// Recurrence issue time of every frame of the first kTraceHeads heads (rank 0).
constexpr int kTraceHeads = 64;
__device__ unsigned long long g_trace_heads[kTraceHeads * kTraceFrames];
// Per CTA (first kTraceCtas): SM id, and the K/V loader's clock when it starts
// its third own frame and its last one.
constexpr int kTraceCtas = 1024;
__device__ unsigned long long g_trace_cta[kTraceCtas * 4];
#define GDN_TRACE_CTA(slot, value)                                     \
  do {                                                                 \
    if (blockIdx.x < kTraceCtas) g_trace_cta[blockIdx.x * 4 + (slot)] = (value); \
  } while (0)
#define GDN_TRACE_EV(ev, idx)                                                              \
  do {                                                                                     \
    if (bh == 0 && (idx) < kTraceFrames)                                                   \
      g_trace[((int)rank * kTraceEvents + (ev)) * kTraceFrames + (idx)] = globaltimer_ns(); \
  } while (0)
#else
#define GDN_TRACE_CTA(slot, value) \
  do {                             \
  } while (0)
#define GDN_TRACE_EV(ev, idx) \
  do {                        \
  } while (0)
#endif

namespace {

using namespace ptx;

constexpr uint64_t kDrainNs = 1000ull * 1000ull * 1000ull;     // 1 s per drain wait
constexpr int kThreads = 512;
constexpr int kD = 64;
constexpr int kTile = 128;                                      // rows per tile
constexpr uint32_t kTileBytes = kTile * kD * 2;                 // 16 KB
constexpr int kKvRows = 64;                                     // rows per K/V tile
constexpr uint32_t kKvTileBytes = kKvRows * kD * 2;             // 8 KB
constexpr uint32_t align1k(uint32_t x) { return (x + 1023u) & ~1023u; }
constexpr int kRing = 16;                                       // frames per head in the ring
constexpr int kStoreRows = 16;                                  // rows per output store box

// Status codes recorded in the device status word (bit per waiting role).
enum : uint32_t {
  kStKvLoad = 1u << 0, kStQLoad = 1u << 1, kStMma = 1u << 2, kStChain = 1u << 3,
  kStProd = 1u << 4, kStOut = 1u << 5, kStDrain = 1u << 6, kStMoEmpty = 1u << 7,
  kStAcEmpty = 1u << 8, kStRing = 1u << 9, kStConfig = 1u << 10
};

template <int P>
struct Layout {
  static constexpr int NKV = 5;                      // K/V tile pairs in flight
  static constexpr int NQ = 4;                       // Q tiles in flight (also output staging)
  static constexpr int NAC = 2;                      // transition-operand slots
  static constexpr int NM = 4;                       // state operand buffers: M_t in t % NM
  static constexpr int NCLAIM = 16;                  // claimed frames (jobs) in flight
  static constexpr uint32_t KV_SLOT = 2 * kKvTileBytes;             // K tile, then V tile
  static constexpr uint32_t AP_BYTES = kD * kD * 2;                 // A' (bf16)
  static constexpr uint32_t C_BYTES = kD * kD * 4;                  // c^T, fp32: row j = column j of c
  static constexpr uint32_t AC_BYTES = AP_BYTES + C_BYTES;          // one bulk copy
  static constexpr uint32_t AC_SLOT = align1k(AC_BYTES);
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
  static constexpr int B_KV_EMPTY = B_KV_FULL + NKV;
  static constexpr int B_Q_FULL = B_KV_EMPTY + NKV;
  static constexpr int B_Q_EMPTY = B_Q_FULL + NQ;
  static constexpr int B_AC_FULL = B_Q_EMPTY + NQ;      // [NAC] operands of the frame ready
  static constexpr int B_AC_EMPTY = B_AC_FULL + NAC;    // [NAC] frame consumed (recurrence warps)
  static constexpr int B_GB_FULL = B_AC_EMPTY + NAC;
  static constexpr int B_GB_FREE = B_GB_FULL + 2;
  static constexpr int B_CHAIN_DONE = B_GB_FREE + 2;
  static constexpr int B_M_READY = B_CHAIN_DONE + 1;
  static constexpr int B_MCH_FULL = B_M_READY + 1;      // [NM] M_t written (4 warps)
  static constexpr int B_MCH_FREE = B_MCH_FULL + NM;    // [NM] read-out MMAs of M_t done
  static constexpr int B_O_FULL = B_MCH_FREE + NM;
  static constexpr int B_O_FREE = B_O_FULL + 2;
  static constexpr int B_DRAIN = B_O_FREE + 2;         // [3] one per MMA issuer
  static constexpr int B_E1_STAGED = B_DRAIN + 3;       // [4] frame's A'/c written (4 warps)
  static constexpr int B_PUB_DONE = B_E1_STAGED + 4;    // [4] frame published to the ring
  static constexpr int B_STAGE = B_PUB_DONE + 4;        // [2] output tile staged (4 warps)
  static constexpr int B_CLAIM = B_STAGE + 2;           // [NCLAIM] frame of job j known
  static constexpr int NBAR = B_CLAIM + NCLAIM;
  static constexpr uint32_t OFF_TMEM_PTR = OFF_BAR + 8 * NBAR;
  static constexpr uint32_t OFF_ABORT = OFF_TMEM_PTR + 4;
  static constexpr uint32_t OFF_CLAIM_CTR = OFF_ABORT + 16;   // u32; rank 0's counts the head's claims
  static constexpr uint32_t OFF_CLAIMS = OFF_CLAIM_CTR + 16;  // [NCLAIM] s32: frame of job j, -1 = done
  static constexpr uint32_t BYTES = OFF_CLAIMS + 4 * NCLAIM;
  static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;              // base alignment slack

  // TMEM columns (each region 128 lanes)
  static constexpr uint32_t T_GB = 0;        // 2 x 64: [G; (K^T V)^T] accumulators
  static constexpr uint32_t T_O = 128;       // 2 x 64: output tile accumulators
  static constexpr uint32_t T_CHAIN = 256;   // 32 columns; value columns 0-31 in lanes
                                             // 32q+0..15, columns 32-63 in lanes 32q+16..31
  static constexpr uint32_t TMEM_COLS = 512;
};

static_assert(Layout<4>::SMEM_ALLOC <= 232448, "shared memory budget (P=4)");
static_assert(Layout<2>::SMEM_ALLOC <= 232448, "shared memory budget (P=2)");
static_assert(Layout<1>::SMEM_ALLOC <= 232448, "shared memory budget (P=1)");

// Scratch of gdn_frame_scan_noalloc, for callers that cannot allocate: the
// ring and its flags (TcParams below) for up to GDN_NOALLOC_MAX_HEADS heads at
// the largest cluster size, 12 MiB + 5 KiB. The ring starts at the base, the
// flags at kNoAllocRingBytes.
constexpr size_t kNoAllocRingBytes = (size_t)GDN_NOALLOC_MAX_HEADS * kRing * Layout<4>::AC_BYTES;
constexpr size_t kNoAllocFlagBytes =
    (size_t)GDN_NOALLOC_MAX_HEADS * (kRing + 4) * sizeof(unsigned long long);
static_assert(Layout<2>::AC_BYTES == Layout<4>::AC_BYTES, "one ring image size for every P");
static_assert(kNoAllocRingBytes % 256 == 0, "flags stay aligned");
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocRingBytes + kNoAllocFlagBytes];

struct TcParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_o;
  const float* gamma;
  const float* beta;
  const float* state_in;
  float* state_out;
  uint16_t* out;           // bf16 bit patterns
  unsigned int* status;
  unsigned long long timeout_ns;   // bound of every role wait
  // Transition operands shared by the CTAs of a head (P > 1), per head:
  // kRing frames of [A' (bf16, K-major, swizzled) | c^T (fp32)], their ready
  // flags and per-CTA progress.
  uint8_t* ring;                     // [heads][kRing][AC_BYTES]
  unsigned long long* ring_flag;     // [heads][kRing]: frame + 1 once published
  unsigned long long* ring_loaded;   // [heads][P]: frames loaded by each CTA
  int T;
  int S;
  int ntile;
  int nkv;          // K/V tiles per frame (kKvRows rows each)
  int chunk;        // output rows per CTA (multiple of 16); CTA r owns [r*chunk, (r+1)*chunk)
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

// Claims the next frame of the head: relaxed atomic add on the counter in the
// shared memory of the cluster's rank 0 (cluster address). Returns the frame.
__device__ __forceinline__ int claim_frame(uint32_t counter) {
  uint32_t old;
  asm volatile("atom.relaxed.cluster.shared::cluster.add.u32 %0, [%1], 1;"
               : "=r"(old)
               : "r"(counter)
               : "memory");
  return (int)old;
}

__device__ __forceinline__ int ld_shared_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// 8 floats -> one 16-byte chunk of bf16 (round to nearest even).
__device__ __forceinline__ uint4 pack8(const float* x) {
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

struct Ctl {
  uint32_t abort_addr;    // local shared address of the abort flag
  unsigned int* status;
  int P;
  uint64_t timeout_ns;    // bound of every role wait (1 s in the shipped library)
};

__device__ __forceinline__ bool aborted(const Ctl& c) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(c.abort_addr) : "memory");
  return v != 0;
}

__device__ __noinline__ void raise_abort(const Ctl& c, uint32_t code) {
  atomicOr(c.status, code);
  for (int q = 0; q < c.P; ++q) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(mapa(c.abort_addr, q)), "r"(1u)
                 : "memory");
  }
  fence_acq_rel_cluster();
}

// Bounded wait on a local mbarrier phase. False if the kernel is aborting or
// the wait ran out (then the abort is raised with `code`).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& c,
                                         uint32_t code) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (aborted(c)) return false;
    if (globaltimer_ns() - t0 > c.timeout_ns) {
      raise_abort(c, code);
      return false;
    }
  }
}

// Bounded poll with a short sleep between tests, for the recurrence's
// latency-critical handoffs: it reacts within tens of nanoseconds without
// taking issue slots from the other warps of its sub-partition.
__device__ __forceinline__ bool poll_bar(uint32_t bar, uint32_t parity, const Ctl& c,
                                         uint32_t code) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 32; ++i) {
      __nanosleep(20);
      if (mbar_test(bar, parity)) return true;
    }
    if (aborted(c)) return false;
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

// Bounded wait that ignores the abort flag (used to drain in-flight copies).
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
  while (true) {
    if (ld_acquire_gpu_u64(ptr) >= v) return true;
    if (aborted(c)) return false;
    if (globaltimer_ns() - t0 > c.timeout_ns) {
      raise_abort(c, code);
      return false;
    }
  }
}

// A'_t M_{t-1} into the recurrence accumulator, committed to `done`: A'_t
// K-major in `ac`, M_{t-1} as two MN-major 32-column blocks from `mprev`. Both
// in bf16: the product is small next to the exact fp32 gamma M term it is added
// to, so its relative rounding error enters the state scaled down by |A'| / gamma.
template <int P>
__device__ __forceinline__ void chain_mma(uint32_t tmem, uint32_t ac, uint32_t mprev, uint32_t done) {
  using L = Layout<P>;
  constexpr uint32_t id_chain = idesc_bf16(64, 32, 0, 1);    // A' K-major, M half MN-major
  tc_fence_after();
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const uint32_t dt = tmem + L::T_CHAIN + ((uint32_t)hf << 20);   // lane offset 16
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t aH = smem_desc(ac + kk * 32, 16, 1024, 2);
      const uint32_t mb = mprev + hf * L::MB_BLOCK + kk * 2 * L::MB_SBO;
      const uint64_t bH = smem_desc(mb, L::MB_BLOCK, L::MB_SBO, 4);
      mma_bf16(dt, aH, bH, id_chain, kk > 0 ? 1u : 0u);
    }
  }
  mma_commit(done);
}

template <int P>
__global__ void __launch_bounds__(kThreads, 1) gdn_tc_kernel(const __grid_constant__ TcParams p) {
  using L = Layout<P>;
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
  const uint32_t sb = (raw + 1023u) & ~1023u;         // 1 KB aligned base, same in every CTA
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int bh = blockIdx.x / P;
  const int T = p.T;
  const int nkv = p.nkv;

  auto bar = [&](int i) -> uint32_t { return sb + L::OFF_BAR + 8u * i; };
  auto kv_slot = [&](int i) -> uint32_t { return sb + L::OFF_KV + i * L::KV_SLOT; };
  auto q_slot = [&](int i) -> uint32_t { return sb + L::OFF_Q + i * kTileBytes; };
  auto ac_slot = [&](int i) -> uint32_t { return sb + L::OFF_AC + i * L::AC_SLOT; };
  auto mch = [&](int i) -> uint32_t { return sb + L::OFF_MCH + i * L::M_BUF; };
  // Frame of this CTA's job j (claimed by its K/V loader), or -1 past the last one.
  auto claim_slot = [&](int j) -> uint32_t { return sb + L::OFF_CLAIMS + 4u * (j % L::NCLAIM); };
  // Output rows of this CTA, in every frame, and its Q tiles.
  const int r0 = (int)rank * p.chunk;
  const int r1 = min(p.S, r0 + p.chunk);
  const int nq = r1 > r0 ? (r1 - r0 + kTile - 1) / kTile : 0;
  const uint32_t tmem_ptr = sb + L::OFF_TMEM_PTR;
  Ctl ctl{sb + L::OFF_ABORT, p.status, P, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NKV; ++i) {
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
    mbar_init(bar(L::B_M_READY), 4);
    for (int i = 0; i < 3; ++i) mbar_init(bar(L::B_DRAIN + i), 1);
    for (int i = 0; i < L::NCLAIM; ++i) mbar_init(bar(L::B_CLAIM + i), 1);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(ctl.abort_addr), "r"(0u) : "memory");
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(sb + L::OFF_CLAIM_CTR), "r"(0u) : "memory");
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    prefetch_tmap(&p.tm_o);
  }
  if (warp == 2) {
    tmem_alloc(tmem_ptr, L::TMEM_COLS);
    tmem_relinquish();
  }
  // The recurrence warps read the initial state before the cluster barrier
  // below. Rank 0 writes the final state only after that barrier, so with
  // state_in == state_out no CTA of the head can read a row rank 0 has
  // already overwritten. Lane l of warp quarter q owns row 16q + (l % 16),
  // value columns 32 (l / 16) .. + 32.
  float m[32];
  if (warp >= 4 && warp < 8) {
    const int row = (warp & 3) * 16 + (lane & 15);
    const int col0 = 32 * (lane >> 4);
#pragma unroll
    for (int jj = 0; jj < 32; ++jj)
      m[jj] = p.state_in ? p.state_in[((size_t)bh * kD + row) * kD + col0 + jj] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();   // the CTAs of a head start together
  uint32_t tmem;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(tmem_ptr) : "memory");

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ K/V loader (claims the frames to produce)
    // The CTAs of a head claim the frames they produce from one counter in
    // rank 0's shared memory, so a CTA that streams faster produces more of
    // them. Each claim is made one frame ahead, and that frame's tiles are
    // prefetched into L2 while the current one loads, so the loads below see L2
    // latency rather than loaded-HBM latency. Inputs are read once: evict them
    // first, keeping L2 for the ring and the prefetches.
    const uint64_t stream_pol = policy_evict_first();
    const uint32_t counter = mapa(sb + L::OFF_CLAIM_CTR, 0);
    auto prefetch_frame = [&](int f) {
      for (int i = 0; i < nkv; ++i) {
        tma_prefetch_3d(&p.tm_k, 0, i * kKvRows, bh * T + f);
        tma_prefetch_3d(&p.tm_v, 0, i * kKvRows, bh * T + f);
      }
    };
    int next = claim_frame(counter);
    if (next < T) prefetch_frame(next);
#ifdef GDN_TRACE
    {
      unsigned int sm;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
      GDN_TRACE_CTA(0, sm);
    }
#endif
    int it = 0;
    for (int j = 0;; ++j) {
      const int f = next < T ? next : -1;
      // Job j's frame for the MMA issuer, the A'/c warps and the publisher. They
      // trail this loop by fewer than NCLAIM jobs, so the slot is free again.
      asm volatile("st.shared.s32 [%0], %1;" ::"r"(claim_slot(j)), "r"(f) : "memory");
      mbar_arrive(bar(L::B_CLAIM + j % L::NCLAIM));
      if (f < 0) {
        GDN_TRACE_CTA(2, globaltimer_ns());
        GDN_TRACE_CTA(3, j);
        break;
      }
      if (j == 2) GDN_TRACE_CTA(1, globaltimer_ns());
      next = claim_frame(counter);
      if (next < T) prefetch_frame(next);
      bool ok = true;
      for (int i = 0; i < nkv; ++i, ++it) {
        const int slot = it % L::NKV;
        if (!wait_bar(bar(L::B_KV_EMPTY + slot), ((it / L::NKV) & 1) ^ 1, ctl, kStKvLoad)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(L::B_KV_FULL + slot), 2 * kKvTileBytes);
        if (i == 0) GDN_TRACE_EV(11, j);
        if (i == nkv - 1) GDN_TRACE_EV(12, j);
        tma_load_3d_hint(kv_slot(slot), &p.tm_k, bar(L::B_KV_FULL + slot), 0, i * kKvRows, bh * T + f,
                         stream_pol);
        tma_load_3d_hint(kv_slot(slot) + kKvTileBytes, &p.tm_v, bar(L::B_KV_FULL + slot), 0,
                         i * kKvRows, bh * T + f, stream_pol);
      }
      if (!ok) break;
    }
    for (int k = it - 1; k >= 0 && k >= it - L::NKV; --k)
      drain_bar(bar(L::B_KV_FULL + k % L::NKV), (k / L::NKV) & 1, ctl);
  } else if (warp == 0 && lane == 16 && P > 1) {
    // ------------------------------------------------ publisher of this CTA's frames
    // The fence and the release below wait for the producer warps' ring writes
    // to be performed; doing them here keeps the producer warps streaming.
    for (int j = 0;; ++j) {
      if (!wait_bar(bar(L::B_CLAIM + j % L::NCLAIM), (j / L::NCLAIM) & 1, ctl, kStProd)) break;
      const int f = ld_shared_s32(claim_slot(j));
      if (f < 0) break;
      if (!wait_bar(bar(L::B_E1_STAGED + (j & 3)), (j >> 2) & 1, ctl, kStProd)) break;
      GDN_TRACE_EV(20, j);
      __threadfence();
      fence_proxy_async_global();
      st_release_gpu_u64(p.ring_flag + (size_t)bh * kRing + f % kRing, (unsigned long long)(f + 1));
      mbar_arrive(bar(L::B_PUB_DONE + (j & 3)));
      GDN_TRACE_EV(8, j);
    }
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
        if (i == 0) GDN_TRACE_EV(13, t / P);
        tma_load_3d_hint(q_slot(slot), &p.tm_q, bar(L::B_Q_FULL + slot), 0, r0 + i * kTile, bh * T + t,
                         stream_pol);
      }
    }
    for (int k = it - 1; k >= 0 && k >= it - L::NQ; --k)
      drain_bar(bar(L::B_Q_FULL + k % L::NQ), (k / L::NQ) & 1, ctl);
  } else if (warp == 2 && lane == 0) {
    // ------------------------------------------------ recurrence MMA issuer
    // tcgen05.commit tracks the MMAs of the issuing thread, so each of the three
    // MMA streams has its own issuer and waits only on its own inputs.
    for (int t = 0; t < T; ++t) {
      if (!poll_bar(bar(L::B_M_READY), t & 1, ctl, kStMma) ||
          !poll_bar(bar(L::B_AC_FULL + t % NAC), (t / NAC) & 1, ctl, kStMma))
        break;
      chain_mma<P>(tmem, ac_slot(t % NAC), mch((t + L::NM - 1) % L::NM), bar(L::B_CHAIN_DONE));
      GDN_TRACE_EV(0, t);
#ifdef GDN_TRACE
      if (rank == 0 && bh < kTraceHeads && t < kTraceFrames)
        g_trace_heads[bh * kTraceFrames + t] = globaltimer_ns();
#endif
    }
    mma_commit(bar(L::B_DRAIN + 0));
    drain_bar(bar(L::B_DRAIN + 0), 0, ctl);
  } else if (warp == 1 && lane == 16) {
    // ------------------------------------------------ [K V]^T K MMA issuer (own frames)
    constexpr uint32_t id_gb = idesc_bf16(128, 64, 1, 1);      // [K V]^T and K, both MN-major
    int kvit = 0;
    bool ok = true;
    for (int j = 0; ok; ++j) {
      if (!wait_bar(bar(L::B_CLAIM + j % L::NCLAIM), (j / L::NCLAIM) & 1, ctl, kStMma)) break;
      if (ld_shared_s32(claim_slot(j)) < 0) break;
      const int b = j & 1;
      if (!wait_bar(bar(L::B_GB_FREE + b), ((j >> 1) & 1) ^ 1, ctl, kStMma)) break;
      for (int i = 0; i < nkv; ++i, ++kvit) {
        const int slot = kvit % L::NKV;
        if (!wait_bar(bar(L::B_KV_FULL + slot), (kvit / L::NKV) & 1, ctl, kStMma)) {
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
      GDN_TRACE_EV(14, j);
    }
    mma_commit(bar(L::B_DRAIN + 1));
    drain_bar(bar(L::B_DRAIN + 1), 0, ctl);
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
        if (i == 0 && t % P == (int)rank) GDN_TRACE_EV(15, t / P);
      }
      if (ok) mma_commit(bar(L::B_MCH_FREE + u));   // M_t no longer read here
    }
    mma_commit(bar(L::B_DRAIN + 2));
    drain_bar(bar(L::B_DRAIN + 2), 0, ctl);
  } else if (warp == 3 && lane == 0 && P > 1) {
    // ------------------------------------------------ loader of the transition operands
    // Every frame, this CTA's own included, arrives through the ring, in frame
    // order, so each slot wait below is for the next phase of its barrier. The
    // bulk load completes the slot's "full" barrier itself.
    // The ring keeps the normal eviction priority: the streams around it are
    // evict-first, so it stays in L2 anyway. With evict-last, lines of rings that
    // earlier launches left at other addresses kept their priority and crowded
    // out the live ring: the same launch then ran up to 7x slower.
    const uint64_t ring_pol = policy_evict_normal();
    int t = 0;
    for (; t < T; ++t) {
      const int s = t % NAC;
      const size_t rs = (size_t)bh * kRing + t % kRing;
      if (!wait_global_ge(p.ring_flag + rs, (unsigned long long)(t + 1), ctl, kStRing)) break;
      GDN_TRACE_EV(16, t);
      if (!wait_bar(bar(L::B_AC_EMPTY + s), ((t / NAC) & 1) ^ 1, ctl, kStRing)) break;
      GDN_TRACE_EV(18, t);
      // Frame t - NAC has been consumed here, so its load (and every earlier one)
      // completed: ring slots up to it may be reused by their producers.
      if (t >= NAC)
        st_relaxed_gpu_u64(p.ring_loaded + (size_t)bh * P + rank, (unsigned long long)(t - NAC + 1));
      fence_proxy_async_global();
      mbar_arrive_expect_tx(bar(L::B_AC_FULL + s), L::AC_BYTES);
      bulk_load_global_hint(ac_slot(s), p.ring + rs * L::AC_BYTES, L::AC_BYTES, bar(L::B_AC_FULL + s),
                            ring_pol);
      GDN_TRACE_EV(17, t);
    }
    // Loads still in flight target this CTA: let them land before it can leave.
    for (int k = t - 1; k >= 0 && k >= t - NAC; --k)
      drain_bar(bar(L::B_AC_FULL + k % NAC), (k / NAC) & 1, ctl);
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------ recurrence epilogue
    // The accumulator holds A' M for the 64 state rows: value columns 0-31 of
    // row 16q+i in TMEM lane 32q+i, columns 32-63 in lane 32q+16+i. So lane l
    // of warp quarter q owns row 16q+(l%16), columns 32*(l/16)..+32.
    const int qd = warp & 3;
    const int hf = lane >> 4;
    const int row = qd * 16 + (lane & 15);
    // m: the fp32 state, row `row`, columns 32hf..32hf+31 (loaded before the
    // first cluster barrier)
    auto store_state = [&](uint32_t buf) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        st_shared_v4(buf + hf * L::MB_BLOCK + swz_off(row, c, L::MB_RW, 2), pack8(&m[8 * c]));
    };
    store_state(mch(L::NM - 1));               // M_{-1} = M_0, read by the first MMA
    fence_proxy_async_cta();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::B_M_READY));
    const float* gam = p.gamma + (size_t)bh * T;
    float g_next = __ldg(gam);
    bool ok = true;
    int t = 0;
    for (; t < T; ++t) {
      const float g = g_next;
      if (t + 1 < T) g_next = __ldg(gam + t + 1);
      const int s = t % NAC;
      const bool acok = warp_wait(bar(L::B_AC_FULL + s), (t / NAC) & 1, ctl, kStChain);
      if (acok && lane == 0 && warp == 4) GDN_TRACE_EV(21, t);
      // M_t goes to buffer t % NM, which held M_{t-NM}: its read-out MMAs must be done.
      uint32_t cd = 0;
      if (acok && lane == 0) cd = poll_bar(bar(L::B_CHAIN_DONE), t & 1, ctl, kStChain) ? 1u : 0u;
      cd = __shfl_sync(0xffffffffu, cd, 0);
      if (cd) mbar_test(bar(L::B_CHAIN_DONE), t & 1);    // acquire for every lane
      if (!acok || !cd ||
          !warp_wait(bar(L::B_MCH_FREE + t % L::NM), ((t / L::NM) & 1) ^ 1, ctl, kStMoEmpty)) {
        ok = false;
        break;
      }
      if (lane == 0 && warp == 4) GDN_TRACE_EV(1, t);
      tc_fence_after();
      uint32_t d[32];
      {
        uint32_t r0[16], r1[16];
        tmem_ld16(tmem + L::T_CHAIN + ((uint32_t)(qd * 32) << 16), r0);
        tmem_ld16(tmem + L::T_CHAIN + 16 + ((uint32_t)(qd * 32) << 16), r1);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          d[e] = r0[e];
          d[16 + e] = r1[e];
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
        mbar_arrive(bar(L::B_M_READY));        // next MMA operand ready; accumulator free
        mbar_arrive(bar(L::B_AC_EMPTY + s));   // A'_t read by its MMA, c_t read here: slot free
        mbar_arrive(bar(L::B_MCH_FULL + t % L::NM));   // M_t ready for the read-out
        if (warp == 4) GDN_TRACE_EV(2, t);
      }
    }
    if (ok && p.state_out && rank == 0) {      // every CTA holds the same state
#pragma unroll
      for (int jj = 0; jj < 32; ++jj)
        p.state_out[((size_t)bh * kD + row) * kD + 32 * hf + jj] = m[jj];
    }
  } else if (warp >= 8 && warp < 12) {
    // ------------------------------------------------ A' and c from [G; (K^T V)^T]
    const int qd = warp & 3;
    const int lrow = qd * 32 + lane;           // accumulator row = TMEM lane
    const float* gam = p.gamma + (size_t)bh * T;
    const float* bet = p.beta + (size_t)bh * T;
    unsigned long long ring_seen = 0;            // lowest CTA progress last read (lane 0)
    for (int j = 0;; ++j) {
      if (!warp_wait(bar(L::B_CLAIM + j % L::NCLAIM), (j / L::NCLAIM) & 1, ctl, kStProd)) break;
      const int f = ld_shared_s32(claim_slot(j));
      if (f < 0) break;
      const int b = j & 1;
      const float g = __ldg(gam + f);
      const float be = __ldg(bet + f);
      if (!warp_wait(bar(L::B_GB_FULL + b), (j >> 1) & 1, ctl, kStProd)) break;
      if (lane == 0 && warp == 8) GDN_TRACE_EV(6, j);
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
      // Convert first, then wait for the slot: after the wait only stores remain.
      // A' rows are packed in place: chunk c (8 values) becomes 4 bf16x2 words in
      // v[8c..8c+3].
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
      const int s = f % NAC;
      uint32_t sent = 1;
      if (P == 1) {
        // Every frame is ours: build it in the local slot once frame f - NAC is consumed.
        if (!warp_wait(bar(L::B_AC_EMPTY + s), ((f / NAC) & 1) ^ 1, ctl, kStAcEmpty)) break;
        if (lane == 0 && warp == 8) GDN_TRACE_EV(7, j);
        const uint32_t slot = ac_slot(s);
        if (lrow < kD) {
          // row lrow of A', bf16 hi + lo, K-major, 128-byte swizzle
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t off = swz_off(lrow, c, 128, 3);
            st_shared_v4(slot + off, make_uint4(v[8 * c], v[8 * c + 1], v[8 * c + 2], v[8 * c + 3]));
          }
        } else {
          // column (lrow - 64) of c = row (lrow - 64) of c^T
          const uint32_t dst = slot + L::AP_BYTES + (lrow - kD) * kD * 4;
#pragma unroll
          for (int i = 0; i < kD; i += 4)
            st_shared_v4(dst + i * 4, make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]));
        }
        fence_proxy_async_cta();     // visible to the MMA
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_E1_STAGED + (j & 3)));
        if (warp == 8 && lane == 0) {
          sent = wait_bar(bar(L::B_E1_STAGED + (j & 3)), (j >> 2) & 1, ctl, kStProd) ? 1u : 0u;
          if (sent) mbar_arrive(bar(L::B_AC_FULL + s));
          GDN_TRACE_EV(8, j);
        }
      } else {
        // Publish to every CTA of the head (this one included) through the ring.
        // Its slot is free once each CTA has loaded frame f - kRing.
        const size_t rs = (size_t)bh * kRing + f % kRing;
        uint32_t ok = 1;
        const unsigned long long need = (unsigned long long)(f - kRing + 1);
        if (lane == 0 && f >= kRing && ring_seen < need) {
          // Re-read the CTAs' progress only when the last reading no longer covers f.
          unsigned long long lo = ~0ull;
          for (int q = 0; q < P && ok; ++q) {
            ok = wait_global_ge(p.ring_loaded + (size_t)bh * P + q, need, ctl, kStRing) ? 1u : 0u;
            const unsigned long long v = ld_acquire_gpu_u64(p.ring_loaded + (size_t)bh * P + q);
            lo = v < lo ? v : lo;
          }
          if (ok) ring_seen = lo;
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if (lane == 0 && warp == 8) GDN_TRACE_EV(7, j);
        uint8_t* img = p.ring + rs * L::AC_BYTES;
        const uint64_t ring_pol = policy_evict_normal();
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
        if (lane == 0 && warp == 8) GDN_TRACE_EV(19, j);
        // The publisher (warp 0, lane 16) fences and raises the ring flag; it must
        // have published own frame j - 4 before its staging barrier is reused.
        if (j >= 4 && !warp_wait(bar(L::B_PUB_DONE + (j & 3)), ((j >> 2) - 1) & 1, ctl, kStProd))
          break;
        if (lane == 0) mbar_arrive(bar(L::B_E1_STAGED + (j & 3)));
      }
      sent = __shfl_sync(0xffffffffu, sent, 0);   // warp-uniform verdict (other warps: abort flag)
      if (!sent) break;
    }
  } else if (warp >= 12) {
    // ------------------------------------------------ output tiles: TMEM -> bf16 -> TMA store
    // Each tile is staged in the Q slot it was computed from (its MMA is done)
    // and written with bulk tensor stores of 16 rows, this CTA's rows only; the
    // slot goes back to the Q loader once the stores have read it. Bulk stores
    // keep the SM's generic write queue short, so the GPU-scope fences elsewhere
    // stay cheap.
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
        if (i == 0 && lane == 0 && warp == 12 && t % P == (int)rank) GDN_TRACE_EV(9, t / P);
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
          if (i == nq - 1 && t % P == (int)rank) GDN_TRACE_EV(10, t / P);
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
  cluster_sync();   // no CTA leaves while a peer may still write into its shared memory
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

// [B*H*T][S][64] bf16 viewed as a 3-D tensor (64, S, B*H*T); 64 x box_rows x 1
// boxes with the 128-byte swizzle. Rows past S inside a frame read as zero and
// are not stored.
bool make_map(CUtensorMap* m, const void* base, int S, long long frames, int box_rows = kTile) {
  return make_frame_map(m, base, kD, S, frames, box_rows);
}

template <int P>
const void* kernel_ptr() {
  return reinterpret_cast<const void*>(&gdn_tc_kernel<P>);
}

// Raises the kernel's dynamic shared-memory limit. The attribute belongs to the
// kernel on each device, so it is set once per device (concurrent first calls
// both set it, which is harmless).
template <int P>
cudaError_t prepare() {
  static std::atomic<bool> done[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel_ptr<P>(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Layout<P>::SMEM_ALLOC);
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

// Clusters of P CTAs (one CTA per SM) that fit on the current device at
// once, or -1 if there is no usable device (host-only planning). A cluster
// sits inside one GPC, so clusters of 4 leave a few SMs of each GPC unused:
// 33 fit on a 148-SM B200, about 9/40 of the SM count; clusters of 2 fill the
// device. Only the cluster size depends on this count (the clusters never
// wait on each other), so it comes from the SM count rather than from the
// driver's cluster-occupancy query: that query, made before the caller's
// large allocations, was followed by scans running 20-45 % slower.
template <int P>
int resident_clusters() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return P == 4 ? sms * 9 / 40 : sms / P;
}

// Address of g_noalloc_scratch on the current device. cudaGetSymbolAddress
// (which allocates nothing) runs once per device, with that device current;
// the address is kept for later calls.
cudaError_t noalloc_scratch(uint8_t** out) {
  static std::atomic<uint8_t*> cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  uint8_t* a = cache[dev].load(std::memory_order_acquire);
  if (!a) {
    void* sym = nullptr;
    e = cudaGetSymbolAddress(&sym, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    a = static_cast<uint8_t*>(sym);
    cache[dev].store(a, std::memory_order_release);
  }
  *out = a;
  return cudaSuccess;
}

// fixed_scratch: null for gdn_frame_scan (stream-ordered scratch when P > 1),
// g_noalloc_scratch's address for gdn_frame_scan_noalloc.
template <int P>
cudaError_t launch_p(const Problem& pr, uint8_t* fixed_scratch) {
  cudaError_t e = prepare<P>();
  if (e != cudaSuccess) return e;
  TcParams p;
  const long long frames = (long long)pr.B * pr.H * pr.T;
  if (!make_map(&p.tm_q, pr.q, pr.S, frames) || !make_map(&p.tm_k, pr.k, pr.S, frames, kKvRows) ||
      !make_map(&p.tm_v, pr.v, pr.S, frames, kKvRows) || !make_map(&p.tm_o, pr.out, pr.S, frames, kStoreRows))
    return cudaErrorInvalidValue;
  unsigned int* status = status_word();
  if (!status) return cudaErrorInvalidDevice;
  p.gamma = pr.gamma;
  p.beta = pr.beta;
  p.state_in = pr.state_in;
  p.state_out = pr.state_out;
  p.out = static_cast<uint16_t*>(pr.out);
  p.status = status;
  p.timeout_ns = wait_budget_ns();
  p.T = pr.T;
  p.S = pr.S;
  p.ntile = (pr.S + kTile - 1) / kTile;
  p.nkv = (pr.S + kKvRows - 1) / kKvRows;
  p.chunk = ((pr.S + P - 1) / P + 15) / 16 * 16;
  p.s = pr.key_scale;
  const double sd = 1.0 / ((double)kD * (double)pr.S);
  p.s2 = (float)sd;
  p.delta = pr.delta ? 1.f : 0.f;

  // Ring of transition operands shared by the CTAs of each head (P > 1):
  // stream-ordered scratch, released right after the launch on the same stream.
  const size_t heads = (size_t)pr.B * pr.H;
  const size_t ring_bytes = heads * kRing * Layout<P>::AC_BYTES;
  const size_t ctrl_bytes = heads * (kRing + P) * sizeof(unsigned long long);
  void* scratch = nullptr;
  p.ring = nullptr;
  p.ring_flag = nullptr;
  p.ring_loaded = nullptr;
  if (P > 1 && fixed_scratch) {
    // The fixed array: nothing to allocate; its flags must start at zero.
    if (heads > (size_t)GDN_NOALLOC_MAX_HEADS) return cudaErrorInvalidValue;
    p.ring = fixed_scratch;
    p.ring_flag = reinterpret_cast<unsigned long long*>(fixed_scratch + kNoAllocRingBytes);
    p.ring_loaded = p.ring_flag + heads * kRing;
    e = cudaMemsetAsync(p.ring_flag, 0, ctrl_bytes, pr.stream);
    if (e != cudaSuccess) return e;
  } else if (P > 1) {
    e = cudaMallocAsync(&scratch, ring_bytes + ctrl_bytes, pr.stream);
    if (e != cudaSuccess) return e;
    p.ring = static_cast<uint8_t*>(scratch);
    p.ring_flag = reinterpret_cast<unsigned long long*>(p.ring + ring_bytes);
    p.ring_loaded = p.ring_flag + heads * kRing;
    e = cudaMemsetAsync(p.ring_flag, 0, ctrl_bytes, pr.stream);
    if (e != cudaSuccess) {
      cudaFreeAsync(scratch, pr.stream);
      return e;
    }
  }

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(pr.B * pr.H * P), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Layout<P>::SMEM_ALLOC;
  cfg.stream = pr.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gdn_tc_kernel<P>, p);
  if (scratch) {
    const cudaError_t ef = cudaFreeAsync(scratch, pr.stream);
    if (e == cudaSuccess) e = ef;
  }
  return e;
}

}  // namespace

int tc_ctas_per_head(int B, int H, int T, int S, int D) {
  if (D != kD) return 0;
  const long long heads = (long long)B * H;
  if (heads * (long long)T >= (1ll << 31) || (long long)S * kD * 2 >= (1ll << 40)) return 0;
  if (heads * 4 > (1ll << 31) - 1) return 0;
  // Tuning override: GDN_TC_CTAS=1|2|4 forces the cluster size.
  if (const char* e = getenv("GDN_TC_CTAS")) {
    const int v = atoi(e);
    if (v == 1 || v == 2 || v == 4) return v;
  }
  if (T == 1) return 1;
  // Largest cluster size whose clusters all fit on the device at once.
  const int c4 = resident_clusters<4>();
  const int c2 = resident_clusters<2>();
  const int sms = 148;                     // planning without a device: a B200
  const long long fit4 = c4 >= 0 ? c4 : sms * 9 / 40;
  const long long fit2 = c2 >= 0 ? c2 : sms / 2;
  if (heads <= fit4) return 4;
  if (heads <= fit2) return 2;
  return 1;
}

cudaError_t launch_tc_bf16(const Problem& p, int ctas_per_head) {
  switch (ctas_per_head) {
    case 1: return launch_p<1>(p, nullptr);
    case 2: return launch_p<2>(p, nullptr);
    case 4: return launch_p<4>(p, nullptr);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_tc_bf16_noalloc(const Problem& p, int ctas_per_head) {
  if ((long long)p.B * p.H > GDN_NOALLOC_MAX_HEADS) return cudaErrorInvalidValue;
  if (ctas_per_head == 1) return launch_p<1>(p, nullptr);   // no ring, no scratch
  uint8_t* scratch = nullptr;
  const cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  switch (ctas_per_head) {
    case 2: return launch_p<2>(p, scratch);
    case 4: return launch_p<4>(p, scratch);
    default: return cudaErrorInvalidValue;
  }
}

#ifdef GDN_TRACE
extern "C" __attribute__((visibility("default"))) int gdn_trace_copy(void* dst, size_t bytes) {
  const size_t n = sizeof(g_trace) < bytes ? sizeof(g_trace) : bytes;
  return cudaMemcpyFromSymbol(dst, g_trace, n) == cudaSuccess ? (int)n : -1;
}
extern "C" __attribute__((visibility("default"))) int gdn_trace_cta_copy(void* dst, size_t bytes) {
  const size_t n = sizeof(g_trace_cta) < bytes ? sizeof(g_trace_cta) : bytes;
  return cudaMemcpyFromSymbol(dst, g_trace_cta, n) == cudaSuccess ? (int)n : -1;
}
extern "C" __attribute__((visibility("default"))) int gdn_trace_heads_copy(void* dst, size_t bytes) {
  const size_t n = sizeof(g_trace_heads) < bytes ? sizeof(g_trace_heads) : bytes;
  return cudaMemcpyFromSymbol(dst, g_trace_heads, n) == cudaSuccess ? (int)n : -1;
}
#endif

}  // namespace gdn
