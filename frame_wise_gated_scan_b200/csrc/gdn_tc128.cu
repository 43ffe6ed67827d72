// tcgen05 kernel of the frame-wise Gated DeltaNet scan for D = 128, bf16 inputs.
//
// The update ("NVIDIA Apresenta SANA-WM ...", acheiumaia.com.br, section
// "A Arquitetura", item "1. Atencao Linear Hibrida com Gated DeltaNet"), per
// head and frame t with s = 1/sqrt(D*S):
//     W = (sK) M,  R = V - gamma W,  M' = gamma M + beta (sK)^T R,  O = Q M'.
// By associativity (sK)^T R = s K^T V - gamma s^2 (K^T K) M, so
//     M' = gamma M + beta s (K^T V + A'' M),   A'' = -gamma s K^T K.
// K^T K and K^T V depend only on the frame's inputs, and the state-dependent
// product A'' M can accumulate straight onto K^T V in the same TMEM
// accumulator: one MMA stream forms [K^T K | K^T V] = K^T [K V] (M = 128,
// N = 256), and the recurrence adds A'' M into its right half.
//
// Work split: a cluster of two CTAs per head, by role, each streaming half of
// a frame's bytes.
//  * rank 0, the producer: streams K and V (64-row tiles, four in flight),
//    forms K^T [K V] into one of two TMEM accumulators, keeps the fp32 state
//    in the registers of eight warps for all T frames, turns K^T K into A''
//    (bf16), issues A'' M_{t-1} onto K^T V, updates M_t = gamma M + beta s D in
//    fp32 and writes its bf16 copy, which one thread pushes into the reader's
//    shared memory with a bulk copy over distributed shared memory;
//  * rank 1, the reader: streams Q (128-row tiles, five in flight), reads out
//    O_t = Q_t M_t on the tensor cores from the pushed M_t, and stores O with
//    TMA from the tile's own Q slot. When the read-out MMAs of a frame are
//    done, a multicast tcgen05.commit tells the producer the slot is free.
// Precision is that of the D = 64 kernel: A'' and M enter their product in
// bf16, accumulation and the state are fp32, O is rounded to bf16.
//
// Every wait is bounded (gdn_wait.cuh). On abort every role stops; after the
// last cluster barrier each CTA drains what its peer may still have in flight
// towards it (pushed state copies, multicast commits) before either leaves.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdlib.h>

#include <atomic>

#include "gdn.h"
#include "gdn_internal.h"
#include "gdn_wait.cuh"
#include "sm100_ptx.h"

namespace gdn {
namespace {

using namespace ptx;
using namespace wait;

constexpr int kD = 128;
constexpr int kThreads = 384;                       // 12 warps
constexpr int kKvRows = 64;                         // rows per K/V tile
constexpr int kQRows = 128;                         // rows per Q / output tile
constexpr uint32_t kBox64 = 64 * 128;               // 64 rows x 64 columns, bf16: 8 KB
constexpr uint32_t kStage = 4 * kBox64;             // K cols 0-63 | K cols 64-127 | V | V: 32 KB
constexpr uint32_t kQTile = 2 * 128 * 128;          // 128 rows x 128 columns, bf16: 32 KB
constexpr uint32_t kMat = 128 * 128 * 2;            // a 128 x 128 bf16 operand: 32 KB
constexpr uint32_t kAtom = 128 * 128;               // 128 rows x 128 bytes: 16 KB
constexpr int NKV = 4;
constexpr int NQ = 5;

// Shared memory, from a 1 KB aligned base. The two roles lay out their data
// differently; barriers sit at one offset in both (the peer addresses them).
constexpr uint32_t OFF_KV = 0;                       // producer: [NKV] stages
constexpr uint32_t OFF_A = OFF_KV + NKV * kStage;    // producer: A'' (K-major, two atoms)
constexpr uint32_t OFF_M = OFF_A + kMat;             // producer: [2] M_t in bf16 (MN-major)
constexpr uint32_t OFF_Q = 0;                        // reader: [NQ] Q tiles, then output staging
constexpr uint32_t OFF_MR = OFF_Q + NQ * kQTile;     // reader: [2] pushed M_t
constexpr uint32_t OFF_BAR = OFF_M + 2 * kMat;
static_assert(OFF_MR + 2 * kMat <= OFF_BAR, "reader data fits below the barriers");
enum {
  // producer
  B_KV_FULL = 0, B_KV_EMPTY = B_KV_FULL + NKV, B_ACC_FULL = B_KV_EMPTY + NKV,
  B_ACC_FREE = B_ACC_FULL + 2, B_A_READY = B_ACC_FREE + 2, B_CHAIN = B_A_READY + 1,
  B_M_READY = B_CHAIN + 1, B_M_WRITTEN = B_M_READY + 1, B_MR_FREE = B_M_WRITTEN + 2,
  B_DRAIN_P = B_MR_FREE + 2,
  // reader
  B_Q_FULL = B_DRAIN_P + 2, B_Q_EMPTY = B_Q_FULL + NQ, B_MR_FULL = B_Q_EMPTY + NQ,
  B_O_FULL = B_MR_FULL + 2, B_O_FREE = B_O_FULL + 2, B_STAGE = B_O_FREE + 2,
  B_DRAIN_R = B_STAGE + 2,
  NBAR = B_DRAIN_R + 1
};
constexpr uint32_t OFF_TMEM_PTR = OFF_BAR + 8 * NBAR;
constexpr uint32_t OFF_ABORT = OFF_TMEM_PTR + 4;
constexpr uint32_t OFF_PUSHED = OFF_ABORT + 4;      // producer: M_t copies issued
constexpr uint32_t OFF_COMMITTED = OFF_PUSHED + 4;  // reader: frames whose release was committed
constexpr uint32_t BYTES = OFF_COMMITTED + 4;
constexpr uint32_t SMEM_ALLOC = BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

enum : uint32_t {
  kStLoad = 1u << 24, kStMma = 1u << 25, kStEpi = 1u << 26, kStPush = 1u << 27,
  kStOut = 1u << 28, kStDrain = 1u << 29, kStConfig = 1u << 30
};

struct Tc128Params {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_o;
  const float* gamma;
  const float* beta;
  const float* state_in;
  float* state_out;
  unsigned int* status;
  unsigned long long timeout_ns;
  int T;
  int S;
  float s;       // key scale 1/sqrt(D*S)
  float delta;   // 1: delta rule; 0: GDN_FLAG_NO_DELTA (A'' = 0)
};

__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t chunk) {
  const uint32_t off = row * 128u + chunk * 16u;
  return off ^ (((off >> 7) & 7u) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Arrives (one) on the mbarrier at the same shared-memory offset in every CTA
// of `mask`, once the tcgen05 operations this thread issued so far complete.
__device__ __forceinline__ void mma_commit_multicast(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// 64 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&v)[64]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t r16[16];
    tmem_ld16(taddr + 16 * c, r16);
#pragma unroll
    for (int e = 0; e < 16; ++e) v[16 * c + e] = r16[e];
  }
  tmem_wait_ld();
}

__global__ void __launch_bounds__(kThreads, 1) gdn_tc128_kernel(const __grid_constant__ Tc128Params p) {
  extern __shared__ uint8_t smem_raw[];
  {
    uint32_t dsmem;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dsmem));
    if (blockDim.x != kThreads || blockDim.y != 1 || blockDim.z != 1 || dsmem < SMEM_ALLOC ||
        cluster_nctarank() != 2u) {
      if (threadIdx.x == 0) atomicOr(p.status, kStConfig);
      return;
    }
  }
  const uint32_t sb = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int bh = blockIdx.x >> 1;
  const int T = p.T;
  const int nkv = (p.S + kKvRows - 1) / kKvRows;
  const int nq = (p.S + kQRows - 1) / kQRows;
  auto bar = [&](int i) -> uint32_t { return sb + OFF_BAR + 8u * i; };
  Ctl ctl{sb + OFF_ABORT, p.status, p.timeout_ns, 2};
  const uint32_t tmem_cols = rank == 0 ? 512u : 256u;

  if (threadIdx.x == 0) {
    if (rank == 0) {
      for (int i = 0; i < NKV; ++i) {
        mbar_init(bar(B_KV_FULL + i), 1);
        mbar_init(bar(B_KV_EMPTY + i), 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(B_ACC_FULL + i), 1);
        mbar_init(bar(B_ACC_FREE + i), 8);
        mbar_init(bar(B_M_WRITTEN + i), 8);
        mbar_init(bar(B_MR_FREE + i), 1);
        mbar_init(bar(B_DRAIN_P + i), 1);
      }
      mbar_init(bar(B_A_READY), 8);
      mbar_init(bar(B_CHAIN), 1);
      mbar_init(bar(B_M_READY), 8);
    } else {
      for (int i = 0; i < NQ; ++i) {
        mbar_init(bar(B_Q_FULL + i), 1);
        mbar_init(bar(B_Q_EMPTY + i), 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(B_MR_FULL + i), 1);
        mbar_init(bar(B_O_FULL + i), 1);
        mbar_init(bar(B_O_FREE + i), 8);
        mbar_init(bar(B_STAGE + i), 8);
      }
      mbar_init(bar(B_DRAIN_R), 1);
    }
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(ctl.abort_addr), "r"(0u) : "memory");
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(sb + OFF_PUSHED), "r"(0u) : "memory");
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(sb + OFF_COMMITTED), "r"(0u) : "memory");
    fence_mbar_init();
  }
  // Producer epilogue warps 4-11: warp quarter q = warp % 4 reads TMEM lanes
  // 32q..32q+31 (state rows), column half h = (warp - 4) / 4. The state is
  // read here, before the first cluster barrier; only this CTA touches it.
  const int eq = warp & 3;
  const int eh = (warp - 4) >> 2;
  const int erow = eq * 32 + lane;
  float m[64];
  if (rank == 0 && warp >= 4) {
#pragma unroll
    for (int j = 0; j < 64; ++j)
      m[j] = p.state_in ? p.state_in[((size_t)bh * kD + erow) * kD + 64 * eh + j] : 0.f;
  }
  if (warp == 2) {
    tmem_alloc(sb + OFF_TMEM_PTR, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();
  const uint32_t tmem = ld_shared_u32(sb + OFF_TMEM_PTR);
  const uint64_t stream_pol = policy_evict_first();

  if (rank == 0) {
    // ============================================================ producer
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------- K/V loader
      int it = 0;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        for (int i = 0; i < nkv; ++i, ++it) {
          const int slot = it % NKV;
          if (!wait_bar(bar(B_KV_EMPTY + slot), ((it / NKV) & 1) ^ 1, ctl, kStLoad)) {
            ok = false;
            break;
          }
          const uint32_t st = sb + OFF_KV + slot * kStage;
          const uint32_t fb = bar(B_KV_FULL + slot);
          mbar_arrive_expect_tx(fb, kStage);
          const int y = i * kKvRows, z = bh * T + t;
          tma_load_3d_hint(st, &p.tm_k, fb, 0, y, z, stream_pol);
          tma_load_3d_hint(st + kBox64, &p.tm_k, fb, 64, y, z, stream_pol);
          tma_load_3d_hint(st + 2 * kBox64, &p.tm_v, fb, 0, y, z, stream_pol);
          tma_load_3d_hint(st + 3 * kBox64, &p.tm_v, fb, 64, y, z, stream_pol);
        }
      }
      for (int k = it - 1; k >= 0 && k >= it - NKV; --k)
        drain_bar(bar(B_KV_FULL + k % NKV), (k / NKV) & 1, ctl, kStDrain);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------- K^T [K V] issuer
      // A = K^T: M = 128 key dims in two 64-column atoms 8 KB apart; B = [K V]:
      // N = 256 in four atoms 8 KB apart; both MN-major views of the tiles.
      constexpr uint32_t idesc = idesc_bf16(128, 256, 1, 1);
      int it = 0;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int b = t & 1;
        if (!wait_bar(bar(B_ACC_FREE + b), ((t >> 1) & 1) ^ 1, ctl, kStMma)) break;
        for (int i = 0; i < nkv; ++i, ++it) {
          const int slot = it % NKV;
          if (!wait_bar(bar(B_KV_FULL + slot), (it / NKV) & 1, ctl, kStMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sb + OFF_KV + slot * kStage;
#pragma unroll
          for (int kk = 0; kk < kKvRows / 16; ++kk) {
            const uint64_t a = smem_desc(st + kk * 2048, kBox64, 1024, 2);
            const uint64_t bd = smem_desc(st + kk * 2048, kBox64, 1024, 2);
            mma_bf16(tmem + 256 * b, a, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(B_KV_EMPTY + slot));
        }
        if (ok) mma_commit(bar(B_ACC_FULL + b));
      }
      mma_commit(bar(B_DRAIN_P + 0));
      drain_bar(bar(B_DRAIN_P + 0), 0, ctl, kStDrain);
    } else if (warp == 2 && lane == 0) {
      // ---------------------------------------------- recurrence issuer: D += A'' M_{t-1}
      // A = A'' (K-major, two 64-column atoms 16 KB apart); B = M_{t-1}
      // (MN-major, value columns in two atoms 16 KB apart); 16 key rows per MMA.
      constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 1);
      for (int t = 0; t < T; ++t) {
        if (!wait_bar(bar(B_A_READY), t & 1, ctl, kStMma) ||
            !wait_bar(bar(B_M_READY), t & 1, ctl, kStMma))
          break;
        tc_fence_after();
        const uint32_t mb = sb + OFF_M + (uint32_t)(t & 1) * kMat;   // M_{t-1}
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = smem_desc(sb + OFF_A + (kk >> 2) * kAtom + (kk & 3) * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(mb + kk * 2048, kAtom, 1024, 2);
          mma_bf16(tmem + 256 * (t & 1) + 128, a, bd, idesc, 1u);
        }
        mma_commit(bar(B_CHAIN));
      }
      mma_commit(bar(B_DRAIN_P + 1));
      drain_bar(bar(B_DRAIN_P + 1), 0, ctl, kStDrain);
    } else if (warp == 3 && lane == 0) {
      // ---------------------------------------------- pusher: M_t into the reader's slot t % 2
      // M_t sits in buffer (t + 1) % 2 as that buffer's ((t + 1) / 2)-th write.
      for (int t = 0; t < T; ++t) {
        const int u = (t + 1) & 1;
        if (!wait_bar(bar(B_M_WRITTEN + u), ((t + 1) >> 1) & 1, ctl, kStPush)) break;
        if (t >= 2 && !wait_bar(bar(B_MR_FREE + (t & 1)), ((t - 2) >> 1) & 1, ctl, kStPush)) break;
        const uint32_t rbar = mapa(bar(B_MR_FULL + (t & 1)), 1);
        mbar_arrive_expect_tx_cluster(rbar, kMat);
        bulk_copy_to_cluster(mapa(sb + OFF_MR + (uint32_t)(t & 1) * kMat, 1),
                             sb + OFF_M + (uint32_t)u * kMat, kMat, rbar);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sb + OFF_PUSHED), "r"((uint32_t)(t + 1))
                     : "memory");
      }
    } else if (warp >= 4) {
      // ---------------------------------------------- A'' and the state update
      const float* gam = p.gamma + (size_t)bh * T;
      const float* bet = p.beta + (size_t)bh * T;
      auto store_m = [&](int buf) {
        const uint32_t base = sb + OFF_M + (uint32_t)buf * kMat + (uint32_t)eh * kAtom;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(base + swz128((uint32_t)erow, (uint32_t)c),
                       make_uint4(pack_bf16x2(m[8 * c], m[8 * c + 1]), pack_bf16x2(m[8 * c + 2], m[8 * c + 3]),
                                  pack_bf16x2(m[8 * c + 4], m[8 * c + 5]),
                                  pack_bf16x2(m[8 * c + 6], m[8 * c + 7])));
      };
      store_m(0);   // M_{-1} = M_0, the operand of frame 0
      fence_proxy_async_cta();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(B_M_READY));
        mbar_arrive(bar(B_M_WRITTEN + 0));
      }
      bool ok = true;
      int t = 0;
      for (; t < T; ++t) {
        const int b = t & 1;
        const float g = __ldg(gam + t);
        const float be = __ldg(bet + t);
        if (!warp_wait(bar(B_ACC_FULL + b), (t >> 1) & 1, ctl, kStEpi)) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          uint32_t v[64];
          tmem_ld64(tmem + 256 * b + 64 * eh + ((uint32_t)(eq * 32) << 16), v);
          const float coef = -g * p.s * p.delta;   // A'' = -gamma s K^T K
          const uint32_t base = sb + OFF_A + (uint32_t)eh * kAtom;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = coef * __uint_as_float(v[8 * c + e]);
            st_shared_v4(base + swz128((uint32_t)erow, (uint32_t)c),
                         make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                    pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7])));
          }
        }
        fence_proxy_async_cta();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_A_READY));
        uint32_t cd = 0;
        if (lane == 0) {
          cd = wait_bar(bar(B_CHAIN), t & 1, ctl, kStEpi) ? 1u : 0u;
        }
        cd = __shfl_sync(0xffffffffu, cd, 0);
        if (!cd) {
          ok = false;
          break;
        }
        mbar_test(bar(B_CHAIN), t & 1);   // acquire for every lane
        tc_fence_after();
        {
          uint32_t d[64];
          tmem_ld64(tmem + 256 * b + 128 + 64 * eh + ((uint32_t)(eq * 32) << 16), d);
          const float bs = be * p.s;
#pragma unroll
          for (int j = 0; j < 64; ++j) m[j] = fmaf(g, m[j], bs * __uint_as_float(d[j]));
        }
        tc_fence_before();
        // M_t replaces M_{t-2} in buffer (t + 1) % 2: its copy to the reader
        // must be done, which the reader's release of frame t - 2 tells.
        if (t >= 2 && !warp_wait(bar(B_MR_FREE + (t & 1)), ((t - 2) >> 1) & 1, ctl, kStEpi)) {
          ok = false;
          break;
        }
        store_m((t + 1) & 1);
        fence_proxy_async_cta();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_M_READY));
          mbar_arrive(bar(B_M_WRITTEN + ((t + 1) & 1)));
          mbar_arrive(bar(B_ACC_FREE + b));
        }
      }
      if (ok && p.state_out) {
#pragma unroll
        for (int j = 0; j < 64; ++j) p.state_out[((size_t)bh * kD + erow) * kD + 64 * eh + j] = m[j];
      }
      // The reader's releases of the last frames arrive here: wait for them all
      // before this CTA may leave (its shared memory is their target).
      if (ok && warp == 4 && lane == 0) {
        for (int f = (T >= 2 ? T - 2 : 0); f < T; ++f)
          wait_bar(bar(B_MR_FREE + (f & 1)), (f >> 1) & 1, ctl, kStEpi);
      }
    }
  } else {
    // ============================================================ reader
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------- Q loader
      int it = 0;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        for (int i = 0; i < nq; ++i, ++it) {
          const int slot = it % NQ;
          if (!wait_bar(bar(B_Q_EMPTY + slot), ((it / NQ) & 1) ^ 1, ctl, kStLoad)) {
            ok = false;
            break;
          }
          const uint32_t qt = sb + OFF_Q + slot * kQTile;
          const uint32_t fb = bar(B_Q_FULL + slot);
          mbar_arrive_expect_tx(fb, kQTile);
          tma_load_3d_hint(qt, &p.tm_q, fb, 0, i * kQRows, bh * T + t, stream_pol);
          tma_load_3d_hint(qt + kAtom, &p.tm_q, fb, 64, i * kQRows, bh * T + t, stream_pol);
        }
      }
      for (int k = it - 1; k >= 0 && k >= it - NQ; --k)
        drain_bar(bar(B_Q_FULL + k % NQ), (k / NQ) & 1, ctl, kStDrain);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------- read-out issuer: O = Q M_t
      constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 1);   // Q K-major, M MN-major
      int qit = 0, on = 0;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t & 1;
        if (!wait_bar(bar(B_MR_FULL + s), (t >> 1) & 1, ctl, kStMma)) break;
        const uint32_t mb = sb + OFF_MR + (uint32_t)s * kMat;
        for (int i = 0; i < nq; ++i, ++qit, ++on) {
          const int slot = qit % NQ;
          const int ob = on & 1;
          if (!wait_bar(bar(B_Q_FULL + slot), (qit / NQ) & 1, ctl, kStMma) ||
              !wait_bar(bar(B_O_FREE + ob), ((on >> 1) & 1) ^ 1, ctl, kStMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qt = sb + OFF_Q + slot * kQTile;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t a = smem_desc(qt + (kk >> 2) * kAtom + (kk & 3) * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(mb + kk * 2048, kAtom, 1024, 2);
            mma_bf16(tmem + 128 * ob, a, bd, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_O_FULL + ob));
        }
        if (ok) {
          // slot s of M is free once these MMAs complete: tell the producer
          mma_commit_multicast(bar(B_MR_FREE + s), (uint16_t)1u);
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(sb + OFF_COMMITTED), "r"((uint32_t)(t + 1))
                       : "memory");
        }
      }
      mma_commit(bar(B_DRAIN_R));
      drain_bar(bar(B_DRAIN_R), 0, ctl, kStDrain);
    } else if (warp >= 4) {
      // ---------------------------------------------- output tiles: TMEM -> bf16 -> TMA store
      // Warp quarter q holds tile rows 32q..32q+31, column half h; the tile is
      // staged in its own Q slot (the MMA that read it is done) and stored as
      // two 64-column boxes by one leader thread.
      const bool leader = warp == 4 && lane == 0;
      int n = 0;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        for (int i = 0; i < nq; ++i, ++n) {
          const int ob = n & 1;
          if (!warp_wait(bar(B_O_FULL + ob), (n >> 1) & 1, ctl, kStOut)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t v[64];
          tmem_ld64(tmem + 128 * ob + 64 * eh + ((uint32_t)(eq * 32) << 16), v);
          tc_fence_before();
          const int slot = n % NQ;
          const uint32_t base = sb + OFF_Q + slot * kQTile + (uint32_t)eh * kAtom;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(base + swz128((uint32_t)erow, (uint32_t)c),
                         make_uint4(pack_bf16x2(__uint_as_float(v[8 * c]), __uint_as_float(v[8 * c + 1])),
                                    pack_bf16x2(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3])),
                                    pack_bf16x2(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5])),
                                    pack_bf16x2(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]))));
          fence_proxy_async_cta();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(bar(B_STAGE + (n & 1)));
            mbar_arrive(bar(B_O_FREE + ob));
          }
          uint32_t stored = 1;
          if (leader) {
            stored = wait_bar(bar(B_STAGE + (n & 1)), (n >> 1) & 1, ctl, kStOut) ? 1u : 0u;
            if (stored) {
              const uint32_t tile = sb + OFF_Q + slot * kQTile;
              tma_store_3d_hint(&p.tm_o, tile, 0, i * kQRows, bh * T + t, stream_pol);
              tma_store_3d_hint(&p.tm_o, tile + kAtom, 64, i * kQRows, bh * T + t, stream_pol);
              bulk_commit();
              bulk_wait_read0();
              mbar_arrive(bar(B_Q_EMPTY + slot));
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
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (aborted(ctl)) {
    // Same verdict in both CTAs. What the peer issued towards this CTA before
    // the barrier above must land before either leaves: pushed copies of M
    // (reader) and release commits (producer).
    // Phases of a barrier complete in order, and a parity wait may only name
    // the current or the previous phase: wait for the last frame of each slot.
    if (threadIdx.x == 0) {
      const uint32_t n = rank == 1 ? ld_cluster_u32(mapa(sb + OFF_PUSHED, 0))
                                   : ld_cluster_u32(mapa(sb + OFF_COMMITTED, 1));
      const int base = rank == 1 ? B_MR_FULL : B_MR_FREE;
      for (uint32_t f = n >= 2 ? n - 2 : 0; f < n; ++f)
        drain_bar(bar(base + (f & 1)), (f >> 1) & 1, ctl, kStDrain);
    }
    __syncthreads();
    cluster_sync();
  }
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// ------------------------------------------------------------------ host side

cudaError_t prepare() {
  static std::atomic<bool> done[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(reinterpret_cast<const void*>(&gdn_tc128_kernel),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

}  // namespace

int tc128_ctas_per_head(int B, int H, int T, int S, int D) {
  if (D != kD) return 0;
  const long long heads = (long long)B * H;
  if (heads * (long long)T >= (1ll << 31) || heads * 2 > (1ll << 31) - 1) return 0;
  (void)S;
  return 2;
}

cudaError_t launch_tc128_bf16(const Problem& pr) {
  if (pr.D != kD) return cudaErrorInvalidValue;
  cudaError_t e = prepare();
  if (e != cudaSuccess) return e;
  Tc128Params p;
  const long long frames = (long long)pr.B * pr.H * pr.T;
  if (!make_frame_map(&p.tm_q, pr.q, kD, pr.S, frames, kQRows) ||
      !make_frame_map(&p.tm_k, pr.k, kD, pr.S, frames, kKvRows) ||
      !make_frame_map(&p.tm_v, pr.v, kD, pr.S, frames, kKvRows) ||
      !make_frame_map(&p.tm_o, pr.out, kD, pr.S, frames, kQRows))
    return cudaErrorInvalidValue;
  p.status = status_word();
  if (!p.status) return cudaErrorInvalidDevice;
  p.gamma = pr.gamma;
  p.beta = pr.beta;
  p.state_in = pr.state_in;
  p.state_out = pr.state_out;
  p.timeout_ns = wait_budget_ns();
  p.T = pr.T;
  p.S = pr.S;
  p.s = pr.key_scale;
  p.delta = pr.delta ? 1.f : 0.f;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(pr.B * pr.H * 2), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cfg.stream = pr.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gdn_tc128_kernel, p);
}

}  // namespace gdn
