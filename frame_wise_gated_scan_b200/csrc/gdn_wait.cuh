// Bounded waits and the abort protocol shared by the cluster kernels.
//
// Every wait on an mbarrier, a peer or a flag gives up after `timeout_ns`
// (1 s in the shipped library; a GDN_DEBUG build takes it from the
// environment so that tests can make waits run out). Drains of copies and
// MMAs already in flight always keep the full bound, kDrainNs. A wait that runs out records its role in the
// device status word (read by gdn_device_status) and raises an abort flag in
// the shared memory of every CTA of the cluster; the other roles see the flag
// and stop waiting, so every CTA reaches the same exit path, drains what is
// still in flight, and returns.
#pragma once

#include <stdint.h>

#include "sm100_ptx.h"

namespace gdn {
namespace wait {

using namespace ptx;

constexpr unsigned long long kDrainNs = 1000ull * 1000ull * 1000ull;   // 1 s

struct Ctl {
  uint32_t abort_addr;            // local shared address of the abort flag
  unsigned int* status;           // device status word
  unsigned long long timeout_ns;  // bound of every wait
  int P;                          // CTAs in the cluster
};

__device__ __forceinline__ bool aborted(const Ctl& c) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(c.abort_addr) : "memory");
  return v != 0;
}

static __device__ __noinline__ void raise_abort(const Ctl& c, uint32_t code) {
  atomicOr(c.status, code);
  for (int q = 0; q < c.P; ++q)
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(mapa(c.abort_addr, q)), "r"(1u) : "memory");
  fence_acq_rel_cluster();
}

// Bounded wait on a local mbarrier phase; false if aborting or out of time.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& c, uint32_t code) {
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

// Warp-uniform bounded wait: lane 0 waits, the verdict is broadcast, and on
// success every lane observes the completed phase itself (acquire).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Ctl& c, uint32_t code) {
  uint32_t ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, c, code) ? 1u : 0u;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) {
    for (int i = 0; i < 1024 && !mbar_try(bar, parity); ++i) {
    }
  }
  return ok != 0;
}

// Bounded wait that ignores the abort flag (draining copies and MMAs in
// flight); its bound is kDrainNs whatever the role-wait budget.
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity, const Ctl& c,
                                          uint32_t code) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainNs) {
      atomicOr(c.status, code);
      return;
    }
  }
}

}  // namespace wait
}  // namespace gdn
