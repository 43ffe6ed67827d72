// Host-side helpers shared by the kernels: TMA tensor maps of the [frames][S][D]
// bf16 arrays, and the device status word that bounded device waits report to.
#include <cuda.h>
#include <cuda_runtime.h>

#include <stdlib.h>

#include <atomic>
#include <mutex>

#include "gdn_internal.h"

namespace gdn {

// Bits are set by a kernel whose bounded wait ran out (or that was launched
// with the wrong shape); read and cleared by gdn_device_status().
__device__ unsigned int g_status = 0;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once per process.
EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

}  // namespace

bool make_frame_map(CUtensorMap* m, const void* base, int D, int S, long long frames,
                    int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)frames};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 1u};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

unsigned int* status_word() {
  static std::atomic<unsigned int*> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  unsigned int* a = cache[dev].load(std::memory_order_acquire);
  if (!a) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status) != cudaSuccess) return nullptr;
    a = static_cast<unsigned int*>(ptr);
    cache[dev].store(a, std::memory_order_release);
  }
  return a;
}

cudaError_t read_status(unsigned int* status) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(status, g_status, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_status, &zero, sizeof(unsigned int));
}

unsigned long long wait_budget_ns() {
#ifdef GDN_DEBUG
  if (const char* e = getenv("GDN_DEBUG_WAIT_NS")) return strtoull(e, nullptr, 10);
#endif
  return 1000ull * 1000ull * 1000ull;
}

}  // namespace gdn
