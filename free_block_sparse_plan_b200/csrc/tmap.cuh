// Host side of the TMA tensor maps: the driver's cuTensorMapEncodeTiled, looked up once
// through the runtime (no link against libcuda).  Returns null when the driver lacks it.
#pragma once
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace spr {

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace spr
