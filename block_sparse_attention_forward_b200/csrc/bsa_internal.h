// Internal helpers shared by the libbsa translation units (host side).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa.h"

namespace bsa {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

inline bsa_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BSA_OK : BSA_ERR_LAUNCH;
}

inline int num_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return sms;
}

}  // namespace bsa
