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

// Stages 2-7 of mask packing (tiled count sort -> row_offsets and schedule,
// the head-mix check of that schedule and, when it mixes many heads, the
// head-major order; then the kept-block lists), for any producer that has
// written every row's
// CRM words and count.  `scratch` holds pack_scratch_bytes(rows, nb_k) bytes,
// 16-byte aligned.  Defined in bsa_pack.cu.
size_t pack_scratch_bytes(int64_t rows, int nb_k);
bsa_status pack_finish(const uint32_t* bits, const int32_t* counts, int rows, int nb_q,
                       int nb_k, int32_t* row_offsets, int32_t* col_idx, int32_t* schedule,
                       void* scratch, cudaStream_t s);
// Largest nb_k the packing stages accept (BSA_ERR_UNSUPPORTED beyond).
constexpr int kPackMaxNbK = 49151;

// The predictor's device-side error word (BSA_ERR_TIMEOUT after a wait of its
// score kernel ran out, else 0), read and cleared; -1 if the copy failed.
// Defined in bsa_predict.cu.
int take_predict_device_error();

}  // namespace bsa
