// status.cuh -- the device status word that kernels write instead of trapping.
#pragma once
#include "himuon.h"

namespace himuon {

constexpr int HIMUON_ERR_TIMEOUT_DEV = HIMUON_ERR_TIMEOUT;

// Record the first error only; later ones keep the first code.
__device__ __forceinline__ void set_status(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace himuon
