// static_scratch.cu -- himuon_ns_static: the staged NS path with its scratch
// in a file-scope device array instead of a caller workspace.
//
// For callers that cannot allocate device memory.  The array is part of the
// library's device image, so every GPU that loads the library holds
// HIMUON_STATIC_SCRATCH_BYTES of it until the process exits.  Host code must
// never hand the symbol itself to a kernel (on the host it names a host-side
// stand-in, not device memory); the device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
#include <cuda_runtime.h>

#include <atomic>

#include "himuon.h"

namespace himuon {

int run_staged_into(int op, const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                    const himuon_ns_params *p, void *scratch, size_t scratch_bytes, cudaStream_t stream);

namespace {

__device__ __align__(256) unsigned char g_static_scratch[HIMUON_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
// Looked-up addresses, one per device.  Host threads may race on a device's
// first call: each then looks the address up itself (the same value) and the
// atomic store keeps the slot well defined.
std::atomic<void *> g_scratch_addr[kMaxDevices];

// Device address of g_static_scratch on the current device (set-up on first use).
int scratch_address(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return HIMUON_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return HIMUON_ERR_NO_DEVICE;
  void *ptr = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!ptr) {
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess || !ptr) {
      cudaGetLastError();
      return HIMUON_ERR_CUDA;
    }
    g_scratch_addr[dev].store(ptr, std::memory_order_release);
  }
  *out = ptr;
  return HIMUON_OK;
}

}  // namespace
}  // namespace himuon

extern "C" int himuon_ns_static(const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                                const himuon_ns_params *p, void *stream) {
  if (!in || !out || !p) return HIMUON_ERR_INVALID;
  if (p->tiles) return HIMUON_ERR_UNSUPPORTED;   // one tile size per call here
  void *scratch = nullptr;
  const int rc = himuon::scratch_address(&scratch);
  if (rc != HIMUON_OK) return rc;
  const int op = p->tile <= 0 ? HIMUON_OP_NS_FULL : HIMUON_OP_NS_TILED;
  return himuon::run_staged_into(op, in, out, n, splits, p, scratch, HIMUON_STATIC_SCRATCH_BYTES,
                                 static_cast<cudaStream_t>(stream));
}
