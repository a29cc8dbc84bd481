// dbf_forward_noalloc: the layer forward for callers that cannot allocate.
//
// dbf_forward needs a caller-provided workspace (a status word and the middle
// activations V).  Some callers have no way to provide one: a plugin running
// inside a host application that owns every byte of device memory and gives
// its extensions no allocator, or a latency-critical thread that must not call
// cudaMalloc because it can block and synchronise the whole device.  This
// entry point serves them by using a fixed buffer that lives in the library
// itself: a file-scope static __device__ array of kNoAllocScratchBytes, which
// every GPU that loads the library keeps until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it
// only names a shadow symbol), so the first call on each device, with that
// device current, looks the address up with cudaGetSymbolAddress and caches
// it; that first call should therefore come before any stream capture.  A
// lookup that fails is not cached: the error it left is cleared and the next
// call tries again.  The call itself allocates nothing: it clears the status
// word with cudaMemsetAsync and hands the buffer to the forward as its
// workspace.  dbf_noalloc_status reads that status word back.  Every call
// shares the one buffer, so calls whose work overlaps on the GPU (different
// streams, or different host threads) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "dbf_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t{2} << 20;  // 2 MiB: status block + V (batch x k fp16)
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the buffer on the current device `device` (cached after
// the first successful lookup).
void* scratch_address(int device, dbf_status* st) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[device] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();  // leave no sticky error for a later launch check
      *st = DBF_ERR_CUDA;
      return nullptr;
    }
    addr[device] = p;
  }
  *st = DBF_OK;
  return addr[device];
}

}  // namespace

extern "C" {

dbf_status dbf_forward_noalloc(const uint16_t* x, const uint32_t* packedA, const uint32_t* packedB,
                               const uint16_t* a, const uint16_t* m, const uint16_t* b, int64_t n, int64_t k,
                               int64_t m_in, int64_t batch, void* y, dbf_dtype y_t, uint32_t flags,
                               struct CUstream_st* stream) {
  dbf_status st = dbf::validate_forward_args(x, packedA, packedB, a, m, b, n, k, m_in, batch, y, y_t, flags);
  if (st != DBF_OK) return st;
  // the buffer holds the status block and V; the optional areas after them
  // (single-launch decode partials, stream-K slots) are used where they fit
  if (dbf::forward_workspace_min_bytes(k, batch) > kNoAllocScratchBytes) return DBF_ERR_WORKSPACE;
  dbf::DeviceInfo dev;
  st = dbf::current_device(&dev);
  if (st != DBF_OK) return st;
  if (dev.device >= kMaxDevices) return DBF_ERR_DEVICE;
  void* ws = scratch_address(dev.device, &st);
  if (st != DBF_OK) return st;
  // The status word must start at zero; the rest of the buffer is overwritten.
  if (cudaMemsetAsync(ws, 0, sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DBF_ERR_CUDA;
  return dbf_forward(x, packedA, packedB, a, m, b, n, k, m_in, batch, y, y_t, ws, kNoAllocScratchBytes, flags,
                     stream);
}

dbf_status dbf_noalloc_status(struct CUstream_st* stream, int32_t* device_status) {
  if (!device_status) return DBF_ERR_INVALID_ARG;
  dbf::DeviceInfo dev;
  dbf_status st = dbf::current_device(&dev);
  if (st != DBF_OK) return st;
  if (dev.device >= kMaxDevices) return DBF_ERR_DEVICE;
  void* ws = scratch_address(dev.device, &st);
  if (st != DBF_OK) return st;
  return dbf_workspace_status(ws, stream, device_status);
}

}  // extern "C"
