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
// it; that first call should therefore come before any stream capture.  The
// call itself allocates nothing: it clears the status word with
// cudaMemsetAsync and hands the buffer to dbf_forward as its workspace.
// Every call shares the one buffer, so calls whose work overlaps on the GPU
// (different streams, or different host threads) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "dbf_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t{2} << 20;  // 2 MiB: status block + V (batch x k fp16)
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* scratch_address(int device, dbf_status* st) {
  static void* addr[kMaxDevices] = {};
  static std::once_flag once[kMaxDevices];
  static cudaError_t err[kMaxDevices] = {};
  std::call_once(once[device], [device] {
    void* p = nullptr;
    err[device] = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // device `device` is current here
    addr[device] = p;
  });
  if (err[device] != cudaSuccess || addr[device] == nullptr) {
    *st = DBF_ERR_CUDA;
    return nullptr;
  }
  *st = DBF_OK;
  return addr[device];
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The synchronous argument checks dbf_forward makes, run before this entry
// point enqueues its status-word clear, so that a rejected call enqueues nothing.
dbf_status precheck(const uint16_t* x, const uint32_t* packedA, const uint32_t* packedB, const uint16_t* a,
                    const uint16_t* m, const uint16_t* b, int64_t n, int64_t k, int64_t m_in, int64_t batch,
                    const void* y, dbf_dtype y_t, uint32_t flags) {
  if (!x || !packedA || !packedB || !a || !m || !b || !y) return DBF_ERR_INVALID_ARG;
  if (n < 1 || k < 1 || m_in < 1 || batch < 1) return DBF_ERR_INVALID_ARG;
  if (k % 64 != 0 || m_in % 64 != 0 || k > (int64_t{1} << 20) || m_in > (int64_t{1} << 20) ||
      n > (int64_t{1} << 24) || batch > (int64_t{1} << 24))
    return DBF_ERR_UNSUPPORTED_SHAPE;
  if (y_t != DBF_F16 && y_t != DBF_F32) return DBF_ERR_INVALID_ARG;
  const uint32_t known = DBF_FWD_WEIGHTS_STATIC | DBF_FWD_FORCE_DECODE | DBF_FWD_FORCE_PREFILL |
                         DBF_FWD_DECODE_SHIFT_EXPAND;
  if ((flags & ~known) != 0 || ((flags & DBF_FWD_FORCE_DECODE) && (flags & DBF_FWD_FORCE_PREFILL)))
    return DBF_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packedA) || !aligned16(packedB) || !aligned16(a) || !aligned16(m) ||
      !aligned16(b) || !aligned16(y))
    return DBF_ERR_MISALIGNED;
  return DBF_OK;
}

}  // namespace

extern "C" {

dbf_status dbf_forward_noalloc(const uint16_t* x, const uint32_t* packedA, const uint32_t* packedB,
                               const uint16_t* a, const uint16_t* m, const uint16_t* b, int64_t n, int64_t k,
                               int64_t m_in, int64_t batch, void* y, dbf_dtype y_t, uint32_t flags,
                               struct CUstream_st* stream) {
  dbf_status st = precheck(x, packedA, packedB, a, m, b, n, k, m_in, batch, y, y_t, flags);
  if (st != DBF_OK) return st;
  if (dbf_forward_workspace_bytes(n, k, m_in, batch) > kNoAllocScratchBytes) return DBF_ERR_WORKSPACE;
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

}  // extern "C"
