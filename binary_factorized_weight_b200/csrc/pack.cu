// Sign packing: a +-1 matrix (int8, fp16 or fp32 entries) -> the packed layout.
//
// The pages store A and B as matrices of +-1 elements ("Addition is almost all
// you need", sciencestack.ai Figure 1; gist.science section 2.1).  One warp
// builds one 32-bit word: word p of a 256-column block holds the column pair
// (16g + 2p, 16g + 2p + 1) of every group g at bits (g, g+16), so lane b reads
// column 16(b%16) + 2p + b/16 of the block and a warp ballot of "value < 0" is
// the word.  Rows are padded to whole blocks with zero bits.
// Not a hot path (weights are packed once).
#include <algorithm>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace dbf {
namespace {

__device__ __forceinline__ bool is_negative(int8_t v) { return v < 0; }
__device__ __forceinline__ bool is_negative(__half v) { return __half2float(v) < 0.f; }  // -0.0, NaN -> false
__device__ __forceinline__ bool is_negative(float v) { return v < 0.f; }

template <typename T>
__global__ void dbf_pack_kernel(const T* __restrict__ src, int64_t rows, int64_t cols, int64_t wpr,
                                uint32_t* __restrict__ packed) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int lane_col = 16 * (lane & 15) + (lane >> 4);  // column (within its block, for pair 0) of bit `lane`
  const int64_t total = rows * wpr;
  for (int64_t word = warp_id; word < total; word += nwarps) {
    const int64_t r = word / wpr;
    const int64_t wi = word - r * wpr;
    const int64_t col = (wi >> 3) * 256 + 2 * (wi & 7) + lane_col;
    const bool neg = col < cols && is_negative(src[r * cols + col]);
    const uint32_t bits = __ballot_sync(0xffffffffu, neg);
    if (lane == 0) packed[word] = bits;
  }
}

}  // namespace

dbf_status launch_pack(const void* src, dbf_dtype src_t, int64_t rows, int64_t cols, uint32_t* packed,
                       const DeviceInfo& dev, cudaStream_t stream) {
  const int64_t wpr = words_per_row(cols);
  const int64_t total = rows * wpr;
  const int threads = 256;
  const int64_t want = (total + (threads / 32) - 1) / (threads / 32);
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(want, static_cast<int64_t>(dev.num_sms) * 16));
  switch (src_t) {
    case DBF_I8:
      return launch_plain(dbf_pack_kernel<int8_t>, dim3(blocks), dim3(threads), 0, stream,
                          static_cast<const int8_t*>(src), rows, cols, wpr, packed);
    case DBF_F16:
      return launch_plain(dbf_pack_kernel<__half>, dim3(blocks), dim3(threads), 0, stream,
                          static_cast<const __half*>(src), rows, cols, wpr, packed);
    case DBF_F32:
      return launch_plain(dbf_pack_kernel<float>, dim3(blocks), dim3(threads), 0, stream,
                          static_cast<const float*>(src), rows, cols, wpr, packed);
    default:
      return DBF_ERR_INVALID_ARG;
  }
}

}  // namespace dbf
