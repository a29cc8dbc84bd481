// Transpose of a packed sign matrix: the packing of S^T from the packing of S.
//
// The transpose product dx = dy W of the factorised W = (a (.) A (.) m^T)(B (.) b^T)
// ("Addition is almost all you need", gist.science technical summary, section
// 2.1) is itself a factorised product, with B^T and A^T in the places of A and
// B.  Both are sign matrices again, so the forward kernels run it unchanged once
// A^T and B^T are packed row-major over their own reduction dimension.
//
// One warp builds one output word, as the pack kernel does: output row r' is
// input column r', and bit `lane` of output word wi is the sign of output column
// c' = (wi/8)*256 + 2*(wi%8) + 16*(lane%16) + lane/16, i.e. of input element
// (row c', column r').  Each lane reads the one input word that holds it; a
// ballot of the bits is the output word.  Padding columns (c' >= rows) are zero.
// Not a hot path (weights are transposed once).
#include <algorithm>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace dbf {
namespace {

__global__ void dbf_transpose_signs_kernel(const uint32_t* __restrict__ in, int64_t rows, int64_t cols, int64_t wpr_in,
                                           int64_t wpr_out, uint32_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int lane_col = 16 * (lane & 15) + (lane >> 4);
  const int64_t total = cols * wpr_out;  // output: cols rows of wpr_out words
  for (int64_t word = warp_id; word < total; word += nwarps) {
    const int64_t r_out = word / wpr_out;  // = input column
    const int64_t wi = word - r_out * wpr_out;
    const int64_t c_out = (wi >> 3) * 256 + 2 * (wi & 7) + lane_col;  // = input row
    // input element (c_out, r_out): block r_out/256, word (e%16)/2, bit e/16 + 16(e%2), e = r_out % 256
    const int e = static_cast<int>(r_out & 255);
    const int64_t in_word = (r_out >> 8) * 8 + packed_word_in_block(e);
    const int in_bit = packed_bit_in_block(e);
    bool neg = false;
    if (c_out < rows) neg = (in[c_out * wpr_in + in_word] >> in_bit) & 1u;
    const uint32_t bits = __ballot_sync(0xffffffffu, neg);
    if (lane == 0) out[word] = bits;
  }
}

}  // namespace

dbf_status launch_transpose_signs(const uint32_t* packed, int64_t rows, int64_t cols, uint32_t* out,
                                  const DeviceInfo& dev, cudaStream_t stream) {
  const int64_t wpr_in = words_per_row(cols);
  const int64_t wpr_out = words_per_row(rows);
  const int64_t total = cols * wpr_out;
  const int threads = 256;
  const int64_t want = (total + (threads / 32) - 1) / (threads / 32);
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(want, static_cast<int64_t>(dev.num_sms) * 16));
  return launch_plain(dbf_transpose_signs_kernel, dim3(blocks), dim3(threads), 0, stream, packed, rows, cols, wpr_in,
                      wpr_out, out);
}

}  // namespace dbf
