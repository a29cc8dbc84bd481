// Dense reconstruction W = (a (.) A (.) m^T)(B (.) b^T) ("Addition is almost
// all you need", gist.science technical summary, section 2.1, factorisation):
//
//   W[i][j] = a_i * b_j * sum_l A[i][l] * mid_l * B[l][j]
//
// Used to check a factorisation against the dense weight it stands for; not a
// hot path.  A 64x64 tile of W per CTA, 256 threads with 4x4 outputs each; the
// middle dimension is walked one packed block (256 values of l) at a time with
// A's block words for the tile's 64 rows and B's block words for 256 rows l
// (the columns j0..j0+63 of those rows) staged in shared memory.  fp32
// accumulation of +-mid_l.
#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace dbf {
namespace {

constexpr int kTile = 64;

template <bool OUT_F32>
__global__ void __launch_bounds__(256) dbf_reconstruct_kernel(const uint32_t* __restrict__ packedA,
                                                              const uint32_t* __restrict__ packedB,
                                                              const __half* __restrict__ a,
                                                              const __half* __restrict__ mid,
                                                              const __half* __restrict__ b, int n, int k, int m_in,
                                                              int64_t wprA, int64_t wprB, void* W) {
  __shared__ uint32_t a_words[kTile][8];   // rows i0.., the 8 words of the l-block
  __shared__ uint32_t b_words[256][9];     // rows l of the block, B's 8 words of block j0/256 (+1 pad)
  __shared__ float mid_s[256];

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int i0 = blockIdx.y * kTile, j0 = blockIdx.x * kTile;
  const int64_t jblock_word = static_cast<int64_t>(j0 / 256) * 8;
  float acc[4][4] = {};

  for (int lb = 0; lb < k; lb += 256) {
    for (int t = tid; t < kTile * 8; t += 256) {
      const int i = i0 + (t >> 3);
      a_words[t >> 3][t & 7] = i < n ? packedA[static_cast<int64_t>(i) * wprA + lb / 32 + (t & 7)] : 0u;
    }
    for (int t = tid; t < 256 * 8; t += 256) {
      const int l = lb + (t >> 3);
      b_words[t >> 3][t & 7] = l < k ? packedB[static_cast<int64_t>(l) * wprB + jblock_word + (t & 7)] : 0u;
    }
    mid_s[tid] = (lb + tid < k) ? __half2float(mid[lb + tid]) : 0.f;
    __syncthreads();
    const int lmax = min(256, k - lb);
    for (int e = 0; e < lmax; ++e) {
      const int aw = packed_word_in_block(e), abit = packed_bit_in_block(e);
      const float m = mid_s[e];
      float sa[4], sb[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) sa[r] = ((a_words[ty * 4 + r][aw] >> abit) & 1u) ? -m : m;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int jc = (j0 + tx * 4 + q) & 255;  // column of B within its block
        sb[q] = ((b_words[e][packed_word_in_block(jc)] >> packed_bit_in_block(jc)) & 1u) ? -1.f : 1.f;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r][q] = fmaf(sa[r], sb[q], acc[r][q]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + ty * 4 + r;
    if (i >= n) continue;
    const float ai = __half2float(a[i]);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + tx * 4 + q;
      if (j >= m_in) continue;
      const float v = (ai * acc[r][q]) * __half2float(b[j]);
      if constexpr (OUT_F32) {
        static_cast<float*>(W)[static_cast<int64_t>(i) * m_in + j] = v;
      } else {
        static_cast<__half*>(W)[static_cast<int64_t>(i) * m_in + j] = __float2half_rn(v);
      }
    }
  }
}

}  // namespace

dbf_status launch_reconstruct(const uint32_t* packedA, const uint32_t* packedB, const __half* a, const __half* mid,
                              const __half* b, int64_t n, int64_t k, int64_t m_in, void* W, bool out_f32,
                              const DeviceInfo& dev, cudaStream_t stream) {
  (void)dev;
  const dim3 grid(static_cast<unsigned>((m_in + kTile - 1) / kTile), static_cast<unsigned>((n + kTile - 1) / kTile));
  if (grid.y > 65535u) return DBF_ERR_UNSUPPORTED_SHAPE;
  const int64_t wprA = words_per_row(k), wprB = words_per_row(m_in);
  auto kernel = out_f32 ? dbf_reconstruct_kernel<true> : dbf_reconstruct_kernel<false>;
  return launch_plain(kernel, grid, dim3(256), 0, stream, packedA, packedB, a, mid, b, static_cast<int>(n),
                      static_cast<int>(k), static_cast<int>(m_in), wprA, wprB, W);
}

}  // namespace dbf
