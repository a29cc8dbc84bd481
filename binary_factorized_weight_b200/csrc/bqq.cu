// Binary Quadratic Quantization (BQQ) forward on the DBF kernels.
//
// The sciencestack.ai page of "Binary Quadratic Quantization: Beyond
// First-Order Quantization for Real-Valued Matrix Compression" (TL;DR) writes
// a compressed matrix as
//     W = sum_{i<p} (r_i Y_i Z_i + s_i Y_i 1_Z + t_i 1_Y Z_i) + u 1
// with binary Y_i (n x k), Z_i (k x m_in), read here as {0, 1} matrices.  With
// the library's sign convention (a set bit is -1) a packed bit IS the binary
// entry: Y = (1 - S_Y) / 2 for the sign matrix S_Y of the packed bits, so
//     Y_i Z_i = (S_Yi S_Zi - S_Yi 1 - 1 S_Zi + k 1) / 4
// and, with S_Y = [S_Y0 .. S_Yp-1] (n x pk) and S_Z = [S_Z0; ..; S_Zp-1]
// (pk x m_in),
//     W x = S_Y diag(mid) S_Z x + c (1^T x) + 1 (d^T x),
//     mid = r_i / 4 on the k middle rows of term i,
//     c   = sum_i (s_i + r_i / 2) rowsum(Y_i)                  (n entries),
//     d   = sum_i (t_i + r_i / 2) colsum(Z_i) + u - k sum_i r_i / 4   (m_in).
// The first term is a DBF layer (a = b = 1) and runs on dbf_forward's
// kernels; c and d depend on the weights only and are computed once by
// dbf_bqq_prepare; the forward adds the rank-two correction in one more pass.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace dbf {
namespace {

constexpr int kThreads = 256;

size_t r256(size_t v) { return (v + 255) / 256 * 256; }

struct PrepLayout {
  size_t mid, ones, c, d, total;
};

PrepLayout prep_layout(int64_t n, int64_t k, int64_t p, int64_t m_in) {
  PrepLayout L;
  L.mid = 0;
  L.ones = r256(static_cast<size_t>(p * k) * 2);
  L.c = L.ones + r256(static_cast<size_t>(n > m_in ? n : m_in) * 2);
  L.d = L.c + r256(static_cast<size_t>(n) * 4);
  L.total = L.d + r256(static_cast<size_t>(m_in) * 4);
  return L;
}

__device__ __forceinline__ int packed_bit(const uint32_t* row, int64_t col) {
  const uint32_t w = row[(col >> 8) * 8 + ((col & 15) >> 1)];
  return static_cast<int>((w >> (((col & 255) >> 4) + 16 * (col & 1))) & 1u);
}

__global__ void bqq_fill_kernel(const __half* r, int64_t k, int64_t p, int64_t ones_len, __half* mid, __half* ones) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < p * k; i += stride)
    mid[i] = __float2half_rn(__half2float(r[i / k]) * 0.25f);  // r_i / 4: exact for normal fp16 r_i
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < ones_len; i += stride)
    ones[i] = __float2half_rn(1.0f);
}

// c[a] = sum_i (s_i + r_i / 2) * (ones of row a of Y in columns [ik, (i+1)k)).
__global__ void bqq_row_kernel(const uint32_t* packedY, int64_t wpr, int64_t n, int64_t k, int64_t p,
                               const __half* r, const __half* s, float* c) {
  const int64_t a = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (a >= n) return;
  const uint32_t* row = packedY + a * wpr;
  float acc = 0.f;
  for (int64_t i = 0; i < p; ++i) {
    int cnt = 0;
    for (int64_t col = i * k; col < (i + 1) * k; ++col) cnt += packed_bit(row, col);
    acc += (__half2float(s[i]) + 0.5f * __half2float(r[i])) * static_cast<float>(cnt);
  }
  c[a] = acc;
}

// d[col] = sum_i (t_i + r_i / 2) * (ones of column col of Z in rows [ik, (i+1)k)) + u - k sum_i r_i / 4.
__global__ void bqq_col_kernel(const uint32_t* packedZ, int64_t wpr, int64_t m_in, int64_t k, int64_t p,
                               const __half* r, const __half* t, const __half* u, float* d) {
  const int64_t col = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (col >= m_in) return;
  float acc = __half2float(*u);
  for (int64_t i = 0; i < p; ++i) {
    int cnt = 0;
    for (int64_t l = i * k; l < (i + 1) * k; ++l) cnt += packed_bit(packedZ + l * wpr, col);
    acc += (__half2float(t[i]) + 0.5f * __half2float(r[i])) * static_cast<float>(cnt) -
           0.25f * static_cast<float>(k) * __half2float(r[i]);
  }
  d[col] = acc;
}

// y[tok][a] = y32[tok][a] + c[a] * sum(x[tok]) + d . x[tok]; one CTA per token.
template <bool OUT_F32>
__global__ void bqq_correct_kernel(const __half* x, int64_t m_in, const float* y32, int64_t n, const float* c,
                                   const float* d, void* y) {
  __shared__ float red[2][kThreads / 32];
  const int64_t tok = blockIdx.x;
  const __half* xt = x + tok * m_in;
  float sx = 0.f, dx = 0.f;
  for (int64_t j = threadIdx.x; j < m_in; j += kThreads) {
    const float v = __half2float(xt[j]);
    sx += v;
    dx = fmaf(d[j], v, dx);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sx += __shfl_xor_sync(0xffffffffu, sx, off);
    dx += __shfl_xor_sync(0xffffffffu, dx, off);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[0][warp] = sx;
    red[1][warp] = dx;
  }
  __syncthreads();
  sx = 0.f;
  dx = 0.f;
  for (int w = 0; w < kThreads / 32; ++w) {  // fixed order: the same on every thread
    sx += red[0][w];
    dx += red[1][w];
  }
  for (int64_t a = threadIdx.x; a < n; a += kThreads) {
    const float v = fmaf(c[a], sx, y32[tok * n + a]) + dx;
    if constexpr (OUT_F32) {
      static_cast<float*>(y)[tok * n + a] = v;
    } else {
      static_cast<__half*>(y)[tok * n + a] = __float2half_rn(v);
    }
  }
}

inline bool aligned16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

dbf_status check_bqq_shape(int64_t n, int64_t k, int64_t p, int64_t m_in) {
  if (n < 1 || k < 1 || p < 1 || m_in < 1) return DBF_ERR_INVALID_ARG;
  if ((p * k) % 64 != 0 || m_in % 64 != 0 || p * k > (int64_t{1} << 20) || m_in > (int64_t{1} << 20) ||
      n > (int64_t{1} << 24) || p > 4096)
    return DBF_ERR_UNSUPPORTED_SHAPE;
  return DBF_OK;
}

}  // namespace
}  // namespace dbf

using namespace dbf;

extern "C" {

size_t dbf_bqq_prepared_bytes(int64_t n, int64_t k, int64_t p, int64_t m_in) {
  if (check_bqq_shape(n, k, p, m_in) != DBF_OK) return 0;
  return prep_layout(n, k, p, m_in).total;
}

dbf_status dbf_bqq_prepare(const uint32_t* packedY, const uint32_t* packedZ, const uint16_t* r, const uint16_t* s,
                           const uint16_t* t, const uint16_t* u, int64_t n, int64_t k, int64_t p, int64_t m_in,
                           void* prepared, size_t prepared_bytes, struct CUstream_st* stream_handle) {
  if (!packedY || !packedZ || !r || !s || !t || !u || !prepared) return DBF_ERR_INVALID_ARG;
  dbf_status st = check_bqq_shape(n, k, p, m_in);
  if (st != DBF_OK) return st;
  if (!aligned16(packedY) || !aligned16(packedZ) || !aligned16(prepared)) return DBF_ERR_MISALIGNED;
  const PrepLayout L = prep_layout(n, k, p, m_in);
  if (prepared_bytes < L.total) return DBF_ERR_WORKSPACE;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != DBF_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_handle);
  char* base = static_cast<char*>(prepared);
  const __half* rh = reinterpret_cast<const __half*>(r);
  const __half* sh = reinterpret_cast<const __half*>(s);
  const __half* th = reinterpret_cast<const __half*>(t);
  const __half* uh = reinterpret_cast<const __half*>(u);
  const int64_t ones_len = n > m_in ? n : m_in;
  st = launch_plain(bqq_fill_kernel, dim3(static_cast<unsigned>(2 * dev.num_sms)), dim3(kThreads), 0, stream, rh, k,
                    p, ones_len, reinterpret_cast<__half*>(base + L.mid), reinterpret_cast<__half*>(base + L.ones));
  if (st != DBF_OK) return st;
  st = launch_plain(bqq_row_kernel, dim3(static_cast<unsigned>((n + kThreads - 1) / kThreads)), dim3(kThreads), 0,
                    stream, packedY, words_per_row(p * k), n, k, p, rh, sh, reinterpret_cast<float*>(base + L.c));
  if (st != DBF_OK) return st;
  return launch_plain(bqq_col_kernel, dim3(static_cast<unsigned>((m_in + kThreads - 1) / kThreads)), dim3(kThreads),
                      0, stream, packedZ, words_per_row(m_in), m_in, k, p, rh, th, uh,
                      reinterpret_cast<float*>(base + L.d));
}

size_t dbf_bqq_workspace_bytes(int64_t n, int64_t k, int64_t p, int64_t m_in, int64_t batch) {
  if (check_bqq_shape(n, k, p, m_in) != DBF_OK || batch < 1) return 0;
  return dbf_forward_workspace_bytes(n, p * k, m_in, batch) + r256(static_cast<size_t>(batch * n) * 4);
}

dbf_status dbf_bqq_forward(const uint16_t* x, const uint32_t* packedY, const uint32_t* packedZ, const void* prepared,
                           int64_t n, int64_t k, int64_t p, int64_t m_in, int64_t batch, void* y, dbf_dtype y_t,
                           void* workspace, size_t ws_bytes, uint32_t flags, struct CUstream_st* stream_handle) {
  if (!prepared) return DBF_ERR_INVALID_ARG;
  dbf_status st = check_bqq_shape(n, k, p, m_in);
  if (st != DBF_OK) return st;
  if (!aligned16(prepared)) return DBF_ERR_MISALIGNED;
  const PrepLayout L = prep_layout(n, k, p, m_in);
  const char* base = static_cast<const char*>(prepared);
  const uint16_t* mid = reinterpret_cast<const uint16_t*>(base + L.mid);
  const uint16_t* ones = reinterpret_cast<const uint16_t*>(base + L.ones);
  st = validate_forward_args(x, packedY, packedZ, ones, mid, ones, n, p * k, m_in, batch, y, y_t, flags);
  if (st != DBF_OK) return st;
  const size_t fwd_ws = dbf_forward_workspace_bytes(n, p * k, m_in, batch);
  if (!workspace || !aligned16(workspace) || ws_bytes < dbf_bqq_workspace_bytes(n, k, p, m_in, batch))
    return DBF_ERR_WORKSPACE;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != DBF_OK) return st;
  float* y32 = reinterpret_cast<float*>(static_cast<char*>(workspace) + fwd_ws);
  // the sign-product term: a DBF layer with a = b = 1 and mid = r_i / 4 per term
  st = dbf_forward(x, packedY, packedZ, ones, mid, ones, n, p * k, m_in, batch, y32, DBF_F32, workspace, fwd_ws,
                   flags, stream_handle);
  if (st != DBF_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_handle);
  const float* c = reinterpret_cast<const float*>(base + L.c);
  const float* d = reinterpret_cast<const float*>(base + L.d);
  const __half* xh = reinterpret_cast<const __half*>(x);  // batch <= 2^24: checked with the forward's arguments
  if (y_t == DBF_F32)
    return launch_plain(bqq_correct_kernel<true>, dim3(static_cast<unsigned>(batch)), dim3(kThreads), 0, stream, xh,
                        m_in, static_cast<const float*>(y32), n, c, d, y);
  return launch_plain(bqq_correct_kernel<false>, dim3(static_cast<unsigned>(batch)), dim3(kThreads), 0, stream, xh,
                      m_in, static_cast<const float*>(y32), n, c, d, y);
}

}  // extern "C"
