// Offline DBF factorisation of a dense weight on the GPU: the alternating
// passes of "Addition is almost all you need" (gist.science technical summary,
// section 2.2, optimisation algorithm): alternating minimisation over the two
// factors, each constrained problem solved by ADMM with the SVID projection
// (sign matrix with rank-one magnitudes) as its constraint step.
//
// The factors are kept as dense fp32 matrices in SVID form,
//     L = diag(a) A diag(mL)  (n x k),   R = diag(mR) B diag(b)  (k x m),
// so W ~= L R = (a (.) A (.) mid^T)(B (.) b^T) with mid = mL (.) mR.
// One pass (dbf_factorize_pass):
//   left:  G = 2 R R^T + rho I, rho = trace(2 R R^T) / k;  Gi = G^-1
//          Z = L, U = 0; repeat: L' = (2 W R^T + rho (Z - U)) Gi,
//                                Z = SVID(L' + U), U += L' - Z
//          L = Z
//   right: the same for R with L fixed (G = 2 L^T L + rho I, R' = Gi (2 L^T W + rho (Z - U)))
//   err  = ||W - L R||_F / ||W||_F
// Dense products are cuBLAS SGEMMs (fp32, no tensor-op math).  G is
// symmetric positive definite with all eigenvalues in [rho, rho + lambda_max]
// (rho is the mean eigenvalue of 2 R R^T, so its condition number is at most
// k + 1), and its inverse comes from a Cholesky factorisation G = C C^T and
// the inverse of the factor (cuSOLVER potrf / potri, about k^3 flops), formed
// once per factor per pass so that every ADMM step is one GEMM.  SVID's rank-one
// magnitude is the leading singular pair of |M| by power iteration from the
// uniform vector (|M| is nonnegative: its leading pair is nonnegative and, for
// the matrices met here, well separated).  Every reduction runs in a fixed
// order (deterministic).
#include <cublas_v2.h>
#include <cuda_runtime.h>
#include <cusolverDn.h>

#include <mutex>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace dbf {
namespace {

constexpr int kT = 256;
constexpr int kPowerSteps = 30;
constexpr int kMaxDev = 64;

size_t al256(size_t v) { return (v + 255) / 256 * 256; }

cublasHandle_t handle_for(int device) {
  static cublasHandle_t h[kMaxDev] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (h[device] == nullptr) {
    cublasHandle_t nh = nullptr;
    if (cublasCreate(&nh) != CUBLAS_STATUS_SUCCESS) return nullptr;
    cublasSetPointerMode(nh, CUBLAS_POINTER_MODE_HOST);
    h[device] = nh;
  }
  return h[device];
}

cusolverDnHandle_t solver_for(int device) {
  static cusolverDnHandle_t h[kMaxDev] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (h[device] == nullptr) {
    cusolverDnHandle_t nh = nullptr;
    if (cusolverDnCreate(&nh) != CUSOLVER_STATUS_SUCCESS) return nullptr;
    h[device] = nh;
  }
  return h[device];
}

// Row-major C (r x c) = alpha op(A) op(B) + beta C, with op(A) r x inner and
// op(B) inner x c; A is stored row-major as (ta ? inner x r : r x inner), B as
// (tb ? c x inner : inner x c).  cuBLAS sees the transposed column-major problem.
bool gemm(cublasHandle_t h, bool ta, bool tb, int64_t r, int64_t c, int64_t inner, float alpha, const float* A,
          const float* B, float beta, float* C) {
  const int lda = static_cast<int>(ta ? r : inner);
  const int ldb = static_cast<int>(tb ? inner : c);
  return cublasSgemm(h, tb ? CUBLAS_OP_T : CUBLAS_OP_N, ta ? CUBLAS_OP_T : CUBLAS_OP_N, static_cast<int>(c),
                     static_cast<int>(r), static_cast<int>(inner), &alpha, B, ldb, A, lda, &beta, C,
                     static_cast<int>(c)) == CUBLAS_STATUS_SUCCESS;
}

// ---------------------------------------------------------------- reductions (one CTA, fixed order)
__device__ float block_sum(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < kT / 32; ++w) s += red[w];
  return s;
}

// Sum of squares of x (count elements) in two launches with a fixed order:
// CTA c sums a strided share (fp64 per thread) into part[c], then one CTA adds
// the kSumCtas parts.
constexpr int kSumCtas = 256;

__global__ void sumsq_part_kernel(const float* x, int64_t count, float* part) {
  __shared__ float red[kT / 32];
  double acc = 0.0;  // long sums: accumulate in fp64 per thread
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kT) + threadIdx.x; i < count;
       i += static_cast<int64_t>(kSumCtas) * kT)
    acc += static_cast<double>(x[i]) * x[i];
  const float s = block_sum(static_cast<float>(acc), red);
  if (threadIdx.x == 0) part[blockIdx.x] = s;
}

__global__ void sum_final_kernel(const float* part, float* out) {
  __shared__ float red[kT / 32];
  static_assert(kSumCtas == kT, "one part per thread");
  const float s = block_sum(part[threadIdx.x], red);
  if (threadIdx.x == 0) out[0] = s;
}

// G (k x k) += rho I with rho = trace(G) / k (G holds 2 R R^T); writes rho
// to scal[0].  One CTA.
__global__ void regularize_kernel(float* G, int64_t k, float* scal) {
  __shared__ float red[kT / 32];
  __shared__ float s_rho;
  float tr = 0.f;
  for (int64_t i = threadIdx.x; i < k; i += kT) tr += G[i * k + i];
  tr = block_sum(tr, red);
  if (threadIdx.x == 0) s_rho = tr > 0.f ? tr / static_cast<float>(k) : 1.f;
  __syncthreads();
  const float rho = s_rho;
  for (int64_t i = threadIdx.x; i < k; i += kT) G[i * k + i] += rho;
  if (threadIdx.x == 0) scal[0] = rho;
}

// Gi (k x k) holds the inverse in its lower triangle (column-major, so the
// upper triangle of the row-major array) after potri: mirror it into the other
// half.  A failed factorisation (*info != 0, only possible for a non-finite
// Gram) leaves NaN everywhere, so the pass's error is NaN and it is rejected.
__global__ void mirror_inverse_kernel(float* Gi, int64_t k, const int* info) {
  const bool bad = *info != 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < k * k;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / k, c = i % k;
    if (bad) {
      Gi[i] = __int_as_float(0x7fc00000);
    } else if (r > c) {
      Gi[i] = Gi[c * k + r];
    }
  }
}

// T = P + rho (Z - U)   (elementwise; P holds 2 W R^T or 2 L^T W)
__global__ void admm_rhs_kernel(const float* P, const float* Z, const float* U, const float* scal, float* T,
                                int64_t count) {
  const float rho = scal[0];
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    T[i] = P[i] + rho * (Z[i] - U[i]);
}

// M = L + U
__global__ void add_kernel(const float* L, const float* U, float* M, int64_t count) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    M[i] = L[i] + U[i];
}

// U += L - Z
__global__ void dual_kernel(const float* L, const float* Z, float* U, int64_t count) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    U[i] += L[i] - Z[i];
}

// u[i] = c for all i (power-iteration start, c = 1/sqrt(rows))
__global__ void fill_kernel(float* u, int64_t count, float c) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    u[i] = c;
}

// part[c][j] = sum over rows i of chunk c of |M[i][j]| u[i] / ||u||   (rows x
// cols row-major; a thread per column and chunk, the chunk's rows in order).
// Every CTA forms ||u|| itself in the same fixed order (no separate
// normalisation launch for u).
constexpr int kRowChunks = 32;
__global__ void abs_gemv_t_part_kernel(const float* M, const float* u, int64_t rows, int64_t cols, float* part) {
  __shared__ float red[kT / 32];
  float q = 0.f;
  for (int64_t i = threadIdx.x; i < rows; i += kT) q = fmaf(u[i], u[i], q);
  q = block_sum(q, red);
  const float nrm = sqrtf(q);
  const float inv = nrm > 0.f ? 1.f / nrm : 0.f;
  const int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t c = blockIdx.y;
  if (j >= cols) return;
  const int64_t per = (rows + kRowChunks - 1) / kRowChunks;
  const int64_t i1 = (c + 1) * per < rows ? (c + 1) * per : rows;
  float s = 0.f;
  for (int64_t i = c * per; i < i1; ++i) s = fmaf(fabsf(M[i * cols + j]), u[i], s);
  part[c * cols + j] = s * inv;
}

// v[j] = sum of the chunks' parts in chunk order
__global__ void sum_parts_kernel(const float* part, int64_t cols, float* v) {
  const int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (j >= cols) return;
  float s = 0.f;
  for (int c = 0; c < kRowChunks; ++c) s += part[c * cols + j];
  v[j] = s;
}

// u[i] = sum_j |M[i][j]| v[j] / ||v||   (a warp per row, lanes over the row,
// fixed-order tree).  Each warp reads all of v for its row, so it forms ||v||
// in the same loop, in the same order in every warp: the power step needs no
// separate normalisation launch for v.
__global__ void abs_gemv_kernel(const float* M, const float* v, int64_t rows, int64_t cols, float* u) {
  const int64_t i = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (i >= rows) return;
  float s = 0.f, q = 0.f;
  for (int64_t j = lane; j < cols; j += 32) {
    const float vj = v[j];
    s = fmaf(fabsf(M[i * cols + j]), vj, s);
    q = fmaf(vj, vj, q);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, off);
    q += __shfl_xor_sync(0xffffffffu, q, off);
  }
  const float nrm = sqrtf(q);
  if (lane == 0) u[i] = nrm > 0.f ? s * (1.f / nrm) : 0.f;
}

// x /= ||x|| (one CTA); if nrm_out, *nrm_out = ||x|| before the division.
__global__ void normalize_kernel(float* x, int64_t count, float* nrm_out) {
  __shared__ float red[kT / 32];
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < count; i += kT) s = fmaf(x[i], x[i], s);
  s = block_sum(s, red);
  const float nrm = sqrtf(s);
  const float inv = nrm > 0.f ? 1.f / nrm : 0.f;
  for (int64_t i = threadIdx.x; i < count; i += kT) x[i] *= inv;
  if (threadIdx.x == 0 && nrm_out) *nrm_out = nrm;
}

// Z[i][j] = (M[i][j] < 0 ? -1 : 1) * sigma * u[i] * v[j]   (u, v unit vectors)
__global__ void svid_rebuild_kernel(const float* M, const float* u, const float* v, const float* sigma, int64_t rows,
                                    int64_t cols, float* Z) {
  const float sg = *sigma;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < rows * cols;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = idx / cols, j = idx - i * cols;
    const float mag = sg * u[i] * v[j];
    Z[idx] = M[idx] < 0.f ? -mag : mag;
  }
}

// E = W - E (elementwise), then out = ||E||_F / ||W||_F (the second via the sumsq kernel)
__global__ void residual_kernel(const float* W, float* E, int64_t count) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    E[i] = W[i] - E[i];
}

__global__ void ratio_sqrt_kernel(const float* num, const float* den, float* out) {
  out[0] = den[0] > 0.f ? sqrtf(num[0] / den[0]) : 0.f;
}

// sigma, u (unit), v (unit) of the leading singular pair of |M| (rows x cols);
// part: kRowChunks * cols floats of scratch.
dbf_status svid_pair(const float* M, int64_t rows, int64_t cols, float* u, float* v, float* sigma, float* part,
                     int grid, cudaStream_t s) {
  fill_kernel<<<grid, kT, 0, s>>>(u, rows, 1.f);
  const unsigned cblocks = static_cast<unsigned>((cols + kT - 1) / kT);
  for (int it = 0; it < kPowerSteps; ++it) {
    abs_gemv_t_part_kernel<<<dim3(cblocks, kRowChunks), kT, 0, s>>>(M, u, rows, cols, part);
    sum_parts_kernel<<<cblocks, kT, 0, s>>>(part, cols, v);
    abs_gemv_kernel<<<static_cast<unsigned>((rows * 32 + kT - 1) / kT), kT, 0, s>>>(M, v, rows, cols, u);
  }
  // u = |M| v / ||v|| of the last step: sigma = ||u||; both vectors to unit
  // length (inside the loop each product normalises its input vector itself)
  normalize_kernel<<<1, kT, 0, s>>>(v, cols, nullptr);
  normalize_kernel<<<1, kT, 0, s>>>(u, rows, sigma);
  return cudaGetLastError() == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

// Y (cols x rows) = X^T for X rows x cols, row-major.
__global__ void transpose_kernel(const float* X, int64_t rows, int64_t cols, float* Y) {
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < rows * cols;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = idx / rows, i = idx - j * rows;  // output row j, column i
    Y[idx] = X[i * cols + j];
  }
}

// out[i] = fp16(sqrt(sigma) * x[i]) (x a unit vector of the SVID pair); optional
// second vector y multiplies in (the middle vector mL (.) mR).
__global__ void scale_half_kernel(const float* x, const float* sigma_x, const float* y, const float* sigma_y,
                                  int64_t count, __half* out) {
  const float sx = sqrtf(*sigma_x);
  const float sy = y ? sqrtf(*sigma_y) : 1.f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v = sx * x[i];
    if (y) v *= sy * y[i];
    out[i] = __float2half_rn(v);
  }
}

struct FactWs {
  float *G, *Gi, *Y, *X2, *P, *T, *Lt, *Z, *U, *M, *E, *u, *v, *part, *scal;
  size_t total;
};

FactWs fact_layout(char* base, int64_t n, int64_t m, int64_t k) {
  const int64_t big = (n > m ? n : m) * k;  // the largest factor
  FactWs w{};
  size_t off = 0;
  auto take = [&](float** p, size_t count) {
    if (base) *p = reinterpret_cast<float*>(base + off);
    off += al256(count * 4);
  };
  take(&w.G, k * k);
  take(&w.Gi, k * k);
  take(&w.Y, k * k);
  take(&w.X2, k * k);
  take(&w.P, big);
  take(&w.T, big);
  take(&w.Lt, big);
  take(&w.Z, big);
  take(&w.U, big);
  take(&w.M, big);
  take(&w.E, n * m);
  take(&w.u, (n > m ? n : m) > k ? (n > m ? n : m) : k);
  take(&w.v, (n > m ? n : m) > k ? (n > m ? n : m) : k);
  take(&w.part, static_cast<size_t>(kRowChunks) * ((n > m ? n : m) > k ? (n > m ? n : m) : k));
  take(&w.scal, 64);
  w.total = off;
  return w;
}

// Gi = G^-1 for G (k x k) symmetric positive definite: Cholesky factor of a
// copy, inverse from the factor, mirrored to a full matrix.  The solver's
// scratch is the k x k pair Y, X2 when its request fits there (large k), else
// a stream-ordered allocation freed on the same stream; its status word sits
// in the scalar area.
dbf_status cholesky_inverse(cusolverDnHandle_t sh, const FactWs& w, int64_t k, int grid, cudaStream_t s) {
  const int kk = static_cast<int>(k);
  const size_t cap = static_cast<size_t>(w.X2 - w.Y) + static_cast<size_t>(k * k);  // floats in Y..X2
  int lw_f = 0, lw_i = 0;
  if (cudaMemcpyAsync(w.Gi, w.G, static_cast<size_t>(k * k) * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return DBF_ERR_CUDA;
  if (cusolverDnSpotrf_bufferSize(sh, CUBLAS_FILL_MODE_LOWER, kk, w.Gi, kk, &lw_f) != CUSOLVER_STATUS_SUCCESS ||
      cusolverDnSpotri_bufferSize(sh, CUBLAS_FILL_MODE_LOWER, kk, w.Gi, kk, &lw_i) != CUSOLVER_STATUS_SUCCESS)
    return DBF_ERR_CUDA;
  const int lw = lw_f > lw_i ? lw_f : lw_i;
  if (lw < 0) return DBF_ERR_CUDA;
  float* scratch = w.Y;
  void* own = nullptr;
  if (static_cast<size_t>(lw) > cap) {
    if (cudaMallocAsync(&own, static_cast<size_t>(lw) * 4, s) != cudaSuccess) return DBF_ERR_CUDA;
    scratch = static_cast<float*>(own);
  }
  int* info = reinterpret_cast<int*>(w.scal + 16);
  const bool ok =
      cusolverDnSpotrf(sh, CUBLAS_FILL_MODE_LOWER, kk, w.Gi, kk, scratch, lw, info) == CUSOLVER_STATUS_SUCCESS &&
      cusolverDnSpotri(sh, CUBLAS_FILL_MODE_LOWER, kk, w.Gi, kk, scratch, lw, info) == CUSOLVER_STATUS_SUCCESS;
  if (own && cudaFreeAsync(own, s) != cudaSuccess) return DBF_ERR_CUDA;
  if (!ok) return DBF_ERR_CUDA;
  mirror_inverse_kernel<<<grid, kT, 0, s>>>(w.Gi, k, info);
  return cudaGetLastError() == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

// One ADMM solve of a factor F (rows x cols, in/out, SVID form) with P = the
// right-hand side product and Gi the inverse; left: F = T Gi, right: F = Gi T.
dbf_status admm_factor(cublasHandle_t h, const FactWs& w, float* F, int64_t rows, int64_t cols, bool left, int steps,
                       int grid, cudaStream_t s) {
  const int64_t count = rows * cols;
  if (cudaMemcpyAsync(w.Z, F, static_cast<size_t>(count) * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemsetAsync(w.U, 0, static_cast<size_t>(count) * 4, s) != cudaSuccess)
    return DBF_ERR_CUDA;
  const int64_t k = left ? cols : rows;
  for (int it = 0; it < steps; ++it) {
    admm_rhs_kernel<<<grid, kT, 0, s>>>(w.P, w.Z, w.U, w.scal, w.T, count);
    const bool ok = left ? gemm(h, false, false, rows, cols, k, 1.f, w.T, w.Gi, 0.f, w.Lt)
                         : gemm(h, false, false, rows, cols, k, 1.f, w.Gi, w.T, 0.f, w.Lt);
    if (!ok) return DBF_ERR_CUDA;
    add_kernel<<<grid, kT, 0, s>>>(w.Lt, w.U, w.M, count);
    dbf_status st = svid_pair(w.M, rows, cols, w.u, w.v, w.scal + 2, w.part, grid, s);
    if (st != DBF_OK) return st;
    svid_rebuild_kernel<<<grid, kT, 0, s>>>(w.M, w.u, w.v, w.scal + 2, rows, cols, w.Z);
    dual_kernel<<<grid, kT, 0, s>>>(w.Lt, w.Z, w.U, count);
  }
  if (cudaMemcpyAsync(F, w.Z, static_cast<size_t>(count) * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return DBF_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

// *err = ||W - L R||_F / ||W||_F
dbf_status rel_error(cublasHandle_t h, const FactWs& w, const float* W, const float* L, const float* R, int64_t n,
                     int64_t m, int64_t k, float* err, int grid, cudaStream_t s) {
  if (!gemm(h, false, false, n, m, k, 1.f, L, R, 0.f, w.E)) return DBF_ERR_CUDA;
  residual_kernel<<<grid, kT, 0, s>>>(W, w.E, n * m);
  sumsq_part_kernel<<<kSumCtas, kT, 0, s>>>(w.E, n * m, w.part);
  sum_final_kernel<<<1, kT, 0, s>>>(w.part, w.scal + 4);
  sumsq_part_kernel<<<kSumCtas, kT, 0, s>>>(W, n * m, w.part);
  sum_final_kernel<<<1, kT, 0, s>>>(w.part, w.scal + 5);
  ratio_sqrt_kernel<<<1, 1, 0, s>>>(w.scal + 4, w.scal + 5, err);
  return cudaGetLastError() == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

// F = SVID(M) (rows x cols), with the pair left in w.u, w.v and sigma in sigma.
dbf_status svid_into(const FactWs& w, const float* M, int64_t rows, int64_t cols, float* F, float* sigma, int grid,
                     cudaStream_t s) {
  dbf_status st = svid_pair(M, rows, cols, w.u, w.v, sigma, w.part, grid, s);
  if (st != DBF_OK) return st;
  svid_rebuild_kernel<<<grid, kT, 0, s>>>(M, w.u, w.v, sigma, rows, cols, F);
  return cudaGetLastError() == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

inline bool aligned16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

dbf_status check_fact_shape(int64_t n, int64_t m, int64_t k) {
  if (n < 1 || m < 1 || k < 1) return DBF_ERR_INVALID_ARG;
  if (n > 65536 || m > 65536 || k > 16384 || n * m > (int64_t{1} << 31) || k * (n > m ? n : m) > (int64_t{1} << 31))
    return DBF_ERR_UNSUPPORTED_SHAPE;
  return DBF_OK;
}

}  // namespace
}  // namespace dbf

using namespace dbf;

extern "C" {

size_t dbf_svid_workspace_bytes(int64_t rows, int64_t cols) {
  if (rows < 1 || cols < 1) return 0;
  return static_cast<size_t>(kRowChunks) * static_cast<size_t>(cols) * 4;
}

size_t dbf_factorize_workspace_bytes(int64_t n, int64_t m, int64_t k) {
  if (check_fact_shape(n, m, k) != DBF_OK) return 0;
  return fact_layout(nullptr, n, m, k).total;
}

dbf_status dbf_svid(const float* M, int64_t rows, int64_t cols, float* u, float* v, float* sigma, void* workspace,
                    size_t ws_bytes, struct CUstream_st* stream_handle) {
  if (!M || !u || !v || !sigma || !workspace) return DBF_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1) return DBF_ERR_INVALID_ARG;
  if (rows * cols > (int64_t{1} << 31)) return DBF_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(M) || !aligned16(u) || !aligned16(v) || !aligned16(sigma) || !aligned16(workspace))
    return DBF_ERR_MISALIGNED;
  if (ws_bytes < dbf_svid_workspace_bytes(rows, cols)) return DBF_ERR_WORKSPACE;
  DeviceInfo dev;
  dbf_status st = current_device(&dev);
  if (st != DBF_OK) return st;
  return svid_pair(M, rows, cols, u, v, sigma, static_cast<float*>(workspace), 2 * dev.num_sms,
                   reinterpret_cast<cudaStream_t>(stream_handle));
}

dbf_status dbf_factorize_pass(const float* W, int64_t n, int64_t m, int64_t k, float* L, float* R, int admm_steps,
                              float* err, void* workspace, size_t ws_bytes, struct CUstream_st* stream_handle) {
  if (!W || !L || !R || !err || !workspace) return DBF_ERR_INVALID_ARG;
  dbf_status st = check_fact_shape(n, m, k);
  if (st != DBF_OK) return st;
  if (admm_steps < 1 || admm_steps > 1000) return DBF_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(L) || !aligned16(R) || !aligned16(err) || !aligned16(workspace))
    return DBF_ERR_MISALIGNED;
  if (ws_bytes < dbf_factorize_workspace_bytes(n, m, k)) return DBF_ERR_WORKSPACE;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != DBF_OK) return st;
  cublasHandle_t h = handle_for(dev.device);
  cusolverDnHandle_t sh = solver_for(dev.device);
  if (!h || !sh) return DBF_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_handle);
  if (cublasSetStream(h, s) != CUBLAS_STATUS_SUCCESS || cusolverDnSetStream(sh, s) != CUSOLVER_STATUS_SUCCESS)
    return DBF_ERR_CUDA;
  const FactWs w = fact_layout(static_cast<char*>(workspace), n, m, k);
  const int grid = 4 * dev.num_sms;

  // left factor, R fixed
  if (!gemm(h, false, true, k, k, m, 2.f, R, R, 0.f, w.G)) return DBF_ERR_CUDA;  // 2 R R^T
  regularize_kernel<<<1, kT, 0, s>>>(w.G, k, w.scal);
  st = cholesky_inverse(sh, w, k, grid, s);
  if (st != DBF_OK) return st;
  if (!gemm(h, false, true, n, k, m, 2.f, W, R, 0.f, w.P)) return DBF_ERR_CUDA;  // 2 W R^T
  st = admm_factor(h, w, L, n, k, true, admm_steps, grid, s);
  if (st != DBF_OK) return st;
  // right factor, L fixed
  if (!gemm(h, true, false, k, k, n, 2.f, L, L, 0.f, w.G)) return DBF_ERR_CUDA;  // 2 L^T L
  regularize_kernel<<<1, kT, 0, s>>>(w.G, k, w.scal);
  st = cholesky_inverse(sh, w, k, grid, s);
  if (st != DBF_OK) return st;
  if (!gemm(h, true, false, k, m, n, 2.f, L, W, 0.f, w.P)) return DBF_ERR_CUDA;  // 2 L^T W
  st = admm_factor(h, w, R, k, m, false, admm_steps, grid, s);
  if (st != DBF_OK) return st;
  return rel_error(h, w, W, L, R, n, m, k, err, grid, s);
}

dbf_status dbf_factorize_start(const float* W, const float* Omega, int64_t n, int64_t m, int64_t k, float* L,
                               float* R, float* err, void* workspace, size_t ws_bytes, struct CUstream_st* stream_handle) {
  if (!W || !Omega || !L || !R || !err || !workspace) return DBF_ERR_INVALID_ARG;
  dbf_status st = check_fact_shape(n, m, k);
  if (st != DBF_OK) return st;
  if (!aligned16(W) || !aligned16(Omega) || !aligned16(L) || !aligned16(R) || !aligned16(err) ||
      !aligned16(workspace))
    return DBF_ERR_MISALIGNED;
  if (ws_bytes < dbf_factorize_workspace_bytes(n, m, k)) return DBF_ERR_WORKSPACE;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != DBF_OK) return st;
  cublasHandle_t h = handle_for(dev.device);
  if (!h) return DBF_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_handle);
  if (cublasSetStream(h, s) != CUBLAS_STATUS_SUCCESS) return DBF_ERR_CUDA;
  const FactWs w = fact_layout(static_cast<char*>(workspace), n, m, k);
  const int grid = 4 * dev.num_sms;
  if (!gemm(h, false, false, n, k, m, 1.f, W, Omega, 0.f, w.M)) return DBF_ERR_CUDA;  // W Omega
  st = svid_into(w, w.M, n, k, L, w.scal + 2, grid, s);
  if (st != DBF_OK) return st;
  transpose_kernel<<<grid, kT, 0, s>>>(Omega, m, k, w.M);  // Omega^T (k x m)
  st = svid_into(w, w.M, k, m, R, w.scal + 2, grid, s);
  if (st != DBF_OK) return st;
  return rel_error(h, w, W, L, R, n, m, k, err, grid, s);
}

dbf_status dbf_factorize_finish(const float* L, const float* R, int64_t n, int64_t m, int64_t k, uint32_t* packedA,
                                uint32_t* packedB, uint16_t* a, uint16_t* mid, uint16_t* b, void* workspace,
                                size_t ws_bytes, struct CUstream_st* stream_handle) {
  if (!L || !R || !packedA || !packedB || !a || !mid || !b || !workspace) return DBF_ERR_INVALID_ARG;
  dbf_status st = check_fact_shape(n, m, k);
  if (st != DBF_OK) return st;
  if (!aligned16(L) || !aligned16(R) || !aligned16(packedA) || !aligned16(packedB) || !aligned16(a) ||
      !aligned16(mid) || !aligned16(b) || !aligned16(workspace))
    return DBF_ERR_MISALIGNED;
  if (ws_bytes < dbf_factorize_workspace_bytes(n, m, k)) return DBF_ERR_WORKSPACE;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != DBF_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_handle);
  const FactWs w = fact_layout(static_cast<char*>(workspace), n, m, k);
  const int grid = 4 * dev.num_sms;
  // L = sigma_L uL vL^T (.) A: a = sqrt(sigma_L) uL, mL = sqrt(sigma_L) vL (kept in w.P)
  st = svid_pair(L, n, k, w.u, w.v, w.scal + 8, w.part, grid, s);
  if (st != DBF_OK) return st;
  scale_half_kernel<<<grid, kT, 0, s>>>(w.u, w.scal + 8, nullptr, nullptr, n, reinterpret_cast<__half*>(a));
  if (cudaMemcpyAsync(w.P, w.v, static_cast<size_t>(k) * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return DBF_ERR_CUDA;
  // R = sigma_R uR vR^T (.) B: mR = sqrt(sigma_R) uR, b = sqrt(sigma_R) vR; mid = mL (.) mR
  st = svid_pair(R, k, m, w.u, w.v, w.scal + 9, w.part, grid, s);
  if (st != DBF_OK) return st;
  scale_half_kernel<<<grid, kT, 0, s>>>(w.v, w.scal + 9, nullptr, nullptr, m, reinterpret_cast<__half*>(b));
  scale_half_kernel<<<grid, kT, 0, s>>>(w.P, w.scal + 8, w.u, w.scal + 9, k, reinterpret_cast<__half*>(mid));
  // signs: a set bit where the factor is negative
  st = launch_pack(L, DBF_F32, n, k, packedA, dev, s);
  if (st != DBF_OK) return st;
  return launch_pack(R, DBF_F32, k, m, packedB, dev, s);
}

}  // extern "C"
