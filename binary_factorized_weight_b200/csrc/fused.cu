// Decode path (batch <= 16) in ONE launch per layer.
//
// "Addition is almost all you need" (gist.science technical summary, section
// 2.1, computation process) evaluates the layer as two products with +-1
// matrices:  t = B (x (.) b),  V = mid (.) t,  y = a (.) (A V).
// At a handful of tokens both products are bound by latency, not arithmetic,
// so this kernel does the whole layer in one grid and hands the middle vector
// from the first product to the second inside the chip.
//
// Work split.  The middle dimension k is cut into J slices of kb rows (kb a
// multiple of 256); slice j belongs to a thread-block cluster of R CTAs
// (R <= 16).  Rank r of cluster j
//   1. multiplies its kb rows of B over its share of the m_in columns
//      (whole 256-column blocks) -> a partial t for the slice;
//   2. the R partials meet through distributed shared memory: rank r' adds the
//      R parts of its kb/R rows in rank order (reduce-scatter), scales them by
//      mid and sends the result to every rank (all-gather), so each rank holds
//      V for the whole slice -- V never leaves the cluster;
//   3. multiplies its nb output rows of A over the slice's kb columns -> a
//      partial z of y;
//   4. the J partials of each output row meet in global memory: cluster 0's
//      rank r waits for the other clusters' partials of its rows (each 64-bit
//      word carries its value and a valid tag, so the data arrives with the
//      wait itself), adds them in cluster order, scales by a and stores y.
// Every wait is bounded; a lost arrival records DBF_ERR_TIMEOUT in the
// workspace status word.
//
// Arithmetic.  The sign products run on the int8 warp MMA (mma.sync
// m16n8k32 s8 x s8 -> s32), exactly.  Activations (x (.) b for the first
// product, V for the second) are written in block fixed point: per token and
// per CTA slice, q = rint(u * 2^e) with e chosen so that |q| < 2^22, split into
// three signed base-256 digits, each digit a column of the MMA's N operand
// (column 3*token + digit).  The signs are the M operand, formed from the
// packed words with one mask per register:
//   class form (<= 2 N tiles): byte i of (w & (0x01010101 << s)) is 2^s (s < 7)
//     or -128 (s = 7) where the sign bit is set, so K step s accumulates into
//     its own set D_s and sum(bit * q) = sum_{s<7} D_s / 2^s - D_7 / 128;
//   shift form (more N tiles): (w >> s) & 0x01010101 gives the bits themselves.
// With Q = sum(q), sum(sign * q) = Q - 2 sum(bit * q), all in int32 (exact),
// recombined over the digits in int64 and scaled by 2^-e into fp32: one
// rounding per CTA partial.  No fp16 rounding of x (.) b or of V happens on
// this path; with integer data every step is exact.
//
// Packed layout (shared with the rest of the library): column e of a 256-column
// block sits in word (e % 16) / 2 at bit e / 16 + 16 (e % 2).  For K step s the
// mask picks bits {s, s+8, s+16, s+24}, i.e. groups s and s + 8 of the block:
// byte i of word p holds column 16 (s + 8 (i & 1)) + 2 p + (i >> 1).  Lane
// (g, c) takes words 2c (k positions 4c..4c+3) and 2c + 1 (16 + 4c..) of rows
// g and g + 8; the activation digits are stored in the same order.
#include <algorithm>
#include <mutex>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace dbf {
namespace {

constexpr int kFThreads = 256;
constexpr int kFWarps = kFThreads / 32;
constexpr int kMaxTok = 16;
constexpr int kFusedSmemBudget = 200 * 1024;

__host__ __device__ inline int align128(int v) { return (v + 127) & ~127; }

// Shared-memory layout of one CTA (host and device compute it the same way).
struct FusedSmem {
  int wB, wA, dig, U, Tb, part, red, z, total;
};

// The partial sums of the first product meet in one all-to-all round (every
// rank sends its whole slice to every peer and adds the R parts itself) when
// the R copies fit in 64 KB of shared memory, else in two rounds
// (reduce-scatter of kb / R rows per rank, then all-gather).
__host__ __device__ inline bool fused_one_round(const FusedArgs& p) {
  return p.R > 1 && p.R * p.batch * p.kb * 4 <= 64 * 1024;
}

__host__ __device__ inline FusedSmem fused_smem_layout(const FusedArgs& p, int ntile) {
  const int ncol = 8 * ntile;
  const int nblkB_max = (p.MB + p.R - 1) / p.R;
  const int nblkA = p.kb / 256;
  const int nblk_max = nblkB_max > nblkA ? nblkB_max : nblkA;
  FusedSmem L;
  int off = 2560;  // mbarriers, abort flag, exponents, per-warp digit sums and token maxima
  L.wB = off;
  off += align128((p.kb / 16) * nblkB_max * 512);
  L.wA = off;
  off += align128((p.nb / 16) * nblkA * 512);
  L.dig = off;
  off += align128(nblk_max * 8 * ncol * 32);
  L.U = off;
  off += align128(p.batch * nblk_max * 256 * 4);
  L.Tb = off;
  off += align128(kFWarps * 16 * ncol * 4);
  L.part = off;
  off += align128(p.batch * p.kb * 4);
  L.red = off;
  off += align128((fused_one_round(p) ? p.R : 1) * p.batch * p.kb * 4);
  L.z = off;
  off += align128(p.batch * p.nb * 4);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void st_async_v4(uint32_t dst_cluster, float4 v, uint32_t bar_cluster) {
  st_async_v4f32(dst_cluster, v.x, v.y, v.z, v.w, bar_cluster);
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Two 64-bit words at a 16-byte aligned address; each word is accessed as a
// unit (a word's value and its tag are never torn).
__device__ __forceinline__ void ld_relaxed_u64x2(const unsigned long long* p, unsigned long long& a,
                                                 unsigned long long& b) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
__device__ __forceinline__ void st_relaxed_u64x2(unsigned long long* p, unsigned long long a, unsigned long long b) {
  asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}

template <bool CLASS>
__device__ __forceinline__ uint32_t sign_bytes(uint32_t w, int s) {
  return CLASS ? (w & (0x01010101u << s)) : ((w >> s) & 0x01010101u);
}

// 2^v as a float for v in [-126, 127].
__device__ __forceinline__ float pow2f(int v) { return __int_as_float((v + 127) << 23); }

// Block fixed point of the activations of one product, for this CTA's slice:
// U[tok][0..cols) fp32 (zero past the valid columns) -> digit bytes in the MMA
// order, per-token exponents exps[tok] and the digit sums Q[3 tok + d].
// 2^lg = kFWarps / batch warps share a token (one warp per token past 4
// tokens; warp w then also takes token w + 8), each taking every 2^lg-th run
// of 32 columns.  Two block barriers inside; Q is complete after the caller's
// next barrier.
__device__ __forceinline__ int warps_per_token_log2(int batch) { return batch == 1 ? 3 : batch == 2 ? 2 : batch <= 4 ? 1 : 0; }

template <int NTILE>
__device__ __forceinline__ void build_digits(const float* U, int cols, int batch, uint8_t* dig, int* exps, int* Q,
                                          float* redmax) {
  constexpr int NCOL = 8 * NTILE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lg = warps_per_token_log2(batch);
  const int part = warp & ((1 << lg) - 1);
  const int tok0 = warp >> lg;
  const int tstep = kFWarps >> lg;  // tokens handled by one pass of all warps
  const int stride = 32 << lg;
  if (threadIdx.x < 3 * kMaxTok) Q[threadIdx.x] = 0;
  // token maxima: each warp over its columns, then across the token's warps
  for (int tok = tok0; tok < batch; tok += tstep) {
    const float* u = U + tok * cols;
    float mx = 0.f;
    for (int col = part * 32 + lane; col < cols; col += stride) mx = fmaxf(mx, fabsf(u[col]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) redmax[tok * kFWarps + part] = mx;
  }
  __syncthreads();
  for (int tok = tok0; tok < batch; tok += tstep) {
    // the token's maximum from its warps' parts (all 8 slots read at once; unused ones are never 0-valued reads
    // of other tokens because only 2^lg of them are combined)
    float mx = 0.f;
#pragma unroll
    for (int q = 0; q < kFWarps; ++q)
      if (q < (1 << lg)) mx = fmaxf(mx, redmax[tok * kFWarps + q]);
    // |q| < 2^22: e = 21 - floor(log2(max)), clamped so that 2^e stays a normal float
    int e = 0;
    if (mx > 0.f) {
      const int emax = ((__float_as_int(mx) >> 23) & 255) - 127;  // max is a normal number or tiny
      e = 21 - (emax < -126 ? -126 : emax);
      e = e > 126 ? 126 : (e < -126 ? -126 : e);
    }
    const float scale = pow2f(e);
    const float* u = U + tok * cols;
    int q0 = 0, q1 = 0, q2 = 0;
    for (int col = part * 32 + lane; col < cols; col += stride) {
      const int q = __float2int_rn(u[col] * scale);
      const int d0 = ((q + 128) & 255) - 128;
      const int r1 = (q - d0) >> 8;
      const int d1 = ((r1 + 128) & 255) - 128;
      const int d2 = (r1 - d1) >> 8;
      q0 += d0;
      q1 += d1;
      q2 += d2;
      const int blk = col >> 8, el = col & 255;
      const int grp = el >> 4, pr = (el & 15) >> 1, h = el & 1;
      const int s = grp & 7, i = (grp >> 3) | (h << 1), cq = pr >> 1, half = pr & 1;
      uint8_t* base = dig + ((blk * 8 + s) * NCOL) * 32 + cq * 8 + half * 4 + i;
      base[(3 * tok + 0) * 32] = static_cast<uint8_t>(d0);
      base[(3 * tok + 1) * 32] = static_cast<uint8_t>(d1);
      base[(3 * tok + 2) * 32] = static_cast<uint8_t>(d2);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      q0 += __shfl_xor_sync(0xffffffffu, q0, off);
      q1 += __shfl_xor_sync(0xffffffffu, q1, off);
      q2 += __shfl_xor_sync(0xffffffffu, q2, off);
    }
    if (lane == 0) {
      if (part == 0) exps[tok] = e;
      atomicAdd(&Q[3 * tok + 0], q0);  // integer sums: the order does not matter
      atomicAdd(&Q[3 * tok + 1], q1);
      atomicAdd(&Q[3 * tok + 2], q2);
    }
  }
}

// One product over this CTA's tiles: out[tok][row] (fp32, rows of the tiles)
// = sum over the slice's blocks of sign(row, col) * u[tok][col], exactly in
// int32 per digit, then 2^-e[tok] * (T2 * 65536 + T1 * 256 + T0).
// w: weight items [tile][blk] of 16 rows x 32 bytes.  Warp w takes tiles w, w + 8, ...
template <int NTILE, bool CLASS>
__device__ __forceinline__ void sign_product(const uint8_t* w, int tiles, int nblk, const uint8_t* dig, const int* exps,
                                          const int* Q, int batch, int* Tb, float* out, int ld_out) {
  constexpr int NCOL = 8 * NTILE;
  constexpr int NACC = CLASS ? 8 : 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  int* T = Tb + warp * 16 * NCOL;
  int qcol[NTILE][2];  // digit sums of this lane's columns (unused columns: anything)
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h) qcol[nt][h] = Q[nt * 8 + 2 * c + h];
  for (int t = warp; t < tiles; t += kFWarps) {
    int acc[NACC][NTILE][4];
#pragma unroll
    for (int a = 0; a < NACC; ++a)
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[a][nt][e] = 0;
    for (int q = 0; q < nblk; ++q) {
      const uint8_t* wi = w + (t * nblk + q) * 512;
      const uint2 wlo = *reinterpret_cast<const uint2*>(wi + g * 32 + c * 8);
      const uint2 whi = *reinterpret_cast<const uint2*>(wi + (g + 8) * 32 + c * 8);
      const uint8_t* dq = dig + q * 8 * NCOL * 32 + g * 32 + c * 8;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t a0 = sign_bytes<CLASS>(wlo.x, s);
        const uint32_t a1 = sign_bytes<CLASS>(whi.x, s);
        const uint32_t a2 = sign_bytes<CLASS>(wlo.y, s);
        const uint32_t a3 = sign_bytes<CLASS>(whi.y, s);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) {
          const uint2 bf = *reinterpret_cast<const uint2*>(dq + (s * NCOL + nt * 8) * 32);
          mma_s8(acc[CLASS ? s : 0][nt], a0, a1, a2, a3, bf.x, bf.y);
        }
      }
    }
    if constexpr (NTILE == 1) {
      // One N tile (batch <= 2): token t's digit columns 3t..3t+2 lie in lanes
      // c = t and c + 1 of the quad, so the combination stays in registers.
      int T[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int bits;
        if constexpr (CLASS) {
          bits = -(acc[7][0][e] >> 7);
#pragma unroll
          for (int s = 0; s < 7; ++s) bits += acc[s][0][e] >> s;
        } else {
          bits = acc[0][0][e];
        }
        T[e] = qcol[0][e & 1] - 2 * bits;
      }
      int Tn[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) Tn[e] = __shfl_down_sync(0xffffffffu, T[e], 1);
      if (c < batch) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {  // rows g and g + 8
          const int e0 = 2 * hr;
          const int d0 = c == 0 ? T[e0] : T[e0 + 1];
          const int d1 = c == 0 ? T[e0 + 1] : Tn[e0];
          const int d2 = c == 0 ? Tn[e0] : Tn[e0 + 1];
          const long long v = static_cast<long long>(d2) * 65536ll + static_cast<long long>(d1) * 256ll + d0;
          out[c * ld_out + t * 16 + g + 8 * hr] = __ll2float_rn(v) * pow2f(-exps[c]);  // one rounding, exact scaling
        }
      }
      continue;
    }
    // T = Q - 2 sum(bit * q) for rows g, g + 8 and columns 2c, 2c + 1 of each N tile
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nt * 8 + 2 * c + (e & 1);
        int bits;
        if constexpr (CLASS) {
          bits = -(acc[7][nt][e] >> 7);
#pragma unroll
          for (int s = 0; s < 7; ++s) bits += acc[s][nt][e] >> s;
        } else {
          bits = acc[0][nt][e];
        }
        const int row = g + 8 * (e >> 1);
        T[row * NCOL + col] = qcol[nt][e & 1] - 2 * bits;
      }
    }
    __syncwarp();
    for (int idx = lane; idx < 16 * batch; idx += 32) {
      const int row = idx & 15, tok = idx >> 4;
      const int* tr = T + row * NCOL + 3 * tok;
      // exact in fp64 (|v| < 2^53), one rounding to fp32, exact power-of-two scaling
      const double v = fma(static_cast<double>(tr[2]), 65536.0, fma(static_cast<double>(tr[1]), 256.0, tr[0]));
      out[tok * ld_out + t * 16 + row] = __double2float_rn(v) * pow2f(-exps[tok]);
    }
    __syncwarp();
  }
}

template <int NTILE, bool CLASS, bool OUT_F32>
__global__ void __launch_bounds__(kFThreads, 2) dbf_decode_fused_kernel(const __grid_constant__ FusedArgs p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const FusedSmem L = fused_smem_layout(p, NTILE);
  uint64_t* bar1 = reinterpret_cast<uint64_t*>(smem);      // reduce-scatter parts landed
  uint64_t* bar2 = reinterpret_cast<uint64_t*>(smem + 8);  // all-gather of V landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 16);
  int* exps = reinterpret_cast<int*>(smem + 64);      // [16]
  float* redmax = reinterpret_cast<float*>(smem + 128);  // [16 tokens][8 warps]
  int* Q = reinterpret_cast<int*>(smem + 640);         // [48]: digit sums of the MMA columns
  uint8_t* wB = smem + L.wB;
  uint8_t* wA = smem + L.wA;
  uint8_t* dig = smem + L.dig;
  float* U = reinterpret_cast<float*>(smem + L.U);
  int* Tb = reinterpret_cast<int*>(smem + L.Tb);
  float* part = reinterpret_cast<float*>(smem + L.part);  // partial t, then V: [tok][kb]
  float* red = reinterpret_cast<float*>(smem + L.red);    // [R][tok][vb] parts of this rank's rows
  float* zb = reinterpret_cast<float*>(smem + L.z);       // [tok][nb] partial of y

  const int tid = threadIdx.x;
  const int R = p.R;
  const int r = R > 1 ? static_cast<int>(cluster_rank()) : 0;
  const int j = static_cast<int>(blockIdx.y);
  const int batch = p.batch;
  const int vb = p.kb / R;

  // this CTA's share
  const int kl0 = j * p.kb;
  const int kbj = min(p.k, kl0 + p.kb) - kl0;  // middle rows of the slice
  const int bB0 = r * p.MB / R, bB1 = (r + 1) * p.MB / R;
  const int nblkB = bB1 - bB0;
  const int colsB = nblkB * 256;
  const int i0 = r * p.nb;
  const int rowsA = max(0, min(p.n, i0 + p.nb) - i0);
  const int nblkA = (kbj + 255) >> 8;
  const int tilesB = (kbj + 15) >> 4;
  const int tilesA = (rowsA + 15) >> 4;
  const bool one_round = fused_one_round(p);
  // bytes each exchange round brings into this CTA
  const uint32_t xbytes = static_cast<uint32_t>((R - 1) * batch * (one_round ? p.kb : vb) * 4);

  if (tid == 0) {
    mbar_init(bar1, 1);
    mbar_init(bar2, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (R > 1) {
    if (tid == 0) {
      mbar_arrive_expect_tx(bar1, xbytes + (p.test_lose_bytes && r == 0 ? 16u : 0u));
      if (!one_round) mbar_arrive_expect_tx(bar2, xbytes);
    }
    cluster_arrive_relaxed();  // peers may send only after this CTA's barriers exist (matching wait below)
  }
  // The next kernel in the stream may start its own prologue now: it cannot
  // read anything this one writes before this grid has completed.
  pdl_launch_dependents();

  // ---- weights: every 16-byte chunk of this CTA's B and A tiles into shared memory
  // (weights that cannot depend on earlier work in the stream are requested
  // before waiting for it, so that they stream in while that work finishes)
  if (!p.weights_early) pdl_wait();
  {
    const int chB = tilesB * nblkB * 32;
    const int chA = tilesA * nblkA * 32;
#pragma unroll 1
    for (int ch = tid; ch < chB + chA; ch += kFThreads) {
      const bool isB = ch < chB;
      const int cc = isB ? ch : ch - chB;
      const int item = cc >> 5, part16 = cc & 31;
      const int row = part16 >> 1, half = part16 & 1;
      const int nblk = isB ? nblkB : nblkA;
      const int t = item / nblk, q = item - t * nblk;
      if (isB) {
        const int gr = kl0 + t * 16 + row;
        const bool ok = t * 16 + row < kbj;
        const uint32_t* src = p.packedB + (ok ? static_cast<int64_t>(gr) * p.wprB + (bB0 + q) * 8 + half * 4 : 0);
        cp_async16(wB + item * 512 + row * 32 + half * 16, src, ok);
      } else {
        const int gr = i0 + t * 16 + row;
        const bool ok = t * 16 + row < rowsA;
        const uint32_t* src =
            p.packedA + (ok ? static_cast<int64_t>(gr) * p.wprA + ((kl0 >> 8) + q) * 8 + half * 4 : 0);
        cp_async16(wA + item * 512 + row * 32 + half * 16, src, ok);
      }
    }
    cp_async_commit();
  }
  if (p.weights_early) pdl_wait();

  // ---- u = x (.) b over this rank's m_in columns, fp32 (exact product of two fp16);
  // 8 columns per thread and load, every thread at once
  {
    const int nvec = colsB / 8;
    for (int idx = tid; idx < batch * nvec; idx += kFThreads) {
      const int tok = idx / nvec, v = idx - tok * nvec;
      const int gc = bB0 * 256 + v * 8;  // m_in is a multiple of 64: all 8 columns are in or out together
      float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
      if (gc < p.m_in) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(tok) * p.ld_x + gc));
        const uint4 bv = __ldg(reinterpret_cast<const uint4*>(p.b + gc));
        const __half2* xh = reinterpret_cast<const __half2*>(&xv);
        const __half2* bh = reinterpret_cast<const __half2*>(&bv);
        const float2 x0 = __half22float2(xh[0]), x1 = __half22float2(xh[1]), x2 = __half22float2(xh[2]),
                     x3 = __half22float2(xh[3]);
        const float2 b0 = __half22float2(bh[0]), b1 = __half22float2(bh[1]), b2 = __half22float2(bh[2]),
                     b3 = __half22float2(bh[3]);
        lo = make_float4(x0.x * b0.x, x0.y * b0.y, x1.x * b1.x, x1.y * b1.y);
        hi = make_float4(x2.x * b2.x, x2.y * b2.y, x3.x * b3.x, x3.y * b3.y);
      }
      float4* dst = reinterpret_cast<float4*>(U + tok * colsB + v * 8);
      dst[0] = lo;
      dst[1] = hi;
    }
  }
  __syncthreads();
  build_digits<NTILE>(U, colsB, batch, dig, exps, Q, redmax);
  cp_async_wait_all();
  __syncthreads();

  // ---- first product: partial t of the slice's rows over this rank's columns
  sign_product<NTILE, CLASS>(wB, tilesB, nblkB, dig, exps, Q, batch, Tb, part, p.kb);
  __syncthreads();

  // ---- V = mid (.) t for the slice, assembled in every rank of the cluster and
  // written (zero past the slice's rows) as the input of the second product
  const int colsA = nblkA * 256;
  bool ok = true;
  if (R > 1) {
    cluster_wait_acquire();  // matches the arrive above: every peer's barriers are initialised
    if (one_round) {
      // every peer gets this rank's partial sums of all kb rows
      const int nv4 = batch * p.kb / 4;
#pragma unroll 1
      for (int r2 = 0; r2 < R; ++r2) {
        if (r2 == r) continue;
        const uint32_t peer_bar = map_to_rank(bar1, r2);
        const uint32_t peer_red = map_to_rank(red + r * batch * p.kb, r2);
#pragma unroll 1
        for (int v4 = tid; v4 < nv4; v4 += kFThreads)
          st_async_v4(peer_red + 16u * v4, reinterpret_cast<const float4*>(part)[v4], peer_bar);
      }
      ok = __syncthreads_and(mbar_wait_cluster_bounded(bar1, 0, p.status));
      if (!ok) return;
#pragma unroll 1
      for (int idx = tid; idx < batch * colsA; idx += kFThreads) {
        const int tok = idx / colsA, col = idx - tok * colsA;
        float v = 0.f;
        if (col < kbj) {
          float t = 0.f;
#pragma unroll 1
          for (int r2 = 0; r2 < R; ++r2)  // rank order: the same sum on every rank
            t += (r2 == r ? part : red + r2 * batch * p.kb)[tok * p.kb + col];
          v = t * __half2float(p.mid[kl0 + col]);
        }
        U[idx] = v;
      }
    } else {
      // reduce-scatter: rank r2 gets this rank's part of its vb rows
      const int nv4 = vb / 4;
#pragma unroll 1
      for (int idx = tid; idx < (R - 1) * batch * nv4; idx += kFThreads) {
        const int peer_i = idx / (batch * nv4);
        const int rem = idx - peer_i * batch * nv4;
        const int tok = rem / nv4, v4 = rem - tok * nv4;
        const int r2 = peer_i < r ? peer_i : peer_i + 1;
        const float4 v = *reinterpret_cast<const float4*>(part + tok * p.kb + r2 * vb + v4 * 4);
        float* dst = red + (r * batch + tok) * vb + v4 * 4;
        st_async_v4(map_to_rank(dst, r2), v, map_to_rank(bar1, r2));
      }
      ok = __syncthreads_and(mbar_wait_cluster_bounded(bar1, 0, p.status));
      if (!ok) return;
      // this rank's rows: add the R parts in rank order, scale by mid, send to every peer
#pragma unroll 1
      for (int idx = tid; idx < batch * nv4; idx += kFThreads) {
        const int tok = idx / nv4, v4 = idx - tok * nv4;
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
        for (int r2 = 0; r2 < R; ++r2) {
          const float4 v = r2 == r ? *reinterpret_cast<const float4*>(part + tok * p.kb + r * vb + v4 * 4)
                                   : *reinterpret_cast<const float4*>(red + (r2 * batch + tok) * vb + v4 * 4);
          sum.x += v.x;
          sum.y += v.y;
          sum.z += v.z;
          sum.w += v.w;
        }
        const int l0 = r * vb + v4 * 4;  // row within the slice
        float4 vv;
        vv.x = l0 + 0 < kbj ? sum.x * __half2float(p.mid[kl0 + l0 + 0]) : 0.f;
        vv.y = l0 + 1 < kbj ? sum.y * __half2float(p.mid[kl0 + l0 + 1]) : 0.f;
        vv.z = l0 + 2 < kbj ? sum.z * __half2float(p.mid[kl0 + l0 + 2]) : 0.f;
        vv.w = l0 + 3 < kbj ? sum.w * __half2float(p.mid[kl0 + l0 + 3]) : 0.f;
        float* own = part + tok * p.kb + l0;
        *reinterpret_cast<float4*>(own) = vv;
#pragma unroll 1
        for (int r2 = 0; r2 < R; ++r2)
          if (r2 != r) st_async_v4(map_to_rank(own, r2), vv, map_to_rank(bar2, r2));
      }
      ok = __syncthreads_and(mbar_wait_cluster_bounded(bar2, 0, p.status));
      if (!ok) return;
#pragma unroll 1
      for (int idx = tid; idx < batch * colsA; idx += kFThreads) {
        const int tok = idx / colsA, col = idx - tok * colsA;
        U[idx] = col < kbj ? part[tok * p.kb + col] : 0.f;
      }
    }
  } else {
#pragma unroll 1
    for (int idx = tid; idx < batch * colsA; idx += kFThreads) {
      const int tok = idx / colsA, col = idx - tok * colsA;
      U[idx] = col < kbj ? part[tok * p.kb + col] * __half2float(p.mid[kl0 + col]) : 0.f;
    }
  }
  __syncthreads();

  // ---- second product: partial z of this rank's output rows over the slice
  if (tilesA > 0) {
    build_digits<NTILE>(U, colsA, batch, dig, exps, Q, redmax);
    __syncthreads();
    sign_product<NTILE, CLASS>(wA, tilesA, nblkA, dig, exps, Q, batch, Tb, zb, p.nb);
  }
  __syncthreads();
  if (rowsA == 0) return;

  // ---- y: cluster 0 adds the other clusters' partials of its rows (cluster order).
  // Slot words: [tok][row][8], word j - 1 from cluster j; the high half of a word
  // is 1 once written, so a row's partials arrive with the loads that wait for them.
  const int n = p.n;
  if (j > 0) {
    for (int idx = tid; idx < batch * rowsA; idx += kFThreads) {
      const int tok = idx / rowsA, rl = idx - tok * rowsA;
      const unsigned long long w =
          (1ull << 32) | static_cast<unsigned long long>(__float_as_uint(zb[tok * p.nb + rl]));
      st_relaxed_u64(p.slots + (static_cast<int64_t>(tok) * n + i0 + rl) * 8 + (j - 1), w);
    }
    return;
  }
  const unsigned long long t0 = globaltimer_ns();
  const int nw = p.J - 1;
  const int items = batch * rowsA;
  constexpr int kItems = 4;  // rows a thread waits for at once
  for (int base = tid; base < items && ok; base += kItems * kFThreads) {
    unsigned long long w[kItems][8];
    uint32_t missing[kItems];
#pragma unroll
    for (int u = 0; u < kItems; ++u) missing[u] = base + u * kFThreads < items ? (1u << nw) - 1u : 0u;
    for (uint32_t it = 0;; ++it) {
      bool pending = false;
#pragma unroll
      for (int u = 0; u < kItems; ++u) {
        if (missing[u] == 0) continue;
        const int idx = base + u * kFThreads;
        const int tok = idx / rowsA, rl = idx - tok * rowsA;
        const unsigned long long* sp = p.slots + (static_cast<int64_t>(tok) * n + i0 + rl) * 8;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (missing[u] & (3u << (2 * q))) ld_relaxed_u64x2(sp + 2 * q, w[u][2 * q], w[u][2 * q + 1]);
      }
#pragma unroll
      for (int u = 0; u < kItems; ++u) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if ((missing[u] >> q & 1u) && (w[u][q] >> 32) == 1ull) missing[u] &= ~(1u << q);
        pending |= missing[u] != 0;
      }
      if (!pending) break;
      if ((it & 15u) == 15u && (*abort_flag || globaltimer_ns() - t0 > kWaitBudgetNs)) {
        if (!*abort_flag) {
          *abort_flag = 1;
          atomicCAS(p.status, 0, kStatusTimeout);
        }
        ok = false;
        break;
      }
    }
    if (!ok) break;
#pragma unroll
    for (int u = 0; u < kItems; ++u) {
      const int idx = base + u * kFThreads;
      if (idx >= items) continue;
      const int tok = idx / rowsA, rl = idx - tok * rowsA;
      const int i = i0 + rl;
      float acc = zb[tok * p.nb + rl];
#pragma unroll
      for (int q = 0; q < kFusedMaxSlices - 1; ++q)
        if (q < nw) acc += __uint_as_float(static_cast<uint32_t>(w[u][q]));
      // consumed: the next forward on this workspace starts from empty slots
      unsigned long long* sp = p.slots + (static_cast<int64_t>(tok) * n + i) * 8;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (2 * q < nw) st_relaxed_u64x2(sp + 2 * q, 0ull, 0ull);
      const float v = acc * __half2float(p.a[i]);
      if constexpr (OUT_F32) {
        static_cast<float*>(p.y)[static_cast<int64_t>(tok) * p.ld_y + i] = v;
      } else {
        static_cast<__half*>(p.y)[static_cast<int64_t>(tok) * p.ld_y + i] = __float2half_rn(v);
      }
    }
  }
}

template <int NTILE, bool CLASS, bool OUT_F32>
dbf_status launch_fused_typed(const FusedArgs& a, size_t smem, cudaStream_t stream) {
  auto kernel = dbf_decode_fused_kernel<NTILE, CLASS, OUT_F32>;
  // attributes once per instantiation (the maximum this path ever asks for)
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmemBudget);
    if (attr_err == cudaSuccess) attr_err = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  });
  if (attr_err != cudaSuccess) return DBF_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.R), static_cast<unsigned>(a.J), 1);
  cfg.blockDim = dim3(kFThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = static_cast<unsigned>(a.R);
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, a) == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

template <bool OUT_F32>
dbf_status launch_fused_out(const FusedArgs& a, int ntile, size_t smem, cudaStream_t stream) {
  switch (ntile) {
    case 1: return launch_fused_typed<1, true, OUT_F32>(a, smem, stream);
    case 2: return launch_fused_typed<2, true, OUT_F32>(a, smem, stream);
    case 3: return launch_fused_typed<3, false, OUT_F32>(a, smem, stream);
    case 4: return launch_fused_typed<4, false, OUT_F32>(a, smem, stream);
    case 5: return launch_fused_typed<5, false, OUT_F32>(a, smem, stream);
    case 6: return launch_fused_typed<6, false, OUT_F32>(a, smem, stream);
  }
  return DBF_ERR_INVALID_ARG;
}

}  // namespace

// Cluster and slice sizes (see the top of this file).  R: the largest power of
// two <= min(16, m_in blocks), so every rank has at least one 256-column block
// of B and kb / R rows of V; kb: the smallest multiple of 256 that cuts k into
// at most kFusedMaxSlices slices; nb: the output rows of a rank, a multiple of 16.
bool plan_fused(int64_t n, int64_t k, int64_t m_in, int batch, FusedArgs* out, size_t* smem_bytes) {
  if (batch < 1 || batch > kMaxTok) return false;
  FusedArgs a{};
  a.n = static_cast<int>(n);
  a.k = static_cast<int>(k);
  a.m_in = static_cast<int>(m_in);
  a.batch = batch;
  a.MB = static_cast<int>((m_in + 255) / 256);
  int R = 1;
  while (R * 2 <= 16 && R * 2 <= a.MB) R *= 2;
  a.R = R;
  int64_t kb = (k + 256 * kFusedMaxSlices - 1) / (256 * kFusedMaxSlices) * 256;
  if (kb < 256) kb = 256;
  a.kb = static_cast<int>(kb);
  a.J = static_cast<int>((k + kb - 1) / kb);
  const int64_t nb = ((n + R - 1) / R + 15) / 16 * 16;
  a.nb = static_cast<int>(nb);
  const int ntile = (3 * batch + 7) / 8;
  const FusedSmem L = fused_smem_layout(a, ntile);
  if (L.total > kFusedSmemBudget) return false;
  *out = a;
  *smem_bytes = static_cast<size_t>(L.total);
  return true;
}

dbf_status launch_fused_decode(const FusedArgs& a, size_t smem, bool out_f32, cudaStream_t stream) {
  const int ntile = (3 * a.batch + 7) / 8;
  return out_f32 ? launch_fused_out<true>(a, ntile, smem, stream) : launch_fused_out<false>(a, ntile, smem, stream);
}

}  // namespace dbf
