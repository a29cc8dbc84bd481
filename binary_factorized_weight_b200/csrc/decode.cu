// Decode path (batch <= 16): one sign-product stage per launch.
//
// "Addition is almost all you need" (gist.science technical summary, section
// 2.1, computation process) evaluates X W^T as two products with +-1 matrices,
// (X (.) b^T) B^T and (. (.) m^T) A^T, each made of additions and sign flips.
// This kernel is one such product for a handful of tokens:
//
//   out[tok][row] = rowscale[row] * sum_K sign(row, K) * u[tok][K]
//
// Stage B: rows = k, K = m_in, u = fp16(x (.) b), rowscale = mid, out = V.
// Stage A: rows = n, K = k,    u = V,             rowscale = a,   out = y.
//
// Mapping onto the GPU.  The signs are the M operand of the legacy warp MMA
// (mma.sync m16n8k16, fp16 operands, fp32 accumulators); the tokens are its N
// operand (8 or 16 columns).  Each warp owns a 16-row tile and each CTA four of
// them (64 rows), so the activation chunk a CTA stages in shared memory is
// shared by 64 rows.  Long reductions are split over the CTAs of a thread-
// block cluster (up to 8 along K) whose partial sums meet in rank 0's shared
// memory through DSMEM and are added in rank order (deterministic).
//
// Sign operands never touch shared memory: each thread loads its own packed
// words straight from global memory (all of them for the first piece, before
// the programmatic-dependent-launch wait when that is allowed) and forms the
// fp16 fragments in registers.  For a 256-element block of one row, word h
// (elements 32h..32h+31) holds element pair (32h + 2s, 32h + 2s + 1) at bits
// (s, s+16).  MMA step s (s = 0..15) of the block feeds the 8 pairs {(h, s)}
// of each row as its 16 k values, so every A register of step s comes from one
// word and one bit pair.  Two ways to form the fp16 pair:
//   shift  ((w << (15 - s)) & 0x80008000) | 0x3C003C00  -> (+-1, +-1);
//   class  w & (1 << s | 1 << (s+16))                   -> (0 or c_s, 0 or c_s)
//          with c_s the fp16 value of bit s alone (a power of two), and
//          (w & 0x80008000) | 0x3C003C00 for s = 15.
// In class form, step s accumulates c_s * sum(set-bit activations) into its
// own accumulator set, and the epilogue recovers
//   t = D_15 + sum_{s<15} (U_s - 2 D_s / c_s),
// U_s being the plain sum of the class-s activations.  That halves the ALU
// work per sign.  Both forms are exact on integer data.
#include <cooperative_groups.h>

#include <algorithm>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace cg = cooperative_groups;

namespace dbf {
namespace {

constexpr int kDecThreads = 128;
constexpr int kRowsPerCta = 64;  // 4 warps x 16-row MMA tiles
constexpr int kPieceBlocks = 8;  // 256-element blocks staged per piece
constexpr int kPieceElems = kPieceBlocks * 256;
// Token row stride in shared memory, in 32-bit words (fp16 pairs): one piece
// of pairs plus 8 words, so the 8-byte fragment loads of a half warp hit 32
// distinct banks.
constexpr int kActStride = kPieceElems / 2 + 8;
constexpr int kMaxClusterK = 8;

// 1 / c_s for the class form: c_s is the fp16 value with only bit s set.
__device__ __forceinline__ constexpr float inv_class_scale(int s) {
  // s < 10: subnormal 2^(s-24); s in 10..14: exponent field 2^(s-10) -> 2^(2^(s-10)-15)
  return s == 0   ? 16777216.0f
         : s == 1 ? 8388608.0f
         : s == 2 ? 4194304.0f
         : s == 3 ? 2097152.0f
         : s == 4 ? 1048576.0f
         : s == 5 ? 524288.0f
         : s == 6 ? 262144.0f
         : s == 7 ? 131072.0f
         : s == 8 ? 65536.0f
         : s == 9 ? 32768.0f
         : s == 10 ? 16384.0f
         : s == 11 ? 8192.0f
         : s == 12 ? 2048.0f
         : s == 13 ? 128.0f
                   : 0.5f;
}

// fp16 pair for MMA step s of a block from packed word w (s is a compile-time
// constant after unrolling, so this folds to one LOP3, or SHF + LOP3).
template <bool CLASS>
__device__ __forceinline__ uint32_t form_pair(uint32_t w, int s) {
  if (CLASS) {
    if (s == 15) return (w & 0x80008000u) | 0x3C003C00u;
    return w & ((1u << s) | (1u << (s + 16)));
  }
  return ((w << (15 - s)) & 0x80008000u) | 0x3C003C00u;
}

template <int NT, bool CLASS, bool KSCALE, bool OUT_F32>
__global__ void __launch_bounds__(kDecThreads) dbf_decode_stage_kernel(const DecodeArgs p) {
  constexpr int NTOK = NT * 8;
  constexpr int NACC = CLASS ? 16 : 4;
  extern __shared__ __align__(16) uint32_t smem[];
  uint32_t* act_s = smem;                                              // NTOK x kActStride
  float* urest_s = reinterpret_cast<float*>(act_s + NTOK * kActStride);  // NTOK
  float* red_s = urest_s + 16;                                          // ks x NTOK x 64

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int ks = static_cast<int>(cluster.num_blocks());

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int m0 = blockIdx.x * kRowsPerCta;
  const int row0 = m0 + warp * 16 + g;
  const int k_lo = rank * p.kchunk;
  const int k_hi = min(p.K, k_lo + p.kchunk);

  const bool r0ok = row0 < p.M;
  const bool r8ok = row0 + 8 < p.M;
  const uint32_t* w_lo = p.packed + static_cast<int64_t>(r0ok ? row0 : 0) * p.wpr;
  const uint32_t* w_hi = p.packed + static_cast<int64_t>(r8ok ? row0 + 8 : 0) * p.wpr;

  float acc[NACC][NT][4];
#pragma unroll
  for (int i = 0; i < NACC; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  uint32_t w[kPieceBlocks][4];
  auto load_weights = [&](int k0, int nblk) {
#pragma unroll
    for (int b = 0; b < kPieceBlocks; ++b) {
      const int64_t word = (k0 >> 5) + b * 8 + c;
      const bool in_b = b < nblk;
      w[b][0] = (in_b && r0ok && word < p.wpr) ? __ldg(w_lo + word) : 0u;
      w[b][1] = (in_b && r8ok && word < p.wpr) ? __ldg(w_hi + word) : 0u;
      w[b][2] = (in_b && r0ok && word + 4 < p.wpr) ? __ldg(w_lo + word + 4) : 0u;
      w[b][3] = (in_b && r8ok && word + 4 < p.wpr) ? __ldg(w_hi + word + 4) : 0u;
    }
  };

  int k0 = k_lo;
  int piece_end = min(k_hi, k0 + kPieceElems);
  int nblk = (piece_end - k0 + 255) >> 8;

  // Weights never depend on the previous kernel when the caller says so (or,
  // for stage A, because stage B only releases its dependents after its own
  // wait): stream them in before waiting for the activations.
  if (p.weights_early) load_weights(k0, nblk);
  pdl_wait();
  pdl_launch_dependents();
  if (!p.weights_early) load_weights(k0, nblk);

  if (tid < 16) urest_s[tid] = 0.f;

  for (;;) {
    // ---- stage this piece of activations (u) in the permuted pair order
    const int npairs = nblk * 128;
    for (int idx = tid; idx < NTOK * npairs; idx += kDecThreads) {
      const int tok = idx / npairs;
      const int P = idx - tok * npairs;
      const int kk = k0 + 2 * P;
      uint32_t u = 0u;
      if (tok < p.batch && kk < k_hi) {
        __half2 x2 = *reinterpret_cast<const __half2*>(p.act + static_cast<int64_t>(tok) * p.ld_act + kk);
        if constexpr (KSCALE) x2 = __hmul2(x2, __ldg(reinterpret_cast<const __half2*>(p.kscale + kk)));
        u = *reinterpret_cast<uint32_t*>(&x2);
      }
      const int blk = P >> 7, hp = P & 127, h = hp >> 4, s = hp & 15;
      act_s[tok * kActStride + blk * 128 + s * 8 + 2 * (h & 3) + (h >> 2)] = u;
    }
    __syncthreads();

    if constexpr (CLASS) {
      // U_rest[tok] += sum of the piece's activations outside class 15
      for (int tok = warp; tok < NTOK; tok += 4) {
        float sum = 0.f;
        for (int sl = lane; sl < npairs; sl += 32) {
          if (((sl & 127) >> 3) != 15) {
            const __half2 u = *reinterpret_cast<const __half2*>(act_s + tok * kActStride + sl);
            sum += __low2float(u) + __high2float(u);
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) urest_s[tok] += sum;
      }
    }

    // ---- sign products
#pragma unroll
    for (int b = 0; b < kPieceBlocks; ++b) {
      if (b < nblk) {
        const uint32_t* ab = act_s + b * 128 + 2 * c;
#pragma unroll
        for (int s = 0; s < 16; ++s) {
          const uint32_t a0 = form_pair<CLASS>(w[b][0], s);
          const uint32_t a1 = form_pair<CLASS>(w[b][1], s);
          const uint32_t a2 = form_pair<CLASS>(w[b][2], s);
          const uint32_t a3 = form_pair<CLASS>(w[b][3], s);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint2 bb = *reinterpret_cast<const uint2*>(ab + (nt * 8 + g) * kActStride + s * 8);
            mma_m16n8k16(acc[CLASS ? s : (s & 3)][nt], a0, a1, a2, a3, bb.x, bb.y);
          }
        }
      }
    }
    __syncthreads();  // act_s is rewritten by the next piece; urest_s read below

    k0 = piece_end;
    if (k0 >= k_hi) break;
    piece_end = min(k_hi, k0 + kPieceElems);
    nblk = (piece_end - k0 + 255) >> 8;
    load_weights(k0, nblk);
  }

  // ---- combine accumulators into this CTA's partial t and hand it to rank 0
  float* red0 = cluster.map_shared_rank(red_s, 0);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = nt * 8 + 2 * c + (e & 1);
      float t;
      if constexpr (CLASS) {
        float corr = 0.f;
#pragma unroll
        for (int s = 0; s < 15; ++s) corr = fmaf(acc[s][nt][e], inv_class_scale(s), corr);
        t = acc[15][nt][e] + urest_s[tok] - 2.f * corr;
      } else {
        t = (acc[0][nt][e] + acc[1][nt][e]) + (acc[2][nt][e] + acc[3][nt][e]);
      }
      const int rl = warp * 16 + g + 8 * (e >> 1);
      red0[(rank * NTOK + tok) * kRowsPerCta + rl] = t;
    }
  }
  cluster.sync();

  if (rank == 0) {
    for (int idx = tid; idx < p.batch * kRowsPerCta; idx += kDecThreads) {
      const int tok = idx >> 6, rl = idx & 63;
      const int row = m0 + rl;
      if (row < p.M) {
        float t = 0.f;
        for (int q = 0; q < ks; ++q) t += red_s[(q * NTOK + tok) * kRowsPerCta + rl];
        const float v = t * __half2float(p.rowscale[row]);
        if constexpr (OUT_F32) {
          static_cast<float*>(p.out)[static_cast<int64_t>(tok) * p.ld_out + row] = v;
        } else {
          static_cast<__half*>(p.out)[static_cast<int64_t>(tok) * p.ld_out + row] = __float2half_rn(v);
        }
      }
    }
  }
}

template <int NT, bool CLASS, bool KSCALE, bool OUT_F32>
dbf_status launch_typed(const DecodeArgs& a, int ks, cudaStream_t stream) {
  auto kernel = dbf_decode_stage_kernel<NT, CLASS, KSCALE, OUT_F32>;
  const size_t smem = (static_cast<size_t>(NT * 8) * kActStride + 16 + static_cast<size_t>(ks) * NT * 8 * kRowsPerCta) *
                      sizeof(uint32_t);
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return DBF_ERR_CUDA;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((a.M + kRowsPerCta - 1) / kRowsPerCta), static_cast<unsigned>(ks), 1);
  cfg.blockDim = dim3(kDecThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = 1;
  attrs[0].val.clusterDim.y = static_cast<unsigned>(ks);
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  err = cudaLaunchKernelEx(&cfg, kernel, a);
  return err == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

}  // namespace

dbf_status launch_decode_stage(const DecodeArgs& args_in, bool class_expand, bool out_f32, const DeviceInfo& dev,
                               cudaStream_t stream) {
  DecodeArgs a = args_in;
  // K split: aim for about two CTAs per SM, at most one cluster of 8 along K.
  const int64_t tiles = (a.M + kRowsPerCta - 1) / kRowsPerCta;
  const int64_t target = 2 * static_cast<int64_t>(dev.num_sms);
  int ks = static_cast<int>(std::min<int64_t>(kMaxClusterK, std::max<int64_t>(1, (target + tiles - 1) / tiles)));
  int64_t kchunk = (a.K + ks - 1) / ks;
  kchunk = (kchunk + 255) / 256 * 256;
  ks = static_cast<int>((a.K + kchunk - 1) / kchunk);
  a.kchunk = static_cast<int>(kchunk);

  const bool nt2 = a.batch > 8;
  const bool kscale = a.kscale != nullptr;
#define DBF_DISPATCH(NT, CL)                                                   \
  if (kscale) {                                                                \
    return out_f32 ? launch_typed<NT, CL, true, true>(a, ks, stream)           \
                   : launch_typed<NT, CL, true, false>(a, ks, stream);         \
  } else {                                                                     \
    return out_f32 ? launch_typed<NT, CL, false, true>(a, ks, stream)          \
                   : launch_typed<NT, CL, false, false>(a, ks, stream);        \
  }
  if (nt2) {
    if (class_expand) {
      DBF_DISPATCH(2, true)
    } else {
      DBF_DISPATCH(2, false)
    }
  } else {
    if (class_expand) {
      DBF_DISPATCH(1, true)
    } else {
      DBF_DISPATCH(1, false)
    }
  }
#undef DBF_DISPATCH
}

}  // namespace dbf
