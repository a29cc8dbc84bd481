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
// them (64 rows), so the activation range a CTA stages in shared memory serves
// 64 rows.  Long reductions are split over the CTAs of a thread-block cluster
// (up to 8 along K); their partial sums meet in rank 0's shared memory through
// DSMEM and are added in rank order (deterministic).
//
// Data movement.  Each thread streams its own packed words from global memory
// into registers, 4 blocks at a time with the next 4 in flight (the first
// group before the programmatic-dependent-launch wait whenever the weights
// cannot depend on the previous kernel).  One thread brings the CTA's
// activation rows (and b) into shared memory with bulk asynchronous copies on
// an mbarrier; a vectorised pass then applies b and forms the class sums.
//
// Sign operands.  In the packed layout word p of a 256-column block holds the
// column pair (16g + 2p, 16g + 2p + 1) at bits (g, g+16) for each group g.
// MMA step s of a block is group s (16 consecutive columns, in natural order),
// so every A register of step s is bit pair s of one word:
//   shift  ((w << (15 - s)) & 0x80008000) | 0x3C003C00  -> (+-1, +-1);
//   class  w & (1 << s | 1 << (s+16))                   -> (0 or c_s, 0 or c_s)
//          with c_s the fp16 value of bit s alone (a power of two), and
//          (w & 0x80008000) | 0x3C003C00 for s = 15.
// In class form, step s accumulates c_s * sum(set-bit activations) into its
// own accumulator set and the epilogue recovers
//   t = D_15 + sum_{s<15} (U_s - 2 D_s / c_s),
// U_s being the plain sum of the class-s activations.  One LOP3 per fp16 pair
// instead of two instructions.  Both forms are exact on integer data.
#include <cooperative_groups.h>

#include <algorithm>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace cg = cooperative_groups;

namespace dbf {
namespace {

constexpr int kDecThreads = 128;
constexpr int kRowsPerCta = 64;  // 4 warps x 16-row MMA tiles
constexpr int kGroupBlocks = 4;  // 256-column blocks per register group of weights
constexpr int kMaxClusterK = 8;
constexpr int kSmemBudget = 100 * 1024;
constexpr int kHeadBytes = 128;  // mbarrier, abort flag, class sums

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

// Shared-memory layout of one CTA (host and device agree on it).
struct DecSmem {
  int piece;       // activation columns staged per piece (multiple of 1024)
  int stride;      // words per staged token row: piece/2 + 8 (= 8 mod 32)
  int act_off;     // byte offsets
  int zero_off;
  int b_off;
  int red_off;
  int total;
};

__host__ __device__ inline DecSmem dec_smem_layout(int piece, int nvalid, int ntok, int ks) {
  DecSmem l;
  l.piece = piece;
  l.stride = piece / 2 + 8;
  l.act_off = kHeadBytes;
  l.zero_off = l.act_off + nvalid * l.stride * 4;
  l.b_off = l.zero_off + l.stride * 4;
  l.red_off = l.b_off + piece * 2;
  l.total = l.red_off + ks * ntok * kRowsPerCta * 4;
  return l;
}

template <int NT, bool CLASS, bool KSCALE, bool OUT_F32>
__global__ void __launch_bounds__(kDecThreads) dbf_decode_stage_kernel(const DecodeArgs p, const int piece) {
  constexpr int NTOK = NT * 8;
  constexpr int NACC = CLASS ? 16 : 4;
  constexpr int D = kGroupBlocks;
  extern __shared__ __align__(128) uint8_t smem[];

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int ks = static_cast<int>(cluster.num_blocks());
  const int nvalid = min(p.batch, NTOK);
  const DecSmem L = dec_smem_layout(piece, nvalid, NTOK, ks);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 8);
  float* urest_s = reinterpret_cast<float*>(smem + 64);
  uint32_t* act_s = reinterpret_cast<uint32_t*>(smem + L.act_off);
  uint32_t* zero_row = reinterpret_cast<uint32_t*>(smem + L.zero_off);
  __half* b_s = reinterpret_cast<__half*>(smem + L.b_off);
  float* red_s = reinterpret_cast<float*>(smem + L.red_off);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int m0 = blockIdx.x * kRowsPerCta;
  const int row0 = m0 + warp * 16 + g;
  const int k_lo = rank * p.kchunk;
  const int k_hi = min(p.K, k_lo + p.kchunk);
  const int blk_hi = (k_hi + 255) >> 8;

  const bool r0ok = row0 < p.M;
  const bool r8ok = row0 + 8 < p.M;
  // uint2 j of a row = words (2j, 2j+1); this lane reads uint2 (4*blk + c) of rows row0 and row0 + 8
  const uint2* w_lo = reinterpret_cast<const uint2*>(p.packed + static_cast<int64_t>(r0ok ? row0 : 0) * p.wpr);
  const uint2* w_hi = reinterpret_cast<const uint2*>(p.packed + static_cast<int64_t>(r8ok ? row0 + 8 : 0) * p.wpr);

  uint2 wa[D][2], wb[D][2];
  auto load_group = [&](uint2 (&wr)[D][2], int blk0) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const int blk = blk0 + d;
      const bool in = blk < blk_hi;
      wr[d][0] = (in && r0ok) ? __ldg(w_lo + 4 * blk + c) : make_uint2(0u, 0u);
      wr[d][1] = (in && r8ok) ? __ldg(w_hi + 4 * blk + c) : make_uint2(0u, 0u);
    }
  };

  float acc[NACC][NT][4];
#pragma unroll
  for (int i = 0; i < NACC; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  // Weights never depend on the previous kernel when the caller says so (or,
  // for stage A, because stage B releases its dependents only after its own
  // wait): start streaming them before waiting for the activations.
  if (p.weights_early) load_group(wa, k_lo >> 8);
  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (tid < 16) urest_s[tid] = 0.f;
  for (int i = tid; i < L.stride; i += kDecThreads) zero_row[i] = 0u;
  pdl_wait();
  pdl_launch_dependents();
  if (!p.weights_early) load_group(wa, k_lo >> 8);
  __syncthreads();

  const uint32_t* arow[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tok = nt * 8 + g;
    arow[nt] = (tok < nvalid ? act_s + tok * L.stride : zero_row) + 2 * c;
  }

  bool ok = true;
  uint32_t phase = 0;
  for (int pk = k_lo; pk < k_hi && ok; pk += piece) {
    const int pe = min(k_hi, pk + piece);
    const int plen = pe - pk;  // multiple of 64
    // ---- bring the activation rows (and b) of this piece into shared memory
    if (tid == 0) {
      const uint32_t row_bytes = static_cast<uint32_t>(plen) * 2;
      mbar_arrive_expect_tx(bar, row_bytes * static_cast<uint32_t>(nvalid + (KSCALE ? 1 : 0)));
      for (int tok = 0; tok < nvalid; ++tok)
        bulk_load(act_s + tok * L.stride, p.act + static_cast<int64_t>(tok) * p.ld_act + pk, row_bytes, bar);
      if constexpr (KSCALE) bulk_load(b_s, p.kscale + pk, row_bytes, bar);
    }
    ok = mbar_wait_bounded(bar, phase, abort_flag, p.status);
    phase ^= 1u;
    ok = __syncthreads_and(ok);
    if (!ok) break;

    // ---- u = fp16(x (.) b) in place; class sums U_rest (all groups but 15)
    if constexpr (KSCALE || CLASS) {
      for (int tok = warp; tok < nvalid; tok += 4) {
        uint4* rowv = reinterpret_cast<uint4*>(act_s + tok * L.stride);
        float sum = 0.f;
        for (int ch = lane; ch < plen / 8; ch += 32) {
          uint4 v = rowv[ch];
          if constexpr (KSCALE) {
            const uint4 sb = reinterpret_cast<const uint4*>(b_s)[ch];
            __half2* h = reinterpret_cast<__half2*>(&v);
            const __half2* hb = reinterpret_cast<const __half2*>(&sb);
            h[0] = __hmul2(h[0], hb[0]);
            h[1] = __hmul2(h[1], hb[1]);
            h[2] = __hmul2(h[2], hb[2]);
            h[3] = __hmul2(h[3], hb[3]);
            rowv[ch] = v;
          }
          if constexpr (CLASS) {
            if (((ch >> 1) & 15) != 15) {  // 8 columns = half a group; group = (8*ch mod 256)/16
              const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
              for (int q = 0; q < 4; ++q) sum += __low2float(h[q]) + __high2float(h[q]);
            }
          }
        }
        if constexpr (CLASS) {
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
          if (lane == 0) urest_s[tok] += sum;
        }
      }
      __syncthreads();
    }

    // ---- sign products over this piece, weights double-buffered in registers
    const int bend = (pe + 255) >> 8;
    for (int gb = pk >> 8; gb < bend; gb += D) {
      if (gb + D < blk_hi) load_group(wb, gb + D);
#pragma unroll
      for (int d = 0; d < D; ++d) {
        const int blk = gb + d;
        if (blk < bend) {
          const int off = (blk * 256 - pk) >> 1;  // word offset of the block in a staged row
          const int nsteps = min(16, (pe - blk * 256) >> 4);
#pragma unroll
          for (int s = 0; s < 16; ++s) {
            if (s < nsteps) {
              const uint32_t a0 = form_pair<CLASS>(wa[d][0].x, s);
              const uint32_t a2 = form_pair<CLASS>(wa[d][0].y, s);
              const uint32_t a1 = form_pair<CLASS>(wa[d][1].x, s);
              const uint32_t a3 = form_pair<CLASS>(wa[d][1].y, s);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const uint2 bb = *reinterpret_cast<const uint2*>(arow[nt] + off + 8 * s);
                mma_m16n8k16(acc[CLASS ? s : (s & 3)][nt], a0, a1, a2, a3, bb.x, bb.y);
              }
            }
          }
        }
      }
#pragma unroll
      for (int d = 0; d < D; ++d) {
        wa[d][0] = wb[d][0];
        wa[d][1] = wb[d][1];
      }
    }
    __syncthreads();  // the next piece overwrites act_s; urest_s is read below
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

  if (rank == 0 && ok) {
    for (int idx = tid; idx < nvalid * kRowsPerCta; idx += kDecThreads) {
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
dbf_status launch_typed(const DecodeArgs& a, int ks, int piece, cudaStream_t stream) {
  auto kernel = dbf_decode_stage_kernel<NT, CLASS, KSCALE, OUT_F32>;
  const DecSmem L = dec_smem_layout(piece, a.batch < NT * 8 ? a.batch : NT * 8, NT * 8, ks);
  const size_t smem = static_cast<size_t>(L.total);
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
  err = cudaLaunchKernelEx(&cfg, kernel, a, piece);
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
  const int ntok = nt2 ? 16 : 8;
  const int nvalid = a.batch < ntok ? a.batch : ntok;
  // Largest piece (multiple of 1024 columns, at most the chunk) that fits the shared-memory budget.
  int piece = static_cast<int>((kchunk + 1023) / 1024 * 1024);
  while (piece > 1024 && dec_smem_layout(piece, nvalid, ntok, ks).total > kSmemBudget) piece -= 1024;

  const bool kscale = a.kscale != nullptr;
#define DBF_DISPATCH(NT, CL)                                                          \
  if (kscale) {                                                                       \
    return out_f32 ? launch_typed<NT, CL, true, true>(a, ks, piece, stream)           \
                   : launch_typed<NT, CL, true, false>(a, ks, piece, stream);         \
  } else {                                                                            \
    return out_f32 ? launch_typed<NT, CL, false, true>(a, ks, piece, stream)          \
                   : launch_typed<NT, CL, false, false>(a, ks, piece, stream);        \
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
