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
#include <mutex>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace cg = cooperative_groups;

namespace dbf {
namespace {

constexpr int kDecThreads = 128;
// 256-column blocks per register group of weights: 4, or 8 for rows of more
// than 8 blocks per warp in launches of at most 1.75 CTAs per SM (long
// reductions stream their weights; a bigger group keeps more of them in flight
// while the previous group is multiplied)
constexpr int kMaxClusterK = 8;
constexpr int kSmemBudget = 100 * 1024;
constexpr int kMaxDynSmem = 227 * 1024;  // opt-in limit of one CTA on sm_100
constexpr int kHeadBytes = 512;  // mbarriers, abort flag, class sums and their per-warp parts

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
  int piece;     // activation columns staged per piece (multiple of 256)
  int stride;    // words per staged token row: piece/2 + 8 (= 8 mod 32)
  int act_off;   // byte offsets
  int zero_off;
  int b_off;
  int rs_off;    // row scales of the CTA's rows (fp32)
  int red_off;   // partial sums: [ks * KW slots][RT*16 rows][NTOK tokens] fp32
  int total;
};

__host__ __device__ inline DecSmem dec_smem_layout(int piece, int nvalid, int ntok, int ks, int rt) {
  DecSmem l;
  l.piece = piece;
  l.stride = piece / 2 + 8;
  l.act_off = kHeadBytes;
  l.zero_off = l.act_off + nvalid * l.stride * 4;
  l.b_off = l.zero_off + l.stride * 4;
  l.rs_off = l.b_off + piece * 2;
  l.red_off = l.rs_off + 64 * 4;
  l.total = l.red_off + ks * (4 / rt) * (rt * 16) * ntok * 4;
  return l;
}

// One launch computes RT*16 rows per CTA.  Its 4 warps form RT row tiles x
// KW = 4/RT K slices; a cluster of ks CTAs along K splits the reduction further.
// The launch may cover several layers that share their input (a group): the
// CTA's tile index picks its layer.
template <int NT, int RT, int D, bool TOKPAR, bool CLASS, bool KSCALE, bool OUT_F32>
__global__ void __launch_bounds__(kDecThreads, 1)
    dbf_decode_stage_kernel(const __grid_constant__ DecodeGroup grp, const int piece) {
  constexpr int NTOK = NT * 8;
  constexpr int NACC = CLASS ? 16 : 4;
  constexpr int KW = 4 / RT;
  constexpr int ROWS = RT * 16;
  extern __shared__ __align__(128) uint8_t smem[];

  int li = 0;
  while (li + 1 < grp.n && static_cast<int>(blockIdx.x) >= grp.tile_start[li + 1]) ++li;
  const DecodeArgs& p = grp.layer[li];

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int ks = static_cast<int>(cluster.num_blocks());
  const int nvalid = min(p.batch, NTOK);
  const DecSmem L = dec_smem_layout(piece, nvalid, NTOK, ks, RT);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);          // activations of the current piece
  uint64_t* bar_b = reinterpret_cast<uint64_t*>(smem + 16);    // b of the current piece
  uint64_t* bar_red = reinterpret_cast<uint64_t*>(smem + 24);  // rank 0: partial sums of the other ranks landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 8);
  float* urest_s = reinterpret_cast<float*>(smem + 64);        // [16 tokens]
  float* upart_s = reinterpret_cast<float*>(smem + 128);       // [4 warps][16 tokens]
  uint32_t* act_s = reinterpret_cast<uint32_t*>(smem + L.act_off);
  uint32_t* zero_row = reinterpret_cast<uint32_t*>(smem + L.zero_off);
  __half* b_s = reinterpret_cast<__half*>(smem + L.b_off);
  float* rs_s = reinterpret_cast<float*>(smem + L.rs_off);
  float* red_s = reinterpret_cast<float*>(smem + L.red_off);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int rt = warp / KW, kw = warp % KW;
  const int m0 = (static_cast<int>(blockIdx.x) - grp.tile_start[li]) * ROWS;
  const int row0 = m0 + rt * 16 + g;
  const int k_lo = rank * p.kchunk;
  const int k_hi = min(p.K, k_lo + p.kchunk);

  const bool r0ok = row0 < p.M;
  const bool r8ok = row0 + 8 < p.M;
  // uint2 j of a row = words (2j, 2j+1); this lane reads uint2 (4*blk + c) of rows row0 and row0 + 8
  const uint2* w_lo = reinterpret_cast<const uint2*>(p.packed + static_cast<int64_t>(r0ok ? row0 : 0) * p.wpr);
  const uint2* w_hi = reinterpret_cast<const uint2*>(p.packed + static_cast<int64_t>(r8ok ? row0 + 8 : 0) * p.wpr);

  // This warp's blocks of a piece [pk, pe): an even share of the piece's blocks.
  auto slice = [&](int pk, int pe, int& b0, int& b1) {
    const int pb0 = pk >> 8, pb1 = (pe + 255) >> 8;
    const int per = (pb1 - pb0 + KW - 1) / KW;
    b0 = min(pb1, pb0 + kw * per);
    b1 = min(pb1, b0 + per);
  };

  uint2 wa[D][2], wb[D][2];
  auto load_group = [&](uint2 (&wr)[D][2], int blk0, int blk_end) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const int blk = blk0 + d;
      const bool in = blk < blk_end;
      wr[d][0] = (in && r0ok) ? __ldg(w_lo + 4 * blk + c) : make_uint2(0u, 0u);
      wr[d][1] = (in && r8ok) ? __ldg(w_hi + 4 * blk + c) : make_uint2(0u, 0u);
    }
  };
  auto load_static = [&](int pk, int pe) {
    if (tid < ROWS) rs_s[tid] = (m0 + tid < p.M) ? __half2float(p.rowscale[m0 + tid]) : 0.f;
    if constexpr (KSCALE) {
      if (tid == 0 && pe > pk) {
        const uint32_t bytes = static_cast<uint32_t>(pe - pk) * 2;
        mbar_arrive_expect_tx(bar_b, bytes);
        bulk_load(b_s, p.kscale + pk, bytes, bar_b);
      }
    }
  };

  float acc[NACC][NT][4];
#pragma unroll
  for (int i = 0; i < NACC; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar_b, 1);
    mbar_init(bar_red, ks > 1 ? (ks - 1) * kDecThreads : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();  // barriers initialised before anyone can arrive on them
  // Other ranks arrive on rank 0's bar_red at the end; the matching cluster wait
  // is deferred to just before that, so this barrier costs nothing up front.
  if (ks > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  int pk = k_lo;
  int pe = min(k_hi, pk + piece);
  int sb0, sb1;
  slice(pk, pe, sb0, sb1);
  // Weights, b and the row scales never depend on the previous kernel when the
  // caller says so (or, for stage A, because stage B releases its dependents
  // only after its own wait): start loading them before waiting.
  if (p.weights_early) {
    load_group(wa, sb0, sb1);
    load_static(pk, pe);
  }
  if (tid < 16) urest_s[tid] = 0.f;
  for (int i = tid; i < L.stride; i += kDecThreads) zero_row[i] = 0u;
  pdl_wait();
  pdl_launch_dependents();
  if (!p.weights_early) {
    load_group(wa, sb0, sb1);
    load_static(pk, pe);
  }

  const uint32_t* arow[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tok = nt * 8 + g;
    arow[nt] = (tok < nvalid ? act_s + tok * L.stride : zero_row) + 2 * c;
  }

  bool ok = true;
  uint32_t phase = 0;
  // In a group, a layer whose K is shorter than the launch's split may leave a
  // rank without columns; its partial sums are zero.
  const bool has_k = k_lo < k_hi;
  while (has_k) {
    const int plen = pe - pk;  // multiple of 64
    // ---- bring the activation rows of this piece into shared memory
    if (tid == 0) {
      const uint32_t row_bytes = static_cast<uint32_t>(plen) * 2;
      mbar_arrive_expect_tx(bar, row_bytes * static_cast<uint32_t>(nvalid));
      for (int tok = 0; tok < nvalid; ++tok)
        bulk_load(act_s + tok * L.stride, p.act + static_cast<int64_t>(tok) * p.ld_act + pk, row_bytes, bar);
    }
    ok = mbar_wait_bounded(bar, phase, abort_flag, p.status);
    if constexpr (KSCALE) ok = ok && mbar_wait_bounded(bar_b, phase, abort_flag, p.status);
    phase ^= 1u;
    ok = __syncthreads_and(ok);
    if (!ok) break;

    // ---- u = fp16(x (.) b) in place; class sums U_rest (all groups but 15),
    // per-warp parts added in warp order (deterministic).
    // Up to 3 tokens: all 128 threads take each token's row in turn.
    // 4 to 16 tokens: warp w owns tokens w, w+4, w+8, w+12; a thread scales and
    // sums only what it owns, so a warp's tokens run side by side.
    if constexpr (!TOKPAR) {
      if constexpr (KSCALE || CLASS) {
        const int nch = plen / 8;
        for (int tok = 0; tok < nvalid; ++tok) {
          uint4* rowv = reinterpret_cast<uint4*>(act_s + tok * L.stride);
          float sum = 0.f;
          for (int ch = tid; ch < nch; ch += kDecThreads) {
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
            if (lane == 0) upart_s[warp * 16 + tok] = sum;
          }
        }
        __syncthreads();
        if constexpr (CLASS) {
          if (tid < nvalid) urest_s[tid] += (upart_s[tid] + upart_s[16 + tid]) + (upart_s[32 + tid] + upart_s[48 + tid]);
        }
      }
    } else {
      if constexpr (KSCALE || CLASS) {
        const int nch = plen / 8;
        float sum[4] = {0.f, 0.f, 0.f, 0.f};
        for (int ch = lane; ch < nch; ch += 32) {
          const bool rest = ((ch >> 1) & 15) != 15;  // 8 columns = half a group; group = (8*ch mod 256)/16
          uint4 sb = make_uint4(0u, 0u, 0u, 0u);
          if constexpr (KSCALE) sb = reinterpret_cast<const uint4*>(b_s)[ch];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int tok = warp + 4 * j;
            if (tok < nvalid) {
              uint4* rowv = reinterpret_cast<uint4*>(act_s + tok * L.stride);
              uint4 v = rowv[ch];
              __half2* h = reinterpret_cast<__half2*>(&v);
              if constexpr (KSCALE) {
                const __half2* hb = reinterpret_cast<const __half2*>(&sb);
                h[0] = __hmul2(h[0], hb[0]);
                h[1] = __hmul2(h[1], hb[1]);
                h[2] = __hmul2(h[2], hb[2]);
                h[3] = __hmul2(h[3], hb[3]);
                rowv[ch] = v;
              }
              if constexpr (CLASS) {
                if (rest) {
#pragma unroll
                  for (int q = 0; q < 4; ++q) sum[j] += __low2float(h[q]) + __high2float(h[q]);
                }
              }
            }
          }
        }
        if constexpr (CLASS) {
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
            for (int j = 0; j < 4; ++j) sum[j] += __shfl_xor_sync(0xffffffffu, sum[j], off);
          }
          if (lane == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (warp + 4 * j < nvalid) upart_s[warp * 16 + warp + 4 * j] = sum[j];
          }
        }
        __syncthreads();
        if constexpr (CLASS) {
          // token t's sum comes from its owner warp t % 4 alone
          if (tid < nvalid) urest_s[tid] += upart_s[(tid & 3) * 16 + tid];
        }
      }
    }

    // ---- sign products over this warp's slice of the piece
    for (int gb = sb0; gb < sb1; gb += D) {
      if (gb + D < sb1) load_group(wb, gb + D, sb1);
      if (gb + D <= sb1 && pe - (gb + D) * 256 >= 0) {
        // D whole blocks: fixed offsets and no per-step predicates
        const int off0 = (gb * 256 - pk) >> 1;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          uint2 bb[16][NT];
#pragma unroll
          for (int s = 0; s < 16; ++s)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              bb[s][nt] = *reinterpret_cast<const uint2*>(arow[nt] + off0 + 128 * d + 8 * s);
#pragma unroll
          for (int s = 0; s < 16; ++s) {
            const uint32_t a0 = form_pair<CLASS>(wa[d][0].x, s);
            const uint32_t a2 = form_pair<CLASS>(wa[d][0].y, s);
            const uint32_t a1 = form_pair<CLASS>(wa[d][1].x, s);
            const uint32_t a3 = form_pair<CLASS>(wa[d][1].y, s);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_m16n8k16(acc[CLASS ? s : (s & 3)][nt], a0, a1, a2, a3, bb[s][nt].x, bb[s][nt].y);
          }
        }
      } else {
#pragma unroll
        for (int d = 0; d < D; ++d) {
          const int blk = gb + d;
          if (blk < sb1) {
            const int off = (blk * 256 - pk) >> 1;  // word offset of the block in a staged row
            const int nsteps = min(16, (pe - blk * 256) >> 4);
            // all of the block's activation fragments first, so the shared-memory
            // loads overlap each other instead of each MMA waiting for its own
            uint2 bb[16][NT];
#pragma unroll
            for (int s = 0; s < 16; ++s)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                bb[s][nt] = s < nsteps ? *reinterpret_cast<const uint2*>(arow[nt] + off + 8 * s) : make_uint2(0u, 0u);
#pragma unroll
            for (int s = 0; s < 16; ++s) {
              if (s < nsteps) {
                const uint32_t a0 = form_pair<CLASS>(wa[d][0].x, s);
                const uint32_t a2 = form_pair<CLASS>(wa[d][0].y, s);
                const uint32_t a1 = form_pair<CLASS>(wa[d][1].x, s);
                const uint32_t a3 = form_pair<CLASS>(wa[d][1].y, s);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                  mma_m16n8k16(acc[CLASS ? s : (s & 3)][nt], a0, a1, a2, a3, bb[s][nt].x, bb[s][nt].y);
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

    pk = pe;
    if (pk >= k_hi) break;
    pe = min(k_hi, pk + piece);
    // The next piece's bulk copies (async proxy) overwrite shared memory this
    // piece wrote (the b-scaled activations) and read with ordinary accesses:
    // order those accesses before the copies.
    fence_proxy_async_smem();
    __syncthreads();  // everyone is done with this piece's activations and b
    slice(pk, pe, sb0, sb1);
    load_group(wa, sb0, sb1);
    load_static(pk, pe);
  }
  __syncthreads();  // urest_s complete

  // ---- combine accumulators into this warp's partial t and hand it to rank 0
  const int slot = rank * KW + kw;
  if (ks > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // rank 0's bar_red is initialised
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
        // the class sums are counted once per CTA: by the K slice 0 warps
        t = acc[15][nt][e] + (kw == 0 ? urest_s[tok] : 0.f) - 2.f * corr;
      } else {
        t = (acc[0][nt][e] + acc[1][nt][e]) + (acc[2][nt][e] + acc[3][nt][e]);
      }
      const int rl = rt * 16 + g + 8 * (e >> 1);
      float* dst = &red_s[(slot * NTOK + tok) * ROWS + rl];
      if (rank == 0) {
        *dst = t;
      } else {
        st_cluster_f32(map_to_rank(dst, 0), t);
      }
    }
  }
  if (ks > 1 && rank != 0) {
    // each thread releases its own stores into rank 0 with its arrival
    mbar_arrive_remote_release(map_to_rank(bar_red, 0));
    return;  // nothing of this CTA's shared memory is read by others
  }
  __syncthreads();  // this CTA's own partials are written
  if (ks > 1) ok = mbar_wait_cluster_bounded(bar_red, 0, p.status) && ok;

  if (rank == 0 && ok) {
    const int nslots = ks * KW;
    for (int idx = tid; idx < nvalid * ROWS; idx += kDecThreads) {
      const int tok = idx / ROWS, rl = idx - tok * ROWS;
      const int row = m0 + rl;
      if (row < p.M) {
        float t = 0.f;
        for (int q = 0; q < nslots; ++q) t += red_s[(q * NTOK + tok) * ROWS + rl];
        const float v = t * rs_s[rl];
        if constexpr (OUT_F32) {
          static_cast<float*>(p.out)[static_cast<int64_t>(tok) * p.ld_out + row] = v;
        } else {
          static_cast<__half*>(p.out)[static_cast<int64_t>(tok) * p.ld_out + row] = __float2half_rn(v);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- one token: table lookup
//
// With a single token an MMA carries one useful column of eight, so the sums
// are formed by table lookup instead: for each nibble of a packed word (four
// sign bits) the CTA builds, once per piece of K, a table of the 16 signed
// sums of the four activations those bits select, and a row's product is the
// sum of one table entry per nibble of its words.  In the packed layout bit i
// of nibble j of word p of a 256-column block is the column
//   16 (4 (j mod 4) + i) + 2p + (j div 4),
// so table (block, p, j) holds T[v] = sum_i (bit i of v ? -u : u)[column_i].
// Tables are fp32 built from u = x (.) b in fp32 (exact for fp16 x and b), so
// this path does not round u to fp16.  Lane = weight row: all 32 lanes of a
// warp read the same 16-entry table at a time (conflict-free).  A CTA has 64
// rows: warp w takes rows 32 (w / 2) .. + 31 and half (w mod 2) of the blocks
// of each piece; K is split over a cluster as in the MMA kernel and the
// partials meet in rank 0 (rank-major, half minor: a fixed order).
constexpr int kLutD = 4;  // blocks of weights per register group

struct LutSmem {
  int act_off, b_off, tab_off, rs_off, red_off, total;
};

__host__ __device__ inline LutSmem lut_smem_layout(int piece, int ks) {
  LutSmem l;
  l.act_off = kHeadBytes;
  l.b_off = l.act_off + piece * 2;
  l.tab_off = (l.b_off + piece * 2 + 15) / 16 * 16;
  l.rs_off = l.tab_off + piece * 16;  // piece / 4 tables of 16 fp32
  l.red_off = l.rs_off + 64 * 4;
  l.total = l.red_off + ks * 2 * 64 * 4;
  return l;
}

template <bool KSCALE, bool OUT_F32>
__global__ void __launch_bounds__(kDecThreads, 1)
    dbf_decode_lut_kernel(const __grid_constant__ DecodeGroup grp, const int piece) {
  extern __shared__ __align__(128) uint8_t smem[];
  int li = 0;
  while (li + 1 < grp.n && static_cast<int>(blockIdx.x) >= grp.tile_start[li + 1]) ++li;
  const DecodeArgs& p = grp.layer[li];

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int ks = static_cast<int>(cluster.num_blocks());
  const LutSmem L = lut_smem_layout(piece, ks);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* bar_b = reinterpret_cast<uint64_t*>(smem + 16);
  uint64_t* bar_red = reinterpret_cast<uint64_t*>(smem + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 8);
  __half* act_s = reinterpret_cast<__half*>(smem + L.act_off);
  __half* b_s = reinterpret_cast<__half*>(smem + L.b_off);
  float* tab_s = reinterpret_cast<float*>(smem + L.tab_off);
  float* rs_s = reinterpret_cast<float*>(smem + L.rs_off);
  float* red_s = reinterpret_cast<float*>(smem + L.red_off);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int rg = warp >> 1, half = warp & 1;
  const int m0 = (static_cast<int>(blockIdx.x) - grp.tile_start[li]) * 64;
  const int row = m0 + 32 * rg + lane;
  const bool rok = row < p.M;
  const int k_lo = rank * p.kchunk;
  const int k_hi = min(p.K, k_lo + p.kchunk);
  const uint4* wrow = reinterpret_cast<const uint4*>(p.packed + static_cast<int64_t>(rok ? row : 0) * p.wpr);

  // this warp's blocks of a piece [pk, pe): its half of the piece's blocks
  auto slice = [&](int pk, int pe, int& b0, int& b1) {
    const int pb0 = pk >> 8, pb1 = (pe + 255) >> 8;
    const int per = (pb1 - pb0 + 1) / 2;
    b0 = min(pb1, pb0 + half * per);
    b1 = min(pb1, b0 + per);
  };
  uint4 wa[kLutD][2], wb[kLutD][2];
  auto load_group = [&](uint4 (&wr)[kLutD][2], int blk0, int blk_end) {
#pragma unroll
    for (int d = 0; d < kLutD; ++d) {
      const bool in = rok && blk0 + d < blk_end;
      wr[d][0] = in ? __ldg(wrow + 2 * (blk0 + d)) : make_uint4(0u, 0u, 0u, 0u);
      wr[d][1] = in ? __ldg(wrow + 2 * (blk0 + d) + 1) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  auto load_static = [&](int pk, int pe) {
    if (tid < 64) rs_s[tid] = (m0 + tid < p.M) ? __half2float(p.rowscale[m0 + tid]) : 0.f;
    if constexpr (KSCALE) {
      if (tid == 0 && pe > pk) {
        const uint32_t bytes = static_cast<uint32_t>(pe - pk) * 2;
        mbar_arrive_expect_tx(bar_b, bytes);
        bulk_load(b_s, p.kscale + pk, bytes, bar_b);
      }
    }
  };

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar_b, 1);
    mbar_init(bar_red, ks > 1 ? (ks - 1) * kDecThreads : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (ks > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  int pk = k_lo;
  int pe = min(k_hi, pk + piece);
  int sb0, sb1;
  slice(pk, pe, sb0, sb1);
  if (p.weights_early) {
    load_group(wa, sb0, sb1);
    load_static(pk, pe);
  }
  pdl_wait();
  pdl_launch_dependents();
  if (!p.weights_early) {
    load_group(wa, sb0, sb1);
    load_static(pk, pe);
  }

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  bool ok = true;
  uint32_t phase = 0;
  const bool has_k = k_lo < k_hi;
  while (has_k) {
    const int plen = pe - pk;  // multiple of 64
    if (tid == 0) {
      const uint32_t bytes = static_cast<uint32_t>(plen) * 2;
      mbar_arrive_expect_tx(bar, bytes);
      bulk_load(act_s, p.act + pk, bytes, bar);
    }
    ok = mbar_wait_bounded(bar, phase, abort_flag, p.status);
    if constexpr (KSCALE) ok = ok && mbar_wait_bounded(bar_b, phase, abort_flag, p.status);
    phase ^= 1u;
    ok = __syncthreads_and(ok);
    if (!ok) break;

    // ---- the tables of this piece: table tb = (block, word p, nibble j)
    const int ntab = ((plen + 255) >> 8) * 64;
    for (int tb = tid; tb < ntab; tb += kDecThreads) {
      const int pw = (tb >> 3) & 7, j = tb & 7;
      const int base = (tb >> 6) * 256 + 2 * pw + (j >> 2) + 64 * (j & 3);
      float u[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = base + 16 * i;
        float v = 0.f;
        if (col < plen) {
          v = __half2float(act_s[col]);
          if constexpr (KSCALE) v *= __half2float(b_s[col]);
        }
        u[i] = v;
      }
      // v = bits (b0 b1 b2 b3): e[v & 3] + f[v >> 2], a set bit negating its term
      const float e0 = u[0] + u[1], e1 = u[1] - u[0], e2 = u[0] - u[1], e3 = -(u[0] + u[1]);
      const float f0 = u[2] + u[3], f1 = u[3] - u[2], f2 = u[2] - u[3], f3 = -(u[2] + u[3]);
      float4* t4 = reinterpret_cast<float4*>(tab_s + tb * 16);
      t4[0] = make_float4(e0 + f0, e1 + f0, e2 + f0, e3 + f0);
      t4[1] = make_float4(e0 + f1, e1 + f1, e2 + f1, e3 + f1);
      t4[2] = make_float4(e0 + f2, e1 + f2, e2 + f2, e3 + f2);
      t4[3] = make_float4(e0 + f3, e1 + f3, e2 + f3, e3 + f3);
    }
    __syncthreads();

    // ---- one lookup per nibble of this lane's words
    const int pb0 = pk >> 8;
    for (int gb = sb0; gb < sb1; gb += kLutD) {
      if (gb + kLutD < sb1) load_group(wb, gb + kLutD, sb1);
#pragma unroll
      for (int d = 0; d < kLutD; ++d) {
        if (gb + d < sb1) {
          const float* tblk = tab_s + (gb + d - pb0) * 64 * 16;
          const uint32_t wd[8] = {wa[d][0].x, wa[d][0].y, wa[d][0].z, wa[d][0].w,
                                  wa[d][1].x, wa[d][1].y, wa[d][1].z, wa[d][1].w};
#pragma unroll
          for (int pw = 0; pw < 8; ++pw) {
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j & 3] += tblk[(pw * 8 + j) * 16 + ((wd[pw] >> (4 * j)) & 15u)];
          }
        }
      }
#pragma unroll
      for (int d = 0; d < kLutD; ++d) {
        wa[d][0] = wb[d][0];
        wa[d][1] = wb[d][1];
      }
    }

    pk = pe;
    if (pk >= k_hi) break;
    pe = min(k_hi, pk + piece);
    fence_proxy_async_smem();  // this piece's shared reads before the next bulk copies overwrite it
    __syncthreads();
    slice(pk, pe, sb0, sb1);
    load_group(wa, sb0, sb1);
    load_static(pk, pe);
  }

  // ---- this warp's partial of its 32 rows, to rank 0
  const int slot = rank * 2 + half;
  if (ks > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  {
    const float t = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    float* dst = &red_s[slot * 64 + 32 * rg + lane];
    if (rank == 0) {
      *dst = t;
    } else {
      st_cluster_f32(map_to_rank(dst, 0), t);
    }
  }
  if (ks > 1 && rank != 0) {
    mbar_arrive_remote_release(map_to_rank(bar_red, 0));
    return;
  }
  __syncthreads();
  if (ks > 1) ok = mbar_wait_cluster_bounded(bar_red, 0, p.status) && ok;
  if (rank == 0 && ok && tid < 64) {
    const int r = m0 + tid;
    if (r < p.M) {
      float t = 0.f;
      for (int q = 0; q < 2 * ks; ++q) t += red_s[q * 64 + tid];
      const float v = t * rs_s[tid];
      if constexpr (OUT_F32) {
        static_cast<float*>(p.out)[r] = v;
      } else {
        static_cast<__half*>(p.out)[r] = __float2half_rn(v);
      }
    }
  }
}

template <bool KSCALE, bool OUT_F32>
dbf_status launch_lut(const DecodeGroup& grp, int ks, int piece, cudaStream_t stream) {
  auto kernel = dbf_decode_lut_kernel<KSCALE, OUT_F32>;
  const size_t smem = static_cast<size_t>(lut_smem_layout(piece, ks).total);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
  });
  if (attr_err != cudaSuccess || smem > static_cast<size_t>(kMaxDynSmem)) return DBF_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grp.tile_start[grp.n]), static_cast<unsigned>(ks), 1);
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
  return cudaLaunchKernelEx(&cfg, kernel, grp, piece) == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

template <int NT, int RT, int D, bool TOKPAR, bool CLASS, bool KSCALE, bool OUT_F32>
dbf_status launch_typed(const DecodeGroup& grp, int batch, int ks, int piece, cudaStream_t stream) {
  auto kernel = dbf_decode_stage_kernel<NT, RT, D, TOKPAR, CLASS, KSCALE, OUT_F32>;
  const DecSmem L = dec_smem_layout(piece, batch < NT * 8 ? batch : NT * 8, NT * 8, ks, RT);
  const size_t smem = static_cast<size_t>(L.total);
  // the shared-memory limit once per instantiation (the largest a CTA may ask for)
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
  });
  if (attr_err != cudaSuccess || smem > static_cast<size_t>(kMaxDynSmem)) return DBF_ERR_CUDA;
  cudaError_t err;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grp.tile_start[grp.n]), static_cast<unsigned>(ks), 1);
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
  err = cudaLaunchKernelEx(&cfg, kernel, grp, piece);
  return err == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

template <int NT, int RT, int D, bool TOKPAR>
dbf_status launch_rt(const DecodeGroup& g, int batch, bool kscale, bool class_expand, bool out_f32, int ks, int piece,
                     cudaStream_t stream) {
  if (class_expand) {
    if (kscale) return out_f32 ? launch_typed<NT, RT, D, TOKPAR, true, true, true>(g, batch, ks, piece, stream)
                               : launch_typed<NT, RT, D, TOKPAR, true, true, false>(g, batch, ks, piece, stream);
    return out_f32 ? launch_typed<NT, RT, D, TOKPAR, true, false, true>(g, batch, ks, piece, stream)
                   : launch_typed<NT, RT, D, TOKPAR, true, false, false>(g, batch, ks, piece, stream);
  }
  if (kscale) return out_f32 ? launch_typed<NT, RT, D, TOKPAR, false, true, true>(g, batch, ks, piece, stream)
                             : launch_typed<NT, RT, D, TOKPAR, false, true, false>(g, batch, ks, piece, stream);
  return out_f32 ? launch_typed<NT, RT, D, TOKPAR, false, false, true>(g, batch, ks, piece, stream)
                 : launch_typed<NT, RT, D, TOKPAR, false, false, false>(g, batch, ks, piece, stream);
}

}  // namespace

// Work split of one stage: RT*16-row CTAs (RT = 4: 64 rows, one 16-row tile
// per warp) and ks CTAs per cluster along K.  Measured on B200 over the layer
// shapes of the workloads at batch 1 and 16, with the weights streamed from HBM:
//  * a warp's weights should fit one register group (4 blocks = 1024 columns),
//    so that all of them are requested before the programmatic-dependent-launch
//    wait and none of their latency is exposed after it: ks >= K / 1024;
//  * more than about two CTAs per SM per launch costs more than it gains: the
//    launch then cannot be resident beside its neighbour in the stream, and its
//    late CTAs start their weight loads only after the wait;
//  * when the other stage of the forward has enough row tiles to fill the GPU on
//    its own (1.5 per SM) and at most 8 tokens are in flight, this stage keeps
//    to about one CTA per SM for the same reason, but splits K at least half as
//    far as the first rule asks;
//  * at least a quarter of the SMs should take part.
// On a 4096 x 4096 layer at 1 bit/weight (k = 2048), batch 1, this split takes
// 7.8 us per layer against 8.8 us for a plain "two CTAs per SM" split.
struct DecodePlan {
  int rt, ks, piece;
  int64_t kchunk;
};

static DecodePlan plan_decode(int64_t M, int64_t K, int batch, int num_sms, int64_t peer_rows) {
  const int ntok = batch > 8 ? 16 : 8;
  const int nvalid = batch < ntok ? batch : ntok;
  const int64_t tiles = (M + 63) / 64;
  const int64_t peer_tiles = (peer_rows + 63) / 64;
  const int64_t ks_pref = std::min<int64_t>(kMaxClusterK, std::max<int64_t>(1, (K + 1023) / 1024));
  const bool peer_fills = batch <= 8 && 2 * peer_tiles >= 3 * static_cast<int64_t>(num_sms);
  const int64_t cap = peer_fills ? num_sms : 2 * num_sms;
  int64_t ks = ks_pref;
  while (ks > 1 && tiles * ks > cap) --ks;
  if (peer_fills) ks = std::max(ks, (ks_pref + 1) / 2);  // long rows still need CTAs in flight
  const int64_t ks_min = std::min<int64_t>(kMaxClusterK, (num_sms + 4 * tiles - 1) / (4 * tiles));
  ks = std::max(ks, ks_min);
  int64_t kchunk = (K + ks - 1) / ks;
  kchunk = (kchunk + 255) / 256 * 256;
  const int ks_eff = static_cast<int>((K + kchunk - 1) / kchunk);
  int piece = static_cast<int>(kchunk);
  while (piece > 256 && dec_smem_layout(piece, nvalid, ntok, ks_eff, 4).total > kSmemBudget) piece -= 256;
  return DecodePlan{4, ks_eff, piece, kchunk};
}

dbf_status launch_decode_group(DecodeGroup& grp, int64_t peer_rows, bool class_expand, bool lut, bool out_f32,
                               const DeviceInfo& dev, cudaStream_t stream) {
  if (grp.n < 1 || grp.n > kMaxGroup) return DBF_ERR_INVALID_ARG;
  const int batch = grp.layer[0].batch;
  const bool kscale = grp.layer[0].kscale != nullptr;
  int64_t tiles = 0, k_max = 0;
  for (int g = 0; g < grp.n; ++g) {
    const DecodeArgs& l = grp.layer[g];
    if (l.batch != batch || (l.kscale != nullptr) != kscale) return DBF_ERR_INVALID_ARG;
    grp.tile_start[g] = static_cast<int>(tiles);
    tiles += (l.M + 63) / 64;
    k_max = std::max<int64_t>(k_max, l.K);
  }
  if (tiles > 0x7fffffffLL) return DBF_ERR_UNSUPPORTED_SHAPE;
  grp.tile_start[grp.n] = static_cast<int>(tiles);
  // one K split for the launch, planned for its rows and its longest K; every
  // layer cuts its own K into that many 256-column-aligned chunks
  const DecodePlan plan = plan_decode(64 * tiles, k_max, batch, dev.num_sms, peer_rows);
  for (int g = 0; g < grp.n; ++g) {
    int64_t kc = (grp.layer[g].K + plan.ks - 1) / plan.ks;
    grp.layer[g].kchunk = static_cast<int>((kc + 255) / 256 * 256);
  }
  if (lut && batch == 1) {
    // one token: the lookup-table kernel (64-row CTAs, the same K split); a
    // piece is the whole K chunk unless the tables would not fit
    int kmax_chunk = 0;
    for (int g = 0; g < grp.n; ++g) kmax_chunk = std::max(kmax_chunk, grp.layer[g].kchunk);
    int piece = kmax_chunk;
    while (piece > 256 && lut_smem_layout(piece, plan.ks).total > kSmemBudget) piece -= 256;
    if (kscale) return out_f32 ? launch_lut<true, true>(grp, plan.ks, piece, stream)
                               : launch_lut<true, false>(grp, plan.ks, piece, stream);
    return out_f32 ? launch_lut<false, true>(grp, plan.ks, piece, stream)
                   : launch_lut<false, false>(grp, plan.ks, piece, stream);
  }
  int64_t max_blocks = 0;
  for (int g = 0; g < grp.n; ++g) max_blocks = std::max<int64_t>(max_blocks, grp.layer[g].kchunk / 256);
  // 8-block groups cost registers: keep them to launches of at most 1.75 CTAs
  // per SM, where the neighbouring launch is not resident beside them anyway
  const bool long_rows = max_blocks > 8 && 4 * tiles * plan.ks <= 7 * static_cast<int64_t>(dev.num_sms);
  // the activation pass: row by row for 1-3 tokens, four tokens per warp side by side from 4
  if (batch > 8) {
    return long_rows ? launch_rt<2, 4, 8, true>(grp, batch, kscale, class_expand, out_f32, plan.ks, plan.piece, stream)
                     : launch_rt<2, 4, 4, true>(grp, batch, kscale, class_expand, out_f32, plan.ks, plan.piece, stream);
  }
  if (batch >= 4) {
    return long_rows ? launch_rt<1, 4, 8, true>(grp, batch, kscale, class_expand, out_f32, plan.ks, plan.piece, stream)
                     : launch_rt<1, 4, 4, true>(grp, batch, kscale, class_expand, out_f32, plan.ks, plan.piece, stream);
  }
  return long_rows ? launch_rt<1, 4, 8, false>(grp, batch, kscale, class_expand, out_f32, plan.ks, plan.piece, stream)
                   : launch_rt<1, 4, 4, false>(grp, batch, kscale, class_expand, out_f32, plan.ks, plan.piece, stream);
}

dbf_status launch_decode_stage(const DecodeArgs& args, bool class_expand, bool lut, bool out_f32, const DeviceInfo& dev,
                               cudaStream_t stream) {
  DecodeGroup grp{};
  grp.n = 1;
  grp.layer[0] = args;
  return launch_decode_group(grp, args.peer_rows, class_expand, lut, out_f32, dev, stream);
}

}  // namespace dbf
