// Prefill path (large batches): one sign-product GEMM per launch on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Same product as the decode stage ("Addition is almost all you need",
// gist.science technical summary, section 2.1, computation process):
//
//   out[tok][row] = rowscale[row] * sum_K sign(row, K) * kscale[K] * act[tok][K]
//
// GEMM1: rows = k, K = m_in, kscale = b, act = x, rowscale = mid, out = V (fp16)
// GEMM2: rows = n, K = k,    no kscale,  act = V, rowscale = a,   out = y
//
// A tile computes D[128 weight rows x NTILE tokens] = S * act^T: the weights
// are the M operand, so each expanded sign tile serves NTILE tokens, each TMEM
// lane holds one weight row (the epilogue scale is a per-thread scalar) and a
// warp store writes 32 consecutive rows of one output token.
//
// The kernel is persistent: one CTA per SM walks the tiles tile = blockIdx.x,
// + gridDim.x, ...; the shared-memory ring runs on across tiles, and two TMEM
// accumulators let the epilogue of one tile overlap the main loop of the next.
// Roles (448 threads):
//   warps 0-7   sign expansion: thread t owns weight row t%128 and word half
//               t/128 of each 8-word block, i.e. pairs 4h..4h+3 of every
//               16-column group.  Per K step it turns 32 sign bits into 32
//               fp16 values (+-1, or +-b_j with b folded in by flipping the
//               scale's sign bit: exact) and stores four 16-byte chunks of the
//               row of a 128B-swizzled K-major tile.  Weight blocks are fetched
//               two blocks ahead and b one K step ahead;
//   warp 8      TMA producer of the activation tile (K-major, 128B swizzle,
//               tokens past the batch read as zero);
//   warp 9      TMEM allocation and the single-thread tcgen05.mma issue loop;
//   warps 10-13 epilogue: TMEM -> registers -> row scale -> a 32x32 transpose
//               in shared memory -> 16-byte global stores (warp w reads TMEM
//               lanes 32*(w%4) .. 32*(w%4)+31).
// Few tiles (small batches): the K range of each 128 x 128 tile is split over a
// cluster of 2-8 CTAs, one (tile, K slice) per CTA.  After the main loop a
// cluster barrier says every CTA's operand rings are idle; all warps then read
// the fp32 partial tile out of TMEM and store each rank's share of the token
// columns straight into that rank's B ring (st.async, completion counted in
// bytes on the rank's mbarrier), and every rank finishes its share, adding the
// parts in rank order.
// Stage hand-off is through mbarriers; every wait is bounded and an expired
// wait records DBF_ERR_TIMEOUT in the workspace status word, raises a CTA-wide
// abort flag and lets all roles fall through to the teardown, which frees TMEM
// only after this CTA's MMAs are known to be complete.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>
#include <type_traits>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace dbf {
namespace {

constexpr int kBM = 128;  // weight rows per tile (TMEM lanes)
constexpr int kBK = 64;   // K per pipeline stage: one 128-byte swizzle row of fp16
constexpr int kExpThreads = 256;
constexpr int kThreads = kExpThreads + 32 + 32 + 128;
constexpr int kWarpTma = kExpThreads / 32;
constexpr int kWarpMma = kWarpTma + 1;
constexpr int kWarpEpi0 = kWarpMma + 1;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kEpiStageBytes = 32 * 32 * 4;  // one warp's 32 tokens x 32 rows (fp32 worst case)

__device__ __forceinline__ void st_release_gpu_u32(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_gpu_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Bounded wait for a stream-K flag raised by another CTA of this grid (the
// same budget and abort protocol as the barrier waits).
__device__ __forceinline__ bool flag_wait_bounded(const unsigned* f, volatile int* abort_flag, int* status) {
  if (ld_acquire_gpu_u32(f) != 0u) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_gpu_u32(f) != 0u) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitBudgetNs) {
        *abort_flag = 1;
        if (status) atomicCAS(status, 0, kStatusTimeout);
        return false;
      }
    }
  }
}

template <int NTILE, bool SPLIT, bool ATMEM>
struct Cfg {
  // TMEM accumulators: two, so that the epilogue of one tile overlaps the
  // main loop of the next, except for 256-token tiles with A in TMEM, where
  // the A ring takes the room of the second one
  static constexpr int kAccBufs = (ATMEM && NTILE == 256) ? 1 : 2;
  static constexpr int kStages = ATMEM ? (NTILE == 256 ? 4 : 8) : (NTILE == 256 ? 4 : 6);
  static constexpr int kAStageBytes = ATMEM ? 0 : kABytes;  // A in TMEM: no shared-memory A ring
  static constexpr int kBBytes = NTILE * kBK * 2;
  static constexpr int kEpiOffset = kStages * (kAStageBytes + kBBytes);
  static constexpr int kBarOffset = kEpiOffset + 4 * kEpiStageBytes;
  // full_a[S], full_b[S], empty[S], acc_full[2], acc_empty[2], mma_done, recv, epi, sk
  static constexpr int kNumBars = 3 * kStages + 8;
  static constexpr int kRsOffset = kBarOffset + kNumBars * 8 + 16;  // after the tmem slot and abort flag
  // + split K: the tile's row scales (fp32), + alignment slack
  static constexpr int kSmemBytes = kRsOffset + kBM * 4 + 1024;
  // TMEM: kAccBufs accumulators of NTILE columns, then (A in TMEM) the A
  // ring, kBK / 2 columns per stage (column c of a stage = the fp16 pair K 2c, 2c+1)
  static constexpr int kTmemA = kAccBufs * NTILE;
  static constexpr int kTmemCols = ATMEM ? 512 : 2 * NTILE;
  static_assert(!ATMEM || kTmemA + kStages * (kBK / 2) <= 512, "A ring must fit in tensor memory");
  // split K: once a CTA's MMAs are done its operand rings are idle; the B ring
  // then receives the peers' parts of this CTA's token columns,
  // [src rank][NTILE/ks/4][128 rows] float4 (at most one whole partial tile).
  static constexpr int kPartialBytes = kBM * NTILE * 4;
  static_assert(!SPLIT || kPartialBytes <= kStages * kBBytes, "split-K parts must fit in the idle B ring");
  static_assert(!SPLIT || 14 * 8 * 32 * 4 <= 4 * kEpiStageBytes, "split-K output transposes must fit the epilogue stage");
};

template <int NTILE, bool SPLIT, bool KSCALE, bool OUT_F32, bool ATMEM, bool SK>
__global__ void __launch_bounds__(kThreads, 1)
    dbf_prefill_gemm_kernel(const __grid_constant__ CUtensorMap act_map, const PrefillArgs p) {
  static_assert(!(SK && SPLIT), "stream-K and the cluster split are separate schedules");
  static_assert(!SK || NTILE * kBM * 4 <= static_cast<int>(kSkSlotBytes), "a partial tile must fit its slot");
  using C = Cfg<NTILE, SPLIT, ATMEM>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_st = smem;
  uint8_t* b_st = smem + S * C::kAStageBytes;
  uint8_t* epi_st = smem + C::kEpiOffset;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* full_a = bars;
  uint64_t* full_b = bars + S;
  uint64_t* empty = bars + 2 * S;
  uint64_t* acc_full = bars + 3 * S;
  uint64_t* acc_empty = bars + 3 * S + 2;
  uint64_t* mma_done = bars + 3 * S + 4;
  uint64_t* recv_bar = bars + 3 * S + 5;  // split K: the peers' parts have landed
  uint64_t* epi_bar = bars + 3 * S + 6;   // stream-K: the four epilogue warps meet (bounded, unlike bar.sync)
  uint64_t* sk_bar = bars + 3 * S + 7;    // stream-K: a partial tile has been copied into the B ring
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* rs_s = reinterpret_cast<float*>(smem + C::kRsOffset);  // split K: row scales of the tile

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int m_tiles = (p.M + kBM - 1) / kBM;
  const int num_tiles = m_tiles * ((p.batch + NTILE - 1) / NTILE);
  const int KT = p.K / kBK;
  const int nblk = (KT + 3) / 4;
  // Work items: (tile, K slice).  Without a split there is one slice per tile
  // and the CTAs walk the items persistently; with a split, the ks CTAs of a
  // cluster take the ks slices of one tile (one item per CTA) and add their
  // partial sums through distributed shared memory.
  const int ks = SPLIT ? static_cast<int>(cluster_size()) : 1;
  const int rank = SPLIT ? static_cast<int>(cluster_rank()) : 0;
  const int num_items = num_tiles * ks;
  const int bper = (nblk + ks - 1) / ks;
  auto item_blocks = [&](int w, int& b0, int& b1) {
    b0 = min(nblk, (w % ks) * bper);
    b1 = min(nblk, b0 + bper);
  };
  // Stream-K: the units (tile, 256-column block), tile-major, are cut into
  // gridDim.x contiguous ranges, one per CTA; a CTA's range is a sequence of
  // segments (tile, blocks b0..b1).  Only a CTA's first segment can start
  // inside a tile (it then leaves an fp32 partial tile in its slot) and only
  // its last can stop inside one (it then finishes that tile: it adds the
  // partials of the CTAs after it whose first segments lie in the tile).
  const int64_t sk_units = static_cast<int64_t>(num_tiles) * nblk;
  auto sk_lo = [&](int64_t c) { return sk_units * c / gridDim.x; };
  const int64_t sk_hi = SK ? sk_lo(blockIdx.x + 1) : 0;
  // A work cursor walks this CTA's work: an item index (one item per tile and
  // K slice, stepping by gridDim.x) or, for stream-K, a unit index.
  const int64_t work_first = SK ? sk_lo(blockIdx.x) : static_cast<int64_t>(blockIdx.x);
  auto work_valid = [&](int64_t c) { return SK ? c < sk_hi : c < num_items; };
  auto work_get = [&](int64_t c, int& tile, int& b0, int& b1) {
    if constexpr (SK) {
      tile = static_cast<int>(c / nblk);
      b0 = static_cast<int>(c % nblk);
      const int64_t end = b0 + (sk_hi - c);
      b1 = end < nblk ? static_cast<int>(end) : nblk;
    } else {
      tile = static_cast<int>(c) / ks;
      item_blocks(static_cast<int>(c), b0, b1);
    }
  };
  auto work_next = [&](int64_t c, int b0, int b1) -> int64_t {
    return SK ? c + (b1 - b0) : c + static_cast<int64_t>(gridDim.x);
  };

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_a[i], kExpThreads);
      mbar_init(&full_b[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    mbar_init(mma_done, 1);
    mbar_init(recv_bar, 1);
    mbar_init(epi_bar, 128);
    mbar_init(sk_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpTma && lane == 0) prefetch_tmap(&act_map);
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Let the next kernel in the stream be scheduled as this grid's CTAs exit
  // (it waits for this grid's completion before it reads anything this grid
  // writes).  Every CTA of this grid is resident once they have all passed
  // here, so a dependent cannot keep one of them from starting; and two CTAs
  // of this kernel never fit on one SM, so a dependent prefill CTA only takes
  // an SM this grid has left.
  pdl_launch_dependents();
  // Peers write into this CTA's receive buffer only after every CTA of the
  // cluster has initialised its barriers (the matching wait comes later).
  if constexpr (SPLIT) cluster_arrive_relaxed();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kWarpTma) {
    // ------------------------------------------------ sign expansion
    // Row r's packed row is a sequence of 8-word blocks of 256 columns; K step
    // kt covers groups 4*(kt%4) .. 4*(kt%4)+3 of block kt/4, and group g's 16
    // columns come from bit pair (g, g+16) of the block's 8 words.
    // A in shared memory: thread (row, h) holds words 4h..4h+3 (column pairs
    // 4h..4h+3 of every group) and writes four 16-byte chunks per K step.
    // A in tensor memory: thread (row, h) holds all 8 words and writes the 16
    // column pairs of groups 2h, 2h+1 of each K step (TMEM columns 16h..16h+15
    // of the stage, one 32x32b.x16 store per warp into its TMEM lane quadrant).
    const int r_local = tid & (kBM - 1);
    const int h = tid >> 7;
    struct Words {
      uint4 lo, hi;  // hi: words 4..7 (A in tensor memory only)
    };
    // block sequence of this CTA: (work, blk) with blk fastest
    int64_t f_cur = work_first;
    int f_tile = 0, f_b0 = 0, f_blk = 0, f_end = 0;
    auto f_seek = [&]() {
      while (work_valid(f_cur)) {
        work_get(f_cur, f_tile, f_b0, f_end);
        f_blk = f_b0;
        if (f_blk < f_end) return;
        f_cur = work_next(f_cur, f_b0, f_end);
      }
    };
    f_seek();
    auto fetch_next = [&]() -> Words {
      Words v{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
      if (work_valid(f_cur)) {
        const int r = (f_tile % m_tiles) * kBM + r_local;
        if (r < p.M) {
          const uint32_t* src = p.packed + static_cast<int64_t>(r) * p.wpr + 8 * f_blk;
          if constexpr (ATMEM) {
            v.lo = ldg_stream_u4(src);
            v.hi = ldg_stream_u4(src + 4);
          } else {
            v.lo = ldg_stream_u4(src + 4 * h);
          }
        }
        if (++f_blk == f_end) {
          f_cur = work_next(f_cur, f_b0, f_end);
          f_seek();
        }
      }
      return v;
    };
    // The scale pairs of this thread's columns of K step kt: A in shared
    // memory, sc[i] = columns 16i + 8h .. +7; A in tensor memory,
    // sc[2j + c] = columns 16(2h + j) + 8c .. +7.
    auto fetch_scale = [&](int kt, uint4 (&sc)[4]) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = ATMEM ? 16 * (2 * h + (i >> 1)) + 8 * (i & 1) : 16 * i + 8 * h;
        sc[i] = __ldg(reinterpret_cast<const uint4*>(p.kscale + kt * kBK + col));
      }
    };
    int first_tile = 0, first_b0 = 0, first_b1 = 0;
    if (work_valid(work_first)) work_get(work_first, first_tile, first_b0, first_b1);
    const int kt_first = min(KT - 1, 4 * first_b0);
    Words w_n1, w_n2, wcur{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    uint4 sc_next[4];
    if (p.weights_early) {
      w_n1 = fetch_next();
      w_n2 = fetch_next();
      if constexpr (KSCALE) fetch_scale(kt_first, sc_next);
    }
    pdl_wait();
    if (!p.weights_early) {
      w_n1 = fetch_next();
      w_n2 = fetch_next();
      if constexpr (KSCALE) fetch_scale(kt_first, sc_next);
    }
    bool ok = true;
    const int swz = r_local & 7;
    const uint32_t a_lane = static_cast<uint32_t>(r_local & ~31) << 16;  // this warp's TMEM lane quadrant
    uint32_t it = 0;
    for (int64_t wc = work_first; work_valid(wc) && ok;) {
      int tile, b0, b1;
      work_get(wc, tile, b0, b1);
      wc = work_next(wc, b0, b1);
      const int kt0 = 4 * b0, kt1 = min(KT, 4 * b1);
      for (int kt = kt0; kt < kt1; ++kt, ++it) {
        const int s = static_cast<int>(it % S);
        const uint32_t use = it / S;
        if ((kt & 3) == 0) {
          wcur = w_n1;
          w_n1 = w_n2;
          w_n2 = fetch_next();
        }
        // the next K step (the next item of a persistent CTA starts again at K step 0)
        const int kt_next = kt + 1 < kt1 ? kt + 1 : (SPLIT ? kt0 : 0);
        uint4 sc[4];
        if constexpr (KSCALE) {
#pragma unroll
          for (int i = 0; i < 4; ++i) sc[i] = sc_next[i];
          fetch_scale(kt_next, sc_next);
        }
        if (it >= S && !mbar_wait_bounded(&empty[s], (use - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        if constexpr (ATMEM) {
          tc_fence_after();  // the MMAs that read this stage have completed
          const uint32_t wd[8] = {wcur.lo.x, wcur.lo.y, wcur.lo.z, wcur.lo.w, wcur.hi.x, wcur.hi.y, wcur.hi.z, wcur.hi.w};
          uint32_t q[16];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int g = 4 * (kt & 3) + 2 * h + j;  // group inside the block
#pragma unroll
            for (int pr = 0; pr < 8; ++pr) {
              if constexpr (KSCALE) {
                const uint4 v = sc[2 * j + (pr >> 2)];
                const uint32_t sp = (pr & 3) == 0 ? v.x : (pr & 3) == 1 ? v.y : (pr & 3) == 2 ? v.z : v.w;
                q[8 * j + pr] = signed_scale_pair_rt(wd[pr], g, sp);
              } else {
                q[8 * j + pr] = pm1_pair_rt(wd[pr], g);
              }
            }
          }
          tmem_st_32x32b_x16(tmem_base + a_lane + static_cast<uint32_t>(C::kTmemA + s * (kBK / 2) + 16 * h), q);
          tmem_st_wait();
          tc_fence_before();
        } else {
          uint8_t* dst = a_st + s * kABytes + (r_local >> 3) * 1024 + swz * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int g = 4 * (kt & 3) + i;  // group inside the block
            uint32_t q[4];
            if constexpr (KSCALE) {
              q[0] = signed_scale_pair_rt(wcur.lo.x, g, sc[i].x);
              q[1] = signed_scale_pair_rt(wcur.lo.y, g, sc[i].y);
              q[2] = signed_scale_pair_rt(wcur.lo.z, g, sc[i].z);
              q[3] = signed_scale_pair_rt(wcur.lo.w, g, sc[i].w);
            } else {
              q[0] = pm1_pair_rt(wcur.lo.x, g);
              q[1] = pm1_pair_rt(wcur.lo.y, g);
              q[2] = pm1_pair_rt(wcur.lo.z, g);
              q[3] = pm1_pair_rt(wcur.lo.w, g);
            }
            // columns 16i + 8h .. 16i + 8h + 7 -> 16-byte chunk 2i + h (128B swizzle)
            *reinterpret_cast<uint4*>(dst + (((2 * i + h) ^ swz) << 4)) = make_uint4(q[0], q[1], q[2], q[3]);
          }
          fence_proxy_async_smem();
        }
        mbar_arrive(&full_a[s]);
      }
    }
  } else if (warp == kWarpTma) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      pdl_wait();
      uint32_t it = 0;
      bool ok = true;
      for (int64_t wc = work_first; work_valid(wc) && ok;) {
        int tile, b0, b1;
        work_get(wc, tile, b0, b1);
        wc = work_next(wc, b0, b1);
        const int n0 = (tile / m_tiles) * NTILE;
        for (int kt = 4 * b0; kt < min(KT, 4 * b1); ++kt, ++it) {
          const int s = static_cast<int>(it % S);
          const uint32_t use = it / S;
          if (it >= S && !mbar_wait_bounded(&empty[s], (use - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_b[s], C::kBBytes);
          tma_load_2d(b_st + s * C::kBBytes, &act_map, kt * kBK, n0, &full_b[s]);
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------ MMA issue
    if (lane == 0) {
      pdl_wait();
      constexpr uint32_t idesc = idesc_f16_f32(kBM, NTILE);
      bool ok = true;
      uint32_t it = 0, local = 0;
      for (int64_t wc = work_first; work_valid(wc) && ok; ++local) {
        const uint32_t buf = local % C::kAccBufs;
        if (local >= C::kAccBufs &&
            !mbar_wait_bounded(&acc_empty[buf], ((local / C::kAccBufs) - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * NTILE;
        int tile, b0, b1;
        work_get(wc, tile, b0, b1);
        wc = work_next(wc, b0, b1);
        const int kt0 = 4 * b0, kt1 = min(KT, 4 * b1);
        for (int kt = kt0; kt < kt1; ++kt, ++it) {
          const int s = static_cast<int>(it % S);
          const uint32_t par = (it / S) & 1;
          if (!mbar_wait_bounded(&full_a[s], par, abort_flag, p.status) ||
              !mbar_wait_bounded(&full_b[s], par, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(a_st + s * C::kAStageBytes);
          const uint32_t b_addr = smem_u32(b_st + s * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t acc = (kt != kt0 || kk != 0) ? 1u : 0u;
            if constexpr (ATMEM) {
              tc_mma_f16_ts(d_tmem, tmem_base + static_cast<uint32_t>(C::kTmemA + s * (kBK / 2) + kk * 8),
                            smem_desc_sw128_kmajor(b_addr + kk * 32), idesc, acc);
            } else {
              tc_mma_f16_ss(d_tmem, smem_desc_sw128_kmajor(a_addr + kk * 32), smem_desc_sw128_kmajor(b_addr + kk * 32),
                            idesc, acc);
            }
          }
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(&acc_full[buf]);
      }
      tc_commit(mma_done);
    }
  } else {
    // ------------------------------------------------ epilogue
    using OutT = typename std::conditional<OUT_F32, float, __half>::type;
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    OutT* out = static_cast<OutT*>(p.out);
    uint32_t local = 0;
    if constexpr (SPLIT) {
      // split K: the exchange and the reduction run on all warps after the
      // role loops; the epilogue warps only stage the tile's row scales here
      if (!p.weights_early) pdl_wait();
      const int r = q * 32 + lane;
      const int row = ((static_cast<int>(blockIdx.x) / ks) % m_tiles) * kBM + r;
      rs_s[r] = row < p.M ? __half2float(p.rowscale[row]) : 0.f;
    } else {
      constexpr int kVec = 16 / sizeof(OutT);  // outputs per 16-byte store
      OutT* stg = reinterpret_cast<OutT*>(epi_st + (warp - kWarpEpi0) * kEpiStageBytes);  // [32 tokens][32 rows]
      const bool ld_ok = (p.ld_out % kVec) == 0;
      const int r = q * 32 + lane;  // row of the tile (TMEM lane)
      uint32_t epi_phase = 0, sk_phase = 0;
      auto epi_sync = [&]() -> bool {
        mbar_arrive(epi_bar);
        return mbar_wait_bounded(epi_bar, (epi_phase++) & 1, abort_flag, p.status);
      };
      for (int64_t wc = work_first; work_valid(wc); ++local) {
        int tile, b0, b1;
        work_get(wc, tile, b0, b1);
        wc = work_next(wc, b0, b1);
        const uint32_t buf = local % C::kAccBufs;
        const int m0 = (tile % m_tiles) * kBM;
        const int n0 = (tile / m_tiles) * NTILE;
        const int row0 = m0 + q * 32;
        const int row = row0 + lane;
        const float rs = (row < p.M) ? __half2float(p.rowscale[row]) : 0.f;  // in flight during the wait
        if (!mbar_wait_bounded(&acc_full[buf], (local / C::kAccBufs) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t acc_addr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * NTILE;
        if (SK && b0 > 0) {
          // stream-K, a later part of a tile: leave the fp32 partial in this
          // CTA's slot, [column / 4][row] float4, and raise the slot's flag
          float4* slot = reinterpret_cast<float4*>(p.sk_slots) + static_cast<size_t>(blockIdx.x) * (kSkSlotBytes / 16);
          for (int col = 0; col < NTILE; col += 32) {
            if (n0 + col >= p.batch) break;  // warp-uniform
            uint32_t v[32];
            tmem_ld_32x32b_x32(acc_addr + static_cast<uint32_t>(col), v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 8; ++i)
              slot[(col / 4 + i) * kBM + r] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                          __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[buf]);
          if (!epi_sync()) break;  // every epilogue thread's part is stored
          if (tid == kWarpEpi0 * 32) {
            __threadfence();
            st_release_gpu_u32(p.sk_flags + blockIdx.x, 1u);
          }
          continue;
        }
        // stream-K, the first part of a tile that later CTAs finish
        // (contributors blockIdx.x+1 .. c_end-1): the MMAs are done, so the B
        // ring is idle; each contributor's partial is bulk-copied into it and
        // added into the accumulator in TMEM, in CTA order
        int c_end = static_cast<int>(blockIdx.x) + 1;
        bool parts_ok = true;
        if (SK && b1 < nblk) {
          const int64_t tile_end = static_cast<int64_t>(tile + 1) * nblk;
          while (c_end < static_cast<int>(gridDim.x) && sk_lo(c_end) < tile_end) ++c_end;
          const int ncols = min(NTILE, (p.batch - n0 + 31) / 32 * 32);  // the columns the parts hold
          const uint32_t bytes = static_cast<uint32_t>(ncols) * kBM * 4;
          const float4* part = reinterpret_cast<const float4*>(b_st);
          for (int c = static_cast<int>(blockIdx.x) + 1; c < c_end && parts_ok; ++c) {
            if (tid == kWarpEpi0 * 32 && flag_wait_bounded(p.sk_flags + c, abort_flag, p.status)) {
              fence_proxy_async_global();  // the part was written through the generic proxy
              mbar_arrive_expect_tx(sk_bar, bytes);
              const char* src = reinterpret_cast<const char*>(p.sk_slots) + static_cast<size_t>(c) * kSkSlotBytes;
              for (uint32_t off = 0; off < bytes; off += 32768u)
                bulk_load(b_st + off, src + off, bytes - off < 32768u ? bytes - off : 32768u, sk_bar);
            }
            parts_ok = mbar_wait_bounded(sk_bar, (sk_phase++) & 1, abort_flag, p.status);
            if (!parts_ok) break;
            for (int col = 0; col < ncols; col += 32) {
              uint32_t v[32];
              tmem_ld_32x32b_x32(acc_addr + static_cast<uint32_t>(col), v);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 t = part[(col / 4 + i) * kBM + r];
                v[4 * i] = __float_as_uint(__uint_as_float(v[4 * i]) + t.x);
                v[4 * i + 1] = __float_as_uint(__uint_as_float(v[4 * i + 1]) + t.y);
                v[4 * i + 2] = __float_as_uint(__uint_as_float(v[4 * i + 2]) + t.z);
                v[4 * i + 3] = __float_as_uint(__uint_as_float(v[4 * i + 3]) + t.w);
              }
              tmem_st_32x32b_x32(acc_addr + static_cast<uint32_t>(col), v);
            }
            tmem_st_wait();
            fence_proxy_async_smem();  // these reads come before the next copy into the ring
            parts_ok = epi_sync();
          }
        }
        const bool rows_full = row0 + 32 <= p.M;
        for (int col = 0; col < NTILE && parts_ok; col += 32) {
          if (n0 + col >= p.batch) break;  // warp-uniform
          uint32_t v[32];
          tmem_ld_32x32b_x32(acc_addr + static_cast<uint32_t>(col), v);
          tmem_ld_wait();
          const int tok0 = n0 + col;
          if (rows_full && ld_ok && tok0 + 32 <= p.batch) {
            // transpose through shared memory, then 16-byte stores of kVec consecutive rows
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float val = rs * __uint_as_float(v[j]);
              if constexpr (OUT_F32) {
                stg[j * 32 + lane] = val;
              } else {
                stg[j * 32 + lane] = __float2half_rn(val);
              }
            }
            __syncwarp();
            constexpr int kChunksPerTok = 32 / kVec;
#pragma unroll
            for (int m = 0; m < 32 * kChunksPerTok / 32; ++m) {
              const int cidx = lane + 32 * m;
              const int tk = cidx / kChunksPerTok, rp = cidx % kChunksPerTok;
              const uint4 val = *reinterpret_cast<const uint4*>(stg + tk * 32 + rp * kVec);
              *reinterpret_cast<uint4*>(out + static_cast<int64_t>(tok0 + tk) * p.ld_out + row0 + rp * kVec) = val;
            }
            __syncwarp();
          } else if (row < p.M) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int tok = tok0 + j;
              if (tok < p.batch) {
                const float val = rs * __uint_as_float(v[j]);
                if constexpr (OUT_F32) {
                  out[static_cast<int64_t>(tok) * p.ld_out + row] = val;
                } else {
                  out[static_cast<int64_t>(tok) * p.ld_out + row] = __float2half_rn(val);
                }
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);
        if (!parts_ok) break;
        if (SK && c_end > static_cast<int>(blockIdx.x) + 1) {
          if (!epi_sync()) break;  // every epilogue thread has read the partials
          if (tid == kWarpEpi0 * 32)
            for (int c = static_cast<int>(blockIdx.x) + 1; c < c_end; ++c) p.sk_flags[c] = 0u;  // zero for the next launch
        }
      }
    }
  }

  // ------------------------------------------------ split K: exchange of the partial tiles
  if constexpr (SPLIT) {
    // Reduce-scatter of the ks partial tiles of one (tile, all K) item: rank j
    // finishes token columns [j*cw, (j+1)*cw).  Once every rank's MMAs are done
    // (a cluster barrier: every operand ring is idle), all 14 warps read the
    // partial tile out of TMEM (warp w may read lanes 32*(w%4) .. 32*(w%4)+31;
    // the warps of a lane quadrant share its 16-column chunks) and store each
    // quad of the other ranks' columns straight into the owning rank's B ring
    // with st.async, counted in bytes on that rank's mbarrier.  This rank's own
    // columns stay in TMEM.
    __syncwarp();  // the single-thread roles rejoin their warps
    constexpr int kWarps = kThreads / 32;
    const int cw = NTILE / ks;
    const int cw4 = cw / 4;
    const uint32_t slice_bytes = static_cast<uint32_t>(kBM * cw * 4);
    float4* recv = reinterpret_cast<float4*>(b_st);  // [src rank][cw4][128 rows]
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int nq = (kWarps - q + 3) / 4;  // warps that may read quadrant q (4, 4, 3, 3)
    const int jq = warp >> 2;             // this warp's index among them
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const bool got = mbar_wait_bounded(&acc_full[0], 0, abort_flag, p.status);
    tc_fence_after();
    int b0, b1;
    item_blocks(blockIdx.x, b0, b1);
    const bool have = __all_sync(0xffffffffu, got) && b1 > b0;  // an empty K slice contributes zeros
    cluster_wait_acquire();    // phase 0: every CTA of the cluster initialised its barriers
    cluster_arrive_release();  // phase 1: this CTA's MMAs are done, its rings are idle
    cluster_wait_acquire();
    if (tid == 0) mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>(ks - 1) * slice_bytes);
    for (int col = 16 * jq; col < NTILE; col += 16 * nq) {
      const int dst = col / cw;  // cw >= 16: a chunk has one owner
      if (dst == rank) continue;
      uint32_t v[16];
      if (have) {
        tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(col), v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
      const int cc40 = (col - dst * cw) >> 2;
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        st_async_v4f32(map_to_rank(&recv[(rank * cw4 + cc40 + j4) * kBM + r], static_cast<uint32_t>(dst)),
                       __uint_as_float(v[4 * j4]), __uint_as_float(v[4 * j4 + 1]), __uint_as_float(v[4 * j4 + 2]),
                       __uint_as_float(v[4 * j4 + 3]), map_to_rank(recv_bar, static_cast<uint32_t>(dst)));
      }
    }

    // Finish this rank's columns once the peers' parts have landed: thread r of
    // quadrant q adds, for its row and 8 of the columns, the ks parts in rank
    // order (its own from TMEM), scales, and the warp writes its 32 rows x 8
    // tokens through a shared-memory transpose with 16-byte stores.
    const bool rcv = __all_sync(0xffffffffu, mbar_wait_cluster_bounded(recv_bar, 0, p.status));
    if (rcv) {
      using OutT = typename std::conditional<OUT_F32, float, __half>::type;
      constexpr int kVec = 16 / sizeof(OutT);  // outputs per 16-byte store
      OutT* out = static_cast<OutT*>(p.out);
      OutT* stg = reinterpret_cast<OutT*>(epi_st + warp * (8 * 32 * sizeof(OutT)));  // [8 tokens][32 rows]
      const int m0 = ((static_cast<int>(blockIdx.x) / ks) % m_tiles) * kBM;
      const int n0 = ((static_cast<int>(blockIdx.x) / ks) / m_tiles) * NTILE + rank * cw;
      const int row0 = m0 + q * 32;
      const int row = row0 + lane;
      const float rs = rs_s[r];
      const bool vec_ok = row0 + 32 <= p.M && (p.ld_out % kVec) == 0;
      for (int ch = jq; ch < cw / 8; ch += nq) {
        uint32_t v[8];
        if (have) {
          tmem_ld_32x32b_x8(lane_base + static_cast<uint32_t>(rank * cw + 8 * ch), v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = 0u;
        }
        float sum[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) sum[j] = 0.f;
        for (int src = 0; src < ks; ++src) {
          float t[8];
          if (src == rank) {
#pragma unroll
            for (int j = 0; j < 8; ++j) t[j] = __uint_as_float(v[j]);
          } else {
            const float4 lo = recv[(src * cw4 + 2 * ch) * kBM + r];
            const float4 hi = recv[(src * cw4 + 2 * ch + 1) * kBM + r];
            t[0] = lo.x; t[1] = lo.y; t[2] = lo.z; t[3] = lo.w;
            t[4] = hi.x; t[5] = hi.y; t[6] = hi.z; t[7] = hi.w;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) sum[j] += t[j];
        }
        const int tok0 = n0 + 8 * ch;
        if (vec_ok && tok0 + 8 <= p.batch) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if constexpr (OUT_F32) {
              stg[j * 32 + lane] = rs * sum[j];
            } else {
              stg[j * 32 + lane] = __float2half_rn(rs * sum[j]);
            }
          }
          __syncwarp();
          constexpr int kChunksPerTok = 32 / kVec;
#pragma unroll
          for (int m = 0; m < 8 * kChunksPerTok / 32; ++m) {
            const int cidx = lane + 32 * m;
            const int tk = cidx / kChunksPerTok, rp = cidx % kChunksPerTok;
            const uint4 val = *reinterpret_cast<const uint4*>(stg + tk * 32 + rp * kVec);
            *reinterpret_cast<uint4*>(out + static_cast<int64_t>(tok0 + tk) * p.ld_out + row0 + rp * kVec) = val;
          }
          __syncwarp();
        } else if (row < p.M) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int tok = tok0 + j;
            if (tok < p.batch) {
              if constexpr (OUT_F32) {
                out[static_cast<int64_t>(tok) * p.ld_out + row] = rs * sum[j];
              } else {
                out[static_cast<int64_t>(tok) * p.ld_out + row] = __float2half_rn(rs * sum[j]);
              }
            }
          }
        }
      }
    }
  }

  // ------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    // Free TMEM once every MMA this CTA issued has finished (the wait is
    // bounded; TMEM must be released before the CTA exits either way).
    (void)mbar_wait_bounded(mma_done, 0, abort_flag, p.status);
    __syncwarp();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if constexpr (SPLIT) {
    // phase 2: no CTA leaves while a peer may still store into its shared
    // memory (every rank has waited for all of its parts)
    cluster_arrive_release();
    cluster_wait_acquire();
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
  });
  return fn;
}

template <int NTILE, bool SPLIT, bool KSCALE, bool OUT_F32, bool ATMEM, bool SK>
dbf_status launch_typed(const PrefillArgs& a, const CUtensorMap& map, int ks, const DeviceInfo& dev,
                        cudaStream_t stream) {
  auto kernel = dbf_prefill_gemm_kernel<NTILE, SPLIT, KSCALE, OUT_F32, ATMEM, SK>;
  constexpr int smem = Cfg<NTILE, SPLIT, ATMEM>::kSmemBytes;
  static std::once_flag once;  // the attribute once per instantiation
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] { attr_err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
  if (attr_err != cudaSuccess) return DBF_ERR_CUDA;
  const int64_t m_tiles = (a.M + kBM - 1) / kBM;
  const int64_t n_tiles = (a.batch + NTILE - 1) / NTILE;
  // split K: one (tile, K slice) item per CTA, the ks slices of a tile in one
  // cluster; stream-K: one range of units per SM (all CTAs resident at once)
  const int64_t grid = SPLIT ? m_tiles * n_tiles * ks
                       : SK  ? std::min<int64_t>(dev.num_sms, kSkMaxCtas)
                             : std::min<int64_t>(m_tiles * n_tiles, dev.num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(SPLIT ? ks : 1);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, map, a) == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

template <int NTILE, bool SPLIT, bool ATMEM, bool SK = false>
dbf_status launch_split(const PrefillArgs& a, const CUtensorMap& map, int ks, bool out_f32, const DeviceInfo& dev,
                        cudaStream_t stream) {
  if (a.kscale != nullptr)
    return out_f32 ? launch_typed<NTILE, SPLIT, true, true, ATMEM, SK>(a, map, ks, dev, stream)
                   : launch_typed<NTILE, SPLIT, true, false, ATMEM, SK>(a, map, ks, dev, stream);
  return out_f32 ? launch_typed<NTILE, SPLIT, false, true, ATMEM, SK>(a, map, ks, dev, stream)
                 : launch_typed<NTILE, SPLIT, false, false, ATMEM, SK>(a, map, ks, dev, stream);
}

}  // namespace

// The activation tensor map of one (pointer, K, rows, tile) on the current
// device: encoded once and kept in a small table (a forward reuses the same
// activation buffers call after call; encoding costs about a microsecond).
static bool activation_map(const __half* act, int64_t K, int64_t rows, int ntile,
                           PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap* out) {
  struct Entry {
    const void* ptr;
    int64_t K, rows;
    int ntile, device;
    CUtensorMap map;
  };
  constexpr int kEntries = 64;
  static Entry table[kEntries];
  static int used = 0, next = 0;
  static std::mutex mu;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i) {
    const Entry& e = table[i];
    if (e.ptr == act && e.K == K && e.rows == rows && e.ntile == ntile && e.device == device) {
      *out = e.map;
      return true;
    }
  }
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(ntile)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(act), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return false;
  Entry& e = table[next];
  e = Entry{act, K, rows, ntile, device, map};
  next = (next + 1) % kEntries;
  if (used < kEntries) ++used;
  *out = map;
  return true;
}

// Tile shape and K split.  128 x 128 tiles with no split when there are enough
// of them to occupy half the SMs (128 x 256 past 128 tokens); otherwise the K
// range of each 128 x 128 tile is split over a cluster of 2, 4 or 8 CTAs: as
// many as fit on the SMs, at most one slice per 256-column block, and no more
// clusters than the GPU can hold at once (a second wave would double the time).
static int prefill_k_split(int64_t M, int64_t K, int64_t batch, int num_sms) {
  const int64_t tiles128 = (M + kBM - 1) / kBM * ((batch + 127) / 128);
  const int64_t nblk = (K / kBK + 3) / 4;
  if (2 * tiles128 > num_sms) return 1;
  int ks = 1;
  while (ks < 8 && tiles128 * ks * 2 <= num_sms && ks * 2 <= nblk) ks *= 2;
  return ks;
}

// Clusters of ks split-K CTAs that can be resident at once (0 if unknown).
static int max_resident_clusters(int device, int ks, int num_sms) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(device, ks);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  auto kernel = dbf_prefill_gemm_kernel<128, true, false, false, true, false>;
  constexpr int smem = Cfg<128, true, true>::kSmemBytes;
  int n = 0;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ks * num_sms), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(ks);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
  }
  cache[key] = n;
  return n;
}

dbf_status launch_prefill_gemm(const PrefillArgs& a, const __half* act, int64_t act_rows, bool out_f32,
                               const DeviceInfo& dev, cudaStream_t stream) {
  auto encode = encode_fn();
  if (!encode) return DBF_ERR_CUDA;

  int ks = prefill_k_split(a.M, a.K, a.batch, dev.num_sms);
  const int64_t tiles128 = static_cast<int64_t>(a.M + kBM - 1) / kBM * ((a.batch + 127) / 128);
  while (ks > 1 && tiles128 > max_resident_clusters(dev.device, ks, dev.num_sms)) ks /= 2;
  // Past 128 tokens, 256-token tiles, unless they would keep fewer than half
  // the SMs busy (few weight rows): then 128-token tiles, which double the
  // tiles at the price of expanding each weight tile twice as often.
  int ntile = 128;
  if (ks == 1 && a.batch > 128) {
    const int64_t tiles256 = static_cast<int64_t>(a.M + kBM - 1) / kBM * ((a.batch + 255) / 256);
    ntile = 2 * tiles256 <= dev.num_sms ? 128 : 256;
  }
  if (static_cast<int64_t>(a.M + kBM - 1) / kBM * ((a.batch + ntile - 1) / ntile) * ks > 0x7fffffffLL)
    return DBF_ERR_UNSUPPORTED_SHAPE;

  // Stream-K past 128 tokens (when the workspace holds its partial-tile slots):
  // the 256-token tiles' (tile, 256-column block) units cut evenly over the
  // SMs.  Chosen where its estimated time beats the plan above, counted in
  // 256 x 256-column block times: stream-K takes units / SMs plus about 5 for
  // its partial tiles (measured: one partial write, one bulk-copied add and
  // the extra epilogue drains per CTA); the plan above takes its rounds of
  // tiles times the blocks per tile, a 128-token tile about 0.77 of a
  // 256-token one (half the work at a lower tensor-pipe rate), a K slice of
  // a cluster split 1/ks of a tile.
  if (a.batch > 128 && a.sk_slots != nullptr && a.sk_flags != nullptr) {
    const int64_t grid = std::min(dev.num_sms, kSkMaxCtas);
    const int64_t m_tiles = (a.M + kBM - 1) / kBM;
    const int64_t nblk = (a.K / kBK + 3) / 4;
    const int64_t units = m_tiles * ((a.batch + 255) / 256) * nblk;
    const int64_t plan_items = m_tiles * ((a.batch + ntile - 1) / ntile) * ks;
    const int64_t plan_rounds = (plan_items + dev.num_sms - 1) / dev.num_sms;
    const double plan_t = static_cast<double>(plan_rounds) * static_cast<double>(nblk) / ks * (ntile == 128 ? 0.77 : 1.0);
    const double sk_t = static_cast<double>(units) / static_cast<double>(grid) + 5.0;
    if (units >= grid && sk_t < 0.95 * plan_t) {
      CUtensorMap map;
      if (!activation_map(act, a.K, act_rows, 256, encode, &map)) return DBF_ERR_CUDA;
      return out_f32 ? launch_split<256, false, false, true>(a, map, 1, true, dev, stream)
                     : launch_split<256, false, true, true>(a, map, 1, false, dev, stream);
    }
  }

  // Wave tail.  Without a split the persistent CTAs walk the tiles in waves of
  // one tile per SM, and a last, nearly empty wave costs a whole tile time (896
  // tiles on 148 SMs: 7 rounds for 6.05 tiles' worth of work).  When leaving
  // out the last few row tiles (at most a quarter of the SMs' worth of tiles)
  // makes the rest whole waves, those rows go to a second launch of their own,
  // which the planner above gives a K split over clusters.
  if (ks == 1) {
    const int64_t m_tiles = (a.M + kBM - 1) / kBM;
    const int64_t n_tiles = (a.batch + ntile - 1) / ntile;
    if (m_tiles * n_tiles > dev.num_sms && (m_tiles * n_tiles) % dev.num_sms != 0) {
      for (int64_t t = 1; t < m_tiles && 4 * t * n_tiles <= dev.num_sms; ++t) {
        if ((m_tiles - t) * n_tiles % dev.num_sms != 0) continue;
        const int64_t rows_main = (m_tiles - t) * kBM;
        PrefillArgs head = a;
        head.M = static_cast<int>(rows_main);
        PrefillArgs tail = a;
        tail.M = a.M - static_cast<int>(rows_main);
        tail.packed = a.packed + rows_main * a.wpr;
        tail.rowscale = a.rowscale + rows_main;
        tail.out = static_cast<char*>(a.out) + rows_main * (out_f32 ? 4 : 2);
        const dbf_status st = launch_prefill_gemm(head, act, act_rows, out_f32, dev, stream);
        if (st != DBF_OK) return st;
        return launch_prefill_gemm(tail, act, act_rows, out_f32, dev, stream);
      }
    }
  }

  CUtensorMap map;
  if (!activation_map(act, a.K, act_rows, ntile, encode, &map)) return DBF_ERR_CUDA;

  if (ks > 1) return launch_split<128, true, true>(a, map, ks, out_f32, dev, stream);
  // 256-token tiles keep A in shared memory for fp32 outputs (the single
  // accumulator's drain would take twice as long)
  if (ntile == 256)
    return out_f32 ? launch_split<256, false, false>(a, map, 1, true, dev, stream)
                   : launch_split<256, false, true>(a, map, 1, false, dev, stream);
  return launch_split<128, false, true>(a, map, 1, out_f32, dev, stream);
}

}  // namespace dbf
