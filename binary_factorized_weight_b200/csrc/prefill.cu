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
// Stage hand-off is through mbarriers; every wait is bounded and an expired
// wait records DBF_ERR_TIMEOUT in the workspace status word, raises a CTA-wide
// abort flag and lets all roles fall through to the teardown, which frees TMEM
// only after this CTA's MMAs are known to be complete.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
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

template <int NTILE>
struct Cfg {
  static constexpr int kStages = NTILE == 256 ? 4 : 6;
  static constexpr int kBBytes = NTILE * kBK * 2;
  static constexpr int kEpiOffset = kStages * (kABytes + kBBytes);
  static constexpr int kBarOffset = kEpiOffset + 4 * kEpiStageBytes;
  // full_a[S], full_b[S], empty[S], acc_full[2], acc_empty[2], mma_done
  static constexpr int kNumBars = 3 * kStages + 5;
  static constexpr int kSmemBytes = kBarOffset + kNumBars * 8 + 16 + 1024;  // + tmem slot/abort + align slack
  static constexpr int kTmemCols = 2 * NTILE;
};

template <int NTILE, bool KSCALE, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    dbf_prefill_gemm_kernel(const __grid_constant__ CUtensorMap act_map, const PrefillArgs p) {
  using C = Cfg<NTILE>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_st = smem;
  uint8_t* b_st = smem + S * kABytes;
  uint8_t* epi_st = smem + C::kEpiOffset;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* full_a = bars;
  uint64_t* full_b = bars + S;
  uint64_t* empty = bars + 2 * S;
  uint64_t* acc_full = bars + 3 * S;
  uint64_t* acc_empty = bars + 3 * S + 2;
  uint64_t* mma_done = bars + 3 * S + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int m_tiles = (p.M + kBM - 1) / kBM;
  const int num_tiles = m_tiles * ((p.batch + NTILE - 1) / NTILE);
  const int KT = p.K / kBK;

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
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kWarpTma) {
    // ------------------------------------------------ sign expansion
    // Row r's packed row is a sequence of 8-word blocks of 256 columns; K step
    // kt covers groups 4*(kt%4) .. 4*(kt%4)+3 of block kt/4, and group g's 16
    // columns come from bit pair (g, g+16) of the block's 8 words.  This thread
    // holds words 4h..4h+3 (column pairs 4h..4h+3 of every group).
    const int r_local = tid & (kBM - 1);
    const int h = tid >> 7;
    const int nblk = (KT + 3) / 4;
    // block sequence of this CTA: (tile, blk) with blk fastest
    int f_tile = blockIdx.x, f_blk = 0;
    auto fetch_next = [&]() -> uint4 {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (f_tile < num_tiles) {
        const int r = (f_tile % m_tiles) * kBM + r_local;
        if (r < p.M) v = ldg_stream_u4(p.packed + static_cast<int64_t>(r) * p.wpr + 8 * f_blk + 4 * h);
        if (++f_blk == nblk) {
          f_blk = 0;
          f_tile += gridDim.x;
        }
      }
      return v;
    };
    auto fetch_scale = [&](int kt, uint4 (&sc)[4]) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        sc[i] = __ldg(reinterpret_cast<const uint4*>(p.kscale + kt * kBK + 16 * i + 8 * h));
    };
    uint4 w_n1, w_n2, wcur = make_uint4(0u, 0u, 0u, 0u);
    uint4 sc_next[4];
    if (p.weights_early) {
      w_n1 = fetch_next();
      w_n2 = fetch_next();
      if constexpr (KSCALE) fetch_scale(0, sc_next);
    }
    pdl_wait();
    if (!p.weights_early) {
      w_n1 = fetch_next();
      w_n2 = fetch_next();
      if constexpr (KSCALE) fetch_scale(0, sc_next);
    }
    bool ok = true;
    const int swz = r_local & 7;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kt = 0; kt < KT; ++kt, ++it) {
        const int s = static_cast<int>(it % S);
        const uint32_t use = it / S;
        if ((kt & 3) == 0) {
          wcur = w_n1;
          w_n1 = w_n2;
          w_n2 = fetch_next();
        }
        uint4 sc[4];
        if constexpr (KSCALE) {
#pragma unroll
          for (int i = 0; i < 4; ++i) sc[i] = sc_next[i];
          fetch_scale(kt + 1 < KT ? kt + 1 : 0, sc_next);
        }
        if (it >= S && !mbar_wait_bounded(&empty[s], (use - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        uint8_t* dst = a_st + s * kABytes + (r_local >> 3) * 1024 + swz * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int g = 4 * (kt & 3) + i;  // group inside the block
          uint32_t q[4];
          if constexpr (KSCALE) {
            q[0] = signed_scale_pair_rt(wcur.x, g, sc[i].x);
            q[1] = signed_scale_pair_rt(wcur.y, g, sc[i].y);
            q[2] = signed_scale_pair_rt(wcur.z, g, sc[i].z);
            q[3] = signed_scale_pair_rt(wcur.w, g, sc[i].w);
          } else {
            q[0] = pm1_pair_rt(wcur.x, g);
            q[1] = pm1_pair_rt(wcur.y, g);
            q[2] = pm1_pair_rt(wcur.z, g);
            q[3] = pm1_pair_rt(wcur.w, g);
          }
          // columns 16i + 8h .. 16i + 8h + 7 -> 16-byte chunk 2i + h (128B swizzle)
          *reinterpret_cast<uint4*>(dst + (((2 * i + h) ^ swz) << 4)) = make_uint4(q[0], q[1], q[2], q[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&full_a[s]);
      }
    }
  } else if (warp == kWarpTma) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      pdl_wait();
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int n0 = (tile / m_tiles) * NTILE;
        for (int kt = 0; kt < KT; ++kt, ++it) {
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
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const uint32_t buf = local & 1;
        if (local >= 2 && !mbar_wait_bounded(&acc_empty[buf], ((local >> 1) - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * NTILE;
        for (int kt = 0; kt < KT; ++kt, ++it) {
          const int s = static_cast<int>(it % S);
          const uint32_t par = (it / S) & 1;
          if (!mbar_wait_bounded(&full_a[s], par, abort_flag, p.status) ||
              !mbar_wait_bounded(&full_b[s], par, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(a_st + s * kABytes);
          const uint32_t b_addr = smem_u32(b_st + s * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            tc_mma_f16_ss(d_tmem, smem_desc_sw128_kmajor(a_addr + kk * 32), smem_desc_sw128_kmajor(b_addr + kk * 32),
                          idesc, (kt | kk) != 0 ? 1u : 0u);
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
    constexpr int kVec = 16 / sizeof(OutT);  // outputs per 16-byte store
    const int q = warp & 3;                  // TMEM lane quadrant this warp may access
    OutT* stg = reinterpret_cast<OutT*>(epi_st + (warp - kWarpEpi0) * kEpiStageBytes);  // [32 tokens][32 rows]
    OutT* out = static_cast<OutT*>(p.out);
    const bool ld_ok = (p.ld_out % kVec) == 0;
    uint32_t local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const uint32_t buf = local & 1;
      if (!mbar_wait_bounded(&acc_full[buf], (local >> 1) & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const int m0 = (tile % m_tiles) * kBM;
      const int n0 = (tile / m_tiles) * NTILE;
      const int row0 = m0 + q * 32;
      const int row = row0 + lane;
      const float rs = (row < p.M) ? __half2float(p.rowscale[row]) : 0.f;
      const bool rows_full = row0 + 32 <= p.M;
      for (int col = 0; col < NTILE; col += 32) {
        if (n0 + col >= p.batch) break;  // warp-uniform
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * NTILE + static_cast<uint32_t>(col),
                           v);
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

template <int NTILE, bool KSCALE, bool OUT_F32>
dbf_status launch_typed(const PrefillArgs& a, const CUtensorMap& map, const DeviceInfo& dev, cudaStream_t stream) {
  auto kernel = dbf_prefill_gemm_kernel<NTILE, KSCALE, OUT_F32>;
  constexpr int smem = Cfg<NTILE>::kSmemBytes;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DBF_ERR_CUDA;
  const int64_t m_tiles = (a.M + kBM - 1) / kBM;
  const int64_t n_tiles = (a.batch + NTILE - 1) / NTILE;
  const int64_t grid = std::min<int64_t>(m_tiles * n_tiles, dev.num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, map, a) == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

}  // namespace

dbf_status launch_prefill_gemm(const PrefillArgs& a, const __half* act, int64_t act_rows, bool out_f32,
                               const DeviceInfo& dev, cudaStream_t stream) {
  auto encode = encode_fn();
  if (!encode) return DBF_ERR_CUDA;
  const int ntile = a.batch > 128 ? 256 : 128;
  if (static_cast<int64_t>(a.M + kBM - 1) / kBM * ((a.batch + ntile - 1) / ntile) > 0x7fffffffLL)
    return DBF_ERR_UNSUPPORTED_SHAPE;

  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(act_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(ntile)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(act), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return DBF_ERR_CUDA;

  const bool ks = a.kscale != nullptr;
  if (ntile == 256) {
    if (ks) return out_f32 ? launch_typed<256, true, true>(a, map, dev, stream) : launch_typed<256, true, false>(a, map, dev, stream);
    return out_f32 ? launch_typed<256, false, true>(a, map, dev, stream) : launch_typed<256, false, false>(a, map, dev, stream);
  }
  if (ks) return out_f32 ? launch_typed<128, true, true>(a, map, dev, stream) : launch_typed<128, true, false>(a, map, dev, stream);
  return out_f32 ? launch_typed<128, false, true>(a, map, dev, stream) : launch_typed<128, false, false>(a, map, dev, stream);
}

}  // namespace dbf
