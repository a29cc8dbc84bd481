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
// Roles (320 threads):
//   warps 0-3  sign expansion: thread r turns row r's packed bits of a K step
//              into 64 fp16 values (+-1, or +-b_j with b folded in by flipping
//              the scale's sign bit: exact) stored as one 128-byte row of a
//              128B-swizzled K-major tile;
//   warp 4     TMA producer of the activation tile (K-major, 128B swizzle,
//              tokens past the batch read as zero);
//   warp 5     TMEM allocation and the single-thread tcgen05.mma issue loop;
//   warps 6-9  epilogue: TMEM -> registers -> row scale -> global stores
//              (warp w reads TMEM lanes 32*(w%4) .. 32*(w%4)+31).
// Stage hand-off is through mbarriers; every wait is bounded and an expired
// wait records DBF_ERR_TIMEOUT in the workspace status word, raises a CTA-wide
// abort flag and lets all roles fall through to the teardown, which frees TMEM
// only after this CTA's MMAs are known to be complete.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "dbf_device.cuh"
#include "dbf_internal.h"

namespace dbf {
namespace {

constexpr int kBM = 128;  // weight rows per tile (TMEM lanes)
constexpr int kBK = 64;   // K per pipeline stage: one 128-byte swizzle row of fp16
constexpr int kThreads = 320;
constexpr int kABytes = kBM * kBK * 2;

template <int NTILE>
struct Cfg {
  static constexpr int kStages = NTILE == 256 ? 4 : 6;
  static constexpr int kBBytes = NTILE * kBK * 2;
  static constexpr int kBarOffset = kStages * (kABytes + kBBytes);
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
      mbar_init(&full_a[i], 128);
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
  if (warp == 4 && lane == 0) prefetch_tmap(&act_map);
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------ sign expansion
    // Row r's packed row is a sequence of 8-word blocks of 256 columns; K step
    // kt covers groups 4*(kt%4) .. 4*(kt%4)+3 of block kt/4.  Group g's 16
    // columns come from bit pair (g, g+16) of the block's 8 words.  The next
    // block (possibly the first block of this CTA's next tile) is always in
    // flight while the current one is expanded.
    const int nblk = (KT + 3) / 4;
    auto block_ptr = [&](int tile, int blk) -> const uint4* {
      const int r = (tile % m_tiles) * kBM + tid;
      if (tile >= num_tiles || r >= p.M) return nullptr;
      return reinterpret_cast<const uint4*>(p.packed + static_cast<int64_t>(r) * p.wpr) + 2 * blk;
    };
    int tile = blockIdx.x;
    uint4 nxt0 = make_uint4(0u, 0u, 0u, 0u), nxt1 = nxt0;
    auto fetch = [&](const uint4* q) {
      if (q) {
        nxt0 = __ldg(q);
        nxt1 = __ldg(q + 1);
      } else {
        nxt0 = nxt1 = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    if (p.weights_early) fetch(block_ptr(tile, 0));
    pdl_wait();
    if (!p.weights_early) fetch(block_ptr(tile, 0));
    uint32_t w[8];
    bool ok = true;
    const int swz = tid & 7;
    uint32_t it = 0;
    for (; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kt = 0; kt < KT; ++kt, ++it) {
        const int s = static_cast<int>(it % S);
        const uint32_t use = it / S;
        if ((kt & 3) == 0) {
          w[0] = nxt0.x; w[1] = nxt0.y; w[2] = nxt0.z; w[3] = nxt0.w;
          w[4] = nxt1.x; w[5] = nxt1.y; w[6] = nxt1.z; w[7] = nxt1.w;
          const int nb = (kt >> 2) + 1;
          fetch(nb < nblk ? block_ptr(tile, nb) : block_ptr(tile + gridDim.x, 0));
        }
        if (it >= S && !mbar_wait_bounded(&empty[s], (use - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        uint8_t* dst = a_st + s * kABytes + (tid >> 3) * 1024 + swz * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int g = 4 * (kt & 3) + i;  // group inside the block
          uint32_t h[8];
          if constexpr (KSCALE) {
            const uint4* sc = reinterpret_cast<const uint4*>(p.kscale + kt * kBK + 16 * i);
            const uint4 s0 = __ldg(sc), s1 = __ldg(sc + 1);
            h[0] = signed_scale_pair_rt(w[0], g, s0.x);
            h[1] = signed_scale_pair_rt(w[1], g, s0.y);
            h[2] = signed_scale_pair_rt(w[2], g, s0.z);
            h[3] = signed_scale_pair_rt(w[3], g, s0.w);
            h[4] = signed_scale_pair_rt(w[4], g, s1.x);
            h[5] = signed_scale_pair_rt(w[5], g, s1.y);
            h[6] = signed_scale_pair_rt(w[6], g, s1.z);
            h[7] = signed_scale_pair_rt(w[7], g, s1.w);
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) h[q] = pm1_pair_rt(w[q], g);
          }
          // columns 16i..16i+7 -> 16-byte chunk 2i, 16i+8..16i+15 -> chunk 2i+1 (128B swizzle)
          *reinterpret_cast<uint4*>(dst + (((2 * i) ^ swz) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(dst + (((2 * i + 1) ^ swz) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&full_a[s]);
      }
    }
  } else if (warp == 4) {
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
  } else if (warp == 5) {
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
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    uint32_t local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const uint32_t buf = local & 1;
      if (!mbar_wait_bounded(&acc_full[buf], (local >> 1) & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const int m0 = (tile % m_tiles) * kBM;
      const int n0 = (tile / m_tiles) * NTILE;
      const int row = m0 + q * 32 + lane;
      const float rs = (row < p.M) ? __half2float(p.rowscale[row]) : 0.f;
      for (int col = 0; col < NTILE; col += 32) {
        if (n0 + col >= p.batch) break;  // warp-uniform
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * NTILE + static_cast<uint32_t>(col),
                           v);
        tmem_ld_wait();
        if (row < p.M) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tok = n0 + col + j;
            if (tok < p.batch) {
              const float val = rs * __uint_as_float(v[j]);
              if constexpr (OUT_F32) {
                static_cast<float*>(p.out)[static_cast<int64_t>(tok) * p.ld_out + row] = val;
              } else {
                static_cast<__half*>(p.out)[static_cast<int64_t>(tok) * p.ld_out + row] = __float2half_rn(val);
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
  if (warp == 5) {
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
