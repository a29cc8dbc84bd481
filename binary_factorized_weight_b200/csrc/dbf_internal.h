// Internal host-side declarations shared by the libdbf translation units.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/dbf.h"

namespace dbf {

// One sign-product stage of the decode path:
//   out[tok][row] = rowscale[row] * sum_K sign(row, K) * u[tok][K],
//   u = fp16(act (.) kscale) (or act itself when kscale is null).
struct DecodeArgs {
  const uint32_t* packed;  // M rows of packed signs, wpr words per row
  int64_t wpr;
  int M;                   // rows (outputs of this stage)
  int K;                   // reduction length (multiple of 64)
  const __half* act;       // batch x K activations, row stride ld_act
  int64_t ld_act;
  const __half* kscale;    // K entries or nullptr
  const __half* rowscale;  // M entries
  void* out;               // batch x M, row stride ld_out (fp16 or fp32)
  int64_t ld_out;
  int batch;               // 1..16
  int kchunk;              // K elements per cluster rank (multiple of 256)
  int weights_early;       // may read packed/kscale/rowscale before the PDL wait
  int peer_rows;           // rows of the forward's other stage (shapes the work split)
  int* status;             // device status word (DBF_ERR_TIMEOUT on a lost wait)
};

// One sign-product GEMM of the prefill path (same formula, tcgen05).
struct PrefillArgs {
  const uint32_t* packed;
  int64_t wpr;
  int M;
  int K;
  const __half* kscale;
  const __half* rowscale;
  void* out;
  int64_t ld_out;
  int batch;
  int weights_early;
  int* status;  // device status word (DBF_ERR_TIMEOUT on a lost wait)
  // stream-K scratch (null: no stream-K schedule): kSkMaxCtas partial tiles of
  // 128 x 256 fp32 and kSkMaxCtas flags, zero between launches
  float* sk_slots;
  unsigned* sk_flags;
};

// Stream-K: at most this many CTAs, one partial tile slot each.
constexpr int kSkMaxCtas = 160;
constexpr size_t kSkFlagBytes = 1024;  // kSkMaxCtas 32-bit flags, padded
constexpr size_t kSkSlotBytes = size_t{128} * 256 * 4;
constexpr size_t kSkBytes = kSkFlagBytes + kSkMaxCtas * kSkSlotBytes;

struct DeviceInfo {
  int device;
  int num_sms;
  int cc_major, cc_minor;
};

dbf_status current_device(DeviceInfo* info);

// The smallest workspace dbf_forward accepts (status block and V); the
// optional areas after it enable the single-launch decode and stream-K.
size_t forward_workspace_min_bytes(int64_t k, int64_t batch);

// The synchronous argument checks of dbf_forward other than the workspace
// (shared by every entry point that runs the layer forward).
dbf_status validate_forward_args(const uint16_t* x, const uint32_t* packedA, const uint32_t* packedB,
                                 const uint16_t* a, const uint16_t* m, const uint16_t* b, int64_t n, int64_t k,
                                 int64_t m_in, int64_t batch, const void* y, dbf_dtype y_t, uint32_t flags);

dbf_status launch_decode_stage(const DecodeArgs& args, bool class_expand, bool lut, bool out_f32, const DeviceInfo& dev,
                               cudaStream_t stream);

// Several decode stages in one launch (layers that share their input: the
// stage-B products of q, k and v, say, or their stage-A products).  Each layer's
// rows are padded to whole 64-row CTA tiles; tile t belongs to the layer g with
// tile_start[g] <= t < tile_start[g+1].  All layers share the kernel variant
// (batch, kscale or not, output type) and the K split of the launch.
constexpr int kMaxGroup = 8;
struct DecodeGroup {
  int n;
  int tile_start[kMaxGroup + 1];
  DecodeArgs layer[kMaxGroup];
};

// Fills tile_start and each layer's kchunk, then launches.  peer_rows: rows of
// the forward's other stage (all layers).
dbf_status launch_decode_group(DecodeGroup& group, int64_t peer_rows, bool class_expand, bool lut, bool out_f32,
                               const DeviceInfo& dev, cudaStream_t stream);

// The single-launch decode forward (fused.cu): grid (R, J), clusters of R
// CTAs along x, one cluster per slice of kb middle rows.
constexpr int kFusedMaxSlices = 8;
struct FusedArgs {
  const __half* x;
  int64_t ld_x;
  const uint32_t* packedB;  // k rows over m_in
  int64_t wprB;
  const uint32_t* packedA;  // n rows over k
  int64_t wprA;
  const __half* a;
  const __half* mid;
  const __half* b;
  void* y;
  int64_t ld_y;
  int n, k, m_in, batch;     // batch 1..16
  int MB;                    // 256-column blocks of m_in
  int R;                     // CTAs per cluster (power of two <= 16)
  int J;                     // clusters (slices of k)
  int kb;                    // middle rows per slice (multiple of 256)
  int nb;                    // output rows per rank (multiple of 16)
  int weights_early;
  int test_lose_bytes;       // test only: rank 0 waits for bytes that never come
  int* status;
  unsigned long long* slots; // batch x n x 8 tagged partials (word j - 1 from slice j)
};

// Fills the sizes of `args` for this shape; false if the shape does not fit
// the single-launch kernel (then the two-launch path runs).
bool plan_fused(int64_t n, int64_t k, int64_t m_in, int batch, FusedArgs* args, size_t* smem_bytes);
dbf_status launch_fused_decode(const FusedArgs& args, size_t smem_bytes, bool out_f32, cudaStream_t stream);

dbf_status launch_prefill_gemm(const PrefillArgs& args, const __half* act, int64_t act_rows, bool out_f32,
                               const DeviceInfo& dev, cudaStream_t stream);

dbf_status launch_pack(const void* src, dbf_dtype src_t, int64_t rows, int64_t cols, uint32_t* packed,
                       const DeviceInfo& dev, cudaStream_t stream);

dbf_status launch_transpose_signs(const uint32_t* packed, int64_t rows, int64_t cols, uint32_t* out,
                                  const DeviceInfo& dev, cudaStream_t stream);

dbf_status launch_reconstruct(const uint32_t* packedA, const uint32_t* packedB, const __half* a, const __half* mid,
                              const __half* b, int64_t n, int64_t k, int64_t m_in, void* W, bool out_f32,
                              const DeviceInfo& dev, cudaStream_t stream);

inline int64_t words_per_row(int64_t cols) { return cols <= 0 ? 0 : ((cols + 255) / 256) * 8; }

// Plain launch that reports this launch's own error (not a pending one).
template <typename... KArgs, typename... Args>
inline dbf_status launch_plain(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.numAttrs = 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess ? DBF_OK : DBF_ERR_CUDA;
}

}  // namespace dbf
