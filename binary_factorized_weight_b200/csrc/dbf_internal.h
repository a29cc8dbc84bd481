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
};

struct DeviceInfo {
  int device;
  int num_sms;
  int cc_major, cc_minor;
};

dbf_status current_device(DeviceInfo* info);

dbf_status launch_decode_stage(const DecodeArgs& args, bool class_expand, bool out_f32, const DeviceInfo& dev,
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
dbf_status launch_decode_group(DecodeGroup& group, int64_t peer_rows, bool class_expand, bool out_f32,
                               const DeviceInfo& dev, cudaStream_t stream);

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
