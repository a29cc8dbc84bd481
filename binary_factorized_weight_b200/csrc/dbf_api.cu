// extern "C" entry points of libdbf (declared in include/dbf.h): argument
// validation, path selection and launches.  Validation runs before anything
// is enqueued; a call that fails it has no effect on the stream.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "dbf_internal.h"

namespace dbf {

namespace {
constexpr int kMaxDevices = 64;
constexpr int64_t kMaxReduce = int64_t{1} << 20;  // k, m_in
constexpr int64_t kMaxRows = int64_t{1} << 24;    // n, batch
constexpr size_t kStatusBytes = 256;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

dbf_status current_device(DeviceInfo* info) {
  static DeviceInfo cache[kMaxDevices];
  static std::once_flag flags[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DBF_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DBF_ERR_DEVICE;
  bool ok = true;
  std::call_once(flags[dev], [&] {
    DeviceInfo d{};
    d.device = dev;
    ok = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
         cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
         cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess;
    if (!ok) d.cc_major = -1;
    cache[dev] = d;
  });
  *info = cache[dev];
  if (info->cc_major < 0) return DBF_ERR_CUDA;
  // The library is built for sm_100a only.
  if (info->cc_major != 10 || info->cc_minor != 0) return DBF_ERR_DEVICE;
  return DBF_OK;
}

}  // namespace dbf

using namespace dbf;

extern "C" {

int64_t dbf_packed_words_per_row(int64_t cols) { return words_per_row(cols); }

int64_t dbf_packed_words(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 0;
  return rows * words_per_row(cols);
}

const char* dbf_status_string(dbf_status s) {
  switch (s) {
    case DBF_OK: return "DBF_OK: success";
    case DBF_ERR_INVALID_ARG: return "DBF_ERR_INVALID_ARG: null pointer, bad size, unknown dtype or flag";
    case DBF_ERR_UNSUPPORTED_SHAPE: return "DBF_ERR_UNSUPPORTED_SHAPE: shape outside the supported contract";
    case DBF_ERR_MISALIGNED: return "DBF_ERR_MISALIGNED: pointer not 16-byte aligned";
    case DBF_ERR_WORKSPACE: return "DBF_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case DBF_ERR_CUDA: return "DBF_ERR_CUDA: a CUDA call or kernel launch failed";
    case DBF_ERR_TIMEOUT: return "DBF_ERR_TIMEOUT: a bounded device-side wait gave up";
    case DBF_ERR_DEVICE: return "DBF_ERR_DEVICE: current device is not sm_100 (B200-class)";
  }
  return "unknown dbf_status";
}

dbf_status dbf_pack_signs(const void* src, dbf_dtype src_t, int64_t rows, int64_t cols, uint32_t* packed,
                          struct CUstream_st* stream) {
  if (!src || !packed) return DBF_ERR_INVALID_ARG;
  if (src_t != DBF_I8 && src_t != DBF_F16 && src_t != DBF_F32) return DBF_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1) return DBF_ERR_INVALID_ARG;
  if (rows > kMaxRows || cols > kMaxRows || rows * words_per_row(cols) > (int64_t{1} << 40))
    return DBF_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(packed)) return DBF_ERR_MISALIGNED;
  const size_t esz = src_t == DBF_I8 ? 1 : (src_t == DBF_F16 ? 2 : 4);
  if ((reinterpret_cast<uintptr_t>(src) % esz) != 0) return DBF_ERR_MISALIGNED;
  DeviceInfo dev;
  dbf_status st = current_device(&dev);
  if (st != DBF_OK) return st;
  return launch_pack(src, src_t, rows, cols, packed, dev, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {
// Workspace layout: status block, V (batch x k fp16, the two-launch and
// tensor-core paths), then either the tagged partials of the single-launch
// decode (batch x n x 8 64-bit words; batch <= 16) or the stream-K flags and
// partial-tile slots of the tensor-core path (batch > 128).  The last area is
// optional: with less room the forward runs a schedule that does not use it.
size_t v_area_end(int64_t k, int64_t batch) {
  const size_t v_bytes = static_cast<size_t>(batch) * static_cast<size_t>(k) * 2;
  return kStatusBytes + (v_bytes + 255) / 256 * 256;
}
size_t sk_area_bytes(int64_t batch) { return batch > 128 ? kSkBytes : 0; }
size_t slot_bytes(int64_t n, int64_t tokens) {
  return static_cast<size_t>(kFusedMaxSlices) * static_cast<size_t>(tokens) * static_cast<size_t>(n) * 8;
}
}  // namespace

size_t dbf::forward_workspace_min_bytes(int64_t k, int64_t batch) {
  if (k < 1 || batch < 1) return 0;
  return v_area_end(k, batch);
}

extern "C" {

size_t dbf_forward_workspace_bytes(int64_t n, int64_t k, int64_t m_in, int64_t batch) {
  if (n < 1 || k < 1 || m_in < 1 || batch < 1) return 0;
  return v_area_end(k, batch) + (batch <= 16 ? slot_bytes(n, batch) : 0) + sk_area_bytes(batch);
}

static dbf_status validate_factors(const uint32_t* packedA, const uint32_t* packedB, const uint16_t* a,
                                   const uint16_t* m, const uint16_t* b, int64_t n, int64_t k, int64_t m_in) {
  if (!packedA || !packedB || !a || !m || !b) return DBF_ERR_INVALID_ARG;
  if (n < 1 || k < 1 || m_in < 1) return DBF_ERR_INVALID_ARG;
  if (k % 64 != 0 || m_in % 64 != 0 || k > kMaxReduce || m_in > kMaxReduce || n > kMaxRows)
    return DBF_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(packedA) || !aligned16(packedB) || !aligned16(a) || !aligned16(m) || !aligned16(b))
    return DBF_ERR_MISALIGNED;
  return DBF_OK;
}

}  // extern "C"

namespace dbf {
dbf_status validate_forward_args(const uint16_t* x, const uint32_t* packedA, const uint32_t* packedB,
                                 const uint16_t* a, const uint16_t* m, const uint16_t* b, int64_t n, int64_t k,
                                 int64_t m_in, int64_t batch, const void* y, dbf_dtype y_t, uint32_t flags) {
  if (!x || !y) return DBF_ERR_INVALID_ARG;
  dbf_status st = validate_factors(packedA, packedB, a, m, b, n, k, m_in);
  if (st != DBF_OK) return st;
  if (batch < 1) return DBF_ERR_INVALID_ARG;
  if (batch > kMaxRows) return DBF_ERR_UNSUPPORTED_SHAPE;
  if (y_t != DBF_F16 && y_t != DBF_F32) return DBF_ERR_INVALID_ARG;
  const uint32_t known = DBF_FWD_WEIGHTS_STATIC | DBF_FWD_FORCE_DECODE | DBF_FWD_FORCE_PREFILL |
                         DBF_FWD_DECODE_SHIFT_EXPAND | DBF_FWD_DECODE_TWO_STAGE | DBF_FWD_DECODE_SINGLE |
                         DBF_FWD_DECODE_TABLE |
                         DBF_FWD_TEST_LOSE_ARRIVAL;
  if ((flags & ~known) != 0) return DBF_ERR_INVALID_ARG;
  if ((flags & DBF_FWD_DECODE_SINGLE) &&
      (flags & (DBF_FWD_DECODE_TWO_STAGE | DBF_FWD_DECODE_SHIFT_EXPAND | DBF_FWD_DECODE_TABLE)))
    return DBF_ERR_INVALID_ARG;
  if ((flags & DBF_FWD_DECODE_TABLE) && (flags & DBF_FWD_DECODE_SHIFT_EXPAND)) return DBF_ERR_INVALID_ARG;
  if ((flags & DBF_FWD_FORCE_DECODE) && (flags & DBF_FWD_FORCE_PREFILL)) return DBF_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return DBF_ERR_MISALIGNED;
  return DBF_OK;
}
}  // namespace dbf

extern "C" {

dbf_status dbf_forward(const uint16_t* x, const uint32_t* packedA, const uint32_t* packedB, const uint16_t* a,
                       const uint16_t* m, const uint16_t* b, int64_t n, int64_t k, int64_t m_in, int64_t batch,
                       void* y, dbf_dtype y_t, void* workspace, size_t ws_bytes, uint32_t flags,
                       struct CUstream_st* stream_handle) {
  dbf_status st = validate_forward_args(x, packedA, packedB, a, m, b, n, k, m_in, batch, y, y_t, flags);
  if (st != DBF_OK) return st;
  if (!workspace || !aligned16(workspace) || ws_bytes < v_area_end(k, batch)) return DBF_ERR_WORKSPACE;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != DBF_OK) return st;

  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_handle);
  const bool out_f32 = y_t == DBF_F32;
  const bool early = (flags & DBF_FWD_WEIGHTS_STATIC) != 0;
  int* status = static_cast<int*>(workspace);
  __half* V = reinterpret_cast<__half*>(static_cast<char*>(workspace) + kStatusBytes);
  const __half* xh = reinterpret_cast<const __half*>(x);
  const __half* ah = reinterpret_cast<const __half*>(a);
  const __half* mh = reinterpret_cast<const __half*>(m);
  const __half* bh = reinterpret_cast<const __half*>(b);
  const size_t y_elt = out_f32 ? 4 : 2;

  const bool decode = (flags & DBF_FWD_FORCE_DECODE) || (!(flags & DBF_FWD_FORCE_PREFILL) && batch <= 16);
  if (decode) {
    const bool class_expand = (flags & DBF_FWD_DECODE_SHIFT_EXPAND) == 0;
    // one token: the lookup-table kernel when asked for
    const bool lut = (flags & DBF_FWD_DECODE_TABLE) != 0;
    // the single-launch kernel when asked for (its measured per-layer time
    // does not yet beat the two launches on any layer shape of the workloads)
    const bool two_stage = (flags & DBF_FWD_DECODE_SINGLE) == 0;
    for (int64_t t0 = 0; t0 < batch; t0 += 16) {
      const int nb = static_cast<int>(batch - t0 < 16 ? batch - t0 : 16);
      // one launch for the whole layer where the shape fits the kernel and the
      // workspace has room for the cross-cluster partials
      FusedArgs fa{};
      size_t fsmem = 0;
      if (!two_stage && plan_fused(n, k, m_in, nb, &fa, &fsmem) &&
          ws_bytes >= v_area_end(k, batch) + slot_bytes(n, nb)) {
        fa.x = xh + t0 * m_in;
        fa.ld_x = m_in;
        fa.packedB = packedB;
        fa.wprB = words_per_row(m_in);
        fa.packedA = packedA;
        fa.wprA = words_per_row(k);
        fa.a = ah;
        fa.mid = mh;
        fa.b = bh;
        fa.y = static_cast<char*>(y) + static_cast<size_t>(t0) * static_cast<size_t>(n) * y_elt;
        fa.ld_y = n;
        fa.weights_early = early ? 1 : 0;
        fa.test_lose_bytes = (flags & DBF_FWD_TEST_LOSE_ARRIVAL) ? 1 : 0;
        fa.status = status;
        fa.slots = reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) + v_area_end(k, batch));
        st = launch_fused_decode(fa, fsmem, out_f32, stream);
        if (st == DBF_OK) continue;
        (void)cudaGetLastError();  // the launch was refused (e.g. no room for the cluster): two launches instead
      }
      DecodeArgs sb{};
      sb.packed = packedB;
      sb.wpr = words_per_row(m_in);
      sb.M = static_cast<int>(k);
      sb.K = static_cast<int>(m_in);
      sb.act = xh + t0 * m_in;
      sb.ld_act = m_in;
      sb.kscale = bh;
      sb.rowscale = mh;
      sb.out = V + t0 * k;
      sb.ld_out = k;
      sb.batch = nb;
      sb.weights_early = early ? 1 : 0;
      sb.peer_rows = static_cast<int>(n);
      sb.status = status;
      st = launch_decode_stage(sb, class_expand, lut, /*out_f32=*/false, dev, stream);
      if (st != DBF_OK) return st;
      DecodeArgs sa{};
      sa.packed = packedA;
      sa.wpr = words_per_row(k);
      sa.M = static_cast<int>(n);
      sa.K = static_cast<int>(k);
      sa.act = V + t0 * k;
      sa.ld_act = k;
      sa.kscale = nullptr;
      sa.rowscale = ah;
      sa.out = static_cast<char*>(y) + static_cast<size_t>(t0) * static_cast<size_t>(n) * y_elt;
      sa.ld_out = n;
      sa.batch = nb;
      sa.weights_early = 1;  // stage B releases stage A only after its own wait
      sa.peer_rows = static_cast<int>(k);
      sa.status = status;
      st = launch_decode_stage(sa, class_expand, lut, out_f32, dev, stream);
      if (st != DBF_OK) return st;
    }
    return DBF_OK;
  }

  // stream-K scratch after V, when the workspace has room for it
  char* sk = ws_bytes >= v_area_end(k, batch) + kSkBytes ? static_cast<char*>(workspace) + v_area_end(k, batch)
                                                         : nullptr;
  PrefillArgs g1{};
  g1.sk_flags = sk ? reinterpret_cast<unsigned*>(sk) : nullptr;
  g1.sk_slots = sk ? reinterpret_cast<float*>(sk + kSkFlagBytes) : nullptr;
  g1.packed = packedB;
  g1.wpr = words_per_row(m_in);
  g1.M = static_cast<int>(k);
  g1.K = static_cast<int>(m_in);
  g1.kscale = bh;
  g1.rowscale = mh;
  g1.out = V;
  g1.ld_out = k;
  g1.batch = static_cast<int>(batch);
  g1.weights_early = early ? 1 : 0;
  g1.status = status;
  st = launch_prefill_gemm(g1, xh, batch, /*out_f32=*/false, dev, stream);
  if (st != DBF_OK) return st;
  PrefillArgs g2{};
  g2.sk_flags = g1.sk_flags;
  g2.sk_slots = g1.sk_slots;
  g2.packed = packedA;
  g2.wpr = words_per_row(k);
  g2.M = static_cast<int>(n);
  g2.K = static_cast<int>(k);
  g2.kscale = nullptr;
  g2.rowscale = ah;
  g2.out = y;
  g2.ld_out = n;
  g2.batch = static_cast<int>(batch);
  g2.weights_early = 1;
  g2.status = status;
  return launch_prefill_gemm(g2, V, batch, out_f32, dev, stream);
}

static size_t grouped_v_offset(const dbf_layer_desc* layers, int g, int64_t batch) {
  size_t off = kStatusBytes;
  for (int h = 0; h < g; ++h) off += (static_cast<size_t>(batch) * static_cast<size_t>(layers[h].k) * 2 + 255) / 256 * 256;
  return off;
}

size_t dbf_forward_grouped_workspace_bytes(const dbf_layer_desc* layers, int num_layers, int64_t m_in,
                                           int64_t batch) {
  if (!layers || num_layers < 1 || num_layers > DBF_MAX_GROUP || m_in < 1 || batch < 1) return 0;
  for (int g = 0; g < num_layers; ++g)
    if (layers[g].n < 1 || layers[g].k < 1) return 0;
  return grouped_v_offset(layers, num_layers, batch) + sk_area_bytes(batch);
}

dbf_status dbf_forward_grouped(const uint16_t* x, int64_t m_in, int64_t batch, const dbf_layer_desc* layers,
                               int num_layers, dbf_dtype y_t, void* workspace, size_t ws_bytes, uint32_t flags,
                               struct CUstream_st* stream_handle) {
  if (!x || !layers) return DBF_ERR_INVALID_ARG;
  if (num_layers < 1 || num_layers > DBF_MAX_GROUP) return DBF_ERR_INVALID_ARG;
  for (int g = 0; g < num_layers; ++g) {
    const dbf_layer_desc& l = layers[g];
    if (!l.y) return DBF_ERR_INVALID_ARG;
    dbf_status st = validate_factors(l.packedA, l.packedB, l.a, l.m, l.b, l.n, l.k, m_in);
    if (st != DBF_OK) return st;
    if (!aligned16(l.y)) return DBF_ERR_MISALIGNED;
  }
  if (batch < 1) return DBF_ERR_INVALID_ARG;
  if (batch > kMaxRows) return DBF_ERR_UNSUPPORTED_SHAPE;
  if (y_t != DBF_F16 && y_t != DBF_F32) return DBF_ERR_INVALID_ARG;
  // (the grouped decode always runs the two-launch kernels: DBF_FWD_DECODE_TWO_STAGE changes nothing here)
  const uint32_t known = DBF_FWD_WEIGHTS_STATIC | DBF_FWD_FORCE_DECODE | DBF_FWD_FORCE_PREFILL |
                         DBF_FWD_DECODE_SHIFT_EXPAND | DBF_FWD_DECODE_TWO_STAGE | DBF_FWD_DECODE_SINGLE |
                         DBF_FWD_DECODE_TABLE;
  if ((flags & ~known) != 0) return DBF_ERR_INVALID_ARG;
  if ((flags & DBF_FWD_DECODE_TABLE) && (flags & DBF_FWD_DECODE_SHIFT_EXPAND)) return DBF_ERR_INVALID_ARG;
  if ((flags & DBF_FWD_FORCE_DECODE) && (flags & DBF_FWD_FORCE_PREFILL)) return DBF_ERR_INVALID_ARG;
  if (!aligned16(x)) return DBF_ERR_MISALIGNED;
  if (!workspace || !aligned16(workspace) || ws_bytes < grouped_v_offset(layers, num_layers, batch))
    return DBF_ERR_WORKSPACE;
  DeviceInfo dev;
  dbf_status st = current_device(&dev);
  if (st != DBF_OK) return st;

  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_handle);
  const bool out_f32 = y_t == DBF_F32;
  const bool early = (flags & DBF_FWD_WEIGHTS_STATIC) != 0;
  int* status = static_cast<int*>(workspace);
  const __half* xh = reinterpret_cast<const __half*>(x);
  const size_t y_elt = out_f32 ? 4 : 2;
  __half* V[DBF_MAX_GROUP];
  int64_t rows_a = 0, rows_b = 0;
  for (int g = 0; g < num_layers; ++g) {
    V[g] = reinterpret_cast<__half*>(static_cast<char*>(workspace) + grouped_v_offset(layers, g, batch));
    rows_a += layers[g].n;
    rows_b += layers[g].k;
  }

  const bool decode = (flags & DBF_FWD_FORCE_DECODE) || (!(flags & DBF_FWD_FORCE_PREFILL) && batch <= 16);
  if (decode) {
    const bool class_expand = (flags & DBF_FWD_DECODE_SHIFT_EXPAND) == 0;
    const bool lut = (flags & DBF_FWD_DECODE_TABLE) != 0;
    for (int64_t t0 = 0; t0 < batch; t0 += 16) {
      const int nb = static_cast<int>(batch - t0 < 16 ? batch - t0 : 16);
      DecodeGroup gb{};
      DecodeGroup ga{};
      gb.n = ga.n = num_layers;
      for (int g = 0; g < num_layers; ++g) {
        const dbf_layer_desc& l = layers[g];
        DecodeArgs& sb = gb.layer[g];
        sb.packed = l.packedB;
        sb.wpr = words_per_row(m_in);
        sb.M = static_cast<int>(l.k);
        sb.K = static_cast<int>(m_in);
        sb.act = xh + t0 * m_in;
        sb.ld_act = m_in;
        sb.kscale = reinterpret_cast<const __half*>(l.b);
        sb.rowscale = reinterpret_cast<const __half*>(l.m);
        sb.out = V[g] + t0 * l.k;
        sb.ld_out = l.k;
        sb.batch = nb;
        sb.weights_early = early ? 1 : 0;
        sb.status = status;
        DecodeArgs& sa = ga.layer[g];
        sa.packed = l.packedA;
        sa.wpr = words_per_row(l.k);
        sa.M = static_cast<int>(l.n);
        sa.K = static_cast<int>(l.k);
        sa.act = V[g] + t0 * l.k;
        sa.ld_act = l.k;
        sa.kscale = nullptr;
        sa.rowscale = reinterpret_cast<const __half*>(l.a);
        sa.out = static_cast<char*>(l.y) + static_cast<size_t>(t0) * static_cast<size_t>(l.n) * y_elt;
        sa.ld_out = l.n;
        sa.batch = nb;
        sa.weights_early = 1;  // the stage-B launch releases this one only after its own wait
        sa.status = status;
      }
      st = launch_decode_group(gb, rows_a, class_expand, lut, /*out_f32=*/false, dev, stream);
      if (st != DBF_OK) return st;
      st = launch_decode_group(ga, rows_b, class_expand, lut, out_f32, dev, stream);
      if (st != DBF_OK) return st;
    }
    return DBF_OK;
  }

  // Large batches are tensor-core bound: one layer after the other.
  for (int g = 0; g < num_layers; ++g) {
    const dbf_layer_desc& l = layers[g];
    const size_t v_end = grouped_v_offset(layers, num_layers, batch);
    char* sk = ws_bytes >= v_end + kSkBytes ? static_cast<char*>(workspace) + v_end : nullptr;
    PrefillArgs g1{};
    g1.sk_flags = sk ? reinterpret_cast<unsigned*>(sk) : nullptr;
    g1.sk_slots = sk ? reinterpret_cast<float*>(sk + kSkFlagBytes) : nullptr;
    g1.packed = l.packedB;
    g1.wpr = words_per_row(m_in);
    g1.M = static_cast<int>(l.k);
    g1.K = static_cast<int>(m_in);
    g1.kscale = reinterpret_cast<const __half*>(l.b);
    g1.rowscale = reinterpret_cast<const __half*>(l.m);
    g1.out = V[g];
    g1.ld_out = l.k;
    g1.batch = static_cast<int>(batch);
    g1.weights_early = early ? 1 : 0;
    g1.status = status;
    st = launch_prefill_gemm(g1, xh, batch, /*out_f32=*/false, dev, stream);
    if (st != DBF_OK) return st;
    PrefillArgs g2{};
    g2.sk_flags = g1.sk_flags;
    g2.sk_slots = g1.sk_slots;
    g2.packed = l.packedA;
    g2.wpr = words_per_row(l.k);
    g2.M = static_cast<int>(l.n);
    g2.K = static_cast<int>(l.k);
    g2.kscale = nullptr;
    g2.rowscale = reinterpret_cast<const __half*>(l.a);
    g2.out = l.y;
    g2.ld_out = l.n;
    g2.batch = static_cast<int>(batch);
    g2.weights_early = 1;
    g2.status = status;
    st = launch_prefill_gemm(g2, V[g], batch, out_f32, dev, stream);
    if (st != DBF_OK) return st;
  }
  return DBF_OK;
}

dbf_status dbf_transpose_signs(const uint32_t* packed, int64_t rows, int64_t cols, uint32_t* out,
                               struct CUstream_st* stream) {
  if (!packed || !out) return DBF_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1) return DBF_ERR_INVALID_ARG;
  if (rows > kMaxRows || cols > kMaxRows || rows * words_per_row(cols) > (int64_t{1} << 40) ||
      cols * words_per_row(rows) > (int64_t{1} << 40))
    return DBF_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(packed) || !aligned16(out)) return DBF_ERR_MISALIGNED;
  DeviceInfo dev;
  dbf_status st = current_device(&dev);
  if (st != DBF_OK) return st;
  return launch_transpose_signs(packed, rows, cols, out, dev, reinterpret_cast<cudaStream_t>(stream));
}

dbf_status dbf_forward_transposed(const uint16_t* dy, const uint32_t* packedAT, const uint32_t* packedBT,
                                  const uint16_t* a, const uint16_t* m, const uint16_t* b, int64_t n, int64_t k,
                                  int64_t m_in, int64_t batch, void* dx, dbf_dtype dx_t, void* workspace,
                                  size_t ws_bytes, uint32_t flags, struct CUstream_st* stream) {
  // dx = b (.) (B^T (m (.) (A^T (a (.) dy)))): the forward with B^T (m_in rows
  // over k) as its first factor and A^T (k rows over n) as its second, a and b
  // exchanged, and n in the place of m_in.
  return dbf_forward(dy, packedBT, packedAT, b, m, a, m_in, k, n, batch, dx, dx_t, workspace, ws_bytes, flags,
                     stream);
}

dbf_status dbf_reconstruct_dense(const uint32_t* packedA, const uint32_t* packedB, const uint16_t* a,
                                 const uint16_t* m, const uint16_t* b, int64_t n, int64_t k, int64_t m_in, void* W,
                                 dbf_dtype W_t, struct CUstream_st* stream) {
  if (!W) return DBF_ERR_INVALID_ARG;
  dbf_status st = validate_factors(packedA, packedB, a, m, b, n, k, m_in);
  if (st != DBF_OK) return st;
  if (W_t != DBF_F16 && W_t != DBF_F32) return DBF_ERR_INVALID_ARG;
  if (!aligned16(W)) return DBF_ERR_MISALIGNED;
  if (n * m_in > (int64_t{1} << 40)) return DBF_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != DBF_OK) return st;
  return launch_reconstruct(packedA, packedB, reinterpret_cast<const __half*>(a), reinterpret_cast<const __half*>(m),
                            reinterpret_cast<const __half*>(b), n, k, m_in, W, W_t == DBF_F32, dev,
                            reinterpret_cast<cudaStream_t>(stream));
}

dbf_status dbf_workspace_status(const void* workspace, struct CUstream_st* stream, int32_t* device_status) {
  if (!workspace || !device_status) return DBF_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return DBF_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return DBF_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DBF_ERR_CUDA;
  *device_status = v;
  return DBF_OK;
}

}  // extern "C"
