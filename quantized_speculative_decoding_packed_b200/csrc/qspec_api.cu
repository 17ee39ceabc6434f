// C ABI of the shared-INT4 QSpec hot path (declared in include/qspec.h).
//
// Host side only: argument validation, workspace layout, TMA descriptors and
// kernel launches.  Every step of the computation runs in the kernels of
// quantize.cuh, gemm.cuh and accept.cuh; there is no host fallback.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "accept.cuh"
#include "attention.cuh"
#include "gemm.cuh"
#include "qspec.h"
#include "quantize.cuh"

namespace qspec {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
};

DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

qspec_status current_device(int* dev_out, DeviceInfo* info_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return QSPEC_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return QSPEC_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return QSPEC_ERR_CUDA;
    }
    d.supported = (major == 10 && minor == 0);
    d.sm_count = sms;
    d.probed = true;
  }
  if (dev_out) *dev_out = dev;
  if (info_out) *info_out = d;
  return d.supported ? QSPEC_OK : QSPEC_ERR_UNSUPPORTED_DEVICE;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
    } else {
      cudaGetLastError();
    }
  });
  return fn;
}

// 2-D row-major tensor [rows][cols] of `elem` bytes, box [box_rows][box_cols].
bool make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, size_t elem, const void* base,
               uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
               CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- GEMM planning
// Every GEMM workspace starts with a 256-byte status block and the split-tile
// tickets, at fixed offsets.
constexpr size_t kStatusAndTicketBytes = 256 + static_cast<size_t>(kMaxGrid) * 4;

struct GemmPlan {
  int mt = 16;               // token tile (MMA N)
  int m_tiles = 1, n_tiles = 1, ku = 1;
  long long units = 0;
  int grid = 1;
  size_t off_counters = 0, off_partials = 0, off_xq = 0, off_sa = 0, total = 0;
};

int pick_mt(int64_t m) {
  if (m > 96) return 128;
  const int r = static_cast<int>((m + 15) / 16) * 16;
  return r;   // 16, 32, 48, 64, 80, 96
}

bool gemm_shape_ok(int64_t m, int64_t n, int64_t k, int32_t group) {
  if (m < 1 || n < 1 || k < 128 || (k % 128) != 0) return false;
  if (group != 64 && group != 128) return false;
  if (m > (1ll << 30) || n > (1ll << 30) || k > (1ll << 30)) return false;
  // the kernel's 32-bit unit arithmetic
  const long long mt = pick_mt(m);
  const long long units = ((m + mt - 1) / mt) * ((n + kTileN - 1) / kTileN) * (k / unit_k(false));
  return units < kMaxUnits;
}

// Decode-sized drafting GEMMs (m <= 32) can quantize their activations in the
// GEMM kernel itself (QSPEC_GEMM_FUSED_QUANT); otherwise the separate
// per-token pre-pass kernel does.
bool fused_act_quant(bool int8_mode, int64_t m) { return int8_mode && m <= 32; }

GemmPlan plan_gemm(bool int8_mode, int64_t m, int64_t n, int64_t k, int sm_count) {
  GemmPlan p;
  p.mt = pick_mt(m);
  p.m_tiles = static_cast<int>((m + p.mt - 1) / p.mt);
  p.n_tiles = static_cast<int>((n + kTileN - 1) / kTileN);
  const int uk = unit_k(int8_mode);
  p.ku = static_cast<int>((k + uk - 1) / uk);   // a last half unit reads zeros past k
  p.units = static_cast<long long>(p.m_tiles) * p.n_tiles * p.ku;
  const int max_grid = sm_count < kMaxGrid ? sm_count : kMaxGrid;
  p.grid = static_cast<int>(p.units < max_grid ? p.units : max_grid);
  // Fixed-position regions first, so that calls of any shape sharing one
  // workspace never see each other's scratch data in their status word or
  // ticket slots; shape-dependent scratch follows.
  size_t off = 256;                                  // status word(s)
  p.off_counters = off;
  off += static_cast<size_t>(kMaxGrid) * 4;
  p.off_partials = off;
  off += round_up(static_cast<size_t>(2) * p.grid * p.mt * kTileN * 4, 256);
  if (int8_mode) {
    p.off_xq = off;
    off += round_up(static_cast<size_t>(m) * k, 256);
    p.off_sa = off;
    off += round_up(static_cast<size_t>(m) * 4, 256);
  }
  p.total = off;
  return p;
}

template <bool kInt8, int MT, bool kDbg, bool kFused = false>
qspec_status launch_qgemm_t(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ts,
                            const GemmArgs& a,
                            int grid, int dev, cudaStream_t stream) {
  using C = GemmCfg<kInt8, MT, kFused>;
  // Set once per device; concurrent first calls may both set it (idempotent).
  static std::atomic<bool> attr_set[kMaxDevices];
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(qgemm_kernel<kInt8, MT, kDbg, kFused>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess) {
      cudaGetLastError();
      return QSPEC_ERR_CUDA;
    }
    attr_set[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  // Programmatic dependent launch: the GEMM's set-up overlaps the end of the
  // preceding kernel (its activation quantization, or the previous GEMM) and,
  // in W4A4 mode, so does its weight stream; it waits for that grid before it
  // reads activations or writes anything.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, qgemm_kernel<kInt8, MT, kDbg, kFused>, tw, tx, ts, a) != cudaSuccess) {
    cudaGetLastError();
    return QSPEC_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? QSPEC_OK : QSPEC_ERR_CUDA;
}

template <bool kInt8>
qspec_status launch_qgemm(int mt, bool fused, const CUtensorMap& tw, const CUtensorMap& tx,
                          const CUtensorMap& ts, const GemmArgs& a,
                          int grid, int dev, cudaStream_t stream) {
  const bool dbg = kInt8 && a.dbg_acc != nullptr;
  if constexpr (kInt8) {
    if (fused) {
      switch (mt) {
        case 16:
          return dbg ? launch_qgemm_t<true, 16, true, true>(tw, tx, ts, a, grid, dev, stream)
                     : launch_qgemm_t<true, 16, false, true>(tw, tx, ts, a, grid, dev, stream);
        case 32:
          return dbg ? launch_qgemm_t<true, 32, true, true>(tw, tx, ts, a, grid, dev, stream)
                     : launch_qgemm_t<true, 32, false, true>(tw, tx, ts, a, grid, dev, stream);
        default: return QSPEC_ERR_INVALID_ARG;
      }
    }
  }
  switch (mt) {
    case 16:
      return dbg ? launch_qgemm_t<kInt8, 16, kInt8>(tw, tx, ts, a, grid, dev, stream)
                 : launch_qgemm_t<kInt8, 16, false>(tw, tx, ts, a, grid, dev, stream);
    case 32:
      return dbg ? launch_qgemm_t<kInt8, 32, kInt8>(tw, tx, ts, a, grid, dev, stream)
                 : launch_qgemm_t<kInt8, 32, false>(tw, tx, ts, a, grid, dev, stream);
    case 48:
      return dbg ? launch_qgemm_t<kInt8, 48, kInt8>(tw, tx, ts, a, grid, dev, stream)
                 : launch_qgemm_t<kInt8, 48, false>(tw, tx, ts, a, grid, dev, stream);
    case 64:
      return dbg ? launch_qgemm_t<kInt8, 64, kInt8>(tw, tx, ts, a, grid, dev, stream)
                 : launch_qgemm_t<kInt8, 64, false>(tw, tx, ts, a, grid, dev, stream);
    case 80:
      return dbg ? launch_qgemm_t<kInt8, 80, kInt8>(tw, tx, ts, a, grid, dev, stream)
                 : launch_qgemm_t<kInt8, 80, false>(tw, tx, ts, a, grid, dev, stream);
    case 96:
      return dbg ? launch_qgemm_t<kInt8, 96, kInt8>(tw, tx, ts, a, grid, dev, stream)
                 : launch_qgemm_t<kInt8, 96, false>(tw, tx, ts, a, grid, dev, stream);
    case 128:
      return dbg ? launch_qgemm_t<kInt8, 128, kInt8>(tw, tx, ts, a, grid, dev, stream)
                 : launch_qgemm_t<kInt8, 128, false>(tw, tx, ts, a, grid, dev, stream);
    default: return QSPEC_ERR_INVALID_ARG;
  }
}

// kInt8: the drafting modes (integer MMA on per-token activation codes of
// act_bits = 4 (W4A4) or 8 (W4A8)); else the W4A16 verifying mode.
// xf (drafting modes only): fp32 input [m][ldx] instead of bf16 x, rounded
// to bf16 as the activation quantizer reads it.
template <bool kInt8>
qspec_status run_gemm(const uint16_t* x, int64_t m, int64_t k, const uint8_t* wq,
                      const uint16_t* ws, int64_t n, int32_t group, float* y, void* workspace,
                      size_t workspace_bytes, int32_t* dbg_acc, uint32_t flags, void* stream_v,
                      int act_bits = 4, const float* xf = nullptr, int64_t ldx = 0) {
  if ((!x && !xf) || !wq || !ws || !y || !workspace) return QSPEC_ERR_INVALID_ARG;
  const uint32_t allowed = QSPEC_GEMM_WEIGHTS_READY | QSPEC_GEMM_TEST_STALL |
                           ((kInt8 && !xf) ? QSPEC_GEMM_FUSED_QUANT : 0u);
  if ((flags & ~allowed) != 0u) return QSPEC_ERR_INVALID_ARG;
  const bool weights_ready = (flags & QSPEC_GEMM_WEIGHTS_READY) != 0u;
  if (!gemm_shape_ok(m, n, k, group)) return QSPEC_ERR_INVALID_ARG;
  if (xf && (!kInt8 || ldx < k || (ldx % 4) != 0 || ldx > (1ll << 40) / m)) return QSPEC_ERR_INVALID_ARG;
  if ((x && !aligned(x, 16)) || (xf && !aligned(xf, 16)) || !aligned(wq, 16) || !aligned(ws, 16) ||
      !aligned(y, 4) || !aligned(workspace, 16) || (dbg_acc && !aligned(dbg_acc, 4)))
    return QSPEC_ERR_INVALID_ARG;
  int dev = 0;
  DeviceInfo info;
  qspec_status st = current_device(&dev, &info);
  if (st != QSPEC_OK) return st;
  const GemmPlan p = plan_gemm(kInt8, m, n, k, info.sm_count);
  if (workspace_bytes < p.total) return QSPEC_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  uint8_t* wsp = static_cast<uint8_t*>(workspace);

  CUtensorMap tw, tx, ts;
  // Each converter thread reads one row of the packed tile: 128 B in int8
  // mode (128-byte swizzle), 64 B in bf16 mode (64-byte swizzle).
  const int uk = unit_k(kInt8);
  if (!make_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq, n, k / 2, kTileN, uk / 2,
                 kInt8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return QSPEC_ERR_CUDA;
  GemmArgs a;
  a.M = static_cast<int>(m);
  a.N = static_cast<int>(n);
  a.K = static_cast<int>(k);
  a.groups_per_row = static_cast<int>(k / group);
  a.groups_per_unit = uk / group;
  a.m_tiles = p.m_tiles;
  a.n_tiles = p.n_tiles;
  a.ku = p.ku;
  a.units = p.units;
  a.weights_ready = weights_ready ? 1 : 0;
  a.test_stall_ns = (flags & QSPEC_GEMM_TEST_STALL) ? 10u * 1000u * 1000u : 0u;   // 10 ms
  a.qmax = (act_bits == 8) ? 127.f : 7.f;
  const bool fused = fused_act_quant(kInt8, m) && (flags & QSPEC_GEMM_FUSED_QUANT) != 0u;
  a.ws = ws;
  a.y = y;
  a.dbg_acc = dbg_acc;
  a.status = reinterpret_cast<uint32_t*>(wsp);
  a.counters = reinterpret_cast<uint32_t*>(wsp + p.off_counters);
  a.partials = reinterpret_cast<float*>(wsp + p.off_partials);
  a.s_a = nullptr;
  a.x = nullptr;
  a.xq = nullptr;
  a.qsync = nullptr;
  if (fused) {
    // the kernel quantizes the bf16 activations itself, into the same
    // workspace regions the pre-pass would have written, and reads them back
    // by TMA; the two counters live in the status block
    a.x = x;
    a.xq = reinterpret_cast<int8_t*>(wsp + p.off_xq);
    a.s_a = reinterpret_cast<float*>(wsp + p.off_sa);
    a.qsync = reinterpret_cast<uint32_t*>(wsp + 64);
    if (!make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.xq, m, k, p.mt, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return QSPEC_ERR_CUDA;
  } else if constexpr (kInt8) {
    int8_t* xq = reinterpret_cast<int8_t*>(wsp + p.off_xq);
    float* sa = reinterpret_cast<float*>(wsp + p.off_sa);
    // Also a programmatic dependent: it waits for the preceding grid itself,
    // and lets the GEMM launch once it has (or, when the weights are ready,
    // at once: the GEMM then reads nothing else before its own waits).
    // 128 threads beside the 16-token GEMM tile (they fit on its SMs), else 256
    const bool small = p.mt == 16;
    cudaLaunchConfig_t qc = {};
    qc.gridDim = dim3(static_cast<unsigned>(m));
    qc.blockDim = dim3(small ? 128 : 256);
    qc.stream = stream;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    qa[0].val.programmaticStreamSerializationAllowed = 1;
    qc.attrs = qa;
    qc.numAttrs = 1;
    void* qout = xq;
    const int early = weights_ready ? 1 : 0;
    const void* xin = xf ? static_cast<const void*>(xf) : static_cast<const void*>(x);
    const int64_t ld = xf ? ldx : k;
    const int64_t kk = k;
    cudaError_t qe;
    if (xf) {
      if (act_bits == 8)
        qe = small ? cudaLaunchKernelEx(&qc, quant_act_kernel<false, 127, true, 128>, xin, ld, kk, qout, sa, early)
                   : cudaLaunchKernelEx(&qc, quant_act_kernel<false, 127, true, 256>, xin, ld, kk, qout, sa, early);
      else
        qe = small ? cudaLaunchKernelEx(&qc, quant_act_kernel<false, 7, true, 128>, xin, ld, kk, qout, sa, early)
                   : cudaLaunchKernelEx(&qc, quant_act_kernel<false, 7, true, 256>, xin, ld, kk, qout, sa, early);
    } else {
      if (act_bits == 8)
        qe = small ? cudaLaunchKernelEx(&qc, quant_act_kernel<false, 127, false, 128>, xin, ld, kk, qout, sa, early)
                   : cudaLaunchKernelEx(&qc, quant_act_kernel<false, 127, false, 256>, xin, ld, kk, qout, sa, early);
      else
        qe = small ? cudaLaunchKernelEx(&qc, quant_act_kernel<false, 7, false, 128>, xin, ld, kk, qout, sa, early)
                   : cudaLaunchKernelEx(&qc, quant_act_kernel<false, 7, false, 256>, xin, ld, kk, qout, sa, early);
    }
    if (qe != cudaSuccess) {
      cudaGetLastError();
      return QSPEC_ERR_CUDA;
    }
    a.s_a = sa;
    if (!make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xq, m, k, p.mt, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return QSPEC_ERR_CUDA;
  } else {
    if (!make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, m, k, p.mt, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return QSPEC_ERR_CUDA;
  }
  // group scales: [n][ldg] fp16, one box = 8 groups x 128 rows (zero-filled
  // past row n-1; groups k/group .. ldg-1 are stored zeros)
  if (!make_tmap(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, ws, n, scale_row_stride(k / group), kTileN, 8,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return QSPEC_ERR_CUDA;
  return launch_qgemm<kInt8>(p.mt, fused, tw, tx, ts, a, p.grid, dev, stream);
}

}  // namespace
}  // namespace qspec

using namespace qspec;

#ifdef QSPEC_TRACE
extern "C" int qspec_debug_set_trace(void* host_mapped) {
  return cudaMemcpyToSymbol(g_qspec_trace, &host_mapped, sizeof(void*)) == cudaSuccess ? 0 : 1;
}
extern "C" int qspec_debug_set_events(void* dev_buffer) {
  const unsigned zero = 0;
  return (cudaMemcpyToSymbol(g_qspec_events, &dev_buffer, sizeof(void*)) == cudaSuccess &&
          cudaMemcpyToSymbol(g_qspec_event_count, &zero, sizeof(zero)) == cudaSuccess)
             ? 0
             : 1;
}
#endif

extern "C" {

qspec_status qspec_quantize_weights(const float* w, int64_t n, int64_t k, int32_t group,
                                    uint8_t* wq, uint16_t* ws, void* stream) {
  if (!w || !wq || !ws) return QSPEC_ERR_INVALID_ARG;
  if (n < 1 || (group != 64 && group != 128) || k < group || (k % group) != 0)
    return QSPEC_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(wq, 2) || !aligned(ws, 16)) return QSPEC_ERR_INVALID_ARG;
  const long long warps = n * (k / group);
  const long long blocks = (warps + 7) / 8;
  if (blocks > 0x7FFFFFFFll) return QSPEC_ERR_INVALID_ARG;
  qspec_status st = current_device(nullptr, nullptr);
  if (st != QSPEC_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (group == 128)
    quantize_weights_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, s>>>(w, n, k, wq, ws);
  else
    quantize_weights_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, s>>>(w, n, k, wq, ws);
  return cudaGetLastError() == cudaSuccess ? QSPEC_OK : QSPEC_ERR_CUDA;
}

qspec_status qspec_quant_act(const uint16_t* x, int64_t m, int64_t k, uint8_t* xq, float* xs,
                             void* stream) {
  if (!x || !xq || !xs) return QSPEC_ERR_INVALID_ARG;
  if (m < 1 || m > 0x7FFFFFFFll || k < 8 || (k % 8) != 0) return QSPEC_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(xq, 4) || !aligned(xs, 4)) return QSPEC_ERR_INVALID_ARG;
  qspec_status st = current_device(nullptr, nullptr);
  if (st != QSPEC_OK) return st;
  quant_act_kernel<true, 7, false, 256><<<static_cast<unsigned>(m), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, k, k, xq, xs, 0);
  return cudaGetLastError() == cudaSuccess ? QSPEC_OK : QSPEC_ERR_CUDA;
}

qspec_status qspec_cast_bf16(const float* y, int64_t m, int64_t ldy, int64_t k, uint16_t* x,
                             void* stream) {
  if (!y || !x) return QSPEC_ERR_INVALID_ARG;
  if (m < 1 || k < 8 || (k % 8) != 0 || ldy < k || (ldy % 4) != 0 || m * (k / 8) > (1ll << 40))
    return QSPEC_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(x, 16)) return QSPEC_ERR_INVALID_ARG;
  qspec_status st = current_device(nullptr, nullptr);
  if (st != QSPEC_OK) return st;
  const long long threads = m * (k / 8);
  const long long blocks = (threads + 255) / 256;
  if (blocks > 0x7FFFFFFFll) return QSPEC_ERR_INVALID_ARG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(256);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, cast_bf16_kernel, y, static_cast<int64_t>(m), static_cast<int64_t>(ldy),
                         static_cast<int64_t>(k), x) != cudaSuccess) {
    cudaGetLastError();
    return QSPEC_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? QSPEC_OK : QSPEC_ERR_CUDA;
}

qspec_status qspec_gemm_w4a4(const uint16_t* x, int64_t m, int64_t k, const uint8_t* wq,
                             const uint16_t* ws, int64_t n, int32_t group, float* y,
                             void* workspace, size_t workspace_bytes, int32_t* dbg_acc,
                             uint32_t flags, void* stream) {
  return run_gemm<true>(x, m, k, wq, ws, n, group, y, workspace, workspace_bytes, dbg_acc, flags,
                        stream);
}

qspec_status qspec_gemm_w4a8(const uint16_t* x, int64_t m, int64_t k, const uint8_t* wq,
                             const uint16_t* ws, int64_t n, int32_t group, float* y,
                             void* workspace, size_t workspace_bytes, int32_t* dbg_acc,
                             uint32_t flags, void* stream) {
  return run_gemm<true>(x, m, k, wq, ws, n, group, y, workspace, workspace_bytes, dbg_acc, flags,
                        stream, 8);
}

qspec_status qspec_gemm_w4a4_f32in(const float* x, int64_t ldx, int64_t m, int64_t k,
                                   const uint8_t* wq, const uint16_t* ws, int64_t n, int32_t group,
                                   float* y, void* workspace, size_t workspace_bytes,
                                   int32_t* dbg_acc, uint32_t flags, void* stream) {
  return run_gemm<true>(nullptr, m, k, wq, ws, n, group, y, workspace, workspace_bytes, dbg_acc,
                        flags, stream, 4, x, ldx);
}

qspec_status qspec_gemm_w4a8_f32in(const float* x, int64_t ldx, int64_t m, int64_t k,
                                   const uint8_t* wq, const uint16_t* ws, int64_t n, int32_t group,
                                   float* y, void* workspace, size_t workspace_bytes,
                                   int32_t* dbg_acc, uint32_t flags, void* stream) {
  return run_gemm<true>(nullptr, m, k, wq, ws, n, group, y, workspace, workspace_bytes, dbg_acc,
                        flags, stream, 8, x, ldx);
}

qspec_status qspec_gemm_w4a16(const uint16_t* x, int64_t m, int64_t k, const uint8_t* wq,
                              const uint16_t* ws, int64_t n, int32_t group, float* y,
                              void* workspace, size_t workspace_bytes, uint32_t flags,
                              void* stream) {
  return run_gemm<false>(x, m, k, wq, ws, n, group, y, workspace, workspace_bytes, nullptr, flags,
                         stream);
}

int32_t qspec_abi_version(void) { return QSPEC_ABI_VERSION; }

qspec_status qspec_spec_accept(const float* p, const float* q, const int32_t* draft,
                               const float* u_acc, const float* u_res, int32_t batch,
                               int32_t gamma, int32_t vocab, int32_t* n_accepted,
                               int32_t* tokens, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (!p || !q || !draft || !u_acc || !u_res || !n_accepted || !tokens)
    return QSPEC_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || gamma < 1 || gamma > 16 || vocab < 4 || vocab > 409600 ||
      (vocab % 4) != 0)
    return QSPEC_ERR_INVALID_ARG;
  if (!aligned(p, 16) || !aligned(q, 16) || !aligned(draft, 4) || !aligned(u_acc, 4) ||
      !aligned(u_res, 4) || !aligned(n_accepted, 4) || !aligned(tokens, 4))
    return QSPEC_ERR_INVALID_ARG;
  if (workspace && (workspace_bytes < 256 || !aligned(workspace, 16)))
    return QSPEC_ERR_WORKSPACE_TOO_SMALL;
  qspec_status st = current_device(nullptr, nullptr);
  if (st != QSPEC_OK) return st;
  const int chunk = ((vocab + 4 * kAcceptCluster - 1) / (4 * kAcceptCluster)) * 4;
  spec_accept_kernel<<<batch * kAcceptCluster, kAcceptThreads, 0,
                       static_cast<cudaStream_t>(stream)>>>(
      p, q, draft, u_acc, u_res, gamma, vocab, chunk, n_accepted, tokens,
      static_cast<uint32_t*>(workspace));
  return cudaGetLastError() == cudaSuccess ? QSPEC_OK : QSPEC_ERR_CUDA;
}

qspec_status qspec_spec_accept_greedy(const float* p, const int32_t* draft, int32_t batch,
                                      int32_t gamma, int32_t vocab, int32_t* n_accepted,
                                      int32_t* tokens, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  if (!p || !draft || !n_accepted || !tokens) return QSPEC_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || gamma < 1 || gamma > 16 || vocab < 4 || vocab > 409600 ||
      (vocab % 4) != 0)
    return QSPEC_ERR_INVALID_ARG;
  if (!aligned(p, 16) || !aligned(draft, 4) || !aligned(n_accepted, 4) || !aligned(tokens, 4))
    return QSPEC_ERR_INVALID_ARG;
  if (workspace && (workspace_bytes < 256 || !aligned(workspace, 16)))
    return QSPEC_ERR_WORKSPACE_TOO_SMALL;
  qspec_status st = current_device(nullptr, nullptr);
  if (st != QSPEC_OK) return st;
  const int chunk = ((vocab + 4 * kAcceptCluster - 1) / (4 * kAcceptCluster)) * 4;
  greedy_accept_kernel<<<batch * kAcceptCluster, kAcceptThreads, 0,
                         static_cast<cudaStream_t>(stream)>>>(
      p, draft, gamma, vocab, chunk, n_accepted, tokens, static_cast<uint32_t*>(workspace));
  return cudaGetLastError() == cudaSuccess ? QSPEC_OK : QSPEC_ERR_CUDA;
}

namespace {

// Shape checks shared by the three KV-cache calls (head_dim fixed at 128).
bool kv_shape_ok(int32_t batch, int32_t t_new, int32_t h_q, int32_t h_kv, int32_t head_dim,
                 int32_t l_max) {
  if (batch < 1 || batch > 65535 || t_new < 1 || h_q < 1 || h_kv < 1 || h_kv > 65535) return false;
  if (head_dim != kHeadDim || (h_q % h_kv) != 0 || l_max < 1) return false;
  return static_cast<int64_t>(t_new) * (h_q / h_kv) <= kAttnMaxRows;
}

int32_t attn_chunks(int32_t ctx_max) { return (ctx_max + kAttnChunk - 1) / kAttnChunk; }

}  // namespace

size_t qspec_attn_workspace_size(int32_t batch, int32_t t_new, int32_t h_q, int32_t h_kv,
                                 int32_t head_dim, int32_t ctx_max) {
  if (!kv_shape_ok(batch, t_new, h_q, h_kv, head_dim, 1)) return 0;
  if (ctx_max < 1 || attn_chunks(ctx_max) > kAttnMaxChunks) return 0;
  const int64_t rows = static_cast<int64_t>(t_new) * (h_q / h_kv);
  return static_cast<size_t>(attn_layout(batch, h_kv, attn_chunks(ctx_max), rows).total);
}

qspec_status qspec_kv_append(const float* qkv, int64_t ld_qkv, int32_t batch, int32_t t_new,
                             int32_t h_q, int32_t h_kv, int32_t head_dim, const int32_t* lens,
                             int32_t offset, uint16_t* k_cache, uint16_t* v_cache, int32_t l_max,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (!qkv || !lens || !k_cache || !v_cache) return QSPEC_ERR_INVALID_ARG;
  if (!kv_shape_ok(batch, t_new, h_q, h_kv, head_dim, l_max) || offset < 0) return QSPEC_ERR_INVALID_ARG;
  if (ld_qkv < static_cast<int64_t>(h_q + 2 * h_kv) * kHeadDim || (ld_qkv % 4) != 0)
    return QSPEC_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch) * t_new > 0x7FFFFFFFll) return QSPEC_ERR_INVALID_ARG;
  if (!aligned(qkv, 16) || !aligned(lens, 4) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return QSPEC_ERR_INVALID_ARG;
  if (workspace && (workspace_bytes < 256 || !aligned(workspace, 16))) return QSPEC_ERR_INVALID_ARG;
  qspec_status st = current_device(nullptr, nullptr);
  if (st != QSPEC_OK) return st;
  kv_append_kernel<<<static_cast<unsigned>(batch * t_new), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      qkv, ld_qkv, t_new, h_q, h_kv, lens, offset, k_cache, v_cache, l_max,
      static_cast<uint32_t*>(workspace));
  return cudaGetLastError() == cudaSuccess ? QSPEC_OK : QSPEC_ERR_CUDA;
}

qspec_status qspec_attn_decode(const float* qkv, int64_t ld_qkv, int32_t batch, int32_t t_new,
                               int32_t h_q, int32_t h_kv, int32_t head_dim, const int32_t* lens,
                               int32_t offset, const uint16_t* k_cache, const uint16_t* v_cache,
                               int32_t l_max, int32_t ctx_max, float* out, int64_t ld_out,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (!qkv || !lens || !k_cache || !v_cache || !out || !workspace) return QSPEC_ERR_INVALID_ARG;
  if (!kv_shape_ok(batch, t_new, h_q, h_kv, head_dim, l_max) || offset < 0) return QSPEC_ERR_INVALID_ARG;
  if (ctx_max < 1 || ctx_max > l_max || attn_chunks(ctx_max) > kAttnMaxChunks) return QSPEC_ERR_INVALID_ARG;
  if (ld_qkv < static_cast<int64_t>(h_q + 2 * h_kv) * kHeadDim || (ld_qkv % 4) != 0 ||
      ld_out < static_cast<int64_t>(h_q) * kHeadDim)
    return QSPEC_ERR_INVALID_ARG;
  if (!aligned(qkv, 16) || !aligned(lens, 4) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(out, 4) || !aligned(workspace, 16))
    return QSPEC_ERR_INVALID_ARG;
  const int32_t chunks = attn_chunks(ctx_max);
  const int32_t rows = t_new * (h_q / h_kv);
  if (workspace_bytes < static_cast<size_t>(attn_layout(batch, h_kv, chunks, rows).total))
    return QSPEC_ERR_WORKSPACE_TOO_SMALL;
  int dev = 0;
  qspec_status st = current_device(&dev, nullptr);
  if (st != QSPEC_OK) return st;
  const size_t smem = static_cast<size_t>(attn_smem_bytes(rows));
  static std::atomic<bool> attr_done[kMaxDevices];
  if (!attr_done[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(attn_smem_bytes(kAttnMaxRows))) !=
        cudaSuccess) {
      cudaGetLastError();
      return QSPEC_ERR_CUDA;
    }
    attr_done[dev].store(true, std::memory_order_release);
  }
  AttnArgs a;
  a.qkv = qkv;
  a.ld = ld_qkv;
  a.lens = lens;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.out = out;
  a.ld_out = ld_out;
  a.work = static_cast<uint8_t*>(workspace);
  a.t_new = t_new;
  a.h_q = h_q;
  a.h_kv = h_kv;
  a.offset = offset;
  a.l_max = l_max;
  a.ctx_max = ctx_max;
  a.chunks = chunks;
  a.rows = rows;
  attn_decode_kernel<<<dim3(static_cast<unsigned>(chunks), static_cast<unsigned>(h_kv),
                            static_cast<unsigned>(batch)),
                       kAttnThreads, smem, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? QSPEC_OK : QSPEC_ERR_CUDA;
}

qspec_status qspec_kv_commit(int32_t* lens, const int32_t* n_accepted, int32_t batch,
                             int32_t l_max, void* workspace, size_t workspace_bytes, void* stream) {
  if (!lens || !n_accepted || batch < 1 || l_max < 1) return QSPEC_ERR_INVALID_ARG;
  if (!aligned(lens, 4) || !aligned(n_accepted, 4)) return QSPEC_ERR_INVALID_ARG;
  if (workspace && (workspace_bytes < 256 || !aligned(workspace, 16))) return QSPEC_ERR_INVALID_ARG;
  qspec_status st = current_device(nullptr, nullptr);
  if (st != QSPEC_OK) return st;
  kv_commit_kernel<<<static_cast<unsigned>((batch + 127) / 128), 128, 0,
                     static_cast<cudaStream_t>(stream)>>>(lens, n_accepted, batch, l_max,
                                                          static_cast<uint32_t*>(workspace));
  return cudaGetLastError() == cudaSuccess ? QSPEC_OK : QSPEC_ERR_CUDA;
}

size_t qspec_workspace_size(int32_t op, int64_t m, int64_t n, int64_t k, int32_t group,
                            int32_t batch, int32_t gamma, int32_t vocab) {
  (void)batch;
  (void)gamma;
  (void)vocab;
  switch (op) {
    case QSPEC_OP_QUANTIZE_WEIGHTS:
    case QSPEC_OP_QUANT_ACT:
      return 0;
    case QSPEC_OP_SPEC_ACCEPT:
      return 256;
    case QSPEC_OP_GEMM_W4A4:
    case QSPEC_OP_GEMM_W4A8:
    case QSPEC_OP_GEMM_W4A16: {
      if (!gemm_shape_ok(m, n, k, group)) return 0;
      DeviceInfo info;
      if (current_device(nullptr, &info) != QSPEC_OK) return 0;
      return plan_gemm(op != QSPEC_OP_GEMM_W4A16, m, n, k, info.sm_count).total;
    }
    default:
      return 0;
  }
}

qspec_status qspec_workspace_status(void* workspace, void* stream) {
  if (!workspace) return QSPEC_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return QSPEC_ERR_CUDA;
  }
  if (word == 0) return QSPEC_OK;
  // A GEMM that gave up (the only kernels that time out) may have left
  // split-tile tickets taken: clear them with the status word, so that the
  // workspace is ready for the next call.  An accept workspace (256 bytes)
  // only ever receives BAD_INPUT.
  const size_t clear = (word & kDevTimeout) ? kStatusAndTicketBytes : 4;
  if (cudaMemsetAsync(workspace, 0, clear, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return QSPEC_ERR_CUDA;
  }
  return (word & kDevTimeout) ? QSPEC_ERR_TIMEOUT : QSPEC_ERR_BAD_INPUT;
}

// ---------------------------------------------------------------- no-allocation variant
// Built-in scratch for callers that cannot allocate device memory: a plugin
// inside a host application that owns all device memory and allows no
// allocation outside its own pools, or code that must not enter the
// allocator at the point of the call (real-time paths that forbid the
// implicit synchronisation cudaMalloc/cudaFree may cause).  Every GPU that
// loads this library holds the array until the process exits; it starts
// zero-filled.
static __device__ __align__(256) unsigned char g_qspec_static_scratch[QSPEC_STATIC_SCRATCH_BYTES];

namespace {
void* g_static_scratch_ptr[kMaxDevices] = {};
std::mutex g_static_scratch_mutex;

// Device address of the built-in array on the current device (looked up once
// per device, with that device current: in host code the array's name only
// stands in for it), or nullptr on failure.
void* static_scratch(int dev) {
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (!g_static_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_qspec_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return nullptr;
    }
    g_static_scratch_ptr[dev] = p;
  }
  return g_static_scratch_ptr[dev];
}
}  // namespace

qspec_status qspec_gemm_w4a16_noalloc(const uint16_t* x, int64_t m, int64_t k, const uint8_t* wq,
                                      const uint16_t* ws, int64_t n, int32_t group, float* y,
                                      uint32_t flags, void* stream) {
  if (!x || !wq || !ws || !y) return QSPEC_ERR_INVALID_ARG;
  if ((flags & ~QSPEC_GEMM_WEIGHTS_READY) != 0u) return QSPEC_ERR_INVALID_ARG;
  if (!gemm_shape_ok(m, n, k, group)) return QSPEC_ERR_INVALID_ARG;
  int dev = 0;
  DeviceInfo info;
  qspec_status st = current_device(&dev, &info);
  if (st != QSPEC_OK) return st;
  // The scratch needed by this shape must fit in the built-in array.
  if (plan_gemm(false, m, n, k, info.sm_count).total > QSPEC_STATIC_SCRATCH_BYTES)
    return QSPEC_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = static_scratch(dev);
  if (!scratch) return QSPEC_ERR_CUDA;
  // The array keeps whatever the previous call left.  The split-tile tickets
  // must start at zero (a call that gave up may have left some taken); the
  // status word is left alone, so that a fault stays visible until
  // qspec_gemm_w4a16_noalloc_status() reads it.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + 256, 0, kStatusAndTicketBytes - 256, s) !=
      cudaSuccess) {
    cudaGetLastError();
    return QSPEC_ERR_CUDA;
  }
  return run_gemm<false>(x, m, k, wq, ws, n, group, y, scratch, QSPEC_STATIC_SCRATCH_BYTES, nullptr,
                         flags, stream);
}

qspec_status qspec_gemm_w4a16_noalloc_status(void* stream) {
  int dev = 0;
  qspec_status st = current_device(&dev, nullptr);
  if (st != QSPEC_OK) return st;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
    scratch = g_static_scratch_ptr[dev];
  }
  if (!scratch) return QSPEC_OK;   // no call has run on this device
  return qspec_workspace_status(scratch, stream);
}

const char* qspec_status_string(qspec_status status) {
  switch (status) {
    case QSPEC_OK: return "ok";
    case QSPEC_ERR_INVALID_ARG: return "invalid argument";
    case QSPEC_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs sm_100)";
    case QSPEC_ERR_CUDA: return "CUDA error";
    case QSPEC_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case QSPEC_ERR_TIMEOUT: return "kernel wait timed out";
    case QSPEC_ERR_BAD_INPUT: return "invalid input data seen by a kernel";
    default: return "unknown status";
  }
}

}  // extern "C"
