// Weight and activation quantizers (QSpec abstract: one INT4 weight set for
// both stages; explainer essay paragraph 2: W4A4 also quantizes activations).
//
// All decisions are taken in IEEE fp32 with round-to-nearest-even:
//   weights:     s = absmax / 7, s_h = fp16(s), q = clamp(rint(w / s_h), -8, 7)
//   activations: s_a = absmax / 7, inv = 7 / absmax, q = clamp(rint(x * inv), -8, 7)
//                (the clamp never binds for finite x; codes of non-finite x are unspecified)
// The explicit __fdiv_rn / __fmul_rn intrinsics pin the rounding regardless of
// compiler flags and forbid contraction into FMAs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "device_common.cuh"

namespace qspec {

__device__ __forceinline__ int clamp_q(int v) { return v < -8 ? -8 : (v > 7 ? 7 : v); }

// One warp per (row n, group g).  Lane l handles GROUP/32 consecutive values.
// ws rows have scale_row_stride(k / GROUP) entries; the padding is zeroed.
template <int GROUP>
__global__ void __launch_bounds__(256) quantize_weights_kernel(const float* __restrict__ w,
                                                               int64_t n_rows, int64_t k,
                                                               uint8_t* __restrict__ wq,
                                                               uint16_t* __restrict__ ws) {
  constexpr int PER_LANE = GROUP / 32;
  const int64_t groups_per_row = k / GROUP;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (gw >= n_rows * groups_per_row) return;
  const int64_t row = gw / groups_per_row;
  const int64_t g = gw - row * groups_per_row;
  const float* src = w + row * k + g * GROUP + lane * PER_LANE;

  float v[PER_LANE];
  if constexpr (PER_LANE == 4) {
    const float4 t = *reinterpret_cast<const float4*>(src);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else {
    const float2 t = *reinterpret_cast<const float2*>(src);
    v[0] = t.x; v[1] = t.y;
  }
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) a = fmaxf(a, fabsf(v[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));

  const float s = __fdiv_rn(a, 7.0f);
  const __half sh = __float2half_rn(s);
  const float sf = __half2float(sh);
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int q = (sf == 0.f) ? 0 : clamp_q(__float2int_rn(__fdiv_rn(v[i], sf)));
    packed |= (static_cast<uint32_t>(q) & 0xFu) << (4 * i);
  }
  uint8_t* dst = wq + row * (k / 2) + g * (GROUP / 2) + lane * (PER_LANE / 2);
  if constexpr (PER_LANE == 4) {
    *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(packed);
  } else {
    *dst = static_cast<uint8_t>(packed);
  }
  const int64_t ldg = scale_row_stride(groups_per_row);
  if (lane == 0) ws[row * ldg + g] = __half_as_ushort(sh);
  // the row's padding entries (a row's last group writes them)
  if (g == groups_per_row - 1 && lane < ldg - groups_per_row)
    ws[row * ldg + groups_per_row + lane] = 0;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

// One CTA per token row.  kPacked: write two nibbles per byte (the ABI
// format); otherwise write one int8 per element (the layout the W4A4 GEMM
// streams into its tensor-core operand tiles).  kQMax: 7 for the 4-bit codes
// of the W4A4 drafter, 127 for the 8-bit codes of the W4A8 drafting variant
// (s_a = absmax / kQMax, inv = kQMax / absmax, q clamped to [-kQMax-1, kQMax]).
// kF32In: x holds fp32 values (a layer's output, row stride ldx) and each one
// is first rounded to bf16 (nearest even): the bf16 glue of chained layers
// folded into the read.  Otherwise x holds bf16 bit patterns, row stride ldx.
// kThreads per row: 128 at most 56 registers each (launch bounds 128 x 9), or
// 256.  The 128-thread CTA with its 16 bytes of static shared memory fits on an
// SM beside a decode GEMM CTA of the 16-token tile (12 warps x 152 allocated
// registers + 4 x 56 = 65536; shared memory 227 KB + 1 KB reserved each), so
// the GEMM launched behind this kernel never waits for an SM it holds (with
// 256 threads the last 16 GEMM CTAs of every drafting call started only when
// these exited).  Rows of other sizes use 256 threads (fewer re-reads of long
// rows).
template <bool kPacked, int kQMax = 7, bool kF32In = false, int kThreads = 256>
__global__ void __launch_bounds__(kThreads, kThreads == 128 ? 9 : 4)
    quant_act_kernel(const void* __restrict__ x, int64_t ldx, int64_t k, void* __restrict__ out,
                     float* __restrict__ scales, int early_trigger) {
  constexpr int kQuantThreads = kThreads;
  __shared__ float red[kQuantThreads / 32];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  constexpr unsigned kTraceKind = 3u;   // trace builds: event-log tags
  const unsigned trace_launch = static_cast<unsigned>(reinterpret_cast<uintptr_t>(out) >> 8);
  (void)kTraceKind;
  (void)trace_launch;
  QSPEC_TRACE_AT(1);
  if (tid == 0) QSPEC_PHASE(0);
  // This kernel may be launched as a programmatic dependent of the previous
  // grid: wait for it (complete, memory flushed; a no-op otherwise) and let
  // the GEMM that consumes our output launch.  By default the GEMM launches
  // only after the wait, so whatever wrote its weights has finished when it
  // streams them; with early_trigger (the caller vouches that the weights
  // are ready) it launches at once.  Either way the GEMM waits for this
  // kernel (griddepcontrol.wait) where it reads x and s_a.
  if (early_trigger) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
  } else {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  if (tid == 0) QSPEC_PHASE(1);
  const uint16_t* xr = static_cast<const uint16_t*>(x) + row * ldx;
  const float* xfr = static_cast<const float*>(x) + row * ldx;
  if (!QSPEC_ALIGN_OK(kF32In ? reinterpret_cast<uintptr_t>(xfr) : reinterpret_cast<uintptr_t>(xr), 16) ||
      !QSPEC_ALIGN_OK(reinterpret_cast<uintptr_t>(out), 8))
    return;
  // elements c .. c+7 of the row as 8 bf16 bit patterns (element 2j in the
  // low half of word j)
  auto load8 = [&](int64_t c) {
    if constexpr (kF32In) {
      const float4 a = *reinterpret_cast<const float4*>(xfr + c);
      const float4 b = *reinterpret_cast<const float4*>(xfr + c + 4);
      auto two = [](float lo, float hi) {
        return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
      };
      return make_uint4(two(a.x, a.y), two(a.z, a.w), two(b.x, b.y), two(b.z, b.w));
    } else {
      return *reinterpret_cast<const uint4*>(xr + c);
    }
  };

  // Each thread's chunks of 8 elements stay in registers between the two
  // passes (up to kCache chunks: rows of up to 16384 elements are read once);
  // longer rows read the rest again.
  constexpr int kCache = 8;
  uint4 cache[kCache];
  // |x| max on bf16 pairs: clear both sign bits, then one packed bf16 max
  // (a max is exact in any format, so this equals the fp32 max of |x|).
  auto absmax8 = [](const uint4& u, __nv_bfloat162 m) {
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t b = w4[j] & 0x7FFF7FFFu;
      __nv_bfloat162 v;
      memcpy(&v, &b, 4);
      m = __hmax2(m, v);
    }
    return m;
  };
  __nv_bfloat162 m2 = __float2bfloat162_rn(0.f);
#pragma unroll
  for (int j = 0; j < kCache; ++j) {
    const int64_t c = (static_cast<int64_t>(tid) + kQuantThreads * j) * 8;
    if (c < k) {
      cache[j] = load8(c);
      m2 = absmax8(cache[j], m2);
    }
  }
  for (int64_t c = (static_cast<int64_t>(tid) + kQuantThreads * kCache) * 8; c < k;
       c += kQuantThreads * 8)
    m2 = absmax8(load8(c), m2);
  float a = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  if ((tid & 31) == 0) red[tid >> 5] = a;
  __syncthreads();
  a = red[0];
#pragma unroll
  for (int i = 1; i < kQuantThreads / 32; ++i) a = fmaxf(a, red[i]);

  static_assert(!kPacked || kQMax == 7, "packed output holds 4-bit codes");
  constexpr float kLevels = static_cast<float>(kQMax);
  const float s = __fdiv_rn(a, kLevels);
  // an all-zero row quantizes to zeros: inv = 0 gives t = 0 for every element
  const float inv = (a == 0.f) ? 0.f : __fdiv_rn(kLevels, a);
  if (tid == 0) scales[row] = s;

  // t = x * inv rounded to fp32, then rint(t) by adding 1.5 x 2^23: for
  // |t| < 2^22 the sum lies where the float spacing is 1, so it rounds t to
  // the nearest integer, ties to even (1.5 x 2^23 is even), and the sum's bit
  // pattern is 0x4B400000 + rint(t): its low byte is the two's-complement
  // code.  For finite x, |t| <= kQMax (1 + 2^-23), so rint(t) already lies in
  // [-kQMax, kQMax] and no clamp is needed.
  auto code_bits = [inv](float v) {
    return __float_as_uint(__fadd_rn(__fmul_rn(v, inv), 12582912.0f));
  };
  // bytes [a.0, b.0, c.0, d.0]
  auto low_bytes = [](uint32_t a4, uint32_t b4, uint32_t c4, uint32_t d4) {
    return __byte_perm(__byte_perm(a4, b4, 0x0040), __byte_perm(c4, d4, 0x0040), 0x5410);
  };
  auto emit = [&](int64_t c, const uint4& u) {
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
    uint32_t e[8];   // element 2j: low half of word j, element 2j + 1: high half
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      e[2 * j] = code_bits(__uint_as_float(w4[j] << 16));
      e[2 * j + 1] = code_bits(__uint_as_float(w4[j] & 0xFFFF0000u));
    }
    if constexpr (kPacked) {
      // nibble j = code j; bytes -> nibbles: byte i's low nibble joins byte
      // i - 1's high nibble, then bytes 0 and 2 of each half are kept
      uint32_t lo = low_bytes(e[0], e[1], e[2], e[3]) & 0x0F0F0F0Fu;
      uint32_t hi = low_bytes(e[4], e[5], e[6], e[7]) & 0x0F0F0F0Fu;
      lo |= lo >> 4;
      hi |= hi >> 4;
      *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(out) + row * (k / 2) + c / 2) =
          __byte_perm(lo, hi, 0x6420);
    } else {
      // int8 operand for the GEMM, each block of 8 channels stored in the
      // order (0,2,4,6,1,3,5,7): the GEMM widens packed weight nibbles into
      // the same order with masks alone, and a dot product does not depend
      // on the order of its terms.
      *reinterpret_cast<uint2*>(static_cast<int8_t*>(out) + row * k + c) =
          make_uint2(low_bytes(e[0], e[2], e[4], e[6]), low_bytes(e[1], e[3], e[5], e[7]));
    }
  };
#pragma unroll
  for (int j = 0; j < kCache; ++j) {
    const int64_t c = (static_cast<int64_t>(tid) + kQuantThreads * j) * 8;
    if (c < k) emit(c, cache[j]);
  }
  for (int64_t c = (static_cast<int64_t>(tid) + kQuantThreads * kCache) * 8; c < k;
       c += kQuantThreads * 8)
    emit(c, load8(c));
  if (tid == 0) QSPEC_PHASE(8);
}

// Glue between chained linear layers: x[i][j] = bf16_RN(y[i][j]) for j < k,
// the next layer's bf16 input from a layer's fp32 output (its first k
// columns, row stride ldy).  One thread per 8 outputs: two 16-byte loads, one
// 16-byte store.  Launched as a programmatic dependent: it lets the next
// kernel launch at once, then waits for the preceding grid (complete, memory
// flushed) before it reads y or writes x.
__global__ void __launch_bounds__(256) cast_bf16_kernel(const float* __restrict__ y, int64_t m,
                                                        int64_t ldy, int64_t k,
                                                        uint16_t* __restrict__ x) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t per_row = k / 8;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= m * per_row) return;
  const int64_t i = t / per_row;
  const int64_t j = (t - i * per_row) * 8;
  const float4 a = *reinterpret_cast<const float4*>(y + i * ldy + j);
  const float4 b = *reinterpret_cast<const float4*>(y + i * ldy + j + 4);
  auto pack = [](float lo, float hi) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
  };
  *reinterpret_cast<uint4*>(x + i * k + j) =
      make_uint4(pack(a.x, a.y), pack(a.z, a.w), pack(b.x, b.y), pack(b.z, b.w));
}

}  // namespace qspec
