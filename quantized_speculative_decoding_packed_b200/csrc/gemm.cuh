// Shared-INT4 GEMM for both QSpec modes on sm_100a tensor cores.
//
// QSpec (abstract) runs one packed INT4 weight set in two modes: W4A4 for
// drafting and W4A16 for verification; the explainer essay (paragraph 4)
// notes that the modes differ mainly in how activations are handled.  This
// one kernel template serves both from the same `wq`/`ws` bytes:
//
//   W4A4  (kInt8 = true):  nibbles widened to int8 in shared memory,
//         tcgen05.mma kind::i8 (s8 x s8 -> s32 in tensor memory), one exact
//         int32 accumulator per weight group; epilogue
//         y = s_a[m] * sum_g s_h[n,g] * acc_g.
//   W4A16 (kInt8 = false): nibbles widened to exact bf16 integers in shared
//         memory, tcgen05.mma kind::f16 (bf16 x bf16 -> f32), one fp32 partial
//         per group; epilogue y = sum_g s_h[n,g] * partial_g, i.e. exactly
//         x . (q * s_h)^T up to fp32 accumulation.
//
// Orientation ("swap AB"): the weight tile is the MMA's M = 128 operand (rows
// n), the tokens are the MMA's N operand (MT columns, 16..128), so decode
// batches of 1..128 tokens fill the instruction without padding to 128.
//
// Work decomposition: a unit is one 128-row weight tile x 128 input channels.
// Units are ordered (n-tile, m-tile, k-chunk) and split evenly over a
// persistent grid of CTAs (stream-K): every CTA gets the same number of
// units +-1, whatever the shape.  A CTA that covers a whole tile writes y
// directly; partial tiles go to workspace slots and the last CTA to finish a
// tile (an atomic ticket, no waiting) adds the slots in K order, so results
// are deterministic.  A split tile starts inside exactly one CTA's range and
// at most one split tile starts in any CTA's range, so the ticket of a tile
// is indexed by its first contributor; tickets return to zero after use.
//
// Warp roles (one CTA per SM):
//   warp 0      TMA producer for packed weight tiles (8-stage ring, 8 KB each)
//   warp 1      TMA producer for activation tiles (128-byte swizzled)
//   warp 2      tensor-memory allocation and the single MMA-issuing thread
//   warp 3      idle
//   8 warps     converters: packed nibbles -> int8 / bf16 operand tiles
//   4..16 warps epilogue: tensor memory -> registers, group scales, output
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "device_common.cuh"

namespace qspec {

constexpr int kTileN = 128;                      // weight rows per tile (MMA M)
constexpr int kUnitK = 128;                      // input channels per unit
constexpr int kPkBytes = kTileN * kUnitK / 2;    // packed bytes per unit
constexpr int kNumPk = 8;                        // packed-weight ring depth
constexpr int kNumAcc = 4;                       // tensor-memory group ring
constexpr int kConvWarps = 8;
constexpr int kCtlWarps = 4;
constexpr int kSmemLimit = 232448;               // sm_100 dynamic shared memory per CTA
constexpr int kMaxGrid = 1024;                   // ticket slots in the workspace

__host__ __device__ constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <bool kInt8, int MT>
struct GemmCfg {
  static_assert(MT % 16 == 0 && MT >= 16 && MT <= 128, "token tile must be 16..128, step 16");
  static constexpr int kElem = kInt8 ? 1 : 2;                    // bytes per widened element
  static constexpr int kAtoms = kUnitK * kElem / 128;            // 128-byte K atoms per row
  static constexpr int kCvBytes = kTileN * kUnitK * kElem;       // widened weight tile
  static constexpr int kXBytes = MT * 128 * kAtoms;              // activation tile
  static constexpr int kMmaK = kInt8 ? 32 : 16;
  static constexpr int kMmas = kUnitK / kMmaK;                   // MMAs per unit
  static constexpr int kTeams = (MT <= 48) ? 1 : (MT <= 96 ? 2 : 4);
  static constexpr int kEpiWarps = 4 * kTeams;
  static constexpr int kCols = MT / kTeams;                      // token columns per epilogue thread
  static_assert(kCols % 8 == 0, "epilogue columns must be a multiple of 8");
  static constexpr int kWarps = kCtlWarps + kConvWarps + kEpiWarps;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kBarBytes = 512;
  static constexpr int kRingBytes = kCvBytes + kXBytes;
  static constexpr int kNumCvRaw = (kSmemLimit - 1024 - kBarBytes - kNumPk * kPkBytes) / kRingBytes;
  static constexpr int kNumCv = kNumCvRaw > 4 ? 4 : kNumCvRaw;
  static_assert(kNumCv >= 2, "shared memory too small for a double-buffered operand ring");
  static constexpr int kSmemBytes = 1024 + kNumPk * kPkBytes + kNumCv * kRingBytes + kBarBytes;
  static constexpr int kTmemCols = pow2_at_least(kNumAcc * MT);
  static_assert(kTmemCols <= 512, "tensor memory overflow");
};

struct GemmArgs {
  int M, N, K;
  int groups_per_row;      // K / group
  int groups_per_unit;     // 128 / group (1 or 2)
  int m_tiles, n_tiles, ku;
  long long units;         // m_tiles * n_tiles * ku
  const uint16_t* ws;      // fp16 scales [N][K/group]
  const float* s_a;        // W4A4: per-token scales [M]
  float* y;                // [M][N]
  int32_t* dbg_acc;        // optional W4A4 per-group accumulators [M][N][K/group]
  uint32_t* status;        // device status word
  uint32_t* counters;      // tickets [kMaxGrid], indexed by a split tile's first CTA
  float* partials;         // [2 * gridDim.x][MT][128]
};

// First unit of CTA c when `units` are split over `grid` CTAs.
__host__ __device__ __forceinline__ long long unit_begin(long long c, long long units,
                                                         long long grid) {
  return (c * units) / grid;
}
// The CTA that owns unit u.
__host__ __device__ __forceinline__ long long unit_owner(long long u, long long units,
                                                         long long grid) {
  return ((u + 1) * grid - 1) / units;
}

__device__ __forceinline__ uint32_t bf16x2_minus_136(uint32_t v) {
  // (128 + u) - 136 = u - 8 = q, exact in bf16.  fma(v, 1.0, -136.0).
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(v), "r"(0x3F803F80u), "r"(0xC308C308u));
  return d;
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7])
      : "r"(taddr)
      : "memory");
}

template <bool kInt8, int MT>
__global__ void __launch_bounds__(GemmCfg<kInt8, MT>::kThreads, 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                 const __grid_constant__ CUtensorMap tmap_x, const GemmArgs args) {
  using C = GemmCfg<kInt8, MT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* pk_buf = smem;
  uint8_t* cv_buf = pk_buf + kNumPk * kPkBytes;
  uint8_t* x_buf = cv_buf + C::kNumCv * C::kCvBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(x_buf + C::kNumCv * C::kXBytes);
  uint64_t* pk_full = bars;
  uint64_t* pk_empty = pk_full + kNumPk;
  uint64_t* cv_full = pk_empty + kNumPk;
  uint64_t* x_full = cv_full + 4;
  uint64_t* cv_empty = x_full + 4;
  uint64_t* acc_full = cv_empty + 4;
  uint64_t* acc_empty = acc_full + kNumAcc;
  uint64_t* mma_done = acc_empty + kNumAcc;
  uint64_t* epi_sync = mma_done + 1;
  uint32_t* misc = reinterpret_cast<uint32_t*>(epi_sync + 1);
  // misc[0]: tensor-memory base; misc[1]: abort flag; misc[2]: reducer flag
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long grid = gridDim.x;
  const long long cta = blockIdx.x;
  const long long units = args.units;
  const long long u_begin = unit_begin(cta, units, grid);
  const long long u_end = unit_begin(cta + 1, units, grid);
  const int ku = args.ku;
  const int gpu = args.groups_per_unit;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNumPk; ++s) {
      mbar_init(smem_u32(&pk_full[s]), 1);
      mbar_init(smem_u32(&pk_empty[s]), kConvWarps);
    }
    for (int s = 0; s < C::kNumCv; ++s) {
      mbar_init(smem_u32(&cv_full[s]), kConvWarps);
      mbar_init(smem_u32(&x_full[s]), 1);
      mbar_init(smem_u32(&cv_empty[s]), 1);
    }
    for (int b = 0; b < kNumAcc; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), C::kEpiWarps);
    }
    mbar_init(smem_u32(mma_done), 1);
    mbar_init(smem_u32(epi_sync), C::kEpiWarps);
    misc[1] = 0;
    misc[2] = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_w);
    prefetch_tensormap(&tmap_x);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&misc[0]), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  QSPEC_TRACE_AT(tmem_base & 0xFFFF);
  if (!QSPEC_ALIGN_OK(smem_u32(smem), 1024) || !QSPEC_ALIGN_OK(smem_u32(bars), 8)) *abort_flag = 1;

  if (warp == 0) {
    // ------------------------------------------------ packed-weight producer
    if (lane == 0) {
      int i = 0;
      for (long long u = u_begin; u < u_end; ++u, ++i) {
        const int s = i % kNumPk;
        const uint32_t ph = (i / kNumPk) & 1;
        if (!mbar_wait(smem_u32(&pk_empty[s]), ph ^ 1, abort_flag, args.status)) break;
        const long long t = u / ku;
        const int kc = static_cast<int>(u - t * ku);
        const int n_tile = static_cast<int>(t / args.m_tiles);
        QSPEC_TRACE_AT(i);
        if (!QSPEC_ALIGN_OK(smem_u32(pk_buf + s * kPkBytes), 128)) break;
        mbar_arrive_expect_tx(smem_u32(&pk_full[s]), kPkBytes);
        tma_load_2d(smem_u32(pk_buf + s * kPkBytes), &tmap_w, smem_u32(&pk_full[s]),
                    kc * (kUnitK / 2), n_tile * kTileN);
      }
      if (*abort_flag) {
        for (int j = (i > kNumPk ? i - kNumPk : 0); j < i; ++j)
          mbar_wait_drain(smem_u32(&pk_full[j % kNumPk]), (j / kNumPk) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ activation producer
    if (lane == 0) {
      int i = 0;
      for (long long u = u_begin; u < u_end; ++u, ++i) {
        const int s = i % C::kNumCv;
        const uint32_t ph = (i / C::kNumCv) & 1;
        if (!mbar_wait(smem_u32(&cv_empty[s]), ph ^ 1, abort_flag, args.status)) break;
        const long long t = u / ku;
        const int kc = static_cast<int>(u - t * ku);
        const int m_tile = static_cast<int>(t % args.m_tiles);
        QSPEC_TRACE_AT(i);
        if (!QSPEC_ALIGN_OK(smem_u32(x_buf + s * C::kXBytes), 1024)) break;
        mbar_arrive_expect_tx(smem_u32(&x_full[s]), C::kXBytes);
#pragma unroll
        for (int a = 0; a < C::kAtoms; ++a) {
          tma_load_2d(smem_u32(x_buf + s * C::kXBytes + a * MT * 128), &tmap_x,
                      smem_u32(&x_full[s]), kc * kUnitK + a * (128 / C::kElem), m_tile * MT);
        }
      }
      if (*abort_flag) {
        for (int j = (i > C::kNumCv ? i - C::kNumCv : 0); j < i; ++j)
          mbar_wait_drain(smem_u32(&x_full[j % C::kNumCv]), (j / C::kNumCv) & 1);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = kInt8 ? idesc_i8(MT) : idesc_bf16(MT);
      const int per_group = C::kMmas / gpu;
      int i = 0, j = 0;
      bool ok = true;
      for (long long u = u_begin; u < u_end && ok; ++u, ++i) {
        const int s = i % C::kNumCv;
        const uint32_t ph = (i / C::kNumCv) & 1;
        if (!mbar_wait(smem_u32(&cv_full[s]), ph, abort_flag, args.status)) break;
        if (!mbar_wait(smem_u32(&x_full[s]), ph, abort_flag, args.status)) break;
        tc_fence_after();
        QSPEC_TRACE_AT(i);
        const uint32_t a_base = smem_u32(cv_buf + s * C::kCvBytes);
        const uint32_t b_base = smem_u32(x_buf + s * C::kXBytes);
        for (int h = 0; h < gpu; ++h, ++j) {
          const int b = j % kNumAcc;
          const uint32_t pha = (j / kNumAcc) & 1;
          if (!mbar_wait(smem_u32(&acc_empty[b]), pha ^ 1, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kk = 0; kk < per_group; ++kk) {
            const uint32_t kbyte = static_cast<uint32_t>(h * per_group + kk) * 32u;
            const uint32_t atom = kbyte >> 7, within = kbyte & 127u;
            const uint64_t a_desc = smem_desc_sw128(a_base + atom * (kTileN * 128) + within);
            const uint64_t b_desc = smem_desc_sw128(b_base + atom * (MT * 128) + within);
            QSPEC_TRACE_AT(0x8000 | (j << 4) | kk);
            if (!QSPEC_ALIGN_OK(a_base + atom * (kTileN * 128) + within, 16) ||
                !QSPEC_ALIGN_OK(b_base + atom * (MT * 128) + within, 16) ||
                !QSPEC_ALIGN_OK(static_cast<uint32_t>(b * MT) & 0xFFFFu, 8))
              continue;
            mma_ss<kInt8>(tmem_base + static_cast<uint32_t>(b * MT), a_desc, b_desc, idesc,
                          kk > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&acc_full[b]));
          QSPEC_TRACE_AT(0x4000 | j);
        }
        if (!ok) break;
        mma_commit(smem_u32(&cv_empty[s]));
      }
      // All MMAs this thread issued have finished once mma_done completes.
      mma_commit(smem_u32(mma_done));
      mbar_wait_drain(smem_u32(mma_done), 0);
    }
    __syncwarp();
  } else if (warp >= kCtlWarps && warp < kCtlWarps + kConvWarps) {
    // ------------------------------------------------ converters
    const int ct = threadIdx.x - kCtlWarps * 32;
    int i = 0;
    for (long long u = u_begin; u < u_end; ++u, ++i) {
      const int sp = i % kNumPk;
      const uint32_t php = (i / kNumPk) & 1;
      const int sc = i % C::kNumCv;
      const uint32_t phc = (i / C::kNumCv) & 1;
      bool ok = mbar_wait(smem_u32(&pk_full[sp]), php, abort_flag, args.status);
      ok = ok && mbar_wait(smem_u32(&cv_empty[sc]), phc ^ 1, abort_flag, args.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint8_t* src = pk_buf + sp * kPkBytes;
      uint8_t* dst = cv_buf + sc * C::kCvBytes;
      QSPEC_TRACE_AT(i);
#pragma unroll
      for (int it = 0; it < kPkBytes / 16 / (kConvWarps * 32); ++it) {
        const int ch = ct + it * kConvWarps * 32;   // 16-byte chunk of the packed tile
        if (!QSPEC_ALIGN_OK(smem_u32(src + ch * 16), 16)) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(src + ch * 16);
        const int r = ch >> 2;                      // weight row within the tile
        const int p = ch & 3;                       // which 32 input channels of the row
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        if constexpr (kInt8) {
          uint32_t o[8];
#pragma unroll
          for (int wi = 0; wi < 4; ++wi) {
            // offset-binary q + 8 per byte: even k in e, odd k in od
            const uint32_t e = (wv[wi] & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t od = ((wv[wi] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t t0 = prmt(e, od, 0x5140u);   // k0 k1 k2 k3
            const uint32_t t1 = prmt(e, od, 0x7362u);   // k4 k5 k6 k7
            // q + 8 in [0,15] -> signed byte q, no carries between bytes
            o[2 * wi] = (t0 + 0x78787878u) ^ 0x80808080u;
            o[2 * wi + 1] = (t1 + 0x78787878u) ^ 0x80808080u;
          }
          uint8_t* row = dst + r * 128;
          const int c0 = 2 * p, c1 = 2 * p + 1;
          if (!QSPEC_ALIGN_OK(smem_u32(row + ((c0 ^ (r & 7)) << 4)), 16) ||
              !QSPEC_ALIGN_OK(smem_u32(row + ((c1 ^ (r & 7)) << 4)), 16))
            continue;
          *reinterpret_cast<uint4*>(row + ((c0 ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(row + ((c1 ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
          uint8_t* row = dst + (p >> 1) * (kTileN * 128) + r * 128;
#pragma unroll
          for (int wi = 0; wi < 4; ++wi) {
            const uint32_t e = (wv[wi] & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t od = ((wv[wi] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t t0 = prmt(e, od, 0x5140u);   // k0 k1 k2 k3 (offset binary)
            const uint32_t t1 = prmt(e, od, 0x7362u);   // k4 k5 k6 k7
            // bf16 bit pattern 0x43uu is the value 128 + u
            const uint32_t b0 = bf16x2_minus_136(prmt(t0, 0x43434343u, 0x4140u));
            const uint32_t b1 = bf16x2_minus_136(prmt(t0, 0x43434343u, 0x4342u));
            const uint32_t b2 = bf16x2_minus_136(prmt(t1, 0x43434343u, 0x4140u));
            const uint32_t b3 = bf16x2_minus_136(prmt(t1, 0x43434343u, 0x4342u));
            const int c = 4 * (p & 1) + wi;
            if (!QSPEC_ALIGN_OK(smem_u32(row + ((c ^ (r & 7)) << 4)), 16)) continue;
            *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = make_uint4(b0, b1, b2, b3);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      QSPEC_TRACE_AT(0x4000 | i);
      if (lane == 0) {
        mbar_arrive(smem_u32(&pk_empty[sp]));
        mbar_arrive(smem_u32(&cv_full[sc]));
      }
    }
  } else if (warp >= kCtlWarps + kConvWarps) {
    // ------------------------------------------------ epilogue (warp 3 is idle and lands nowhere)
    const int ew = warp - (kCtlWarps + kConvWarps);
    const int quad = warp & 3;                 // tensor-memory lanes this warp may read
    const int team = ew >> 2;
    const int col0 = team * C::kCols;
    const int row = quad * 32 + lane;
    const int et = ew * 32 + lane;             // 0 .. kEpiWarps*32-1
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    volatile int* reducer_flag = reinterpret_cast<volatile int*>(&misc[2]);
    float run[C::kCols];
    int j = 0;
    bool ok = true;
    uint32_t epi_phase = 0;
    // All epilogue warps meet here; bounded, unlike a hardware named barrier.
    auto epi_barrier = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(epi_sync));
      const bool fine = __all_sync(0xffffffffu, mbar_wait(smem_u32(epi_sync), epi_phase, abort_flag, args.status));
      epi_phase ^= 1u;
      return fine;
    };
    long long u = u_begin;
    while (u < u_end && ok) {
      const long long t = u / ku;
      const long long seg_start = u;
      const long long tile_u0 = t * ku;
      const long long seg_end = (u_end < tile_u0 + ku) ? u_end : tile_u0 + ku;
      const int n_tile = static_cast<int>(t / args.m_tiles);
      const int m_tile = static_cast<int>(t - static_cast<long long>(n_tile) * args.m_tiles);
      const int n = n_tile * kTileN + row;
      const int m0 = m_tile * MT + col0;
#pragma unroll
      for (int c = 0; c < C::kCols; ++c) run[c] = 0.f;
      for (; u < seg_end && ok; ++u) {
        const int kc = static_cast<int>(u - tile_u0);
        for (int h = 0; h < gpu; ++h, ++j) {
          const int b = j % kNumAcc;
          const uint32_t pha = (j / kNumAcc) & 1;
          const int g = kc * gpu + h;
          const float sc = (n < args.N)
                               ? __half2float(__ushort_as_half(args.ws[static_cast<long long>(n) * args.groups_per_row + g]))
                               : 0.f;
          ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full[b]), pha, abort_flag, args.status));
          if (!ok) break;
          tc_fence_after();
          const uint32_t taddr = lane_addr + static_cast<uint32_t>(b * MT + col0);
          QSPEC_TRACE_AT(j);
#pragma unroll
          for (int c = 0; c < C::kCols; c += 8) {
            uint32_t v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (QSPEC_ALIGN_OK((taddr + c) & 0xFFFFu, 8)) tmem_ld8(taddr + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float a = kInt8 ? static_cast<float>(static_cast<int>(v[e])) : __uint_as_float(v[e]);
              run[c + e] = fmaf(sc, a, run[c + e]);
            }
            if constexpr (kInt8) {
              if (args.dbg_acc != nullptr && n < args.N) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const int m = m0 + c + e;
                  if (m < args.M)
                    args.dbg_acc[(static_cast<long long>(m) * args.N + n) * args.groups_per_row + g] =
                        static_cast<int>(v[e]);
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          QSPEC_TRACE_AT(0x4000 | j);
          if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
        }
      }
      if (!ok) break;

      const bool full = (seg_start == tile_u0) && (seg_end == tile_u0 + ku);
      QSPEC_TRACE_AT(full ? 0x2001 : 0x2000);
      bool write_out = full;
      if (!full) {
        // Publish this CTA's share of the tile, then take a ticket.
        const int slot = static_cast<int>(2 * cta + (seg_start == u_begin ? 0 : 1));
        float* mine = args.partials + static_cast<long long>(slot) * MT * kTileN;
#pragma unroll
        for (int c = 0; c < C::kCols; ++c) mine[(col0 + c) * kTileN + row] = run[c];
        __threadfence();
        if (!epi_barrier()) break;
        const long long c_lo = unit_owner(tile_u0, units, grid);
        const long long c_hi = unit_owner(tile_u0 + ku - 1, units, grid);
        if (et == 0) {
          const uint32_t old = atomicAdd(&args.counters[c_lo], 1u);
          *reducer_flag = (old == static_cast<uint32_t>(c_hi - c_lo)) ? 1 : 0;
        }
        if (!epi_barrier()) break;
        write_out = (*reducer_flag != 0);
        QSPEC_TRACE_AT(write_out ? 0x3001 : 0x3000);
        if (write_out) {
          __threadfence();
#pragma unroll
          for (int c = 0; c < C::kCols; ++c) run[c] = 0.f;
          for (long long cc = c_lo; cc <= c_hi; ++cc) {
            const int s2 = static_cast<int>(2 * cc + (unit_begin(cc, units, grid) >= tile_u0 ? 0 : 1));
            const float* src = args.partials + static_cast<long long>(s2) * MT * kTileN;
#pragma unroll
            for (int c = 0; c < C::kCols; ++c) run[c] += __ldcg(src + (col0 + c) * kTileN + row);
          }
          if (et == 0) args.counters[c_lo] = 0u;   // ready for the next launch
        }
      }
      if (write_out && n < args.N) {
#pragma unroll
        for (int c = 0; c < C::kCols; ++c) {
          const int m = m0 + c;
          if (m < args.M) {
            const float v = kInt8 ? args.s_a[m] * run[c] : run[c];
            args.y[static_cast<long long>(m) * args.N + n] = v;
          }
        }
      }
    }
  }

  QSPEC_TRACE_AT(0xFFF0);
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  QSPEC_TRACE_AT(0xFFFF);
}

}  // namespace qspec
