// Shared-INT4 GEMM for both QSpec modes on sm_100a tensor cores.
//
// QSpec (abstract) runs one packed INT4 weight set in two modes: W4A4 for
// drafting and W4A16 for verification; the explainer essay (paragraph 4)
// notes that the modes differ mainly in how activations are handled.  This
// one kernel template serves both from the same `wq`/`ws` bytes:
//
//   W4A4  (kInt8 = true):  nibbles widened to int8 (as 16 q, three integer
//         ops per 8 weights, each 8 channels in the order 0,2,4,6,1,3,5,7,
//         which the activation quantizer matches) in shared memory, tcgen05.mma
//         kind::i8 (s8 x s8 -> s32 in tensor memory), one exact int32
//         accumulator per weight group (16 acc_g); epilogue
//         y = (s_a[m] / 16) * sum_g s_h[n,g] * (16 acc_g), bit-identical to
//         s_a[m] * sum_g s_h[n,g] * acc_g since only powers of two differ.
//   W4A16 (kInt8 = false): nibbles widened to exact bf16 integers in shared
//         memory, tcgen05.mma kind::f16 (bf16 x bf16 -> f32), one fp32 partial
//         per group; epilogue y = sum_g s_h[n,g] * partial_g, i.e. exactly
//         x . (q * s_h)^T up to fp32 accumulation.
//
// Orientation ("swap AB"): the weight tile is the MMA's M = 128 operand (rows
// n), the tokens are the MMA's N operand (MT columns, 16..128), so decode
// batches of 1..128 tokens fill the instruction without padding to 128.
//
// Work decomposition: a unit is one 128-row weight tile x 256 input channels
// (int8 mode) or x 128 (bf16 mode).  Units are ordered (n-tile, m-tile,
// k-chunk) and split evenly over a persistent grid of CTAs (stream-K): every
// CTA gets the same number of units +-1, whatever the shape.  A CTA that
// covers a whole tile writes y directly; partial tiles go to workspace slots
// and the last CTA to finish a tile (an atomic ticket, no waiting) adds the
// slots in K order, so results are deterministic.  The weight producer takes
// the tickets, so the epilogue goes straight on to the next tile; when the
// other contributor of the CTA's last tile has already published, the
// epilogue adds its share directly.  A split tile starts inside exactly one
// CTA's range and at most one split tile starts in any CTA's range, so the
// ticket of a tile is indexed by its first contributor; tickets return to
// zero after use.
//
// Warp roles (one CTA per SM):
//   warp 0      TMA producer for packed weight tiles and group-scale tiles;
//               split-tile tickets
//   warp 1      TMA producer for activation tiles (128-byte swizzled ring)
//   warps 2, 3  MMA issuers for even / odd units (warp 2 also owns the
//               tensor-memory allocation)
//   4 or 8      converters (one team in int8 mode, two in bf16 mode): packed
//   warps       nibbles -> int8 / bf16 operand tiles in tensor memory
//   4..16 warps epilogue: tensor memory -> registers, group scales, output
//
// Rings decouple the latencies: packed weights (HBM latency), widened weights
// (converter -> tensor core), activations (L2 latency), group scales, and the
// per-group accumulators in tensor memory (MMA -> epilogue).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "device_common.cuh"

namespace qspec {

constexpr int kTileN = 128;                      // weight rows per tile (MMA M)
// Input channels per unit: 256 in int8 mode (16 KB of packed weights per
// hand-off), 128 in bf16 mode (whose activation tiles are 4x larger).
__host__ __device__ constexpr int unit_k(bool int8_mode) { return int8_mode ? 256 : 128; }
constexpr int kConvTeamWarps = 4;                // a converter team: one warp per lane quadrant
constexpr int kCtlWarps = 4;
constexpr int kSmemLimit = 232448;               // sm_100 dynamic shared memory per CTA
constexpr int kMaxGrid = 1024;                   // ticket slots in the workspace
// (at most 7 activation slots: the int8 16-token tile then leaves an SM room
// for a CTA of the activation quantizer beside it)
constexpr int kMaxPk = 24, kMaxA = 8, kMaxAcc = 8, kMaxX = 7;
// Group scales arrive by TMA, 8 groups x 128 rows (2 KB) per tile, into a ring.
constexpr int kScaleTileGroups = 8;
constexpr int kScaleTileBytes = kTileN * kScaleTileGroups * 2;
constexpr int kNumSc = 8;
constexpr int kTmemCols = 512;                   // all of tensor memory: one CTA per SM
// mbarriers (rings, MMA drain, scale tiles, split-tile hand-offs) and 8 words
// of flags share a 1 KB block, in this order: pk_full, pk_empty, a_full,
// a_empty, x_full, x_empty, acc_full, acc_empty, mma_done, sc_full, sc_empty,
// flush[2], ticket[2], tail, stall.
namespace bar {
constexpr int kPkFull = 0, kPkEmpty = kPkFull + kMaxPk, kAFull = kPkEmpty + kMaxPk;
constexpr int kAEmpty = kAFull + kMaxA, kXFull = kAEmpty + kMaxA, kXEmpty = kXFull + kMaxX;
constexpr int kAccFull = kXEmpty + kMaxX, kAccEmpty = kAccFull + kMaxAcc;
constexpr int kMmaDone = kAccEmpty + kMaxAcc, kScFull = kMmaDone + 1, kScEmpty = kScFull + kNumSc;
constexpr int kFlush = kScEmpty + kNumSc, kTicket = kFlush + 2, kTail = kTicket + 2;
constexpr int kStall = kTail + 1;   // never signalled: the test hook's wait
constexpr int kCount = kStall + 1;
// Fused activation quantization only, in a block of their own: the barrier
// that hands the token scales to the epilogue, the one on which the epilogue
// warps combine a row's absmax, then the row partials and the token scales.
constexpr int kScaleReady = 0, kRowAmax = 1;
constexpr int kFusedCount = kRowAmax + 1;
}  // namespace bar
constexpr int kNumBars = bar::kCount;
// The flag words follow the barriers on a 16-byte boundary: with them 8 bytes
// off it (one barrier more), every call's set-up took several microseconds
// longer on B200 (measured: +17 to +35 % per decode GEMM call).
constexpr int kMiscOffset = (kNumBars * 8 + 15) / 16 * 16;
static_assert(kMiscOffset + 8 * 4 <= 1024, "barrier block overflow");
// The fused block: its barriers, the row absmax partials of up to 4 epilogue
// warps (double-buffered), then the token scales (token tiles <= 32).
constexpr int kRowPartOffset = (bar::kFusedCount * 8 + 15) / 16 * 16;
constexpr int kTokScaleOffset = kRowPartOffset + 2 * 4 * 4;
constexpr int kFusedBlockBytes = 1024;
static_assert(kTokScaleOffset + 32 * 4 <= kFusedBlockBytes, "fused block overflow");

// Arrival count of barrier b in that order.
__device__ __forceinline__ uint32_t bar_count(int b, int epi_warps) {
  if (b >= bar::kPkEmpty && b < bar::kAEmpty) return kConvTeamWarps;   // pk_empty, a_full
  if (b >= bar::kAccEmpty && b < bar::kMmaDone) return epi_warps;      // acc_empty
  if (b == bar::kMmaDone) return 2;                                    // both MMA warps
  if (b >= bar::kScEmpty && b < bar::kTicket) return epi_warps;        // sc_empty, flush
  return 1;
}


__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

// kFused (drafting modes, token tiles of 16 or 32): the kernel quantizes the
// bf16 activations itself (see qgemm_kernel) instead of a separate pre-pass
// kernel doing it.
template <bool kInt8, int MT, bool kFused = false>
struct GemmCfg {
  static_assert(MT % 16 == 0 && MT >= 16 && MT <= 128, "token tile must be 16..128, step 16");
  static_assert(!kFused || (kInt8 && MT <= 32), "fused activation quantization: int8, MT <= 32");
  static constexpr int kUnitK = unit_k(kInt8);
  static constexpr int kPkBytes = kTileN * kUnitK / 2;           // packed bytes per unit
  static constexpr int kElem = kInt8 ? 1 : 2;                    // bytes per widened element
  static constexpr int kAtoms = kUnitK * kElem / 128;            // 128-byte K atoms per row
  static constexpr int kXBytes = MT * 128 * kAtoms;              // activation tile
  // Widened weight units live in tensor memory (lane = weight row, 32-bit
  // columns along K): 32 columns of int8 or 64 of bf16 per unit, then the
  // per-group accumulators (MT columns each) in what is left.
  static constexpr int kACols = kUnitK * kElem / 4;
  static constexpr int kNumA = kInt8 ? (MT <= 32 ? 6 : (MT <= 64 ? 4 : 2)) : 4;
  static constexpr int kAccCol0 = kNumA * kACols;
  static constexpr int kNumAcc = cmin(kMaxAcc, (kTmemCols - kAccCol0) / MT);
  static_assert(kNumAcc >= 2, "tensor memory too small for two accumulators");
  static constexpr int kMmaK = kInt8 ? 32 : 16;
  static constexpr int kMmas = kUnitK / kMmaK;                   // MMAs per unit
  static constexpr int kTeams = (MT <= 48) ? 1 : (MT <= 96 ? 2 : 4);   // column teams
  static constexpr int kEpiWarps = 4 * kTeams;
  static constexpr int kCols = MT / kTeams;                      // token columns per epilogue thread
  static_assert(kCols % 8 == 0, "epilogue columns must be a multiple of 8");
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  // Converter teams take alternate units: two in bf16 mode (13 integer/bf16
  // ops per 8 weights), one in int8 mode (3), where a second team's warps
  // cost the other roles more issue slots than they save.
  static constexpr int kConvTeams = kInt8 ? 1 : 2;
  static constexpr int kConvWarps = kConvTeamWarps * kConvTeams;
  static constexpr int kWarps = kCtlWarps + kConvWarps + kEpiWarps;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kBarBytes = 1024 + (kFused ? kFusedBlockBytes : 0);
  static constexpr int kScaleBytes = kNumSc * kScaleTileBytes;
  // Ring depths from the shared-memory budget: packed weights first (they
  // cover HBM latency), activations (an L2 hit) with what is left.
  static constexpr int kAvail = kSmemLimit - 1024 - kBarBytes - kScaleBytes;
  static constexpr int kNumX = cmin(kMaxX, cmax(3, (kAvail - 128 * 1024) / kXBytes));
  static constexpr int kNumPk = cmin(kMaxPk, (kAvail - kNumX * kXBytes) / kPkBytes);
  static_assert(kNumX >= 3 && kNumPk >= 6, "shared memory too small for the rings");
  static constexpr int kSmemBytes =
      1024 + kNumPk * kPkBytes + kNumX * kXBytes + kScaleBytes + kBarBytes;
  static_assert(kSmemBytes <= kSmemLimit, "shared memory overflow");
};

struct GemmArgs {
  int M, N, K;
  int groups_per_row;      // K / group
  int groups_per_unit;     // 128 / group (1 or 2)
  int m_tiles, n_tiles, ku;
  long long units;         // m_tiles * n_tiles * ku
  int weights_ready;       // wq/ws may be read before the preceding grid completes
  uint32_t test_stall_ns;  // test hook (0 = off): the weight producer first waits this
                           // long on a barrier that nothing signals, then gives up
  float qmax;              // activation codes: 7 (4-bit) or 127 (8-bit)
  const uint16_t* x;       // fused: bf16 activations [M][K]
  int8_t* xq;              // fused: int8 codes [M][K] written by this kernel (workspace)
  uint32_t* qsync;         // fused: [0] rows quantized, [1] CTAs that have seen them all
  const uint16_t* ws;      // fp16 scales [N][K/group]
  const float* s_a;        // drafting modes: per-token scales [M] (fused: written by this kernel)
  float* y;                // [M][N]
  int32_t* dbg_acc;        // optional W4A4 per-group accumulators [M][N][K/group]
  uint32_t* status;        // device status word
  uint32_t* counters;      // tickets [kMaxGrid], indexed by a split tile's first CTA
  float* partials;         // [2 * gridDim.x][MT][128]
};

// Unit arithmetic is 32-bit (the host keeps units below kMaxUnits and the
// grid at most kMaxGrid, so no product reaches 2^32): a 64-bit division is a
// long software sequence on the GPU.
constexpr long long kMaxUnits = 1ll << 22;

// First unit of CTA c when `units` are split over `grid` CTAs.
__host__ __device__ __forceinline__ uint32_t unit_begin(uint32_t c, uint32_t units,
                                                        uint32_t grid) {
  return (c * units) / grid;
}
// The CTA that owns unit u.
__host__ __device__ __forceinline__ uint32_t unit_owner(uint32_t u, uint32_t units,
                                                        uint32_t grid) {
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

// Coordinates of a unit, advanced without divisions inside the hot loops
// (64-bit integer division is a long software sequence on the GPU).
struct UnitCursor {
  int kc, m_tile, n_tile;
  __device__ __forceinline__ void init(long long u, int ku, int m_tiles) {
    const uint32_t t = static_cast<uint32_t>(u) / static_cast<uint32_t>(ku);
    kc = static_cast<int>(static_cast<uint32_t>(u) - t * static_cast<uint32_t>(ku));
    n_tile = static_cast<int>(t / static_cast<uint32_t>(m_tiles));
    m_tile = static_cast<int>(t - static_cast<uint32_t>(n_tile) * static_cast<uint32_t>(m_tiles));
  }
  __device__ __forceinline__ void next(int ku, int m_tiles) {
    if (++kc == ku) {
      kc = 0;
      if (++m_tile == m_tiles) {
        m_tile = 0;
        ++n_tile;
      }
    }
  }
};

// Position in a ring of n slots (slot, phase parity) for item index i,
// advanced without divisions: step(by) for any by <= n.
struct RingPos {
  int slot;
  uint32_t phase;
  __device__ __forceinline__ void init(int i, int n) {
    slot = i % n;
    phase = static_cast<uint32_t>(i / n) & 1u;
  }
  __device__ __forceinline__ void step(int by, int n) {
    slot += by;
    if (slot >= n) {
      slot -= n;
      phase ^= 1u;
    }
  }
};

// Programmatic dependent launch: wait for the grid this one depends on (a
// no-op when launched without the attribute); let dependents start early.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Ticket of split tile t after this CTA published its share (one thread).
// Returns true for the tile's last contributor, which then adds the shares;
// the last contributor also returns the ticket to zero for the next launch
// (nobody else touches it once every contributor has arrived).
__device__ __forceinline__ bool take_tile_ticket(const GemmArgs& args, long long t,
                                                 long long units, long long grid) {
  const long long tile_u0 = t * args.ku;
  const long long c_lo = unit_owner(tile_u0, units, grid);
  const long long c_hi = unit_owner(tile_u0 + args.ku - 1, units, grid);
  // Release: this CTA's share (seen by this thread through an mbarrier) is
  // published with the ticket.  Acquire: the last contributor sees every share.
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;"
               : "=r"(old)
               : "l"(args.counters + c_lo)
               : "memory");
  const bool last = old == static_cast<uint32_t>(c_hi - c_lo);
  if (last) args.counters[c_lo] = 0u;
  return last;
}

// Number of contributors that have ticketed split tile t so far (relaxed;
// pair with fence_acquire_gpu before reading their shares).
__device__ __forceinline__ uint32_t peek_ticket(const uint32_t* counter) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acquire_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_cta(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_cta(uint32_t* p, uint32_t v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// Fused activation quantization of one token row by the NW epilogue warps of
// a CTA, with the arithmetic of quant_act_kernel: a = max_k |x|, s_a = a / qmax
// and inv = qmax / a (IEEE fp32 divisions), q = rint(x * inv) with the product
// rounded to fp32 (within [-qmax, qmax] for finite x), a zero row giving 0; the codes are
// stored as the GEMM reads them, each 8 channels in the order 0,2,4,6,1,3,5,7.
// Each thread keeps up to kCache 16-byte chunks of the row in registers between
// the two passes (all its loads in flight at once); rows longer than
// 8 * kCache * 32 * NW elements read the rest twice.  The warps combine their
// absmax partials through shared memory and the barrier `row_bar` (count NW,
// one phase per row; `part` is double-buffered by that phase).  Returns false
// if the wait gave up.  K is a multiple of 8; rows are 16-byte aligned.
template <int NW>
__device__ __forceinline__ bool quantize_row_team(const uint16_t* xr, int K, int8_t* qr,
                                                  float* s_out, float qmax, int ew, int lane,
                                                  float* part, uint32_t row_bar, uint32_t phase,
                                                  volatile int* abort_flag, uint32_t* status) {
  constexpr int T = NW * 32;
  constexpr int kCache = 8;
  const int t = ew * 32 + lane;
  auto bf = [](uint32_t bits16) { return __uint_as_float(bits16 << 16); };
  auto absmax8 = [&](const uint4& u, float m) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf(w[j] & 0xFFFFu)), fabsf(bf(w[j] >> 16))));
    return m;
  };
  uint4 cache[kCache];
#pragma unroll
  for (int j = 0; j < kCache; ++j) {
    const int c = (t + T * j) * 8;
    if (c < K) cache[j] = __ldcg(reinterpret_cast<const uint4*>(xr + c));   // written by the preceding grid
  }
  float a = 0.f;
#pragma unroll
  for (int j = 0; j < kCache; ++j)
    if ((t + T * j) * 8 < K) a = absmax8(cache[j], a);
  for (int c = (t + T * kCache) * 8; c < K; c += T * 8)
    a = absmax8(__ldcg(reinterpret_cast<const uint4*>(xr + c)), a);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  float* pp = part + (phase & 1u) * 4;
  if (lane == 0) pp[ew] = a;
  __syncwarp();
  if (lane == 0) mbar_arrive(row_bar);
  if (!warp_wait(row_bar, phase & 1u, abort_flag, status)) return false;
  a = pp[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) a = fmaxf(a, pp[w]);
  // rint(x * inv) by an fp32 add of 1.5 x 2^23 (the code lands in the low
  // byte; finite x never needs the clamp), as in quant_act_kernel
  const float inv = (a == 0.f) ? 0.f : __fdiv_rn(qmax, a);
  if (t == 0) *s_out = __fdiv_rn(a, qmax);
  auto code = [inv](float v) { return __float_as_uint(__fadd_rn(__fmul_rn(v, inv), 12582912.0f)); };
  auto low4 = [](uint32_t a4, uint32_t b4, uint32_t c4, uint32_t d4) {
    return __byte_perm(__byte_perm(a4, b4, 0x0040), __byte_perm(c4, d4, 0x0040), 0x5410);
  };
  auto emit = [&](int c, const uint4& u) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t e[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      e[2 * j] = code(bf(w[j] & 0xFFFFu));
      e[2 * j + 1] = code(bf(w[j] >> 16));
    }
    *reinterpret_cast<uint2*>(qr + c) =
        make_uint2(low4(e[0], e[2], e[4], e[6]), low4(e[1], e[3], e[5], e[7]));
  };
#pragma unroll
  for (int j = 0; j < kCache; ++j) {
    const int c = (t + T * j) * 8;
    if (c < K) emit(c, cache[j]);
  }
  for (int c = (t + T * kCache) * 8; c < K; c += T * 8)
    emit(c, __ldcg(reinterpret_cast<const uint4*>(xr + c)));
  return true;
}

// kDbg (int8 mode only): also write the per-group integer accumulators.  A
// separate instantiation keeps those stores out of the hot loop's code.
// kFused: see GemmCfg.
template <bool kInt8, int MT, bool kDbg, bool kFused>
__global__ void __launch_bounds__(GemmCfg<kInt8, MT, kFused>::kThreads, 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                 const __grid_constant__ CUtensorMap tmap_x,
                 const __grid_constant__ CUtensorMap tmap_s, const __grid_constant__ GemmArgs args) {
  using C = GemmCfg<kInt8, MT, kFused>;
  constexpr int NPK = C::kNumPk, NA = C::kNumA, NX = C::kNumX, NACC = C::kNumAcc;
  constexpr unsigned kTraceKind = kInt8 ? 1u : 2u;   // trace builds: event-log tags
  const unsigned trace_launch = static_cast<unsigned>(reinterpret_cast<uintptr_t>(args.status) >> 8);
  (void)kTraceKind;
  (void)trace_launch;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* pk_buf = smem;
  uint8_t* x_buf = pk_buf + NPK * C::kPkBytes;
  uint8_t* sc_buf = x_buf + NX * C::kXBytes;     // group-scale tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sc_buf + C::kScaleBytes);
  uint64_t* pk_full = bars + bar::kPkFull;
  uint64_t* pk_empty = bars + bar::kPkEmpty;
  uint64_t* a_full = bars + bar::kAFull;     // widened unit in tensor memory
  uint64_t* a_empty = bars + bar::kAEmpty;
  uint64_t* x_full = bars + bar::kXFull;
  uint64_t* x_empty = bars + bar::kXEmpty;
  uint64_t* acc_full = bars + bar::kAccFull;
  uint64_t* acc_empty = bars + bar::kAccEmpty;
  uint64_t* mma_done = bars + bar::kMmaDone;
  uint64_t* sc_full = bars + bar::kScFull;   // [kNumSc]: a scale tile has landed
  uint64_t* sc_empty = bars + bar::kScEmpty; // [kNumSc]: the epilogue is done with it
  // [0]: the head split tile's share is published, [1]: the tail split tile's
  uint64_t* flush_bar = bars + bar::kFlush;
  uint64_t* ticket_bar = bars + bar::kTicket;  // ... and its ticket taken (misc[3], misc[6])
  uint64_t* tail_bar = bars + bar::kTail;      // the other contributor's tail share is out
  uint64_t* fbars = bars + 1024 / 8;                // the fused block (fused configurations only)
  uint64_t* scale_ready = fbars + bar::kScaleReady;  // the token scales are in s_tok_scale
  uint64_t* row_amax = fbars + bar::kRowAmax;        // the epilogue warps' row partials are in
  float* s_row_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(fbars) + kRowPartOffset);
  float* s_tok_scale = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(fbars) + kTokScaleOffset);
  uint32_t* misc = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(bars) + kMiscOffset);
  // misc[0]: tensor-memory base; misc[1]: abort flag; misc[3]: this CTA is the
  // last contributor of its head split tile; misc[5]: some epilogue warp left
  // its tail-tile share in the workspace; misc[6]: ... and this CTA is the
  // tail tile's last contributor; misc[7]: the preceding grid has completed
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
  // The CTA's last segment [max(u_begin, tail_u0), u_end) lies in tile t_tail;
  // it is a split tile unless it covers the whole tile.  When this CTA holds
  // the tile's first unit and exactly one other CTA (the next one, which
  // meets the tile at the start of its range) holds the rest, that CTA's
  // share is normally published long before this one gets there: the tail
  // then takes a fast path that adds the share directly (tail_fast).
  const long long t_tail =
      (u_begin < u_end) ? static_cast<uint32_t>(u_end - 1) / static_cast<uint32_t>(ku) : 0;
  const long long tail_u0 = t_tail * ku;
  const bool tail_split = (u_begin < u_end) && !(u_begin <= tail_u0 && u_end == tail_u0 + ku);
  const bool tail_fast = tail_split && u_begin <= tail_u0 &&
                         unit_owner(tail_u0 + ku - 1, units, grid) == cta + 1;

  if (threadIdx.x == 0) QSPEC_PHASE(0);
  if (warp == 0) {
    // The 32 lanes of warp 0 initialise the barriers in a compact loop.  (One
    // thread walking all of them compiled, depending on their number, into a
    // set-up several microseconds long: +20 to +45 % per decode call.)
#pragma unroll 1
    for (int b = lane; b < kNumBars; b += 32) mbar_init(smem_u32(&bars[b]), bar_count(b, C::kEpiWarps));
    if constexpr (kFused) {
      if (lane == 0) {
        mbar_init(smem_u32(scale_ready), 1);
        mbar_init(smem_u32(row_amax), C::kEpiWarps);
      }
    }
    fence_barrier_init();   // each lane's inits, before the async proxy uses them
    if (lane == 0) {
      misc[1] = 0;
      misc[3] = 0;
      misc[5] = 0;
      misc[6] = 0;
      misc[7] = 0;
    }
    __syncwarp();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_w);
    prefetch_tensormap(&tmap_x);
    prefetch_tensormap(&tmap_s);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&misc[0]), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  QSPEC_TRACE_AT(tmem_base & 0xFFFF);
  if (threadIdx.x == 0) QSPEC_PHASE(1);
  // The next grid may be scheduled as SMs free up; it waits for this one to
  // complete before it reads inputs or writes anything.
  if (threadIdx.x == 0) grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------ packed-weight producer
    // (the whole warp walks the loop; an elected lane issues the copies)
    // This warp also takes the split tiles' tickets: the CTA's first tile's
    // when its share is published (probed once per unit, far enough ahead
    // that the ticket's latency costs the pipeline nothing), the last tile's
    // after its loop (see below); any reduction is left to the epilogue's
    // many threads.
    const long long t_head = static_cast<uint32_t>(u_begin) / static_cast<uint32_t>(ku);
    const long long head_end = (u_end < (t_head + 1) * ku) ? u_end : (t_head + 1) * ku;
    bool head_pending = (u_begin < u_end) && head_end < u_end && u_begin != t_head * ku;
    // The weights may come from the preceding grid unless the caller vouches
    // otherwise.  W4A4 with the activation pre-pass runs behind that kernel,
    // which then launches this grid only after the grid before it has completed.
    if constexpr (!kInt8 || kFused) {
      if (!args.weights_ready) grid_dependency_wait();
    }
    // Test hook: a wait that nothing completes runs out, and the CTA gives up
    // as it would on a real stall (abort flag, device status, every role
    // stops at its next wait, copies in flight are drained).
    bool run = true;
    if (args.test_stall_ns != 0u)
      run = __all_sync(0xffffffffu, mbar_wait_slow(smem_u32(bars + bar::kStall), 0, abort_flag,
                                                   args.status, args.test_stall_ns));
    // Group scales: one TMA tile (8 groups x 128 rows) whenever a unit starts a
    // new run of 8 groups of its tile, or is this CTA's first unit; the
    // epilogue walks the same sequence.
    RingPos rs;
    rs.init(0, kNumSc);
    int n_sc = 0;
    bool tail_seen = false;
    bool poll_pending = false;
    uint32_t poll_val = 0;
    int i = 0;
    UnitCursor cur;
    cur.init(u_begin, ku, args.m_tiles);
    for (long long u = u_begin; run && u < u_end; ++u, ++i, cur.next(ku, args.m_tiles)) {
      const int s = i % NPK;
      const uint32_t ph = (i / NPK) & 1;
      if (!warp_wait(smem_u32(&pk_empty[s]), ph ^ 1, abort_flag, args.status)) break;
      if (elect_one_lane()) {
        mbar_arrive_expect_tx(smem_u32(&pk_full[s]), C::kPkBytes);
        tma_load_2d(smem_u32(pk_buf + s * C::kPkBytes), &tmap_w, smem_u32(&pk_full[s]),
                    cur.kc * (C::kUnitK / 2), cur.n_tile * kTileN);
        if (i == 0) QSPEC_PHASE(4);
        if (u + 1 == u_end) QSPEC_PHASE(9);
      }
      __syncwarp();
      const int g0 = cur.kc * gpu;
      if (u == u_begin || (g0 & (kScaleTileGroups - 1)) == 0) {
        if (!warp_wait(smem_u32(&sc_empty[rs.slot]), rs.phase ^ 1u, abort_flag, args.status)) break;
        if (elect_one_lane()) {
          mbar_arrive_expect_tx(smem_u32(&sc_full[rs.slot]), kScaleTileBytes);
          tma_load_2d(smem_u32(sc_buf + rs.slot * kScaleTileBytes), &tmap_s, smem_u32(&sc_full[rs.slot]),
                      g0 & ~(kScaleTileGroups - 1), cur.n_tile * kTileN);
        }
        __syncwarp();
        rs.step(1, kNumSc);
        ++n_sc;
      }
      // (only once the epilogue has seen the preceding grid complete: its
      // tickets may still be in use before that)
      if (tail_fast && u >= tail_u0 && lane == 0 && !tail_seen && ld_acquire_cta(&misc[7]) != 0u) {
        if (poll_pending && poll_val == 1u) {
          fence_acquire_gpu();
          mbar_arrive(smem_u32(tail_bar));
          tail_seen = true;
        } else {
          poll_val = peek_ticket(args.counters + cta);
          poll_pending = true;
        }
      }
      __syncwarp();
      if (head_pending && __all_sync(0xffffffffu, mbar_test_wait(smem_u32(flush_bar), 0))) {
        if (lane == 0) {
          misc[3] = take_tile_ticket(args, t_head, units, grid) ? 1u : 0u;
          mbar_arrive(smem_u32(ticket_bar));
        }
        __syncwarp();
        head_pending = false;
      }
    }
    if (head_pending && warp_wait(smem_u32(flush_bar), 0, abort_flag, args.status)) {
      if (lane == 0) {
        misc[3] = take_tile_ticket(args, t_head, units, grid) ? 1u : 0u;
        mbar_arrive(smem_u32(ticket_bar));
      }
      __syncwarp();
    }
    // Tail split tile: once this warp has issued every unit, watch the other
    // contributor's ticket (fast-path tiles) until it arrives or the epilogue
    // has finished the tail segment; then take this CTA's ticket if any
    // epilogue warp left its share in the workspace.  If every warp took the
    // fast path, this CTA was the last contributor and only returns the
    // ticket to zero.
    if (tail_split && !*abort_flag) {
      grid_dependency_wait();   // the preceding grid's tickets are settled
      bool fine = true;
      tail_seen = __shfl_sync(0xffffffffu, tail_seen ? 1 : 0, 0) != 0;
      if (tail_fast && !tail_seen) {
        const uint64_t start = global_timer_ns();
        for (;;) {
          if (__all_sync(0xffffffffu, mbar_test_wait(smem_u32(&flush_bar[1]), 0))) break;
          uint32_t c = 0;
          if (lane == 0) c = peek_ticket(args.counters + cta);
          if (__shfl_sync(0xffffffffu, c, 0) == 1u) {
            if (lane == 0) {
              fence_acquire_gpu();
              mbar_arrive(smem_u32(tail_bar));
            }
            __syncwarp();
            break;
          }
          if (*abort_flag) {
            fine = false;
            break;
          }
          if (global_timer_ns() - start > kWaitLimitNs) {
            if (lane == 0) {
              *abort_flag = 1;
              if (args.status) atomicOr(args.status, kDevTimeout);
            }
            fine = false;
            break;
          }
        }
      }
      fine = fine && warp_wait(smem_u32(&flush_bar[1]), 0, abort_flag, args.status);
      if (fine && lane == 0) {
        if (misc[5] != 0u) {
          misc[6] = take_tile_ticket(args, t_tail, units, grid) ? 1u : 0u;
          mbar_arrive(smem_u32(&ticket_bar[1]));
        } else {
          args.counters[cta] = 0u;
        }
      }
      __syncwarp();
    }
    if (*abort_flag) {
      for (int j = (i > NPK ? i - NPK : 0); j < i; ++j)
        mbar_wait_drain(smem_u32(&pk_full[j % NPK]), (j / NPK) & 1);
      for (int j = (n_sc > kNumSc ? n_sc - kNumSc : 0); j < n_sc; ++j)
        mbar_wait_drain(smem_u32(&sc_full[j % kNumSc]), (j / kNumSc) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ activation producer
    grid_dependency_wait();   // activations may come from the preceding kernel
    if (lane == 0) QSPEC_PHASE(10);
    bool xok = true;
    if constexpr (kFused) {
      // Every token row is quantized by the epilogue warps of CTA (row mod
      // grid), each warp counting its share: wait (bounded) until all M rows
      // are in the workspace, hand the token scales to the epilogue, and count
      // this CTA as having seen them; the last CTA to do so returns the
      // counters to zero for the next call.
      const uint64_t start = global_timer_ns();
      for (;;) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(args.qsync) : "memory");
        if (v >= static_cast<uint32_t>(args.M * C::kEpiWarps)) break;
        if (*abort_flag || global_timer_ns() - start > kWaitLimitNs) {
          if (lane == 0) {
            *abort_flag = 1;
            if (args.status) atomicOr(args.status, kDevTimeout);
          }
          xok = false;
          break;
        }
        __nanosleep(64);
      }
      xok = __all_sync(0xffffffffu, xok);
      if (lane == 0) QSPEC_PHASE(13);
      // the codes were written by other CTAs' generic stores; TMA reads them
      if (xok) asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    int i = 0;
    UnitCursor cur;
    cur.init(u_begin, ku, args.m_tiles);
    for (long long u = u_begin; xok && u < u_end; ++u, ++i, cur.next(ku, args.m_tiles)) {
      const int s = i % NX;
      const uint32_t ph = (i / NX) & 1;
      if (!warp_wait(smem_u32(&x_empty[s]), ph ^ 1, abort_flag, args.status)) break;
      if (elect_one_lane()) {
        mbar_arrive_expect_tx(smem_u32(&x_full[s]), C::kXBytes);
        if (i == 0) QSPEC_PHASE(14);
#pragma unroll
        for (int a = 0; a < C::kAtoms; ++a) {
          tma_load_2d(smem_u32(x_buf + s * C::kXBytes + a * MT * 128), &tmap_x,
                      smem_u32(&x_full[s]), cur.kc * C::kUnitK + a * (128 / C::kElem),
                      cur.m_tile * MT);
        }
      }
      __syncwarp();
      if constexpr (kFused) {
        // Off the critical path (the first activation tiles are on their way):
        // hand the token scales to the epilogue, and count this CTA as having
        // seen every row; the last CTA to do so zeroes the counters for the
        // next call.
        if (i == 0) {
          if (lane < args.M) s_tok_scale[lane] = __ldcg(args.s_a + lane);
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(smem_u32(scale_ready));
            if (atomicAdd(args.qsync + 1, 1u) == gridDim.x - 1) {
              args.qsync[0] = 0u;
              args.qsync[1] = 0u;
            }
          }
          __syncwarp();
        }
      }
    }
    if (*abort_flag) {
      for (int j = (i > NX ? i - NX : 0); j < i; ++j)
        mbar_wait_drain(smem_u32(&x_full[j % NX]), (j / NX) & 1);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------ MMA issuers (even / odd units)
    // The whole warp walks the loop (waits are warp-uniform); one elected lane
    // issues the tcgen05 instructions.  A (the widened weights) is read from
    // tensor memory, B (the activations) from shared memory.
    constexpr uint32_t idesc = kInt8 ? idesc_i8(MT) : idesc_bf16(MT);
    const int per_group = C::kMmas / gpu;
    const int parity = warp - 2;
    int i = parity;
    bool ok = true;
    RingPos ra, rx, racc;
    ra.init(parity, NA);
    rx.init(parity, NX);
    for (long long u = u_begin + parity; u < u_end && ok;
         u += 2, i += 2, ra.step(2, NA), rx.step(2, NX)) {
      const int sa = ra.slot;
      const int sx = rx.slot;
      racc.init(i * gpu, NACC);
      ok = warp_wait(smem_u32(&a_full[sa]), ra.phase, abort_flag, args.status);
      ok = ok && warp_wait(smem_u32(&x_full[sx]), rx.phase, abort_flag, args.status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t a_col = tmem_base + static_cast<uint32_t>(sa * C::kACols);
      const uint32_t b_base = smem_u32(x_buf + sx * C::kXBytes);
      for (int h = 0; h < gpu; ++h, racc.step(1, NACC)) {
        const int b = racc.slot;
        ok = warp_wait(smem_u32(&acc_empty[b]), racc.phase ^ 1u, abort_flag, args.status);
        if (!ok) break;
        tc_fence_after();
        // One elected lane issues the group's MMAs and its commit back to back.
        if (elect_one_lane()) {
          const uint32_t d = tmem_base + static_cast<uint32_t>(C::kAccCol0 + b * MT);
          for (int kk = 0; kk < per_group; ++kk) {
            const int step = h * per_group + kk;            // 32 bytes of K per step
            const uint32_t kbyte = static_cast<uint32_t>(step) * 32u;
            const uint32_t atom = kbyte >> 7, within = kbyte & 127u;
            const uint64_t b_desc = smem_desc_sw128(b_base + atom * (MT * 128) + within);
            mma_ts<kInt8>(d, a_col + static_cast<uint32_t>(step * 8), b_desc, idesc,
                          kk > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&acc_full[b]));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one_lane()) {
        mma_commit(smem_u32(&a_empty[sa]));
        mma_commit(smem_u32(&x_empty[sx]));
      }
      __syncwarp();
      if (i == 0 && lane == 0) QSPEC_PHASE(3);
    }
    // All MMAs this warp issued have finished once mma_done completes.
    if (elect_one_lane()) mma_commit(smem_u32(mma_done));
    __syncwarp();
    mbar_wait_drain(smem_u32(mma_done), 0);
    __syncwarp();
  } else if (warp >= kCtlWarps && warp < kCtlWarps + C::kConvWarps) {
    // ------------------------------------------------ converters
    // Teams of four warps (one per tensor-memory lane quadrant) take
    // alternate units.  Thread = weight row = tensor-memory lane: it reads the
    // row's packed bytes (int8 mode: 128 B, the TMA's 128-byte swizzle puts
    // 16-byte chunk c of row r at c ^ (r & 7); bf16 mode: 64 B, the 64-byte
    // swizzle puts it at c ^ ((r >> 1) & 3); either way a quarter warp hits
    // eight distinct bank groups), widens them in registers and stores them
    // to its own lane.
    constexpr int kChunks = C::kUnitK / 32;    // 16-byte packed chunks per row
    const int cteam = (warp - kCtlWarps) / kConvTeamWarps;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t swz = static_cast<uint32_t>(kInt8 ? (r & 7) : ((r >> 1) & 3));
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    int i = cteam;
    RingPos rp, ra;
    rp.init(cteam, NPK);
    ra.init(cteam, NA);
    for (long long u = u_begin + cteam; u < u_end;
         u += C::kConvTeams, i += C::kConvTeams, rp.step(C::kConvTeams, NPK),
         ra.step(C::kConvTeams, NA)) {
      const int sp = rp.slot;
      const int sa = ra.slot;
      bool ok = warp_wait(smem_u32(&pk_full[sp]), rp.phase, abort_flag, args.status);
      ok = ok && warp_wait(smem_u32(&a_empty[sa]), ra.phase ^ 1u, abort_flag, args.status);
      if (!ok) break;
      if (i == 0 && r == 0) QSPEC_PHASE(2);
      const uint8_t* rowp = pk_buf + sp * C::kPkBytes + r * (C::kUnitK / 2);
      uint4 v[kChunks];
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
        v[c] = *reinterpret_cast<const uint4*>(rowp + ((static_cast<uint32_t>(c) ^ swz) << 4));
      // The packed slot may be refilled (by the async proxy) once every
      // lane's reads are done.
      fence_proxy_async_smem();
      __syncwarp();
      if (elect_one_lane()) mbar_arrive(smem_u32(&pk_empty[sp]));
      __syncwarp();
      const uint32_t a_col = lane_base + static_cast<uint32_t>(sa * C::kACols);
      if constexpr (kInt8) {
        // A two's-complement nibble in the high half of a byte is the signed
        // byte 16 q, so masking alone widens: odd k are already there, even k
        // move up by 4 bits.  The accumulators come out as 16 x the exact
        // sums; the epilogue divides by 16 exactly.  Each 8 channels land in
        // the order (0,2,4,6,1,3,5,7), the order in which the activation
        // quantizer stores them for this GEMM.
#pragma unroll
        for (int half = 0; half < kChunks / 4; ++half) {   // 128 channels = 32 columns
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 vc = v[4 * half + c];
            const uint32_t wv[4] = {vc.x, vc.y, vc.z, vc.w};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
              o[8 * c + 2 * wi] = (wv[wi] << 4) & 0xF0F0F0F0u;   // 16 q of k0 k2 k4 k6
              o[8 * c + 2 * wi + 1] = wv[wi] & 0xF0F0F0F0u;      // 16 q of k1 k3 k5 k7
            }
          }
          tmem_st16(a_col + 32 * half, o);
          tmem_st16(a_col + 32 * half + 16, o + 16);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t wv[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
          uint32_t o[16];
#pragma unroll
          for (int wi = 0; wi < 4; ++wi) {
            const uint32_t e = (wv[wi] & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t od = ((wv[wi] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t t0 = prmt(e, od, 0x5140u);   // k0 k1 k2 k3 (offset binary)
            const uint32_t t1 = prmt(e, od, 0x7362u);   // k4 k5 k6 k7
            // bf16 bit pattern 0x43uu is the value 128 + u
            o[4 * wi] = bf16x2_minus_136(prmt(t0, 0x43434343u, 0x4140u));
            o[4 * wi + 1] = bf16x2_minus_136(prmt(t0, 0x43434343u, 0x4342u));
            o[4 * wi + 2] = bf16x2_minus_136(prmt(t1, 0x43434343u, 0x4140u));
            o[4 * wi + 3] = bf16x2_minus_136(prmt(t1, 0x43434343u, 0x4342u));
          }
          tmem_st16(a_col + 16 * c, o);   // k = 32c .. 32c+31, two per column
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (elect_one_lane()) mbar_arrive(smem_u32(&a_full[sa]));
      __syncwarp();
    }
  } else if (warp >= kCtlWarps + C::kConvWarps) {
    // ------------------------------------------------ epilogue
    const int ew = warp - (kCtlWarps + C::kConvWarps);
    const int quad = warp & 3;                 // tensor-memory lanes this warp may read
    const int team = ew >> 2;                  // column team
    const int col0 = team * C::kCols;
    const int row = quad * 32 + lane;
    const int et = ew * 32 + lane;             // 0 .. kEpiThreads-1
    const int G = args.groups_per_row;
    grid_dependency_wait();   // no global write before the preceding grid is done
    if (et == 0) st_release_cta(&misc[7], 1u);   // ... and its tickets are settled
    bool epi_ok = true;
    if constexpr (kFused) {
      // Fused activation quantization: this CTA's epilogue warps together
      // quantize token rows blockIdx.x, blockIdx.x + grid, ... into the
      // workspace; each warp counts its share of a row as done (every lane's
      // stores fenced, then one release of the count), M * kEpiWarps in all.
      static_assert(C::kEpiWarps <= 4, "row partials for up to 4 epilogue warps");
      uint32_t rphase = 0;
      for (long long m = cta; epi_ok && m < args.M; m += grid, ++rphase) {
        if (et == 0) QSPEC_PHASE(11);
        epi_ok = quantize_row_team<C::kEpiWarps>(
            args.x + m * args.K, args.K, args.xq + m * args.K, const_cast<float*>(args.s_a) + m,
            args.qmax, ew, lane, s_row_part, smem_u32(row_amax), rphase, abort_flag, args.status);
        // every lane's code stores are ordered before lane 0's release by the
        // warp barrier (the release is cumulative over what lane 0 has seen)
        __syncwarp();
        if (epi_ok && lane == 0)
          asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(args.qsync) : "memory");
        if (et == 0) QSPEC_PHASE(12);
      }
      epi_ok = epi_ok && warp_wait(smem_u32(scale_ready), 0, abort_flag, args.status);
    }
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);

    // Group scales come as TMA tiles of 8 groups x 128 rows from the weight
    // producer, in the order it meets them: a new tile with this CTA's first
    // group and whenever a group index g of a tile reaches a multiple of 8.
    // Groups g >= k/group (a half unit at the end of k) read the stored zeros.
    RingPos rsc;              // next scale tile
    rsc.init(0, kNumSc);
    int sc_cur = -1;          // scale tile being read
    const uint32_t sc_row = smem_u32(sc_buf) + static_cast<uint32_t>(row * kScaleTileGroups * 2);

    float run[C::kCols];
    // y rows m0 .. m0+kCols-1 of output column n from run[]
    auto write_y = [&](int n, int m0) {
      if (n >= args.N) return;
      if constexpr (kInt8 && !kFused) grid_dependency_wait();   // s_a comes from the preceding kernel
#pragma unroll
      for (int c = 0; c < C::kCols; ++c) {
        const int m = m0 + c;
        if (m < args.M) {
          // int8 mode: run holds 16 x the sums; s_a / 16 is exact and so is
          // the product's rounding relative to the unscaled one
          const float sa = kFused ? s_tok_scale[m] : (kInt8 ? args.s_a[m] : 1.f);
          const float v = kInt8 ? (sa * 0.0625f) * run[c] : run[c];
          args.y[static_cast<long long>(m) * args.N + n] = v;
        }
      }
    };
    // As the last contributor of split tile t: add every share in K order
    // (the CTA owning the tile's first unit first) and write y.  Contributor
    // c_lo wrote its head slot if its range starts at the tile, else its tail
    // slot; every later contributor starts inside the tile.
    auto reduce_tile = [&](long long t) {
      const long long tile_u0 = t * ku;
      const long long c_lo = unit_owner(tile_u0, units, grid);
      const long long c_hi = unit_owner(tile_u0 + ku - 1, units, grid);
      const int lo_k = (unit_begin(c_lo, units, grid) == tile_u0) ? 0 : 1;
      const float* src = args.partials + (2 * c_lo + lo_k) * static_cast<long long>(MT * kTileN);
#pragma unroll
      for (int c = 0; c < C::kCols; ++c) run[c] = __ldcg(src + (col0 + c) * kTileN + row);
      for (long long cc = c_lo + 1; cc <= c_hi; ++cc) {
        src = args.partials + 2 * cc * static_cast<long long>(MT * kTileN);
#pragma unroll
        for (int c = 0; c < C::kCols; ++c) run[c] += __ldcg(src + (col0 + c) * kTileN + row);
      }
      const uint32_t n_tile = static_cast<uint32_t>(t) / static_cast<uint32_t>(args.m_tiles);
      const uint32_t m_tile = static_cast<uint32_t>(t) - n_tile * static_cast<uint32_t>(args.m_tiles);
      write_y(static_cast<int>(n_tile) * kTileN + row, static_cast<int>(m_tile) * MT + col0);
    };
    const long long t_head = static_cast<uint32_t>(u_begin) / static_cast<uint32_t>(ku);
    const long long head_end = (u_end < (t_head + 1) * ku) ? u_end : (t_head + 1) * ku;
    const bool head_handoff = (u_begin < u_end) && head_end < u_end && u_begin != t_head * ku;
    RingPos acc;              // accumulator ring position of the next group
    acc.init(0, NACC);
    bool ok = epi_ok;
    bool tail_slow = false;   // this warp left its tail-tile share for the ticket
    long long u = u_begin;
    UnitCursor tc;            // the tile of the next segment (no divisions per segment)
    tc.init(u_begin, ku, args.m_tiles);
    while (u < u_end && ok) {
      // one tile segment: units [seg_start, seg_end) of tile t
      const int n_tile = tc.n_tile, m_tile = tc.m_tile;
      const long long t = static_cast<long long>(n_tile) * args.m_tiles + m_tile;
      const long long tile_u0 = t * ku;
      const long long seg_start = u;
      const long long seg_end = (u_end < tile_u0 + ku) ? u_end : tile_u0 + ku;
      tc.kc = 0;
      if (++tc.m_tile == args.m_tiles) {
        tc.m_tile = 0;
        ++tc.n_tile;
      }
      const int n = n_tile * kTileN + row;
      const int m0 = m_tile * MT + col0;
#pragma unroll
      for (int c = 0; c < C::kCols; ++c) run[c] = 0.f;
      const bool full = (seg_start == tile_u0) && (seg_end == tile_u0 + ku);
      const bool fast_tail = tail_fast && seg_end >= u_end;
      const int seg_groups = static_cast<int>(seg_end - seg_start) * gpu;
      int g = static_cast<int>(seg_start - tile_u0) * gpu;   // the row's scale group
      for (int jj = 0; jj < seg_groups; ++jj, ++g) {
        if (sc_cur < 0 || (g & (kScaleTileGroups - 1)) == 0) {
          if (sc_cur >= 0) {   // done with the previous tile
            __syncwarp();
            if (elect_one_lane()) mbar_arrive(smem_u32(&sc_empty[sc_cur]));
            __syncwarp();
          }
          ok = warp_wait(smem_u32(&sc_full[rsc.slot]), rsc.phase, abort_flag, args.status);
          if (!ok) break;
          sc_cur = rsc.slot;
          rsc.step(1, kNumSc);
        }
        uint16_t hbits;
        asm volatile("ld.shared.u16 %0, [%1];"
                     : "=h"(hbits)
                     : "r"(sc_row + static_cast<uint32_t>(sc_cur * kScaleTileBytes +
                                                          (g & (kScaleTileGroups - 1)) * 2)));
        const float sc = __half2float(__ushort_as_half(hbits));
        ok = warp_wait(smem_u32(&acc_full[acc.slot]), acc.phase, abort_flag, args.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr =
            lane_addr + static_cast<uint32_t>(C::kAccCol0 + acc.slot * MT + col0);
#pragma unroll
        for (int c0 = 0; c0 < C::kCols; c0 += 16) {
          uint32_t v[16];
          tmem_ld8(taddr + c0, v);
          if (c0 + 8 < C::kCols) tmem_ld8(taddr + c0 + 8, v + 8);
          tmem_ld_wait();
          if (c0 + 16 >= C::kCols) {
            // all columns of this group are in registers: hand the buffer back
            tc_fence_before();
            __syncwarp();
            if (elect_one_lane()) mbar_arrive(smem_u32(&acc_empty[acc.slot]));
            __syncwarp();
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            if (c0 + e < C::kCols) {
              const float a = kInt8 ? static_cast<float>(static_cast<int>(v[e])) : __uint_as_float(v[e]);
              run[c0 + e] = fmaf(sc, a, run[c0 + e]);
            }
          }
          if constexpr (kInt8 && kDbg) {
            if (n < args.N && g < G) {
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int m = m0 + c0 + e;
                if (c0 + e < C::kCols && m < args.M)
                  args.dbg_acc[(static_cast<long long>(m) * args.N + n) * G + g] =
                      static_cast<int>(v[e]) >> 4;   // exact: a multiple of 16
              }
            }
          }
        }
        acc.step(1, NACC);
      }
      if (!ok) break;
      u = seg_end;
      if (et == 0) QSPEC_PHASE(u >= u_end ? 5 : 7);

      if (full) {
        write_y(n, m0);
      } else {
        // A split tile.  Fast tail: the other contributor has published, so
        // this warp adds its share (same order as the reduction: this CTA's
        // share first) and writes y.  Otherwise the share goes to the
        // workspace and the weight producer takes the ticket (the head tile
        // right away, the tail tile once every warp is done with it).
        const bool last_seg = seg_end >= u_end;
        bool fast = false;
        if (fast_tail) {
          fast = __all_sync(0xffffffffu, mbar_test_wait(smem_u32(tail_bar), 0));
          if (fast) {
            // the next CTA's share sits in its head slot
            const float* src = args.partials + static_cast<long long>(2 * (cta + 1)) * MT * kTileN;
#pragma unroll
            for (int c = 0; c < C::kCols; ++c) run[c] += __ldcg(src + (col0 + c) * kTileN + row);
            write_y(n, m0);
          }
        }
        if (!fast) {
          const int k = (seg_start == u_begin) ? 0 : 1;
          float* mine = args.partials + static_cast<long long>(2 * cta + k) * MT * kTileN;
#pragma unroll
          for (int c = 0; c < C::kCols; ++c) mine[(col0 + c) * kTileN + row] = run[c];
        }
        __syncwarp();
        if (elect_one_lane()) {
          if (last_seg && !fast) misc[5] = 1u;
          mbar_arrive(smem_u32(&flush_bar[last_seg ? 1 : 0]));
        }
        __syncwarp();
        tail_slow = last_seg && !fast;
      }
    }
    // The split tiles whose last ticket came to this CTA are added up here,
    // after the CTA's own tiles.
    if (ok && head_handoff) {
      ok = warp_wait(smem_u32(&ticket_bar[0]), 0, abort_flag, args.status);
      if (ok && misc[3] != 0u) reduce_tile(t_head);
    }
    if (ok && tail_slow) {
      ok = warp_wait(smem_u32(&ticket_bar[1]), 0, abort_flag, args.status);
      if (ok && misc[6] != 0u) reduce_tile(t_tail);
    }
  }

  QSPEC_TRACE_AT(0xFFF0);
  if ((threadIdx.x & 31) == 0 && warp == kCtlWarps + C::kConvWarps)
    QSPEC_PHASE(6);
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) QSPEC_PHASE(8);
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace qspec
