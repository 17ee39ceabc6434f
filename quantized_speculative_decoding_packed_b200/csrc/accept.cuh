// Batched speculative accept / residual resample (SpecQuant review,
// paragraph 5: verification by "the usual Leviathan rule"; the rule itself is
// the one of "Fast Inference from Transformers via Speculative Decoding" and
// "Accelerating Large Language Model Decoding with Speculative Sampling").
//
// Per sequence b:
//   n = first i < gamma with NOT (u_acc[b][i] * q[b][i][x_i] < p[b][i][x_i]), else gamma
//   r = max(0, p[b][n] - q[b][n])  if n < gamma,  else p[b][gamma]
//   F_j = floor(r_j * 2^62), C_j = sum_{i<=j} F_i, S = C_{V-1}, T = floor(u_res[b] * S)
//   token = min{ j : C_j > T };  if S == 0 the draw repeats on r = p[b][n].
// The ratio test is evaluated exactly (fp32 x fp32 products are exact in
// fp64) and the draw in 64-bit integers, so the result does not depend on
// the order in which the vocabulary is summed.
//
// Layout on B200: one cluster of kAcceptCluster CTAs per sequence.  Each CTA
// streams one contiguous chunk of the row(s) from HBM once, keeps r in shared
// memory, and publishes its chunk total; the CTAs read each other's totals
// through distributed shared memory, and the CTA whose chunk holds the
// threshold finds the token with a block scan over its shared-memory copy.
#pragma once

#include <cooperative_groups.h>
#include <cstdint>

#include "device_common.cuh"

namespace qspec {

// 8 CTAs per sequence (16, a non-portable size, measured 1.7x slower at vocab
// 128256, batch 64).
constexpr int kAcceptCluster = 8;
// Vocabulary iterations whose loads a thread keeps in flight together.
constexpr int kAcceptUnroll = 8;
constexpr int kAcceptThreads = 256;

__device__ __forceinline__ uint64_t fixed_point_weight(float r) {
  // r * 2^62 is exact in fp64; truncation toward zero is floor for r >= 0.
  return (r > 0.f) ? __double2ull_rz(static_cast<double>(r) * 4611686018427387904.0) : 0ull;
}

// floor(u * s) for an fp32 u in [0, 1), computed exactly with a 128-bit product.
__device__ __forceinline__ uint64_t fixed_point_threshold(float u, uint64_t s) {
  const uint32_t bits = __float_as_uint(u);
  const uint32_t e = (bits >> 23) & 0xFFu;
  uint64_t mant = bits & 0x7FFFFFu;
  int shift;
  if (e == 0) {
    shift = 149;                       // subnormal: mant * 2^-149
  } else {
    mant |= 0x800000u;
    shift = 150 - static_cast<int>(e);  // mant * 2^(e - 150)
  }
  if (mant == 0 || shift >= 128) return 0;
  const uint64_t lo = mant * s;
  const uint64_t hi = __umul64hi(mant, s);
  if (shift >= 64) return hi >> (shift - 64);
  if (shift <= 0) return ~0ull;        // u >= 1: caller clamps
  return (lo >> shift) | (hi << (64 - shift));
}

__device__ __forceinline__ uint64_t block_sum_u64(uint64_t v, uint64_t* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  uint64_t t = 0;
#pragma unroll
  for (int i = 0; i < kAcceptThreads / 32; ++i) t += red[i];
  __syncthreads();
  return t;
}

struct AcceptShared {
  uint64_t chunk_sum[2];                    // per pass; read by the other CTAs of the cluster
  uint64_t red[kAcceptThreads / 32];
  int n_acc;
  int token;
};

__global__ void __cluster_dims__(kAcceptCluster, 1, 1) __launch_bounds__(kAcceptThreads)
    spec_accept_kernel(const float* __restrict__ p, const float* __restrict__ q,
                       const int32_t* __restrict__ draft, const float* __restrict__ u_acc,
                       const float* __restrict__ u_res, int gamma, int vocab, int chunk,
                       int32_t* __restrict__ n_accepted, int32_t* __restrict__ tokens,
                       uint32_t* __restrict__ status) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) float r_s[];
  __shared__ AcceptShared sh;

  const int b = blockIdx.x / kAcceptCluster;
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;

  // Phase 1: ratio test at every draft position at once (lane i of the first
  // warp takes position i: one round of scattered reads instead of gamma
  // dependent ones); n = the first failing position, found by a ballot.
  if (tid < 32) {
    bool fail = false;
    bool bad = false;
    if (tid < gamma) {
      const int x = draft[b * gamma + tid];
      if (x < 0 || x >= vocab) {
        fail = bad = true;
      } else {
        const double pv = p[(static_cast<int64_t>(b) * (gamma + 1) + tid) * vocab + x];
        const double qv = q[(static_cast<int64_t>(b) * gamma + tid) * vocab + x];
        fail = !(static_cast<double>(u_acc[b * gamma + tid]) * qv < pv);
      }
    }
    const uint32_t fails = __ballot_sync(0xffffffffu, fail);
    const int n_first = fails ? (__ffs(fails) - 1) : gamma;
    // only an invalid draft the rule actually reached counts as bad input
    if (bad && tid == n_first && status && crank == 0) atomicOr(status, kDevBadInput);
    if (tid == 0) {
      sh.n_acc = n_first;
      sh.token = -1;
    }
  }
  __syncthreads();
  const int n = sh.n_acc;
  const int lo = crank * chunk;
  const int hi = min(vocab, lo + chunk);
  const int len = max(0, hi - lo);

  const float* prow;
  const float* qrow;
  if (n < gamma) {
    prow = p + (static_cast<int64_t>(b) * (gamma + 1) + n) * vocab;
    qrow = q + (static_cast<int64_t>(b) * gamma + n) * vocab;
  } else {
    prow = p + (static_cast<int64_t>(b) * (gamma + 1) + gamma) * vocab;
    qrow = nullptr;
  }

  uint64_t total = 0, prefix = 0;
  for (int pass = 0; pass < 2; ++pass) {
    // Stream this CTA's chunk once: r into shared memory, F summed on the
    // fly; each thread keeps kAcceptUnroll iterations' loads in flight.
    uint64_t part = 0;
    for (int j0 = tid * 4; j0 < len; j0 += kAcceptThreads * 4 * kAcceptUnroll) {
      float4 pv[kAcceptUnroll], qv[kAcceptUnroll];
#pragma unroll
      for (int t = 0; t < kAcceptUnroll; ++t) {
        const int j = j0 + t * kAcceptThreads * 4;
        if (j < len) {
          pv[t] = __ldcs(reinterpret_cast<const float4*>(prow + lo + j));
          if (qrow) qv[t] = __ldcs(reinterpret_cast<const float4*>(qrow + lo + j));
        }
      }
#pragma unroll
      for (int t = 0; t < kAcceptUnroll; ++t) {
        const int j = j0 + t * kAcceptThreads * 4;
        if (j < len) {
          float4 v = pv[t];
          if (qrow) {
            v.x = fmaxf(0.f, __fsub_rn(v.x, qv[t].x));
            v.y = fmaxf(0.f, __fsub_rn(v.y, qv[t].y));
            v.z = fmaxf(0.f, __fsub_rn(v.z, qv[t].z));
            v.w = fmaxf(0.f, __fsub_rn(v.w, qv[t].w));
          }
          *reinterpret_cast<float4*>(r_s + j) = v;
          part += fixed_point_weight(v.x) + fixed_point_weight(v.y) + fixed_point_weight(v.z) +
                  fixed_point_weight(v.w);
        }
      }
    }
    const uint64_t mine = block_sum_u64(part, sh.red);
    if (tid == 0) sh.chunk_sum[pass] = mine;
    cluster.sync();
    total = 0;
    prefix = 0;
    for (int c = 0; c < kAcceptCluster; ++c) {
      const uint64_t* remote = cluster.map_shared_rank(&sh.chunk_sum[pass], c);
      const uint64_t v = *remote;
      if (c < crank) prefix += v;
      total += v;
    }
    if (total != 0 || pass == 1) break;
    // Empty residual (possible only through fp32 rounding): draw from p[b][n].
    prow = p + (static_cast<int64_t>(b) * (gamma + 1) + n) * vocab;
    qrow = nullptr;
    __syncthreads();
  }

  // The CTA whose chunk holds the threshold finds the token: per-thread
  // contiguous sub-ranges of the shared-memory copy, an exclusive scan of
  // their sums, then a sequential search inside the one sub-range that
  // straddles the threshold.
  __syncthreads();
  if (total != 0) {
    const int per = (len + kAcceptThreads - 1) / kAcceptThreads;
    const int a0 = min(len, tid * per);
    const int a1 = min(len, a0 + per);
    uint64_t s = 0;
    for (int j = a0; j < a1; ++j) s += fixed_point_weight(r_s[j]);
    // Exclusive scan of the per-thread sums: inclusive scans inside each warp
    // by shuffles, then the warp totals (exact integer sums, any order).
    const int lane = tid & 31, wid = tid >> 5;
    uint64_t incl = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint64_t o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) sh.red[wid] = incl;
    __syncthreads();
    uint64_t warp_base = 0;
#pragma unroll
    for (int w = 0; w < kAcceptThreads / 32; ++w)
      if (w < wid) warp_base += sh.red[w];
    uint64_t t = fixed_point_threshold(u_res[b], total);
    if (t >= total) t = total - 1;
    const uint64_t base = prefix + warp_base + (incl - s);
    if (s != 0 && base <= t && t < base + s) {
      uint64_t c = base;
      for (int j = a0; j < a1; ++j) {
        c += fixed_point_weight(r_s[j]);
        if (c > t) {
          sh.token = lo + j;
          break;
        }
      }
    }
    __syncthreads();
    if (tid == 0 && sh.token >= 0) tokens[static_cast<int64_t>(b) * (gamma + 1) + n] = sh.token;
  }

  if (crank == 0) {
    for (int i = tid; i <= gamma; i += kAcceptThreads) {
      if (i < n) tokens[static_cast<int64_t>(b) * (gamma + 1) + i] = draft[b * gamma + i];
      if (i > n || (i == n && total == 0)) tokens[static_cast<int64_t>(b) * (gamma + 1) + i] = -1;
    }
    if (tid == 0) n_accepted[b] = n;
  }
  // Keep this CTA's shared memory alive until every CTA of the cluster has read it.
  cluster.sync();
}

// ---------------------------------------------------------------------------
// Greedy verification (SpecQuant review, paragraph 5: a draft that matches in
// full is kept; at the first mismatch the target model's own choice replaces
// the draft token).  The target's choice at position i is t_i = argmax_j
// p[b][i][j], ties to the lowest index; n = first i < gamma with
// draft[b][i] != t_i (gamma if none); the new token is t_n.
//
// One cluster of kAcceptCluster CTAs per sequence walks the rows in order and
// stops at the first mismatch, so only rows 0..n are read from HBM.  Each CTA
// reduces its chunk of a row to (largest value, lowest index holding it),
// publishes the pair in distributed shared memory, and after one cluster
// barrier every CTA combines the same eight pairs into the same t_i, so the
// whole cluster takes the same branch without further communication.
struct ArgMax {
  float v;
  int i;
};

// The better of two candidates: larger value, or equal value and lower index.
__device__ __forceinline__ ArgMax argmax_pick(ArgMax a, ArgMax b) {
  return (b.v > a.v || (b.v == a.v && b.i < a.i)) ? b : a;
}

struct GreedyShared {
  ArgMax part[2];                      // this CTA's pair for the current row (by parity)
  ArgMax red[kAcceptThreads / 32];
};

__global__ void __cluster_dims__(kAcceptCluster, 1, 1) __launch_bounds__(kAcceptThreads)
    greedy_accept_kernel(const float* __restrict__ p, const int32_t* __restrict__ draft, int gamma,
                         int vocab, int chunk, int32_t* __restrict__ n_accepted,
                         int32_t* __restrict__ tokens, uint32_t* __restrict__ status) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ GreedyShared sh;
  const int b = blockIdx.x / kAcceptCluster;
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int lo = crank * chunk;
  const int len = max(0, min(vocab, lo + chunk) - lo);

  int n = gamma;
  int token = -1;
  bool bad = false;
  for (int i = 0; i <= gamma; ++i) {
    const float* row = p + (static_cast<int64_t>(b) * (gamma + 1) + i) * vocab + lo;
    // thread-local scan: increasing indices, strict '>' keeps the first
    // maximum; kAcceptUnroll iterations' loads in flight together
    ArgMax best{-__int_as_float(0x7f800000), 0x7fffffff};
    for (int j0 = tid * 4; j0 < len; j0 += kAcceptThreads * 4 * kAcceptUnroll) {
      float4 vv[kAcceptUnroll];
#pragma unroll
      for (int t = 0; t < kAcceptUnroll; ++t) {
        const int j = j0 + t * kAcceptThreads * 4;
        if (j < len) vv[t] = __ldcs(reinterpret_cast<const float4*>(row + j));
      }
#pragma unroll
      for (int t = 0; t < kAcceptUnroll; ++t) {
        const int j = j0 + t * kAcceptThreads * 4;
        if (j < len) {
          const float4 v = vv[t];
          if (v.x > best.v) best = ArgMax{v.x, lo + j};
          if (v.y > best.v) best = ArgMax{v.y, lo + j + 1};
          if (v.z > best.v) best = ArgMax{v.z, lo + j + 2};
          if (v.w > best.v) best = ArgMax{v.w, lo + j + 3};
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      ArgMax o;
      o.v = __shfl_xor_sync(0xffffffffu, best.v, off);
      o.i = __shfl_xor_sync(0xffffffffu, best.i, off);
      best = argmax_pick(best, o);
    }
    if ((tid & 31) == 0) sh.red[tid >> 5] = best;
    __syncthreads();
    if (tid == 0) {
      ArgMax c = sh.red[0];
#pragma unroll
      for (int w = 1; w < kAcceptThreads / 32; ++w) c = argmax_pick(c, sh.red[w]);
      sh.part[i & 1] = c;
    }
    cluster.sync();
    ArgMax t{-__int_as_float(0x7f800000), 0x7fffffff};
    for (int c = 0; c < kAcceptCluster; ++c)
      t = argmax_pick(t, *cluster.map_shared_rank(&sh.part[i & 1], c));
    if (i == gamma) {
      token = t.i;
      break;
    }
    const int x = draft[b * gamma + i];
    if (x < 0 || x >= vocab) bad = true;
    if (x != t.i) {
      n = i;
      token = t.i;
      break;
    }
  }
  if (crank == 0) {
    if (bad && status && tid == 0) atomicOr(status, kDevBadInput);
    for (int i = tid; i <= gamma; i += kAcceptThreads)
      tokens[static_cast<int64_t>(b) * (gamma + 1) + i] =
          (i < n) ? draft[b * gamma + i] : (i == n ? token : -1);
    if (tid == 0) n_accepted[b] = n;
  }
  // Keep this CTA's shared memory alive until every CTA of the cluster has read it.
  cluster.sync();
}

}  // namespace qspec
