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

constexpr int kAcceptCluster = 8;
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
  uint64_t scan[kAcceptThreads];
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

  // Phase 1: ratio test along the draft (a few scattered reads).
  if (tid == 0) {
    int n = gamma;
    for (int i = 0; i < gamma; ++i) {
      const int x = draft[b * gamma + i];
      if (x < 0 || x >= vocab) {
        if (status && crank == 0) atomicOr(status, kDevBadInput);
        n = i;
        break;
      }
      const double pv = p[(static_cast<int64_t>(b) * (gamma + 1) + i) * vocab + x];
      const double qv = q[(static_cast<int64_t>(b) * gamma + i) * vocab + x];
      if (!(static_cast<double>(u_acc[b * gamma + i]) * qv < pv)) {
        n = i;
        break;
      }
    }
    sh.n_acc = n;
    sh.token = -1;
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
    // Stream this CTA's chunk once: r into shared memory, F summed on the fly.
    uint64_t part = 0;
    for (int j = tid * 4; j < len; j += kAcceptThreads * 4) {
      float4 pv = *reinterpret_cast<const float4*>(prow + lo + j);
      if (qrow) {
        const float4 qv = *reinterpret_cast<const float4*>(qrow + lo + j);
        pv.x = fmaxf(0.f, __fsub_rn(pv.x, qv.x));
        pv.y = fmaxf(0.f, __fsub_rn(pv.y, qv.y));
        pv.z = fmaxf(0.f, __fsub_rn(pv.z, qv.z));
        pv.w = fmaxf(0.f, __fsub_rn(pv.w, qv.w));
      }
      *reinterpret_cast<float4*>(r_s + j) = pv;
      part += fixed_point_weight(pv.x) + fixed_point_weight(pv.y) + fixed_point_weight(pv.z) +
              fixed_point_weight(pv.w);
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
    sh.scan[tid] = s;
    __syncthreads();
    // Exclusive scan of the per-thread sums (256 entries, simple and exact).
    if (tid == 0) {
      uint64_t run = 0;
      for (int i = 0; i < kAcceptThreads; ++i) {
        const uint64_t v = sh.scan[i];
        sh.scan[i] = run;
        run += v;
      }
    }
    __syncthreads();
    uint64_t t = fixed_point_threshold(u_res[b], total);
    if (t >= total) t = total - 1;
    const uint64_t base = prefix + sh.scan[tid];
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

}  // namespace qspec
