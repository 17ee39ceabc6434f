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
// streams one contiguous chunk of the row(s) from HBM once (each warp a
// contiguous sub-chunk, coalesced), records the F sums of its blocks of 128 x
// k floats in shared memory and publishes its chunk total; the CTAs read each
// other's totals through distributed shared memory, and the CTA whose chunk
// holds the threshold locates it among its recorded sums and re-reads only
// that block (an L2 hit) to find the token.  Without a copy of the chunk in
// shared memory a batch of 64 sequences (512 CTAs) is resident in one wave.
#pragma once

#include <cooperative_groups.h>
#include <cstdint>

#include "device_common.cuh"

namespace qspec {

// 8 CTAs per sequence (16, a non-portable size, measured 1.7x slower at vocab
// 128256, batch 64).
constexpr int kAcceptCluster = 8;
// Vocabulary iterations whose loads a thread keeps in flight together (the
// sampler keeps fewer: it runs four CTAs per SM, so within 64 registers).
constexpr int kAcceptUnroll = 8;
constexpr int kSampleUnroll = 4;
constexpr int kAcceptThreads = 256;

__device__ __forceinline__ uint64_t fixed_point_weight(float r) {
  // r * 2^62 only moves the exponent (exact in fp32 for 0 <= r < 4); the
  // conversion truncates toward zero, which is floor for r >= 0.
  return (r > 0.f) ? __float2ull_rz(__fmul_rn(r, 4611686018427387904.0f)) : 0ull;
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

// Block sums recorded per warp: a warp's sub-chunk is read as iterations of
// 128 floats (one float4 per lane), and every AcceptSplit::per_blk
// consecutive iterations (kSampleUnroll up to a vocabulary of 8 x 8 x 64 x 128
// x kSampleUnroll) form one recorded block.
constexpr int kAcceptWarps = kAcceptThreads / 32;
constexpr int kAcceptMaxBlocks = 64;

struct AcceptShared {
  uint64_t chunk_sum[2];                    // per pass; read by the other CTAs of the cluster
  uint64_t red[kAcceptWarps];               // this CTA's warp totals
  uint64_t blk[kAcceptWarps][kAcceptMaxBlocks];
  int n_acc;
  int token;
};

__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__device__ __forceinline__ uint64_t warp_incl_scan_u64(uint64_t v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint64_t o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

// Split of a CTA's chunk of `len` floats (a multiple of 4) among its warps:
// warp w owns [w * wlen, min(len, (w + 1) * wlen)), read in `its` iterations
// of 128 floats, recorded in blocks of `per_blk` iterations.
struct AcceptSplit {
  int wlen, its, per_blk;
  __device__ __forceinline__ void init(int len) {
    wlen = ((len + 4 * kAcceptWarps - 1) / (4 * kAcceptWarps)) * 4;
    its = (wlen + 127) / 128;
    // at least kSampleUnroll iterations per block: one warp reduction per
    // batch of loads
    per_blk = (its + kAcceptMaxBlocks - 1) / kAcceptMaxBlocks;
    if (per_blk < kSampleUnroll) per_blk = kSampleUnroll;
  }
};

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__global__ void __cluster_dims__(kAcceptCluster, 1, 1) __launch_bounds__(kAcceptThreads, 4)
    spec_accept_kernel(const float* __restrict__ p, const float* __restrict__ q,
                       const int32_t* __restrict__ draft, const float* __restrict__ u_acc,
                       const float* __restrict__ u_res, int gamma, int vocab, int chunk,
                       int32_t* __restrict__ n_accepted, int32_t* __restrict__ tokens,
                       uint32_t* __restrict__ status) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ AcceptShared sh;

  const int b = blockIdx.x / kAcceptCluster;
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;

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
  AcceptSplit sp;
  sp.init(len);
  const int w0 = min(len, wid * sp.wlen);
  const int w1 = min(len, w0 + sp.wlen);

  const float* prow;
  const float* qrow;
  if (n < gamma) {
    prow = p + (static_cast<int64_t>(b) * (gamma + 1) + n) * vocab;
    qrow = q + (static_cast<int64_t>(b) * gamma + n) * vocab;
  } else {
    prow = p + (static_cast<int64_t>(b) * (gamma + 1) + gamma) * vocab;
    qrow = nullptr;
  }
  // r at chunk offset j (a multiple of 4), four at a time
  auto r4 = [&](int j) {
    float4 v = __ldcg(reinterpret_cast<const float4*>(prow + lo + j));
    if (qrow) {
      const float4 w = __ldcg(reinterpret_cast<const float4*>(qrow + lo + j));
      v.x = fmaxf(0.f, __fsub_rn(v.x, w.x));
      v.y = fmaxf(0.f, __fsub_rn(v.y, w.y));
      v.z = fmaxf(0.f, __fsub_rn(v.z, w.z));
      v.w = fmaxf(0.f, __fsub_rn(v.w, w.w));
    }
    return v;
  };

  uint64_t total = 0, prefix = 0, mine = 0;
  for (int pass = 0; pass < 2; ++pass) {
    // Stream this CTA's chunk once, each warp its own sub-chunk, coalesced
    // (lane l reads floats 4l..4l+3 of each 128), kSampleUnroll iterations'
    // loads in flight; record the warp's F sum per block of iterations.
    uint64_t wsum = 0, lsum = 0;
    for (int k0 = 0; k0 < sp.its; k0 += kSampleUnroll) {
      float4 pv[kSampleUnroll], qv[kSampleUnroll];
#pragma unroll
      for (int t = 0; t < kSampleUnroll; ++t) {
        const int j = w0 + (k0 + t) * 128 + lane * 4;
        if (k0 + t < sp.its && j < w1) {
          pv[t] = __ldcs(reinterpret_cast<const float4*>(prow + lo + j));
          if (qrow) qv[t] = __ldcs(reinterpret_cast<const float4*>(qrow + lo + j));
        }
      }
#pragma unroll
      for (int t = 0; t < kSampleUnroll; ++t) {
        const int it = k0 + t;
        if (it < sp.its) {   // warp-uniform
          const int j = w0 + it * 128 + lane * 4;
          uint64_t f = 0;
          if (j < w1) {
            float4 v = pv[t];
            if (qrow) {
              v.x = fmaxf(0.f, __fsub_rn(v.x, qv[t].x));
              v.y = fmaxf(0.f, __fsub_rn(v.y, qv[t].y));
              v.z = fmaxf(0.f, __fsub_rn(v.z, qv[t].z));
              v.w = fmaxf(0.f, __fsub_rn(v.w, qv[t].w));
            }
            f = fixed_point_weight(v.x) + fixed_point_weight(v.y) + fixed_point_weight(v.z) +
                fixed_point_weight(v.w);
          }
          lsum += f;
          if ((it + 1) % sp.per_blk == 0 || it + 1 == sp.its) {
            const uint64_t bsum = warp_sum_u64(lsum);
            if (lane == 0) sh.blk[wid][it / sp.per_blk] = bsum;
            wsum += bsum;
            lsum = 0;
          }
        }
      }
    }
    if (lane == 0) sh.red[wid] = wsum;
    __syncthreads();
    mine = 0;
#pragma unroll
    for (int w = 0; w < kAcceptWarps; ++w) mine += sh.red[w];
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
  }
  // Done with the other CTAs' shared memory (they wait for this arrival
  // before exiting, so theirs stays readable until here).
  cluster_arrive_release();

  // The CTA whose chunk holds the threshold T draws the token: its first warp
  // finds the warp sub-chunk and the recorded block holding T, then re-reads
  // that one block (from L2) and finds the lane and the element.
  if (total != 0 && wid == 0) {
    uint64_t t = fixed_point_threshold(u_res[b], total);
    if (t >= total) t = total - 1;
    if (prefix <= t && t < prefix + mine) {
      // warp sub-chunk: lanes 0..7 hold the warp totals
      uint64_t v = (lane < kAcceptWarps) ? sh.red[lane] : 0;
      uint64_t incl = warp_incl_scan_u64(v, lane);
      uint32_t hit = __ballot_sync(0xffffffffu, lane < kAcceptWarps && prefix + incl > t);
      const int ws = hit ? __ffs(hit) - 1 : 0;   // T < prefix + mine: always a hit
      uint64_t base = prefix + __shfl_sync(0xffffffffu, incl - v, ws);
      // recorded block inside that sub-chunk
      const int sw0 = min(len, ws * sp.wlen), sw1 = min(len, sw0 + sp.wlen);
      const int nblk = (sp.its + sp.per_blk - 1) / sp.per_blk;
      int blk = -1;
      for (int b0 = 0; b0 < nblk && blk < 0; b0 += 32) {
        v = (b0 + lane < nblk) ? sh.blk[ws][b0 + lane] : 0;
        incl = warp_incl_scan_u64(v, lane);
        hit = __ballot_sync(0xffffffffu, b0 + lane < nblk && base + incl > t);
        if (hit) {
          const int l = __ffs(hit) - 1;
          blk = b0 + l;
          base += __shfl_sync(0xffffffffu, incl - v, l);
        } else {
          base += __shfl_sync(0xffffffffu, incl, 31);
        }
      }
      // re-read the block's iterations (loads of kSampleUnroll of them in
      // flight) and walk them in order
      const int it1 = min(sp.its, (blk + 1) * sp.per_blk);
      bool done = blk < 0;
      for (int i0 = blk * sp.per_blk; !done && i0 < it1; i0 += kSampleUnroll) {
        float4 rv[kSampleUnroll];
#pragma unroll
        for (int u = 0; u < kSampleUnroll; ++u) {
          const int j = sw0 + (i0 + u) * 128 + lane * 4;
          rv[u] = (i0 + u < it1 && j < sw1) ? r4(j) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kSampleUnroll; ++u) {
          if (done || i0 + u >= it1) break;   // warp-uniform
          const float e[4] = {rv[u].x, rv[u].y, rv[u].z, rv[u].w};
          const uint64_t s = fixed_point_weight(e[0]) + fixed_point_weight(e[1]) +
                             fixed_point_weight(e[2]) + fixed_point_weight(e[3]);
          incl = warp_incl_scan_u64(s, lane);
          hit = __ballot_sync(0xffffffffu, base + incl > t);
          if (hit) {
            if (lane == __ffs(hit) - 1) {
              const int j = sw0 + (i0 + u) * 128 + lane * 4;
              uint64_t c = base + incl - s;
#pragma unroll
              for (int e4 = 0; e4 < 4; ++e4) {
                c += fixed_point_weight(e[e4]);
                if (c > t) {
                  tokens[static_cast<int64_t>(b) * (gamma + 1) + n] = lo + j + e4;
                  break;
                }
              }
            }
            done = true;
          } else {
            base += __shfl_sync(0xffffffffu, incl, 31);
          }
        }
      }
    }
  }

  if (crank == 0) {
    for (int i = tid; i <= gamma; i += kAcceptThreads) {
      if (i < n) tokens[static_cast<int64_t>(b) * (gamma + 1) + i] = draft[b * gamma + i];
      if (i > n || (i == n && total == 0)) tokens[static_cast<int64_t>(b) * (gamma + 1) + i] = -1;
    }
    if (tid == 0) n_accepted[b] = n;
  }
  cluster_wait_acquire();
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
