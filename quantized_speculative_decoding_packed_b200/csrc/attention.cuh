// The KV cache shared by the drafting and the verifying stage (QSpec
// abstract: both stages reuse the KV cache as well as the weights), with the
// decode attention that reads it.
//
// Cache: per layer, K and V each [B][H_kv][L_max][128] bf16.  A pass over T
// new tokens per sequence (drafting pass j: T = 1 at offset j; verifying
// pass: T = gamma + 1 at offset 0, overwriting the drafted entries) appends
// the tokens' keys and values at positions lens[b] + offset + t, taken from
// the fused QKV projection (row b*T + t: H query heads, then H_kv key heads,
// then H_kv value heads, 128 columns each), rounded to bf16.  Token (b, t)
// then attends to positions 0 .. lens[b] + offset + t with the scaled
// dot-product softmax, query head h reading KV head h / (H / H_kv).  After
// the accept step lens[b] grows by n_accepted[b] + 1; the entries past it
// (rejected drafts) are overwritten by the next round.
//
// Layout on B200 (decode attention is HBM-bound: every key and value is
// read once per pass): one CTA per (sequence, KV head, chunk of 128 keys),
// so the cache streams through all SMs whatever the batch.  A CTA copies its
// chunk's keys and values (32 KB each, contiguous) into shared memory with
// two TMA bulk copies; each lane then owns one key for the scores, the
// softmax of the chunk is exact (its own maximum), and for the values each
// lane owns one column of the head.  Each CTA leaves its (max, sum, weighted
// values) per query row in the workspace; the last CTA of a (sequence, KV
// head) to arrive merges the chunks in chunk order, so the result does not
// depend on which CTA finishes last.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "device_common.cuh"

namespace qspec {

constexpr int kHeadDim = 128;
constexpr int kAttnChunk = 128;              // keys per CTA
constexpr int kAttnThreads = 128;            // 4 warps
constexpr int kAttnMaxRows = 32;             // (query heads per KV head) x new tokens
constexpr int kAttnRowBlock = 8;             // query rows per register block
constexpr int kAttnMaxChunks = 256;          // context up to 32768 keys
constexpr float kInvSqrtHeadDim = 0.08838834764831845f;   // 1 / sqrt(128)

// Workspace of the attention call: status word, then one arrival counter per
// (sequence, KV head), then per chunk and query row the partial results.
struct AttnLayout {
  int64_t off_counters, off_ml, off_o, total;
};

__host__ __device__ inline AttnLayout attn_layout(int64_t batch, int64_t h_kv, int64_t chunks,
                                                  int64_t rows) {
  AttnLayout l;
  auto up = [](int64_t v) { return (v + 255) / 256 * 256; };
  l.off_counters = 256;
  l.off_ml = up(l.off_counters + batch * h_kv * 4);
  l.off_o = up(l.off_ml + batch * h_kv * chunks * rows * 2 * 4);
  l.total = up(l.off_o + batch * h_kv * chunks * rows * kHeadDim * 4);
  return l;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
}

// One CTA per new token (b, t): its H_kv key heads and H_kv value heads,
// rounded to bf16, into the caches at position lens[b] + offset + t.  A
// position outside [0, l_max) writes nothing and sets the bad-input status.
__global__ void __launch_bounds__(256) kv_append_kernel(
    const float* __restrict__ qkv, int64_t ld, int t_new, int h_q, int h_kv,
    const int32_t* __restrict__ lens, int offset, uint16_t* __restrict__ k_cache,
    uint16_t* __restrict__ v_cache, int l_max, uint32_t* __restrict__ status) {
  const int b = blockIdx.x / t_new;
  const int t = blockIdx.x % t_new;
  const int64_t pos = static_cast<int64_t>(lens[b]) + offset + t;
  if (lens[b] < 0 || pos < 0 || pos >= l_max) {
    if (threadIdx.x == 0 && status) atomicOr(status, kDevBadInput);
    return;
  }
  const float* row = qkv + (static_cast<int64_t>(b) * t_new + t) * ld + static_cast<int64_t>(h_q) * kHeadDim;
  const int per_half = h_kv * kHeadDim;                // elements of the K (or V) part
  for (int e = threadIdx.x * 4; e < 2 * per_half; e += blockDim.x * 4) {
    const int which = e >= per_half;                   // 0: key, 1: value
    const int ei = e - which * per_half;
    const int g = ei / kHeadDim;
    const int i = ei % kHeadDim;
    const float4 v = *reinterpret_cast<const float4*>(row + e);
    uint16_t* cache = which ? v_cache : k_cache;
    const int64_t dst = ((static_cast<int64_t>(b) * h_kv + g) * l_max + pos) * kHeadDim + i;
    *reinterpret_cast<uint2*>(cache + dst) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

// lens[b] += n_accepted[b] + 1 (one thread per sequence); a count outside
// [0, l_max - lens[b] - 1] leaves lens[b] unchanged and sets the bad-input status.
__global__ void kv_commit_kernel(int32_t* __restrict__ lens, const int32_t* __restrict__ n_acc,
                                 int batch, int l_max, uint32_t* __restrict__ status) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  const int64_t nl = static_cast<int64_t>(lens[b]) + n_acc[b] + 1;
  if (lens[b] < 0 || n_acc[b] < 0 || nl > l_max) {
    if (status) atomicOr(status, kDevBadInput);
    return;
  }
  lens[b] = static_cast<int32_t>(nl);
}

struct AttnArgs {
  const float* qkv;
  int64_t ld;
  const int32_t* lens;
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  float* out;
  int64_t ld_out;
  uint8_t* work;
  int t_new, h_q, h_kv, offset, l_max, ctx_max, chunks, rows;
};

// Dynamic shared memory of one CTA: the chunk's keys and values (bf16,
// [kAttnChunk][128] each, copied by TMA), the queries [rows][128] and the
// weights [rows][kAttnChunk] in fp32.
__host__ __device__ inline int64_t attn_smem_bytes(int rows) {
  return 2ll * kAttnChunk * kHeadDim * 2 + static_cast<int64_t>(rows) * (kHeadDim + kAttnChunk) * 4;
}

// grid (chunks, h_kv, batch), kAttnThreads threads.
__global__ void __launch_bounds__(kAttnThreads, 4) attn_decode_kernel(const AttnArgs a) {
  extern __shared__ __align__(128) uint8_t attn_smem[];
  uint16_t* const k_s = reinterpret_cast<uint16_t*>(attn_smem);                  // [chunk][128]
  uint16_t* const v_s = k_s + kAttnChunk * kHeadDim;                              // [chunk][128]
  float* const q_s = reinterpret_cast<float*>(v_s + kAttnChunk * kHeadDim);       // [rows][128]
  float* const p_s = q_s + a.rows * kHeadDim;                                     // [rows][chunk]
  __shared__ __align__(8) uint64_t kv_bar;
  __shared__ float row_m[kAttnMaxRows], row_l[kAttnMaxRows];
  __shared__ int is_last;
  __shared__ int abort_flag;

  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int group = a.h_q / a.h_kv;
  const int rows = a.rows;                                          // t_new * group
  const AttnLayout lay = attn_layout(gridDim.z, a.h_kv, a.chunks, rows);
  uint32_t* const status = reinterpret_cast<uint32_t*>(a.work);

  // keys the last row of this sequence may see; a length outside the cache
  // or the declared context makes the sequence empty and is reported
  const int64_t len = a.lens[b];
  int64_t n_ctx = len + a.offset + a.t_new;
  if (len < 0 || n_ctx > a.ctx_max || n_ctx > a.l_max) {
    if (tid == 0 && chunk == 0) atomicOr(status, kDevBadInput);
    n_ctx = 0;
  }
  const int64_t k0 = static_cast<int64_t>(chunk) * kAttnChunk;
  const int64_t left = n_ctx - k0;
  const int n_keys = left <= 0 ? 0 : (left >= kAttnChunk ? kAttnChunk : static_cast<int>(left));
  // row r = t * group + hh: token t, query head g * group + hh
  auto row_limit = [&](int r) { return len + a.offset + r / group; };   // last visible key

  const uint16_t* const kc = a.k_cache + ((static_cast<int64_t>(b) * a.h_kv + g) * a.l_max + k0) * kHeadDim;
  const uint16_t* const vc = a.v_cache + ((static_cast<int64_t>(b) * a.h_kv + g) * a.l_max + k0) * kHeadDim;
  const uint32_t bar = static_cast<uint32_t>(__cvta_generic_to_shared(&kv_bar));
  // The chunk's keys and values are contiguous rows of 256 bytes: one bulk
  // copy each into shared memory, completing on one transaction barrier.
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(bar, 1);
    fence_barrier_init();
    if (n_keys > 0) {
      const uint32_t bytes = static_cast<uint32_t>(n_keys) * kHeadDim * 2;
      mbar_arrive_expect_tx(bar, 2 * bytes);
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
          ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(k_s))), "l"(kc), "r"(bytes), "r"(bar)
          : "memory");
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
          ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(v_s))), "l"(vc), "r"(bytes), "r"(bar)
          : "memory");
    }
  }
  // queries of this KV head's rows into shared memory meanwhile
  for (int e = tid * 4; e < rows * kHeadDim; e += kAttnThreads * 4) {
    const int r = e / kHeadDim, i = e % kHeadDim;
    const int t = r / group, h = g * group + r % group;
    const float4 v = *reinterpret_cast<const float4*>(
        a.qkv + (static_cast<int64_t>(b) * a.t_new + t) * a.ld + static_cast<int64_t>(h) * kHeadDim + i);
    *reinterpret_cast<float4*>(q_s + e) = v;
  }
  __syncthreads();
  const bool ok = __syncthreads_and(n_keys == 0 || mbar_wait(bar, 0, &abort_flag, status));
  if (!ok && tid == 0) {
    // the copies did not land in time (reported): let them finish before
    // the shared memory is released, and leave an empty partial
    mbar_wait_drain(bar, 0);
  }
  const int n_live = ok ? n_keys : 0;

  // ---- scores: lane = key.  Lane l reads its row's 16-byte pieces in the
  // order (c + l) mod 16, so the 8 lanes of a quarter warp hit 8 different
  // bank groups; the queries are read at the same pieces.
  {
    const int jl = warp * 32 + lane;
    const bool have = jl < n_live;
    const uint4* krow = reinterpret_cast<const uint4*>(k_s + jl * kHeadDim);
    for (int r0 = 0; r0 < rows; r0 += kAttnRowBlock) {
      float acc[kAttnRowBlock];
#pragma unroll
      for (int rr = 0; rr < kAttnRowBlock; ++rr) acc[rr] = 0.f;
      if (have) {
#pragma unroll 4
        for (int c = 0; c < kHeadDim / 8; ++c) {
          const int cc = (c + lane) & (kHeadDim / 8 - 1);
          const uint4 kw = krow[cc];
          const float kf[8] = {bf16_lo(kw.x), bf16_hi(kw.x), bf16_lo(kw.y), bf16_hi(kw.y),
                               bf16_lo(kw.z), bf16_hi(kw.z), bf16_lo(kw.w), bf16_hi(kw.w)};
#pragma unroll
          for (int rr = 0; rr < kAttnRowBlock; ++rr) {
            if (r0 + rr < rows) {
              const float4 qa = *reinterpret_cast<const float4*>(q_s + (r0 + rr) * kHeadDim + cc * 8);
              const float4 qb = *reinterpret_cast<const float4*>(q_s + (r0 + rr) * kHeadDim + cc * 8 + 4);
              acc[rr] = fmaf(qa.x, kf[0], acc[rr]);
              acc[rr] = fmaf(qa.y, kf[1], acc[rr]);
              acc[rr] = fmaf(qa.z, kf[2], acc[rr]);
              acc[rr] = fmaf(qa.w, kf[3], acc[rr]);
              acc[rr] = fmaf(qb.x, kf[4], acc[rr]);
              acc[rr] = fmaf(qb.y, kf[5], acc[rr]);
              acc[rr] = fmaf(qb.z, kf[6], acc[rr]);
              acc[rr] = fmaf(qb.w, kf[7], acc[rr]);
            }
          }
        }
      }
#pragma unroll
      for (int rr = 0; rr < kAttnRowBlock; ++rr) {
        const int r = r0 + rr;
        if (r < rows) {
          const bool visible = have && k0 + jl <= row_limit(r);
          p_s[r * kAttnChunk + jl] = visible ? acc[rr] * kInvSqrtHeadDim : -INFINITY;
        }
      }
    }
  }
  __syncthreads();

  // ---- softmax of the chunk per row (its own maximum): a warp per row
  for (int r = warp; r < rows; r += kAttnThreads / 32) {
    float* pr = p_s + r * kAttnChunk;
    float m = -INFINITY;
    for (int j = lane; j < kAttnChunk; j += 32) m = fmaxf(m, pr[j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int j = lane; j < kAttnChunk; j += 32) {
      const float p = (m == -INFINITY) ? 0.f : expf(pr[j] - m);
      pr[j] = p;
      l += p;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      row_m[r] = m;
      row_l[r] = l;
    }
  }
  __syncthreads();

  // ---- weighted values: warp w owns head columns 32w .. 32w+31 (lane = one
  // column) over all the chunk's keys, so no cross-warp sum is needed
  const int64_t part = (static_cast<int64_t>(b) * a.h_kv + g) * a.chunks + chunk;
  float* const part_o = reinterpret_cast<float*>(a.work + lay.off_o) + part * rows * kHeadDim;
  float* const part_ml = reinterpret_cast<float*>(a.work + lay.off_ml) + part * rows * 2;
  const int d = warp * 32 + lane;
  for (int r0 = 0; r0 < rows; r0 += kAttnRowBlock) {
    float o[kAttnRowBlock];
#pragma unroll
    for (int rr = 0; rr < kAttnRowBlock; ++rr) o[rr] = 0.f;
    const int n4 = n_live & ~3;
    for (int j = 0; j < n4; j += 4) {
      const float v0 = __uint_as_float(static_cast<uint32_t>(v_s[(j + 0) * kHeadDim + d]) << 16);
      const float v1 = __uint_as_float(static_cast<uint32_t>(v_s[(j + 1) * kHeadDim + d]) << 16);
      const float v2 = __uint_as_float(static_cast<uint32_t>(v_s[(j + 2) * kHeadDim + d]) << 16);
      const float v3 = __uint_as_float(static_cast<uint32_t>(v_s[(j + 3) * kHeadDim + d]) << 16);
#pragma unroll
      for (int rr = 0; rr < kAttnRowBlock; ++rr) {
        if (r0 + rr < rows) {
          const float4 p = *reinterpret_cast<const float4*>(p_s + (r0 + rr) * kAttnChunk + j);
          o[rr] = fmaf(p.x, v0, o[rr]);
          o[rr] = fmaf(p.y, v1, o[rr]);
          o[rr] = fmaf(p.z, v2, o[rr]);
          o[rr] = fmaf(p.w, v3, o[rr]);
        }
      }
    }
    for (int j = n4; j < n_live; ++j) {
      const float v = __uint_as_float(static_cast<uint32_t>(v_s[j * kHeadDim + d]) << 16);
#pragma unroll
      for (int rr = 0; rr < kAttnRowBlock; ++rr)
        if (r0 + rr < rows) o[rr] = fmaf(p_s[(r0 + rr) * kAttnChunk + j], v, o[rr]);
    }
#pragma unroll
    for (int rr = 0; rr < kAttnRowBlock; ++rr)
      if (r0 + rr < rows) part_o[(r0 + rr) * kHeadDim + d] = o[rr];
  }
  if (tid < rows) {
    part_ml[tid * 2] = ok ? row_m[tid] : -INFINITY;
    part_ml[tid * 2 + 1] = ok ? row_l[tid] : 0.f;
  }

  // ---- the last chunk of this (sequence, KV head) to arrive merges all chunks
  uint32_t* const counter = reinterpret_cast<uint32_t*>(a.work + lay.off_counters) +
                            static_cast<int64_t>(b) * a.h_kv + g;
  __syncthreads();
  if (tid == 0) {
    __threadfence();                                   // this CTA's partials before its arrival
    const uint32_t prev = atomicAdd(counter, 1u);
    is_last = prev == static_cast<uint32_t>(a.chunks - 1);
    if (is_last) __threadfence();                      // ... and the others' before the reads below
  }
  __syncthreads();
  if (!is_last) return;
  const float* const all_o = reinterpret_cast<const float*>(a.work + lay.off_o) +
                             (static_cast<int64_t>(b) * a.h_kv + g) * a.chunks * rows * kHeadDim;
  const float* const all_ml = reinterpret_cast<const float*>(a.work + lay.off_ml) +
                              (static_cast<int64_t>(b) * a.h_kv + g) * a.chunks * rows * 2;
  for (int r = 0; r < rows; ++r) {
    float mx = -INFINITY;
    for (int c = 0; c < a.chunks; ++c) mx = fmaxf(mx, __ldcg(all_ml + (c * rows + r) * 2));
    float l = 0.f, acc = 0.f;
    if (mx != -INFINITY) {
      for (int c = 0; c < a.chunks; ++c) {
        const float mc = __ldcg(all_ml + (c * rows + r) * 2);
        if (mc == -INFINITY) continue;                 // no visible key in that chunk
        const float sc = expf(mc - mx);
        l = fmaf(__ldcg(all_ml + (c * rows + r) * 2 + 1), sc, l);
        acc = fmaf(__ldcg(all_o + (static_cast<int64_t>(c) * rows + r) * kHeadDim + tid), sc, acc);
      }
    }
    const int t = r / group, h = g * group + r % group;
    a.out[(static_cast<int64_t>(b) * a.t_new + t) * a.ld_out + static_cast<int64_t>(h) * kHeadDim + tid] =
        l > 0.f ? acc / l : 0.f;
  }
  if (tid == 0) *counter = 0u;                         // ready for the next call
}

}  // namespace qspec
