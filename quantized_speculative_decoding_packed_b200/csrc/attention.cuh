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
// read once per pass): one CTA per (sequence, KV head, chunk of 256 keys),
// so the cache streams through all SMs whatever the batch.  In a CTA each
// lane owns one key for the scores (its 256-byte row in registers, the
// queries broadcast from shared memory), the softmax of the chunk is exact
// (its own maximum), and for the values the lanes span the head dimension
// (4 columns each, a warp per 64 keys).  Each CTA leaves its (max, sum,
// weighted values) per query row in the workspace; the last CTA of a
// (sequence, KV head) to arrive merges the chunks in chunk order, so the
// result does not depend on which CTA finishes last.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "device_common.cuh"

namespace qspec {

constexpr int kHeadDim = 128;
constexpr int kAttnChunk = 256;              // keys per CTA
constexpr int kAttnThreads = 128;            // 4 warps
constexpr int kAttnMaxRows = 32;             // (query heads per KV head) x new tokens
constexpr int kAttnRowBlock = 8;             // query rows per register block
constexpr int kAttnMaxChunks = 128;          // context up to 32768 keys
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

// grid (chunks, h_kv, batch), kAttnThreads threads; dynamic shared memory:
// queries [rows][128] + weights [rows][256] + merge [4][8][128] floats.
__global__ void __launch_bounds__(kAttnThreads, 4) attn_decode_kernel(const AttnArgs a) {
  extern __shared__ float4 attn_smem4[];
  float* const q_s = reinterpret_cast<float*>(attn_smem4);          // [rows][128]
  float* const p_s = q_s + a.rows * kHeadDim;                       // [rows][256]
  float* const red = p_s + a.rows * kAttnChunk;                     // [4][8][128]
  __shared__ float row_m[kAttnMaxRows], row_l[kAttnMaxRows];
  __shared__ int is_last;

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

  // queries of this KV head's rows into shared memory
  for (int e = tid * 4; e < rows * kHeadDim; e += kAttnThreads * 4) {
    const int r = e / kHeadDim, i = e % kHeadDim;
    const int t = r / group, h = g * group + r % group;
    const float4 v = *reinterpret_cast<const float4*>(
        a.qkv + (static_cast<int64_t>(b) * a.t_new + t) * a.ld + static_cast<int64_t>(h) * kHeadDim + i);
    *reinterpret_cast<float4*>(q_s + e) = v;
  }
  __syncthreads();

  const uint16_t* const kc = a.k_cache + (static_cast<int64_t>(b) * a.h_kv + g) * a.l_max * kHeadDim;
  const uint16_t* const vc = a.v_cache + (static_cast<int64_t>(b) * a.h_kv + g) * a.l_max * kHeadDim;

  // ---- scores: lane = key (two keys of 32 per warp pass, 64 per warp)
  for (int pass = 0; pass < 2; ++pass) {
    const int jl = warp * 64 + pass * 32 + lane;                    // key within the chunk
    const bool have = jl < n_keys;
    uint4 kr[kHeadDim / 8];
    if (have) {
      const uint4* src = reinterpret_cast<const uint4*>(kc + (k0 + jl) * kHeadDim);
#pragma unroll
      for (int c = 0; c < kHeadDim / 8; ++c) kr[c] = __ldcs(src + c);
    }
    for (int r0 = 0; r0 < rows; r0 += kAttnRowBlock) {
      float acc[kAttnRowBlock];
#pragma unroll
      for (int rr = 0; rr < kAttnRowBlock; ++rr) acc[rr] = 0.f;
      if (have) {
#pragma unroll
        for (int c = 0; c < kHeadDim / 8; ++c) {
          const float kf[8] = {bf16_lo(kr[c].x), bf16_hi(kr[c].x), bf16_lo(kr[c].y), bf16_hi(kr[c].y),
                               bf16_lo(kr[c].z), bf16_hi(kr[c].z), bf16_lo(kr[c].w), bf16_hi(kr[c].w)};
#pragma unroll
          for (int rr = 0; rr < kAttnRowBlock; ++rr) {
            if (r0 + rr < rows) {
              const float4 qa = *reinterpret_cast<const float4*>(q_s + (r0 + rr) * kHeadDim + c * 8);
              const float4 qb = *reinterpret_cast<const float4*>(q_s + (r0 + rr) * kHeadDim + c * 8 + 4);
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

  // ---- weighted values: a warp per 64 keys, lanes over the head dimension
  const int64_t part = (static_cast<int64_t>(b) * a.h_kv + g) * a.chunks + chunk;
  float* const part_o = reinterpret_cast<float*>(a.work + lay.off_o) + part * rows * kHeadDim;
  float* const part_ml = reinterpret_cast<float*>(a.work + lay.off_ml) + part * rows * 2;
  const int j_lo = warp * 64;
  const int j_hi = min(j_lo + 64, n_keys);
  for (int r0 = 0; r0 < rows; r0 += kAttnRowBlock) {
    float o[kAttnRowBlock][4];
#pragma unroll
    for (int rr = 0; rr < kAttnRowBlock; ++rr)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[rr][i] = 0.f;
    for (int j = j_lo; j < j_hi; ++j) {
      const uint2 vr = __ldcs(reinterpret_cast<const uint2*>(vc + (k0 + j) * kHeadDim + lane * 4));
      const float vf[4] = {bf16_lo(vr.x), bf16_hi(vr.x), bf16_lo(vr.y), bf16_hi(vr.y)};
#pragma unroll
      for (int rr = 0; rr < kAttnRowBlock; ++rr) {
        if (r0 + rr < rows) {
          const float p = p_s[(r0 + rr) * kAttnChunk + j];
#pragma unroll
          for (int i = 0; i < 4; ++i) o[rr][i] = fmaf(p, vf[i], o[rr][i]);
        }
      }
    }
#pragma unroll
    for (int rr = 0; rr < kAttnRowBlock; ++rr)
      *reinterpret_cast<float4*>(red + (warp * kAttnRowBlock + rr) * kHeadDim + lane * 4) =
          make_float4(o[rr][0], o[rr][1], o[rr][2], o[rr][3]);
    __syncthreads();
    // the four warps' sums in warp order; thread = column of the head
    for (int rr = 0; rr < kAttnRowBlock && r0 + rr < rows; ++rr) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kAttnThreads / 32; ++w) s += red[(w * kAttnRowBlock + rr) * kHeadDim + tid];
      part_o[(r0 + rr) * kHeadDim + tid] = s;
    }
    __syncthreads();
  }
  if (tid < rows) {
    part_ml[tid * 2] = row_m[tid];
    part_ml[tid * 2 + 1] = row_l[tid];
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
