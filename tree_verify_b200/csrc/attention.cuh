// attention.cuh -- tree attention for the verification pass (EAGLE summary, section 3
// "Drafting and verification": the target verifies the tree-structured draft in a single
// forward pass using tree attention; appendix A.1 "Tree Structure").
//
// For sequence b, node i, query head h (kv head g = h / G):
//     out[b,i,h] = sum_j softmax_j(scale * q[b,i,h] . k_j) v_j
// over the prefix positions 0 .. L_b-1 of kv head g and the tree nodes on the path from
// i to the root (i included).
//
// This file holds what both precisions share (parameters, the 128-byte-swizzled tile
// layout of 128-key K/V tiles), the log-sum-exp merge of split partials, and the fp32
// path.  The bf16 path runs on the tensor cores (attention_tc.cuh).
//
// f32 path: one warp per output row, fp32 SIMT, keys streamed in order (small shapes).
#pragma once

#include "device_common.cuh"

namespace eagle {

constexpr int kAttnKeys = 128;       // keys per tile

struct AttnParams {
  const __nv_bfloat16* q;       // [B,N,Hq,D]
  const __nv_bfloat16* k_tree;  // [B,N,Hkv,D]
  const __nv_bfloat16* v_tree;
  const int32_t* prefix_lens;   // [B]
  const int32_t* parents;       // [B,N]
  __nv_bfloat16* out;           // [B,N,Hq,D] (single split)
  float* part_acc;              // [B*N*Hq, splits, D]
  float* part_ml;               // [B*N*Hq, splits, 2]
  int32_t B, N, Hq, Hkv, G, Lmax;
  int32_t num_splits, tiles_per_split;
  float scale_log2;             // softmax scale * log2(e)
};

// Byte offset of element (row, d) in a kAttnKeys-row tile stored as D/64 boxes of
// [kAttnKeys][64] bf16 with the 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t attn_swz(int row, int d) {
  const int half = d >> 6;
  const int chunk = (d & 63) >> 3;
  return static_cast<uint32_t>(half * (kAttnKeys * 128) + row * 128 + ((chunk ^ (row & 7)) << 4) +
                               ((d & 7) << 1));
}

// Log-sum-exp merge of split partials: one warp per output row.  The splits' (m, l) and
// accumulators are loaded eight splits at a time with every load issued before any is
// used, so a row costs about one memory round trip per eight splits.
template <int D>
__global__ void __launch_bounds__(128)
    tree_attn_combine_kernel(const float* __restrict__ part_acc, const float* __restrict__ part_ml,
                             __nv_bfloat16* __restrict__ out, int rows, int splits) {
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int kPer = D / 32;
  constexpr int kBatch = 8;
  const float* ml = part_ml + static_cast<size_t>(row) * splits * 2;
  float mmax = -INFINITY;
  for (int s = lane; s < splits; s += 32) mmax = fmaxf(mmax, ml[2 * s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, off));
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float den = 0.f;
  for (int s0 = 0; s0 < splits; s0 += kBatch) {
    float2 mls[kBatch];
    float v[kBatch][kPer];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int s = s0 + k;
      if (s < splits) {
        mls[k] = *reinterpret_cast<const float2*>(ml + 2 * s);
        const float* src = part_acc + (static_cast<size_t>(row) * splits + s) * D + lane * kPer;
        if constexpr (kPer == 4) {
          const float4 t = *reinterpret_cast<const float4*>(src);
          v[k][0] = t.x;
          v[k][1] = t.y;
          v[k][2] = t.z;
          v[k][3] = t.w;
        } else {
          const float2 t = *reinterpret_cast<const float2*>(src);
          v[k][0] = t.x;
          v[k][1] = t.y;
        }
      } else {
        mls[k] = make_float2(-INFINITY, 0.f);
      }
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (s0 + k >= splits || mls[k].x == -INFINITY) continue;
      const float w = exp2f(mls[k].x - mmax);
      den += w * mls[k].y;
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] += w * v[k][e];
    }
  }
  const float inv = 1.0f / den;
  __nv_bfloat16* dst = out + static_cast<size_t>(row) * D + lane * kPer;
#pragma unroll
  for (int e = 0; e < kPer; e += 2)
    *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
}

// ------------------------------------------------------------------ fp32 path
// One warp per output row.  Keys go 32 at a time: lane j scores key c + j against the row's
// query (kept in shared memory, read as a broadcast), the warp folds the 32 scores into
// the running maximum and denominator, then every lane accumulates its D/32 output
// columns over those keys (coalesced V rows).  The loads of a chunk are independent of
// one another, so a row costs a few memory round trips per 32 keys rather than one per key.

template <int D>
__global__ void __launch_bounds__(128)
    tree_attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ kp,
                         const float* __restrict__ vp, const int32_t* __restrict__ prefix_lens,
                         const float* __restrict__ kt, const float* __restrict__ vt,
                         const int32_t* __restrict__ parents, float* __restrict__ out, int B, int N,
                         int Hq, int Hkv, int Lmax, float scale) {
  __shared__ float q_s[4][D];
  __shared__ int path_s[4][64];
  const int wid = threadIdx.x >> 5;
  const int row = blockIdx.x * 4 + wid;
  const int lane = threadIdx.x & 31;
  if (row >= B * N * Hq) return;
  const int b = row / (N * Hq);
  const int i = (row / Hq) % N;
  const int h = row % Hq;
  const int g = h / (Hq / Hkv);
  constexpr int kPer = D / 32;
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    q_s[wid][lane + 32 * e] = q[static_cast<size_t>(row) * D + lane + 32 * e];
    acc[e] = 0.f;
  }
  // the node's path to the root (a link that does not point to an earlier node ends it)
  int np = 0;
  if (lane == 0) {
    int a = i;
    for (int guard = 0; guard < 64 && a >= 0; ++guard) {
      path_s[wid][np++] = a;
      const int p = parents[static_cast<size_t>(b) * N + a];
      a = (p >= 0 && p < a) ? p : -1;
    }
  }
  np = __shfl_sync(0xffffffffu, np, 0);
  __syncwarp();
  int L = prefix_lens[b];
  if ((L < 0 || L > Lmax) && lane == 0) record_error(kErrAttnPrefixLen);
  L = L < 0 ? 0 : (L > Lmax ? Lmax : L);
  const size_t pbase = (static_cast<size_t>(b) * Hkv + g) * Lmax;
  auto key_row = [&](int j, const float* pre, const float* tree) -> const float* {
    return j < L ? pre + (pbase + j) * D
                 : tree + ((static_cast<size_t>(b) * N + path_s[wid][j - L]) * Hkv + g) * D;
  };
  const int nk = L + np;
  float m = -INFINITY, l = 0.f;
  for (int c = 0; c < nk; c += 32) {
    const int j = c + lane;
    float s = -INFINITY;
    if (j < nk) {
      const float* kr = key_row(j, kp, kt);
      // the whole key row is loaded before the dot product starts (one round trip)
      float kv[D];
#pragma unroll
      for (int d = 0; d < D; d += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(kr + d);
        kv[d] = k4.x;
        kv[d + 1] = k4.y;
        kv[d + 2] = k4.z;
        kv[d + 3] = k4.w;
      }
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int d = 0; d < D; d += 2) {
        d0 = fmaf(q_s[wid][d], kv[d], d0);
        d1 = fmaf(q_s[wid][d + 1], kv[d + 1], d1);
      }
      s = (d0 + d1) * scale;
    }
    float cm = s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
    const float mn = fmaxf(m, cm);
    const float corr = expf(m - mn);
    const float p = j < nk ? expf(s - mn) : 0.f;
    float ps = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * corr + ps;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] *= corr;
    const int cnt = min(32, nk - c);
    // eight keys' V loads in flight before their products are added (in key order)
    for (int t0 = 0; t0 < cnt; t0 += 8) {
      float vv[8][kPer];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float* vr = key_row(min(c + t0 + t, nk - 1), vp, vt);
#pragma unroll
        for (int e = 0; e < kPer; ++e) vv[t][e] = vr[lane + 32 * e];
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float pt = __shfl_sync(0xffffffffu, p, t0 + t < 32 ? t0 + t : 31);
        if (t0 + t < cnt) {
#pragma unroll
          for (int e = 0; e < kPer; ++e) acc[e] = fmaf(pt, vv[t][e], acc[e]);
        }
      }
    }
    m = mn;
  }
  const float inv = 1.0f / l;
#pragma unroll
  for (int e = 0; e < kPer; ++e) out[static_cast<size_t>(row) * D + lane + 32 * e] = acc[e] * inv;
}

}  // namespace eagle
