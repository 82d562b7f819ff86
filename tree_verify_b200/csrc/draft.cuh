// draft.cuh -- children of draft nodes (EAGLE summary, appendix A.1 "Tree Structure": in
// greedy decoding a node's children are the top k tokens by probability, in non-greedy
// decoding k tokens are sampled; section 3: the draft samples its next token through the
// LM head).  Row r = (sequence b, draft node f) of the draft LM head's logits:
//   T == 0: the k largest logits in decreasing order, ties to the lower index;
//   T  > 0: k independent samples of p = softmax(logits / T), each an exponential race
//           argmin_v ln(-ln u_v) - ln p_v with Philox uniforms (node f, purpose 2 + j);
//   each child's confidence is its probability (the input of EAGLE-2 reranking), and the
//   row's p may be written out as the draft distribution the accept walk reads.
//
// One CTA of 512 threads per row: a max and a sum-exp reduction, then either k rounds of a
// block argmax below the previous pick (T == 0) or one pass in which every thread keeps k
// running race minima in registers followed by k block argmins (T > 0).  Bound by the row
// read (V floats) at T == 0 and by the k Philox draws per entry at T > 0.
#pragma once

#include <limits.h>

#include "device_common.cuh"
#include "philox.cuh"

namespace eagle {

constexpr int kDraftThreads = 512;
constexpr int kDraftWarps = kDraftThreads / 32;
constexpr int kDraftMaxK = 16;

struct DraftParams {
  const float* logits;  // [R, V], R = B * F
  int32_t* tokens;      // [R, k]
  float* conf;          // [R, k]
  float* probs;         // [R, V] or null
  int32_t F, V, k;
  float T;
  uint64_t seed, offset;
};

// (value, index) pairs: `better` is larger value, then lower index (argmax); the race uses
// smaller key, then lower index, passed in as the negated key.
__device__ __forceinline__ bool draft_better(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

// Block-wide argmax of (value, index); every thread returns the winner.
__device__ __forceinline__ void draft_block_argmax(float& val, int& idx, float* sval, int* sidx) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, val, off);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
    if (draft_better(ov, oi, val, idx)) {
      val = ov;
      idx = oi;
    }
  }
  if (lane == 0) {
    sval[warp] = val;
    sidx[warp] = idx;
  }
  __syncthreads();
  val = sval[0];
  idx = sidx[0];
  for (int w = 1; w < kDraftWarps; ++w)
    if (draft_better(sval[w], sidx[w], val, idx)) {
      val = sval[w];
      idx = sidx[w];
    }
  __syncthreads();  // the slots are reused by the next reduction
}

__device__ __forceinline__ float draft_block_sum(float x, float* sval) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  if (lane == 0) sval[warp] = x;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < kDraftWarps; ++w) s += sval[w];
  __syncthreads();
  return s;
}

template <bool kGreedy>
__global__ void __launch_bounds__(kDraftThreads) draft_select_kernel(const DraftParams p) {
  __shared__ float sval[kDraftWarps];
  __shared__ int sidx[kDraftWarps];
  const int r = blockIdx.x;
  const int b = r / p.F, f = r % p.F;
  const int V = p.V, k = p.k;
  const float* row = p.logits + static_cast<size_t>(r) * V;
  const float invT = kGreedy ? 1.0f : 1.0f / p.T;
  const int tid = threadIdx.x;

  // softmax statistics of y = logit * invT
  float m = -INFINITY;
  for (int v = tid; v < V; v += kDraftThreads) m = fmaxf(m, row[v] * invT);
  int dummy = 0;
  draft_block_argmax(m, dummy, sval, sidx);
  float z = 0.f;
  if (m != -INFINITY)
    for (int v = tid; v < V; v += kDraftThreads) z += expf(row[v] * invT - m);
  z = draft_block_sum(z, sval);
  const float invZ = z > 0.f ? 1.0f / z : 0.f;

  if (p.probs != nullptr) {
    float* out = p.probs + static_cast<size_t>(r) * V;
    for (int v = tid; v < V; v += kDraftThreads) out[v] = expf(row[v] * invT - m) * invZ;
  }

  int32_t* tok = p.tokens + static_cast<size_t>(r) * k;
  float* conf = p.conf + static_cast<size_t>(r) * k;
  if (kGreedy) {
    // round j: the best logit strictly below the previous pick in (value desc, index asc)
    float pv = INFINITY;
    int pi = -1;
    for (int j = 0; j < k; ++j) {
      float best = -INFINITY;
      int bi = INT_MAX;
      for (int v = tid; v < V; v += kDraftThreads) {
        const float x = row[v];
        const bool below = x < pv || (x == pv && v > pi);
        if (below && draft_better(x, v, best, bi)) {
          best = x;
          bi = v;
        }
      }
      draft_block_argmax(best, bi, sval, sidx);
      const bool found = bi != INT_MAX && !(best == -INFINITY && bi == INT_MAX);
      if (tid == 0) {
        tok[j] = found ? bi : -1;
        conf[j] = found ? expf(row[bi] * invT - m) * invZ : 0.f;
      }
      if (!found) {
        for (int jj = j + 1 + tid; jj < k; jj += kDraftThreads) {
          tok[jj] = -1;
          conf[jj] = 0.f;
        }
        break;
      }
      pv = best;
      pi = bi;
    }
  } else {
    // k races in one pass: thread-local minima of key = ln(-ln u) - (y - m)
    float key[kDraftMaxK];
    int arg[kDraftMaxK];
#pragma unroll
    for (int j = 0; j < kDraftMaxK; ++j) {
      key[j] = INFINITY;
      arg[j] = INT_MAX;
    }
    for (int v0 = 4 * tid; v0 < V; v0 += 4 * kDraftThreads) {
      float lw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) lw[e] = v0 + e < V ? row[v0 + e] * invT - m : -INFINITY;
#pragma unroll
      for (int j = 0; j < kDraftMaxK; ++j) {
        if (j >= k) break;
        const Philox4 u = philox_group(p.seed, p.offset, static_cast<uint32_t>(b),
                                       static_cast<uint32_t>(f), static_cast<uint32_t>(2 + j),
                                       static_cast<uint32_t>(v0) >> 2);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (lw[e] == -INFINITY) continue;
          const float kk = logf(-logf(word_to_uniform(u.w[e]))) - lw[e];
          if (kk < key[j]) {
            key[j] = kk;
            arg[j] = v0 + e;
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kDraftMaxK; ++j) {
      if (j >= k) break;
      float nk = -key[j];  // argmin of the key = argmax of its negation, lower index on ties
      int a = arg[j];
      draft_block_argmax(nk, a, sval, sidx);
      if (tid == 0) {
        const bool found = a != INT_MAX;
        tok[j] = found ? a : -1;
        conf[j] = found ? expf(row[a] * invT - m) * invZ : 0.f;
      }
    }
  }
}

}  // namespace eagle
