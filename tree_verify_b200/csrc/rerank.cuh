// rerank.cuh -- EAGLE-2 reranking: from an expanded candidate tree, keep the m candidates
// the target is most likely to accept and renumber them as the tree to verify (EAGLE-2
// blog, section 1: a draft token's confidence approximates the probability that the target
// accepts it; section 4: after expansion, reranking keeps the tokens with the highest
// acceptance probability as the target's input).  A candidate is reached only if its whole
// path is accepted, so its value is the product of the confidences along the path.
//
// One CTA of up to 1024 threads per sequence, one thread per candidate:
//   values   v_0 = 1, v_i = v_parent * clamp(c_i, 0, 1) (NaN counts as 0), float32, root
//            first -- computed level by level (a node takes its value once its parent's is
//            known), so every product is rounded exactly as in the sequential definition;
//   rank     the number of candidates with a higher value, or an equal value and a lower
//            index; kept iff rank < min(m, M) (with c <= 1 a kept node's ancestors are kept);
//   renumber by a block-wide prefix count of the kept flags (candidate order is topological);
//   masks    each kept node ORs the new indices of its ancestors and itself.
#pragma once

#include "device_common.cuh"

namespace eagle {

constexpr int kRerankThreads = 1024;
constexpr int kRerankMaxSelect = 64;

struct RerankParams {
  const int32_t* parents;      // [B, M]
  const int32_t* tokens;       // [B, M]
  const float* confidence;     // [B, M]
  int32_t* sel;                // [B, m]
  int32_t* parents_out;        // [B, m]
  int32_t* tokens_out;         // [B, m]
  uint64_t* masks_out;         // [B, m]
  int32_t* num_selected;       // [B]
  int32_t M, m;
};

__global__ void __launch_bounds__(kRerankThreads) rerank_kernel(const RerankParams p) {
  __shared__ int32_t par_s[kRerankThreads];
  __shared__ float v_s[kRerankThreads];
  __shared__ uint8_t ready[kRerankThreads];
  __shared__ int32_t newidx[kRerankThreads];
  __shared__ int32_t warp_kept[kRerankThreads / 32];
  const int b = blockIdx.x;
  const int i = threadIdx.x;
  const int M = p.M, m = p.m;
  const size_t row = static_cast<size_t>(b) * M;
  const size_t orow = static_cast<size_t>(b) * m;
  const bool live = i < M;
  int32_t pi = -1;
  float ci = 0.f;
  int ok = 1;
  if (live) {
    pi = p.parents[row + i];
    const float c = p.confidence[row + i];
    ci = c > 0.f ? (c < 1.f ? c : 1.f) : 0.f;
    ok = i == 0 ? pi == -1 : (pi >= 0 && pi < i);
    par_s[i] = pi;
    v_s[i] = 1.f;
    ready[i] = i == 0;
  }
  // padding of the outputs past the kept count (and everything for a bad tree)
  if (__syncthreads_and(ok) == 0) {
    if (i < m) {
      p.sel[orow + i] = -1;
      p.parents_out[orow + i] = -1;
      p.tokens_out[orow + i] = -1;
      p.masks_out[orow + i] = 0;
    }
    if (i == 0) p.num_selected[b] = -1;
    return;
  }
  // path values, one tree level per round: read at the start of the round, write after
  for (;;) {
    const bool step = live && !ready[i] && ready[pi];
    const float val = step ? v_s[pi] * ci : 0.f;
    __syncthreads();
    if (step) {
      v_s[i] = val;
      ready[i] = 1;
    }
    if (__syncthreads_or(step) == 0) break;
  }
  const int k = m < M ? m : M;
  int rank = 0;
  if (live) {
    const float vi = v_s[i];
    for (int j = 0; j < M; ++j) {
      const float vj = v_s[j];
      rank += (vj > vi || (vj == vi && j < i)) ? 1 : 0;
    }
  }
  const bool kept = live && rank < k;
  // new index = number of kept candidates before i
  const int lane = i & 31, warp = i >> 5;
  const uint32_t ballot = __ballot_sync(0xffffffffu, kept);
  if (lane == 0) warp_kept[warp] = __popc(ballot);
  __syncthreads();
  int before = __popc(ballot & ((1u << lane) - 1u));
  for (int w = 0; w < warp; ++w) before += warp_kept[w];
  if (live) newidx[i] = kept ? before : -1;
  __syncthreads();
  if (kept) {
    const int t = before;
    p.sel[orow + t] = i;
    p.parents_out[orow + t] = i == 0 ? -1 : newidx[pi];
    p.tokens_out[orow + t] = p.tokens[row + i];
    uint64_t mask = 0;
    for (int a = i; a >= 0; a = par_s[a]) mask |= 1ull << newidx[a];
    p.masks_out[orow + t] = mask;
  }
  if (i >= k && i < m) {
    p.sel[orow + i] = -1;
    p.parents_out[orow + i] = -1;
    p.tokens_out[orow + i] = -1;
    p.masks_out[orow + i] = 0;
  }
  if (i == 0) p.num_selected[b] = k;
}

}  // namespace eagle
