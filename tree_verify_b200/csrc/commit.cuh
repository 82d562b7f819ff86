// commit.cuh -- post-accept commit: the root and the accepted nodes of each sequence are
// appended to the prefix K/V cache and their hidden rows gathered for the next drafting
// round (EAGLE summary, section 3 "Drafting and verification": accepted draft tokens extend
// the target's context, and the accepted tokens' features feed the next draft).
//
// Pure data movement, bound by memory latency at these sizes: a step commits at most 64
// rows per sequence.  Grid (B, Hkv + N): block (b, g < Hkv) copies the K and V rows of kv
// head g (one warp per row, 16-byte vectors); block (b, Hkv + t) copies feature row t.
// Every block validates the path itself (at most 64 nodes), so no block waits on another.
#pragma once

#include "device_common.cuh"

namespace eagle {

constexpr int kCommitThreads = 128;

struct CommitParams {
  uint8_t* k_prefix;            // [B, Hkv, Lmax, D] elements of `esize` bytes
  uint8_t* v_prefix;
  const int32_t* prefix_lens;   // [B]
  const uint8_t* k_tree;        // [B, N, Hkv, D]
  const uint8_t* v_tree;
  const uint8_t* hidden;        // [B*N, H]
  const int32_t* parents;       // [B, N]
  const int32_t* accepted_nodes;
  const int32_t* accept_len;    // [B]
  int32_t* new_lens;            // [B]
  uint8_t* feat;                // [B, N, H]
  int32_t N, Hkv, Lmax;
  int32_t row_bytes;            // D * esize, a multiple of 16
  int32_t hrow_bytes;           // H * esize, a multiple of 4
};

// Copies `bytes` from src to dst with the threads [t0, t0 + nthr) of the block.
__device__ __forceinline__ void commit_copy(uint8_t* dst, const uint8_t* src, int bytes, int t0,
                                            int nthr) {
  if ((bytes & 15) == 0) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* d = reinterpret_cast<uint4*>(dst);
    for (int i = t0; i < bytes / 16; i += nthr) d[i] = s[i];
  } else {
    const uint32_t* s = reinterpret_cast<const uint32_t*>(src);
    uint32_t* d = reinterpret_cast<uint32_t*>(dst);
    for (int i = t0; i < bytes / 4; i += nthr) d[i] = s[i];
  }
}

__global__ void __launch_bounds__(kCommitThreads) commit_kernel(const CommitParams p) {
  __shared__ int32_t path[64];
  const int b = blockIdx.x;
  const int N = p.N;
  const size_t seq = static_cast<size_t>(b) * N;
  const int32_t L = p.prefix_lens[b];
  const int32_t a = p.accept_len[b];
  if (a == -1) {  // the walk found the tree invalid: nothing committed, length unchanged
    if (blockIdx.y == 0 && threadIdx.x == 0) p.new_lens[b] = L;
    return;
  }
  // the path is the root, then accepted node t-1 at position t; node t+1 must be a child of
  // node t
  const bool shape_ok = a >= 0 && a <= N - 1 && L >= 0 && L <= p.Lmax && L + a + 1 <= p.Lmax;
  int ok = 1;
  if (threadIdx.x == 0) path[0] = 0;
  if (shape_ok && threadIdx.x < a) {
    const int32_t c = p.accepted_nodes[seq + threadIdx.x];
    const int32_t prev = threadIdx.x == 0 ? 0 : p.accepted_nodes[seq + threadIdx.x - 1];
    ok = c >= 1 && c < N && p.parents[seq + c] == prev;
    path[threadIdx.x + 1] = c;
  }
  ok = __syncthreads_and(ok) && shape_ok;
  if (!ok) {
    if (blockIdx.y == 0 && threadIdx.x == 0) p.new_lens[b] = -1;
    return;
  }
  const int n = a + 1;
  if (blockIdx.y == 0 && threadIdx.x == 0) p.new_lens[b] = L + n;
  const int y = blockIdx.y;
  if (y < p.Hkv) {
    // K and V rows of kv head g: 2n rows, one warp per row
    const int g = y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp; r < 2 * n; r += kCommitThreads / 32) {
      const int t = r >> 1;
      const bool is_v = r & 1;
      const size_t src = ((seq + path[t]) * p.Hkv + g) * p.row_bytes;
      const size_t dst = ((static_cast<size_t>(b) * p.Hkv + g) * p.Lmax + L + t) * p.row_bytes;
      commit_copy((is_v ? p.v_prefix : p.k_prefix) + dst, (is_v ? p.v_tree : p.k_tree) + src,
                  p.row_bytes, lane, 32);
    }
  } else {
    const int t = y - p.Hkv;
    if (t >= n) return;
    commit_copy(p.feat + (seq + t) * p.hrow_bytes, p.hidden + (seq + path[t]) * p.hrow_bytes,
                p.hrow_bytes, threadIdx.x, kCommitThreads);
  }
}

}  // namespace eagle
