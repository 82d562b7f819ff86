// accept.cuh -- the accept / resample walk over the draft tree (EAGLE summary, section 2
// "Preliminaries": accept a drafted token t with probability min(1, p(t)/p_hat(t)); after
// a rejection discard the rest of that branch and resample; appendix A.2 "Multi-Round
// Speculative Sampling" and appendix B "Algorithm 1": the rule runs over the k candidates
// of a node with an adjusted distribution after each rejection).
//
// One thread-block cluster walks one sequence.  The vocabulary is split into contiguous
// slices, one per CTA, so every pass over V (row statistics, residual update, final
// sample) runs on CL SMs at once with 128-bit loads; the residual distribution
// r = max(0, p - p_hat) stays in the CTAs' shared memory (two buffers, so that a rejected
// update with zero mass can keep the previous one) and the single entry r[t] that an
// accept test needs is read from its owner through distributed shared memory.  Each
// cluster-wide reduction combines per-CTA partials in rank order, so every CTA reaches
// bit-identical decisions and the walk stays in lockstep without further communication.
// Only the accepted node indices, their count and the one extra token are written.
#pragma once

#include <limits.h>

#include "device_common.cuh"
#include "philox.cuh"

namespace eagle {

constexpr int kAccThreads = 256;
constexpr int kAccWarps = kAccThreads / 32;
constexpr int kAccMaxCluster = 8;

struct AccParams {
  const float* logits;       // [B,N,V]
  const float* draft;        // [B,N,V]
  const int32_t* tokens;     // [B,N]
  const int32_t* parents;    // [B,N]
  int32_t* accepted_nodes;   // [B,N]
  int32_t* accept_len;       // [B]
  int32_t* next_token;       // [B]
  int32_t N, V, slice;       // slice: vocabulary entries per CTA, multiple of 4
  float T;
  uint64_t seed, offset;
};

// ---------------------------------------------------------------- reduction operators
// Payload float4: .x/.y carry the value pair, .z/.w unused.
struct OpMaxSum {  // (max y, sum exp(y - max))
  __device__ __forceinline__ float4 operator()(float4 a, float4 b) const {
    const float m = fmaxf(a.x, b.x);
    if (m == -INFINITY) return make_float4(-INFINITY, 0.f, 0.f, 0.f);
    return make_float4(m, a.y * expf(a.x - m) + b.y * expf(b.x - m), 0.f, 0.f);
  }
};
struct OpArgMax {  // (value, index bits): larger value, then lower index
  __device__ __forceinline__ float4 operator()(float4 a, float4 b) const {
    const int ia = __float_as_int(a.y), ib = __float_as_int(b.y);
    return (a.x > b.x || (a.x == b.x && ia < ib)) ? a : b;
  }
};
struct OpArgMin {  // (key, index bits): smaller key, then lower index
  __device__ __forceinline__ float4 operator()(float4 a, float4 b) const {
    const int ia = __float_as_int(a.y), ib = __float_as_int(b.y);
    return (a.x < b.x || (a.x == b.x && ia < ib)) ? a : b;
  }
};
struct OpSum {
  __device__ __forceinline__ float4 operator()(float4 a, float4 b) const {
    return make_float4(a.x + b.x, 0.f, 0.f, 0.f);
  }
};

struct AccShared {
  float4 slot[2];           // per-CTA partial exposed to the cluster (double buffered)
  float4 warp_part[kAccWarps];
  float4 bcast;
  int32_t child_start[65];
  int32_t child_list[64];
  int32_t acc_nodes[64];
  int32_t valid;
};

__device__ __forceinline__ float4 shfl_xor4(float4 v, int off) {
  v.x = __shfl_xor_sync(0xffffffffu, v.x, off);
  v.y = __shfl_xor_sync(0xffffffffu, v.y, off);
  return v;
}

// Block reduction, then cluster exchange in rank order; every thread of every CTA returns
// the same value.  Operators are commutative, so the butterfly leaves all lanes equal.
template <class Op>
__device__ __forceinline__ float4 cluster_reduce(AccShared& sh, float4 v, Op op, int& round,
                                                 uint32_t CL) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = op(v, shfl_xor4(v, off));
  if (lane == 0) sh.warp_part[warp] = v;
  __syncthreads();
  const int buf = round & 1;
  if (threadIdx.x == 0) {
    float4 t = sh.warp_part[0];
    for (int w = 1; w < kAccWarps; ++w) t = op(t, sh.warp_part[w]);
    sh.slot[buf] = t;
  }
  cluster_sync_all();
  if (warp == 0) {
    float4 mine = make_float4(0.f, 0.f, 0.f, 0.f);
    if (static_cast<uint32_t>(lane) < CL) mine = dsmem_ld_f4(dsmem_map(smem_u32(&sh.slot[buf]), lane));
    float4 t = make_float4(__shfl_sync(0xffffffffu, mine.x, 0), __shfl_sync(0xffffffffu, mine.y, 0),
                           0.f, 0.f);
    for (uint32_t r = 1; r < CL; ++r) {
      const float4 o = make_float4(__shfl_sync(0xffffffffu, mine.x, r),
                                   __shfl_sync(0xffffffffu, mine.y, r), 0.f, 0.f);
      t = op(t, o);
    }
    if (lane == 0) sh.bcast = t;
  }
  __syncthreads();
  ++round;
  return sh.bcast;
}

template <bool kVec4>
__device__ __forceinline__ float4 load4(const float* base, int v, int V) {
  if (kVec4) return *reinterpret_cast<const float4*>(base + v);
  float4 r;
  r.x = v < V ? base[v] : 0.f;
  r.y = v + 1 < V ? base[v + 1] : 0.f;
  r.z = v + 2 < V ? base[v + 2] : 0.f;
  r.w = v + 3 < V ? base[v + 3] : 0.f;
  return r;
}

template <bool kVec4>
__global__ void __launch_bounds__(kAccThreads) tree_accept_kernel(const AccParams prm) {
  __shared__ AccShared sh;
  extern __shared__ float acc_rbuf[];  // [2][slice]
  const uint32_t CL = cluster_nctarank();
  const uint32_t cr = cluster_ctarank();
  const int b = blockIdx.x / CL;
  const int N = prm.N, V = prm.V, slice = prm.slice;
  const int v_lo = static_cast<int>(cr) * slice;
  const int v_hi = min(V, v_lo + slice);
  const float T = prm.T;
  const size_t seq = static_cast<size_t>(b) * N;
  const int tid = threadIdx.x;

  if (tid == 0) {
    const int32_t* par = prm.parents + seq;
    const int32_t* tok = prm.tokens + seq;
    int ok = par[0] == -1;
    for (int i = 1; i < N; ++i) {
      const int p = par[i];
      if (p < 0 || p >= i) ok = 0;
      if (tok[i] < 0 || tok[i] >= V) ok = 0;
    }
    sh.valid = ok;
    if (ok) {  // children lists in ascending index (counting sort over parents)
      for (int i = 0; i <= N; ++i) sh.child_start[i] = 0;
      for (int i = 1; i < N; ++i) sh.child_start[par[i] + 1]++;
      for (int i = 0; i < N; ++i) sh.child_start[i + 1] += sh.child_start[i];
      int fill[64];
      for (int i = 0; i < N; ++i) fill[i] = sh.child_start[i];
      for (int i = 1; i < N; ++i) sh.child_list[fill[par[i]]++] = i;
    }
  }
  __syncthreads();
  if (!sh.valid) {
    if (cr == 0 && tid == 0) {
      for (int i = 0; i < N; ++i) prm.accepted_nodes[seq + i] = -1;
      prm.accept_len[b] = -1;
      prm.next_token[b] = -1;
    }
    return;  // every CTA of the cluster takes this branch; no shared memory was exchanged
  }

  float* rbuf0 = acc_rbuf;
  int round = 0;
  int cur = 0, nacc = 0, next = -1;
  for (int depth = 0; depth < N; ++depth) {
    const float* row = prm.logits + (seq + cur) * V;
    if (T == 0.f) {
      // greedy: argmax of the target logits, lowest index on ties
      float4 best = make_float4(-INFINITY, __int_as_float(INT_MAX), 0.f, 0.f);
      for (int v = v_lo + 4 * tid; v < v_hi; v += 4 * kAccThreads) {
        const float4 x = load4<kVec4>(row, v, V);
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (v + e < v_hi && xs[e] > best.x) best = make_float4(xs[e], __int_as_float(v + e), 0.f, 0.f);
      }
      const float4 r = cluster_reduce(sh, best, OpArgMax(), round, CL);
      int m = __float_as_int(r.y);
      if (m < 0 || m >= V) m = 0;  // all-NaN row
      int match = -1;
      for (int ci = sh.child_start[cur]; ci < sh.child_start[cur + 1]; ++ci) {
        const int c = sh.child_list[ci];
        if (prm.tokens[seq + c] == m) {
          match = c;
          break;
        }
      }
      if (match >= 0) {
        if (tid == 0) sh.acc_nodes[nacc] = match;
        ++nacc;
        cur = match;
        continue;
      }
      next = m;
      break;
    }

    // p = softmax(logits[cur] / T): row statistics (M, Z) of y = l / T
    float4 ms = make_float4(-INFINITY, 0.f, 0.f, 0.f);
    for (int v = v_lo + 4 * tid; v < v_hi; v += 4 * kAccThreads) {
      const float4 x = load4<kVec4>(row, v, V);
      const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (v + e >= v_hi) break;
        const float y = xs[e] / T;
        if (y > ms.x) {
          ms.y = ms.y * expf(ms.x - y) + 1.f;
          ms.x = y;
        } else {
          ms.y += expf(y - ms.x);
        }
      }
    }
    const float4 st = cluster_reduce(sh, ms, OpMaxSum(), round, CL);
    const float M = st.x, Z = st.y;

    bool has_res = false;
    int cb = 0;
    float Zr = 0.f;
    int accepted = -1;
    for (int ci = sh.child_start[cur]; ci < sh.child_start[cur + 1]; ++ci) {
      const int c = sh.child_list[ci];
      const int x = prm.tokens[seq + c];
      float px;
      if (has_res) {
        const int owner = x / slice;
        const uint32_t la = smem_u32(rbuf0 + cb * slice + (x - owner * slice));
        px = dsmem_ld_f32(dsmem_map(la, owner)) / Zr;
      } else {
        px = expf(row[x] / T - M) / Z;
      }
      const float* qrow = prm.draft + (seq + c) * V;
      const float qx = qrow[x];
      const float u = uniform_at(prm.seed, prm.offset, b, c, 0, 0);
      if (qx == 0.f || u < px / qx) {
        accepted = c;
        break;
      }
      // rejected: p <- norm(max(0, p - p_hat_c)); stored unnormalised with its mass
      const int nb = has_res ? (cb ^ 1) : cb;
      float* dst = rbuf0 + nb * slice;
      const float* src = rbuf0 + cb * slice;
      float part = 0.f;
      for (int v = v_lo + 4 * tid; v < v_hi; v += 4 * kAccThreads) {
        const float4 q4 = load4<kVec4>(qrow, v, V);
        float pv[4];
        if (has_res) {
#pragma unroll
          for (int e = 0; e < 4; ++e) pv[e] = src[v - v_lo + e] / Zr;
        } else {
          const float4 x4 = load4<kVec4>(row, v, V);
          pv[0] = expf(x4.x / T - M) / Z;
          pv[1] = expf(x4.y / T - M) / Z;
          pv[2] = expf(x4.z / T - M) / Z;
          pv[3] = expf(x4.w / T - M) / Z;
        }
        const float qs[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float r = (v + e < v_hi) ? fmaxf(pv[e] - qs[e], 0.f) : 0.f;
          dst[v - v_lo + e] = r;
          part += r;
        }
      }
      const float4 tot = cluster_reduce(sh, make_float4(part, 0.f, 0.f, 0.f), OpSum(), round, CL);
      if (tot.x > 0.f) {
        cb = nb;
        Zr = tot.x;
        has_res = true;
      }
    }
    if (accepted >= 0) {
      if (tid == 0) sh.acc_nodes[nacc] = accepted;
      ++nacc;
      cur = accepted;
      continue;
    }

    // no child accepted: exponential race over the current distribution,
    // key_v = ln(-ln u_v) - ln w_v with w = residual r or exp(y - M)
    float4 best = make_float4(INFINITY, __int_as_float(INT_MAX), 0.f, 0.f);
    const float* src = rbuf0 + cb * slice;
    for (int v = v_lo + 4 * tid; v < v_hi; v += 4 * kAccThreads) {
      const Philox4 rnd = philox_group(prm.seed, prm.offset, b, cur, 1, static_cast<uint32_t>(v) >> 2);
      float lw[4];
      if (has_res) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float r = src[v - v_lo + e];
          lw[e] = r > 0.f ? logf(r) : -INFINITY;
        }
      } else {
        const float4 x4 = load4<kVec4>(row, v, V);
        lw[0] = x4.x / T - M;
        lw[1] = x4.y / T - M;
        lw[2] = x4.z / T - M;
        lw[3] = x4.w / T - M;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (v + e >= v_hi || lw[e] == -INFINITY) continue;
        const float u = word_to_uniform(rnd.w[e]);
        const float key = logf(-logf(u)) - lw[e];
        if (key < best.x) best = make_float4(key, __int_as_float(v + e), 0.f, 0.f);
      }
    }
    const float4 r = cluster_reduce(sh, best, OpArgMin(), round, CL);
    next = __float_as_int(r.y);
    if (next < 0 || next >= V) next = 0;
    break;
  }

  if (cr == 0 && tid == 0) {
    for (int i = 0; i < N; ++i) prm.accepted_nodes[seq + i] = i < nacc ? sh.acc_nodes[i] : -1;
    prm.accept_len[b] = nacc;
    prm.next_token[b] = next;
  }
  // no CTA may leave while a peer can still read its shared memory
  cluster_sync_all();
}

}  // namespace eagle
