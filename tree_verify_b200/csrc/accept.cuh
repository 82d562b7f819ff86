// accept.cuh -- the accept / resample walk over the draft tree (EAGLE summary, section 2
// "Preliminaries": accept a drafted token t with probability min(1, p(t)/p_hat(t)); after
// a rejection discard the rest of that branch and resample; appendix A.2 "Multi-Round
// Speculative Sampling" and appendix B "Algorithm 1": the rule runs over the k candidates
// of a node with an adjusted distribution after each rejection).
//
// One thread-block cluster walks one sequence; the vocabulary is split into contiguous
// slices, one per CTA.  The walk is a chain of dependent decisions, so the kernel is built
// for latency:
//   - at each visited node the CTA's slice of the node's logits row and of the first
//     children's draft rows come into shared memory at once by bulk async copies (one
//     mbarrier per buffer); p_hat_c(t_c) and the accept uniforms are fetched or computed
//     in the same round trip, so each later pass over V reads shared memory; the root's
//     race keys (ln(-ln u_v)) are computed before the logits are awaited, those of every
//     later node while its first reduction waits for the peers;
//   - the root's draft rows are fetched before waiting for the LM-head grid (programmatic
//     dependent launch), so they arrive while the logits are still being produced;
//   - the residual r = max(0, p - p_hat) stays in the owners' shared memory (two buffers,
//     so that a zero-mass update can keep the previous one); the scalars the next accept
//     test needs (r[t], logits[t]) ride along with the reduction that precedes it;
//   - every reduction (max / sum-exp, argmax, sum, race argmin) is a warp butterfly, a
//     combine of the CTA's warps, and a push of the CTA's partial into every peer's shared
//     memory with a remote mbarrier arrival; each CTA then folds the CL partials with a
//     butterfly, so all CTAs reach bit-identical decisions without a cluster-wide barrier;
//     the max / sum-exp statistics combine in two passes at each level (the maximum, then
//     one exponential per partial and a sum), which keeps the dependent chain short.
// Only the accepted node indices, their count and the one extra token are written.
#pragma once

#include <limits.h>

#include "device_common.cuh"
#include "philox.cuh"

namespace eagle {

constexpr int kAccThreads = 512;
constexpr int kAccWarps = kAccThreads / 32;
constexpr int kAccMaxCluster = 16;
constexpr int kAccMaxQBuf = 4;
constexpr int kAccFixedBufs = 4;  // logits row, two residual buffers, race keys

struct AccParams {
  const float* logits;       // [B,N,V]
  const float* draft;        // [B,N,V]
  const int32_t* tokens;     // [B,N]
  const int32_t* parents;    // [B,N]
  int32_t* accepted_nodes;   // [B,N]
  int32_t* accept_len;       // [B]
  int32_t* next_token;       // [B]
  int32_t N, V, slice;       // slice: vocabulary entries per CTA, multiple of 4
  int32_t nq;                // draft-row prefetch buffers per CTA
  float T;
  uint64_t seed, offset;
};

// ---------------------------------------------------------------- reduction operators
// Payload float4.  Every operator is commutative bit for bit, so a butterfly leaves all
// lanes equal.  Components .y/.z/.w of OpSum (and .z of the max / sum-exp reduction) are
// "owner fields": exactly one CTA contributes a nonzero value (a scalar it alone holds in
// shared memory) and the others contribute 0, so adding them broadcasts that scalar
// exactly.
struct OpArgMax {  // (value, index bits): larger value, then lower index
  static __device__ __forceinline__ float4 identity() {
    return make_float4(-INFINITY, __int_as_float(INT_MAX), 0.f, 0.f);
  }
  __device__ __forceinline__ float4 operator()(float4 a, float4 b) const {
    const int ia = __float_as_int(a.y), ib = __float_as_int(b.y);
    return (a.x > b.x || (a.x == b.x && ia < ib)) ? a : b;
  }
};
struct OpArgMin {  // (key, index bits): smaller key, then lower index
  static __device__ __forceinline__ float4 identity() {
    return make_float4(INFINITY, __int_as_float(INT_MAX), 0.f, 0.f);
  }
  __device__ __forceinline__ float4 operator()(float4 a, float4 b) const {
    const int ia = __float_as_int(a.y), ib = __float_as_int(b.y);
    return (a.x < b.x || (a.x == b.x && ia < ib)) ? a : b;
  }
};
struct OpSum {  // (sum, owner fields)
  static __device__ __forceinline__ float4 identity() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ float4 operator()(float4 a, float4 b) const {
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
  }
};

// What a reduction is about, pushed beside its partial: (site << 24) | (node << 16) |
// (candidate << 8) | residual-in-use.  Every CTA folds all CL tags of a round, so if one
// CTA's control flow has left the others' (a decision taken differently), every CTA sees
// the mismatch in the same round and they all leave the walk together.
enum AccSite : uint32_t { kSiteArgMax = 1, kSiteMaxSum = 2, kSiteSum = 3, kSiteRace = 4 };
__device__ __forceinline__ uint32_t acc_tag(uint32_t site, int node, int cand, bool res) {
  return (site << 24) | (static_cast<uint32_t>(node) << 16) | (static_cast<uint32_t>(cand) << 8) |
         (res ? 1u : 0u);
}

struct AccShared {
  float4 wpart[kAccWarps];             // this CTA's warp partials
  float4 cslot[2][kAccMaxCluster];     // partial of CTA r, pushed by r (double buffered)
  uint2 ctag[2][kAccMaxCluster];       // (tag, failed-copy flag) of CTA r's push
  uint64_t cbar[2];                    // counts the CL pushes of a round
  uint64_t done_bar;                   // closing handshake: counts the CL "no more pushes"
  uint64_t row_bar;
  uint64_t q_bar[kAccMaxQBuf];
  int32_t par[64];
  int32_t tok[64];
  int32_t child_start[65];
  int32_t child_list[64];
  int32_t acc_nodes[64];
  float qx[64];                        // p_hat_c(t_c) of every drafted node c (T > 0)
  float ux[64];                        // node c's accept-test uniform (T > 0)
};

// Butterfly over lanes `offs..1` that moves only the first NC components (the ones the
// operator actually reduces); the other components stay this lane's own.
template <int NC, class Op>
__device__ __forceinline__ float4 warp_reduce_nc(float4 v, Op op, int offs) {
  for (int off = offs; off > 0; off >>= 1) {
    float4 o = Op::identity();
    o.x = __shfl_xor_sync(0xffffffffu, v.x, off);
    if (NC > 1) o.y = __shfl_xor_sync(0xffffffffu, v.y, off);
    v = op(v, o);
  }
  return v;
}

struct NoOwner {
  template <class Op>
  __device__ __forceinline__ float4 operator()(Op) const {
    return Op::identity();
  }
};
struct NoWork {
  __device__ __forceinline__ void operator()() const {}
};

// Cluster-wide reduction; every thread of every CTA returns the same bits.  NC components
// are reduced over all threads; `owner(op)` is evaluated by warp 0 after the CTA's threads
// have synchronised (so it may read what they wrote to shared memory) and folded into this
// CTA's partial.  Each CTA pushes its partial, its `tag` and whether any of its threads saw
// a copy fail (`failed`) into every peer's slot and arrives on the peer's barrier; `work()`
// runs while the peers' partials are on their way; then each warp folds the CL slots with
// a butterfly.  `bad` comes back set, the same in every thread of every CTA that got all
// CL pushes, when the CL tags differ or a CTA flagged a failed copy; it is also set in a
// CTA whose wait for the pushes gave up.
template <int NC, class Op, class Owner = NoOwner, class Work = NoWork>
__device__ __forceinline__ float4 cluster_reduce(AccShared& sh, float4 v, Op op, int& round,
                                                 uint32_t CL, uint32_t cr, uint32_t tag, int failed,
                                                 bool& bad, Owner owner = Owner(), Work work = Work()) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int buf = round & 1;
  v = warp_reduce_nc<NC>(v, op, 16);
  if (lane == 0) sh.wpart[warp] = v;
  const int any_failed = __syncthreads_or(failed);
  if (warp == 0) {
    float4 t = lane < kAccWarps ? sh.wpart[lane] : Op::identity();
    t = op(warp_reduce_nc<NC>(t, op, kAccWarps / 2), owner(op));
    if (static_cast<uint32_t>(lane) < CL) {
      dsmem_st_f4(dsmem_map(smem_u32(&sh.cslot[buf][cr]), lane), t);
      dsmem_st_u2(dsmem_map(smem_u32(&sh.ctag[buf][cr]), lane), make_uint2(tag, any_failed ? 1u : 0u));
      mbar_arrive_remote(dsmem_map(smem_u32(&sh.cbar[buf]), lane));
    }
  }
  work();
  const bool arrived = mbar_wait_cluster(smem_u32(&sh.cbar[buf]), (round >> 1) & 1, kErrAccClusterWait);
  // lane r folds CTA r's partial; a butterfly over all 32 lanes (all four components: the
  // owner fields ride along) leaves the same bits in every lane of every warp.  Every
  // thread must get the result: the walk's control flow is decided from it, and a thread
  // that decided differently would desynchronise the CTA's barriers.
  const int slot = static_cast<uint32_t>(lane) < CL ? lane : 0;
  float4 t = static_cast<uint32_t>(lane) < CL ? sh.cslot[buf][slot] : Op::identity();
  const uint2 tg = sh.ctag[buf][slot];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    float4 o;
    o.x = __shfl_xor_sync(0xffffffffu, t.x, off);
    o.y = __shfl_xor_sync(0xffffffffu, t.y, off);
    o.z = __shfl_xor_sync(0xffffffffu, t.z, off);
    o.w = __shfl_xor_sync(0xffffffffu, t.w, off);
    t = op(t, o);
  }
  const bool mismatch = __reduce_min_sync(0xffffffffu, tg.x) != __reduce_max_sync(0xffffffffu, tg.x);
  const bool flagged = __reduce_or_sync(0xffffffffu, tg.y) != 0u;
  if (mismatch && threadIdx.x == 0) record_error(kErrAccDiverged);
  // one verdict per CTA, so its threads keep to the same barriers
  bad = __syncthreads_or(!arrived || mismatch || flagged) != 0;
  ++round;
  return t;
}

// Cluster-wide (max y, sum exp(y - max)) of the row's statistics, with the same push /
// tag / wait protocol as cluster_reduce.  Each level combines in two passes -- the maximum
// by a butterfly, then every partial rescaled to it with one exponential and summed by a
// butterfly -- instead of merging pairs with two exponentials per step, so the dependent
// chain of exponentials is one per level.  Every thread of every CTA returns the same bits
// (fmaxf and fp32 addition are commutative bit for bit).  (m, s): this thread's partial,
// s taken relative to m.  `owner_z`: warp 0's contribution to the owner field .z.
template <class Work = NoWork>
__device__ __forceinline__ float4 cluster_maxsum(AccShared& sh, float m, float s, int& round, uint32_t CL,
                                                 uint32_t cr, uint32_t tag, int failed, bool& bad,
                                                 float owner_z, Work work = Work()) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int buf = round & 1;
  // warp: max, then rescale and sum
  float wm = m;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, off));
  float ws = wm == -INFINITY ? 0.f : s * __expf(m - wm);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, off);
  if (lane == 0) sh.wpart[warp] = make_float4(wm, ws, 0.f, 0.f);
  const int any_failed = __syncthreads_or(failed);
  if (warp == 0) {
    const float4 p = lane < kAccWarps ? sh.wpart[lane] : make_float4(-INFINITY, 0.f, 0.f, 0.f);
    float cm = p.x;
#pragma unroll
    for (int off = kAccWarps / 2; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
    float cs = cm == -INFINITY ? 0.f : p.y * __expf(p.x - cm);
#pragma unroll
    for (int off = kAccWarps / 2; off > 0; off >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, off);
    const float4 t = make_float4(cm, cs, owner_z, 0.f);
    if (static_cast<uint32_t>(lane) < CL) {
      dsmem_st_f4(dsmem_map(smem_u32(&sh.cslot[buf][cr]), lane), t);
      dsmem_st_u2(dsmem_map(smem_u32(&sh.ctag[buf][cr]), lane), make_uint2(tag, any_failed ? 1u : 0u));
      mbar_arrive_remote(dsmem_map(smem_u32(&sh.cbar[buf]), lane));
    }
  }
  work();
  const bool arrived = mbar_wait_cluster(smem_u32(&sh.cbar[buf]), (round >> 1) & 1, kErrAccClusterWait);
  const int slot = static_cast<uint32_t>(lane) < CL ? lane : 0;
  const float4 p = static_cast<uint32_t>(lane) < CL ? sh.cslot[buf][slot] : make_float4(-INFINITY, 0.f, 0.f, 0.f);
  const uint2 tg = sh.ctag[buf][slot];
  float M = p.x;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float Z = M == -INFINITY ? 0.f : p.y * __expf(p.x - M);
  float z = p.z, wv = p.w;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    Z += __shfl_xor_sync(0xffffffffu, Z, off);
    z += __shfl_xor_sync(0xffffffffu, z, off);
    wv += __shfl_xor_sync(0xffffffffu, wv, off);
  }
  const bool mismatch = __reduce_min_sync(0xffffffffu, tg.x) != __reduce_max_sync(0xffffffffu, tg.x);
  const bool flagged = __reduce_or_sync(0xffffffffu, tg.y) != 0u;
  if (mismatch && threadIdx.x == 0) record_error(kErrAccDiverged);
  bad = __syncthreads_or(!arrived || mismatch || flagged) != 0;
  ++round;
  return make_float4(M, Z, z, wv);
}

// Bulk async copy of `bytes` (multiple of 16, both ends 16-byte aligned) into shared memory,
// completing on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Fills buf[0 .. n) from src: one bulk copy (kBulk) or a cooperative copy.  With kBulk the
// caller waits on `bar` before reading; without it the copy is complete after the next
// wait_slice.
template <bool kBulk>
__device__ __forceinline__ void fetch_slice(float* buf, const float* src, int n, uint64_t* bar) {
  if (kBulk) {
    if (threadIdx.x == 0 && n > 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(smem_u32(bar), static_cast<uint32_t>(n) * 4u);
      bulk_g2s(smem_u32(buf), src, static_cast<uint32_t>(n) * 4u, smem_u32(bar));
    }
  } else {
    for (int i = threadIdx.x; i < n; i += kAccThreads) buf[i] = src[i];
  }
}

// Returns false if the wait gave up (the copy is then treated as failed).
template <bool kBulk>
__device__ __forceinline__ bool wait_slice(uint64_t* bar, uint32_t& phase, int n) {
  bool ok = true;
  if (kBulk) {
    if (n > 0) {
      ok = mbar_wait(smem_u32(bar), phase, kErrAccWait);
      phase ^= 1u;
    }
  } else {
    __syncthreads();
  }
  return ok;
}

// ln(-ln u_v) for tokens v .. v+3 of the race at `node` (v a multiple of 4).  The inner
// logarithm is the accurate one (for u near 1, -ln u is tiny and a fast logarithm's absolute
// error would be a large relative one); the outer one only needs a small absolute error.
__device__ __forceinline__ float4 race_keys(uint64_t seed, uint64_t offset, int b, int node, int v) {
  const Philox4 rnd = philox_group(seed, offset, b, node, 1, static_cast<uint32_t>(v) >> 2);
  return make_float4(__logf(-logf(word_to_uniform(rnd.w[0]))), __logf(-logf(word_to_uniform(rnd.w[1]))),
                     __logf(-logf(word_to_uniform(rnd.w[2]))), __logf(-logf(word_to_uniform(rnd.w[3]))));
}

template <bool kBulk>
__global__ void __launch_bounds__(kAccThreads, 1) tree_accept_kernel(const AccParams prm) {
  __shared__ AccShared sh;
  extern __shared__ __align__(16) float acc_dyn[];  // row | r0 | r1 | race keys | q[0..nq)
  const uint32_t CL = cluster_nctarank();
  const uint32_t cr = cluster_ctarank();
  const int b = blockIdx.x / CL;
  const int N = prm.N, V = prm.V, slice = prm.slice, NQ = prm.nq;
  const int v_lo = static_cast<int>(cr) * slice;
  const int n_loc = max(0, min(V, v_lo + slice) - v_lo);  // entries this CTA owns
  const float T = prm.T;
  const size_t seq = static_cast<size_t>(b) * N;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  float* rowbuf = acc_dyn;
  float* rbuf = acc_dyn + slice;          // [2][slice]
  float* ebuf = acc_dyn + 3 * slice;      // ln(-ln u_v) of one node's race
  float* qbuf = acc_dyn + 4 * slice;      // [NQ][slice]

  // ---- tree set-up (inputs only; runs while the LM-head grid may still be running)
  int ok = 1;
  if (tid < N) {
    const int p = prm.parents[seq + tid];
    const int t = prm.tokens[seq + tid];
    sh.par[tid] = p;
    sh.tok[tid] = t;
    ok = tid == 0 ? (p == -1) : (p >= 0 && p < tid && t >= 0 && t < V);
  }
  if (tid == 0) {
    mbar_init(smem_u32(&sh.cbar[0]), CL);
    mbar_init(smem_u32(&sh.cbar[1]), CL);
    mbar_init(smem_u32(&sh.done_bar), CL);
    mbar_init(smem_u32(&sh.row_bar), 1);
    for (int q = 0; q < kAccMaxQBuf; ++q) mbar_init(smem_u32(&sh.q_bar[q]), 1);
    fence_mbar_init();
  }
  ok = __syncthreads_and(ok);
  if (ok && T > 0.f && tid >= 1 && tid < N) {
    // what the accept test of node tid needs besides the target row: the draft probability
    // of its token in the row it was drafted from, and its uniform; loaded once here, before
    // the LM head has finished, rather than on the walk's path
    sh.qx[tid] = prm.draft[(seq + tid) * V + sh.tok[tid]];
    sh.ux[tid] = uniform_at(prm.seed, prm.offset, b, tid, 0, 0);
  }
  if (ok && tid <= N) {
    // start of node u's children list = number of drafted nodes whose parent is < u
    int start = 0;
    for (int i = 1; i < N; ++i) start += sh.par[i] < tid;
    sh.child_start[tid] = start;
  }
  __syncthreads();
  if (ok && tid >= 1 && tid < N) {
    // children in ascending index: earlier siblings come first
    const int p = sh.par[tid];
    int pos = sh.child_start[p];
    for (int j = 1; j < tid; ++j) pos += sh.par[j] == p;
    sh.child_list[pos] = tid;
  }
  // peers' barriers must be initialised before anyone pushes to them
  cluster_sync_all();
  if (!ok) {
    pdl_wait();
    if (cr == 0 && tid == 0) {
      for (int i = 0; i < N; ++i) prm.accepted_nodes[seq + i] = -1;
      prm.accept_len[b] = -1;
      prm.next_token[b] = -1;
    }
    return;  // every CTA of the cluster takes this branch; nothing was exchanged
  }

  uint32_t row_phase = 0, q_phase[kAccMaxQBuf] = {0u, 0u, 0u, 0u};
  // bulk copies issued and not yet waited for (bit q: draft buffer q; bit 4: the row);
  // the same in every thread, since every thread takes the same path
  uint32_t pending = 0;
  int failed = 0;     // a copy wait of this thread gave up
  bool bad = false;   // the last reduction says the cluster must stop
  bool done_sent = false;
  int round = 0;
  int cur = 0, nacc = 0, next = -1;
  const float invT = T > 0.f ? 1.0f / T : 0.f;
  // does this CTA own vocabulary entry x (and is x a real token)?
  auto owns = [&](int x) { return x >= v_lo && x < v_lo + n_loc; };
  auto wait_q = [&](int qb) {
    if (!kBulk || (pending >> qb) & 1u) failed |= !wait_slice<kBulk>(&sh.q_bar[qb], q_phase[qb], n_loc);
    pending &= ~(1u << qb);
  };
  // a buffer whose previous copy is still in flight (a prefetch for a candidate that was
  // never tested) is landed before it is refilled
  auto fetch_q = [&](int qb, int c) {
    if (kBulk && ((pending >> qb) & 1u)) wait_q(qb);
    fetch_slice<kBulk>(qbuf + qb * slice, prm.draft + (seq + c) * V + v_lo, n_loc, &sh.q_bar[qb]);
    if (kBulk && n_loc > 0) pending |= 1u << qb;
  };
  // this CTA will push nothing more: tell every peer (lane l of warp 0 made every push to
  // peer l, so its arrival also releases them)
  auto send_done = [&]() {
    if (warp == 0 && static_cast<uint32_t>(lane) < CL)
      mbar_arrive_remote(dsmem_map(smem_u32(&sh.done_bar), lane));
    done_sent = true;
  };

  // draft side of a node: the candidates' draft rows (their p_hat_c(t_c) and uniforms were
  // loaded for every node at set-up)
  auto issue_draft = [&](int node) {
    const int c_begin = sh.child_start[node];
    const int kids = sh.child_start[node + 1] - c_begin;
    const int pre = min(kids, NQ);
    // buffers still holding an untested candidate's copy: every thread sees it land before
    // one thread re-arms the barrier (a thread polling after the next phase completed would
    // otherwise wait for a phase that never comes)
    if (kBulk && (pending & ((1u << pre) - 1u))) {
      for (int j = 0; j < pre; ++j) wait_q(j);
      __syncthreads();
    }
    for (int j = 0; j < pre; ++j) fetch_q(j, sh.child_list[c_begin + j]);
  };
  // ebuf holds the race keys of node `ekey`: the root's, computed now (the walk most often
  // ends there), later those of each visited node, computed while its first reduction
  // waits for the peers; each thread keeps the keys of the entries it later races over
  int ekey = 0;
  auto fill_keys = [&](int node) {
    for (int i = 4 * tid; i < n_loc; i += 4 * kAccThreads)
      *reinterpret_cast<float4*>(ebuf + i) = race_keys(prm.seed, prm.offset, b, node, v_lo + i);
  };
  if (T > 0.f) {
    issue_draft(0);
    fill_keys(0);
  }

  // the logits come from the LM-head grid launched just before this one
  pdl_wait();
  // the kernel queued after this one (tree attention) does not read anything this walk
  // writes; let it fill the SMs the walk leaves idle
  pdl_launch_dependents();

  for (int depth = 0; depth < N; ++depth) {
    const float* row = prm.logits + (seq + cur) * V;
    const int c_begin = sh.child_start[cur], c_end = sh.child_start[cur + 1];
    const int kids = c_end - c_begin;
    // the row's copy first, so the draft side's loads overlap it
    fetch_slice<kBulk>(rowbuf, row + v_lo, n_loc, &sh.row_bar);
    if (depth > 0 && T > 0.f) issue_draft(cur);
    failed |= !wait_slice<kBulk>(&sh.row_bar, row_phase, n_loc);
    __syncthreads();  // the row slice is in shared memory for every thread

    if (T == 0.f) {
      // greedy: argmax of the target logits, lowest index on ties
      float4 best = OpArgMax::identity();
      for (int i = 4 * tid; i < n_loc; i += 4 * kAccThreads) {
        const float4 x = *reinterpret_cast<const float4*>(rowbuf + i);
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (i + e < n_loc && xs[e] > best.x)
            best = make_float4(xs[e], __int_as_float(v_lo + i + e), 0.f, 0.f);
      }
      const float4 r = cluster_reduce<2>(sh, best, OpArgMax(), round, CL, cr,
                                         acc_tag(kSiteArgMax, cur, 0, false), failed, bad);
      if (bad) break;
      int m = __float_as_int(r.y);
      if (m < 0 || m >= V) m = 0;  // all-NaN row
      int match = -1;
      for (int ci = c_begin; ci < c_end; ++ci) {
        const int c = sh.child_list[ci];
        if (sh.tok[c] == m) {
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

    // p = softmax(logits[cur] / T): statistics (M, Z) of y = l / T, in two passes over the
    // slice (the maximum, then the exponentials: independent operations, no chain); the
    // owner of the first candidate's token also broadcasts its logit
    const int x0 = kids > 0 ? sh.tok[sh.child_list[c_begin]] : -1;
    float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    for (int i = 4 * tid; i < n_loc; i += 4 * kAccThreads) {
      const float4 x = *reinterpret_cast<const float4*>(rowbuf + i);
      mq[0] = fmaxf(mq[0], x.x);
      if (i + 1 < n_loc) mq[1] = fmaxf(mq[1], x.y);
      if (i + 2 < n_loc) mq[2] = fmaxf(mq[2], x.z);
      if (i + 3 < n_loc) mq[3] = fmaxf(mq[3], x.w);
    }
    const float mt = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * invT;
    float sq[4] = {0.f, 0.f, 0.f, 0.f};
    if (mt != -INFINITY) {
      for (int i = 4 * tid; i < n_loc; i += 4 * kAccThreads) {
        const float4 x = *reinterpret_cast<const float4*>(rowbuf + i);
        sq[0] += __expf(x.x * invT - mt);
        if (i + 1 < n_loc) sq[1] += __expf(x.y * invT - mt);
        if (i + 2 < n_loc) sq[2] += __expf(x.z * invT - mt);
        if (i + 3 < n_loc) sq[3] += __expf(x.w * invT - mt);
      }
    }
    const float st_own = owns(x0) ? rowbuf[x0 - v_lo] : 0.f;
    const bool new_keys = ekey != cur;
    const float4 st = cluster_maxsum(sh, mt, (sq[0] + sq[1]) + (sq[2] + sq[3]), round, CL, cr,
                                     acc_tag(kSiteMaxSum, cur, 0, false), failed, bad, st_own, [&]() {
                                       // this node's race keys, in case the walk ends here
                                       if (new_keys) fill_keys(cur);
                                     });
    ekey = cur;
    if (bad) break;
    const float M = st.x, invZ = 1.0f / st.y;
    float px_next = __expf(st.z * invT - M) * invZ;  // p at the first candidate's token

    bool has_res = false;
    int cb = 0;
    float invZr = 0.f;
    int j_acc = -1;
    for (int j = 0; j < kids; ++j) {
      const int c = sh.child_list[c_begin + j];
      const float px = px_next;
      const float qx = sh.qx[c];
      if (qx == 0.f || sh.ux[c] < px / qx) {
        j_acc = j;
        break;
      }
      // rejected: p <- norm(max(0, p - p_hat_c)); stored unnormalised with its mass
      const int qb = j % NQ;
      float* q = qbuf + qb * slice;
      if (!kBulk && j >= NQ) fetch_q(qb, c);
      wait_q(qb);
      const int nb = has_res ? (cb ^ 1) : cb;
      float* dst = rbuf + nb * slice;
      const float* src = rbuf + cb * slice;
      float part = 0.f;
      for (int i = 4 * tid; i < n_loc; i += 4 * kAccThreads) {
        const float4 q4 = *reinterpret_cast<const float4*>(q + i);
        float4 p4;
        if (has_res) {
          const float4 s4 = *reinterpret_cast<const float4*>(src + i);
          p4 = make_float4(s4.x * invZr, s4.y * invZr, s4.z * invZr, s4.w * invZr);
        } else {
          const float4 x4 = *reinterpret_cast<const float4*>(rowbuf + i);
          p4 = make_float4(__expf(x4.x * invT - M) * invZ, __expf(x4.y * invT - M) * invZ,
                           __expf(x4.z * invT - M) * invZ, __expf(x4.w * invT - M) * invZ);
        }
        float4 r4 = make_float4(fmaxf(p4.x - q4.x, 0.f), fmaxf(p4.y - q4.y, 0.f),
                                fmaxf(p4.z - q4.z, 0.f), fmaxf(p4.w - q4.w, 0.f));
        if (i + 1 >= n_loc) r4.y = 0.f;
        if (i + 2 >= n_loc) r4.z = 0.f;
        if (i + 3 >= n_loc) r4.w = 0.f;
        *reinterpret_cast<float4*>(dst + i) = r4;
        part += (r4.x + r4.y) + (r4.z + r4.w);
      }
      // the owner of the next candidate's token broadcasts what its accept test may need:
      // the new residual there, the previous one, and the logit
      const int xn = j + 1 < kids ? sh.tok[sh.child_list[c_begin + j + 1]] : -1;
      const float4 tot = cluster_reduce<1>(sh, make_float4(part, 0.f, 0.f, 0.f), OpSum(), round, CL, cr,
                                           acc_tag(kSiteSum, cur, j, has_res), failed, bad,
                                           [&](OpSum) {
                                             float4 o = OpSum::identity();
                                             if (owns(xn)) {
                                               o.y = dst[xn - v_lo];
                                               o.z = has_res ? src[xn - v_lo] : 0.f;
                                               o.w = rowbuf[xn - v_lo];
                                             }
                                             return o;
                                           });
      if (bad) break;
      if (tot.x > 0.f) {
        cb = nb;
        invZr = 1.0f / tot.x;
        has_res = true;
        px_next = tot.y * invZr;
      } else {
        // zero residual mass: p is kept
        px_next = has_res ? tot.z * invZr : __expf(tot.w * invT - M) * invZ;
      }
      // every thread of this CTA is past its reads of buffer qb (the reduction above
      // synchronised the CTA): refill it with a later candidate's row
      if (kBulk && j + NQ < kids) fetch_q(qb, sh.child_list[c_begin + j + NQ]);
    }
    if (bad) break;
    if (j_acc >= 0) {
      const int c = sh.child_list[c_begin + j_acc];
      if (tid == 0) sh.acc_nodes[nacc] = c;
      ++nacc;
      // candidates [j_acc, j_acc + NQ) may still have draft-row copies in flight: they stay
      // pending until their buffers are refilled (or the walk ends), so the next node's
      // row request does not wait for them
      __syncthreads();
      cur = c;
      continue;
    }

    // no child accepted: exponential race over the current distribution,
    // key_v = ln(-ln u_v) - ln w_v with w = residual r or exp(y - M)
    float4 best = OpArgMin::identity();
    const float* src = rbuf + cb * slice;
    for (int i = 4 * tid; i < n_loc; i += 4 * kAccThreads) {
      const float4 e4 = *reinterpret_cast<const float4*>(ebuf + i);  // keys of node cur
      const float es[4] = {e4.x, e4.y, e4.z, e4.w};
      float lw[4];
      if (has_res) {
        const float4 s4 = *reinterpret_cast<const float4*>(src + i);
        lw[0] = s4.x > 0.f ? __logf(s4.x) : -INFINITY;
        lw[1] = s4.y > 0.f ? __logf(s4.y) : -INFINITY;
        lw[2] = s4.z > 0.f ? __logf(s4.z) : -INFINITY;
        lw[3] = s4.w > 0.f ? __logf(s4.w) : -INFINITY;
      } else {
        const float4 x4 = *reinterpret_cast<const float4*>(rowbuf + i);
        lw[0] = x4.x * invT - M;
        lw[1] = x4.y * invT - M;
        lw[2] = x4.z * invT - M;
        lw[3] = x4.w * invT - M;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (i + e >= n_loc || lw[e] == -INFINITY) continue;
        const float key = es[e] - lw[e];
        if (key < best.x) best = make_float4(key, __int_as_float(v_lo + i + e), 0.f, 0.f);
      }
    }
    // the race ends every walk at T > 0: this CTA's push is its last, so it announces that
    // while the peers' partials are on their way
    const float4 r = cluster_reduce<2>(sh, best, OpArgMin(), round, CL, cr,
                                       acc_tag(kSiteRace, cur, 0, has_res), failed, bad, NoOwner(),
                                       send_done);
    if (bad) break;
    next = __float_as_int(r.y);
    if (next < 0 || next >= V) next = 0;
    break;
  }

  if (cr == 0 && tid == 0) {
    // a walk the cluster stopped (its CTAs disagreed, or a wait gave up) reports like an
    // invalid tree; the device error word says why
    for (int i = 0; i < N; ++i) prm.accepted_nodes[seq + i] = (!bad && i < nacc) ? sh.acc_nodes[i] : -1;
    prm.accept_len[b] = bad ? -1 : nacc;
    prm.next_token[b] = bad ? -1 : next;
  }
  // Closing handshake.  A CTA leaves only once every peer has said it will push nothing
  // more, so no push can reach the shared memory of a CTA that has exited, even if the
  // cluster's control flow split (the tags make every CTA stop in the round after a split;
  // a CTA that stopped on its own waits here for the others' rounds to give up).  The wait
  // is twice as long as a reduction's, so a peer that timed out in its round still arrives
  // in time.  Copies this CTA issued and did not consume land first.
  if (!done_sent) send_done();
  for (int qb = 0; qb < kAccMaxQBuf; ++qb)
    if ((pending >> qb) & 1u) wait_q(qb);
  if (tid == 0) mbar_wait_cluster(smem_u32(&sh.done_bar), 0, kErrAccClusterWait, 2 * kWaitLimitNs);
}

}  // namespace eagle
