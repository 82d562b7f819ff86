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
// A row is split over a thread-block cluster of S <= 16 CTAs (S = 1 when there are enough
// rows to fill the GPU), CTA s owning the vocabulary slice [s*W, (s+1)*W) with W a multiple
// of 4 (one Philox group per 4 entries).  Each CTA pushes its slice's (max, sum exp) into
// every peer's shared memory; after a hardware cluster barrier every CTA holds the row's
// (M, Z).  Then, over its slice:
//   T == 0: one pass keeps each thread's 16 best (logit desc, index asc) in registers; k
//           rounds of warp argmax merge a warp's lists, then warp 0 merges the warps';
//   T  > 0: race j keeps each thread's smallest key ln(-ln u) - (y - M), starting from the
//           key of the slice's most probable entry; an entry whose 1 - u (a lower bound of
//           -ln u) already puts its key above the thread's best skips the two logarithms,
//           so for a peaked distribution nearly every entry costs one Philox word and one
//           approximate exponential; warp minima per race, then warp 0 takes each race's
//           minimum over the warps.
// Each CTA pushes its k winners to CTA 0, which after a second barrier merges them into the
// row's k children.  Control flow is the same in every CTA, so both barriers are reached
// by all of them and no CTA reads a peer after the second one.  Bound by issued
// instructions (the Philox words at T > 0).
#pragma once

#include <limits.h>

#include "device_common.cuh"
#include "philox.cuh"

namespace eagle {

constexpr int kDraftThreads = 512;
constexpr int kDraftWarps = kDraftThreads / 32;
constexpr int kDraftMaxK = 16;
constexpr int kDraftMaxCluster = 16;      // 16 needs the non-portable cluster size
constexpr int kDraftPortableCluster = 8;
constexpr size_t kDraftMaxSmem = 192 * 1024;  // a CTA's staged slice: V <= 8 * 49152

struct DraftParams {
  const float* logits;  // [R, V], R = B * F
  int32_t* tokens;      // [R, k]
  float* conf;          // [R, k]
  float* probs;         // [R, V] or null
  int32_t F, V, k;
  int32_t slice;        // entries per CTA of a row's cluster, a multiple of 4
  int32_t vec16;        // every row starts 16-byte aligned (V % 4 == 0, aligned logits)
  float T;
  uint64_t seed, offset;
};

struct DraftShared {
  float sval[kDraftWarps];
  int sidx[kDraftWarps];
  float2 stats[kDraftMaxCluster];             // (max y, sum exp(y - max)) of CTA s's slice
  float key0[kDraftMaxK];                      // race j's key at the slice's most probable entry
  float warp_v[kDraftWarps][kDraftMaxK];       // warp w's j-th winner in this CTA
  int warp_i[kDraftWarps][kDraftMaxK];
  float best_v[kDraftMaxCluster][kDraftMaxK];  // CTA 0 only: CTA s's j-th winner
  int best_i[kDraftMaxCluster][kDraftMaxK];
};

// (value, index) pairs: `better` is larger value, then lower index (argmax); the race uses
// smaller key, then lower index, passed in as the negated key.
__device__ __forceinline__ bool draft_better(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

// Warp-wide argmax of (value, index); every lane returns the winner.  `draft_better` is a
// strict total order on the pairs that reach it (no NaN values), so all lanes agree.
__device__ __forceinline__ void draft_warp_argmax(float& val, int& idx) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, val, off);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
    if (draft_better(ov, oi, val, idx)) {
      val = ov;
      idx = oi;
    }
  }
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

// Asynchronous global -> shared copies (every thread's copies in flight at once).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void dsmem_st_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void dsmem_st_s32(uint32_t addr, int v) {
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Kernel modes: the top k logits (T == 0), k independent races (T > 0, siblings drawn with
// replacement), the k smallest keys of one race (T > 0, siblings drawn without replacement).
constexpr int kDraftTopK = 0;
constexpr int kDraftRaces = 1;
constexpr int kDraftDistinct = 2;

// Inserts (cv, ci) into a thread's list of its 16 best entries, sorted by draft_better.
__device__ __forceinline__ void draft_list_insert(float (&lv)[kDraftMaxK], int (&li)[kDraftMaxK], float cv,
                                                  int ci) {
  if (!draft_better(cv, ci, lv[kDraftMaxK - 1], li[kDraftMaxK - 1])) return;
#pragma unroll
  for (int s = 0; s < kDraftMaxK; ++s)
    if (draft_better(cv, ci, lv[s], li[s])) {  // carry the displaced entry down
      const float tv = lv[s];
      const int ti = li[s];
      lv[s] = cv;
      li[s] = ci;
      cv = tv;
      ci = ti;
    }
}

template <int kMode>
__global__ void __launch_bounds__(kDraftThreads) draft_select_kernel(const DraftParams p) {
  constexpr bool kGreedy = kMode == kDraftTopK;
  constexpr bool kList = kMode != kDraftRaces;  // winners from per-thread sorted lists
  __shared__ DraftShared sh;
  const uint32_t S = cluster_nctarank();
  const uint32_t cr = cluster_ctarank();
  const int r = static_cast<int>(blockIdx.x / S);
  const int b = r / p.F, f = r % p.F;
  const int V = p.V, k = p.k;
  const int v_lo = static_cast<int>(cr) * p.slice;
  const int v_hi = min(V, v_lo + p.slice);  // v_lo >= v_hi: an empty slice
  const float* row = p.logits + static_cast<size_t>(r) * V;
  const float invT = kGreedy ? 1.0f : 1.0f / p.T;
  const int tid = threadIdx.x;

  // the slice, staged in shared memory once (16-byte copies when rows start 16-byte aligned)
  extern __shared__ __align__(16) float xs[];
  const int n = max(0, v_hi - v_lo);
  if (p.vec16) {
    for (int i = 4 * tid; i < n; i += 4 * kDraftThreads) cp_async16(xs + i, row + v_lo + i);
  } else {
    for (int i = tid; i < n; i += kDraftThreads) cp_async4(xs + i, row + v_lo + i);
  }
  cp_async_wait_all();
  __syncthreads();

  // softmax statistics of y = logit * invT over this slice, then over the row
  float m = -INFINITY;
  int mi = INT_MAX;  // the slice's most probable entry (lowest index among ties)
  for (int i = tid; i < n; i += kDraftThreads) {
    const float y = xs[i] * invT;
    if (y > m) {
      m = y;
      mi = i;
    }
  }
  draft_block_argmax(m, mi, sh.sval, sh.sidx);
  float z = 0.f;
  if (m != -INFINITY)
    for (int i = tid; i < n; i += kDraftThreads) z += expf(xs[i] * invT - m);
  z = draft_block_sum(z, sh.sval);
  if (static_cast<uint32_t>(tid) < S)
    dsmem_st_f2(dsmem_map(smem_u32(&sh.stats[cr]), static_cast<uint32_t>(tid)), make_float2(m, z));
  cluster_sync_all();
  float M = -INFINITY;
  for (uint32_t s = 0; s < S; ++s) M = fmaxf(M, sh.stats[s].x);
  float Z = 0.f;
  for (uint32_t s = 0; s < S; ++s)
    if (sh.stats[s].x != -INFINITY) Z += sh.stats[s].y * expf(sh.stats[s].x - M);
  const float invZ = Z > 0.f ? 1.0f / Z : 0.f;

  // the distribution, and at T > 0 the slice rewritten in place as lw = y - M for the races
  float* out = p.probs == nullptr ? nullptr : p.probs + static_cast<size_t>(r) * V + v_lo;
  for (int i = tid; i < n; i += kDraftThreads) {
    const float lw = xs[i] * invT - M;
    if (!kGreedy) xs[i] = lw;
    if (out != nullptr) out[i] = expf(lw) * invZ;
  }
  if (!kGreedy) __syncthreads();  // the races read other threads' entries

  // this slice's k winners (index INT_MAX: none), pushed to CTA 0
  const int lane = tid & 31, warp = tid >> 5;
  const uint32_t to0_v = dsmem_map(smem_u32(&sh.best_v[cr][0]), 0);
  const uint32_t to0_i = dsmem_map(smem_u32(&sh.best_i[cr][0]), 0);
  if (kList) {
    // each thread's 16 best entries, sorted; NaN never enters (draft_better is false).  The
    // value is the logit (top k) or the negated race key (without replacement: the k
    // smallest keys of one race, purpose 2, are successive draws)
    float lv[kDraftMaxK];
    int li[kDraftMaxK];
#pragma unroll
    for (int s = 0; s < kDraftMaxK; ++s) {
      lv[s] = -INFINITY;
      li[s] = INT_MAX;
    }
    if (kGreedy) {
      for (int i = tid; i < n; i += kDraftThreads) draft_list_insert(lv, li, xs[i], v_lo + i);
    } else {
      for (int i0 = 4 * tid; i0 < n; i0 += 4 * kDraftThreads) {
        const Philox4 u = philox_group(p.seed, p.offset, static_cast<uint32_t>(b), static_cast<uint32_t>(f),
                                       2u, static_cast<uint32_t>(v_lo + i0) >> 2);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (i0 + e >= n) break;
          const float lw = xs[i0 + e];
          if (lw == -INFINITY) continue;
          draft_list_insert(lv, li, lw - logf(-logf(word_to_uniform(u.w[e]))), v_lo + i0 + e);
        }
      }
    }
    // the warp's k best: k rounds of a warp argmax over the lists' heads
    for (int j = 0; j < k; ++j) {
      float wv = lv[0];
      int wi = li[0];
      draft_warp_argmax(wv, wi);
      if (li[0] == wi) {  // indices are unique, so one lane (or, once all are spent, none)
#pragma unroll
        for (int s = 0; s + 1 < kDraftMaxK; ++s) {
          lv[s] = lv[s + 1];
          li[s] = li[s + 1];
        }
        lv[kDraftMaxK - 1] = -INFINITY;
        li[kDraftMaxK - 1] = INT_MAX;
      }
      if (lane == 0) {
        sh.warp_v[warp][j] = wv;
        sh.warp_i[warp][j] = wi;
      }
    }
    __syncthreads();
    if (warp == 0) {
      // the CTA's k best: lane w walks warp w's list
      int h = 0;
      for (int j = 0; j < k; ++j) {
        const bool live = lane < kDraftWarps && h < k;
        float cv = live ? sh.warp_v[lane][h] : -INFINITY;
        int ci = live ? sh.warp_i[lane][h] : INT_MAX;
        const int mine = ci;
        draft_warp_argmax(cv, ci);
        if (live && mine == ci && ci != INT_MAX) ++h;
        if (lane == 0) {
          dsmem_st_f32(to0_v + 4u * j, cv);
          dsmem_st_s32(to0_i + 4u * j, ci);
        }
      }
    }
  } else {
    // Every thread's race j starts from the key of the slice's most probable entry: a key
    // the slice's minimum cannot exceed, and for a peaked distribution one that nearly every
    // other entry's bound below already beats, so whole warps skip the logarithms.
    if (tid < k)
      sh.key0[tid] = mi == INT_MAX ? INFINITY
                                   : logf(-logf(uniform_at(p.seed, p.offset, static_cast<uint32_t>(b),
                                                           static_cast<uint32_t>(f),
                                                           static_cast<uint32_t>(v_lo + mi),
                                                           static_cast<uint32_t>(2 + tid)))) -
                                         xs[mi];
    __syncthreads();
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
      // the smallest key = ln(-ln u) - (y - M) over the thread's entries and the slice's
      // most probable one, ties to the lower index
      float key = sh.key0[j];
      int arg = mi == INT_MAX ? INT_MAX : v_lo + mi;
#pragma unroll 2
      for (int i0 = 4 * tid; i0 < n; i0 += 4 * kDraftThreads) {
        const int v0 = v_lo + i0;
        const Philox4 u = philox_group(p.seed, p.offset, static_cast<uint32_t>(b),
                                       static_cast<uint32_t>(f), static_cast<uint32_t>(2 + j),
                                       static_cast<uint32_t>(v0) >> 2);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (i0 + e >= n) break;
          const float lw = xs[i0 + e];
          if (lw == -INFINITY) continue;
          const float ue = word_to_uniform(u.w[e]);
          // -ln u >= 1 - u (exact in float: u is a multiple of 2^-24).  If 1 - u is at least
          // exp(key + lw) with a margin well above the rounding of key + lw, of the
          // approximate exponential and of the key below, this entry's key is above `key`.
          const float bound = __expf(key + lw + 1e-4f + 2.5e-7f * (fabsf(key) + fabsf(lw)));
          if (1.0f - ue >= bound) continue;
          const float kk = logf(-logf(ue)) - lw;
          if (kk < key || (kk == key && v0 + e < arg)) {
            key = kk;
            arg = v0 + e;
          }
        }
      }
      float nk = -key;  // argmin of the key = argmax of its negation, lower index on ties
      draft_warp_argmax(nk, arg);
      if (lane == 0) {
        sh.warp_v[warp][j] = nk;
        sh.warp_i[warp][j] = arg;
      }
    }
    __syncthreads();
    if (warp == 0 && lane < k) {
      // race `lane`: the smallest key over the warps
      float cv = -INFINITY;
      int ci = INT_MAX;
      for (int w = 0; w < kDraftWarps; ++w)
        if (draft_better(sh.warp_v[w][lane], sh.warp_i[w][lane], cv, ci)) {
          cv = sh.warp_v[w][lane];
          ci = sh.warp_i[w][lane];
        }
      dsmem_st_f32(to0_v + 4u * lane, cv);
      dsmem_st_s32(to0_i + 4u * lane, ci);
    }
  }
  cluster_sync_all();  // the last access to another CTA's shared memory is above
  if (cr != 0 || warp != 0) return;

  // CTA 0, warp 0: the row's k children; lane j writes child j
  int pick = INT_MAX;
  if (kList) {
    int h = 0;  // lane s walks CTA s's list
    for (int j = 0; j < k; ++j) {
      const bool live = static_cast<uint32_t>(lane) < S && h < k;
      float cv = live ? sh.best_v[lane][h] : -INFINITY;
      int ci = live ? sh.best_i[lane][h] : INT_MAX;
      const int mine = ci;
      draft_warp_argmax(cv, ci);
      if (live && mine == ci && ci != INT_MAX) ++h;
      if (lane == j) pick = ci;
    }
  } else if (lane < k) {
    float cv = -INFINITY;
    for (uint32_t s = 0; s < S; ++s)
      if (draft_better(sh.best_v[s][lane], sh.best_i[s][lane], cv, pick)) {
        cv = sh.best_v[s][lane];
        pick = sh.best_i[s][lane];
      }
  }
  if (lane < k) {
    const bool found = pick != INT_MAX;
    p.tokens[static_cast<size_t>(r) * k + lane] = found ? pick : -1;
    p.conf[static_cast<size_t>(r) * k + lane] = found ? expf(row[pick] * invT - M) * invZ : 0.f;
  }
}

// The row each sibling was drawn from, for siblings drawn without replacement: child j of
// row r was drawn from p_r with tokens[r][0 .. j-1] removed, so its row is p_r over the rest,
// renormalised by the remaining mass R_j summed directly over the kept entries (not 1 minus
// the removed mass, which cancels when the earlier siblings carry most of it).
//
// A row is split over a cluster of C <= 8 CTAs, CTA c owning entries [c*W, (c+1)*W).  Each
// entry v has a position pos(v) = i if v is sibling i's token, else k: it stays in rows
// j <= pos(v).  Each CTA sums its entries into the k partial masses, pushes them into every
// peer's shared memory, and after one hardware cluster barrier every CTA holds R_0..R_{k-1}
// and writes its chunk of all k rows.  A token -1 (or out of range) before sibling j leaves
// rows j.. all zeros.
constexpr int kChildThreads = 512;
constexpr int kChildMaxCluster = 8;

struct ChildParams {
  const float* probs;     // [R, V]
  const int32_t* tokens;  // [R, k]
  float* child;           // [R, k, V]
  int32_t V, k, chunk;    // chunk: entries per CTA
};

__global__ void __launch_bounds__(kChildThreads) draft_child_rows_kernel(const ChildParams p) {
  __shared__ int32_t tok[kDraftMaxK];
  __shared__ float red[kChildThreads / 32][kDraftMaxK];
  __shared__ float part[kChildMaxCluster][kDraftMaxK];  // CTA c's partial masses, pushed by c
  const uint32_t C = cluster_nctarank();
  const uint32_t cr = cluster_ctarank();
  const int r = static_cast<int>(blockIdx.x / C);
  const int V = p.V, k = p.k, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  if (tid < k) tok[tid] = p.tokens[static_cast<size_t>(r) * k + tid];
  __syncthreads();
  int live = k;  // rows j < live are defined: no -1 / out-of-range token before them
  for (int i = 0; i < k; ++i)
    if (tok[i] < 0 || tok[i] >= V) {
      live = i + 1;  // row i itself is still defined (its earlier tokens are valid)
      break;
    }
  const int v_lo = static_cast<int>(cr) * p.chunk;
  const int v_hi = min(V, v_lo + p.chunk);
  const float* row = p.probs + static_cast<size_t>(r) * V;
  auto pos_of = [&](int v) {
    int q = k;
    for (int i = 0; i < k; ++i)
      if (tok[i] == v) {
        q = i;
        break;
      }
    return q;
  };

  // this chunk's partial masses: entry v counts in rows j <= pos(v)
  float acc[kDraftMaxK];
#pragma unroll
  for (int j = 0; j < kDraftMaxK; ++j) acc[j] = 0.f;
  for (int v = v_lo + tid; v < v_hi; v += kChildThreads) {
    const float x = row[v];
    const int q = pos_of(v);
#pragma unroll
    for (int j = 0; j < kDraftMaxK; ++j)
      if (j <= q) acc[j] += x;
  }
#pragma unroll
  for (int j = 0; j < kDraftMaxK; ++j) {
    float t = acc[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (lane == 0) red[warp][j] = t;
  }
  __syncthreads();
  if (tid < k) {
    float t = 0.f;
    for (int w = 0; w < kChildThreads / 32; ++w) t += red[w][tid];
    for (uint32_t c = 0; c < C; ++c) dsmem_st_f32(dsmem_map(smem_u32(&part[cr][tid]), c), t);
  }
  cluster_sync_all();  // the only exchange: no CTA reads a peer afterwards

  float inv[kDraftMaxK];
#pragma unroll
  for (int j = 0; j < kDraftMaxK; ++j) {
    float R = 0.f;
    if (j < k)
      for (uint32_t c = 0; c < C; ++c) R += part[c][j];
    inv[j] = (j < live && R > 0.f) ? 1.0f / R : 0.f;
  }
  float* out = p.child + static_cast<size_t>(r) * k * V;
  for (int v = v_lo + tid; v < v_hi; v += kChildThreads) {
    const float x = row[v];
    const int q = pos_of(v);
#pragma unroll
    for (int j = 0; j < kDraftMaxK; ++j)
      if (j < k) out[static_cast<size_t>(j) * V + v] = (inv[j] == 0.f || q < j) ? 0.f : x * inv[j];
  }
}

}  // namespace eagle
