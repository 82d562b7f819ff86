// attention.cuh -- tree attention for the verification pass (EAGLE summary, section 3
// "Drafting and verification": the target verifies the tree-structured draft in a single
// forward pass using tree attention; appendix A.1 "Tree Structure").
//
// For sequence b, node i, query head h (kv head g = h / G):
//     out[b,i,h] = sum_j softmax_j(scale * q[b,i,h] . k_j) v_j
// over the prefix positions 0 .. L_b-1 of kv head g and the tree nodes on the path from
// i to the root (i included).
//
// bf16 path (decode-style, split-KV over the prefix): one CTA owns one (sequence, kv head,
// block of 64 query rows, prefix split).  The query rows of a kv head are the G heads x N
// nodes that share it (row r -> node r / G, head g*G + r % G), so every prefix K/V tile is
// brought from HBM into shared memory once by TMA (128-byte swizzled boxes) and used by
// all of them.  A producer warp streams 64-key K/V tiles through a multi-stage mbarrier
// ring (a split's tiles are all in flight at once); four consumer warps each own 16 query
// rows and run S = Q K^T and O += P V with warp-level bf16 MMAs and an online softmax kept
// in registers (quad shuffles for the row max).  The CTA of the last split also runs the
// tree tile: the N tree keys, masked by the per-node ancestor bitmask (node i and every
// node up its parent chain) built in shared memory.  Splits write (m, l, acc) partials
// that a second kernel merges by log-sum-exp; with a single split the CTA normalises and
// writes the output itself.
//
// f32 path: one warp per output row, fp32 SIMT, keys streamed in order (small shapes).
#pragma once

#include "device_common.cuh"

namespace eagle {

constexpr int kAttnKeys = 64;        // keys per tile
constexpr int kAttnRows = 64;        // query rows per CTA (4 consumer warps x 16)
constexpr int kAttnConsumerWarps = 4;
constexpr int kAttnThreads = 32 * (kAttnConsumerWarps + 1);

// K/V ring depth: the kernel's registers allow one CTA per SM, so the ring takes most of
// the shared memory and a split's tiles are all in flight at once.
template <int D>
constexpr int attn_stages() {
  return D == 128 ? 4 : 8;
}

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

// Byte offset of element (row, d) in a 64-row tile stored as D/64 boxes of [64][64] bf16
// with the 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t attn_swz(int row, int d) {
  const int half = d >> 6;
  const int chunk = (d & 63) >> 3;
  return static_cast<uint32_t>(half * (kAttnKeys * 128) + row * 128 + ((chunk ^ (row & 7)) << 4) +
                               ((d & 7) << 1));
}

template <int D>
struct AttnSmem {
  static constexpr int kStages = attn_stages<D>();
  static constexpr int kTileBytes = kAttnKeys * D * 2;  // one K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kTreeOffset = kStages * kStageBytes;
  static constexpr int kAncOffset = kTreeOffset + kStageBytes;
  static constexpr int kParOffset = kAncOffset + 64 * 8;
  static constexpr int kBarOffset = kParOffset + 64 * 4;
  static constexpr int kBytes = kBarOffset + 2 * kStages * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

// Per-warp online-softmax state and the S / PV tile computation.
template <int D>
struct AttnWarp {
  uint32_t qf[D / 16][4];  // A fragments of the warp's 16 query rows
  float o[D / 8][4];       // output accumulators (rows g and g + 8)
  float m[2];              // running max (log2 domain)
  float l[2];              // running denominator (this thread's columns only)

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
  }

  // mask(row_half, key) -> key is visible to this thread's row (row_half 0: g, 1: g + 8)
  template <class Mask>
  __device__ __forceinline__ void tile(uint32_t k_base, uint32_t v_base, float scale_log2,
                                       const Mask& mask) {
    const int lane = threadIdx.x & 31;
    const int tig = lane & 3;
    float sc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int kk = 0; kk < D / 16; kk += 2) {
      // consecutive MMAs go to different accumulators (no back-to-back dependency)
      uint32_t bh[8][2];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        uint32_t b0, b1;
        ldmatrix_x4(k_base + attn_swz(nt * 8 + rr, kk * 16 + mi * 8), b0, b1, bh[nt][0], bh[nt][1]);
        mma_bf16_16816(sc[nt], qf[kk], b0, b1);
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mma_bf16_16816(sc[nt], qf[kk + 1], bh[nt][0], bh[nt][1]);
    }
    // scale, mask, row max
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = nt * 8 + tig * 2 + (e & 1);
        const int half = e >> 1;
        const float s = mask(half, key) ? sc[nt][e] * scale_log2 : -INFINITY;
        sc[nt][e] = s;
        mx[half] = fmaxf(mx[half], s);
      }
    }
    float corr[2], mu[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      const float mn = fmaxf(m[h], mx[h]);
      mu[h] = (mn == -INFINITY) ? 0.f : mn;
      corr[h] = exp2f(m[h] - mu[h]);
      m[h] = mn;
      l[h] *= corr[h];
    }
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) {
      o[dt][0] *= corr[0];
      o[dt][1] *= corr[0];
      o[dt][2] *= corr[1];
      o[dt][3] *= corr[1];
    }
    // P = exp2(S - m) rounded to bf16; the denominator sums the rounded values
    uint32_t pk[8][2];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = exp2f(sc[nt][0] - mu[0]);
      const float p1 = exp2f(sc[nt][1] - mu[0]);
      const float p2 = exp2f(sc[nt][2] - mu[1]);
      const float p3 = exp2f(sc[nt][3] - mu[1]);
      pk[nt][0] = pack_bf16x2(p0, p1);
      pk[nt][1] = pack_bf16x2(p2, p3);
      const __nv_bfloat162 q01 = *reinterpret_cast<const __nv_bfloat162*>(&pk[nt][0]);
      const __nv_bfloat162 q23 = *reinterpret_cast<const __nv_bfloat162*>(&pk[nt][1]);
      l[0] += __low2float(q01) + __high2float(q01);
      l[1] += __low2float(q23) + __high2float(q23);
    }
    // O += P V
#pragma unroll
    for (int kk2 = 0; kk2 < 4; ++kk2) {
      const uint32_t a[4] = {pk[2 * kk2][0], pk[2 * kk2][1], pk[2 * kk2 + 1][0], pk[2 * kk2 + 1][1]};
#pragma unroll
      for (int dt = 0; dt < D / 8; dt += 2) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(v_base + attn_swz(kk2 * 16 + (mi & 1) * 8 + rr, (dt + (mi >> 1)) * 8), b0,
                          b1, b2, b3);
        mma_bf16_16816(o[dt], a, b0, b1);
        mma_bf16_16816(o[dt + 1], a, b2, b3);
      }
    }
  }
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads)
    tree_attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const AttnParams prm) {
  using SM = AttnSmem<D>;
  extern __shared__ uint8_t attn_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int kStages = SM::kStages;
  uint64_t* anc = reinterpret_cast<uint64_t*>(smem + SM::kAncOffset);
  int32_t* par_s = reinterpret_cast<int32_t*>(smem + SM::kParOffset);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kBarOffset);
  uint64_t* empty = full + kStages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rb = blockIdx.x;
  const int split = blockIdx.y;
  const int bk = blockIdx.z;
  const int b = bk / prm.Hkv;
  const int kvh = bk % prm.Hkv;
  const int N = prm.N, G = prm.G, R = G * N;
  const int row0 = rb * kAttnRows;
  int L = prm.prefix_lens[b];
  L = L < 0 ? 0 : (L > prm.Lmax ? prm.Lmax : L);
  const int ntiles = (L + kAttnKeys - 1) / kAttnKeys;
  const int t_begin = split * prm.tiles_per_split;
  const int t_end = min(ntiles, t_begin + prm.tiles_per_split);
  const int nt = t_end > t_begin ? t_end - t_begin : 0;
  const bool last = split == prm.num_splits - 1;
  const uint32_t smem_base = smem_u32(smem);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), kAttnConsumerWarps);
    }
    fence_mbar_init();
  }
  if (last && threadIdx.x < N) par_s[threadIdx.x] = prm.parents[static_cast<size_t>(b) * N + threadIdx.x];
  if (last && warp < kAttnConsumerWarps) {
    // tree K/V of (b, kvh) -> swizzled shared tile; rows >= N are zero
    const uint32_t kt = smem_base + SM::kTreeOffset;
    const uint32_t vt = kt + SM::kTileBytes;
    for (int idx = threadIdx.x; idx < kAttnKeys * (D / 8); idx += 32 * kAttnConsumerWarps) {
      const int j = idx / (D / 8);
      const int d = (idx % (D / 8)) * 8;
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (j < N) {
        const size_t off = ((static_cast<size_t>(b) * N + j) * prm.Hkv + kvh) * D + d;
        kv = *reinterpret_cast<const uint4*>(prm.k_tree + off);
        vv = *reinterpret_cast<const uint4*>(prm.v_tree + off);
      }
      const uint32_t o = attn_swz(j, d);
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(kt + o), "r"(kv.x), "r"(kv.y),
                   "r"(kv.z), "r"(kv.w));
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(vt + o), "r"(vv.x), "r"(vv.y),
                   "r"(vv.z), "r"(vv.w));
    }
  }
  __syncthreads();
  if (last && threadIdx.x < N) {
    // ancestor bitmask of node i: itself and every node up its parent chain; a parent link
    // that does not point to an earlier node ends the chain
    int a = threadIdx.x;
    uint64_t m = 0;
    for (int guard = 0; guard < 64 && a >= 0; ++guard) {
      m |= 1ull << a;
      const int p = par_s[a];
      a = (p >= 0 && p < a) ? p : -1;
    }
    anc[threadIdx.x] = m;
  }
  __syncthreads();

  if (warp == kAttnConsumerWarps) {
    // ---------------- producer: prefix K/V tiles of this split
    if (lane == 0) {
      const uint32_t bytes = 2 * SM::kTileBytes;
      int issued = 0;
      bool ok = true;
      for (int t = 0; t < nt; ++t) {
        const int s = t % kStages;
        const int n = t / kStages;
        if (n > 0 && !mbar_wait(smem_u32(&empty[s]), (n - 1) & 1, kErrAttnProducerWait)) {
          ok = false;
          break;
        }
        const uint32_t fb = smem_u32(&full[s]);
        const uint32_t kdst = smem_base + s * SM::kStageBytes;
        const uint32_t vdst = kdst + SM::kTileBytes;
        const int key0 = (t_begin + t) * kAttnKeys;
        mbar_arrive_expect_tx(fb, bytes);
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(kdst + h * kAttnKeys * 128, &tm_k, fb, h * 64, key0, bk);
          tma_load_3d(vdst + h * kAttnKeys * 128, &tm_v, fb, h * 64, key0, bk);
        }
        issued = t + 1;
      }
      if (!ok) {
        for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
          mbar_wait(smem_u32(&full[t % kStages]), (t / kStages) & 1, kErrAttnProducerWait);
      }
    }
    return;
  }

  // ---------------- consumers
  const int g = lane >> 2, tig = lane & 3;
  AttnWarp<D> st;
  st.init();
  int node[2], head[2];
  bool rvalid[2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int r = row0 + warp * 16 + g + hf * 8;
    rvalid[hf] = r < R;
    node[hf] = rvalid[hf] ? r / G : 0;
    head[hf] = kvh * G + (rvalid[hf] ? r % G : 0);
  }
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int hf = e & 1;
      const int d = kk * 16 + tig * 2 + (e >> 1) * 8;
      uint32_t v = 0;
      if (rvalid[hf]) {
        const size_t off = ((static_cast<size_t>(b) * N + node[hf]) * prm.Hq + head[hf]) * D + d;
        v = *reinterpret_cast<const uint32_t*>(prm.q + off);
      }
      st.qf[kk][e] = v;
    }
  }

  bool ok = true;
  for (int t = 0; t < nt; ++t) {
    const int s = t % kStages;
    if (!mbar_wait(smem_u32(&full[s]), (t / kStages) & 1, kErrAttnConsumerWait)) {
      ok = false;
      break;
    }
    const uint32_t kb = smem_base + s * SM::kStageBytes;
    const uint32_t vb = kb + SM::kTileBytes;
    const int key0 = (t_begin + t) * kAttnKeys;
    const int valid = min(kAttnKeys, L - key0);
    if (valid < kAttnKeys) {
      // keys past L_b must not reach P V even if the padding holds non-finite values
      for (int idx = lane; idx < (kAttnKeys - valid) * (D / 8); idx += 32) {
        const int j = valid + idx / (D / 8);
        const int d = (idx % (D / 8)) * 8;
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vb + attn_swz(j, d)), "r"(0));
      }
      __syncwarp();
    }
    st.tile(kb, vb, prm.scale_log2, [&](int, int key) { return key < valid; });
    // the zero rows written above precede the next TMA write into this stage
    if (valid < kAttnKeys) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
  }
  if (ok && last) {
    const uint32_t kt = smem_base + SM::kTreeOffset;
    const uint64_t m0 = anc[node[0]], m1 = anc[node[1]];
    st.tile(kt, kt + SM::kTileBytes, prm.scale_log2, [&](int hf, int key) {
      return key < N && (((hf ? m1 : m0) >> key) & 1ull);
    });
  }
  if (!ok) return;

  // ---------------- epilogue
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    st.l[hf] += __shfl_xor_sync(0xffffffffu, st.l[hf], 1);
    st.l[hf] += __shfl_xor_sync(0xffffffffu, st.l[hf], 2);
  }
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    if (!rvalid[hf]) continue;
    const size_t prow = (static_cast<size_t>(b) * N + node[hf]) * prm.Hq + head[hf];
    if (prm.num_splits == 1) {
      const float inv = 1.0f / st.l[hf];
      __nv_bfloat16* dst = prm.out + prow * D;
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        const int d = dt * 8 + tig * 2;
        *reinterpret_cast<uint32_t*>(dst + d) =
            pack_bf16x2(st.o[dt][hf * 2] * inv, st.o[dt][hf * 2 + 1] * inv);
      }
    } else {
      float* dst = prm.part_acc + (prow * prm.num_splits + split) * D;
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        const int d = dt * 8 + tig * 2;
        *reinterpret_cast<float2*>(dst + d) = make_float2(st.o[dt][hf * 2], st.o[dt][hf * 2 + 1]);
      }
      if (tig == 0) {
        *reinterpret_cast<float2*>(prm.part_ml + (prow * prm.num_splits + split) * 2) =
            make_float2(st.m[hf], st.l[hf]);
      }
    }
  }
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

template <int D>
__global__ void __launch_bounds__(128)
    tree_attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ kp,
                         const float* __restrict__ vp, const int32_t* __restrict__ prefix_lens,
                         const float* __restrict__ kt, const float* __restrict__ vt,
                         const int32_t* __restrict__ parents, float* __restrict__ out, int B, int N,
                         int Hq, int Hkv, int Lmax, float scale) {
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= B * N * Hq) return;
  const int b = row / (N * Hq);
  const int i = (row / Hq) % N;
  const int h = row % Hq;
  const int g = h / (Hq / Hkv);
  constexpr int kPer = D / 32;
  float qv[kPer], acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    qv[e] = q[static_cast<size_t>(row) * D + lane + 32 * e];
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  auto visit = [&](const float* kr, const float* vr) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) s = fmaf(qv[e], kr[lane + 32 * e], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    s *= scale;
    const float mn = fmaxf(m, s);
    const float corr = expf(m - mn);
    const float p = expf(s - mn);
    l = l * corr + p;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = fmaf(p, vr[lane + 32 * e], acc[e] * corr);
    m = mn;
  };
  int L = prefix_lens[b];
  L = L < 0 ? 0 : (L > Lmax ? Lmax : L);
  const size_t pbase = (static_cast<size_t>(b) * Hkv + g) * Lmax;
  for (int j = 0; j < L; ++j) visit(kp + (pbase + j) * D, vp + (pbase + j) * D);
  int a = i;
  for (;;) {
    const size_t off = ((static_cast<size_t>(b) * N + a) * Hkv + g) * D;
    visit(kt + off, vt + off);
    const int p = parents[static_cast<size_t>(b) * N + a];
    if (p < 0 || p >= a) break;
    a = p;
  }
  const float inv = 1.0f / l;
#pragma unroll
  for (int e = 0; e < kPer; ++e) out[static_cast<size_t>(row) * D + lane + 32 * e] = acc[e] * inv;
}

}  // namespace eagle
