// attention_tc.cuh -- tree attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// What it computes is the same as attention.cuh (EAGLE summary, section 3: the target
// scores every draft node in one pass with tree attention; each node sees the prefix and
// its own ancestors).  One CTA owns one (sequence, kv head, block of up to 128 query rows,
// prefix split).  The query rows of a kv head are its G heads x the tree nodes (row
// r -> node i0 + r / G, head kvh*G + r % G), so one 128-row MMA tile covers all of them and
// every prefix K/V tile is read from HBM once.
//
//   warp 8 (lane 0)  TMA: the Q tile once (a 3-D box over [B*N, Hq, D]) and 64-key K/V
//                    tiles of this split into a multi-stage mbarrier ring;
//   warp 9 (lane 0)  tcgen05.mma: S = Q K^T (M 128, N 64, K = D) into one of two TMEM
//                    buffers, then O += P V (M 128, N = D, K 64) with V read as an
//                    MN-major operand straight from its TMA tile;
//   warps 0-7        two threads per query row (= TMEM lane): warps w and w + 4 share the
//                    lane quarter w and take 32 of the tile's 64 scores each (tcgen05.ld),
//                    mask them (prefix length, or the ancestor bitmask for the tree tile),
//                    exchange the row maximum through shared memory, and write their half
//                    of P (bf16) into shared memory in the MMA's 128-byte-swizzled K-major
//                    layout.
// S(t+1) is computed while the softmax of tile t runs.  O lives in TMEM and is rescaled
// lazily: only when a row's maximum grows by more than 2^8 over the reference the row's P
// values were taken against (otherwise P <= 2^8, well inside bf16/fp32 range).  The last
// split also runs the tree tile, whose K/V rows the softmax warps copy into shared memory
// before the main loop.  Splits write (m, l, acc) partials for the log-sum-exp merge; a
// single split normalises and writes the output.
#pragma once

#include "attention.cuh"
#include "device_common.cuh"

namespace eagle {

constexpr int kTcRows = 128;  // MMA M: query rows per CTA
constexpr int kTcSoftmaxWarps = 8;
constexpr int kTcTmaWarp = kTcSoftmaxWarps;
constexpr int kTcMmaWarp = kTcSoftmaxWarps + 1;
constexpr int kTcThreads = 32 * (kTcSoftmaxWarps + 2);
constexpr float kTcRescaleThreshold = 8.0f;  // log2 units

// Lite: the compact layout for a CTA that runs exactly one tile (one prefix tile, or the
// tree tile in a CTA of its own): one K/V stage, which the tree tile shares, and one P
// buffer.  It is small enough to share an SM with two LM-head CTAs.
template <int D, bool Lite = false>
struct TcSmem {
  static constexpr int kStages = Lite ? 1 : (D == 128 ? 3 : 6);
  static constexpr int kPBufs = Lite ? 1 : 2;
  static constexpr int kTile = kAttnKeys * D * 2;  // one K or V tile (D/64 boxes of 64 x 128 B)
  static constexpr int kQ = kTcRows * D * 2;        // D/64 boxes of 128 rows x 128 B
  static constexpr int kP = kTcRows * kAttnKeys * 2;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kQOff + kQ;
  static constexpr int kTreeOff = Lite ? kKVOff : kKVOff + kStages * 2 * kTile;
  static constexpr int kPOff = kKVOff + kStages * 2 * kTile + (Lite ? 0 : 2 * kTile);
  static constexpr int kAncOff = kPOff + kPBufs * kP;
  static constexpr int kParOff = kAncOff + 64 * 8;
  // row-maximum exchange [tile parity][half][row] and, after the loop, the denominator
  // exchange [2][half][row]: three [2][128] float regions
  static constexpr int kXchOff = kParOff + 64 * 4;
  static constexpr int kBarOff = kXchOff + 3 * 2 * kTcRows * 4;
  // q_full, kv_full[S], kv_empty[S], tree_ready, s_full[2], s_free[2], p_full[2],
  // pv_done[2], o_final
  static constexpr int kNumBars = 1 + 2 * kStages + 1 + 2 + 2 + 2 + 2 + 1;
  static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 256;  // S0 [0,64), S1 [64,128), O [128, 128 + D)
};

struct TcAttnParams {
  AttnParams a;
  int32_t nodes_per_block;  // NB: nodes per 128-row tile (G * NB <= 128)
};

template <int D, bool Lite = false>
__global__ void __launch_bounds__(kTcThreads, 1)
    tree_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const TcAttnParams tp) {
  using SM = TcSmem<D, Lite>;
  constexpr int S = SM::kStages;
  const AttnParams& prm = tp.a;
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* anc = reinterpret_cast<uint64_t*>(smem + SM::kAncOff);
  int32_t* par_s = reinterpret_cast<int32_t*>(smem + SM::kParOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + S;
  uint64_t* tree_ready = kv_empty + S;
  uint64_t* s_full = tree_ready + 1;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_final = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_final + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rb = blockIdx.x, split = blockIdx.y, bk = blockIdx.z;
  const int b = bk / prm.Hkv, kvh = bk % prm.Hkv;
  const int N = prm.N, G = prm.G, NB = tp.nodes_per_block;
  const int i0 = rb * NB;
  const int rows_blk = NB * G;
  int L = prm.prefix_lens[b];
  L = L < 0 ? 0 : (L > prm.Lmax ? prm.Lmax : L);
  const int ntiles = (L + kAttnKeys - 1) / kAttnKeys;
  const int t_begin = split * prm.tiles_per_split;
  const int t_end = min(ntiles, t_begin + prm.tiles_per_split);
  int nt = t_end > t_begin ? t_end - t_begin : 0;
  bool last = split == prm.num_splits - 1;
  if (Lite && nt + (last ? 1 : 0) > 1) {
    // a plan that gives a compact-layout CTA two tiles: flag it and run nothing
    if (threadIdx.x == 0) record_error(kErrAttnPlan);
    nt = 0;
    last = false;
  }
  const int T = nt + (last ? 1 : 0);  // tiles this CTA runs (prefix tiles, then the tree tile)

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_empty[s]), 1);
    }
    mbar_init(smem_u32(tree_ready), 32 * kTcSoftmaxWarps);  // every softmax thread
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), 32 * kTcSoftmaxWarps);
      mbar_init(smem_u32(&p_full[i]), 32 * kTcSoftmaxWarps);
      mbar_init(smem_u32(&pv_done[i]), 1);
    }
    mbar_init(smem_u32(o_final), 1);
    fence_mbar_init();
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), SM::kTmemCols);
    tmem_relinquish();
  }
  if (last && threadIdx.x < N) par_s[threadIdx.x] = prm.parents[static_cast<size_t>(b) * N + threadIdx.x];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t q_s = sbase + SM::kQOff;
  const uint32_t tree_s = sbase + SM::kTreeOff;
  const uint32_t p_s = sbase + SM::kPOff;
  auto kv_stage = [&](int s) { return sbase + SM::kKVOff + static_cast<uint32_t>(s) * 2 * SM::kTile; };

  if (warp == kTcTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(smem_u32(q_full), static_cast<uint32_t>(rows_blk * D * 2));
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(q_s + h * kTcRows * 128, &tm_q, smem_u32(q_full), h * 64, kvh * G, b * N + i0);
      int issued = 0;
      for (int t = 0; t < nt; ++t) {
        const int s = t % S, n = t / S;
        if (n > 0 && !mbar_wait(smem_u32(&kv_empty[s]), (n - 1) & 1, kErrAttnProducerWait)) break;
        const uint32_t fb = smem_u32(&kv_full[s]);
        mbar_arrive_expect_tx(fb, 2 * SM::kTile);
        const int key0 = (t_begin + t) * kAttnKeys;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(kv_stage(s) + h * kAttnKeys * 128, &tm_k, fb, h * 64, key0, bk);
          tma_load_3d(kv_stage(s) + SM::kTile + h * kAttnKeys * 128, &tm_v, fb, h * 64, key0, bk);
        }
        issued = t + 1;
      }
      // every issued copy lands before the CTA can leave
      for (int t = (issued > S ? issued - S : 0); t < issued; ++t)
        mbar_wait(smem_u32(&kv_full[t % S]), (t / S) & 1, kErrAttnProducerWait);
      mbar_wait(smem_u32(q_full), 0, kErrAttnProducerWait);
    }
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTcRows, kAttnKeys);
      const uint32_t idesc_o = idesc_bf16_f32_bmn(kTcRows, D);
      const uint32_t o_tmem = tmem + 128;
      bool ok = mbar_wait(smem_u32(q_full), 0, kErrAttnMmaWait);
      auto issue_s = [&](int t) {
        uint32_t kb;
        if (t < nt) {
          const int s = t % S;
          ok = ok && mbar_wait(smem_u32(&kv_full[s]), (t / S) & 1, kErrAttnMmaWait);
          kb = kv_stage(s);
        } else {
          ok = ok && mbar_wait(smem_u32(tree_ready), 0, kErrAttnMmaWait);
          kb = tree_s;
        }
        if (t >= 2) ok = ok && mbar_wait(smem_u32(&s_free[t & 1]), ((t - 2) >> 1) & 1, kErrAttnMmaWait);
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>((t & 1) * kAttnKeys);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int h = kk >> 2, k4 = kk & 3;
          const uint64_t a = smem_desc_k_sw128(q_s + h * kTcRows * 128) + 2 * k4;
          const uint64_t bdesc = smem_desc_k_sw128(kb + h * kAttnKeys * 128) + 2 * k4;
          if (ok) tc_mma_f16(d_tmem, a, bdesc, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&s_full[t & 1]));
      };
      if (T > 0) issue_s(0);
      for (int t = 0; t < T; ++t) {
        if (t + 1 < T) issue_s(t + 1);
        ok = ok && mbar_wait(smem_u32(&p_full[t & 1]), (t >> 1) & 1, kErrAttnMmaWait);
        tc_fence_after();
        const uint32_t vb = (t < nt ? kv_stage(t % S) : tree_s) + SM::kTile;
        const uint32_t pb = p_s + static_cast<uint32_t>((t % SM::kPBufs) * SM::kP);
#pragma unroll
        for (int kk = 0; kk < kAttnKeys / 16; ++kk) {
          const uint64_t a = smem_desc_k_sw128(pb) + 2 * kk;
          // 16 keys = two 8-key groups of 1024 B; the second 64-column group of V is the
          // next TMA box, one tile-half (64 keys x 128 B) further
          const uint64_t bdesc = smem_desc_mn_sw128(vb + kk * 2048, kAttnKeys * 128, 1024);
          if (ok) tc_mma_f16(o_tmem, a, bdesc, idesc_o, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(smem_u32(&pv_done[t & 1]));
        if (t < nt) tc_commit(smem_u32(&kv_empty[t % S]));
      }
      tc_commit(smem_u32(o_final));
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    constexpr int kSoftThreads = 32 * kTcSoftmaxWarps;
    const int quarter = warp & 3;           // TMEM lane quarter = row block of 32
    const int half = warp >> 2;             // which 32 of the 64 scores, which half of O
    const int r = quarter * 32 + lane;      // query row = TMEM lane
    const int node = i0 + r / G;
    const int head = kvh * G + r % G;
    const bool rvalid = r < rows_blk && node < N;
    const int tid = threadIdx.x;            // 0 .. kSoftThreads-1
    float* xch = reinterpret_cast<float*>(smem + SM::kXchOff);
    const uint32_t pair_bar = 2 + quarter;  // named barrier of the two warps sharing a row
    auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory"); };
    if (last) {
      // tree K/V of (b, kvh) -> swizzled shared tile; rows >= N are zero
      for (int idx = tid; idx < kAttnKeys * (D / 8); idx += kSoftThreads) {
        const int j = idx / (D / 8);
        const int d = (idx % (D / 8)) * 8;
        uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
        if (j < N) {
          const size_t off = ((static_cast<size_t>(b) * N + j) * prm.Hkv + kvh) * D + d;
          kv = *reinterpret_cast<const uint4*>(prm.k_tree + off);
          vv = *reinterpret_cast<const uint4*>(prm.v_tree + off);
        }
        const uint32_t o = attn_swz(j, d);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(tree_s + o), "r"(kv.x), "r"(kv.y),
                     "r"(kv.z), "r"(kv.w));
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(tree_s + SM::kTile + o), "r"(vv.x),
                     "r"(vv.y), "r"(vv.z), "r"(vv.w));
      }
      if (tid < N) {
        // ancestor bitmask: node tid and every node up its parent chain (a link that does
        // not point to an earlier node ends the chain)
        int a = tid;
        uint64_t m = 0;
        for (int guard = 0; guard < 64 && a >= 0; ++guard) {
          m |= 1ull << a;
          const int p = par_s[a];
          a = (p >= 0 && p < a) ? p : -1;
        }
        anc[tid] = m;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      // named barrier of the softmax warps: the masks are read below
      asm volatile("bar.sync 1, %0;" ::"r"(kSoftThreads) : "memory");
      mbar_arrive(smem_u32(tree_ready));
    }
    // this thread's 32 key columns of the tree tile, as a bit mask
    const uint32_t tree_bits =
        (last && rvalid) ? static_cast<uint32_t>(anc[node] >> (32 * half)) : 0u;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    float m_ref = -INFINITY, l = 0.f;
    for (int t = 0; t < T; ++t) {
      const bool tree = t >= nt;
      mbar_wait(smem_u32(&s_full[t & 1]), (t >> 1) & 1, kErrAttnConsumerWait);
      tc_fence_after();
      __syncwarp();  // the TMEM load below is warp-wide
      uint32_t sv[32];
      tmem_ld_32x32b_x32(lane_base + (t & 1) * kAttnKeys + 32 * half, sv);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&s_free[t & 1]));
      // visibility of this thread's 32 keys
      uint32_t vis;
      if (tree) {
        vis = tree_bits & (N - 32 * half >= 32 ? 0xffffffffu
                                               : (N - 32 * half <= 0 ? 0u : ((1u << (N - 32 * half)) - 1u)));
      } else {
        const int valid = min(kAttnKeys, L - (t_begin + t) * kAttnKeys) - 32 * half;
        vis = valid >= 32 ? 0xffffffffu : (valid <= 0 ? 0u : ((1u << valid) - 1u));
      }
      if (!rvalid) vis = 0u;
      float x[32];
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        x[j] = ((vis >> j) & 1u) ? __uint_as_float(sv[j]) * prm.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, x[j]);
      }
      // row maximum of the tile: combine with the partner warp's half
      xch[((t & 1) * 2 + half) * kTcRows + r] = tmax;
      pair_sync();
      tmax = fmaxf(tmax, xch[((t & 1) * 2 + (half ^ 1)) * kTcRows + r]);
      const float m_new = fmaxf(m_ref, tmax);
      const bool rebase =
          m_new != -INFINITY && (m_ref == -INFINITY || m_new > m_ref + kTcRescaleThreshold);
      const bool scale_o = rebase && m_ref != -INFINITY;  // O holds P V taken against m_ref
      const float f = scale_o ? fast_exp2(m_ref - m_new) : 1.0f;
      // TMEM loads/stores are warp-wide: the warp rescales if any of its rows must
      if (__any_sync(0xffffffffu, scale_o)) {
        mbar_wait(smem_u32(&pv_done[(t - 1) & 1]), ((t - 1) >> 1) & 1, kErrAttnConsumerWait);
        tc_fence_after();
        __syncwarp();
#pragma unroll 1
        for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 32) {
          uint32_t ov[32];
          tmem_ld_32x32b_x32(lane_base + 128 + c, ov);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * f);
          tmem_st_32x32b_x32(lane_base + 128 + c, ov);
        }
        tmem_st_wait();
      }
      if (rebase) {
        l *= f;
        m_ref = m_new;
      }
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;  // masked keys give exp2(-inf) = 0
      // P buffer t&1 was last read by PV(t - 2)
      if (t >= 2) mbar_wait(smem_u32(&pv_done[t & 1]), ((t - 2) >> 1) & 1, kErrAttnConsumerWait);
      const uint32_t prow = p_s + static_cast<uint32_t>((t % SM::kPBufs) * SM::kP) + static_cast<uint32_t>(r * 128);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = c * 8 + e * 2;
          w[e] = pack_bf16x2(fast_exp2(x[j] - m_use), fast_exp2(x[j + 1] - m_use));
          // the denominator sums the rounded values the MMA multiplies
          l += __uint_as_float(w[e] << 16) + __uint_as_float(w[e] & 0xffff0000u);
        }
        const int chunk = half * 4 + c;
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(prow + ((chunk ^ (r & 7)) << 4)),
                     "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]));
      }
      if (!tree) {
        const int valid = min(kAttnKeys, L - (t_begin + t) * kAttnKeys);
        if (valid < kAttnKeys) {
          // keys past L_b must not reach P V even if the padding holds non-finite values
          const uint32_t vb = kv_stage(t % S) + SM::kTile;
          for (int idx = tid; idx < (kAttnKeys - valid) * (D / 8); idx += kSoftThreads) {
            const int j = valid + idx / (D / 8);
            const int d = (idx % (D / 8)) * 8;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vb + attn_swz(j, d)), "r"(0));
          }
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(smem_u32(&p_full[t & 1]));
    }

    // ------------------------------------------------------------ epilogue
    // row denominator: this thread's columns plus the partner's
    xch[(4 + half) * kTcRows + r] = l;
    pair_sync();
    l += xch[(4 + (half ^ 1)) * kTcRows + r];
    if (T > 0) {
      mbar_wait(smem_u32(o_final), 0, kErrAttnConsumerWait);
      tc_fence_after();
    }
    const size_t prow_g = (static_cast<size_t>(b) * N + node) * prm.Hq + head;
    const bool single = prm.num_splits == 1;
    const float inv = (l > 0.f) ? 1.0f / l : 0.f;
    for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 32) {
      uint32_t ov[32];
      __syncwarp();  // the TMEM load below is warp-wide
      if (T > 0) {
        tmem_ld_32x32b_x32(lane_base + 128 + c, ov);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) ov[k] = 0u;
      }
      if (!rvalid) {
      } else if (single) {
        uint4* dst = reinterpret_cast<uint4*>(prm.out + prow_g * D + c);
#pragma unroll
        for (int k = 0; k < 32; k += 8) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(ov[k]) * inv, __uint_as_float(ov[k + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(ov[k + 2]) * inv, __uint_as_float(ov[k + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(ov[k + 4]) * inv, __uint_as_float(ov[k + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(ov[k + 6]) * inv, __uint_as_float(ov[k + 7]) * inv);
          dst[k / 8] = w;
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(prm.part_acc + (prow_g * prm.num_splits + split) * D + c);
#pragma unroll
        for (int k = 0; k < 32; k += 4)
          dst[k / 4] = make_float4(__uint_as_float(ov[k]), __uint_as_float(ov[k + 1]),
                                   __uint_as_float(ov[k + 2]), __uint_as_float(ov[k + 3]));
      }
    }
    if (rvalid && !single && half == 0)
      *reinterpret_cast<float2*>(prm.part_ml + (prow_g * prm.num_splits + split) * 2) = make_float2(m_ref, l);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    // every MMA has completed before the softmax warps passed o_final; wait here too in
    // case this CTA ran no tiles' epilogue wait
    if (lane == 0) mbar_wait(smem_u32(o_final), 0, kErrAttnMmaWait);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, SM::kTmemCols);
  }
}

}  // namespace eagle
