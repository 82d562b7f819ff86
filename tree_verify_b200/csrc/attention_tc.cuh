// attention_tc.cuh -- tree attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// What it computes is the same as attention.cuh (EAGLE summary, section 3: the target
// scores every draft node in one pass with tree attention; each node sees the prefix and
// its own ancestors).  One CTA owns one (sequence, kv head, block of up to 128 query rows,
// prefix split).  The query rows of a kv head are its G heads x the tree nodes (row
// r -> node i0 + r / G, head kvh*G + r % G), so one 128-row MMA tile covers all of them and
// every prefix K/V tile is read from HBM once.
//
//   warp 16 lane 0    TMA: the Q tile once (a 3-D box over [B*N, Hq, D]) and the 128-key K
//                     tiles of this split into the K ring;
//   warp 16 lane 1    TMA: the matching V tiles into the V ring (its own ring and barriers,
//                     so a K slot is refilled as soon as S = Q K^T has read it, a tile
//                     earlier than its V slot);
//   warp 17 (lane 0)  tcgen05.mma: S = Q K^T (M 128, N 128, K = D) into one of two TMEM
//                     buffers, then O += P V (M 128, N = D, K 128) with P read from TMEM and
//                     V as an MN-major operand straight from its TMA tile (128-key tiles:
//                     fewer, larger MMA instructions per key);
//   warps 0-15        four threads per query row (= TMEM lane): warps w, w + 4, w + 8 and
//                     w + 12 share the lane quarter w % 4 and take 32 of the tile's 128 scores
//                     each (tcgen05.ld), mask them (prefix length, or the ancestor bitmask
//                     for the tree tile), exchange the row maximum through shared memory,
//                     and store their quarter of P (bf16 pairs) back into TMEM (tcgen05.st).
//                     Four warps per SM sub-partition keep the exponential unit fed.  A
//                     warp whose 32 rows are all padding only keeps the barriers.
// S(t+1) is computed while the softmax of tile t runs (two S and two P buffers in TMEM).
// O lives in TMEM and is rescaled lazily: only when a row's maximum grows by more than 2^8
// over the reference the row's P values were taken against (otherwise P <= 2^8, well
// inside bf16/fp32 range).  The last split also runs the tree tile: its K/V rows come by
// TMA from a 4-D view of the tree K/V ([B][N][Hkv][D], rows past N zero-filled) into the
// next ring slots.  Splits write (m, l, acc) partials for the log-sum-exp merge; a single
// split normalises and writes the output.
#pragma once

#include "attention.cuh"
#include "device_common.cuh"

namespace eagle {

constexpr int kTcRows = 128;  // MMA M: query rows per CTA
constexpr int kTcSoftmaxWarps = 16;
constexpr int kTcParts = kTcSoftmaxWarps / 4;       // warps sharing one TMEM lane quarter
constexpr int kTcCols = kAttnKeys / kTcParts;       // score columns per softmax thread
constexpr int kTcLoadWarp = kTcSoftmaxWarps;       // lane 0: Q and K tiles; lane 1: V tiles
constexpr int kTcMmaWarp = kTcSoftmaxWarps + 1;
constexpr int kTcThreads = 32 * (kTcSoftmaxWarps + 2);
constexpr float kTcRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct TcSmem {
  static constexpr int kKStages = D == 128 ? 3 : 5;
  static constexpr int kVStages = D == 128 ? 2 : 5;
  // S and P buffers in TMEM: two of each, so S(t + 1) is computed while the softmax of tile
  // t runs
  static constexpr int kSBufs = 2;
  static constexpr int kTile = kAttnKeys * D * 2;  // one K or V tile (D/64 boxes of 128 x 128 B)
  static constexpr int kQ = kTcRows * D * 2;        // D/64 boxes of 128 rows x 128 B
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQ;
  static constexpr int kVOff = kKOff + kKStages * kTile;
  static constexpr int kAncOff = kVOff + kVStages * kTile;
  static constexpr int kParOff = kAncOff + 64 * 8;
  // row-maximum exchange [tile parity][part][row] and, after the loop, the denominator
  // exchange [part][row]
  static constexpr int kXchOff = kParOff + 64 * 4;
  static constexpr int kBarOff = kXchOff + 3 * kTcParts * kTcRows * 4;
  // q_full, k_full[SK], k_empty[SK], v_full[SV], v_empty[SV], s_full[2], s_free[2],
  // p_full[2], pv_done[2], o_final
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 4 * kSBufs + 1;
  static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
  // TMEM columns: S0 / S1 128 columns each [0, 256), O [256, 256 + D), P0 / P1 64 columns
  // each (128 bf16 per row, two to a column) after O
  static constexpr uint32_t kOCol = kSBufs * kAttnKeys;
  static constexpr uint32_t kPCol = kOCol + D;
  static constexpr uint32_t kTmemCols = 512;
};

struct TcAttnParams {
  AttnParams a;
  int32_t nodes_per_block;  // NB: nodes per 128-row tile (G * NB <= 128)
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    tree_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kt,
                        const __grid_constant__ CUtensorMap tm_vt, const TcAttnParams tp) {
  using SM = TcSmem<D>;
  constexpr int SK = SM::kKStages;
  constexpr int SV = SM::kVStages;
  const AttnParams& prm = tp.a;
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* anc = reinterpret_cast<uint64_t*>(smem + SM::kAncOff);
  int32_t* par_s = reinterpret_cast<int32_t*>(smem + SM::kParOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + SK;
  uint64_t* v_full = k_empty + SK;
  uint64_t* v_empty = v_full + SV;
  constexpr int NS = SM::kSBufs;
  uint64_t* s_full = v_empty + SV;
  uint64_t* s_free = s_full + NS;
  uint64_t* p_full = s_free + NS;
  uint64_t* pv_done = p_full + NS;
  uint64_t* o_final = pv_done + NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_final + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rb = blockIdx.x, split = blockIdx.y, bk = blockIdx.z;
  const int b = bk / prm.Hkv, kvh = bk % prm.Hkv;
  const int N = prm.N, G = prm.G, NB = tp.nodes_per_block;
  const int i0 = rb * NB;
  const int rows_blk = NB * G;
  int L = prm.prefix_lens[b];
  if ((L < 0 || L > prm.Lmax) && threadIdx.x == 0 && rb == 0 && split == 0) record_error(kErrAttnPrefixLen);
  L = L < 0 ? 0 : (L > prm.Lmax ? prm.Lmax : L);
  const int ntiles = (L + kAttnKeys - 1) / kAttnKeys;
  const int t_begin = split * prm.tiles_per_split;
  const int t_end = min(ntiles, t_begin + prm.tiles_per_split);
  const int nt = t_end > t_begin ? t_end - t_begin : 0;
  const bool last = split == prm.num_splits - 1;
  const int T = nt + (last ? 1 : 0);  // tiles this CTA runs (prefix tiles, then the tree tile)

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < SK; ++s) {
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);
    }
    for (int s = 0; s < SV; ++s) {
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
    }
    for (int i = 0; i < NS; ++i) {
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
  auto k_stage = [&](int s) { return sbase + SM::kKOff + static_cast<uint32_t>(s) * SM::kTile; };
  auto v_stage = [&](int s) { return sbase + SM::kVOff + static_cast<uint32_t>(s) * SM::kTile; };

  if (warp == kTcLoadWarp) {
    // ------------------------------------------------------------ TMA producers (K, V)
    if (lane < 2) {
      const bool is_k = lane == 0;
      const int S = is_k ? SK : SV;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      const CUtensorMap* tmap = is_k ? &tm_kt : &tm_vt;
      prefetch_tmap(tmap);
      if (is_k) {
        mbar_arrive_expect_tx(smem_u32(q_full), static_cast<uint32_t>(rows_blk * D * 2));
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(q_s + h * kTcRows * 128, &tm_q, smem_u32(q_full), h * 64, kvh * G, b * N + i0);
      }
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % S, n = t / S;
        if (n > 0 && !mbar_wait(smem_u32(&empty[s]), (n - 1) & 1, kErrAttnProducerWait)) break;
        const uint32_t fb = smem_u32(&full[s]);
        const uint32_t dst = is_k ? k_stage(s) : v_stage(s);
        mbar_arrive_expect_tx(fb, SM::kTile);
        if (t < nt) {
          const int key0 = (t_begin + t) * kAttnKeys;
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_load_3d(dst + h * kAttnKeys * 128, map, fb, h * 64, key0, bk);
        } else {
          // the tree tile: nodes 0..63 of (b, kvh); nodes past N are zero-filled
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_load_4d(dst + h * kAttnKeys * 128, tmap, fb, h * 64, kvh, 0, b);
        }
        issued = t + 1;
      }
      // every issued copy lands before the CTA can leave
      for (int t = (issued > S ? issued - S : 0); t < issued; ++t)
        mbar_wait(smem_u32(&full[t % S]), (t / S) & 1, kErrAttnProducerWait);
      if (is_k) mbar_wait(smem_u32(q_full), 0, kErrAttnProducerWait);
    }
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTcRows, kAttnKeys);
      const uint32_t idesc_o = idesc_bf16_f32_bmn(kTcRows, D);
      const uint32_t o_tmem = tmem + SM::kOCol;
      bool ok = mbar_wait(smem_u32(q_full), 0, kErrAttnMmaWait);
      auto issue_s = [&](int t) {
        const int s = t % SK, sb = t % NS;
        ok = ok && mbar_wait(smem_u32(&k_full[s]), (t / SK) & 1, kErrAttnMmaWait);
        // buffer sb was last read (into registers) by the softmax of tile t - NS
        if (t >= NS) ok = ok && mbar_wait(smem_u32(&s_free[sb]), (t / NS - 1) & 1, kErrAttnMmaWait);
        tc_fence_after();
        const uint32_t kb = k_stage(s);
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(sb * kAttnKeys);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int h = kk >> 2, k4 = kk & 3;
          const uint64_t a = smem_desc_k_sw128(q_s + h * kTcRows * 128) + 2 * k4;
          const uint64_t bdesc = smem_desc_k_sw128(kb + h * kAttnKeys * 128) + 2 * k4;
          if (ok) tc_mma_f16(d_tmem, a, bdesc, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&s_full[sb]));
        tc_commit(smem_u32(&k_empty[s]));  // the K slot is free once S(t) has read it
      };
      // S(t + 1) is queued before PV(t) waits for the softmax of tile t
      if (T > 0) issue_s(0);
      for (int t = 0; t < T; ++t) {
        if (t + 1 < T) issue_s(t + 1);
        const int s = t % SV, pb = t % NS;
        ok = ok && mbar_wait(smem_u32(&p_full[pb]), (t / NS) & 1, kErrAttnMmaWait);
        ok = ok && mbar_wait(smem_u32(&v_full[s]), (t / SV) & 1, kErrAttnMmaWait);
        tc_fence_after();
        const uint32_t vb = v_stage(s);
        const uint32_t pa = tmem + SM::kPCol + static_cast<uint32_t>(pb * (kAttnKeys / 2));
#pragma unroll
        for (int kk = 0; kk < kAttnKeys / 16; ++kk) {
          // 16 keys = 8 TMEM columns of P (bf16 pairs) and two 8-key groups of 1024 B of V;
          // the second 64-column group of V is the next TMA box, kAttnKeys x 128 B further
          const uint64_t bdesc = smem_desc_mn_sw128(vb + kk * 2048, kAttnKeys * 128, 1024);
          if (ok) tc_mma_f16_ts(o_tmem, pa + 8 * kk, bdesc, idesc_o, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(smem_u32(&pv_done[pb]));
        tc_commit(smem_u32(&v_empty[s]));
      }
      tc_commit(smem_u32(o_final));
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    constexpr int kSoftThreads = 32 * kTcSoftmaxWarps;
    constexpr int C = kTcCols;              // score columns of this thread
    constexpr int OC = D / kTcParts;        // output columns of this thread
    const int quarter = warp & 3;           // TMEM lane quarter = row block of 32
    const int part = warp >> 2;             // which C of the 64 scores, which OC of O
    const int r = quarter * 32 + lane;      // query row = TMEM lane
    const int node = i0 + r / G;
    const int head = kvh * G + r % G;
    const bool rvalid = r < rows_blk && node < N;
    // a warp with no real row skips the score and output work (its rows of P and O are
    // never read for an output), but keeps every barrier; the warps of a quarter cover the
    // same rows, so they are live together
    const bool live = __any_sync(0xffffffffu, rvalid);
    const int tid = threadIdx.x;            // 0 .. kSoftThreads-1
    float* xch = reinterpret_cast<float*>(smem + SM::kXchOff);
    const uint32_t quarter_bar = 2 + quarter;  // named barrier of the warps sharing a quarter
    auto quarter_sync = [&]() {
      asm volatile("bar.sync %0, %1;" ::"r"(quarter_bar), "r"(32 * kTcParts) : "memory");
    };
    if (last) {
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
      // named barrier of the softmax warps: the masks are read below
      asm volatile("bar.sync 1, %0;" ::"r"(kSoftThreads) : "memory");
    }
    constexpr uint32_t kColMask = C == 32 ? 0xffffffffu : ((1u << C) - 1u);
    // this thread's C key columns of the tree tile, as a bit mask
    const uint32_t tree_bits = (last && rvalid && C * part < 64)
                                   ? static_cast<uint32_t>(anc[node] >> (C * part)) & kColMask : 0u;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    float m_ref = -INFINITY, l = 0.f;
    for (int t = 0; t < T; ++t) {
      const bool tree = t >= nt;
      const int sb = t % NS;
      mbar_wait(smem_u32(&s_full[sb]), (t / NS) & 1, kErrAttnConsumerWait);
      tc_fence_after();
      uint32_t sv[C];
      if (live) {
        __syncwarp();  // the TMEM load below is warp-wide
        tmem_ld_cols<C>(lane_base + sb * kAttnKeys + C * part, sv);
        tmem_ld_wait();
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&s_free[sb]));
      if (live) {
        // visibility of this thread's C keys
        const int first = tree ? 0 : (t_begin + t) * kAttnKeys;
        const int valid = (tree ? N : min(kAttnKeys, L - first)) - C * part;
        uint32_t vis = valid >= C ? kColMask : (valid <= 0 ? 0u : ((1u << valid) - 1u));
        if (tree) vis &= tree_bits;
        if (!rvalid) vis = 0u;
        // raw scores; masked ones (past L_b, outside the ancestor set, padding rows) become
        // -inf, which also drops any non-finite value the padding holds
        float x[C];
#pragma unroll
        for (int j = 0; j < C; ++j) x[j] = __uint_as_float(sv[j]);
        if (vis != kColMask) {
#pragma unroll
          for (int j = 0; j < C; ++j) x[j] = ((vis >> j) & 1u) ? x[j] : -INFINITY;
        }
        // tile maximum by a tree (short dependency chains)
        float mx[C / 4];
#pragma unroll
        for (int j = 0; j < C / 4; ++j)
          mx[j] = fmaxf(fmaxf(x[j], x[j + C / 4]), fmaxf(x[j + C / 2], x[j + 3 * C / 4]));
#pragma unroll
        for (int w2 = C / 8; w2 >= 1; w2 >>= 1)
#pragma unroll
          for (int j = 0; j < w2; ++j) mx[j] = fmaxf(mx[j], mx[j + w2]);
        float tmax = mx[0];
        // row maximum of the tile: combine with the other parts of the row; in scaled log2
        // units (the scale is positive, so the maximum commutes with it)
        xch[((t & 1) * kTcParts + part) * kTcRows + r] = tmax;
        quarter_sync();
#pragma unroll
        for (int o = 1; o < kTcParts; ++o)
          tmax = fmaxf(tmax, xch[((t & 1) * kTcParts + ((part + o) % kTcParts)) * kTcRows + r]);
        tmax *= prm.scale_log2;
        const float m_new = fmaxf(m_ref, tmax);
        const bool rebase =
            m_new != -INFINITY && (m_ref == -INFINITY || m_new > m_ref + kTcRescaleThreshold);
        const bool scale_o = rebase && m_ref != -INFINITY;  // O holds P V taken against m_ref
        const float f = scale_o ? fast_exp2(m_ref - m_new) : 1.0f;
        // TMEM loads/stores are warp-wide: the warp rescales if any of its rows must
        if (__any_sync(0xffffffffu, scale_o)) {
          mbar_wait(smem_u32(&pv_done[(t - 1) % NS]), ((t - 1) / NS) & 1, kErrAttnConsumerWait);
          tc_fence_after();
          __syncwarp();
#pragma unroll 1
          for (int c0 = 0; c0 < OC; c0 += 16) {
            uint32_t ov[16];
            tmem_ld_cols<16>(lane_base + SM::kOCol + OC * part + c0, ov);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * f);
            tmem_st_cols<16>(lane_base + SM::kOCol + OC * part + c0, ov);
          }
          tmem_st_wait();
        }
        if (rebase) {
          l *= f;
          m_ref = m_new;
        }
        // p = 2^(s * scale_log2 - m), one fused multiply-add per score; masked keys give
        // exp2(-inf) = 0 (and m = 0 while every key so far was masked)
        const float c = prm.scale_log2;
        const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
        // P buffer t % 2 was last read by PV(t - 2)
        if (t >= NS) mbar_wait(smem_u32(&pv_done[sb]), (t / NS - 1) & 1, kErrAttnConsumerWait);
        uint32_t w[C / 2];
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < C / 2; ++e) {
          const float p0 = fast_exp2(fmaf(x[2 * e], c, neg_m));
          const float p1 = fast_exp2(fmaf(x[2 * e + 1], c, neg_m));
          w[e] = pack_bf16x2(p0, p1);
          // the denominator sums the fp32 values; the MMA multiplies their bf16 roundings
          // (round to nearest: the difference averages out far below the bf16 tolerance)
          ls[e & 3] += p0 + p1;
        }
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        __syncwarp();
        tmem_st_cols<C / 2>(lane_base + SM::kPCol + sb * (kAttnKeys / 2) + (C / 2) * part, w);
        tmem_st_wait();
      }
      if (!tree) {
        const int valid = min(kAttnKeys, L - (t_begin + t) * kAttnKeys);
        if (valid < kAttnKeys) {
          // keys past L_b must not reach P V even if the padding holds non-finite values:
          // zero those rows of this tile's V slot once it has landed
          const int s = t % SV;
          mbar_wait(smem_u32(&v_full[s]), (t / SV) & 1, kErrAttnConsumerWait);
          const uint32_t vb = v_stage(s);
          for (int idx = tid; idx < (kAttnKeys - valid) * (D / 8); idx += kSoftThreads) {
            const int j = valid + idx / (D / 8);
            const int d = (idx % (D / 8)) * 8;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vb + attn_swz(j, d)), "r"(0));
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&p_full[sb]));
    }

    // ------------------------------------------------------------ epilogue
    // row denominator: this thread's columns plus the other parts'
    if (live) {
      float* lx = xch + 2 * kTcParts * kTcRows;
      lx[part * kTcRows + r] = l;
      quarter_sync();
#pragma unroll
      for (int o = 1; o < kTcParts; ++o) l += lx[((part + o) % kTcParts) * kTcRows + r];
    }
    if (T > 0) {
      mbar_wait(smem_u32(o_final), 0, kErrAttnConsumerWait);
      tc_fence_after();
    }
    const size_t prow_g = (static_cast<size_t>(b) * N + node) * prm.Hq + head;
    const bool single = prm.num_splits == 1;
    const float inv = (l > 0.f) ? 1.0f / l : 0.f;
    if (live) {
#pragma unroll 1
      for (int cc = 0; cc < OC; cc += 16) {
        uint32_t ov[16];
        __syncwarp();  // the TMEM load below is warp-wide
        if (T > 0) {
          tmem_ld_cols<16>(lane_base + SM::kOCol + OC * part + cc, ov);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) ov[k] = 0u;
        }
        const int c0 = OC * part + cc;
        if (!rvalid) {
        } else if (single) {
          uint4* dst = reinterpret_cast<uint4*>(prm.out + prow_g * D + c0);
#pragma unroll
          for (int k = 0; k < 16; k += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ov[k]) * inv, __uint_as_float(ov[k + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ov[k + 2]) * inv, __uint_as_float(ov[k + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ov[k + 4]) * inv, __uint_as_float(ov[k + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ov[k + 6]) * inv, __uint_as_float(ov[k + 7]) * inv);
            dst[k / 8] = w;
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(prm.part_acc + (prow_g * prm.num_splits + split) * D + c0);
#pragma unroll
          for (int k = 0; k < 16; k += 4)
            dst[k / 4] = make_float4(__uint_as_float(ov[k]), __uint_as_float(ov[k + 1]),
                                     __uint_as_float(ov[k + 2]), __uint_as_float(ov[k + 3]));
        }
      }
    }
    if (rvalid && !single && part == 0)
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
