// attention_tc.cuh -- tree attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// What it computes is the same as attention.cuh (EAGLE summary, section 3: the target
// scores every draft node in one pass with tree attention; each node sees the prefix and
// its own ancestors).  One CTA owns one (sequence, kv head, block of up to 128 query rows,
// prefix split).  The query rows of a kv head are its G heads x the tree nodes (row
// r -> node i0 + r / G, head kvh*G + r % G), so one 128-row MMA tile covers all of them and
// every prefix K/V tile is read from HBM once.
//
// Keys arrive in tiles of 128 (one TMA box per 64 columns of D).  Each tile is split
// between two softmax groups: group 0 takes keys 0-63 of every tile, group 1 keys 64-127,
// one thread per query row in each.  The two threads of a row swap their halves' maxima
// through shared memory once per tile, so both take the same running maximum, and their
// P values feed one output accumulator O: per tile the tensor core runs two MMA chains
// (S and PV), and a switch between chains with different accumulators costs it a pipeline
// drain of a few hundred clocks.
//
//   warps 0-3 / 4-7   softmax groups 0 / 1 (TMEM lane = row, warp w serves lane quarter
//                     w % 4): tcgen05.ld of the group's 64 scores, mask (prefix length, or
//                     the ancestor bitmask on the tree tile), the half's maximum, the swap,
//                     P = 2^(s * c - m), tcgen05.st of P (bf16 pairs);
//   warp 8 lane 0     TMA: the Q tile once (a 3-D box over [B*N, Hq, D]), then the K tiles;
//   warp 8 lane 1     TMA: the V tiles (their own ring, so a K slot refills as soon as the
//                     S MMAs have read it, ahead of its V slot);
//   warp 9 lane 0     tcgen05.mma: S = Q K^T (M 128, N 128, K = D) and O += P V (M 128,
//                     N = D, K 128; P read from TMEM, V an MN-major operand straight from
//                     its TMA tile), in the order PV(t), S(t + 2);
//   warps 10-11       no role (a 384-thread block caps registers at 168, which three warps
//                     per SM sub-partition can hold).
// TMEM: three S buffers of 128 columns, then O (D columns).  S(t) goes to buffer t % 3, so
// the tensor core computes S(t + 1) while the groups work on tile t; the bf16 P of each
// half is written over the first 32 columns of that half of S(t).  S(t + 2) is issued after
// PV(t) into the buffer of S(t - 1) and P(t - 1), once the issuer has seen PV(t - 1)
// complete (pv_done): the ordering rests on barriers, not on the order in which the
// tensor core runs MMAs of different accumulators.  The groups wait for PV(t - 1) before
// they rescale O, and before they announce P(t), so they never run two barrier phases
// ahead of the MMA issuer.  O is rescaled lazily (each group its half of the columns),
// only when the row maximum grows by more than 2^8 over the reference the P values were
// taken against.  The last split also runs the tree tile: its K/V rows come by TMA from a
// 4-D view of the tree K/V ([B][N][Hkv][D], rows past N zero-filled).  Splits write
// (m, l, acc) partials for the log-sum-exp merge; a single split normalises and writes the
// output.
#pragma once

#include "attention.cuh"
#include "device_common.cuh"

namespace eagle {

constexpr int kTcRows = 128;                  // MMA M: query rows per CTA
constexpr int kTcHalf = kAttnKeys / 2;        // keys of a tile per softmax group
constexpr int kTcSoftmaxWarps = 8;            // two groups of four
constexpr int kTcLoadWarp = 8;                // lane 0: Q and K tiles; lane 1: V tiles
constexpr int kTcMmaWarp = 9;
constexpr int kTcThreads = 32 * 12;
constexpr float kTcRescaleThreshold = 8.0f;   // log2 units
// Of every 8 pairs of scores a softmax thread exponentiates, this many go through the
// polynomial 2^x on the FMA pipe (exp2_poly2) and the rest through the SFU, whose 16
// results per clock per SM would otherwise bound the softmax.
constexpr int kTcPolyPairs = 2;

template <int D>
struct TcSmem {
  static constexpr int kKStages = D == 128 ? 3 : 5;
  static constexpr int kVStages = D == 128 ? 2 : 5;
  static constexpr int kTile = kAttnKeys * D * 2;  // one K or V tile (D/64 boxes of 128 x 128 B)
  static constexpr int kQ = kTcRows * D * 2;        // D/64 boxes of 128 rows x 128 B
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQ;
  static constexpr int kVOff = kKOff + kKStages * kTile;
  static constexpr int kAncOff = kVOff + kVStages * kTile;
  static constexpr int kParOff = kAncOff + 64 * 8;
  // the halves' maxima per row and tile parity, [parity][group][row]; then the groups'
  // denominators per row for the epilogue, [group][row]
  static constexpr int kXchOff = kParOff + 64 * 4;
  static constexpr int kLOff = kXchOff + 2 * 2 * kTcRows * 4;
  static constexpr int kBarOff = kLOff + 2 * kTcRows * 4;
  // q_full, k_full[SK], k_empty[SK], v_full[SV], v_empty[SV], s_full[buffer], p_full,
  // pv_done, o_final
  static constexpr int kSBufs = 3;
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + kSBufs + 1 + 1 + 1;
  static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
  // TMEM columns: S(t) in buffer u = t % kSBufs at kSCol + kAttnKeys u (keys in column
  // order; the P of group g over the kTcHalf / 2 columns from kTcHalf g), O at kOCol
  static constexpr uint32_t kSCol = 0;
  static constexpr uint32_t kOCol = kSBufs * kAttnKeys;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kOCol + D <= kTmemCols, "TMEM columns");
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
  float* xch = reinterpret_cast<float*>(smem + SM::kXchOff);
  float* l_s = reinterpret_cast<float*>(smem + SM::kLOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + SK;
  uint64_t* v_full = k_empty + SK;
  uint64_t* v_empty = v_full + SV;
  uint64_t* s_full = v_empty + SV;  // [buffer]
  uint64_t* p_full = s_full + SM::kSBufs;
  uint64_t* pv_done = p_full + 1;
  uint64_t* o_final = pv_done + 1;
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
    for (int u = 0; u < SM::kSBufs; ++u) mbar_init(smem_u32(&s_full[u]), 1);
    mbar_init(smem_u32(p_full), kTcSoftmaxWarps);  // one arrival per softmax warp
    mbar_init(smem_u32(pv_done), 1);
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
          // the tree tile: nodes 0..127 of (b, kvh); nodes past N are zero-filled
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
      bool ok = mbar_wait(smem_u32(q_full), 0, kErrAttnMmaWait);
      // S(t) = Q K^T over the 128 keys of tile t, one M 128 x N 128 chain into buffer t % 3.
      // That buffer last held S(t - 3) and P(t - 3): both groups arrived on p_full before
      // PV(t - 3) was issued, and the issuer saw PV(t - 3) complete before it issued PV(t - 2),
      // which precedes this chain.
      auto issue_s = [&](int t) {
        const int s = t % SK;
        ok = ok && mbar_wait(smem_u32(&k_full[s]), (t / SK) & 1, kErrAttnMmaWait);
        tc_fence_after();
        const uint32_t kb = k_stage(s);
        const uint32_t d_tmem = tmem + SM::kSCol + static_cast<uint32_t>((t % SM::kSBufs) * kAttnKeys);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int h = kk >> 2, k4 = kk & 3;
          const uint64_t a = smem_desc_k_sw128(q_s + h * kTcRows * 128) + 2 * k4;
          const uint64_t bdesc = smem_desc_k_sw128(kb + h * kAttnKeys * 128) + 2 * k4;
          if (ok) tc_mma_f16(d_tmem, a, bdesc, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&s_full[t % SM::kSBufs]));
        tc_commit(smem_u32(&k_empty[s]));
      };
      // O += P V over the tile's 128 keys: 8 MMAs of 16 keys (8 TMEM columns of P from the
      // half that holds them, two 8-key groups of 1024 B of V; the second 64-column group
      // of V is the next TMA box)
      auto issue_pv = [&](int t) {
        const int s = t % SV;
        ok = ok && mbar_wait(smem_u32(p_full), t & 1, kErrAttnMmaWait);
        // PV(t - 1) complete: S(t + 2), issued next, may overwrite its P.  Waited for before
        // this PV's commit, so the barrier is never two phases ahead of this wait.
        if (t > 0) ok = ok && mbar_wait(smem_u32(pv_done), (t - 1) & 1, kErrAttnMmaWait);
        ok = ok && mbar_wait(smem_u32(&v_full[s]), (t / SV) & 1, kErrAttnMmaWait);
        tc_fence_after();
        const uint32_t vb = v_stage(s);
        const uint32_t pa = tmem + SM::kSCol + static_cast<uint32_t>((t % SM::kSBufs) * kAttnKeys);
        const uint32_t o_tmem = tmem + SM::kOCol;
#pragma unroll
        for (int kk = 0; kk < kAttnKeys / 16; ++kk) {
          const uint32_t a_col = static_cast<uint32_t>((kk >> 2) * kTcHalf + 8 * (kk & 3));
          const uint64_t bdesc = smem_desc_mn_sw128(vb + kk * 2048, kAttnKeys * 128, 1024);
          if (ok) tc_mma_f16_ts(o_tmem, pa + a_col, bdesc, idesc_o, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(smem_u32(pv_done));
        tc_commit(smem_u32(&v_empty[s]));
      };
      for (int t = 0; t < T && t < 2; ++t) issue_s(t);
      for (int t = 0; t < T; ++t) {
        issue_pv(t);
        if (t + 2 < T) issue_s(t + 2);
      }
      tc_commit(smem_u32(o_final));
    }
  } else if (warp < kTcSoftmaxWarps) {
    // ------------------------------------------------------------ softmax groups
    const int grp = warp >> 2;              // keys [64 grp, 64 grp + 64) of every tile
    const int quarter = warp & 3;           // TMEM lane quarter = row block of 32
    const int r = quarter * 32 + lane;      // query row = TMEM lane
    const int node = i0 + r / G;
    const int head = kvh * G + r % G;
    const bool rvalid = r < rows_blk && node < N;
    // a warp with no real row skips the score and output work (its rows of P and O are
    // never read for an output), but keeps every barrier
    const bool live = __any_sync(0xffffffffu, rvalid);
    const int tid = threadIdx.x;            // 0 .. 255
    constexpr int kSoftThreads = 32 * kTcSoftmaxWarps;
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
    // the tree keys are nodes 0..N-1 <= 63: all in group 0's half of the tree tile
    const uint64_t tree_bits = (last && rvalid && grp == 0) ? anc[node] : 0ull;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    // the half of O's columns this group rescales and writes out
    const uint32_t o_col = lane_base + SM::kOCol + static_cast<uint32_t>(grp * (D / 2));
    const float c = prm.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    for (int t = 0; t < T; ++t) {
      const bool tree = t >= nt;
      mbar_wait(smem_u32(&s_full[t % SM::kSBufs]), (t / SM::kSBufs) & 1, kErrAttnConsumerWait);
      tc_fence_after();
      // this group's half of S(t), and its P(t) over the half's first 32 columns
      const uint32_t s_col =
          lane_base + SM::kSCol + static_cast<uint32_t>((t % SM::kSBufs) * kAttnKeys + grp * kTcHalf);
      float tmax_half = -INFINITY;
      float x[kTcHalf];
      if (live) {
        uint32_t sa[32], sb[32];
        __syncwarp();  // the TMEM loads below are warp-wide
        tmem_ld_cols<32>(s_col, sa);
        tmem_ld_cols<32>(s_col + 32, sb);
        tmem_ld_wait();
        // visibility of this group's 64 keys
        const int first = tree ? 0 : (t_begin + t) * kAttnKeys;
        const int valid = (tree ? N : min(kAttnKeys, L - first)) - grp * kTcHalf;
        uint64_t vis = valid >= kTcHalf ? ~0ull : (valid <= 0 ? 0ull : ((1ull << valid) - 1ull));
        if (tree) vis &= tree_bits;
        if (!rvalid) vis = 0ull;
        // raw scores; masked ones (past L_b, outside the ancestor set, padding rows) become
        // -inf, which also drops any non-finite value the padding holds
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          x[j] = __uint_as_float(sa[j]);
          x[j + 32] = __uint_as_float(sb[j]);
        }
        if (vis != ~0ull) {
#pragma unroll
          for (int j = 0; j < kTcHalf; ++j) x[j] = ((vis >> j) & 1ull) ? x[j] : -INFINITY;
        }
        // row maximum by a tree of three-input maxima (32 instructions for 64 values)
        float m3[22];
#pragma unroll
        for (int j = 0; j < 21; ++j) m3[j] = fmax3f(x[3 * j], x[3 * j + 1], x[3 * j + 2]);
        m3[21] = x[63];
        float n3[8];
#pragma unroll
        for (int j = 0; j < 7; ++j) n3[j] = fmax3f(m3[3 * j], m3[3 * j + 1], m3[3 * j + 2]);
        n3[7] = m3[21];
        // in scaled log2 units (the scale is positive, so the maximum commutes with it)
        tmax_half =
            fmax3f(fmax3f(n3[0], n3[1], n3[2]), fmax3f(n3[3], n3[4], n3[5]), fmaxf(n3[6], n3[7])) * c;
      }
      // swap the halves' maxima: both threads of a row take the same maximum, so their P
      // values share one reference and one accumulator.  The slot of tile t is written again
      // at tile t + 2, after the other group has passed the swap of tile t + 1.
      float* xm = xch + (t & 1) * 2 * kTcRows;
      xm[grp * kTcRows + r] = tmax_half;
      asm volatile("bar.sync 1, %0;" ::"r"(kSoftThreads) : "memory");
      const float tmax = fmaxf(tmax_half, xm[(grp ^ 1) * kTcRows + r]);
      if (live) {
        const float m_new = fmaxf(m_ref, tmax);
        const bool rebase =
            m_new != -INFINITY && (m_ref == -INFINITY || m_new > m_ref + kTcRescaleThreshold);
        const bool scale_o = rebase && m_ref != -INFINITY;  // O holds P V taken against m_ref
        const float f = scale_o ? fast_exp2(m_ref - m_new) : 1.0f;
        if (rebase) {
          l *= f;
          m_ref = m_new;
        }
        // p = 2^(s * scale_log2 - m), one fused multiply-add per score; masked keys give
        // 2^-inf = 0 (and m = 0 while every key so far was masked)
        const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
        uint32_t w[kTcHalf / 2];
        float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < kTcHalf / 2; ++e) {
          const float2 y = ffma2(make_float2(x[2 * e], x[2 * e + 1]), make_float2(c, c), make_float2(neg_m, neg_m));
          float2 pe;
          if ((e & 7) < kTcPolyPairs) {
            pe = exp2_poly2(y);
          } else {
            pe.x = fast_exp2(y.x);
            pe.y = fast_exp2(y.y);
          }
          w[e] = pack_bf16x2(pe.x, pe.y);
          // the denominator sums the fp32 values; the MMA multiplies their bf16 roundings
          // (round to nearest: the difference averages out far below the bf16 tolerance)
          if (e & 1)
            ls1 = fadd2(ls1, pe);
          else
            ls0 = fadd2(ls0, pe);
        }
        ls0 = fadd2(ls0, ls1);
        l += ls0.x + ls0.y;
        // every score of this half of S(t) is in registers: its P goes over them
        tmem_st_cols<32>(s_col, w);
        // O holds P V taken against the old reference: rescale this group's half of its
        // columns once PV(t - 1) has landed.  TMEM loads/stores are warp-wide: the warp
        // rescales if any of its rows must (the other group's warp on the same rows decides
        // the same).
        if (__any_sync(0xffffffffu, scale_o)) {
          if (t > 0) mbar_wait(smem_u32(pv_done), (t - 1) & 1, kErrAttnConsumerWait);
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < D / 2; c0 += 16) {
            uint32_t ov[16];
            tmem_ld_cols<16>(o_col + c0, ov);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * f);
            tmem_st_cols<16>(o_col + c0, ov);
          }
        }
        tmem_st_wait();
      }
      if (!tree) {
        const int valid = min(kAttnKeys, L - (t_begin + t) * kAttnKeys);
        const int lo = max(valid, grp * kTcHalf), hi = (grp + 1) * kTcHalf;
        if (lo < hi) {
          // keys past L_b must not reach P V even if the padding holds non-finite values:
          // zero this group's rows of them in the tile's V slot once it has landed
          const int s = t % SV;
          mbar_wait(smem_u32(&v_full[s]), (t / SV) & 1, kErrAttnConsumerWait);
          const uint32_t vb = v_stage(s);
          const int gtid = tid & 127;
          for (int idx = gtid; idx < (hi - lo) * (D / 8); idx += 128) {
            const int j = lo + idx / (D / 8);
            const int d = (idx % (D / 8)) * 8;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vb + attn_swz(j, d)), "r"(0));
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
      }
      // PV(t - 1) issued means the issuer has taken p_full phase t - 1: arriving for phase t
      // cannot complete two phases ahead of its wait
      if (t > 0) mbar_wait(smem_u32(pv_done), (t - 1) & 1, kErrAttnConsumerWait);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(p_full));
    }

    // ------------------------------------------------------------ epilogue
    // both groups hold the same m_ref; the row's denominator is the sum of the halves'
    l_s[grp * kTcRows + r] = l;
    asm volatile("bar.sync 1, %0;" ::"r"(kSoftThreads) : "memory");
    const float mm = m_ref;
    const float lt = l_s[r] + l_s[kTcRows + r];
    if (T > 0) {
      mbar_wait(smem_u32(o_final), 0, kErrAttnConsumerWait);
      tc_fence_after();
    }
    const size_t prow_g = (static_cast<size_t>(b) * N + node) * prm.Hq + head;
    const bool single = prm.num_splits == 1;
    const float inv = (lt > 0.f) ? 1.0f / lt : 0.f;
    if (live) {
#pragma unroll 1
      for (int cc = grp * (D / 2); cc < (grp + 1) * (D / 2); cc += 16) {
        uint32_t a0[16];
        float ov[16];
        __syncwarp();  // the TMEM loads below are warp-wide
        if (T > 0) {
          tmem_ld_cols<16>(lane_base + SM::kOCol + cc, a0);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) ov[k] = __uint_as_float(a0[k]);
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) ov[k] = 0.f;
        }
        if (!rvalid) {
        } else if (single) {
          uint4* dst = reinterpret_cast<uint4*>(prm.out + prow_g * D + cc);
#pragma unroll
          for (int k = 0; k < 16; k += 8) {
            uint4 wv;
            wv.x = pack_bf16x2(ov[k] * inv, ov[k + 1] * inv);
            wv.y = pack_bf16x2(ov[k + 2] * inv, ov[k + 3] * inv);
            wv.z = pack_bf16x2(ov[k + 4] * inv, ov[k + 5] * inv);
            wv.w = pack_bf16x2(ov[k + 6] * inv, ov[k + 7] * inv);
            dst[k / 8] = wv;
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(prm.part_acc + (prow_g * prm.num_splits + split) * D + cc);
#pragma unroll
          for (int k = 0; k < 16; k += 4) dst[k / 4] = make_float4(ov[k], ov[k + 1], ov[k + 2], ov[k + 3]);
        }
      }
    }
    if (rvalid && !single && grp == 0)
      *reinterpret_cast<float2*>(prm.part_ml + (prow_g * prm.num_splits + split) * 2) = make_float2(mm, lt);
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
