// lm_head.cuh -- LM-head logits for every tree node:
//     logits[r, v] = sum_k hidden[r, k] * W[v, k]
// (EAGLE summary, section 3 "Draft model": the LM head turns the target's features into
// token distributions; every tree node is scored in the one verification pass).
//
// bf16 path: a tcgen05 tensor-core GEMM computed "swap-AB": the vocabulary is the MMA M
// dimension (128 rows of W per CTA) and the few tree rows are the MMA N dimension, so
// the weight W -- the only large operand -- streams through TMA once while the tree rows
// (tens to a few hundred) ride along.  One CTA = one 128-token vocabulary tile x one
// chunk of up to 256 tree rows.  Warp roles: warp 0 lane 0 issues TMA, warp 1 owns TMEM
// and lane 0 issues the MMAs, then all four warps drain TMEM and store fp32 logits with
// coalesced 128-byte rows (lane = vocabulary entry).
//
// f32 path: a plain fp32 SIMT tile GEMM (tensor cores cannot give fp32-exact products).
#pragma once

#include "device_common.cuh"

namespace eagle {

constexpr int kLmBlockV = 128;      // vocabulary rows per CTA (MMA M)
constexpr int kLmBlockK = 64;       // bf16 elements per 128-byte swizzle row
constexpr int kLmThreads = 128;

struct LmTcParams {
  float* logits;
  int32_t M;       // tree rows (B * N)
  int32_t V;
  int32_t H;
  int32_t bn;      // rows per CTA, multiple of 16, <= 256 (MMA N)
  int32_t stages;
  int32_t tmem_cols;
};

__host__ __device__ inline uint32_t lm_stage_bytes(int bn) {
  return static_cast<uint32_t>(kLmBlockV * kLmBlockK * 2 + bn * kLmBlockK * 2);
}

__global__ void __launch_bounds__(kLmThreads, 1)
    lm_head_tc_kernel(const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_h, const LmTcParams prm) {
  extern __shared__ uint8_t lm_smem_raw[];
  // 1024-byte alignment for the 128B-swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lm_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = prm.stages;
  const int bn = prm.bn;
  uint8_t* a_tiles = smem;                                    // S x 16 KB
  uint8_t* b_tiles = smem + S * kLmBlockV * kLmBlockK * 2;    // S x bn*128 B
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_tiles + S * bn * kLmBlockK * 2);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* accum = bars + 2 * S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 1);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * bn;
  const int v0 = blockIdx.y * kLmBlockV;
  const int KB = (prm.H + kLmBlockK - 1) / kLmBlockK;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_h);
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(accum), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(prm.tmem_cols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // the walk that consumes these logits may start its prologue now; it waits for this
  // grid's completion before reading them
  pdl_launch_dependents();

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    const uint32_t bytes = lm_stage_bytes(bn);
    const uint64_t pol_w = l2_policy_evict_first();  // W streams through once
    const uint64_t pol_h = l2_policy_evict_last();   // every vocabulary tile re-reads hidden
    int issued = 0;
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % S;
      const int n = kb / S;
      if (n > 0 && !mbar_wait(smem_u32(&empty[s]), (n - 1) & 1, kErrLmProducerWait)) {
        *abort_flag = 1;
        break;
      }
      if (*abort_flag) break;
      const uint32_t fb = smem_u32(&full[s]);
      mbar_arrive_expect_tx(fb, bytes);
      tma_load_2d_hint(smem_u32(a_tiles + s * kLmBlockV * kLmBlockK * 2), &tm_w, fb, kb * kLmBlockK,
                       v0, pol_w);
      tma_load_2d_hint(smem_u32(b_tiles + s * bn * kLmBlockK * 2), &tm_h, fb, kb * kLmBlockK, r0,
                       pol_h);
      issued = kb + 1;
    }
    if (*abort_flag) {
      // Drain: every issued load must land before this CTA's shared memory is released.
      for (int kb = (issued > S ? issued - S : 0); kb < issued; ++kb)
        mbar_wait(smem_u32(&full[kb % S]), (kb / S) & 1, kErrLmProducerWait);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kLmBlockV, bn);
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % S;
      if (!mbar_wait(smem_u32(&full[s]), (kb / S) & 1, kErrLmMmaWait)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a_addr = smem_u32(a_tiles + s * kLmBlockV * kLmBlockK * 2);
      const uint32_t b_addr = smem_u32(b_tiles + s * bn * kLmBlockK * 2);
      const uint64_t a_desc = smem_desc_k_sw128(a_addr);
      const uint64_t b_desc = smem_desc_k_sw128(b_addr);
#pragma unroll
      for (int k = 0; k < kLmBlockK / 16; ++k) {
        // +32 bytes per 16-element K step inside the 128-byte swizzle row (>> 4 = 2)
        tc_mma_f16(tmem, a_desc + 2 * k, b_desc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
      }
      tc_commit(smem_u32(&empty[s]));
    }
    // Always signal: on the abort path this still orders the TMEM release after every
    // MMA already issued.
    tc_commit(smem_u32(accum));
  }
  __syncwarp();

  // ---------------- epilogue: TMEM -> registers -> global (all 4 warps)
  const bool have = mbar_wait(smem_u32(accum), 0, kErrLmEpilogueWait);
  tc_fence_after();
  if (have && !*abort_flag) {
    const int v = v0 + warp * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float* out = prm.logits;
    for (int c0 = 0; c0 < bn; c0 += 16) {
      uint32_t r[16];
      __syncwarp();  // the TMEM load below is warp-wide
      tmem_ld_32x32b_x16(lane_base + c0, r);
      tmem_ld_wait();
      if (v < prm.V) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int row = r0 + c0 + j;
          if (row < prm.M) out[static_cast<size_t>(row) * prm.V + v] = __uint_as_float(r[j]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(prm.tmem_cols));
  }
}

// ------------------------------------------------------------------ persistent bf16 path
// For many tree rows (M > 256, where the GEMM is bound by the tensor cores rather than by
// the weight stream): one CTA per SM walks a list of (vocabulary tile, row chunk) tiles,
// row chunk fastest, so the CTAs working on the chunks of one vocabulary tile run side by
// side and W is read from HBM about once.  Warp roles: warp 0 lane 0 issues TMA (W boxes and
// a hidden box per k block, one ring), warp 1 owns TMEM and lane 0 issues the MMAs, warps 2-5
// drain TMEM (warp w reads TMEM lanes 32 * (w % 4) ..) and store fp32 logits in coalesced
// 128-byte rows.  Two tile shapes (kVB vocabulary blocks of 128 rows per tile):
//   kVB = 1  two TMEM accumulators (2 x 256 columns): the epilogue drains tile j while the
//            MMAs of tile j + 1 run;
//   kVB = 2  one accumulator per block (the same 512 columns): every k block's hidden tile
//            feeds two MMAs, so a tile moves a third fewer bytes through shared memory per
//            MMA (the bound of this GEMM: TMA writes plus operand reads per stage), at the
//            price of the MMAs waiting for each tile's epilogue.

constexpr int kLmpThreads = 192;
constexpr int kLmpAccCols = 256;  // columns per accumulator

struct LmpParams {
  float* logits;
  int32_t M, V, H;
  int32_t bn;       // rows per chunk, multiple of 16, <= 256
  int32_t chunks;   // row chunks (ceil(M / bn))
  int32_t vtiles;   // vocabulary tiles of 128 * kVB
  int32_t stages;
};

__host__ __device__ inline uint32_t lmp_stage_bytes(int vb, int bn) {
  return static_cast<uint32_t>(vb * kLmBlockV * kLmBlockK * 2 + bn * kLmBlockK * 2);
}
__host__ __device__ inline size_t lmp_smem_bytes(int vb, int bn, int stages) {
  return 1024 + static_cast<size_t>(stages) * lmp_stage_bytes(vb, bn) + (2 * stages + 5) * 8 + 16;
}

template <int kVB>
__global__ void __launch_bounds__(kLmpThreads, 1)
    lm_head_tc_persist_kernel(const __grid_constant__ CUtensorMap tm_w,
                              const __grid_constant__ CUtensorMap tm_h, const LmpParams prm) {
  static_assert(kVB == 1 || kVB == 2, "one or two vocabulary blocks per tile");
  constexpr int NA = kVB == 1 ? 2 : 1;  // accumulator sets in flight
  constexpr uint32_t kWBox = kLmBlockV * kLmBlockK * 2;
  extern __shared__ uint8_t lmp_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lmp_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = prm.stages;
  const int bn = prm.bn;
  uint8_t* a_tiles = smem;                                    // S x kVB x 16 KB
  uint8_t* b_tiles = smem + S * kVB * kWBox;                  // S x bn*128 B
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_tiles + S * bn * kLmBlockK * 2);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* acc_full = bars + 2 * S;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = (prm.H + kLmBlockK - 1) / kLmBlockK;
  const int num_tiles = prm.vtiles * prm.chunks;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_h);
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 4);  // one arrival per epilogue warp
    }
    mbar_init(smem_u32(mma_done), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kLmpAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      const uint32_t bytes = lmp_stage_bytes(kVB, bn);
      const uint64_t pol_h = l2_policy_evict_last();  // every tile re-reads hidden
      int it = 0, issued = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
        const int c = tile % prm.chunks, v0 = (tile / prm.chunks) * (kVB * kLmBlockV);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S, n = it / S;
          if (n > 0 && !mbar_wait(smem_u32(&empty[s]), (n - 1) & 1, kErrLmProducerWait)) {
            *abort_flag = 1;
            break;
          }
          const uint32_t fb = smem_u32(&full[s]);
          mbar_arrive_expect_tx(fb, bytes);
#pragma unroll
          for (int vb = 0; vb < kVB; ++vb)
            tma_load_2d(smem_u32(a_tiles + (s * kVB + vb) * kWBox), &tm_w, fb, kb * kLmBlockK,
                        v0 + vb * kLmBlockV);
          tma_load_2d_hint(smem_u32(b_tiles + s * bn * kLmBlockK * 2), &tm_h, fb, kb * kLmBlockK, c * bn,
                           pol_h);
          issued = it + 1;
        }
      }
      // every issued load lands before this CTA's shared memory can be released
      for (int k = (issued > S ? issued - S : 0); k < issued; ++k)
        mbar_wait(smem_u32(&full[k % S]), (k / S) & 1, kErrLmProducerWait);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kLmBlockV, bn);
      int it = 0, j = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x, ++j) {
        const int a = j % NA;
        if (j >= NA && !mbar_wait(smem_u32(&acc_empty[a]), (j / NA - 1) & 1, kErrLmMmaWait)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        // accumulator of block vb: set a (kVB = 1) or block vb (kVB = 2), 256 columns each
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(a * kLmpAccCols);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(smem_u32(&full[s]), (it / S) & 1, kErrLmMmaWait)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t b_desc = smem_desc_k_sw128(smem_u32(b_tiles + s * bn * kLmBlockK * 2));
#pragma unroll
          for (int k = 0; k < kLmBlockK / 16; ++k)
#pragma unroll
            for (int vb = 0; vb < kVB; ++vb) {
              const uint64_t a_desc = smem_desc_k_sw128(smem_u32(a_tiles + (s * kVB + vb) * kWBox));
              tc_mma_f16(d_tmem + static_cast<uint32_t>(vb * kLmpAccCols), a_desc + 2 * k, b_desc + 2 * k, idesc,
                         (kb | k) != 0 ? 1u : 0u);
            }
          tc_commit(smem_u32(&empty[s]));
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        tc_commit(smem_u32(&acc_full[a]));
      }
      // orders the TMEM release after every MMA issued
      tc_commit(smem_u32(mma_done));
    }
  } else {
    // ---------------- epilogue: TMEM -> registers -> global (warps 2-5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int j = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++j) {
      const int a = j % NA;
      if (!mbar_wait(smem_u32(&acc_full[a]), (j / NA) & 1, kErrLmEpilogueWait)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int c = tile % prm.chunks, v0 = (tile / prm.chunks) * (kVB * kLmBlockV);
      const int r0 = c * bn;
      float* out = prm.logits;
      for (int vb = 0; vb < kVB; ++vb) {
        const int v = v0 + vb * kLmBlockV + q * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>((a + vb) * kLmpAccCols);
        for (int c0 = 0; c0 < bn; c0 += 16) {
          uint32_t r[16];
          __syncwarp();  // the TMEM load below is warp-wide
          tmem_ld_32x32b_x16(lane_base + c0, r);
          tmem_ld_wait();
          if (v < prm.V) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int row = r0 + c0 + e;
              if (row < prm.M) out[static_cast<size_t>(row) * prm.V + v] = __uint_as_float(r[e]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[a]));
    }
  }
  __syncwarp();
  if (warp == 1) {
    if (lane == 0) mbar_wait(smem_u32(mma_done), 0, kErrLmMmaWait);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kLmpAccCols);
  }
}

// ------------------------------------------------------------------ fp32 SIMT path

constexpr int kLmF32TileV = 64;
constexpr int kLmF32TileR = 16;
constexpr int kLmF32TileK = 128;  // 41 KB of tiles: few dependent memory round trips per row

__global__ void __launch_bounds__(256)
    lm_head_f32_kernel(const float* __restrict__ hidden, const float* __restrict__ w,
                       float* __restrict__ logits, int M, int V, int H) {
  __shared__ float ws[kLmF32TileV][kLmF32TileK + 1];
  __shared__ float hs[kLmF32TileR][kLmF32TileK + 1];
  const int tv = threadIdx.x % kLmF32TileV;      // vocabulary entry within the tile
  const int tr = threadIdx.x / kLmF32TileV;      // 0..3: rows tr*4 .. tr*4+3
  const int v0 = blockIdx.x * kLmF32TileV;
  const int r0 = blockIdx.y * kLmF32TileR;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < H; k0 += kLmF32TileK) {
    // every load of the tile is issued before any is stored, so a tile costs one memory
    // round trip (a load-store loop would wait for each load in turn)
    constexpr int kWPer = kLmF32TileV * kLmF32TileK / 256, kHPer = kLmF32TileR * kLmF32TileK / 256;
    float wr[kWPer], hr[kHPer];
#pragma unroll
    for (int e = 0; e < kWPer; ++e) {
      const int idx = threadIdx.x + e * 256;
      const int vv = idx / kLmF32TileK, kk = idx % kLmF32TileK;
      const int gv = v0 + vv, gk = k0 + kk;
      wr[e] = (gv < V && gk < H) ? w[static_cast<size_t>(gv) * H + gk] : 0.f;
    }
#pragma unroll
    for (int e = 0; e < kHPer; ++e) {
      const int idx = threadIdx.x + e * 256;
      const int rr = idx / kLmF32TileK, kk = idx % kLmF32TileK;
      const int gr = r0 + rr, gk = k0 + kk;
      hr[e] = (gr < M && gk < H) ? hidden[static_cast<size_t>(gr) * H + gk] : 0.f;
    }
#pragma unroll
    for (int e = 0; e < kWPer; ++e) {
      const int idx = threadIdx.x + e * 256;
      ws[idx / kLmF32TileK][idx % kLmF32TileK] = wr[e];
    }
#pragma unroll
    for (int e = 0; e < kHPer; ++e) {
      const int idx = threadIdx.x + e * 256;
      hs[idx / kLmF32TileK][idx % kLmF32TileK] = hr[e];
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kLmF32TileK; ++kk) {
      const float wv = ws[tv][kk];
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] = fmaf(hs[tr * 4 + j][kk], wv, acc[j]);
    }
    __syncthreads();
  }
  const int v = v0 + tv;
  if (v < V) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = r0 + tr * 4 + j;
      if (row < M) logits[static_cast<size_t>(row) * V + v] = acc[j];
    }
  }
}

}  // namespace eagle
