// eagle_verify.cu -- C ABI of the draft-tree verification library (declared in
// include/eagle_verify.h): argument validation, launch planning, TMA descriptor encoding
// and the launches of the tree-attention, LM-head and accept kernels.
//
// Everything the host can check is checked before anything is enqueued; no entry point
// allocates memory or synchronises the caller's stream.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/eagle_verify.h"
#include "accept.cuh"
#include "attention.cuh"
#include "attention_tc.cuh"
#include "commit.cuh"
#include "draft.cuh"
#include "rerank.cuh"
#include "device_common.cuh"
#include "lm_head.cuh"

namespace eagle {
namespace {

constexpr int kNumSMs = 148;            // B200; launch planning targets this count
constexpr int kMaxDevices = 64;

// ------------------------------------------------------------------ validation

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

eagle_status_t check_shape(const eagle_shape_t* s) {
  if (s == nullptr) return EAGLE_ERR_INVALID_ARGUMENT;
  if (s->batch < 1 || s->batch > 65535) return EAGLE_ERR_INVALID_ARGUMENT;
  // N <= 64 also keeps node indices inside the Philox counter's 8-bit node field
  static_assert(64 - 1 <= kPhiloxMaxField, "tree nodes must fit the counter's node field");
  if (s->num_nodes < 1 || s->num_nodes > 64) return EAGLE_ERR_INVALID_ARGUMENT;
  if (s->num_q_heads < 1 || s->num_kv_heads < 1 || s->num_q_heads % s->num_kv_heads != 0)
    return EAGLE_ERR_INVALID_ARGUMENT;
  if (s->head_dim != 64 && s->head_dim != 128) return EAGLE_ERR_INVALID_ARGUMENT;
  if (s->max_prefix_len < 1) return EAGLE_ERR_INVALID_ARGUMENT;
  if (s->hidden < 1 || s->vocab < 1) return EAGLE_ERR_INVALID_ARGUMENT;
  if (s->dtype != EAGLE_DTYPE_F32 && s->dtype != EAGLE_DTYPE_BF16) return EAGLE_ERR_INVALID_ARGUMENT;
  if (s->dtype == EAGLE_DTYPE_BF16 && s->hidden % 8 != 0) return EAGLE_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(s->softmax_scale)) return EAGLE_ERR_INVALID_ARGUMENT;
  return EAGLE_OK;
}

float softmax_scale(const eagle_shape_t* s) {
  return s->softmax_scale > 0.f ? s->softmax_scale : 1.0f / std::sqrt(static_cast<float>(s->head_dim));
}

// ------------------------------------------------------------------ planning

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct AttnPlan {
  int nodes_per_block;
  int row_blocks;
  int splits;
  int tiles_per_split;
  size_t acc_bytes;  // split partials (0 with a single split)
  size_t ml_bytes;
};

// Split the prefix so that (sequences x kv heads x row blocks x splits) runs in as few
// waves of one CTA per SM as the work allows (the kernel's shared memory allows one).
AttnPlan plan_attention(const eagle_shape_t* s) {
  AttnPlan p{};
  const int G = s->num_q_heads / s->num_kv_heads;
  if (s->dtype == EAGLE_DTYPE_BF16) {
    // tensor-core path: a 128-row tile holds floor(128 / G) nodes x G heads
    p.nodes_per_block = G <= kTcRows ? kTcRows / G : 1;
    p.row_blocks = (s->num_nodes + p.nodes_per_block - 1) / p.nodes_per_block;
  } else {
    p.nodes_per_block = 0;
    p.row_blocks = 1;
  }
  const int max_tiles = (s->max_prefix_len + kAttnKeys - 1) / kAttnKeys;
  // pick the split count that minimises waves x (tiles per split + a CTA's fixed cost,
  // about two tiles' time: set-up, pipeline fill, the tree tile, the partials it writes
  // for the merge)
  const long base = static_cast<long>(s->batch) * s->num_kv_heads * p.row_blocks;
  int best_splits = 1;
  long best_cost = -1;
  for (int sp = 1; sp <= (max_tiles > 0 ? max_tiles : 1); ++sp) {
    const long tiles_per = max_tiles > 0 ? (max_tiles + sp - 1) / sp : 0;
    if (sp > 1 && (tiles_per - 1) * sp >= max_tiles) continue;  // same split count as a smaller sp
    const long waves = (base * sp + kNumSMs - 1) / kNumSMs;
    const long cost = waves * (tiles_per + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_splits = sp;
    }
  }
  int tiles_per = max_tiles > 0 ? (max_tiles + best_splits - 1) / best_splits : 1;
  if (tiles_per < 1) tiles_per = 1;
  p.tiles_per_split = tiles_per;
  p.splits = max_tiles > 0 ? (max_tiles + tiles_per - 1) / tiles_per : 1;
  if (s->dtype != EAGLE_DTYPE_BF16 || p.splits == 1) {
    p.splits = s->dtype == EAGLE_DTYPE_BF16 ? p.splits : 1;
    p.acc_bytes = p.ml_bytes = 0;
    return p;
  }
  const size_t rows = static_cast<size_t>(s->batch) * s->num_nodes * s->num_q_heads;
  p.acc_bytes = align256(rows * p.splits * s->head_dim * sizeof(float));
  p.ml_bytes = align256(rows * p.splits * 2 * sizeof(float));
  return p;
}

struct LmPlan {
  int chunks;
  int bn;
  int stages;
  int tmem_cols;
  size_t smem;
};

LmPlan plan_lm_head(const eagle_shape_t* s, int max_stages = 8) {
  LmPlan p{};
  const long M = static_cast<long>(s->batch) * s->num_nodes;
  p.chunks = static_cast<int>((M + 255) / 256);
  const long per = (M + p.chunks - 1) / p.chunks;
  p.bn = static_cast<int>(((per + 15) / 16) * 16);
  const uint32_t stage = lm_stage_bytes(p.bn);
  // small row counts: keep two CTAs per SM in flight; large ones: deepest ring in one CTA
  if (stage * 4 <= 104 * 1024) {
    p.stages = static_cast<int>((104 * 1024) / stage);
  } else {
    p.stages = static_cast<int>((200 * 1024) / stage);
  }
  if (p.stages > max_stages) p.stages = max_stages;
  if (p.stages < 2) p.stages = 2;
  int cols = 32;
  while (cols < p.bn) cols <<= 1;
  p.tmem_cols = cols;
  p.smem = 1024 + static_cast<size_t>(p.stages) * stage + (2 * p.stages + 1) * 8 + 16;
  return p;
}

struct AccPlan {
  int cluster;
  int slice;
  int nq;
  size_t smem;
};

constexpr size_t kAccSmemBudget = 200 * 1024;

// One cluster per sequence: 16 CTAs (a non-portable size) for large vocabularies, fewer
// for small ones; each CTA holds its slice of the logits row, two residual buffers and
// up to four prefetched draft rows (plus the race keys of the current node).
AccPlan plan_accept(const eagle_shape_t* s, int max_cluster = kAccMaxCluster) {
  AccPlan p{};
  int cl = s->vocab >= 16384 ? 16 : (s->vocab + 2047) / 2048;
  if (cl < 1) cl = 1;
  if (cl > max_cluster) cl = max_cluster;
  p.cluster = cl;
  const int per = (s->vocab + cl - 1) / cl;
  p.slice = ((per + 3) / 4) * 4;
  const size_t row = static_cast<size_t>(p.slice) * sizeof(float);
  const long nq = static_cast<long>(kAccSmemBudget / row) - kAccFixedBufs;
  p.nq = static_cast<int>(nq < 0 ? 0 : (nq > kAccMaxQBuf ? kAccMaxQBuf : nq));
  p.smem = static_cast<size_t>(kAccFixedBufs + (p.nq > 0 ? p.nq : 1)) * row;
  return p;
}

constexpr size_t kAccMaxSmem = kAccSmemBudget;

// ------------------------------------------------------------------ workspace

size_t attention_ws_bytes(const eagle_shape_t* s) {
  const AttnPlan p = plan_attention(s);
  return p.acc_bytes + p.ml_bytes;
}

// ------------------------------------------------------------------ driver entry point

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_bf16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUresult r =
      enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
          dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ per-device state

struct DeviceState {
  std::once_flag attrs_once;
  bool attrs_ok = false;
  int max_cluster = 8;
  // eagle_verify_step's second stream and its fork/join events, made on first use
  std::once_flag side_once;
  bool side_ok = false;
  cudaStream_t side = nullptr;
  cudaEvent_t lm_mark = nullptr;  // LM head completed
  cudaEvent_t attn_done = nullptr;
  std::mutex step_mu;  // one step's fork/join sequence at a time on the shared side stream
  // eagle_draft_select: shared-memory limits set once; clusters of S CTAs resident at once,
  // [kernel mode][log2 S][slice bytes in 4 KB steps], stored + 1 (0: not queried yet)
  std::once_flag draft_once;
  bool draft_ok = false;
  int draft_max_cluster = kDraftPortableCluster;  // 16 where the device co-schedules them
  std::mutex draft_mu;
  int draft_clusters[3][5][kDraftMaxSmem / 4096 + 1] = {};
};
DeviceState g_dev[kMaxDevices];

bool current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return false;
  return *dev >= 0 && *dev < kMaxDevices;
}

bool ensure_attributes(int dev) {
  DeviceState& st = g_dev[dev];
  std::call_once(st.attrs_once, [&] {
    bool ok = true;
    ok &= cudaFuncSetAttribute(lm_head_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) == cudaSuccess;
    ok &= cudaFuncSetAttribute(lm_head_tc_persist_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) == cudaSuccess;
    ok &= cudaFuncSetAttribute(lm_head_tc_persist_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tree_attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               TcSmem<64>::kAlloc) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tree_attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               TcSmem<128>::kAlloc) == cudaSuccess;
    const void* walks[2] = {reinterpret_cast<const void*>(tree_accept_kernel<true>),
                            reinterpret_cast<const void*>(tree_accept_kernel<false>)};
    bool nonportable = true;
    for (const void* k : walks) {
      ok &= cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kAccMaxSmem)) == cudaSuccess;
      nonportable &= cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    }
    // 16-CTA clusters if the device can co-schedule them, else the portable 8
    st.max_cluster = 8;
    if (nonportable) {
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(16);
      cfg.blockDim = dim3(kAccThreads);
      cfg.dynamicSmemBytes = kAccMaxSmem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 16;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, tree_accept_kernel<true>, &cfg) == cudaSuccess && n >= 1)
        st.max_cluster = 16;
    }
    cudaGetLastError();
    st.attrs_ok = ok;
  });
  return st.attrs_ok;
}

bool ensure_side(int dev) {
  DeviceState& st = g_dev[dev];
  std::call_once(st.side_once, [&] {
    st.side_ok = cudaStreamCreateWithFlags(&st.side, cudaStreamNonBlocking) == cudaSuccess &&
                 cudaEventCreateWithFlags(&st.lm_mark, cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&st.attn_done, cudaEventDisableTiming) == cudaSuccess;
    cudaGetLastError();
  });
  return st.side_ok;
}

eagle_status_t launch_status() {
  return cudaGetLastError() == cudaSuccess ? EAGLE_OK : EAGLE_ERR_CUDA;
}

// ------------------------------------------------------------------ launches

eagle_status_t run_attention(const eagle_shape_t* s, const void* q, const void* kp, const void* vp,
                             const int32_t* lens, const void* kt, const void* vt,
                             const int32_t* parents, void* out, void* ws, cudaStream_t st) {
  const int B = s->batch, N = s->num_nodes, Hq = s->num_q_heads, Hkv = s->num_kv_heads;
  const int D = s->head_dim, Lmax = s->max_prefix_len;
  const float scale = softmax_scale(s);
  if (s->dtype == EAGLE_DTYPE_F32) {
    const int rows = B * N * Hq;
    const dim3 grid((rows + 3) / 4);
    if (D == 64)
      tree_attn_f32_kernel<64><<<grid, 128, 0, st>>>(
          static_cast<const float*>(q), static_cast<const float*>(kp), static_cast<const float*>(vp), lens,
          static_cast<const float*>(kt), static_cast<const float*>(vt), parents, static_cast<float*>(out), B,
          N, Hq, Hkv, Lmax, scale);
    else
      tree_attn_f32_kernel<128><<<grid, 128, 0, st>>>(
          static_cast<const float*>(q), static_cast<const float*>(kp), static_cast<const float*>(vp), lens,
          static_cast<const float*>(kt), static_cast<const float*>(vt), parents, static_cast<float*>(out), B,
          N, Hq, Hkv, Lmax, scale);
    return launch_status();
  }
  const AttnPlan plan = plan_attention(s);
  const int G = Hq / Hkv;
  CUtensorMap tq, tk, tv, tkt, tvt;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Lmax),
                              static_cast<cuuint64_t>(B) * Hkv};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Lmax) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kAttnKeys), 1};
  // queries viewed as [B*N, Hq, D]: one box = G heads x nodes_per_block nodes of a kv head
  const cuuint64_t qdims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hq),
                               static_cast<cuuint64_t>(B) * s->num_nodes};
  const cuuint64_t qstrides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Hq) * D * 2};
  const cuuint32_t qbox[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(plan.nodes_per_block)};
  // tree K/V viewed as [B][N][Hkv][D]: one box = the 64 node rows of (b, kv head), rows
  // past N outside the tensor (zero-filled)
  const cuuint64_t tdims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv),
                               static_cast<cuuint64_t>(s->num_nodes), static_cast<cuuint64_t>(B)};
  const cuuint64_t tstrides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Hkv) * D * 2,
                                  static_cast<cuuint64_t>(s->num_nodes) * Hkv * D * 2};
  const cuuint32_t tbox[4] = {64, 1, static_cast<cuuint32_t>(kAttnKeys), 1};
  if (!encode_bf16(&tk, kp, 3, dims, strides, box) || !encode_bf16(&tv, vp, 3, dims, strides, box) ||
      !encode_bf16(&tq, q, 3, qdims, qstrides, qbox) || !encode_bf16(&tkt, kt, 4, tdims, tstrides, tbox) ||
      !encode_bf16(&tvt, vt, 4, tdims, tstrides, tbox))
    return EAGLE_ERR_CUDA;
  TcAttnParams tp{};
  AttnParams& prm = tp.a;
  tp.nodes_per_block = plan.nodes_per_block;
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.k_tree = static_cast<const __nv_bfloat16*>(kt);
  prm.v_tree = static_cast<const __nv_bfloat16*>(vt);
  prm.prefix_lens = lens;
  prm.parents = parents;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.part_acc = static_cast<float*>(ws);
  prm.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + plan.acc_bytes);
  prm.B = B;
  prm.N = s->num_nodes;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = G;
  prm.Lmax = Lmax;
  prm.num_splits = plan.splits;
  prm.tiles_per_split = plan.tiles_per_split;
  prm.scale_log2 = scale * 1.4426950408889634f;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(plan.row_blocks, plan.splits, B * Hkv);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = D == 64 ? TcSmem<64>::kAlloc : TcSmem<128>::kAlloc;
  cfg.stream = st;
  cudaError_t e;
  e = D == 64 ? cudaLaunchKernelEx(&cfg, tree_attn_tc_kernel<64>, tq, tk, tv, tkt, tvt, tp)
              : cudaLaunchKernelEx(&cfg, tree_attn_tc_kernel<128>, tq, tk, tv, tkt, tvt, tp);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EAGLE_ERR_CUDA;
  }
  eagle_status_t rc = launch_status();
  if (rc != EAGLE_OK || plan.splits == 1) return rc;
  const int rows = B * N * Hq;
  const dim3 cgrid((rows + 3) / 4);
  if (D == 64)
    tree_attn_combine_kernel<64><<<cgrid, 128, 0, st>>>(prm.part_acc, prm.part_ml, prm.out, rows, plan.splits);
  else
    tree_attn_combine_kernel<128><<<cgrid, 128, 0, st>>>(prm.part_acc, prm.part_ml, prm.out, rows, plan.splits);
  return launch_status();
}

// Many tree rows (more than one chunk of 256): the persistent kernel, one CTA per SM, the
// chunks of a vocabulary tile on neighbouring CTAs.  Tiles of two 128-row vocabulary blocks
// (a third fewer shared-memory bytes per MMA; each tile's epilogue not overlapped) when
// there are enough of them to keep the last round of tiles short (six per SM), else single
// blocks with the epilogue of one tile under the MMAs of the next.
eagle_status_t run_lm_head_persistent(const eagle_shape_t* s, const void* hidden, const void* w,
                                      float* logits, cudaStream_t st, const LmPlan& plan) {
  const int M = s->batch * s->num_nodes, V = s->vocab, H = s->hidden;
  CUtensorMap tw, th;
  const cuuint64_t wd[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(V)};
  const cuuint64_t hd[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(M)};
  const cuuint64_t stride[1] = {static_cast<cuuint64_t>(H) * 2};
  const cuuint32_t wbox[2] = {static_cast<cuuint32_t>(kLmBlockK), static_cast<cuuint32_t>(kLmBlockV)};
  const cuuint32_t hbox[2] = {static_cast<cuuint32_t>(kLmBlockK), static_cast<cuuint32_t>(plan.bn)};
  if (!encode_bf16(&tw, w, 2, wd, stride, wbox) || !encode_bf16(&th, hidden, 2, hd, stride, hbox))
    return EAGLE_ERR_CUDA;
  const long wide_tiles = static_cast<long>((V + 2 * kLmBlockV - 1) / (2 * kLmBlockV)) * plan.chunks;
  const int vb = wide_tiles >= 6L * kNumSMs ? 2 : 1;
  const int vtiles = (V + vb * kLmBlockV - 1) / (vb * kLmBlockV);
  int stages = 2;
  while (stages < 8 && lmp_smem_bytes(vb, plan.bn, stages + 1) <= 220 * 1024) ++stages;
  LmpParams prm{logits, M, V, H, plan.bn, plan.chunks, vtiles, stages};
  const size_t smem = lmp_smem_bytes(vb, plan.bn, stages);
  const long tiles = static_cast<long>(vtiles) * plan.chunks;
  const int grid = static_cast<int>(tiles < kNumSMs ? tiles : kNumSMs);
  if (vb == 2)
    lm_head_tc_persist_kernel<2><<<grid, kLmpThreads, smem, st>>>(tw, th, prm);
  else
    lm_head_tc_persist_kernel<1><<<grid, kLmpThreads, smem, st>>>(tw, th, prm);
  return launch_status();
}

eagle_status_t run_lm_head(const eagle_shape_t* s, const void* hidden, const void* w, float* logits,
                           cudaStream_t st) {
  const int M = s->batch * s->num_nodes, V = s->vocab, H = s->hidden;
  if (s->dtype == EAGLE_DTYPE_F32) {
    const dim3 grid((V + kLmF32TileV - 1) / kLmF32TileV, (M + kLmF32TileR - 1) / kLmF32TileR);
    lm_head_f32_kernel<<<grid, 256, 0, st>>>(static_cast<const float*>(hidden), static_cast<const float*>(w),
                                             logits, M, V, H);
    return launch_status();
  }
  const LmPlan plan = plan_lm_head(s);
  if (plan.chunks > 1) return run_lm_head_persistent(s, hidden, w, logits, st, plan);
  CUtensorMap tw, th;
  const cuuint64_t wd[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(V)};
  const cuuint64_t hd[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(M)};
  const cuuint64_t stride[1] = {static_cast<cuuint64_t>(H) * 2};
  const cuuint32_t wbox[2] = {static_cast<cuuint32_t>(kLmBlockK), static_cast<cuuint32_t>(kLmBlockV)};
  const cuuint32_t hbox[2] = {static_cast<cuuint32_t>(kLmBlockK), static_cast<cuuint32_t>(plan.bn)};
  if (!encode_bf16(&tw, w, 2, wd, stride, wbox) || !encode_bf16(&th, hidden, 2, hd, stride, hbox))
    return EAGLE_ERR_CUDA;
  LmTcParams prm{logits, M, V, H, plan.bn, plan.stages, plan.tmem_cols};
  const dim3 grid(plan.chunks, (V + kLmBlockV - 1) / kLmBlockV);
  lm_head_tc_kernel<<<grid, kLmThreads, plan.smem, st>>>(tw, th, prm);
  return launch_status();
}

eagle_status_t run_accept(const eagle_shape_t* s, const float* logits, const float* draft,
                          const int32_t* tokens, const int32_t* parents, float T, uint64_t seed,
                          uint64_t offset, int32_t* acc, int32_t* alen, int32_t* next,
                          cudaStream_t st, bool pdl = false) {
  int dev = 0;
  cudaGetDevice(&dev);
  const AccPlan plan = plan_accept(s, g_dev[dev].max_cluster);
  AccParams prm{};
  prm.logits = logits;
  prm.draft = draft;
  prm.tokens = tokens;
  prm.parents = parents;
  prm.accepted_nodes = acc;
  prm.accept_len = alen;
  prm.next_token = next;
  prm.N = s->num_nodes;
  prm.V = s->vocab;
  prm.slice = plan.slice;
  prm.nq = plan.nq > 0 ? plan.nq : 1;
  prm.T = T;
  prm.seed = seed;
  prm.offset = offset;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(s->batch * plan.cluster);
  cfg.blockDim = dim3(kAccThreads);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // with `pdl` (right behind the LM head of the same step): may start while the LM head
  // drains; the kernel waits for that grid before it reads the logits
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  cudaError_t e;
  if (s->vocab % 4 == 0)
    e = cudaLaunchKernelEx(&cfg, tree_accept_kernel<true>, prm);
  else
    e = cudaLaunchKernelEx(&cfg, tree_accept_kernel<false>, prm);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EAGLE_ERR_CUDA;
  }
  return launch_status();
}

eagle_status_t run_commit(const eagle_shape_t* s, void* kp, void* vp, const int32_t* lens,
                          const void* kt, const void* vt, const void* hidden, const int32_t* parents,
                          const int32_t* acc, const int32_t* alen, int32_t* new_lens, void* feat,
                          cudaStream_t st) {
  const int esize = s->dtype == EAGLE_DTYPE_BF16 ? 2 : 4;
  CommitParams p{};
  p.k_prefix = static_cast<uint8_t*>(kp);
  p.v_prefix = static_cast<uint8_t*>(vp);
  p.prefix_lens = lens;
  p.k_tree = static_cast<const uint8_t*>(kt);
  p.v_tree = static_cast<const uint8_t*>(vt);
  p.hidden = static_cast<const uint8_t*>(hidden);
  p.parents = parents;
  p.accepted_nodes = acc;
  p.accept_len = alen;
  p.new_lens = new_lens;
  p.feat = static_cast<uint8_t*>(feat);
  p.N = s->num_nodes;
  p.Hkv = s->num_kv_heads;
  p.Lmax = s->max_prefix_len;
  p.row_bytes = s->head_dim * esize;
  p.hrow_bytes = s->hidden * esize;
  const dim3 grid(s->batch, s->num_kv_heads + s->num_nodes);
  commit_kernel<<<grid, kCommitThreads, 0, st>>>(p);
  return launch_status();
}

// ------------------------------------------------------------------ argument checks

eagle_status_t check_attention_args(const eagle_shape_t* s, const void* q, const void* kp,
                                    const void* vp, const int32_t* lens, const void* kt,
                                    const void* vt, const int32_t* parents, const void* out,
                                    const void* ws, size_t ws_bytes, size_t need) {
  eagle_status_t rc = check_shape(s);
  if (rc != EAGLE_OK) return rc;
  if (!aligned16(q) || !aligned16(kp) || !aligned16(vp) || !aligned16(kt) || !aligned16(vt) ||
      !aligned16(out) || lens == nullptr || parents == nullptr)
    return EAGLE_ERR_INVALID_ARGUMENT;
  if (static_cast<long>(s->batch) * s->num_kv_heads > 65535) return EAGLE_ERR_UNSUPPORTED;
  if (s->dtype == EAGLE_DTYPE_BF16 && s->num_q_heads / s->num_kv_heads > kTcRows) return EAGLE_ERR_UNSUPPORTED;
  if (ws_bytes < need) return EAGLE_ERR_WORKSPACE_TOO_SMALL;
  if (need > 0 && (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0))
    return EAGLE_ERR_INVALID_ARGUMENT;
  return EAGLE_OK;
}

eagle_status_t check_lm_args(const eagle_shape_t* s, const void* hidden, const void* w,
                             const float* logits) {
  eagle_status_t rc = check_shape(s);
  if (rc != EAGLE_OK) return rc;
  if (!aligned16(hidden) || !aligned16(w) || !aligned16(logits)) return EAGLE_ERR_INVALID_ARGUMENT;
  return EAGLE_OK;
}

eagle_status_t check_accept_args(const eagle_shape_t* s, const float* logits, const float* draft,
                                 const int32_t* tokens, const int32_t* parents, float T,
                                 const int32_t* acc, const int32_t* alen, const int32_t* next) {
  eagle_status_t rc = check_shape(s);
  if (rc != EAGLE_OK) return rc;
  if (!aligned16(logits) || !aligned16(draft) || tokens == nullptr || parents == nullptr ||
      acc == nullptr || alen == nullptr || next == nullptr)
    return EAGLE_ERR_INVALID_ARGUMENT;
  if (!(T >= 0.f) || !std::isfinite(T)) return EAGLE_ERR_INVALID_ARGUMENT;
  // host-only bound: the largest cluster any device offers; device_accept_supported()
  // checks the current device before anything is enqueued
  const AccPlan ap = plan_accept(s, kAccMaxCluster);
  if (ap.nq < 1 || ap.smem > kAccMaxSmem) return EAGLE_ERR_UNSUPPORTED;
  return EAGLE_OK;
}

eagle_status_t check_commit_args(const eagle_shape_t* s, const void* kp, const void* vp,
                                 const int32_t* lens, const void* kt, const void* vt,
                                 const void* hidden, const int32_t* parents, const int32_t* acc,
                                 const int32_t* alen, const int32_t* new_lens, const void* feat) {
  eagle_status_t rc = check_shape(s);
  if (rc != EAGLE_OK) return rc;
  if (!aligned16(kp) || !aligned16(vp) || !aligned16(kt) || !aligned16(vt) || !aligned16(hidden) ||
      !aligned16(feat) || lens == nullptr || parents == nullptr || acc == nullptr ||
      alen == nullptr || new_lens == nullptr)
    return EAGLE_ERR_INVALID_ARGUMENT;
  // the kernel reads prefix_lens[b] in every block while one block writes new_lens[b]
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(lens), b0 = reinterpret_cast<uintptr_t>(new_lens);
  const uintptr_t span = static_cast<uintptr_t>(s->batch) * sizeof(int32_t);
  if (a0 < b0 + span && b0 < a0 + span) return EAGLE_ERR_INVALID_ARGUMENT;
  if (s->num_kv_heads + s->num_nodes > 65535) return EAGLE_ERR_UNSUPPORTED;
  return EAGLE_OK;
}

// The accept plan on the current device (its largest co-schedulable cluster).
bool device_accept_supported(const eagle_shape_t* s, int dev) {
  const AccPlan ap = plan_accept(s, g_dev[dev].max_cluster);
  return ap.nq >= 1 && ap.smem <= kAccMaxSmem;
}

const void* draft_kernel(int mode) {
  switch (mode) {
    case kDraftTopK: return reinterpret_cast<const void*>(draft_select_kernel<kDraftTopK>);
    case kDraftRaces: return reinterpret_cast<const void*>(draft_select_kernel<kDraftRaces>);
    default: return reinterpret_cast<const void*>(draft_select_kernel<kDraftDistinct>);
  }
}

int draft_active_clusters(int mode, int S, size_t smem) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(S));
  cfg.blockDim = dim3(kDraftThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, draft_kernel(mode), &cfg) != cudaSuccess) n = 0;
  cudaGetLastError();
  return n;
}

// Entries per CTA when a row of V entries is split over S CTAs (a multiple of 4).
int draft_slice(int V, int S) { return (((V + S - 1) / S + 3) / 4) * 4; }

// Cluster size for `rows` rows of V entries, each CTA staging its slice in shared memory:
// the largest S in {16, 8, 4, 2} whose clusters are all resident at once, with slices of at
// least 1024 entries; else the smallest S whose slice fits (more rows than one wave holds
// gain nothing from splitting).  0: no S fits.
int draft_cluster(int dev, long rows, int V, int mode) {
  DeviceState& ds = g_dev[dev];
  int first_fit = 0;
  for (int lg = 0; lg < 4; ++lg) {  // portable sizes only
    const int S = 1 << lg;
    if (static_cast<size_t>(draft_slice(V, S)) * 4 <= kDraftMaxSmem) {
      first_fit = S;
      break;
    }
  }
  if (first_fit == 0) return 0;
  for (int lg = 4; lg >= 1; --lg) {
    const int S = 1 << lg;
    const size_t bytes = static_cast<size_t>(draft_slice(V, S)) * 4;
    if (S > ds.draft_max_cluster || S < first_fit || V < S * 1024 || bytes > kDraftMaxSmem) continue;
    const size_t bucket = (bytes + 4095) / 4096;
    int n;
    {
      std::lock_guard<std::mutex> lock(ds.draft_mu);
      int& slot = ds.draft_clusters[mode][lg][bucket];
      if (slot == 0) slot = 1 + draft_active_clusters(mode, S, bucket * 4096);
      n = slot - 1;
    }
    if (rows <= n) return S;
  }
  return first_fit;
}

bool ensure_draft(int dev) {
  DeviceState& ds = g_dev[dev];
  std::call_once(ds.draft_once, [&] {
    const int bytes = static_cast<int>(kDraftMaxSmem);
    bool ok = true, wide = true;
    for (int mode = 0; mode < 3; ++mode) {
      ok &= cudaFuncSetAttribute(draft_kernel(mode), cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
            cudaSuccess;
      wide &= cudaFuncSetAttribute(draft_kernel(mode), cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
              cudaSuccess;
    }
    for (int mode = 0; mode < 3 && wide; ++mode) wide &= draft_active_clusters(mode, 16, 4096) >= 1;
    ds.draft_ok = ok;
    if (wide) ds.draft_max_cluster = 16;
    cudaGetLastError();
  });
  return ds.draft_ok;
}

// eagle_draft_select / eagle_draft_select_distinct: argument checks, then one cluster launch.
eagle_status_t draft_launch(int mode, int32_t batch, int32_t rows_per_seq, int32_t vocab, int32_t k,
                            const float* logits, float temperature, uint64_t seed, uint64_t offset,
                            int32_t* tokens, float* conf, float* probs, void* stream) {
  if (batch < 1 || batch > 65535 || rows_per_seq < 1 || rows_per_seq > 256 || k < 1 ||
      k > kDraftMaxK || vocab < k)
    return EAGLE_ERR_INVALID_ARGUMENT;
  // the Philox counter packs b (16 bits), the purpose 2 + j and the row f (8 bits each)
  static_assert(kDraftMaxK + 2 <= 256, "race purposes must fit the counter's 8-bit field");
  if (rows_per_seq - 1 > kPhiloxMaxField || k + 1 > kPhiloxMaxField) return EAGLE_ERR_INVALID_ARGUMENT;
  if (!(temperature >= 0.f) || !std::isfinite(temperature)) return EAGLE_ERR_INVALID_ARGUMENT;
  if (logits == nullptr || tokens == nullptr || conf == nullptr) return EAGLE_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(logits) & 3) != 0) return EAGLE_ERR_INVALID_ARGUMENT;
  if (static_cast<size_t>(draft_slice(vocab, kDraftPortableCluster)) * 4 > kDraftMaxSmem)
    return EAGLE_ERR_UNSUPPORTED;  // a row must fit the shared memory of one cluster
  if (temperature == 0.f) mode = kDraftTopK;
  int dev;
  if (!current_device(&dev) || !ensure_draft(dev)) return EAGLE_ERR_CUDA;
  const long rows = static_cast<long>(batch) * rows_per_seq;
  const int S = draft_cluster(dev, rows, vocab, mode);
  if (S == 0) return EAGLE_ERR_UNSUPPORTED;
  const int slice = draft_slice(vocab, S);
  const int vec16 = (vocab % 4 == 0 && aligned16(logits)) ? 1 : 0;
  DraftParams p{logits, tokens, conf, probs, rows_per_seq, vocab, k, slice, vec16, temperature, seed, offset};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * S));
  cfg.blockDim = dim3(kDraftThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(slice) * 4;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  switch (mode) {
    case kDraftTopK: e = cudaLaunchKernelEx(&cfg, draft_select_kernel<kDraftTopK>, p); break;
    case kDraftRaces: e = cudaLaunchKernelEx(&cfg, draft_select_kernel<kDraftRaces>, p); break;
    default: e = cudaLaunchKernelEx(&cfg, draft_select_kernel<kDraftDistinct>, p); break;
  }
  if (e != cudaSuccess) return EAGLE_ERR_CUDA;
  return launch_status();
}

}  // namespace
}  // namespace eagle

using namespace eagle;

extern "C" {

const char* eagle_status_string(eagle_status_t status) {
  switch (status) {
    case EAGLE_OK: return "EAGLE_OK";
    case EAGLE_ERR_INVALID_ARGUMENT: return "EAGLE_ERR_INVALID_ARGUMENT";
    case EAGLE_ERR_UNSUPPORTED: return "EAGLE_ERR_UNSUPPORTED";
    case EAGLE_ERR_WORKSPACE_TOO_SMALL: return "EAGLE_ERR_WORKSPACE_TOO_SMALL";
    case EAGLE_ERR_CUDA: return "EAGLE_ERR_CUDA";
  }
  return "EAGLE_ERR_UNKNOWN";
}

size_t eagle_workspace_bytes(const eagle_shape_t* shape) {
  if (check_shape(shape) != EAGLE_OK) return 0;
  return attention_ws_bytes(shape);
}

eagle_status_t eagle_tree_attention(const eagle_shape_t* shape, const void* q, const void* k_prefix,
                                    const void* v_prefix, const int32_t* prefix_lens,
                                    const void* k_tree, const void* v_tree, const int32_t* parents,
                                    void* out, void* workspace, size_t workspace_bytes, void* stream) {
  eagle_status_t rc = check_attention_args(shape, q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree,
                                           parents, out, workspace, workspace_bytes,
                                           eagle_workspace_bytes(shape));
  if (rc != EAGLE_OK) return rc;
  int dev;
  if (!current_device(&dev) || !ensure_attributes(dev)) return EAGLE_ERR_CUDA;
  return run_attention(shape, q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree, parents, out,
                       workspace, static_cast<cudaStream_t>(stream));
}

eagle_status_t eagle_lm_head_logits(const eagle_shape_t* shape, const void* hidden, const void* w_lm,
                                    float* logits, void* stream) {
  eagle_status_t rc = check_lm_args(shape, hidden, w_lm, logits);
  if (rc != EAGLE_OK) return rc;
  int dev;
  if (!current_device(&dev) || !ensure_attributes(dev)) return EAGLE_ERR_CUDA;
  return run_lm_head(shape, hidden, w_lm, logits, static_cast<cudaStream_t>(stream));
}

eagle_status_t eagle_tree_accept(const eagle_shape_t* shape, const float* logits, const float* draft_probs,
                                 const int32_t* tokens, const int32_t* parents, float temperature,
                                 uint64_t seed, uint64_t offset, int32_t* accepted_nodes,
                                 int32_t* accept_len, int32_t* next_token, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  eagle_status_t rc = check_accept_args(shape, logits, draft_probs, tokens, parents, temperature,
                                        accepted_nodes, accept_len, next_token);
  if (rc != EAGLE_OK) return rc;
  int dev;
  if (!current_device(&dev) || !ensure_attributes(dev)) return EAGLE_ERR_CUDA;
  if (!device_accept_supported(shape, dev)) return EAGLE_ERR_UNSUPPORTED;
  return run_accept(shape, logits, draft_probs, tokens, parents, temperature, seed, offset,
                    accepted_nodes, accept_len, next_token, static_cast<cudaStream_t>(stream));
}

eagle_status_t eagle_verify_step(const eagle_shape_t* shape, const void* q, const void* k_prefix,
                                 const void* v_prefix, const int32_t* prefix_lens, const void* k_tree,
                                 const void* v_tree, const int32_t* parents, const void* hidden,
                                 const void* w_lm, const float* draft_probs, const int32_t* tokens,
                                 float temperature, uint64_t seed, uint64_t offset, void* out,
                                 float* logits, int32_t* accepted_nodes, int32_t* accept_len,
                                 int32_t* next_token, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  eagle_status_t rc = check_attention_args(shape, q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree,
                                           parents, out, workspace, workspace_bytes,
                                           eagle_workspace_bytes(shape));
  if (rc == EAGLE_OK) rc = check_lm_args(shape, hidden, w_lm, logits);
  if (rc == EAGLE_OK)
    rc = check_accept_args(shape, logits, draft_probs, tokens, parents, temperature, accepted_nodes,
                           accept_len, next_token);
  if (rc != EAGLE_OK) return rc;
  int dev;
  if (!current_device(&dev) || !ensure_attributes(dev)) return EAGLE_ERR_CUDA;
  if (!device_accept_supported(shape, dev)) return EAGLE_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (shape->dtype == EAGLE_DTYPE_BF16 && ensure_side(dev)) {
    // Two streams.  The LM head streams W over the whole GPU and the accept walk follows it
    // on the caller's stream (programmatic dependent launch: the walk's set-up overlaps the
    // LM head's drain).  Tree attention, whose output the walk does not read, runs with its
    // merge on a library-owned side stream once the LM head has completed, beside the walk,
    // and the caller's stream waits for it after the walk.  No kernel is ever launched as a
    // programmatic dependent of the walk.
    DeviceState& ds = g_dev[dev];
    std::lock_guard<std::mutex> lock(ds.step_mu);
    rc = run_lm_head(shape, hidden, w_lm, logits, st);
    if (rc != EAGLE_OK) return rc;
    if (cudaEventRecord(ds.lm_mark, st) != cudaSuccess) return EAGLE_ERR_CUDA;
    if (cudaStreamWaitEvent(ds.side, ds.lm_mark, 0) != cudaSuccess) return EAGLE_ERR_CUDA;
    rc = run_attention(shape, q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree, parents, out,
                       workspace, ds.side);
    if (rc != EAGLE_OK) return rc;
    if (cudaEventRecord(ds.attn_done, ds.side) != cudaSuccess) return EAGLE_ERR_CUDA;
    rc = run_accept(shape, logits, draft_probs, tokens, parents, temperature, seed, offset,
                    accepted_nodes, accept_len, next_token, st, /*pdl=*/true);
    if (rc != EAGLE_OK) return rc;
    if (cudaStreamWaitEvent(st, ds.attn_done, 0) != cudaSuccess) return EAGLE_ERR_CUDA;
    return EAGLE_OK;
  }
  // fp32 (and bf16 if the side stream could not be made): one stream -- the LM head, the
  // walk (programmatic dependent launch), then tree attention once the walk has completed
  rc = run_lm_head(shape, hidden, w_lm, logits, st);
  if (rc != EAGLE_OK) return rc;
  rc = run_accept(shape, logits, draft_probs, tokens, parents, temperature, seed, offset,
                  accepted_nodes, accept_len, next_token, st, /*pdl=*/true);
  if (rc != EAGLE_OK) return rc;
  return run_attention(shape, q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree, parents, out,
                       workspace, st);
}

eagle_status_t eagle_commit_accepted(const eagle_shape_t* shape, void* k_prefix, void* v_prefix,
                                     const int32_t* prefix_lens, const void* k_tree,
                                     const void* v_tree, const void* hidden, const int32_t* parents,
                                     const int32_t* accepted_nodes, const int32_t* accept_len,
                                     int32_t* new_prefix_lens, void* feat, void* stream) {
  const eagle_status_t rc = check_commit_args(shape, k_prefix, v_prefix, prefix_lens, k_tree, v_tree,
                                              hidden, parents, accepted_nodes, accept_len,
                                              new_prefix_lens, feat);
  if (rc != EAGLE_OK) return rc;
  return run_commit(shape, k_prefix, v_prefix, prefix_lens, k_tree, v_tree, hidden, parents,
                    accepted_nodes, accept_len, new_prefix_lens, feat, static_cast<cudaStream_t>(stream));
}

eagle_status_t eagle_tree_rerank(int32_t batch, int32_t num_candidates, int32_t num_select,
                                 const int32_t* cand_parents, const int32_t* cand_tokens,
                                 const float* confidence, int32_t* sel, int32_t* parents_out,
                                 int32_t* tokens_out, uint64_t* masks_out, int32_t* num_selected,
                                 void* stream) {
  if (batch < 1 || batch > 65535 || num_candidates < 1 || num_candidates > kRerankThreads ||
      num_select < 1 || num_select > kRerankMaxSelect)
    return EAGLE_ERR_INVALID_ARGUMENT;
  if (cand_parents == nullptr || cand_tokens == nullptr || confidence == nullptr || sel == nullptr ||
      parents_out == nullptr || tokens_out == nullptr || num_selected == nullptr ||
      masks_out == nullptr || (reinterpret_cast<uintptr_t>(masks_out) & 7u) != 0)
    return EAGLE_ERR_INVALID_ARGUMENT;
  RerankParams p{cand_parents, cand_tokens, confidence, sel,        parents_out,
                 tokens_out,   masks_out,   num_selected, num_candidates, num_select};
  rerank_kernel<<<batch, kRerankThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return launch_status();
}

eagle_status_t eagle_draft_select(int32_t batch, int32_t rows_per_seq, int32_t vocab, int32_t k,
                                  const float* logits, float temperature, uint64_t seed,
                                  uint64_t offset, int32_t* tokens, float* conf, float* probs,
                                  void* stream) {
  return draft_launch(kDraftRaces, batch, rows_per_seq, vocab, k, logits, temperature, seed, offset,
                      tokens, conf, probs, stream);
}

eagle_status_t eagle_draft_select_distinct(int32_t batch, int32_t rows_per_seq, int32_t vocab, int32_t k,
                                           const float* logits, float temperature, uint64_t seed,
                                           uint64_t offset, int32_t* tokens, float* conf, float* probs,
                                           void* stream) {
  return draft_launch(kDraftDistinct, batch, rows_per_seq, vocab, k, logits, temperature, seed, offset,
                      tokens, conf, probs, stream);
}

eagle_status_t eagle_draft_child_rows(int32_t batch, int32_t rows_per_seq, int32_t vocab, int32_t k,
                                      const float* probs, const int32_t* tokens, float* child_probs,
                                      void* stream) {
  if (batch < 1 || batch > 65535 || rows_per_seq < 1 || rows_per_seq > 256 || k < 1 ||
      k > kDraftMaxK || vocab < 1)
    return EAGLE_ERR_INVALID_ARGUMENT;
  if (probs == nullptr || tokens == nullptr || child_probs == nullptr) return EAGLE_ERR_INVALID_ARGUMENT;
  const long rows = static_cast<long>(batch) * rows_per_seq;
  int C = (vocab + 4095) / 4096;  // chunks of at least 4096 entries, up to 8 per row
  if (C > kChildMaxCluster) C = kChildMaxCluster;
  if (C < 1) C = 1;
  ChildParams p{probs, tokens, child_probs, vocab, k, (vocab + C - 1) / C};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * C));
  cfg.blockDim = dim3(kChildThreads);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, draft_child_rows_kernel, p) != cudaSuccess) return EAGLE_ERR_CUDA;
  return launch_status();
}

eagle_status_t eagle_device_error(int32_t* code, int32_t reset) {
  if (code == nullptr) return EAGLE_ERR_INVALID_ARGUMENT;
  int32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return EAGLE_ERR_CUDA;
  *code = v;
  if (reset) {
    const int32_t zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess) return EAGLE_ERR_CUDA;
  }
  return EAGLE_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ allocation-free variant
// Tree attention whose split partials live in a fixed array of this library instead of a
// caller workspace, for callers that cannot allocate device memory at call time.

namespace eagle {
namespace {

static __device__ __align__(256) uint8_t g_static_scratch[EAGLE_STATIC_SCRATCH_BYTES];

struct StaticScratch {
  std::mutex mu;
  void* ptr = nullptr;  // set only by a lookup that succeeded
};
StaticScratch g_scratch[kMaxDevices];

// The host-side name of the array is not a device address; look the address up per
// device, with that device current.  Only a successful lookup is kept: one that failed
// (say, made during a stream capture) is retried by the next call.
void* static_scratch_address(int dev) {
  StaticScratch& s = g_scratch[dev];
  std::lock_guard<std::mutex> lock(s.mu);
  if (s.ptr == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) == cudaSuccess) s.ptr = p;
    else cudaGetLastError();
  }
  return s.ptr;
}

}  // namespace
}  // namespace eagle

extern "C" eagle_status_t eagle_tree_attention_static(const eagle_shape_t* shape, const void* q,
                                                      const void* k_prefix, const void* v_prefix,
                                                      const int32_t* prefix_lens, const void* k_tree,
                                                      const void* v_tree, const int32_t* parents,
                                                      void* out, void* stream) {
  if (check_shape(shape) != EAGLE_OK) return EAGLE_ERR_INVALID_ARGUMENT;
  if (attention_ws_bytes(shape) > EAGLE_STATIC_SCRATCH_BYTES) return EAGLE_ERR_UNSUPPORTED;
  int dev;
  if (!current_device(&dev)) return EAGLE_ERR_CUDA;
  void* scratch = static_scratch_address(dev);
  if (scratch == nullptr) return EAGLE_ERR_CUDA;
  eagle_status_t rc = check_attention_args(shape, q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree,
                                           parents, out, scratch, EAGLE_STATIC_SCRATCH_BYTES,
                                           attention_ws_bytes(shape));
  if (rc != EAGLE_OK) return rc;
  if (!ensure_attributes(dev)) return EAGLE_ERR_CUDA;
  return run_attention(shape, q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree, parents, out,
                       scratch, static_cast<cudaStream_t>(stream));
}
