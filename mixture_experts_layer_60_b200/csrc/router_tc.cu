// Fused router of the DeepSeekMoE layer ("DeepSeek-V3 技術報告", section
// 方法 / 2): the affinity s_{i,t} = Sigmoid(u_t^T e_i), the K largest keys
// s + b (g'-equation; optionally within the best groups), the gates
// normalised from the unbiased s, and the per-expert load, in one tcgen05
// kernel.  The float32 logits never go to memory, except for the rows of the
// few tokens whose routing hinged on a key gap below the refine gap, which
// the float64 tie-break (router.cu) re-routes.
//
// Tiling.  A CTA pair (tcgen05 cta_group::2) owns 256 tokens: each CTA keeps
// 128 token rows of u in its shared memory (the MMA's M side) and half of the
// centroid rows E (N = N_r, split across the pair), and every MMA leaves each
// CTA the full N_r-wide logit rows of its own 128 tokens in TMEM.  Sharing the
// centroid operand across the pair halves the centroid bytes each SM streams.
// To fill the GPU when tokens are few, S pairs of one cluster (2S CTAs) split
// the d-long contraction in S slices; the pairs holding slices 1..S-1 stage
// their partial logits in shared memory and the first pair adds them over
// distributed shared memory, in slice order.  With S = 1 pairs loop over
// tiles (persistent).
//
// Roles (192 threads per CTA): warp 0 TMA producer (both CTAs of a pair;
// loads complete on the pair leader's barrier), warp 1 TMEM allocation and,
// in the leader, the MMA issuer, warps 2-5 the epilogue: thread = token row
// (TMEM lane), which walks the token's N_r logits once: sigmoid, key, a
// sorted top-(K+1) list in registers, then gates, the load histogram (shared
// memory, then global atomics) and, for near-ties, the tie-break listing.
//
// Every wait is bounded (1 s of %globaltimer); on expiry the kernel records
// ERR_GEMM_TIMEOUT in the device error word and every role drains to the
// closing cluster barrier.
#include <math.h>

#include "launch.h"
#include "router_warp.cuh"
#include "sm100.cuh"

namespace moe {

moe_status make_tmap_2d(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                        int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer);

namespace {

using namespace sm100;

constexpr int BK = 64;                 // bf16 K elements per 128-byte swizzle row
constexpr int TM = 128;                // token rows per CTA (TMEM lanes)
constexpr int kMaxN = 256;             // N_r limit of the pair MMA
constexpr int kParts = 4;              // epilogue warps per TMEM lane quarter (column parts)
constexpr int kEpiWarps = 4 * kParts;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 64 + kEpiThreads;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr int kEpiBarrier = 1;         // named barrier of the epilogue warps
constexpr int STAGES = 4;
constexpr int HALF_ROWS = TM / 2;      // token rows staged in shared memory at a time

constexpr int A_BYTES = TM * BK * 2;                  // 16 KB
constexpr int B_MAX_BYTES = (kMaxN / 2) * BK * 2;     // 16 KB
constexpr int XLD = kMaxN + 4;                        // float stride of a staged logit row
constexpr int OFF_B = STAGES * A_BYTES;
constexpr int RING_BYTES = OFF_B + STAGES * B_MAX_BYTES;
// S > 1: each CTA stages its partial logits of the rows other slices own in
// [TM][XLD] floats from offset 0 (over the ring, free once the tile's MMAs
// are done), then the logits of its own rows go to sX
constexpr int STAGE_BYTES = TM * XLD * 4;
constexpr int OFF_X = RING_BYTES > STAGE_BYTES ? RING_BYTES : STAGE_BYTES;   // [HALF_ROWS][XLD]
constexpr int OFF_WK = OFF_X + HALF_ROWS * XLD * 4;   // float [kEpiWarps][kMaxN] group keys
constexpr int OFF_BAR = OFF_WK + kEpiWarps * kMaxN * 4;
constexpr int N_BARS = 2 * STAGES + 4;     // full, empty, tfull, tempty, peer_ready, mma_done
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;        // tmem slot, abort flag
constexpr int OFF_BIAS = OFF_MISC + 16;               // float [kMaxN]
constexpr int OFF_HIST = OFF_BIAS + kMaxN * 4;        // int [kMaxN]
constexpr int SMEM_BYTES = OFF_HIST + kMaxN * 4;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

struct RouterParams {
  const float* bias;     // [N_r]
  int T, N_r, K;
  int nk;                // d / BK
  int n_tiles;           // ceil(T / 256)
  int parts;             // column parts actually used (<= kParts), N_r / parts % 16 == 0
  int n_groups, topk_groups;
  int32_t* idx;
  float* gate;
  int32_t* counts;
  float* logits;         // [T, N_r]: written for listed tokens only
  RefineLists rl;
  float refine_gap, near;
  int* err;
};

__device__ __forceinline__ void raise_abort(volatile int* abort, int* err) {
  *abort = 1;
  atomicOr(err, ERR_GEMM_TIMEOUT);
}

__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync %0, %1;" ::"n"(kEpiBarrier), "n"(kEpiThreads) : "memory");
}
// True on every epilogue thread when `v` is true on any of them (a barrier).
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kEpiBarrier), "n"(kEpiThreads)
      : "memory");
  return r != 0;
}

// Logits of this thread's token for columns [c, c + CH): the partial sums
// of the S slices of the contraction added in slice order, this CTA's own
// (slice `slice`) from TMEM, the others from their staged copies.
constexpr int CH = 16;                 // columns per TMEM load in the epilogue
template <int S>
__device__ __forceinline__ void load_logits(uint32_t tmem_row, int c, int slice, uint32_t half,
                                            uint32_t stage_addr, float* x) {
  uint32_t r[CH];
  tmem_ld_32x32b_x16(tmem_row + c, r);
  tmem_wait_ld();
  if constexpr (S == 1) {
#pragma unroll
    for (int j = 0; j < CH; ++j) x[j] = __uint_as_float(r[j]);
  } else {
#pragma unroll
    for (int j = 0; j < CH; ++j) x[j] = 0.f;
#pragma unroll
    for (int q = 0; q < S; ++q) {
      if (q == slice) {
#pragma unroll
        for (int j = 0; j < CH; ++j) x[j] += __uint_as_float(r[j]);
      } else {
        const uint32_t peer = map_shared_to(stage_addr, half + 2u * (uint32_t)q);
#pragma unroll
        for (int v = 0; v < CH / 4; ++v) {
          const float4 f = ld_shared_cluster_v4(peer + (uint32_t)(c + 4 * v) * 4u);
          x[4 * v] += f.x;
          x[4 * v + 1] += f.y;
          x[4 * v + 2] += f.z;
          x[4 * v + 3] += f.w;
        }
      }
    }
  }
}

template <int S, int V>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmU,
                     const __grid_constant__ CUtensorMap tmE, const RouterParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + OFF_B;
  float* sX = reinterpret_cast<float*>(smem + OFF_X);
  float* s_wkeys = reinterpret_cast<float*>(smem + OFF_WK);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* peer_ready = tempty + 1;
  uint64_t* mma_done = peer_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  float* s_bias = reinterpret_cast<float*>(smem + OFF_BIAS);
  int* s_hist = reinterpret_cast<int*>(smem + OFF_HIST);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t half = rank & 1u;                   // which 128 tokens / which half of E
  const int slice = (int)(rank >> 1);                // which slice of the contraction
  const uint32_t leader = rank & ~1u;
  const bool is_leader = rank == leader;
  const uint16_t pair_mask = (uint16_t)(3u << leader);
  const int N = p.N_r;
  const int b_bytes = (N / 2) * BK * 2;
  const int kb0 = slice * p.nk / S, kb1 = (slice + 1) * p.nk / S;
  const int first_tile = (int)cluster_id_x();
  const int tile_step = S == 1 ? (int)n_clusters_x() : p.n_tiles;   // S > 1: one tile per cluster
  const uint32_t tmem_cols = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(tfull, 1);
    mbar_init(tempty, 2 * kEpiWarps);                // epilogue warps of both CTAs of the pair
    mbar_init(peer_ready, S > 1 ? (S - 1) * kEpiWarps : 1);   // staging warps of the other slices
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmE);
  }
  if (warp == 1) {
    tmem2_alloc(tmem_slot, tmem_cols);
    tmem2_relinquish();
  }
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    s_bias[i] = p.bias[i];
    s_hist[i] = 0;
  }
  tc_fence_before();
  cluster_sync_all();          // barriers of every CTA initialised, TMEM allocated in each pair
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t full_leader0 = map_shared_to(smem_u32(&full[0]), leader);
  const uint32_t tempty_leader = map_shared_to(smem_u32(tempty), leader);

  if (warp == 0) {
    // ------------------------------------------------------------ producer (every CTA)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t bytes = 2u * (uint32_t)(A_BYTES + b_bytes);   // both CTAs' loads
      for (int tile = first_tile; tile < p.n_tiles && ok; tile += tile_step) {
        const int row0 = tile * 2 * TM + (int)half * TM;
        const int e0 = (int)half * (N / 2);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          if (is_leader) mbar_arrive_expect_tx(&full[stage], bytes);
          const uint32_t fb = full_leader0 + stage * 8;
          tma_load_2d_pair(sA + stage * A_BYTES, &tmU, kb * BK, row0, fb);
          tma_load_2d_pair(sB + stage * B_MAX_BYTES, &tmE, kb * BK, e0, fb);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // the leader waits until every armed stage's copies have landed
      if (is_leader)
        for (int s = 0; s < STAGES; ++s)
          mbar_wait_bounded(&full[s], ((s < stage) ? phase : phase ^ 1), nullptr, kWaitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (pair leader)
    if (is_leader && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * TM, N);
      int stage = 0;
      uint32_t phase = 0, tphase = 0;
      bool ok = true;
      for (int tile = first_tile; tile < p.n_tiles && ok; tile += tile_step) {
        if (!mbar_wait_bounded(tempty, tphase ^ 1, abort_flag, kWaitNs)) {
          raise_abort(abort_flag, p.err);
          break;
        }
        tc_fence_after();
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * B_MAX_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma2_f16_ss(tmem_base, smem_desc_k_sw128(a0 + k * 32), smem_desc_k_sw128(b0 + k * 32),
                        idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          mma2_commit_mask(&empty[stage], pair_mask);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma2_commit_mask(tfull, pair_mask);
        tphase ^= 1;
      }
      mma2_commit_local(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue (every CTA)
    // Warp w: TMEM lane quarter q = w % 4 (its 32 token rows) and column part
    // `part` (columns [part*cols, +cols) of those rows) when reading TMEM; one
    // token per warp when routing.
    const int ew = warp - 2;                      // epilogue warp 0 .. kEpiWarps-1
    const int q = warp & 3;
    const int part = ew >> 2;
    const int row = q * 32 + lane;                // token row of this CTA
    const int P = p.parts;
    const int cols = N / P;
    const int c0 = part * cols;
    const bool active = part < P;
    const uint32_t tmem_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    float* stage_row = reinterpret_cast<float*>(smem) + (size_t)row * XLD;
    float* wkeys = s_wkeys + ew * kMaxN;
    // rows of the tile this CTA routes: all of them (S == 1) or slice
    // `slice`'s share of TM / S rows (S > 1; the other slices' CTAs route the rest)
    const int own0 = S == 1 ? 0 : slice * (TM / S);
    const int own1 = S == 1 ? TM : own0 + TM / S;
    uint32_t tphase = 0;
    for (int tile = first_tile; tile < p.n_tiles; tile += tile_step) {
      const bool got = mbar_wait_bounded(tfull, tphase, abort_flag, kWaitNs);
      if (epi_any(!got)) {
        if (lane == 0) raise_abort(abort_flag, p.err);
        break;
      }
      tc_fence_after();
      if (S > 1) {
        // stage this slice's partial logits of the rows the other slices own,
        // signal their CTAs, wait for theirs of this CTA's rows
        if (active && (row < own0 || row >= own1)) {
          for (int c = c0; c < c0 + cols; c += CH) {
            uint32_t r[CH];
            tmem_ld_32x32b_x16(tmem_row + c, r);
            tmem_wait_ld();
#pragma unroll
            for (int v = 0; v < CH / 4; ++v)
              *reinterpret_cast<uint4*>(stage_row + c + 4 * v) =
                  make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
          }
        }
        __syncwarp();
        if (lane == 0)
          for (int s2 = 0; s2 < S; ++s2)
            if (s2 != slice)
              mbar_arrive_remote(map_shared_to(smem_u32(peer_ready), half + 2u * (uint32_t)s2));
        const bool ready = mbar_wait_cluster_bounded(peer_ready, 0, abort_flag, kWaitNs);
        if (epi_any(!ready)) {
          if (lane == 0) raise_abort(abort_flag, p.err);
          break;
        }
      }
      const int tok0 = tile * 2 * TM + (int)half * TM;
      // own rows in blocks of HALF_ROWS (lane quarters 2h, 2h+1)
      for (int h0 = own0; h0 < own1; h0 += HALF_ROWS) {
        const int h1 = min(own1, h0 + HALF_ROWS);
        if (active && row >= h0 && row < h1) {
          float* xr = sX + (size_t)(row - h0) * XLD;
          for (int c = c0; c < c0 + cols; c += CH) {
            float x[CH];
            load_logits<S>(tmem_row, c, slice, half, smem_u32(stage_row), x);
#pragma unroll
            for (int v = 0; v < CH / 4; ++v)
              *reinterpret_cast<float4*>(xr + c + 4 * v) =
                  make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
          }
        }
        tc_fence_before();
        epi_sync();
        if (h1 == own1 && lane == 0)
          mbar_arrive_remote(tempty_leader);    // TMEM read: the next tile's MMA may go
        // one token per warp
        for (int r = ew; r < h1 - h0; r += kEpiWarps) {
          const int t = tok0 + h0 + r;
          if (t < p.T)
            route_token_warp<V>(sX + (size_t)r * XLD, s_bias, t, N, p.K, p.n_groups,
                                p.topk_groups, wkeys, p.idx, p.gate, s_hist, p.rl, p.refine_gap,
                                p.near, p.logits);
        }
        epi_sync();                             // sX is rewritten next
      }
      tphase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  for (int i = threadIdx.x; i < N; i += blockDim.x)
    if (s_hist[i]) atomicAdd(&p.counts[i], s_hist[i]);
  cluster_sync_all();          // no CTA leaves while another may read its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem2_dealloc(tmem_base, tmem_cols);
  }
}

template <int S, int V>
moe_status router_launch(const CUtensorMap& tmU, const CUtensorMap& tmE, const RouterParams& p,
                         int n_clusters, cudaStream_t s) {
  auto kern = router_tc_kernel<S, V>;
  static bool attr_done[kMaxSmemDevices] = {};
  const moe_status st = ensure_max_smem(reinterpret_cast<const void*>(kern), SMEM_ALLOC,
                                        attr_done, "router_tc smem attribute");
  if (st != MOE_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * S * n_clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2 * S;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, kern, tmU, tmE, p), "router_tc launch");
}

// Clusters of 2S CTAs of this kernel that fit on the device at once.
template <int S, int V>
int resident_clusters() {
  static int cached[kMaxSmemDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSmemDevices) return 0;
  if (cached[dev]) return cached[dev];
  auto kern = router_tc_kernel<S, V>;
  static bool attr_done[kMaxSmemDevices] = {};
  if (ensure_max_smem(reinterpret_cast<const void*>(kern), SMEM_ALLOC, attr_done,
                      "router_tc smem attribute") != MOE_OK)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * S * (sm_count() / (2 * S)));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2 * S;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(kern), &cfg) !=
          cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    return 0;
  }
  cached[dev] = n;
  return n;
}

template <int V>
moe_status router_dispatch_s(const CUtensorMap& tmU, const CUtensorMap& tmE,
                             const RouterParams& p, cudaStream_t s) {
  // the largest slice count whose clusters all run in one wave and whose
  // slices each get at least one 64-wide block of the contraction
  if (p.nk >= 4 && resident_clusters<4, V>() >= p.n_tiles)
    return router_launch<4, V>(tmU, tmE, p, p.n_tiles, s);
  if (p.nk >= 2 && resident_clusters<2, V>() >= p.n_tiles)
    return router_launch<2, V>(tmU, tmE, p, p.n_tiles, s);
  const int pairs = resident_clusters<1, V>();
  if (pairs <= 0) return fail(MOE_ERR_CUDA, "router_tc: no resident CTA pair");
  return router_launch<1, V>(tmU, tmE, p, pairs < p.n_tiles ? pairs : p.n_tiles, s);
}

}  // namespace

bool router_tc_supported(moe_dtype dt, int d, int N_r, int K, int n_groups, int topk_groups) {
  (void)topk_groups;
  if (dt != MOE_BF16 || d % BK != 0 || N_r % 32 != 0 || N_r < 32 || N_r > kMaxN) return false;
  if (K < 1 || K > N_r) return false;
  return n_groups >= 1 && n_groups <= 32;
}

moe_status launch_router_tc(const void* u, const void* E, const float* b, int T, int d, int N_r,
                            int K, int n_groups, int topk_groups, int32_t* idx, float* gate,
                            int32_t* counts, float* logits, RefineLists rl, float refine_gap,
                            float near, cudaStream_t s) {
  if (T <= 0) return MOE_OK;
  CUtensorMap tmU, tmE;
  moe_status st = make_tmap_2d(&tmU, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, T, BK, TM);
  if (st != MOE_OK) return st;
  st = make_tmap_2d(&tmE, E, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N_r, BK, N_r / 2);
  if (st != MOE_OK) return st;
  RouterParams p;
  p.bias = b;
  p.T = T;
  p.N_r = N_r;
  p.K = K;
  p.nk = d / BK;
  p.n_tiles = (T + 2 * TM - 1) / (2 * TM);
  // column parts per token row when reading TMEM: the most (<= 4) that
  // split N_r into 16-column pieces
  p.parts = 1;
  for (int parts = kParts; parts > 1; --parts)
    if ((N_r / CH) % parts == 0) { p.parts = parts; break; }
  p.n_groups = n_groups;
  p.topk_groups = topk_groups;
  p.idx = idx;
  p.gate = gate;
  p.counts = counts;
  p.logits = logits;
  p.rl = rl;
  p.refine_gap = refine_gap;
  p.near = near;
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  const int V = N_r / 32;
  if (V <= 1) return router_dispatch_s<1>(tmU, tmE, p, s);
  if (V <= 2) return router_dispatch_s<2>(tmU, tmE, p, s);
  if (V <= 4) return router_dispatch_s<4>(tmU, tmE, p, s);
  return router_dispatch_s<8>(tmU, tmE, p, s);
}

}  // namespace moe
