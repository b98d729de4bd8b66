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
#include "sm100.cuh"

namespace moe {

moe_status make_tmap_2d(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                        int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer);

namespace {

using namespace sm100;

constexpr int BK = 64;                 // bf16 K elements per 128-byte swizzle row
constexpr int TM = 128;                // token rows per CTA (TMEM lanes)
constexpr int STAGES = 6;
constexpr int kMaxN = 256;             // N_r limit of the pair MMA
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr uint64_t kWaitNs = 1000000000ull;

constexpr int A_BYTES = TM * BK * 2;                  // 16 KB
constexpr int B_MAX_BYTES = (kMaxN / 2) * BK * 2;     // 16 KB
constexpr int OFF_B = STAGES * A_BYTES;
constexpr int OFF_BAR = OFF_B + STAGES * B_MAX_BYTES;
constexpr int N_BARS = 2 * STAGES + 4;                // full, empty, tfull, tempty, peer_ready, mma_done
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;        // tmem slot, abort flag
constexpr int OFF_BIAS = OFF_MISC + 16;               // float [kMaxN]
constexpr int OFF_HIST = OFF_BIAS + kMaxN * 4;        // int [kMaxN]
constexpr int OFF_GS = OFF_HIST + kMaxN * 4;          // float [32 groups][128 rows]
constexpr int SMEM_BYTES = OFF_GS + 32 * TM * 4;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
constexpr int STAGE_LD = kMaxN + 4;                   // float stride of a staged partial row

struct RouterParams {
  const float* bias;     // [N_r]
  int T, N_r, K;
  int nk;                // d / BK
  int n_tiles;           // ceil(T / 256)
  int n_groups, topk_groups, gshift;   // grouped: group of expert e is e >> gshift
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

__device__ __forceinline__ float affinity32(float x) { return 1.0f / (1.0f + expf(-x)); }

// Logits of this thread's token for columns [c*32, c*32+32): its own TMEM
// partial plus, in slice order, the partials the other S-1 pairs staged.
template <int S>
__device__ __forceinline__ void load_logits32(uint32_t tmem_row, int c, const uint32_t* peer_row,
                                              float* x) {
  uint32_t r[32];
  tmem_ld_32x32b_x32(tmem_row + c * 32, r);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(r[j]);
#pragma unroll
  for (int q = 1; q < S; ++q) {
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const float4 f = ld_shared_cluster_v4(peer_row[q] + (uint32_t)(c * 32 + 4 * v) * 4u);
      x[4 * v] += f.x;
      x[4 * v + 1] += f.y;
      x[4 * v + 2] += f.z;
      x[4 * v + 3] += f.w;
    }
  }
}

// Inserts (key, e, s) into the list sorted by (key desc, index asc): slots
// [0, K] hold the K+1 best so far; a new key equal to a listed one goes
// after it (experts arrive in ascending order).
template <int KMAX>
__device__ __forceinline__ void insert_top(float key, int e, float s, int K, float* tk, int* te,
                                           float* ts) {
#pragma unroll
  for (int j = KMAX; j >= 1; --j) {
    if (j <= K) {
      if (key > tk[j - 1]) {
        tk[j] = tk[j - 1];
        te[j] = te[j - 1];
        ts[j] = ts[j - 1];
      } else if (key > tk[j]) {
        tk[j] = key;
        te[j] = e;
        ts[j] = s;
      }
    }
  }
  if (key > tk[0]) {
    tk[0] = key;
    te[0] = e;
    ts[0] = s;
  }
}

template <int KMAX>
__device__ __forceinline__ float slot_value(const float* a, int k) {
  float v = a[0];
#pragma unroll
  for (int j = 1; j <= KMAX; ++j)
    if (j == k) v = a[j];
  return v;
}

template <int S, int KMAX, bool GROUPED>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmU,
                     const __grid_constant__ CUtensorMap tmE, const RouterParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + OFF_B;
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
  float* s_gscore = reinterpret_cast<float*>(smem + OFF_GS);

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
    const int q = warp & 3;                       // TMEM lane quarter
    const int row = q * 32 + lane;                // token row of this CTA
    const uint32_t tmem_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    float* stage_row = reinterpret_cast<float*>(smem) + (size_t)row * STAGE_LD;
    uint32_t tphase = 0;
    for (int tile = first_tile; tile < p.n_tiles; tile += tile_step) {
      const bool got = mbar_wait_bounded(tfull, tphase, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, got)) {
        raise_abort(abort_flag, p.err);
        break;
      }
      tc_fence_after();
      if (slice > 0) {
        // stage this slice's partial logits for the first pair, then signal it
        for (int c = 0; c < N / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem_row + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int v = 0; v < 8; ++v)
            *reinterpret_cast<uint4*>(stage_row + c * 32 + 4 * v) =
                make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
        }
        __syncwarp();
        if (lane == 0)
          mbar_arrive_remote(map_shared_to(smem_u32(peer_ready), rank - 2u * (uint32_t)slice));
        tc_fence_before();
        break;                                  // S > 1: one tile per cluster
      }
      uint32_t peer_row[S > 1 ? S : 1];
      if (S > 1) {
        const bool ready = mbar_wait_cluster_bounded(peer_ready, 0, abort_flag, kWaitNs);
        if (!__all_sync(0xffffffffu, ready)) {
          raise_abort(abort_flag, p.err);
          break;
        }
#pragma unroll
        for (int s2 = 1; s2 < S; ++s2)
          peer_row[s2] = map_shared_to(smem_u32(stage_row), rank + 2u * (uint32_t)s2);
      }
      const int t = tile * 2 * TM + (int)half * TM + row;
      const bool tv = t < p.T;
      const int K = p.K;
      // ---- group limit: group scores, kept groups, the kept-vs-excluded gap
      float margin = INFINITY, next_group = INFINITY;
      unsigned kept = 0xffffffffu;
      if (GROUPED) {
        const int G = p.n_groups;
        for (int g = 0; g < G; ++g) s_gscore[g * TM + row] = -INFINITY;
        for (int c = 0; c < N / 32; ++c) {
          float x[32];
          load_logits32<S>(tmem_row, c, peer_row, x);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int e = c * 32 + j;
            const float key = affinity32(x[j]) + s_bias[e];
            float* gs = &s_gscore[(e >> p.gshift) * TM + row];
            *gs = fmaxf(*gs, key);
          }
        }
        // topk_groups rounds of (score desc, group asc), plus one round that
        // finds the best excluded group
        kept = 0u;
        float last_kept = INFINITY;
        for (int r = 0; r <= p.topk_groups; ++r) {
          float bk = -INFINITY;
          int bg = -1;
          for (int g = 0; g < G; ++g) {
            const float v = s_gscore[g * TM + row];
            if (!((kept >> g) & 1u) && (bg < 0 || v > bk)) { bk = v; bg = g; }
          }
          if (r < p.topk_groups) {
            kept |= 1u << bg;
            last_kept = bk;
          } else {
            margin = last_kept - bk;
            next_group = bk;
          }
        }
      }
      // ---- top-(K+1) of the eligible keys, sorted by (key desc, index asc)
      float tk[KMAX + 1], ts[KMAX + 1];
      int te[KMAX + 1];
#pragma unroll
      for (int j = 0; j <= KMAX; ++j) {
        tk[j] = -INFINITY;
        ts[j] = 0.f;
        te[j] = 0x7fffffff;
      }
      float thr = -INFINITY;                        // the (K+1)-th key so far
      for (int c = 0; c < N / 32; ++c) {
        float x[32];
        load_logits32<S>(tmem_row, c, peer_row, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int e = c * 32 + j;
          const float s = affinity32(x[j]);
          const float key = s + s_bias[e];
          const bool elig = !GROUPED || ((kept >> (e >> p.gshift)) & 1u);
          if (elig && key > thr) {
            insert_top<KMAX>(key, e, s, K, tk, te, ts);
            thr = slot_value<KMAX>(tk, K);
          }
        }
      }
      // ---- gates, outputs, load
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < K) sum += ts[j];
      if (tv) {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (j < K) {
            p.idx[(size_t)t * K + j] = te[j];
            p.gate[(size_t)t * K + j] = ts[j] / sum;
            atomicAdd(&s_hist[te[j]], 1);
          }
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (j < K) margin = fminf(margin, tk[j] - tk[j + 1]);   // tk[K] = -inf when K = N_r
      }
      // ---- near-tie listing: the token, every expert whose key lies within
      // `near` of the lowest key a decision hinged on, and its logit row
      const bool listed = tv && margin < p.refine_gap;
      if (__any_sync(0xffffffffu, listed)) {
        const float lim = fminf(thr, next_group) - p.near;
        int cnt = 0;
        int32_t* pr = p.rl.pair + (size_t)t * N;
        float* lg = p.logits + (size_t)t * N;
        for (int c = 0; c < N / 32; ++c) {
          float x[32];
          load_logits32<S>(tmem_row, c, peer_row, x);
          if (listed) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int e = c * 32 + j;
              lg[e] = x[j];
              const float key = affinity32(x[j]) + s_bias[e];
              if (key >= lim) pr[cnt++] = t * N + e;
            }
          }
        }
        if (listed) {
          const int slot = atomicAdd(&p.rl.hdr[0], 1);
          p.rl.tok[slot] = t;
          p.rl.start[slot] = t * N;
          p.rl.num[slot] = cnt;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_leader);
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

template <int S, int KMAX, bool GROUPED>
moe_status router_launch(const CUtensorMap& tmU, const CUtensorMap& tmE, const RouterParams& p,
                         int n_clusters, cudaStream_t s) {
  auto kern = router_tc_kernel<S, KMAX, GROUPED>;
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
template <int S, int KMAX, bool GROUPED>
int resident_clusters() {
  static int cached[kMaxSmemDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSmemDevices) return 0;
  if (cached[dev]) return cached[dev];
  auto kern = router_tc_kernel<S, KMAX, GROUPED>;
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

template <int KMAX, bool GROUPED>
moe_status router_dispatch_s(const CUtensorMap& tmU, const CUtensorMap& tmE,
                             const RouterParams& p, cudaStream_t s) {
  // the largest slice count whose clusters all run in one wave and whose
  // slices each get at least one 64-wide block of the contraction
  if (p.nk >= 4 && resident_clusters<4, KMAX, GROUPED>() >= p.n_tiles)
    return router_launch<4, KMAX, GROUPED>(tmU, tmE, p, p.n_tiles, s);
  if (p.nk >= 2 && resident_clusters<2, KMAX, GROUPED>() >= p.n_tiles)
    return router_launch<2, KMAX, GROUPED>(tmU, tmE, p, p.n_tiles, s);
  const int pairs = resident_clusters<1, KMAX, GROUPED>();
  if (pairs <= 0) return fail(MOE_ERR_CUDA, "router_tc: no resident CTA pair");
  return router_launch<1, KMAX, GROUPED>(tmU, tmE, p, pairs < p.n_tiles ? pairs : p.n_tiles, s);
}

}  // namespace

bool router_tc_supported(moe_dtype dt, int d, int N_r, int K, int n_groups, int topk_groups) {
  if (dt != MOE_BF16 || d % BK != 0 || N_r % 32 != 0 || N_r < 32 || N_r > kMaxN) return false;
  if (K < 1 || K > 16) return false;
  if (n_groups > 1 && topk_groups < n_groups) {
    const int gs = N_r / n_groups;
    if (n_groups > 32 || (gs & (gs - 1)) != 0) return false;
  }
  return true;
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
  const bool grouped = n_groups > 1 && topk_groups < n_groups;
  p.n_groups = grouped ? n_groups : 1;
  p.topk_groups = grouped ? topk_groups : 1;
  p.gshift = 0;
  if (grouped)
    while ((1 << p.gshift) < N_r / n_groups) ++p.gshift;
  p.idx = idx;
  p.gate = gate;
  p.counts = counts;
  p.logits = logits;
  p.rl = rl;
  p.refine_gap = refine_gap;
  p.near = near;
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  if (K <= 8)
    return grouped ? router_dispatch_s<8, true>(tmU, tmE, p, s)
                   : router_dispatch_s<8, false>(tmU, tmE, p, s);
  return grouped ? router_dispatch_s<16, true>(tmU, tmE, p, s)
                 : router_dispatch_s<16, false>(tmU, tmE, p, s);
}

}  // namespace moe
