// Weights-stationary grouped bf16 GEMM on CTA pairs (tcgen05 cta_group::2)
// for the forward down projections (the W_down product of FFN_i in the
// h'-equation, "DeepSeek-V3 技術報告", section 方法 / 2): routed groups, and the
// shared experts as extra groups.
//
// A tile is 256 weight rows x up to 256 token rows, computed by the two CTAs
// of a cluster as one M = 256 MMA per 16-element K slice:
//   CTA r holds weight rows [128 r, 128 r + 128) of the tile (its A operand)
//   and token rows [r N/2, (r+1) N/2) (its half of B), and keeps the
//   accumulator rows of its own weight rows for all N tokens in its TMEM:
//   y[tok, nt*256 + 128r + n] = bf16(D[n, tok]).
// N is the tile's token count rounded up to 16 (each half a multiple of 8
// rows, one swizzle atom); an expert with M tokens is cut into ceil(M/256)
// equal token tiles.  Each CTA's accumulator is 128 lanes x N <= 256
// columns, so TMEM (512 columns) holds two: the epilogue of one tile runs
// while the MMA of the next accumulates into the other buffer.  A pipeline
// stage spans 128 K elements (two 128-byte swizzle atoms): one TMA operation
// brings this CTA's 128 weight rows (32 KB, a 3-d map of K atoms) and one its
// token rows (a 64- or 128-row box; the box may read past the tile's rows,
// which the epilogue never stores).  Output values go through a
// shared-memory patch per warp so that global stores are 16-byte vectors
// along token rows.
//
// Roles (each CTA): warp 0 TMA producer (its own weight rows and token rows;
// completion counted on the pair leader's barrier), warp 1 TMEM allocator and,
// in the leader, MMA issuer; warps 2-9 epilogue (lane quarter warp % 4,
// alternate 32-token chunks).  Every wait is bounded (1 s) and reported
// through the device error word.  Every CTA loads its own tiles.
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace moe {

moe_status make_tmap_col_blocks(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                                int elem_bytes, uint64_t cols, uint64_t rows, uint32_t bc,
                                uint32_t box_rows, uint32_t box_blocks);

namespace {

using namespace sm100;

constexpr int TMAX = 256;           // max token rows per tile (MMA N)
constexpr int TGRAN = 16;           // token rows per tile are a multiple of this (MMA N)
constexpr int BK = 64;              // bf16 elements per 128-byte swizzle atom
constexpr int KA = 2;               // swizzle atoms per pipeline stage
constexpr int BKS = BK * KA;        // K elements per stage
constexpr int STAGES = 3;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxGroups = 1024;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t TMEM_COLS = 512;   // two accumulators of up to 256 columns

constexpr int ATOM_W = 128 * BK * 2;            // 16 KB: 128 weight rows x one atom
constexpr int W_BYTES = KA * ATOM_W;            // 32 KB per stage
constexpr int X_BYTES = KA * (TMAX / 2) * BK * 2;   // 32 KB: at most 128 token rows
constexpr int OFF_X = STAGES * W_BYTES;
constexpr int OFF_PATCH = OFF_X + STAGES * X_BYTES;   // 2 KB output patch per epilogue warp
constexpr int OFF_BAR = OFF_PATCH + kEpiWarps * 2048;
constexpr int N_BARS = 2 * STAGES + 5;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int OFF_TAB = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_TAB + 2 * (kMaxGroups + 1) * 4;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory");

struct Ws2Params {
  const int32_t* offsets;   // [n_groups+1] or nullptr (one group of `rows`)
  int n_groups;
  int rows;
  int N;                    // output columns (d)
  int K;
  int b_rows_per_group;     // rows of W per group
  __nv_bfloat16* C;
  int ldc;
  int n_extra;              // extra groups after the routed ones (0: none)
  int T_extra;              // rows of each extra group
  int x_extra_local;        // 1: extra groups read X rows [0, T_extra); 0: their C rows
  int* err;
};

// Token tiling of a group of m rows: tiles of `step` rows (a multiple of
// TGRAN, at most TMAX), n_t = ceil(m / step) tiles, the last possibly shorter.
__device__ __forceinline__ void token_tiling(int m, int& n_t, int& step) {
  if (m <= 0) { n_t = 0; step = TGRAN; return; }
  const int n0 = (m + TMAX - 1) / TMAX;
  step = ((m + n0 - 1) / n0 + TGRAN - 1) / TGRAN * TGRAN;
  n_t = (m + step - 1) / step;
}

__device__ __forceinline__ void group_span(int g, int G, const int* roff, const Ws2Params& p,
                                           int& base, int& m) {
  if (g < G) {
    base = roff[g];
    m = roff[g + 1] - roff[g];
  } else {
    base = p.rows + (g - G) * p.T_extra;
    m = p.T_extra;
  }
}

// Tile t -> group g, weight tile nt, first C row tok0, rows count, first X row.
__device__ __forceinline__ void decode_tile(int t, const int* prefix, const int* roff, int G,
                                            int Gtot, const Ws2Params& p, int& g, int& nt,
                                            int& tok0, int& count, int& xrow0) {
  int lo = 0, hi = Gtot - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  g = lo;
  int base, m;
  group_span(g, G, roff, p, base, m);
  int n_t, step;
  token_tiling(m, n_t, step);
  const int local = t - prefix[g];
  nt = local / n_t;
  const int ti = local - nt * n_t;
  tok0 = base + ti * step;
  count = min(step, m - ti * step);
  xrow0 = (g >= G && p.x_extra_local) ? ti * step : tok0;
}

__device__ __forceinline__ void raise_abort(volatile int* abort, int* err) {
  *abort = 1;
  atomicOr(err, ERR_GEMM_TIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 1)
    ws2_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ CUtensorMap tmXb,
                    const __grid_constant__ CUtensorMap tmW2,
                    const __grid_constant__ CUtensorMap tmX2,
                    const __grid_constant__ CUtensorMap tmX2b, const Ws2Params p) {
  constexpr int OUT_COLS = 256;                    // output columns per weight tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sW = smem;
  uint8_t* sX = smem + OFF_X;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;   // [2]
  uint64_t* tempty = tfull + 2;       // [2] (leader: epilogue warps of both CTAs)
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  int* prefix = reinterpret_cast<int*>(smem + OFF_TAB);
  int* roff = prefix + kMaxGroups + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();        // 0: leader, 1: peer
  const bool is_leader = rank == 0;
  const uint16_t pair_mask = 3u;
  const int G = p.offsets ? p.n_groups : 1;
  const int Gtot = G + p.n_extra;
  const int n_wt = p.N / OUT_COLS;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 2 * kEpiWarps); }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmXb);
    if (p.n_extra) {
      tma_prefetch_desc(&tmW2);
      tma_prefetch_desc(&tmX2);
      tma_prefetch_desc(&tmX2b);
    }
  }
  if (warp == 1) {
    tmem2_alloc(tmem_slot, TMEM_COLS);
    tmem2_relinquish();
  }
  if (warp == 2) {
    // tile table (the same in both CTAs): prefix[g] = first tile of group g;
    // a group's tiles run weight-tile major, token-tile fastest
    load_offsets_warp(p.offsets, G, p.rows, roff, p.err);
    const int per = (Gtot + 31) / 32;
    const int g0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int g = g0 + i;
      if (g < Gtot) {
        int base, m, n_t, step;
        group_span(g, G, roff, p, base, m);
        token_tiling(m, n_t, step);
        local += n_t * n_wt;
      }
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    __syncwarp();
    int run = incl - local;
    for (int i = 0; i < per; ++i) {
      const int g = g0 + i;
      if (g < Gtot) {
        prefix[g] = run;
        int base, m, n_t, step;
        group_span(g, G, roff, p, base, m);
        token_tiling(m, n_t, step);
        run += n_t * n_wt;
      }
    }
    if (lane == 31) prefix[Gtot] = incl;
  }
  tc_fence_before();
  cluster_sync_all();          // barriers of both CTAs initialised, TMEM allocated in the pair
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = prefix[Gtot];
  const int nk = p.K / BKS;
  const int first_tile = (int)cluster_id_x();
  const int tile_step = (int)n_clusters_x();
  const uint32_t full_leader0 = map_shared_to(smem_u32(&full[0]), 0);
  const uint32_t tempty_leader0 = map_shared_to(smem_u32(&tempty[0]), 0);

  if (warp == 0) {
    // ---------------------------------------------------------------- producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = first_tile; t < total && ok; t += tile_step) {
        int g, nt, tok0, count, xrow0;
        decode_tile(t, prefix, roff, G, Gtot, p, g, nt, tok0, count, xrow0);
        const bool extra = g >= G;
        const CUtensorMap* tw = extra ? &tmW2 : &tmW;
        const int half = (count + TGRAN - 1) / TGRAN * (TGRAN / 2);   // token rows per CTA
        const bool big = half > 64;                                     // 128-row token box
        const CUtensorMap* tx = extra ? (big ? &tmX2b : &tmX2) : (big ? &tmXb : &tmX);
        const uint32_t bytes = 2u * (uint32_t)(W_BYTES + KA * (big ? 128 : 64) * BK * 2);
        const int gw = (extra ? g - G : g) * p.b_rows_per_group;
        const int wrow = gw + nt * 256 + (int)rank * 128;
        const int xrow = xrow0 + (int)rank * half;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          if (is_leader) mbar_arrive_expect_tx(&full[stage], bytes);
          const uint32_t fb = full_leader0 + stage * 8;
          tma_load_3d_pair(sW + stage * W_BYTES, tw, 0, wrow, kb * KA, fb);   // [atom][128 rows]
          tma_load_3d_pair(sX + stage * X_BYTES, tx, 0, xrow, kb * KA, fb);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // the leader waits until every armed stage's copies (both CTAs') have landed
      if (is_leader)
        for (int s = 0; s < STAGES; ++s)
          mbar_wait_bounded(&full[s], ((s < stage) ? phase : phase ^ 1), nullptr, kWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    if (is_leader && lane == 0) {
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = first_tile; t < total && ok; t += tile_step, ++it) {
        int g, nt, tok0, count, xrow0;
        decode_tile(t, prefix, roff, G, Gtot, p, g, nt, tok0, count, xrow0);
        const int n_mma = (count + TGRAN - 1) / TGRAN * TGRAN;
        const uint32_t idesc = idesc_bf16_f32(256, n_mma);
        const int a = it & 1;
        if (!mbar_wait_cluster_bounded(&tempty[a], ((it >> 1) & 1) ^ 1, abort_flag, kWaitNs)) {
          raise_abort(abort_flag, p.err);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)a * 256u;
        const uint32_t x_atom = (n_mma / 2 > 64 ? 128u : 64u) * BK * 2;   // token box rows x 128 B
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w0 = smem_u32(sW + stage * W_BYTES);
          const uint32_t x0 = smem_u32(sX + stage * X_BYTES);
#pragma unroll
          for (int at = 0; at < KA; ++at)
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              mma2_f16_ss(d_tmem, smem_desc_k_sw128(w0 + at * ATOM_W + k * 32),
                          smem_desc_k_sw128(x0 + at * x_atom + k * 32), idesc,
                          (kb | at | k) != 0 ? 1u : 0u);
          mma2_commit_mask(&empty[stage], pair_mask);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma2_commit_mask(&tfull[a], pair_mask);
      }
      mma2_commit_local(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr, kWaitNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;                       // TMEM lane quarter
    const int ch = (warp - 2) >> 2;               // alternate 32-token chunks
    uint16_t* patch = reinterpret_cast<uint16_t*>(smem + OFF_PATCH + (warp - 2) * 2048);
    int it = 0;
    for (int t = first_tile; t < total; t += tile_step, ++it) {
      int g, nt, tok0, count, xrow0;
      decode_tile(t, prefix, roff, G, Gtot, p, g, nt, tok0, count, xrow0);
      const int a = it & 1;
      const bool got = mbar_wait_bounded(&tfull[a], (it >> 1) & 1, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) raise_abort(abort_flag, p.err);
        break;
      }
      tc_fence_after();
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (uint32_t)a * 256u;
      const int nch = (count + 31) / 32;
      for (int c = ch; c < nch; c += 2) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tl + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          patch[j * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[j])));
        __syncwarp();
        const int col = nt * 256 + (int)rank * 128 + q * 32 + (lane & 3) * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = i * 8 + (lane >> 2);
          const int tok = c * 32 + j;
          const uint4 v = *reinterpret_cast<const uint4*>(patch + j * 32 + (lane & 3) * 8);
          if (tok < count && in_bounds(tok0 + tok < p.rows + p.n_extra * p.T_extra, p.err))
            *reinterpret_cast<uint4*>(p.C + (size_t)(tok0 + tok) * p.ldc + col) = v;
        }
        __syncwarp();                             // the patch is rewritten next
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_leader0 + (uint32_t)a * 8u);   // accumulator read
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();          // neither CTA leaves while the pair's MMA or loads may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem2_dealloc(tmem_base, TMEM_COLS);
  }
}

int ws2_resident_pairs() {
  static int cached[kMaxSmemDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSmemDevices) return 0;
  if (cached[dev]) return cached[dev];
  auto kern = ws2_gemm_kernel;
  static bool attr_done[kMaxSmemDevices] = {};
  if (ensure_max_smem(reinterpret_cast<const void*>(kern), SMEM_ALLOC, attr_done,
                      "ws2_gemm smem attribute") != MOE_OK)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sm_count() / 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
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

moe_status ws2_launch(const void* X, const void* W, int b_rows_per_group, const int32_t* offsets,
                      int n_groups, int rows, int N, int K, void* C, const WsExtraGroups& ex,
                      cudaStream_t s) {
  constexpr int OUT_COLS = 256;
  CUtensorMap tmW, tmX, tmXb, tmW2, tmX2, tmX2b;
  const int G = offsets ? n_groups : 1;
  long long x_rows = ex.n_extra && !ex.x_local ? rows + (long long)ex.n_extra * ex.T : rows;
  if (x_rows == 0) x_rows = ex.T;   // no routed rows: a map over the extra X, never read
  // weights [atom][128 rows][64 k]; tokens [atom][64 or 128 rows][64 k]
  auto wmap = [&](CUtensorMap* tm, const void* base, long long groups) {
    return make_tmap_col_blocks(tm, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K,
                                (uint64_t)(groups * b_rows_per_group), BK, 128, KA);
  };
  auto xmap = [&](CUtensorMap* tm, const void* base, long long n, uint32_t box_rows) {
    return make_tmap_col_blocks(tm, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, (uint64_t)n,
                                BK, box_rows, KA);
  };
  moe_status st = wmap(&tmW, W, G);
  if (st != MOE_OK) return st;
  if ((st = xmap(&tmX, X, x_rows, 64)) != MOE_OK) return st;
  if ((st = xmap(&tmXb, X, x_rows, 128)) != MOE_OK) return st;
  tmW2 = tmW;
  tmX2 = tmX;
  tmX2b = tmXb;
  if (ex.n_extra) {
    if ((st = wmap(&tmW2, ex.W, ex.n_extra)) != MOE_OK) return st;
    if (ex.x_local) {
      if ((st = xmap(&tmX2, ex.X, ex.T, 64)) != MOE_OK) return st;
      if ((st = xmap(&tmX2b, ex.X, ex.T, 128)) != MOE_OK) return st;
    }
  }
  auto kern = ws2_gemm_kernel;
  static bool attr_done[kMaxSmemDevices] = {};
  {
    const moe_status sst = ensure_max_smem(reinterpret_cast<const void*>(kern), SMEM_ALLOC,
                                           attr_done, "ws2_gemm smem attribute");
    if (sst != MOE_OK) return sst;
  }
  Ws2Params p;
  p.offsets = offsets;
  p.n_groups = n_groups;
  p.rows = rows;
  p.N = N;
  p.K = K;
  p.b_rows_per_group = b_rows_per_group;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.ldc = N;
  p.n_extra = ex.n_extra;
  p.T_extra = ex.T;
  p.x_extra_local = ex.x_local ? 1 : 0;
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  const long long max_tiles =
      ((long long)(rows + TMAX - 1) / TMAX + (offsets ? G : 0) +
       (long long)ex.n_extra * ((ex.T + TMAX - 1) / TMAX)) * (N / OUT_COLS);
  int pairs = ws2_resident_pairs();
  if (pairs <= 0) return fail(MOE_ERR_CUDA, "ws2_gemm: no resident CTA pair");
  if (max_tiles < pairs) pairs = (int)(max_tiles > 0 ? max_tiles : 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, kern, tmW, tmX, tmXb, tmW2, tmX2, tmX2b, p),
                    "ws2_gemm launch");
}

}  // namespace

bool ws2_gemm_supported(int N, int K, int n_groups, bool grouped) {
  if (K <= 0 || K % BKS) return false;
  if (grouped && n_groups > kMaxGroups) return false;
  return N % 256 == 0;
}

moe_status launch_ws2_gemm(const void* X, const void* W, int b_rows_per_group,
                           const int32_t* offsets, int n_groups, int rows, int N, int K, void* C,
                           cudaStream_t s, const WsExtraGroups* extra) {
  const WsExtraGroups none{};
  const WsExtraGroups& ex = extra ? *extra : none;
  if (rows <= 0 && (ex.n_extra == 0 || ex.T <= 0)) return MOE_OK;
  if (!ws2_gemm_supported(N, K, n_groups, offsets != nullptr))
    return fail(MOE_ERR_UNSUPPORTED, "ws2 gemm: N=%d K=%d not supported", N, K);
  return ws2_launch(X, W, b_rows_per_group, offsets, n_groups, rows, N, K, C, ex, s);
}

}  // namespace moe
