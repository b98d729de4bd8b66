// Weights-stationary grouped bf16 GEMM on CTA pairs (tcgen05 cta_group::2)
// for the expert FFNs (FFN_i of the h'-equation, "DeepSeek-V3 技術報告",
// section 方法 / 2).
//
// A cluster of two CTAs on two SMs computes one tile: 2 x 256 weight rows by
// up to 256 of an expert's tokens.  Each tcgen05.mma.cta_group::2 (M = 256,
// N = the tile's token count rounded to 16) takes 128 weight rows (A) and
// half of the tokens (B) from each CTA's shared memory and leaves each CTA
// 128 rows x N columns of the result in its own TMEM.  Per 16-K slice the
// leader issues two such MMAs:
//   SWIGLU  gate rows [nt*256, +256) and the matching up rows: CTA r holds h
//           columns nt*256 + r*128 + [0, 128)
//   STORE   output rows nt*512 + [0, 256) and nt*512 + 256 + [0, 256): CTA r
//           holds columns nt*512 + hh*256 + r*128 + [0, 128), hh = 0, 1
// so an SM moves 32 KB of weights and at most 16 KB of tokens per 64-wide K
// step (1024 MMA cycles), and four 48 KB stages fit in shared memory.
//
// Synchronisation: both CTAs' TMA loads complete on the leader's "full"
// barrier (cta_group::2 loads name it); the leader's commits arrive on both
// CTAs' "empty" and "tmem full" barriers (multicast commit); both CTAs'
// epilogue warps arrive on the leader's "tmem empty" barrier.  Every wait is
// bounded (1 s, reported through the device error word); the two cluster
// barriers at start and end are reached by every thread in bounded time.
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace moe {

moe_status make_tmap_2d(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                        int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer);

namespace {

using namespace sm100;

constexpr int TMAX = 256;            // max tokens per tile (MMA N)
constexpr int BK = 64;               // bf16 elements per 128-byte swizzle row
constexpr int XBOX = 64;             // token rows per TMA box
constexpr int STAGES = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxGroups = 1024;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t TMEM_COLS = 512;

constexpr int W_BYTES = 256 * BK * 2;          // this CTA's 2 x 128 weight rows: 32 KB
constexpr int X_BYTES = (TMAX / 2) * BK * 2;   // this CTA's half of the tokens: 16 KB
constexpr int XBOX_BYTES = XBOX * BK * 2;      // 8 KB
constexpr int OFF_X = STAGES * W_BYTES;
constexpr int OFF_PATCH = OFF_X + STAGES * X_BYTES;
constexpr int OFF_BAR = OFF_PATCH + kEpiWarps * 2048;
constexpr int N_BARS = 2 * STAGES + 3;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int OFF_TAB = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_TAB + 2 * (kMaxGroups + 1) * 4;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

struct Ws2Params {
  const int32_t* offsets;
  int n_groups;
  int rows;
  int N;               // output columns
  int K;
  int b_rows_per_group;
  int half_b;          // SWIGLU: I
  __nv_bfloat16* C;
  int* err;
};

// ------------------------------------------------------------- pair PTX
__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_cta(uint32_t saddr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
  return out;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA tile load into this CTA's shared memory, completing on the pair leader's barrier.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* tm, int c0,
                                                 int c1, uint32_t leader_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(leader_bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void mma2_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// Arrives once on the barrier at this offset in both CTAs of the pair.
__device__ __forceinline__ void mma2_commit_both(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], m;\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mma2_commit_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem2_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem2_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem2_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// ------------------------------------------------------------- tiling
__device__ __forceinline__ void token_tiling(int m, int& n_t, int& step) {
  if (m <= 0) { n_t = 0; step = 16; return; }
  const int n0 = (m + TMAX - 1) / TMAX;
  step = ((m + n0 - 1) / n0 + 15) / 16 * 16;
  n_t = (m + step - 1) / step;
}

__device__ __forceinline__ void decode_tile(int t, const int* prefix, const int* roff, int G,
                                            int& g, int& nt, int& tok0, int& count) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  g = lo;
  const int m = roff[g + 1] - roff[g];
  int n_t, step;
  token_tiling(m, n_t, step);
  const int local = t - prefix[g];
  nt = local / n_t;
  const int ti = local - nt * n_t;
  tok0 = roff[g] + ti * step;
  count = min(step, m - ti * step);
}

__device__ __forceinline__ void raise_abort(volatile int* abort, int* err) {
  *abort = 1;
  atomicOr(err, ERR_GEMM_TIMEOUT);
}

__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

template <bool SWIGLU>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    ws2_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                    const __grid_constant__ CUtensorMap tmX, const Ws2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sW = smem;
  uint8_t* sX = smem + OFF_X;
  uint8_t* sPatch = smem + OFF_PATCH;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* mma_done = tempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  int* prefix = reinterpret_cast<int*>(smem + OFF_TAB);
  int* roff = prefix + kMaxGroups + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int G = p.offsets ? p.n_groups : 1;
  const int OUT = SWIGLU ? 256 : 512;            // output columns per pair tile
  const int n_wt = p.N / OUT;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(tfull, 1);
    mbar_init(tempty, 2 * kEpiWarps);            // one arrival per epilogue warp of both CTAs
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem2_alloc(tmem_slot, TMEM_COLS);
    tmem2_relinquish();
  }
  if (warp == 2) {
    const int per = (G + 31) / 32;
    const int g0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int g = g0 + i;
      if (g < G) {
        const int a = p.offsets ? p.offsets[g] : 0;
        const int b = p.offsets ? p.offsets[g + 1] : p.rows;
        int n_t, step;
        token_tiling(b - a, n_t, step);
        roff[g] = a;
        if (g == G - 1) roff[G] = b;
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
      if (g < G) {
        prefix[g] = run;
        int n_t, step;
        token_tiling(roff[g + 1] - roff[g], n_t, step);
        run += n_t * n_wt;
      }
    }
    if (lane == 31) prefix[G] = incl;
  }
  tc_fence_before();
  cluster_sync();          // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = prefix[G];
  const int nk = p.K / BK;
  const uint32_t full_leader0 = map_to_cta(smem_u32(&full[0]), 0);
  const uint32_t tempty_leader = map_to_cta(smem_u32(tempty), 0);

  if (warp == 0) {
    // ---------------------------------------------------------------- producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += n_pairs) {
        int g, nt, tok0, count;
        decode_tile(t, prefix, roff, G, g, nt, tok0, count);
        const int n_mma = (count + 15) / 16 * 16;
        const int half = n_mma / 2;                  // token rows this CTA supplies
        const int nbox = (half + XBOX - 1) / XBOX;
        const uint32_t bytes = 2 * (W_BYTES + nbox * XBOX_BYTES);   // both CTAs' loads
        const int wbase = g * p.b_rows_per_group;
        const int w0 = SWIGLU ? wbase + nt * 256 + rank * 128 : wbase + nt * 512 + rank * 128;
        const int w1 = SWIGLU ? w0 + p.half_b : w0 + 256;
        const int xrow = tok0 + rank * half;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
          const uint32_t fb = full_leader0 + stage * 8;
          uint8_t* w_dst = sW + stage * W_BYTES;
          tma_load_2d_pair(w_dst, &tmW, kb * BK, w0, fb);
          tma_load_2d_pair(w_dst + W_BYTES / 2, &tmW, kb * BK, w1, fb);
          uint8_t* x_dst = sX + stage * X_BYTES;
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_pair(x_dst + b * XBOX_BYTES, &tmX, kb * BK, xrow + b * XBOX, fb);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (leader)
        for (int s = 0; s < STAGES; ++s)
          mbar_wait_bounded(&full[s], ((s < stage) ? phase : phase ^ 1), nullptr, kWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0, tphase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += n_pairs) {
        int g, nt, tok0, count;
        decode_tile(t, prefix, roff, G, g, nt, tok0, count);
        const int n_mma = (count + 15) / 16 * 16;
        const uint32_t idesc = idesc_bf16_f32(256, n_mma);
        if (!mbar_wait_bounded(tempty, tphase ^ 1, abort_flag, kWaitNs)) {
          raise_abort(abort_flag, p.err);
          break;
        }
        tc_fence_after();
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
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t xd = smem_desc_k_sw128(x0 + k * 32);
            const uint32_t acc = (kb | k) != 0;
            mma2_f16_ss(tmem_base, smem_desc_k_sw128(w0 + k * 32), xd, idesc, acc);
            mma2_f16_ss(tmem_base + 256, smem_desc_k_sw128(w0 + W_BYTES / 2 + k * 32), xd, idesc,
                        acc);
          }
          mma2_commit_both(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        mma2_commit_both(tfull);
        tphase ^= 1;
      }
      mma2_commit_local(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr, kWaitNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int ch = (warp - 2) >> 2;
    uint16_t* patch = reinterpret_cast<uint16_t*>(sPatch + (warp - 2) * 2048);
    uint32_t tphase = 0;
    for (int t = pair; t < total; t += n_pairs) {
      int g, nt, tok0, count;
      decode_tile(t, prefix, roff, G, g, nt, tok0, count);
      const bool got = mbar_wait_bounded(tfull, tphase, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, got)) {
        raise_abort(abort_flag, p.err);
        break;
      }
      tc_fence_after();
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      const int nch = (count + 31) / 32;
      for (int c = ch; c < nch; c += 2) {
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(tl + c * 32, r0);
        tmem_ld_32x32b_x32(tl + 256 + c * 32, r1);
        tmem_wait_ld();
        const int half_n = SWIGLU ? 1 : 2;
#pragma unroll
        for (int hh = 0; hh < half_n; ++hh) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float v;
            if (SWIGLU) v = silu_f(__uint_as_float(r0[j])) * __uint_as_float(r1[j]);
            else v = __uint_as_float(hh == 0 ? r0[j] : r1[j]);
            patch[j * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
          }
          __syncwarp();
          const int col0 = SWIGLU ? nt * 256 + rank * 128 + q * 32
                                  : nt * 512 + hh * 256 + rank * 128 + q * 32;
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int j = it * 8 + (lane >> 2);
            const int tok = c * 32 + j;
            const uint4 v = *reinterpret_cast<const uint4*>(patch + j * 32 + (lane & 3) * 8);
            if (tok < count) {
              __nv_bfloat16* dst = p.C + (size_t)(tok0 + tok) * p.N + col0 + (lane & 3) * 8;
              *reinterpret_cast<uint4*>(dst) = v;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_remote(tempty_leader);
      tphase ^= 1;
    }
  }

  tc_fence_before();
  cluster_sync();          // no CTA leaves while its pair may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem2_dealloc(tmem_base, TMEM_COLS);
  }
}

template <bool SWIGLU>
moe_status ws2_launch(const void* X, const void* W, int b_rows_per_group, const int32_t* offsets,
                      int n_groups, int rows, int N, int K, void* C, cudaStream_t s) {
  CUtensorMap tmW, tmX;
  const int G = offsets ? n_groups : 1;
  moe_status st = make_tmap_2d(&tmW, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K,
                               (uint64_t)G * b_rows_per_group, BK, 128);
  if (st != MOE_OK) return st;
  st = make_tmap_2d(&tmX, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, rows, BK, XBOX);
  if (st != MOE_OK) return st;
  auto kern = ws2_gemm_kernel<SWIGLU>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
    if (e != cudaSuccess) return cuda_check(e, "ws2_gemm smem attribute");
    attr_set = true;
  }
  Ws2Params p;
  p.offsets = offsets;
  p.n_groups = n_groups;
  p.rows = rows;
  p.N = N;
  p.K = K;
  p.b_rows_per_group = b_rows_per_group;
  p.half_b = SWIGLU ? b_rows_per_group / 2 : 0;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  const int OUT = SWIGLU ? 256 : 512;
  const long long max_tiles = ((long long)(rows + TMAX - 1) / TMAX + (offsets ? G : 0)) * (N / OUT);
  // Persistent pairs: launch only as many as can be resident at once (GPCs
  // with an odd number of usable SMs leave some SMs without a partner).
  static int resident_pairs = 0;
  if (!resident_pairs) {
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
    cudaError_t e = cudaOccupancyMaxActiveClusters(&n, (const void*)kern, &cfg);
    if (e != cudaSuccess || n <= 0) return cuda_check(e != cudaSuccess ? e : cudaErrorInvalidConfiguration,
                                                       "ws2_gemm cluster occupancy");
    resident_pairs = n;
  }
  int pairs = resident_pairs;
  if (max_tiles < pairs) pairs = (int)(max_tiles > 0 ? max_tiles : 1);
  kern<<<2 * pairs, kThreads, SMEM_ALLOC, s>>>(tmW, tmX, p);
  return cuda_check(cudaGetLastError(), "ws2_gemm launch");
}

}  // namespace

bool ws2_supports(bool swiglu, int N) { return swiglu ? (N % 256 == 0) : (N % 512 == 0); }

moe_status launch_ws2_gemm(const void* X, const void* W, int b_rows_per_group,
                           const int32_t* offsets, int n_groups, int rows, int N, int K,
                           bool swiglu, void* C, cudaStream_t s) {
  if (rows <= 0) return MOE_OK;
  if (K % BK) return fail(MOE_ERR_UNSUPPORTED, "ws2 gemm: K=%d not a multiple of %d", K, BK);
  if (offsets && n_groups > kMaxGroups)
    return fail(MOE_ERR_UNSUPPORTED, "ws2 gemm: at most %d groups", kMaxGroups);
  if (!ws2_supports(swiglu, N)) return fail(MOE_ERR_UNSUPPORTED, "ws2 gemm: N=%d", N);
  if (swiglu) return ws2_launch<true>(X, W, b_rows_per_group, offsets, n_groups, rows, N, K, C, s);
  return ws2_launch<false>(X, W, b_rows_per_group, offsets, n_groups, rows, N, K, C, s);
}

}  // namespace moe
