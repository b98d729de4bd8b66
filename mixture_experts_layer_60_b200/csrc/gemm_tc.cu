// Grouped bf16 GEMM on the 5th-generation tensor cores (tcgen05), the dense
// contraction inside the expert FFNs (FFN_i of the h'-equation in
// "DeepSeek-V3 技術報告", section 方法 / 2) and of the router logits
// (u_t^T e_i, affinity line of the same section).
//
// For every group g and every row r in [offsets[g], offsets[g+1]):
//   acc[r, n] = sum_k A[r, k] * B[g * b_rows + n, k]        (A, B K-major bf16)
// and one of three epilogues:
//   STORE_BF16  C[r, n] = bf16(acc)
//   STORE_F32   C[r, n] = acc
//   SWIGLU      B holds W_gate rows [0, I) and W_up rows [I, 2I) of a group;
//               C[r, n] = bf16(SiLU(acc_gate) * acc_up), n < I.
//
// Structure: a persistent kernel, one CTA per SM, 6 warps:
//   warp 0     TMA producer: 128-byte-swizzled A and B tiles into a ring of
//              shared-memory stages (mbarrier "full" with transaction bytes)
//   warp 1     allocates TMEM; one lane issues tcgen05.mma (M=128, N=BN,
//              K=16 each) into one of two TMEM accumulators and releases a
//              stage with tcgen05.commit on its "empty" mbarrier
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//              lanes 32*(w%4)..+31 = tile rows), fused SiLU*up / casts,
//              16-byte stores; then frees the accumulator.
// Tiles are (group, n-tile, m-tile) with the m-tile fastest, so the CTAs
// that share one weight tile run side by side and the second read hits L2.
// Every wait is bounded (1 s); on expiry the kernel records
// ERR_GEMM_TIMEOUT in the device error word, and every role drains and exits.
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = 128;            // tile rows (TMEM lanes)
constexpr int BK = 64;             // bf16 elements per 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kMaxGroups = 1024;
constexpr uint64_t kWaitNs = 1000000000ull;

struct TcParams {
  const int32_t* offsets;  // [n_groups+1], or nullptr for one group of `rows` rows
  int n_groups;
  int rows;
  int N;                   // output columns
  int K;
  int b_rows_per_group;
  int half_b;              // SWIGLU: row offset of W_up inside a group (= I)
  void* C;
  int* err;
};

template <int BN, int STAGES>
struct Layout {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int OFF_B = STAGES * A_BYTES;
  static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
  static constexpr int N_BARS = 2 * STAGES + 5;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;     // tmem slot, abort flag
  static constexpr int OFF_TAB = OFF_MISC + 16;             // tile prefix, row offsets
  static constexpr int BYTES = OFF_TAB + 2 * (kMaxGroups + 1) * 4;
  static constexpr int ALLOC = BYTES + 1024;                 // room to align the base
};

template <int BN>
constexpr int tmem_cols() { return 2 * BN < 32 ? 32 : 2 * BN; }

__device__ __forceinline__ void decode_tile(int t, const int* prefix, const int* roff, int G,
                                            int& g, int& nt, int& row0, int& m_valid) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  g = lo;
  const int m = roff[g + 1] - roff[g];
  const int mtc = (m + BM - 1) / BM;
  const int local = t - prefix[g];
  nt = local / mtc;
  const int mt = local - nt * mtc;
  row0 = roff[g] + mt * BM;
  m_valid = min(BM, m - mt * BM);
}

__device__ __forceinline__ void raise_abort(volatile int* abort, int* err, int bit) {
  *abort = 1;
  atomicOr(err, bit);
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + __expf(-x)); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&p);
}

template <int BN, int EPI, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const TcParams p) {
  using L = Layout<BN, STAGES>;
  constexpr int BN_OUT = (EPI == TC_EPI_SWIGLU_BF16) ? BN / 2 : BN;
  constexpr uint32_t TMEM_COLS = tmem_cols<BN>();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + L::OFF_B;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;  // teardown: all issued MMAs complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  int* prefix = reinterpret_cast<int*>(smem + L::OFF_TAB);
  int* roff = prefix + kMaxGroups + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.offsets ? p.n_groups : 1;
  const int n_tiles_n = p.N / BN_OUT;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 4); }   // one per epilogue warp
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2) {
    // Tile table: prefix[g] = first tile of group g (tiles ordered n-major, m
    // fastest), from offsets clamped into disjoint ranges of [0, rows).
    load_offsets_warp(p.offsets, G, p.rows, roff, p.err);
    const int per = (G + 31) / 32;
    const int g0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int g = g0 + i;
      if (g < G) local += ((roff[g + 1] - roff[g] + BM - 1) / BM) * n_tiles_n;
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    __syncwarp();  // roff[] written by other lanes is read below
    int run = incl - local;
    for (int i = 0; i < per; ++i) {
      const int g = g0 + i;
      if (g < G) {
        prefix[g] = run;
        run += ((roff[g + 1] - roff[g] + BM - 1) / BM) * n_tiles_n;
      }
    }
    if (lane == 31) prefix[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = prefix[G];
  const int nk = p.K / BK;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int g, nt, row0, mv;
        decode_tile(t, prefix, roff, G, g, nt, row0, mv);
        const int brow = g * p.b_rows_per_group + nt * BN_OUT;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err, ERR_GEMM_TIMEOUT);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L::STAGE_BYTES);
          tma_load_2d(sA + stage * L::A_BYTES, &tmA, kb * BK, row0, &full[stage]);
          if (EPI == TC_EPI_SWIGLU_BF16) {
            tma_load_2d(sB + stage * L::B_BYTES, &tmB, kb * BK, brow, &full[stage]);
            tma_load_2d(sB + stage * L::B_BYTES + L::B_BYTES / 2, &tmB, kb * BK, brow + p.half_b,
                        &full[stage]);
          } else {
            tma_load_2d(sB + stage * L::B_BYTES, &tmB, kb * BK, brow, &full[stage]);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // Drain: every armed stage's copy must land before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        mbar_wait_bounded(&full[s], ((s < stage) ? phase : phase ^ 1), nullptr, kWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, kWaitNs)) {
          raise_abort(abort_flag, p.err, ERR_GEMM_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err, ERR_GEMM_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * L::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * L::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_f16_ss(d_tmem, smem_desc_k_sw128(a0 + k * 32), smem_desc_k_sw128(b0 + k * 32),
                       idesc, (kb | k) != 0);
          mma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        mma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // Let every issued MMA finish before TMEM is released.  A barrier of its
      // own: a commit on tfull[] here could complete a phase the epilogue has
      // not waited for yet and make its parity wait ambiguous.
      mma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr, kWaitNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int sub = warp & 3;
    const int rit = sub * 32 + lane;  // row inside the tile = TMEM lane
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      int g, nt, row0, mv;
      decode_tile(t, prefix, roff, G, g, nt, row0, mv);
      const bool got = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, got)) {  // warp-uniform: tcgen05.ld needs the whole warp
        raise_abort(abort_flag, p.err, ERR_GEMM_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + acc * BN;
      const size_t orow = static_cast<size_t>(row0 + rit);
      const bool valid = rit < mv && in_bounds(orow < (size_t)p.rows, p.err);
      if (EPI == TC_EPI_SWIGLU_BF16) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.C) + orow * p.N + nt * BN_OUT;
#pragma unroll 1
        for (int c = 0; c < BN_OUT; c += 32) {
          uint32_t gr[32], ur[32];
          tmem_ld_32x32b_x32(tb + c, gr);
          tmem_ld_32x32b_x32(tb + BN_OUT + c, ur);
          tmem_wait_ld();
          if (valid) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float h0 = silu_f(__uint_as_float(gr[2 * j])) * __uint_as_float(ur[2 * j]);
              const float h1 =
                  silu_f(__uint_as_float(gr[2 * j + 1])) * __uint_as_float(ur[2 * j + 1]);
              w[j] = pack_bf16(h0, h1);
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              d4[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          }
        }
      } else if (EPI == TC_EPI_STORE_BF16) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.C) + orow * p.N + nt * BN_OUT;
#pragma unroll 1
        for (int c = 0; c < BN_OUT; c += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tb + c, r);
          tmem_wait_ld();
          if (valid) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              w[j] = pack_bf16(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              d4[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          }
        }
      } else {
        float* dst = static_cast<float*>(p.C) + orow * p.N + nt * BN_OUT;
#pragma unroll 1
        for (int c = 0; c < BN_OUT; c += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tb + c, r);
          tmem_wait_ld();
          if (valid) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              d4[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

// Shared with the other tcgen05 kernels: 128-byte swizzle.
moe_status make_tmap_2d_swz(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                            int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                            uint32_t box_outer, CUtensorMapSwizzle swz);
moe_status make_tmap_2d(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                        int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer) {
  return make_tmap_2d_swz(tm, base, dtype, elem_bytes, inner, outer, box_inner, box_outer,
                          CU_TENSOR_MAP_SWIZZLE_128B);
}

moe_status make_tmap_2d_swz(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                            int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                            uint32_t box_outer, CUtensorMapSwizzle swz) {
  static EncodeTiledFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled not available");
    encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0)
    return fail(MOE_ERR_INVALID_ARG, "TMA operand base %p is not 16-byte aligned", base);
  if ((inner * elem_bytes) % 16 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "TMA row pitch %llu bytes is not a multiple of 16",
                (unsigned long long)(inner * elem_bytes));
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * elem_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(tm, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOE_OK;
}

// A row-major [rows, cols] matrix seen as blocks of `bc` columns: dimensions
// (bc columns, rows, cols/bc blocks) with strides (row pitch, bc * elem bytes),
// so that one box of (bc, box_rows, box_blocks) lands in shared memory as
// box_blocks consecutive [box_rows][bc] tiles (128-byte swizzle, bc * elem = 128).
moe_status make_tmap_col_blocks(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                                int elem_bytes, uint64_t cols, uint64_t rows, uint32_t bc,
                                uint32_t box_rows, uint32_t box_blocks) {
  static EncodeTiledFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled not available");
    encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0)
    return fail(MOE_ERR_INVALID_ARG, "TMA operand base %p is not 16-byte aligned", base);
  if ((cols * elem_bytes) % 16 != 0 || cols % bc != 0)
    return fail(MOE_ERR_UNSUPPORTED, "TMA column blocks: %llu columns",
                (unsigned long long)cols);
  cuuint64_t dims[3] = {bc, rows, cols / bc};
  cuuint64_t strides[2] = {cols * elem_bytes, (cuuint64_t)bc * elem_bytes};
  cuuint32_t box[3] = {bc, box_rows, box_blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(tm, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (column blocks) failed (%d)", (int)r);
  return MOE_OK;
}

namespace {

template <int BN, int EPI, int STAGES>
moe_status tc_launch(const void* A, const void* B, int b_rows_per_group, const int32_t* offsets,
                     int n_groups, int rows, int N, int K, void* C, cudaStream_t s) {
  using L = Layout<BN, STAGES>;
  constexpr int BN_OUT = (EPI == TC_EPI_SWIGLU_BF16) ? BN / 2 : BN;
  CUtensorMap tmA, tmB;
  moe_status st = make_tmap_2d(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, rows, BK, BM);
  if (st != MOE_OK) return st;
  const int G = offsets ? n_groups : 1;
  st = make_tmap_2d(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K,
                    (uint64_t)G * b_rows_per_group, BK, BN_OUT);
  if (st != MOE_OK) return st;
  auto kern = tc_gemm_kernel<BN, EPI, STAGES>;
  static bool attr_done[kMaxSmemDevices] = {};   // per instantiation and device
  {
    const moe_status sst = ensure_max_smem(reinterpret_cast<const void*>(kern), L::ALLOC,
                                           attr_done, "tc_gemm smem attribute");
    if (sst != MOE_OK) return sst;
  }
  TcParams p;
  p.offsets = offsets;
  p.n_groups = n_groups;
  p.rows = rows;
  p.N = N;
  p.K = K;
  p.b_rows_per_group = b_rows_per_group;
  p.half_b = (EPI == TC_EPI_SWIGLU_BF16) ? b_rows_per_group / 2 : 0;
  p.C = C;
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  const long long max_tiles =
      ((long long)(rows + BM - 1) / BM + (offsets ? G : 0)) * (N / BN_OUT);
  int grid = sm_count();
  if (max_tiles < grid) grid = (int)(max_tiles > 0 ? max_tiles : 1);
  kern<<<grid, kThreads, L::ALLOC, s>>>(tmA, tmB, p);
  return cuda_check(cudaGetLastError(), "tc_gemm launch");
}

}  // namespace

moe_status launch_tc_gemm(const void* A, const void* B, int b_rows_per_group,
                          const int32_t* offsets, int n_groups, int rows, int N, int K,
                          TcEpilogue epi, void* C, cudaStream_t s) {
  if (rows <= 0) return MOE_OK;
  if (K % BK != 0) return fail(MOE_ERR_UNSUPPORTED, "tc gemm: K=%d not a multiple of %d", K, BK);
  if (offsets && n_groups > kMaxGroups)
    return fail(MOE_ERR_UNSUPPORTED, "tc gemm: at most %d groups", kMaxGroups);
  switch (epi) {
    case TC_EPI_SWIGLU_BF16:
      if (N % 128) return fail(MOE_ERR_UNSUPPORTED, "tc gemm swiglu: N=%d %% 128", N);
      return tc_launch<256, TC_EPI_SWIGLU_BF16, 4>(A, B, b_rows_per_group, offsets, n_groups,
                                                    rows, N, K, C, s);
    case TC_EPI_STORE_BF16:
      if (N % 256 == 0)
        return tc_launch<256, TC_EPI_STORE_BF16, 4>(A, B, b_rows_per_group, offsets, n_groups,
                                                     rows, N, K, C, s);
      if (N % 128 == 0)
        return tc_launch<128, TC_EPI_STORE_BF16, 6>(A, B, b_rows_per_group, offsets, n_groups,
                                                     rows, N, K, C, s);
      return fail(MOE_ERR_UNSUPPORTED, "tc gemm store: N=%d %% 128", N);
    case TC_EPI_STORE_F32: {
      // Router logits: one group of `rows` tokens.  Take narrower N tiles
      // while the wide ones would leave a quarter of the SMs idle.
      const long long m_tiles = (rows + BM - 1) / BM;
      const long long busy = (3LL * sm_count()) / 4;
      int bn = (N % 256 == 0) ? 256 : (N % 128 == 0) ? 128 : 64;
      while (bn > 64 && N % (bn / 2) == 0 && m_tiles * (N / bn) < busy) bn /= 2;
      if (N % bn) return fail(MOE_ERR_UNSUPPORTED, "tc gemm f32: N=%d %% 64", N);
      if (bn == 256)
        return tc_launch<256, TC_EPI_STORE_F32, 4>(A, B, b_rows_per_group, offsets, n_groups,
                                                    rows, N, K, C, s);
      if (bn == 128)
        return tc_launch<128, TC_EPI_STORE_F32, 6>(A, B, b_rows_per_group, offsets, n_groups,
                                                    rows, N, K, C, s);
      return tc_launch<64, TC_EPI_STORE_F32, 8>(A, B, b_rows_per_group, offsets, n_groups, rows,
                                                 N, K, C, s);
    }
  }
  return fail(MOE_ERR_INVALID_ARG, "tc gemm: bad epilogue");
}

}  // namespace moe
