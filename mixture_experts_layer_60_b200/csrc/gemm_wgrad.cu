// Grouped weight-gradient GEMM on tcgen05 (the Wgrad pass that "DeepSeek V3 &
// R1 論文研究", section FP8 mixed precision, names beside Fprop and Dgrad):
// for every expert g with token rows [off_g, off_g+1),
//   C_g[m, n] = sum over those rows r of A[r, m] * B[r, n]
// A [rows, M] and B [rows, N] are row-major activations, so both MMA operands
// are MN-major (the contraction runs over rows).  dW_down = dy^T h and
// dW_gate_up = dA^T x are the two uses.
//
// Tile: 128 rows of C (one M=128 MMA) x 256 columns (N=256), 64 token rows per
// K step, 4 shared-memory stages of 48 KB (A: two [64 tok][64 m] TMA boxes,
// B: four [64 tok][64 n] boxes, 128-byte swizzle), two TMEM accumulators of
// 256 columns so the epilogue of one tile overlaps the MMAs of the next.
// The last K step of a group is ragged: its A rows come from a side buffer
// of per-group tail blocks written beforehand by launch_wgrad_tails (rows
// past the group's end are zero there, so the next expert's tokens never
// enter), and only ceil(valid/16) MMAs are issued.  A group with no tokens
// gets C_g = 0 from the epilogue without touching TMEM.
//
// Roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps 2-17
// epilogue (warp w
// reads TMEM lanes 32*(w%4).. = C rows and one 64-column quarter of the
// tile; each 32x32 block is converted to bf16 into a 2 KB shared-memory
// patch laid out as a 64-byte-swizzled [32 rows][32 cols] TMA box and written
// to global memory by one TMA store).  Every wait
// is bounded (1 s) and reported through the device error word.
#include "launch.h"
#include "sm100.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;              // token rows per stage
constexpr int STAGES = 4;
constexpr int kEpiWarps = 16;       // 4 per TMEM lane quarter, 64 columns each
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t TMEM_COLS = 512;

constexpr int BOX_BYTES = 64 * BK * 2;         // one [64 tok][64 mn] bf16 box: 8 KB
constexpr int A_BYTES = 2 * BOX_BYTES;         // 16 KB
constexpr int B_BYTES = 4 * BOX_BYTES;         // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int OFF_PATCH = STAGES * STAGE_BYTES;        // one 2 KB transpose patch per epilogue warp
constexpr int OFF_BAR = OFF_PATCH + kEpiWarps * 2048;
constexpr int N_BARS = 2 * STAGES + 5;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

struct WgParams {
  const int32_t* offsets;   // [n_groups+1] or nullptr (one group of `rows`)
  int n_groups;
  int rows;
  int M, N;
  __nv_bfloat16* C;         // [G, M, N]
  int* err;
};

// Rows [r0, r0 + cnt) of group g, clamped into [0, rows) (ERR_BAD_OFFSETS on a clamp).
__device__ __forceinline__ void group_rows(const WgParams& p, int g, int& r0, int& cnt) {
  int r1;
  clamp_group_rows(p.offsets, g, p.rows, p.err, r0, r1);
  cnt = r1 - r0;
}

__device__ __forceinline__ void raise_abort(volatile int* abort, int* err) {
  *abort = 1;
  atomicOr(err, ERR_GEMM_TIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 1)
    wgrad_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmC,
                      const __grid_constant__ CUtensorMap tmAt, const WgParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;      // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.offsets ? p.n_groups : 1;
  const int n_m = p.M / BM, n_n = p.N / BN;
  const int per_group = n_m * n_n;
  const int total = G * per_group;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], kEpiWarps); }
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int g = t / per_group, loc = t - g * per_group;
        const int mt = loc / n_n, nt = loc - mt * n_n;
        int r0, cnt;
        group_rows(p, g, r0, cnt);
        const int nkb = (cnt + BK - 1) / BK;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          uint8_t* a_dst = smem + stage * STAGE_BYTES;
          uint8_t* b_dst = a_dst + A_BYTES;
          const int row = r0 + kb * BK;
          // one TMA per operand: 2 (A) / 4 (B) consecutive [64 tok][64 col] tiles;
          // a group's last block of A comes from its zero-padded tail block
          if (kb == nkb - 1)
            tma_load_3d(a_dst, &tmAt, 0, g * BK, mt * (BM / 64), &full[stage]);
          else
            tma_load_3d(a_dst, &tmA, 0, row, mt * (BM / 64), &full[stage]);
          tma_load_3d(b_dst, &tmB, 0, row, nt * (BN / 64), &full[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      for (int s = 0; s < STAGES; ++s)
        mbar_wait_bounded(&full[s], ((s < stage) ? phase : phase ^ 1), nullptr, kWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0, used = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16_f32_major(BM, BN, true, true);
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int g = t / per_group;
        int r0, cnt;
        group_rows(p, g, r0, cnt);
        if (cnt <= 0) continue;
        const int ab = used & 1;
        const uint32_t tpar = ((used >> 1) & 1) ^ 1;
        ++used;
        if (!mbar_wait_bounded(&tempty[ab], tpar, abort_flag, kWaitNs)) {
          raise_abort(abort_flag, p.err);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * BN;
        const int nkb = (cnt + BK - 1) / BK;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          tc_fence_after();
          const int valid = min(BK, cnt - kb * BK);
          const int nks = (valid + 15) / 16;
          const uint32_t a0 = smem_u32(smem + stage * STAGE_BYTES), b0 = a0 + A_BYTES;
          for (int k = 0; k < nks; ++k)
            mma_f16_ss(d_tmem, smem_desc_mn_sw128(a0 + k * 2048, BOX_BYTES),
                       smem_desc_mn_sw128(b0 + k * 2048, BOX_BYTES), idesc, (kb | k) != 0);
          mma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        mma_commit(&tfull[ab]);
      }
      mma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr, kWaitNs);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                       // TMEM lane quarter = C rows q*32..
    const int cq = (warp - 2) >> 2;               // 64-column quarter of the tile
    uint4* patch = reinterpret_cast<uint4*>(smem + OFF_PATCH + (warp - 2) * 2048);   // [32][4]
    int used = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const int g = t / per_group, loc = t - g * per_group;
      const int mt = loc / n_n, nt = loc - mt * n_n;
      int r0, cnt;
      group_rows(p, g, r0, cnt);
      const int m = mt * BM + q * 32 + lane;
      __nv_bfloat16* dst_row = p.C + ((size_t)g * p.M + m) * p.N + nt * BN + cq * 64;
      if (cnt <= 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          reinterpret_cast<uint4*>(dst_row)[i] = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      const int ab = used & 1;
      const uint32_t tpar = (used >> 1) & 1;
      ++used;
      const bool got = mbar_wait_bounded(&tfull[ab], tpar, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) raise_abort(abort_flag, p.err);
        break;
      }
      tc_fence_after();
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * BN + cq * 64;
      uint32_t r[2][32];
      tmem_ld_32x32b_x32(tl, r[0]);
      tmem_ld_32x32b_x32(tl + 32, r[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);   // accumulator read: the next tile's MMAs may start
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        // the previous TMA store must have read the patch before it is rewritten
        if (lane == 0) tma_store_wait_read_all();
        __syncwarp();
        // row `lane` (64 bytes) into the patch, 64-byte swizzle: 16-byte slot i
        // of row r sits at i ^ ((r >> 1) & 3) (also spreads 8 lanes over 8 bank groups)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t w4[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(r[c][8 * i + 2 * k]),
                                                      __uint_as_float(r[c][8 * i + 2 * k + 1]));
            w4[k] = *reinterpret_cast<uint32_t*>(&pr);
          }
          patch[lane * 4 + (i ^ ((lane >> 1) & 3))] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmC, patch, nt * BN + cq * 64 + c * 32, g * p.M + mt * BM + q * 32);
          tma_store_commit();
        }
      }
    }
  }

  if (warp >= 2 && lane == 0) tma_store_wait_all();   // stores done before the CTA exits
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

moe_status make_tmap_2d(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                        int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer);
moe_status make_tmap_2d_swz(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                            int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                            uint32_t box_outer, CUtensorMapSwizzle swz);
moe_status make_tmap_col_blocks(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                                int elem_bytes, uint64_t cols, uint64_t rows, uint32_t bc,
                                uint32_t box_rows, uint32_t box_blocks);

namespace {

// T[g][i] = row (start of g's last block) + i of A if it lies inside group g, else 0.
__global__ void __launch_bounds__(256) wgrad_tails_kernel(const uint4* __restrict__ A,
                                                          int row_vec, int block_rows,
                                                          const int32_t* __restrict__ offsets,
                                                          int rows, uint4* __restrict__ T) {
  const int g = blockIdx.x, i = blockIdx.y;
  int r0, r1;
  clamp_group_rows(offsets, g, rows, nullptr, r0, r1);   // the GEMM reports a clamp
  const int cnt = r1 - r0;
  if (cnt <= 0) return;
  const int row = r0 + ((cnt - 1) / block_rows) * block_rows + i;
  uint4* dst = T + ((size_t)g * block_rows + i) * row_vec;
  if (row < r1) {
    const uint4* src = A + (size_t)row * row_vec;
    for (int c = threadIdx.x; c < row_vec; c += blockDim.x) dst[c] = src[c];
  } else {
    for (int c = threadIdx.x; c < row_vec; c += blockDim.x) dst[c] = make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace

moe_status launch_wgrad_tails(const void* A, size_t row_bytes, int block_rows,
                              const int32_t* offsets, int n_groups, int rows, void* T,
                              cudaStream_t s) {
  const int G = offsets ? n_groups : 1;
  if (G <= 0 || rows <= 0) return MOE_OK;
  dim3 grid(G, block_rows);
  wgrad_tails_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(A), (int)(row_bytes / 16),
                                          block_rows, offsets, rows, static_cast<uint4*>(T));
  return cuda_check(cudaGetLastError(), "wgrad tails launch");
}

size_t wgrad_tail_bytes(size_t row_bytes, int block_rows, int n_groups) {
  return align_up((size_t)n_groups * block_rows * row_bytes, 256);
}

moe_status launch_wgrad_gemm(const void* A, int M, const void* B, int N, const int32_t* offsets,
                             int n_groups, int rows, void* A_tail, void* C, cudaStream_t s) {
  const int G = offsets ? n_groups : 1;
  if (G <= 0) return MOE_OK;
  if (M % BM || N % BN)
    return fail(MOE_ERR_UNSUPPORTED, "wgrad gemm: M=%d must be a multiple of %d, N=%d of %d", M,
                BM, N, BN);
  if (rows <= 0) {
    // every group is empty: C = 0
    return cuda_check(cudaMemsetAsync(C, 0, (size_t)G * M * N * 2, s), "wgrad zero fill");
  }
  // the A operand's tail blocks: [G * BK rows][M] (launch_wgrad_tails)
  moe_status st = launch_wgrad_tails(A, (size_t)M * 2, BK, offsets, G, rows, A_tail, s);
  if (st != MOE_OK) return st;
  CUtensorMap tmA, tmB, tmC, tmAt;
  st = make_tmap_col_blocks(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, rows, 64, BK, BM / 64);
  if (st != MOE_OK) return st;
  st = make_tmap_col_blocks(&tmAt, A_tail, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M,
                            (uint64_t)G * BK, 64, BK, BM / 64);
  if (st != MOE_OK) return st;
  st = make_tmap_col_blocks(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, rows, 64, BK, BN / 64);
  if (st != MOE_OK) return st;
  // output: [G*M rows][N cols], stored in [32 rows][32 cols] boxes with 64-byte swizzle
  st = make_tmap_2d_swz(&tmC, C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, (uint64_t)G * M, 32, 32,
                        CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != MOE_OK) return st;
  static bool attr_done[kMaxSmemDevices] = {};   // per instantiation and device
  {
    const moe_status sst = ensure_max_smem(reinterpret_cast<const void*>(wgrad_gemm_kernel), SMEM_ALLOC,
                                           attr_done, "wgrad smem attribute");
    if (sst != MOE_OK) return sst;
  }
  WgParams p;
  p.offsets = offsets;
  p.n_groups = G;
  p.rows = rows;
  p.M = M;
  p.N = N;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  const long long tiles = (long long)G * (M / BM) * (N / BN);
  int grid = sm_count();
  if (tiles < grid) grid = (int)tiles;
  wgrad_gemm_kernel<<<grid, kThreads, SMEM_ALLOC, s>>>(tmA, tmB, tmC, tmAt, p);
  return cuda_check(cudaGetLastError(), "wgrad gemm launch");
}

}  // namespace moe
