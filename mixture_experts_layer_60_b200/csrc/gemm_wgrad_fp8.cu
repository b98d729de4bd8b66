// FP8 weight-gradient GEMM (the Wgrad pass under the FP8 recipe of
// "DeepSeek-V3 技術報告", section 核心概念: E4M3 operands, 1x128 activation
// tiles, FP32 promotion every N_c = 128).  The contraction runs over an
// expert's tokens, so an activation tile is 128 consecutive rows of one
// expert (blocks start at the expert's first row) x 1 column:
//   C_g[m, n] = sum over g's blocks b of
//               (sum_{r in b} qa[r, m] qb[r, n]) * sa[b, m] * sb[b, n]
// qa [rows, M], qb [rows, N] e4m3 row-major (both MMA operands MN-major);
// sa [blocks, M], sb [blocks, N] float32; C [G, M, N] bf16.
//
// Tile 128 x 256 outputs; each shared-memory stage is one 128-row block
// (A: one [128 tok][128 m] box, B: two [128 tok][128 n] boxes, 128-byte
// swizzle, 48 KB), 4 stages; with every stage the producer also copies the
// block's scales sa[b, m0:m0+128] and sb[b, n0:n0+256] into a ring of 6
// scale slots (bulk copies on their own barriers).  The MMA warp writes each
// block's partial product into one of two TMEM buffers (tcgen05.mma
// kind::f8f6f4, K = 32 per instruction; the A rows of an expert's ragged last
// block come from its zero-padded tail block, and only ceil(valid/32) MMAs are
// issued); 16 epilogue warps read it back (warp w: TMEM lanes
// 32*(w%4).. = C rows, 64 columns), add P * (sa * sb) into float32 registers
// with paired multiplies and FMAs, and after the expert's last block write
// bf16 rows to global memory.  Waits are bounded (1 s).
#include "launch.h"
#include "sm100.cuh"

namespace moe {

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

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;             // token rows per stage = one promotion block
constexpr int STAGES = 4;
constexpr int kEpiWarps = 16;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t TMEM_COLS = 512;

constexpr int BOX_BYTES = 128 * BK;            // [128 tok][128 e4m3]: 16 KB
constexpr int A_BYTES = BOX_BYTES;
constexpr int B_BYTES = 2 * BOX_BYTES;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SSLOTS = 6;                       // scale ring: sa [128] + sb [256] float32 per block
constexpr int SLOT_BYTES = (BM + BN) * 4;
constexpr int OFF_SCALE = STAGES * STAGE_BYTES;
constexpr int OFF_BAR = OFF_SCALE + SSLOTS * SLOT_BYTES;
constexpr int N_BARS = 2 * STAGES + 5 + 2 * SSLOTS;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

struct Wg8Params {
  const int32_t* offsets;
  int n_groups;
  int rows;
  int M, N;
  const float* sa;            // [blocks, M]
  const float* sb;            // [blocks, N]
  const int32_t* block_start; // [G+1]
  __nv_bfloat16* Cp;          // [G, M, N]
  int* err;
  __device__ __nv_bfloat16* C(int g, int m, int n) const {
    return Cp + ((size_t)g * M + m) * N + n;
  }
};

// Rows [r0, r0 + cnt) of group g, clamped into [0, rows) (ERR_BAD_OFFSETS on a clamp).
__device__ __forceinline__ void group_rows(const Wg8Params& p, int g, int& r0, int& cnt) {
  int r1;
  clamp_group_rows(p.offsets, g, p.rows, p.err, r0, r1);
  cnt = r1 - r0;
}

__device__ __forceinline__ void raise_abort(volatile int* abort, int* err) {
  *abort = 1;
  atomicOr(err, ERR_GEMM_FP8_TIMEOUT);
}

__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint64_t lds_b64(uint32_t a) {
  uint64_t v;
  asm volatile("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(a));
  return v;
}
// (a0, a1) * (b0, b1), elementwise, rounded like two fmul
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// c += (x0, x1) * s2 with x0, x1 the raw bits of two float32 TMEM words
__device__ __forceinline__ uint64_t fma2_bits(uint32_t x0, uint32_t x1, uint64_t s2, uint64_t c) {
  asm("{\n\t.reg .b64 t;\n\tmov.b64 t, {%1, %2};\n\tfma.rn.f32x2 %0, t, %3, %0;\n\t}"
      : "+l"(c)
      : "r"(x0), "r"(x1), "l"(s2));
  return c;
}

// 18 warps put 5 on two of the SM's four sub-partitions, whose 16K-register
// files then cap a thread at 96 registers (__launch_bounds__ below).
__global__ void __launch_bounds__(kThreads, 1)
    wgrad_fp8_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmAt, const Wg8Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* pfull = empty + STAGES;      // [2] partial product ready
  uint64_t* pempty = pfull + 2;          // [2] partial product read by the epilogue
  uint64_t* mma_done = pempty + 2;
  uint64_t* sfull = mma_done + 1;        // [SSLOTS] scales landed
  uint64_t* sempty = sfull + SSLOTS;     // [SSLOTS] scales read by the epilogue
  float* scales = reinterpret_cast<float*>(smem + OFF_SCALE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.offsets ? p.n_groups : 1;
  const int n_m = p.M / BM, n_n = p.N / BN;
  const int per_group = n_m * n_n;
  const int total = G * per_group;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&pfull[b], 1); mbar_init(&pempty[b], kEpiWarps); }
    mbar_init(mma_done, 1);
    for (int i = 0; i < SSLOTS; ++i) { mbar_init(&sfull[i], 1); mbar_init(&sempty[i], kEpiWarps); }
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
      int stage = 0, ss = 0;
      uint32_t phase = 0, sphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int g = t / per_group, loc = t - g * per_group;
        const int mt = loc / n_n, nt = loc - mt * n_n;
        int r0, cnt;
        group_rows(p, g, r0, cnt);
        const int nkb = (cnt + BK - 1) / BK;
        const int blk0 = nkb > 0 ? p.block_start[g] : 0;
        for (int kb = 0; kb < nkb; ++kb) {
          // this block's scales into the next slot of the ring
          if (!mbar_wait_bounded(&sempty[ss], sphase ^ 1, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sfull[ss], SLOT_BYTES);
          float* sl = scales + ss * (BM + BN);
          bulk_load(sl, p.sa + (size_t)(blk0 + kb) * p.M + mt * BM, BM * 4, &sfull[ss]);
          bulk_load(sl + BM, p.sb + (size_t)(blk0 + kb) * p.N + nt * BN, BN * 4, &sfull[ss]);
          if (++ss == SSLOTS) { ss = 0; sphase ^= 1; }
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          uint8_t* a_dst = smem + stage * STAGE_BYTES;
          const int row = r0 + kb * BK;
          if (kb == nkb - 1)   // the expert's last block of A: its zero-padded tail block
            tma_load_2d(a_dst, &tmAt, mt * BM, g * BK, &full[stage]);
          else
            tma_load_2d(a_dst, &tmA, mt * BM, row, &full[stage]);
          tma_load_3d(a_dst + A_BYTES, &tmB, 0, row, nt * (BN / 128), &full[stage]);   // 2 tiles
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      for (int s = 0; s < STAGES; ++s)
        mbar_wait_bounded(&full[s], ((s < stage) ? phase : phase ^ 1), nullptr, kWaitNs);
      for (int i = 0; i < SSLOTS; ++i)
        mbar_wait_bounded(&sfull[i], ((i < ss) ? sphase : sphase ^ 1), nullptr, kWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0, pb = 0;
      uint32_t phase = 0, pphase = 0;
      bool ok = true;
      const uint32_t idesc = idesc_e4m3_f32(BM, BN) | (1u << 15) | (1u << 16);   // A, B MN-major
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int g = t / per_group;
        int r0, cnt;
        group_rows(p, g, r0, cnt);
        const int nkb = (cnt + BK - 1) / BK;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&pempty[pb], pphase ^ 1, abort_flag, kWaitNs) ||
              !mbar_wait_bounded(&full[stage], phase, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          tc_fence_after();
          const int valid = min(BK, cnt - kb * BK);
          const int nks = (valid + 31) / 32;
          const uint32_t a0 = smem_u32(smem + stage * STAGE_BYTES), b0 = a0 + A_BYTES;
          const uint32_t d_tmem = tmem_base + pb * BN;
          for (int k = 0; k < nks; ++k)
            mma_f8_ss(d_tmem, smem_desc_mn_sw128(a0 + k * 4096, BOX_BYTES),
                      smem_desc_mn_sw128(b0 + k * 4096, BOX_BYTES), idesc, k != 0);
          mma_commit(&empty[stage]);
          mma_commit(&pfull[pb]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
          if (++pb == 2) { pb = 0; pphase ^= 1; }
        }
      }
      mma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr, kWaitNs);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                       // TMEM lane quarter = C rows q*32..
    const int cq = (warp - 2) >> 2;               // 64-column quarter of the tile
    int pb = 0, ss = 0;
    uint32_t pphase = 0, sphase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int g = t / per_group, loc = t - g * per_group;
      const int mt = loc / n_n, nt = loc - mt * n_n;
      int r0, cnt;
      group_rows(p, g, r0, cnt);
      if (cnt <= 0) {
        uint4* dst = reinterpret_cast<uint4*>(p.C(g, mt * BM + q * 32 + lane, nt * BN + cq * 64));
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      uint64_t acc2[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc2[i] = 0ull;
      const int nkb = (cnt + BK - 1) / BK;
      for (int kb = 0; kb < nkb; ++kb) {
        const bool gs = mbar_wait_bounded(&sfull[ss], sphase, abort_flag, kWaitNs);
        const bool got = gs && mbar_wait_bounded(&pfull[pb], pphase, abort_flag, kWaitNs);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) raise_abort(abort_flag, p.err);
          ok = false;
          break;
        }
        tc_fence_after();
        // 32-bit shared addresses keep the hot loop's register count down
        const uint32_t sl = smem_u32(scales) + ss * (BM + BN) * 4;
        const float sa = lds_f32(sl + (q * 32 + lane) * 4);
        const uint64_t sa2 = f2_pack(sa, sa);
        const uint32_t sb = sl + (BM + cq * 64) * 4;                           // column pairs
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + pb * BN + cq * 64;
        // eight 8-column pieces
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t r[8];
          tmem_ld_32x32b_x8(tb + c * 8, r);
          tmem_wait_ld();
          if (c == 7) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[pb]);   // partial read: the MMA may overwrite it
          }
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint64_t s2 = mul2(sa2, lds_b64(sb + (c * 8 + 2 * v) * 4));   // broadcast read
            acc2[c * 4 + v] = fma2_bits(r[2 * v], r[2 * v + 1], s2, acc2[c * 4 + v]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[ss]);   // this block's scales are no longer read
        if (++pb == 2) { pb = 0; pphase ^= 1; }
        if (++ss == SSLOTS) { ss = 0; sphase ^= 1; }
      }
      if (!ok) break;
      uint4* dst = reinterpret_cast<uint4*>(p.C(g, mt * BM + q * 32 + lane, nt * BN + cq * 64));
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t w4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float x0, x1;
          f2_unpack(acc2[4 * i + k], x0, x1);
          __nv_bfloat162 pr = __floats2bfloat162_rn(x0, x1);
          w4[k] = *reinterpret_cast<uint32_t*>(&pr);
        }
        dst[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

moe_status launch_wgrad_tails(const void* A, size_t row_bytes, int block_rows,
                              const int32_t* offsets, int n_groups, int rows, void* T,
                              cudaStream_t s);

moe_status launch_wgrad_fp8(const void* qa, const float* sa, int M, const void* qb,
                            const float* sb, int N, const int32_t* offsets, int n_groups,
                            int rows, const int32_t* block_start, void* qa_tail, void* C,
                            cudaStream_t s) {
  const int G = offsets ? n_groups : 1;
  if (G <= 0) return MOE_OK;
  if (M % BM || N % BN)
    return fail(MOE_ERR_UNSUPPORTED, "fp8 wgrad: M=%d must be a multiple of %d, N=%d of %d", M,
                BM, N, BN);
  if (rows <= 0)
    return cuda_check(cudaMemsetAsync(C, 0, (size_t)G * M * N * 2, s), "fp8 wgrad zero fill");
  moe_status st = launch_wgrad_tails(qa, (size_t)M, BK, offsets, G, rows, qa_tail, s);
  if (st != MOE_OK) return st;
  CUtensorMap tmA, tmB, tmAt;
  st = make_tmap_2d(&tmA, qa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, rows, 128, BK);
  if (st != MOE_OK) return st;
  st = make_tmap_2d(&tmAt, qa_tail, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, (uint64_t)G * BK, 128, BK);
  if (st != MOE_OK) return st;
  st = make_tmap_col_blocks(&tmB, qb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, rows, 128, BK, BN / 128);
  if (st != MOE_OK) return st;
  static bool attr_done[kMaxSmemDevices] = {};   // per instantiation and device
  {
    const moe_status sst = ensure_max_smem(reinterpret_cast<const void*>(wgrad_fp8_kernel), SMEM_ALLOC,
                                           attr_done, "fp8 wgrad smem attribute");
    if (sst != MOE_OK) return sst;
  }
  Wg8Params p;
  p.offsets = offsets;
  p.n_groups = G;
  p.rows = rows;
  p.M = M;
  p.N = N;
  p.sa = sa;
  p.sb = sb;
  p.block_start = block_start;
  p.Cp = static_cast<__nv_bfloat16*>(C);
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  const long long tiles = (long long)G * (M / BM) * (N / BN);
  int grid = sm_count();
  if (tiles < grid) grid = (int)tiles;
  wgrad_fp8_kernel<<<grid, kThreads, SMEM_ALLOC, s>>>(tmA, tmB, tmAt, p);
  return cuda_check(cudaGetLastError(), "fp8 wgrad launch");
}

}  // namespace moe
