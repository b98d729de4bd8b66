// FP8 grouped GEMM with fine-grained scales and FP32 promotion every 128
// K-elements: the FP8 recipe of "DeepSeek-V3 技術報告", section 核心概念
// (E4M3 operands, 1x128 activation-tile scales, 128x128 weight-block scales,
// N_c = 128), applied to the expert FFNs of the h'-equation (section 方法 / 2).
//
//   acc[r, n] = sum_kb  P_kb[r, n] * sa[r, kb] * sw[g, n / 128, kb]
//   P_kb[r, n] = sum_{k in kb} qa[r, k] qw[g*b_rows + n, k]      (tensor cores)
//
// Each 128-wide K block is one shared-memory stage (128 bytes per row, the
// 128-byte swizzle width).  The MMA warp writes P_kb into one of two TMEM
// partial buffers (4 x tcgen05.mma kind::f8f6f4, K = 32 each); two epilogue
// warpgroups read it back with tcgen05.ld, multiply by the two scales and add
// into float32 registers (4 warpgroups, 64 columns each), then release the
// buffer.  After the last block:
//   SWIGLU   h = SiLU(acc_gate) * acc_up (float32), quantised 1x128 to E4M3
//            with scale amax/448 (the 128 columns of a row span the four
//            warpgroups: their amax meet in shared memory)
//   STORE    y = bf16(acc)
//   SWIGLU_SAVE  SWIGLU that also writes the float32 gate and up values as
//            bf16 pre-activations S [rows, 2I] for the backward
//   DSWIGLU  the Dgrad of the down projection fused with the SwiGLU backward:
//            dh = acc; a, b = S[:, 0:I], S[:, I:2I] (bf16);
//            dA = [dh * b * SiLU'(a) | dh * SiLU(a)] written as bf16 (C2) and
//            quantised 1x128 to E4M3 (C, c_scale); a 128-column tile spans two
//            warpgroups, whose amax meet in shared memory
// B_MN: the weight is stored [K rows][N cols] (a Dgrad reads W_down [d, I]
// and W_gate_up [2I, d] as they are); its 128x128 block scales are then
// indexed [K/128][N/128], and the MMA reads B as an MN-major operand.
// Warp roles: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2-17 epilogue
// (warpgroup w = warps 2+4w .. 5+4w).  Waits are bounded.
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace moe {

moe_status make_tmap_2d(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                        int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer);
moe_status make_tmap_col_blocks(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                                int elem_bytes, uint64_t cols, uint64_t rows, uint32_t bc,
                                uint32_t box_rows, uint32_t box_blocks);

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 256;               // MMA N: SWIGLU = 128 gate + 128 up columns
constexpr int BK = 128;               // e4m3 bytes per row = one promotion block
constexpr int STAGES = 4;
constexpr int kEpiWG = 4;             // epilogue warpgroups; each owns BN / kEpiWG columns
constexpr int kThreads = 64 + 128 * kEpiWG;
constexpr int kMaxGroups = 1024;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t TMEM_COLS = 512;   // two partial buffers of BN columns

constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int OFF_B = STAGES * A_BYTES;
constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
constexpr int N_BARS = 2 * STAGES + 7;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int OFF_AMAX = OFF_MISC + 16;                 // [2 slots][2][kEpiWG][BM] float
// STORE: [32 rows][16 cols] bf16 per warp, read and written as 16-byte vectors
constexpr int OFF_PATCH = (OFF_AMAX + 2 * 2 * kEpiWG * BM * 4 + 127) / 128 * 128;
static_assert(OFF_PATCH % 16 == 0, "16-byte vectors");
constexpr int OFF_TAB = OFF_PATCH + 4 * kEpiWG * 1024;
constexpr int SMEM_BYTES = OFF_TAB + 2 * (kMaxGroups + 1) * 4;
static_assert(SMEM_BYTES + 1024 <= 227 * 1024, "shared memory");
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

struct Fp8Params {
  const int32_t* offsets;
  int n_groups;
  int rows;
  int N;                // output columns
  int K;
  int b_rows_per_group;
  int half_b;           // SWIGLU: I
  const float* a_scale; // [rows, K/128]
  const float* b_scale; // [G, b_rows/128, K/128] (B_MN: [G, K/128, N/128])
  void* C;              // SWIGLU: e4m3 [rows, N]; STORE: bf16 [rows, N]; DSWIGLU: e4m3 [rows, 2N]
  float* c_scale;       // SWIGLU: [rows, N/128]; DSWIGLU: [rows, 2N/128]
  __nv_bfloat16* S;     // SWIGLU_SAVE: pre-activations out; DSWIGLU: in ([rows, lds])
  int lds;
  __nv_bfloat16* C2;    // DSWIGLU: bf16 dA [rows, 2N]
  int* err;
};

template <int EPI>
struct Fp8Tile {
  static constexpr bool SW = EPI == F8_SWIGLU || EPI == F8_SWIGLU_SAVE;
  static constexpr int BN_OUT = SW ? BN / 2 : BN;
};

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

__device__ __forceinline__ void raise_abort(volatile int* abort, int* err) {
  *abort = 1;
  atomicOr(err, ERR_GEMM_FP8_TIMEOUT);
}

// Packed pair of float32 in one 64-bit register, and the sm_100 paired FMA
// (two IEEE fused multiply-adds per instruction, each rounded like fmaf).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
// c += (x0, x1) * s2, x0/x1 the raw bits of two float32 TMEM words
__device__ __forceinline__ uint64_t fma2_bits(uint32_t x0, uint32_t x1, uint64_t s2, uint64_t c) {
  asm("{\n\t.reg .b64 t;\n\tmov.b64 t, {%1, %2};\n\tfma.rn.f32x2 %0, t, %3, %0;\n\t}"
      : "+l"(c)
      : "r"(x0), "r"(x1), "l"(s2));
  return c;
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  return (uint32_t)__nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3) |
         ((uint32_t)__nv_cvt_float_to_fp8(b, __NV_SATFINITE, __NV_E4M3) << 8) |
         ((uint32_t)__nv_cvt_float_to_fp8(c, __NV_SATFINITE, __NV_E4M3) << 16) |
         ((uint32_t)__nv_cvt_float_to_fp8(d, __NV_SATFINITE, __NV_E4M3) << 24);
}

template <int EPI, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB, const Fp8Params p) {
  constexpr bool SWIGLU = Fp8Tile<EPI>::SW;
  constexpr int BN_OUT = Fp8Tile<EPI>::BN_OUT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + OFF_B;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* pfull = empty + STAGES;   // [2] partial ready
  uint64_t* pempty = pfull + 2;       // [2] partial consumed (256 arrivals)
  uint64_t* mma_done = pempty + 2;
  uint64_t* xbar = mma_done + 1;      // [2] amax exchange between the warpgroups (one arrival per warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  float* amax_x = reinterpret_cast<float*>(smem + OFF_AMAX);
  int* prefix = reinterpret_cast<int*>(smem + OFF_TAB);
  int* roff = prefix + kMaxGroups + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.offsets ? p.n_groups : 1;
  const int n_tiles_n = p.N / BN_OUT;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&pfull[a], 1); mbar_init(&pempty[a], 4 * kEpiWG); }   // one arrival per epilogue warp
    mbar_init(mma_done, 1);
    mbar_init(&xbar[0], 4 * kEpiWG);                 // one arrival per epilogue warp
    mbar_init(&xbar[1], 4 * kEpiWG);
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
    // tile table from offsets clamped into disjoint ranges of [0, rows)
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
    __syncwarp();
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
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          tma_load_2d(sA + stage * A_BYTES, &tmA, kb * BK, row0, &full[stage]);
          if (B_MN) {
            // [128 K rows][128 N cols] x 2 tiles of columns nt*256 .. in one 3D box
            tma_load_3d(sB + stage * B_BYTES, &tmB, 0, g * p.K + kb * BK, nt * (BN / 128),
                        &full[stage]);
          } else if (SWIGLU) {
            tma_load_2d(sB + stage * B_BYTES, &tmB, kb * BK, brow, &full[stage]);
            tma_load_2d(sB + stage * B_BYTES + B_BYTES / 2, &tmB, kb * BK, brow + p.half_b,
                        &full[stage]);
          } else {
            tma_load_2d(sB + stage * B_BYTES, &tmB, kb * BK, brow, &full[stage]);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      for (int s = 0; s < STAGES; ++s)
        mbar_wait_bounded(&full[s], ((s < stage) ? phase : phase ^ 1), nullptr, kWaitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN) | (B_MN ? (1u << 16) : 0u);
      int stage = 0, pb = 0;
      uint32_t phase = 0, pphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&pempty[pb], pphase ^ 1, abort_flag, kWaitNs) ||
              !mbar_wait_bounded(&full[stage], phase, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
          const uint32_t d_tmem = tmem_base + pb * BN;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_f8_ss(d_tmem, smem_desc_k_sw128(a0 + k * 32),
                      B_MN ? smem_desc_mn_sw128(b0 + k * 4096, B_BYTES / 2)
                           : smem_desc_k_sw128(b0 + k * 32),
                      idesc, k != 0);
          mma_commit(&empty[stage]);
          mma_commit(&pfull[pb]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
          if (++pb == 2) { pb = 0; pphase ^= 1; }
        }
      }
      mma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr, kWaitNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // kEpiWG warpgroups; warpgroup wg owns, for every row of the tile,
    //   SWIGLU: gate columns [wg*32, +32) and the matching up columns 128 + [wg*32, +32)
    //   STORE:  output columns [wg*64, +64)
    constexpr int CW = BN / kEpiWG;     // 64 accumulator columns per thread
    const int wg = (warp - 2) >> 2;
    const int sub = warp & 3;           // TMEM lane quarter of this warp
    const int rit = sub * 32 + lane;    // row inside the tile
    const int nkb_a = p.K / BK;
    int pb = 0;
    uint32_t pphase = 0;
    bool ok = true;
    int it = 0;  // tiles done by this CTA (amax exchange slot and phase)
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
      int g, nt, row0, mv;
      decode_tile(t, prefix, roff, G, g, nt, row0, mv);
      const bool valid = rit < mv && in_bounds(row0 + rit < p.rows, p.err);
      const int arow = valid ? row0 + rit : row0;   // clamp scale reads for padding rows
      const float* sa_row = p.a_scale + (size_t)arow * nkb_a;
      // weight N blocks per group; block scales [nbw][K/128], or [K/128][nbw] for B_MN
      const int nbw = B_MN ? p.N / 128 : p.b_rows_per_group / 128;
      const float* sw_g = p.b_scale + (size_t)g * nbw * nkb_a;
      // weight row blocks of this thread's two 32-column chunks
      int blk0, blk1;
      uint32_t col0, col1;
      if (SWIGLU) {
        blk0 = nt;                                   // gate rows nt*128 ..
        blk1 = (p.half_b / 128) + nt;                // up rows I + nt*128 ..
        col0 = wg * 32;
        col1 = 128 + wg * 32;
      } else {
        blk0 = blk1 = 2 * nt + (wg * CW) / 128;      // output columns nt*256 + wg*64 ..
        col0 = wg * CW;
        col1 = wg * CW + 32;
      }
      uint64_t acc2[CW / 2];   // accumulator pairs: columns (2i, 2i+1) of this thread's chunks
#pragma unroll
      for (int i = 0; i < CW / 2; ++i) acc2[i] = 0ull;
      float sa = sa_row[0];
      for (int kb = 0; kb < nk; ++kb) {
        const float sa_next = (kb + 1 < nk) ? sa_row[kb + 1] : 0.f;
        const float s0 = sa * (B_MN ? sw_g[(size_t)kb * nbw + blk0] : sw_g[(size_t)blk0 * nkb_a + kb]);
        const float s1 = sa * (B_MN ? sw_g[(size_t)kb * nbw + blk1] : sw_g[(size_t)blk1 * nkb_a + kb]);
        const bool got = mbar_wait_bounded(&pfull[pb], pphase, abort_flag, kWaitNs);
        if (!__all_sync(0xffffffffu, got)) {
          raise_abort(abort_flag, p.err);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + pb * BN;
        // Four 16-column pieces; many warps per sub-partition hide the load latency.
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(tb + (c < 2 ? col0 : col1) + (c & 1) * 16, r);
          tmem_wait_ld();
          if (c == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[pb]);   // partial read: the MMA may overwrite it
          }
          const uint64_t sc2 = c < 2 ? f2_pack(s0, s0) : f2_pack(s1, s1);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc2[c * 8 + i] = fma2_bits(r[2 * i], r[2 * i + 1], sc2, acc2[c * 8 + i]);
        }
        if (++pb == 2) { pb = 0; pphase ^= 1; }
        sa = sa_next;
      }
      if (!ok) break;
      float acc[CW];
#pragma unroll
      for (int i = 0; i < CW / 2; ++i) f2_unpack(acc2[i], acc[2 * i], acc[2 * i + 1]);
      if (EPI == F8_SWIGLU_SAVE && valid) {
        // gate / up pre-activations (float32 values rounded to bf16) for the backward
        __nv_bfloat16* sg = p.S + (size_t)(row0 + rit) * p.lds + nt * 128 + wg * 32;
        __nv_bfloat16* su = sg + p.half_b;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t wg4[4], wu4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 a2 = __floats2bfloat162_rn(acc[q4 * 8 + 2 * i], acc[q4 * 8 + 2 * i + 1]);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[32 + q4 * 8 + 2 * i], acc[32 + q4 * 8 + 2 * i + 1]);
            wg4[i] = *reinterpret_cast<uint32_t*>(&a2);
            wu4[i] = *reinterpret_cast<uint32_t*>(&b2);
          }
          reinterpret_cast<uint4*>(sg)[q4] = make_uint4(wg4[0], wg4[1], wg4[2], wg4[3]);
          reinterpret_cast<uint4*>(su)[q4] = make_uint4(wu4[0], wu4[1], wu4[2], wu4[3]);
        }
      }
      if (EPI == F8_DSWIGLU) {
        // acc = dh for columns c0 .. c0+63 of this row; a, b from the saved pre-activations
        const int I = p.N;
        const int c0 = nt * BN + wg * CW;
        const size_t row = (size_t)(valid ? row0 + rit : row0);
        const __nv_bfloat16* sa_p = p.S + row * p.lds + c0;
        const __nv_bfloat16* sb_p = sa_p + I;
        float ma = 0.f, mb = 0.f;
        // pass 1: dA in bf16, and the amax of this thread's 64 da and 64 db values
#pragma unroll
        for (int j8 = 0; j8 < CW / 8; ++j8) {
          float fa[8], fb[8], da[8], db[8];
          if (valid) {
            const uint4 av = reinterpret_cast<const uint4*>(sa_p)[j8];
            const uint4 bv = reinterpret_cast<const uint4*>(sb_p)[j8];
            Vec<__nv_bfloat16>::load(av, fa);
            Vec<__nv_bfloat16>::load(bv, fb);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float dhv = acc[j8 * 8 + i];
              const float sg = __fdividef(1.0f, 1.0f + __expf(-fa[i]));
              da[i] = dhv * fb[i] * (sg * (1.0f + fa[i] * (1.0f - sg)));
              db[i] = dhv * fa[i] * sg;
              ma = fmaxf(ma, fabsf(da[i]));
              mb = fmaxf(mb, fabsf(db[i]));
            }
            reinterpret_cast<uint4*>(p.C2 + row * (2 * I) + c0)[j8] = Vec<__nv_bfloat16>::store(da);
            reinterpret_cast<uint4*>(p.C2 + row * (2 * I) + I + c0)[j8] = Vec<__nv_bfloat16>::store(db);
          }
        }
        // a 128-column tile of da (and of db) spans warpgroups wg and wg ^ 1
        const int sl = it & 1;
        float* slot = amax_x + sl * 2 * kEpiWG * BM;
        slot[wg * BM + rit] = ma;
        slot[(kEpiWG + wg) * BM + rit] = mb;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xbar[sl]);   // this warp's amax values are in place
        const bool xok = mbar_wait_bounded(&xbar[sl], (it >> 1) & 1, abort_flag, kWaitNs);
        if (!xok) {
          raise_abort(abort_flag, p.err);
          break;
        }
        ma = fmaxf(ma, slot[(wg ^ 1) * BM + rit]);
        mb = fmaxf(mb, slot[(kEpiWG + (wg ^ 1)) * BM + rit]);
        const float sca = ma == 0.f ? 1.f : __fdiv_rn(ma, 448.f);
        const float scb = mb == 0.f ? 1.f : __fdiv_rn(mb, 448.f);
        if (valid) {
          // pass 2: the same float32 da, db again, quantised with the tile scales
          uint8_t* qa_p = static_cast<uint8_t*>(p.C) + row * (2 * I) + c0;
          uint8_t* qb_p = qa_p + I;
#pragma unroll
          for (int j16 = 0; j16 < CW / 16; ++j16) {
            uint32_t wa[4], wb[4];
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
              float fa[8], fb[8];
              Vec<__nv_bfloat16>::load(reinterpret_cast<const uint4*>(sa_p)[j16 * 2 + h8], fa);
              Vec<__nv_bfloat16>::load(reinterpret_cast<const uint4*>(sb_p)[j16 * 2 + h8], fb);
              float da[8], db[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float dhv = acc[j16 * 16 + h8 * 8 + i];
                const float sg = __fdividef(1.0f, 1.0f + __expf(-fa[i]));
                da[i] = dhv * fb[i] * (sg * (1.0f + fa[i] * (1.0f - sg)));
                db[i] = dhv * fa[i] * sg;
              }
              wa[h8 * 2] = e4m3x4(__fdiv_rn(da[0], sca), __fdiv_rn(da[1], sca),
                                  __fdiv_rn(da[2], sca), __fdiv_rn(da[3], sca));
              wa[h8 * 2 + 1] = e4m3x4(__fdiv_rn(da[4], sca), __fdiv_rn(da[5], sca),
                                      __fdiv_rn(da[6], sca), __fdiv_rn(da[7], sca));
              wb[h8 * 2] = e4m3x4(__fdiv_rn(db[0], scb), __fdiv_rn(db[1], scb),
                                  __fdiv_rn(db[2], scb), __fdiv_rn(db[3], scb));
              wb[h8 * 2 + 1] = e4m3x4(__fdiv_rn(db[4], scb), __fdiv_rn(db[5], scb),
                                      __fdiv_rn(db[6], scb), __fdiv_rn(db[7], scb));
            }
            reinterpret_cast<uint4*>(qa_p)[j16] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
            reinterpret_cast<uint4*>(qb_p)[j16] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
          }
          if ((wg & 1) == 0) {
            const int tile = c0 / 128;
            p.c_scale[row * (2 * I / 128) + tile] = sca;
            p.c_scale[row * (2 * I / 128) + I / 128 + tile] = scb;
          }
        }
      } else if (SWIGLU) {
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float gt = acc[j];
          acc[j] = __fdividef(gt, 1.0f + __expf(-gt)) * acc[32 + j];
          amax = fmaxf(amax, fabsf(acc[j]));
        }
        // The row's 128 h columns are spread over the warpgroups: exchange amax.
        const int sl = it & 1;
        float* slot = amax_x + sl * 2 * kEpiWG * BM;
        slot[wg * BM + rit] = amax;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xbar[sl]);   // this warp's amax values are in place
        const bool xok = mbar_wait_bounded(&xbar[sl], (it >> 1) & 1, abort_flag, kWaitNs);
        if (!xok) {
          raise_abort(abort_flag, p.err);
          break;
        }
#pragma unroll
        for (int o = 0; o < kEpiWG; ++o) amax = fmaxf(amax, slot[o * BM + rit]);
        const float sc = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
        if (valid) {
          uint8_t* dst = static_cast<uint8_t*>(p.C) + (size_t)(row0 + rit) * p.N + nt * 128 + wg * 32;
          uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int j = q * 16 + i * 4;
              w[i] = e4m3x4(__fdiv_rn(acc[j], sc), __fdiv_rn(acc[j + 1], sc),
                            __fdiv_rn(acc[j + 2], sc), __fdiv_rn(acc[j + 3], sc));
            }
            d4[q] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          if (wg == 0) p.c_scale[(size_t)(row0 + rit) * (p.N / 128) + nt] = sc;
        }
      } else {
        // STORE: 16 columns at a time through a 1 KB patch per warp, so that
        // each store instruction writes 16 rows x 32 bytes (whole sectors)
        // instead of 32 rows x 16 bytes
        uint4* patch = reinterpret_cast<uint4*>(smem + OFF_PATCH + (warp - 2) * 1024);   // [32][2]
        __nv_bfloat16* cbase = static_cast<__nv_bfloat16*>(p.C) + nt * BN + wg * CW;
#pragma unroll
        for (int q16 = 0; q16 < CW / 16; ++q16) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int j = q16 * 16 + h * 8 + 2 * i;
              __nv_bfloat162 pr = __floats2bfloat162_rn(acc[j], acc[j + 1]);
              w[i] = *reinterpret_cast<uint32_t*>(&pr);
            }
            patch[lane * 2 + h] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int piece = i * 32 + lane;
            const int r = piece >> 1;                    // row of this warp's 32
            const int rr = sub * 32 + r;                 // row inside the tile
            if (rr < mv && in_bounds(row0 + rr < p.rows, p.err))
              *reinterpret_cast<uint4*>(cbase + (size_t)(row0 + rr) * p.N + q16 * 16 +
                                        (piece & 1) * 8) = patch[piece];
          }
          __syncwarp();
        }
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

template <int EPI, bool B_MN>
moe_status fp8_launch(const void* A, const float* a_scale, const void* B, const float* b_scale,
                      int b_rows_per_group, const int32_t* offsets, int n_groups, int rows, int N,
                      int K, void* C, float* c_scale, void* S, int lds, void* C2,
                      cudaStream_t s) {
  constexpr int BN_OUT = Fp8Tile<EPI>::BN_OUT;
  CUtensorMap tmA, tmB;
  moe_status st = make_tmap_2d(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, rows, BK, BM);
  if (st != MOE_OK) return st;
  const int G = offsets ? n_groups : 1;
  if (B_MN)
    st = make_tmap_col_blocks(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, (uint64_t)G * K, 128,
                              BK, BN / 128);
  else
    st = make_tmap_2d(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, (uint64_t)G * b_rows_per_group,
                      BK, Fp8Tile<EPI>::SW ? 128 : BN);
  if (st != MOE_OK) return st;
  auto kern = fp8_gemm_kernel<EPI, B_MN>;
  static bool attr_done[kMaxSmemDevices] = {};   // per instantiation and device
  {
    const moe_status sst = ensure_max_smem(reinterpret_cast<const void*>(kern), SMEM_ALLOC,
                                           attr_done, "fp8_gemm smem attribute");
    if (sst != MOE_OK) return sst;
  }
  Fp8Params p;
  p.offsets = offsets;
  p.n_groups = n_groups;
  p.rows = rows;
  p.N = N;
  p.K = K;
  p.b_rows_per_group = b_rows_per_group;
  p.half_b = Fp8Tile<EPI>::SW ? b_rows_per_group / 2 : 0;
  p.a_scale = a_scale;
  p.b_scale = b_scale;
  p.C = C;
  p.c_scale = c_scale;
  p.S = static_cast<__nv_bfloat16*>(S);
  p.lds = lds;
  p.C2 = static_cast<__nv_bfloat16*>(C2);
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  const long long max_tiles = ((long long)(rows + BM - 1) / BM + (offsets ? G : 0)) * (N / BN_OUT);
  int grid = sm_count();
  if (max_tiles < grid) grid = (int)(max_tiles > 0 ? max_tiles : 1);
  kern<<<grid, kThreads, SMEM_ALLOC, s>>>(tmA, tmB, p);
  return cuda_check(cudaGetLastError(), "fp8_gemm launch");
}

}  // namespace

moe_status launch_fp8_gemm(const void* A, const float* a_scale, const void* B,
                           const float* b_scale, int b_rows_per_group, const int32_t* offsets,
                           int n_groups, int rows, int N, int K, bool swiglu, void* C,
                           float* c_scale, cudaStream_t s) {
  return launch_fp8_gemm_ex(A, a_scale, B, b_scale, b_rows_per_group, offsets, n_groups, rows, N,
                            K, swiglu ? F8_SWIGLU : F8_STORE, false, C, c_scale, nullptr, 0,
                            nullptr, s);
}

moe_status launch_fp8_gemm_ex(const void* A, const float* a_scale, const void* B,
                              const float* b_scale, int b_rows_per_group, const int32_t* offsets,
                              int n_groups, int rows, int N, int K, Fp8Epi epi, bool b_mn,
                              void* C, float* c_scale, void* S, int lds, void* C2,
                              cudaStream_t s) {
  if (rows <= 0) return MOE_OK;
  if (K % BK) return fail(MOE_ERR_UNSUPPORTED, "fp8 gemm: K=%d not a multiple of 128", K);
  if (offsets && n_groups > kMaxGroups)
    return fail(MOE_ERR_UNSUPPORTED, "fp8 gemm: at most %d groups", kMaxGroups);
  const bool sw = epi == F8_SWIGLU || epi == F8_SWIGLU_SAVE;
  if (sw && N % 128) return fail(MOE_ERR_UNSUPPORTED, "fp8 gemm swiglu: N=%d %% 128", N);
  if (!sw && N % 256) return fail(MOE_ERR_UNSUPPORTED, "fp8 gemm: N=%d must be a multiple of 256", N);
  if (sw && b_mn) return fail(MOE_ERR_UNSUPPORTED, "fp8 gemm: MN-major weights with swiglu");
  if (epi == F8_DSWIGLU && !b_mn) return fail(MOE_ERR_UNSUPPORTED, "fp8 dswiglu needs MN-major W");
  switch (epi) {
    case F8_SWIGLU:
      return fp8_launch<F8_SWIGLU, false>(A, a_scale, B, b_scale, b_rows_per_group, offsets,
                                          n_groups, rows, N, K, C, c_scale, S, lds, C2, s);
    case F8_SWIGLU_SAVE:
      return fp8_launch<F8_SWIGLU_SAVE, false>(A, a_scale, B, b_scale, b_rows_per_group, offsets,
                                               n_groups, rows, N, K, C, c_scale, S, lds, C2, s);
    case F8_STORE:
      return b_mn ? fp8_launch<F8_STORE, true>(A, a_scale, B, b_scale, b_rows_per_group, offsets,
                                               n_groups, rows, N, K, C, c_scale, S, lds, C2, s)
                  : fp8_launch<F8_STORE, false>(A, a_scale, B, b_scale, b_rows_per_group, offsets,
                                                n_groups, rows, N, K, C, c_scale, S, lds, C2, s);
    case F8_DSWIGLU:
      return fp8_launch<F8_DSWIGLU, true>(A, a_scale, B, b_scale, b_rows_per_group, offsets,
                                          n_groups, rows, N, K, C, c_scale, S, lds, C2, s);
  }
  return fail(MOE_ERR_INVALID_ARG, "fp8 gemm: unknown epilogue %d", (int)epi);
}

}  // namespace moe
