// Weights-stationary grouped bf16 GEMM on tcgen05 for the expert FFNs
// (FFN_i of the h'-equation, "DeepSeek-V3 技術報告", section 方法 / 2).
//
// The MMA's M side is the weight matrix and its N side the expert's tokens:
//   D[n, j] = sum_k W[g*b_rows + w0 + n, k] * X[tok0 + j, k]
// A tile is 256 weight rows x up to 256 token rows.  Each 64-wide K step
// issues two M=128 MMAs per 16-element slice (SWIGLU: the 128 gate rows and
// the 128 matching up rows of one h-column block; STORE: output columns
// [0,128) and [128,256) of a 256-column block), both with N = the tile's token
// count rounded up to 16.  An expert with M tokens is cut into
// ceil(M/256) token tiles of equal size (multiples of 16), so ragged expert
// loads cost at most 15 padding rows per tile instead of a 128-row tail.
//
// Epilogue (8 warps; warp w owns TMEM lanes 32*(w%4).. = weight rows, and
// every other 32-token chunk):
//   SWIGLU  h[tok0+j, nt*128 + n] = bf16(SiLU(D_gate[n,j]) * D_up[n,j])
//   STORE   y[tok0+j, nt*256 + n] = bf16(D0[n,j]), y[.., nt*256+128+n] = bf16(D1[n,j])
// Values are transposed through a 2 KB shared-memory patch per warp so that
// global stores are 16-byte vectors along token rows.
//
// Roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps 2-9
// epilogue.  3 shared-memory stages of 64 KB; one TMEM accumulator pair
// (512 columns).  Every wait is bounded (1 s) and reported through the
// device error word.
//
// Extra groups (the shared experts of the h'-equation, weight 1): n_extra
// groups of T_extra rows each run in the same launch after the routed
// groups, with their own weight map (group j = row block j of W_extra) and
// token map (gate/up: the layer input u, rows [0, T_extra); down: the same
// h buffer as the routed rows).  Extra group j's output rows are
// rows + j*T_extra + [0, T_extra) of C.
#include <math.h>

#include "launch.h"
#include "sm100.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int WROWS = 256;          // weight rows per tile (two M=128 MMAs)
constexpr int TMAX = 256;           // max token rows per tile (MMA N)
constexpr int BK = 64;              // bf16 elements per 128-byte swizzle row
constexpr int STAGES = 3;
constexpr int kEpiWarps = 8;        // two warps per TMEM lane quarter, alternating token chunks
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxGroups = 1024;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t TMEM_COLS = 512;

constexpr int W_BYTES = WROWS * BK * 2;       // 32 KB
constexpr int X_BYTES = TMAX * BK * 2;        // 32 KB
constexpr int WBOX_MN_BYTES = 64 * BK * 2;    // MN-major weights: one [64 K][64 N] box, 8 KB
constexpr int OFF_X = STAGES * W_BYTES;
constexpr int OFF_STAGE_OUT = OFF_X + STAGES * X_BYTES;   // one 2 KB transpose patch per epilogue warp
constexpr int OFF_BAR = OFF_STAGE_OUT + kEpiWarps * 2048;
constexpr int N_BARS = 2 * STAGES + 3;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int OFF_TAB = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_TAB + 2 * (kMaxGroups + 1) * 4;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

struct WsParams {
  const int32_t* offsets;   // [n_groups+1] or nullptr (one group of `rows`)
  int n_groups;
  int rows;
  int N;                    // output columns (SWIGLU*: I; STORE: d; DSWIGLU: I)
  int K;
  int b_rows_per_group;     // K-major weights: rows of W per group
  int half_b;               // SWIGLU*: I (row offset of W_up inside a group)
  __nv_bfloat16* C;
  int ldc;                  // row stride of C in elements
  __nv_bfloat16* S;         // SWIGLU_SAVE: pre-activations written; DSWIGLU: read
  int lds;                  // row stride of S (2I)
  int n_extra;              // extra groups after the routed ones (0: none)
  int T_extra;              // rows of each extra group
  int x_extra_local;        // 1: extra groups read X rows [0, T_extra); 0: their C rows
  int* err;
};

template <int EPI>
struct TileMath {
  static constexpr bool SW = EPI == WS_SWIGLU || EPI == WS_SWIGLU_SAVE;
  static constexpr int OUT_COLS = SW ? 128 : 256;   // output columns per weight tile
};

// Token tiling of a group of m rows: tiles of `step` rows (a multiple of 16,
// at most 256, about m / ceil(m/256)); n_t = ceil(m / step) tiles, each with
// at least one row, the last one possibly shorter.
__device__ __forceinline__ void token_tiling(int m, int& n_t, int& step) {
  if (m <= 0) { n_t = 0; step = 16; return; }
  const int n0 = (m + TMAX - 1) / TMAX;
  step = ((m + n0 - 1) / n0 + 15) / 16 * 16;
  n_t = (m + step - 1) / step;
}

// Rows of group g: routed groups from roff, extra group j = g - G at
// C rows base = rows + j * T_extra.
__device__ __forceinline__ void group_span(int g, int G, const int* roff, const WsParams& p,
                                           int& base, int& m) {
  if (g < G) {
    base = roff[g];
    m = roff[g + 1] - roff[g];
  } else {
    base = p.rows + (g - G) * p.T_extra;
    m = p.T_extra;
  }
}

// Tile t -> group g, weight tile nt, first C row tok0, rows count, and the
// first row xrow0 of X that the tile reads.
__device__ __forceinline__ void decode_tile(int t, const int* prefix, const int* roff, int G,
                                            int Gtot, const WsParams& p, int& g, int& nt,
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

// SiLU for a bf16 result: fast exponential and division are well inside bf16 rounding.
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

template <int EPI, bool WMN>
__global__ void __launch_bounds__(kThreads, 1)
    ws_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmX128,
                   const __grid_constant__ CUtensorMap tmX256,
                   const __grid_constant__ CUtensorMap tmW2,
                   const __grid_constant__ CUtensorMap tmX2,
                   const __grid_constant__ CUtensorMap tmX2_128,
                   const __grid_constant__ CUtensorMap tmX2_256, const WsParams p) {
  constexpr int OUT_COLS = TileMath<EPI>::OUT_COLS;
  constexpr bool SWIGLU = TileMath<EPI>::SW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sW = smem;
  uint8_t* sX = smem + OFF_X;
  uint8_t* sOut = smem + OFF_STAGE_OUT;
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
  const int G = p.offsets ? p.n_groups : 1;
  const int Gtot = G + p.n_extra;
  const int n_wt = p.N / OUT_COLS;   // weight tiles per group

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(tfull, 1);
    mbar_init(tempty, kEpiWarps);      // one arrival per epilogue warp
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmX128);
    tma_prefetch_desc(&tmX256);
    if (p.n_extra) {
      tma_prefetch_desc(&tmW2);
      tma_prefetch_desc(&tmX2);
      tma_prefetch_desc(&tmX2_128);
      tma_prefetch_desc(&tmX2_256);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2) {
    // Tile table: prefix[g] = first tile of group g; tiles of a group are
    // ordered weight-tile major, token-tile fastest.  Offsets are clamped
    // into disjoint ranges of [0, rows) first.
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
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = prefix[Gtot];
  const int nk = p.K / BK;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int g, nt, tok0, count, xrow0;
        decode_tile(t, prefix, roff, G, Gtot, p, g, nt, tok0, count, xrow0);
        const bool extra = g >= G;
        const CUtensorMap* tw = extra ? &tmW2 : &tmW;
        // one token box per stage: 64, 128 or 256 rows (it may read past the
        // tile's rows, which the MMA's N or the epilogue leaves unused)
        const int xb = count <= 64 ? 64 : count <= 128 ? 128 : 256;
        const CUtensorMap* tx = xb == 64 ? (extra ? &tmX2 : &tmX)
                                : xb == 128 ? (extra ? &tmX2_128 : &tmX128)
                                            : (extra ? &tmX2_256 : &tmX256);
        const uint32_t bytes = W_BYTES + (uint32_t)xb * BK * 2;
        const int wrow = (extra ? g - G : g) * p.b_rows_per_group + nt * (SWIGLU ? 128 : 256);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, kWaitNs)) {
            raise_abort(abort_flag, p.err);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], bytes);
          uint8_t* w_dst = sW + stage * W_BYTES;
          if (WMN) {
            // weights stored [K rows][N cols]: four [64 K][64 N] boxes of columns nt*256 + 64j
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_2d(w_dst + j * WBOX_MN_BYTES, &tmW, nt * 256 + 64 * j,
                          g * p.K + kb * BK, &full[stage]);
          } else {
            tma_load_2d(w_dst, tw, kb * BK, wrow, &full[stage]);
            tma_load_2d(w_dst + W_BYTES / 2, tw, kb * BK, wrow + (SWIGLU ? p.half_b : 128),
                        &full[stage]);
          }
          tma_load_2d(sX + stage * X_BYTES, tx, kb * BK, xrow0, &full[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      for (int s = 0; s < STAGES; ++s)
        mbar_wait_bounded(&full[s], ((s < stage) ? phase : phase ^ 1), nullptr, kWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, tphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int g, nt, tok0, count, xrow0;
        decode_tile(t, prefix, roff, G, Gtot, p, g, nt, tok0, count, xrow0);
        const int n_mma = (count + 15) / 16 * 16;
        const uint32_t idesc = idesc_bf16_f32_major(128, n_mma, WMN, false);
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
            const uint64_t a0 = WMN ? smem_desc_mn_sw128(w0 + k * 2048, WBOX_MN_BYTES)
                                    : smem_desc_k_sw128(w0 + k * 32);
            const uint64_t a1 = WMN ? smem_desc_mn_sw128(w0 + W_BYTES / 2 + k * 2048,
                                                         WBOX_MN_BYTES)
                                    : smem_desc_k_sw128(w0 + W_BYTES / 2 + k * 32);
            mma_f16_ss(tmem_base, a0, xd, idesc, acc);
            mma_f16_ss(tmem_base + 256, a1, xd, idesc, acc);
          }
          mma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        mma_commit(tfull);
        tphase ^= 1;
      }
      mma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr, kWaitNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                       // TMEM lane quarter
    const int ch = (warp - 2) >> 2;               // which alternate 32-token chunks this warp takes
    uint16_t* patch = reinterpret_cast<uint16_t*>(sOut + (warp - 2) * 2048);   // [32 tok][32 col]
    uint32_t tphase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      int g, nt, tok0, count, xrow0;
      decode_tile(t, prefix, roff, G, Gtot, p, g, nt, tok0, count, xrow0);
      const bool got = mbar_wait_bounded(tfull, tphase, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, got)) {
        raise_abort(abort_flag, p.err);
        break;
      }
      tc_fence_after();
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      const int nch = (count + 31) / 32;
      if (EPI == WS_DSWIGLU) {
        // dh[tok, col] from TMEM; a = S[tok, col], b = S[tok, I + col]:
        //   dA[tok, col] = dh * b * SiLU'(a),  dA[tok, I + col] = dh * SiLU(a).
        // dh goes through a float32 [16 tok][32 col] patch so that every
        // global access is a 16-byte vector along a token row.
        float* pf = reinterpret_cast<float*>(patch);
        for (int c = ch; c < nch; c += 2) {
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(tl + c * 32, r0);
          tmem_ld_32x32b_x32(tl + 256 + c * 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                pf[j * 32 + lane] = __uint_as_float(hh == 0 ? r0[sub * 16 + j] : r1[sub * 16 + j]);
              __syncwarp();
              // both 16-byte pieces of this lane first, then the arithmetic
              uint4 av[2], bv[2];
              size_t grow[2];
              int col[2], c8[2], row[2];
              bool ok[2];
#pragma unroll
              for (int it = 0; it < 2; ++it) {
                const int idx = it * 32 + lane;
                row[it] = idx >> 2;
                c8[it] = (idx & 3) * 8;
                const int tok = c * 32 + sub * 16 + row[it];
                ok[it] = tok < count &&
                         in_bounds(tok0 + tok < p.rows + p.n_extra * p.T_extra, p.err);
                grow[it] = (size_t)(tok0 + (ok[it] ? tok : 0));
                col[it] = nt * 256 + hh * 128 + q * 32 + c8[it];
                if (ok[it]) {
                  av[it] = *reinterpret_cast<const uint4*>(p.S + grow[it] * p.lds + col[it]);
                  bv[it] = *reinterpret_cast<const uint4*>(p.S + grow[it] * p.lds + p.N + col[it]);
                }
              }
#pragma unroll
              for (int it = 0; it < 2; ++it) {
                if (ok[it]) {
                  const float4 d0 = *reinterpret_cast<const float4*>(pf + row[it] * 32 + c8[it]);
                  const float4 d1 = *reinterpret_cast<const float4*>(pf + row[it] * 32 + c8[it] + 4);
                  const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
                  float fa[8], fb[8], oa[8], ob[8];
                  Vec<__nv_bfloat16>::load(av[it], fa);
                  Vec<__nv_bfloat16>::load(bv[it], fb);
#pragma unroll
                  for (int i = 0; i < 8; ++i) {
                    const float sg = __fdividef(1.0f, 1.0f + __expf(-fa[i]));
                    oa[i] = dv[i] * fb[i] * (sg * (1.0f + fa[i] * (1.0f - sg)));
                    ob[i] = dv[i] * fa[i] * sg;
                  }
                  *reinterpret_cast<uint4*>(p.C + grow[it] * p.ldc + col[it]) =
                      Vec<__nv_bfloat16>::store(oa);
                  *reinterpret_cast<uint4*>(p.C + grow[it] * p.ldc + p.N + col[it]) =
                      Vec<__nv_bfloat16>::store(ob);
                }
              }
              __syncwarp();
            }
          }
        }
      } else
      for (int c = ch; c < nch; c += 2) {
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(tl + c * 32, r0);
        tmem_ld_32x32b_x32(tl + 256 + c * 32, r1);
        tmem_wait_ld();
        // outputs: SWIGLU h; SWIGLU_SAVE h, gate and up pre-activations; STORE two halves
        constexpr int n_out = EPI == WS_SWIGLU_SAVE ? 3 : (SWIGLU ? 1 : 2);
#pragma unroll
        for (int hh = 0; hh < n_out; ++hh) {
          // patch[j][lane] = value of token (c*32 + j), column (q*32 + lane)
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float v;
            if (SWIGLU && hh == 0) v = silu_f(__uint_as_float(r0[j])) * __uint_as_float(r1[j]);
            else if (SWIGLU) v = __uint_as_float(hh == 1 ? r0[j] : r1[j]);
            else v = __uint_as_float(hh == 0 ? r0[j] : r1[j]);
            patch[j * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
          }
          __syncwarp();
          // 32 token rows x 64 bytes: lane -> (row lane/4 + 8*it, 16-byte chunk lane%4)
          __nv_bfloat16* base;
          int ld, col0;
          if (!SWIGLU) { base = p.C; ld = p.ldc; col0 = nt * OUT_COLS + hh * 128 + q * 32; }
          else if (hh == 0) { base = p.C; ld = p.ldc; col0 = nt * 128 + q * 32; }
          else { base = p.S; ld = p.lds; col0 = (hh == 2 ? p.N : 0) + nt * 128 + q * 32; }
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int j = it * 8 + (lane >> 2);
            const int tok = c * 32 + j;
            const uint4 v = *reinterpret_cast<const uint4*>(patch + j * 32 + (lane & 3) * 8);
            if (tok < count && in_bounds(tok0 + tok < p.rows + p.n_extra * p.T_extra, p.err)) {
              __nv_bfloat16* dst = base + (size_t)(tok0 + tok) * ld + col0 + (lane & 3) * 8;
              *reinterpret_cast<uint4*>(dst) = v;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);
      tphase ^= 1;
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

moe_status make_tmap_2d(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                        int elem_bytes, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer);

namespace {

template <int EPI, bool WMN>
moe_status ws_launch(const void* X, const void* W, int b_rows_per_group, const int32_t* offsets,
                     int n_groups, int rows, int N, int K, void* C, int ldc, void* S, int lds,
                     const WsExtraGroups& ex, cudaStream_t s) {
  constexpr int OUT_COLS = TileMath<EPI>::OUT_COLS;
  CUtensorMap tmW, tmX, tmX128, tmX256, tmW2, tmX2, tmX2_128, tmX2_256;
  const int G = offsets ? n_groups : 1;
  long long x_rows = ex.n_extra && !ex.x_local ? rows + (long long)ex.n_extra * ex.T : rows;
  if (x_rows == 0) x_rows = ex.T;   // no routed rows: a map over the extra X, never read
  moe_status st = WMN ? make_tmap_2d(&tmW, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N,
                                     (uint64_t)G * K, 64, BK)
                      : make_tmap_2d(&tmW, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K,
                                     (uint64_t)G * b_rows_per_group, BK, 128);
  if (st != MOE_OK) return st;
  auto xmaps = [&](const void* base, uint64_t n, CUtensorMap* m64, CUtensorMap* m128,
                   CUtensorMap* m256) -> moe_status {
    moe_status r = make_tmap_2d(m64, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, n, BK, 64);
    if (r == MOE_OK) r = make_tmap_2d(m128, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, n, BK, 128);
    if (r == MOE_OK) r = make_tmap_2d(m256, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, n, BK, 256);
    return r;
  };
  st = xmaps(X, (uint64_t)x_rows, &tmX, &tmX128, &tmX256);
  if (st != MOE_OK) return st;
  tmW2 = tmW;
  tmX2 = tmX;
  tmX2_128 = tmX128;
  tmX2_256 = tmX256;
  if (ex.n_extra) {
    st = make_tmap_2d(&tmW2, ex.W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K,
                      (uint64_t)ex.n_extra * b_rows_per_group, BK, 128);
    if (st != MOE_OK) return st;
    if (ex.x_local) {
      st = xmaps(ex.X, (uint64_t)ex.T, &tmX2, &tmX2_128, &tmX2_256);
      if (st != MOE_OK) return st;
    }
  }
  auto kern = ws_gemm_kernel<EPI, WMN>;
  static bool attr_done[kMaxSmemDevices] = {};   // per instantiation and device
  {
    const moe_status sst = ensure_max_smem(reinterpret_cast<const void*>(kern), SMEM_ALLOC,
                                           attr_done, "ws_gemm smem attribute");
    if (sst != MOE_OK) return sst;
  }
  WsParams p;
  p.offsets = offsets;
  p.n_groups = n_groups;
  p.rows = rows;
  p.N = N;
  p.K = K;
  p.b_rows_per_group = b_rows_per_group;
  p.half_b = TileMath<EPI>::SW ? b_rows_per_group / 2 : 0;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.ldc = ldc;
  p.S = static_cast<__nv_bfloat16*>(S);
  p.lds = lds;
  p.n_extra = ex.n_extra;
  p.T_extra = ex.T;
  p.x_extra_local = ex.x_local ? 1 : 0;
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  const long long max_tiles =
      ((long long)(rows + TMAX - 1) / TMAX + (offsets ? G : 0) +
       (long long)ex.n_extra * ((ex.T + TMAX - 1) / TMAX)) * (N / OUT_COLS);
  int grid = sm_count();
  if (max_tiles < grid) grid = (int)(max_tiles > 0 ? max_tiles : 1);
  kern<<<grid, kThreads, SMEM_ALLOC, s>>>(tmW, tmX, tmX128, tmX256, tmW2, tmX2, tmX2_128, tmX2_256, p);
  return cuda_check(cudaGetLastError(), "ws_gemm launch");
}

}  // namespace

moe_status launch_ws_gemm(const void* X, const void* W, int b_rows_per_group,
                          const int32_t* offsets, int n_groups, int rows, int N, int K,
                          bool swiglu, void* C, cudaStream_t s, const WsExtraGroups* extra) {
  // the down projection (STORE) runs on CTA pairs where the shape allows
  if (!swiglu && ws2_gemm_supported(N, K, n_groups, offsets != nullptr))
    return launch_ws2_gemm(X, W, b_rows_per_group, offsets, n_groups, rows, N, K, C, s, extra);
  return launch_ws_gemm_ex(X, W, b_rows_per_group, offsets, n_groups, rows, N, K,
                           swiglu ? WS_SWIGLU : WS_STORE, false, C, N, nullptr, 0, s, extra);
}

moe_status launch_ws_gemm_ex(const void* X, const void* W, int b_rows_per_group,
                             const int32_t* offsets, int n_groups, int rows, int N, int K,
                             WsEpi epi, bool w_mn, void* C, int ldc, void* S, int lds,
                             cudaStream_t s, const WsExtraGroups* extra) {
  const WsExtraGroups none{};
  const WsExtraGroups& ex = extra ? *extra : none;
  if (ex.n_extra && (epi == WS_SWIGLU_SAVE || epi == WS_DSWIGLU || w_mn))
    return fail(MOE_ERR_UNSUPPORTED, "ws gemm: extra groups only with the forward epilogues");
  if (rows <= 0 && (ex.n_extra == 0 || ex.T <= 0)) return MOE_OK;
  if (K % BK) return fail(MOE_ERR_UNSUPPORTED, "ws gemm: K=%d not a multiple of %d", K, BK);
  if (offsets && n_groups > kMaxGroups)
    return fail(MOE_ERR_UNSUPPORTED, "ws gemm: at most %d groups", kMaxGroups);
  const bool sw = epi == WS_SWIGLU || epi == WS_SWIGLU_SAVE;
  if (sw && N % 128) return fail(MOE_ERR_UNSUPPORTED, "ws gemm swiglu: N=%d %% 128", N);
  if (!sw && N % 256) return fail(MOE_ERR_UNSUPPORTED, "ws gemm: N=%d %% 256", N);
  if (w_mn && sw) return fail(MOE_ERR_UNSUPPORTED, "ws gemm: MN-major weights with swiglu");
  switch (epi) {
    case WS_SWIGLU:
      return ws_launch<WS_SWIGLU, false>(X, W, b_rows_per_group, offsets, n_groups, rows, N, K,
                                         C, ldc, S, lds, ex, s);
    case WS_SWIGLU_SAVE:
      return ws_launch<WS_SWIGLU_SAVE, false>(X, W, b_rows_per_group, offsets, n_groups, rows,
                                              N, K, C, ldc, S, lds, ex, s);
    case WS_STORE:
      return w_mn ? ws_launch<WS_STORE, true>(X, W, b_rows_per_group, offsets, n_groups, rows, N,
                                              K, C, ldc, S, lds, ex, s)
                  : ws_launch<WS_STORE, false>(X, W, b_rows_per_group, offsets, n_groups, rows,
                                               N, K, C, ldc, S, lds, ex, s);
    case WS_DSWIGLU:
      if (!w_mn) return fail(MOE_ERR_UNSUPPORTED, "ws gemm dswiglu: needs MN-major weights");
      return ws_launch<WS_DSWIGLU, true>(X, W, b_rows_per_group, offsets, n_groups, rows, N, K,
                                         C, ldc, S, lds, ex, s);
  }
  return fail(MOE_ERR_INVALID_ARG, "ws gemm: unknown epilogue %d", (int)epi);
}

}  // namespace moe
