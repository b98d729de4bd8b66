// FP8 quantisers of the fine-grained recipe in "DeepSeek-V3 技術報告",
// section 核心概念 (FP8 bullet): E4M3 values with one float32 scale per 1x128
// activation tile or per 128x128 weight block.
//   scale = amax / 448 (1 for an all-zero tile)
//   q     = E4M3 round-to-nearest-even, saturated to +-448, of x / scale
// x / scale is an IEEE float32 division so the code of every element is a
// function of the stored inputs alone.
#include "launch.h"

namespace moe {

namespace {

__device__ __forceinline__ float tile_scale(float amax) {
  return amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
}

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

// One half-warp per (row, 128-column tile): lane l of the half holds columns
// 8l..8l+7 (one 16-byte load); each half-warp quantises kQU tiles, their
// loads issued together so that enough bytes are in flight per SM.
constexpr int kQU = 4;

__global__ void __launch_bounds__(256) quant_1x128_kernel(const __nv_bfloat16* __restrict__ x,
                                                          int rows, int cols,
                                                          uint8_t* __restrict__ q,
                                                          float* __restrict__ scale) {
  const int l16 = threadIdx.x & 15;
  const int tiles_per_row = cols / 128;
  const long long n_tiles = (long long)rows * tiles_per_row;
  const long long n_half = (long long)gridDim.x * (blockDim.x >> 4);
  const long long h = (long long)blockIdx.x * (blockDim.x >> 4) + (threadIdx.x >> 4);
  uint4 raw[kQU];
  size_t base[kQU];
#pragma unroll
  for (int k = 0; k < kQU; ++k) {
    const long long t = h + k * n_half;
    base[k] = 0;
    raw[k] = make_uint4(0u, 0u, 0u, 0u);
    if (t < n_tiles) {
      const long long r = t / tiles_per_row;
      const int tb = (int)(t - r * tiles_per_row);
      base[k] = (size_t)r * cols + (size_t)tb * 128 + l16 * 8;
      raw[k] = *reinterpret_cast<const uint4*>(x + base[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < kQU; ++k) {
    const long long t = h + k * n_half;
    const uint32_t w[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    // the tile's 16 lanes (every lane shuffles: the offsets stay inside a half)
#pragma unroll
    for (int off = 8; off > 0; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (t < n_tiles) {
      const float sc = tile_scale(amax);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        lo |= (uint32_t)to_e4m3(__fdiv_rn(v[i], sc)) << (8 * i);
        hi |= (uint32_t)to_e4m3(__fdiv_rn(v[4 + i], sc)) << (8 * i);
      }
      *reinterpret_cast<uint2*>(q + base[k]) = make_uint2(lo, hi);
      if (l16 == 0) scale[(size_t)t] = sc;
    }
  }
}

// One 256-thread block per 128x128 block of one group.
__global__ void __launch_bounds__(256) quant_128x128_kernel(const __nv_bfloat16* __restrict__ w,
                                                            int rows, int cols,
                                                            uint8_t* __restrict__ q,
                                                            float* __restrict__ scale) {
  __shared__ float red[8];
  const int cb = blockIdx.x, rb = blockIdx.y, g = blockIdx.z;
  const int nrb = rows / 128, ncb = cols / 128;
  const __nv_bfloat16* src = w + ((size_t)g * rows + (size_t)rb * 128) * cols + (size_t)cb * 128;
  uint8_t* dst = q + ((size_t)g * rows + (size_t)rb * 128) * cols + (size_t)cb * 128;
  // thread -> (row = tid/16 + 16*i, 8 columns at (tid%16)*8), i = 0..7
  const int c8 = (threadIdx.x & 15) * 8;
  const int r0 = threadIdx.x >> 4;
  float v[8][8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 raw = *reinterpret_cast<const uint4*>(src + (size_t)(r0 + 16 * i) * cols + c8);
    const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[i][2 * j] = __uint_as_float(wv[j] << 16);
      v[i][2 * j + 1] = __uint_as_float(wv[j] & 0xffff0000u);
      amax = fmaxf(amax, fmaxf(fabsf(v[i][2 * j]), fabsf(v[i][2 * j + 1])));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float sc = tile_scale(amax);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      lo |= (uint32_t)to_e4m3(__fdiv_rn(v[i][j], sc)) << (8 * j);
      hi |= (uint32_t)to_e4m3(__fdiv_rn(v[i][4 + j], sc)) << (8 * j);
    }
    *reinterpret_cast<uint2*>(dst + (size_t)(r0 + 16 * i) * cols + c8) = make_uint2(lo, hi);
  }
  if (threadIdx.x == 0) scale[((size_t)g * nrb + rb) * ncb + cb] = sc;
}

}  // namespace

moe_status launch_quant_1x128(const void* x, int rows, int cols, uint8_t* q, float* scale,
                              cudaStream_t s) {
  const long long tiles = (long long)rows * (cols / 128);
  const int per_block = (256 / 16) * kQU;        // 16 half-warps, kQU tiles each
  const long long blocks = (tiles + per_block - 1) / per_block;
  if (blocks > 0x7fffffffLL) return fail(MOE_ERR_UNSUPPORTED, "quantize_1x128: too many tiles");
  if (blocks == 0) return MOE_OK;
  quant_1x128_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(x), rows, cols, q, scale);
  return cuda_check(cudaGetLastError(), "quant_1x128 launch");
}

moe_status launch_quant_128x128(const void* w, int groups, int rows, int cols, uint8_t* q,
                                float* scale, cudaStream_t s) {
  if (groups > 65535 || rows / 128 > 65535)
    return fail(MOE_ERR_UNSUPPORTED, "quantize_128x128: grid too large");
  dim3 grid(cols / 128, rows / 128, groups);
  quant_128x128_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), rows, cols, q,
                                            scale);
  return cuda_check(cudaGetLastError(), "quant_128x128 launch");
}

namespace {

// ---------------------------------------------------------------- Wgrad operands
// 128x1 tiles along the rows of each group (the contraction of a weight
// gradient runs over an expert's tokens): blocks of 128 consecutive rows start
// at every group's first row, the last block of a group may be shorter, and
// every column of a block gets its own scale.

// block_start[g] = sum over g' < g of ceil(rows of g' / 128); block_start[G] = total.
// A group's rows are clamped into [0, rows) (its size is never negative), so
// the total never exceeds ceil(rows / 128) + G.
__global__ void __launch_bounds__(1024) block_table_kernel(const int32_t* __restrict__ offsets,
                                                           int G, int rows,
                                                           int32_t* __restrict__ block_start) {
  __shared__ int warp_sum[32];
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  int run = 0;
  for (int base = 0; base < G; base += 1024) {
    const int g = base + t;
    int c = 0;
    if (g < G) {
      int r0, r1;
      clamp_group_rows(offsets, g, rows, nullptr, r0, r1);
      c = (r1 - r0 + 127) / 128;
    }
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sum[w] = incl;
    __syncthreads();
    if (w == 0) {
      int ws = warp_sum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += v;
      }
      warp_sum[lane] = ws;
    }
    __syncthreads();
    const int before = (w > 0 ? warp_sum[w - 1] : 0) + incl - c;
    if (g < G) block_start[g] = run + before;
    const int chunk_total = warp_sum[31];
    __syncthreads();
    run += chunk_total;
  }
  if (t == 0) block_start[G] = run;
}

__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// Two columns per thread, 256 columns per block; blockIdx.x = 128-row block.
// SWIGLU_IN: the value of (row, c) is SiLU(x[row, c]) * x[row, cols + c].
template <bool SWIGLU_IN>
__global__ void __launch_bounds__(128) quant_128x1_kernel(
    const __nv_bfloat16* __restrict__ x, int ldx, const int32_t* __restrict__ src_rows, int rows,
    int cols, const int32_t* __restrict__ offsets, int G, const int32_t* __restrict__ block_start,
    uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int blk = blockIdx.x;
  if (blk >= block_start[G]) return;
  int lo = 0, hi = G - 1;                  // last group whose first block is <= blk
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (block_start[mid] <= blk) lo = mid; else hi = mid - 1;
  }
  int g0, g1;
  clamp_group_rows(offsets, lo, rows, nullptr, g0, g1);
  const int r0 = g0 + (blk - block_start[lo]) * 128;
  const int r1 = min(r0 + 128, g1);
  const int c = (blockIdx.y * 128 + threadIdx.x) * 2;
  if (c >= cols) return;
  auto load = [&](int r, float& v0, float& v1) {
    const size_t row = (size_t)(src_rows ? src_rows[r] : r);
    const uint32_t a = *reinterpret_cast<const uint32_t*>(x + row * ldx + c);
    v0 = __uint_as_float(a << 16);
    v1 = __uint_as_float(a & 0xffff0000u);
    if (SWIGLU_IN) {
      const uint32_t b = *reinterpret_cast<const uint32_t*>(x + row * ldx + cols + c);
      v0 = silu_fast(v0) * __uint_as_float(b << 16);
      v1 = silu_fast(v1) * __uint_as_float(b & 0xffff0000u);
    }
  };
  float m0 = 0.f, m1 = 0.f;
#pragma unroll 4
  for (int r = r0; r < r1; ++r) {
    float v0, v1;
    load(r, v0, v1);
    m0 = fmaxf(m0, fabsf(v0));
    m1 = fmaxf(m1, fabsf(v1));
  }
  const float s0 = tile_scale(m0), s1 = tile_scale(m1);
#pragma unroll 4
  for (int r = r0; r < r1; ++r) {
    float v0, v1;
    load(r, v0, v1);
    const uint16_t pk = (uint16_t)to_e4m3(__fdiv_rn(v0, s0)) | ((uint16_t)to_e4m3(__fdiv_rn(v1, s1)) << 8);
    *reinterpret_cast<uint16_t*>(q + (size_t)r * cols + c) = pk;
  }
  *reinterpret_cast<float2*>(scale + (size_t)blk * cols + c) = make_float2(s0, s1);
}

}  // namespace

moe_status launch_block_table(const int32_t* offsets, int n_groups, int rows,
                              int32_t* block_start, cudaStream_t s) {
  block_table_kernel<<<1, 1024, 0, s>>>(offsets, n_groups, rows, block_start);
  return cuda_check(cudaGetLastError(), "block_table launch");
}

moe_status launch_quant_128x1(const void* x, int ldx, const int32_t* src_rows, bool swiglu_in,
                              int rows, int cols, const int32_t* offsets, int n_groups,
                              const int32_t* block_start, uint8_t* q, float* scale,
                              cudaStream_t s) {
  if (rows <= 0) return MOE_OK;
  const int G = offsets ? n_groups : 1;
  dim3 grid((rows + 127) / 128 + G, (cols + 255) / 256), block(128);
  auto X = static_cast<const __nv_bfloat16*>(x);
  if (swiglu_in)
    quant_128x1_kernel<true><<<grid, block, 0, s>>>(X, ldx, src_rows, rows, cols, offsets, G,
                                                    block_start, q, scale);
  else
    quant_128x1_kernel<false><<<grid, block, 0, s>>>(X, ldx, src_rows, rows, cols, offsets, G,
                                                     block_start, q, scale);
  return cuda_check(cudaGetLastError(), "quant_128x1 launch");
}

}  // namespace moe
