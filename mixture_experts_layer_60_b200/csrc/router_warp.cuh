// One token's routing by one warp, shared by the top-K kernel (logits from
// memory) and the fused router's epilogue (logits staged in shared memory):
// the affinity s = Sigmoid(x) of every expert, the K largest keys s + b
// (g'-equation of "DeepSeek-V3 技術報告", section 方法 / 2), optionally inside
// the best expert groups, the gates normalised from the unbiased s, the load
// histogram and the near-tie listing for the float64 tie-break.
//
// Lane l holds experts e = j*32 + l (j < V), read from x_row with coalesced
// loads.  K rounds of a warp-wide arg-max on order-preserving integer keys
// (two redux.sync reductions: the largest key, then the lowest expert id
// holding it) give the selection in the documented output order (key
// descending, lower index first on ties); lane k keeps the k-th winner
// (k < 32) so the gates are normalised and written from registers.  One
// more round measures the (K+1)-th key.
//
// Group limit (n_groups > 1, topk_groups < n_groups): experts form n_groups
// groups of N_r/n_groups consecutive indices; a group's score is its largest
// key s+b; only the topk_groups best groups (ties to the lower group index)
// stay eligible.  This is the per-token node limit of "DeepSeek V3 & R1
// 論文研究", section Cross-Node All-to-All; the score rule is this library's
// reading (the pages give only the limit).
//
// A token whose selection or order was decided by a key gap below refine_gap
// is listed: rl.tok / start / num get the token, its region of pair codes
// pair[t*N_r, t*N_r + num) the experts whose key lies within `near` of the
// keys of those close decisions (the span from the lowest to the highest of
// them), and, when logits_out is given, its logit row is copied there for
// the tie-break.  A decision between keys further apart than refine_gap is
// right in float32 as long as each key is within refine_gap / 2 of its
// float64 value; an expert further than `near` from every close key keeps
// that margin to the refined keys too.
#pragma once

#include "launch.h"

namespace moe {

// Order-preserving map of a float key to an unsigned integer (every real key
// maps above 0; -0 is taken as +0, so equal keys map to equal integers).
__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t b = __float_as_uint(f + 0.0f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord_float(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

template <int V>
__device__ __forceinline__ void route_token_warp(
    const float* x_row, const float* bias, int t, int N_r, int K, int n_groups, int topk_groups,
    float* wkeys, int32_t* __restrict__ idx, float* __restrict__ gate, int* hist,
    const RefineLists& rl, float refine_gap, float near, float* logits_out) {
  const int lane = threadIdx.x & 31;
  const bool grouped = n_groups > 1 && topk_groups < n_groups;
  float key[V], sv[V], kb[V], xv[V];
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int e = j * 32 + lane;
    if (e < N_r) {
      const float x = x_row[e];
      const float s = router_affinity(x);
      xv[j] = x;
      sv[j] = s;
      key[j] = s + bias[e];
    } else {
      xv[j] = 0.f;
      sv[j] = 0.f;
      key[j] = -INFINITY;
    }
    kb[j] = key[j];
  }
  // span of the keys of the decisions closer than refine_gap
  float close_lo = INFINITY, close_hi = -INFINITY;
  if (grouped) {
    const int gs = N_r / n_groups;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int e = j * 32 + lane;
      if (e < N_r) wkeys[e] = key[j];
    }
    __syncwarp();
    float gscore = -INFINITY;                       // lane g holds group g's score
    if (lane < n_groups)
      for (int i = 0; i < gs; ++i) gscore = fmaxf(gscore, wkeys[lane * gs + i]);
    __syncwarp();
    unsigned kept = 0;
    float last_kept = INFINITY;
    for (int r = 0; r <= topk_groups; ++r) {    // one extra round: the best excluded group
      float bk = (lane < n_groups && !((kept >> lane) & 1u)) ? gscore : -INFINITY;
      int bg = lane < n_groups && !((kept >> lane) & 1u) ? lane : 0x7fffffff;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
        const int og = __shfl_xor_sync(0xffffffffu, bg, off);
        if (ok > bk || (ok == bk && og < bg)) { bk = ok; bg = og; }
      }
      if (r < topk_groups) {
        kept |= 1u << bg;
        last_kept = bk;
      } else if (last_kept - bk < refine_gap) {   // kept vs excluded group scores
        close_lo = bk;
        close_hi = last_kept;
      }
    }
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int e = j * 32 + lane;
      if (e < N_r && !((kept >> (e / gs)) & 1u)) key[j] = -INFINITY;
    }
  }
  // K+1 rounds of a warp arg-max: each lane keeps the best of its own keys
  // (ties to the lower index), the warp takes the largest with one reduction
  // and the lowest expert id holding it with another; the winner's lane then
  // drops it (compared by expert id so that the arrays stay in registers) and
  // rescans its keys.
  uint32_t ko[V];
#pragma unroll
  for (int j = 0; j < V; ++j) ko[j] = j * 32 + lane < N_r ? ord_key(key[j]) : 0u;
  uint32_t lb = 0u;
  int lj = 0;
#pragma unroll
  for (int j = 0; j < V; ++j)
    if (ko[j] > lb) { lb = ko[j]; lj = j; }
  float sum = 0.f, prev = INFINITY;
  int my_e = 0;
  float my_s = 0.f;
  for (int k = 0; k <= K; ++k) {             // round K only measures the next key
    const uint32_t m = __reduce_max_sync(0xffffffffu, lb);
    if (m == 0u) break;                       // no key left (only after the K-th round)
    const int be = __reduce_min_sync(0xffffffffu, lb == m ? lj * 32 + lane : 0x7fffffff);
    const float bk = ord_float(m);
    if (prev - bk < refine_gap) {             // adjacent selected keys, and K-th vs next
      close_lo = fminf(close_lo, bk);
      close_hi = fmaxf(close_hi, prev);
    }
    prev = bk;
    if (k == K) break;
    float s_win = 0.f;
    uint32_t nb = 0u;
    int nj = 0;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (j * 32 + lane == be) { s_win = sv[j]; ko[j] = 0u; }
      if (ko[j] > nb) { nb = ko[j]; nj = j; }
    }
    lb = nb;
    lj = nj;
    s_win = __shfl_sync(0xffffffffu, s_win, be & 31);
    sum += s_win;
    if (k < 32) {
      if (lane == k) { my_e = be; my_s = s_win; }
    } else if (lane == 0) {
      idx[(size_t)t * K + k] = be;
      gate[(size_t)t * K + k] = s_win;
      atomicAdd(&hist[be], 1);
    }
  }
  if (lane < K) {
    idx[(size_t)t * K + lane] = my_e;
    gate[(size_t)t * K + lane] = my_s / sum;
    atomicAdd(&hist[my_e], 1);
  }
  if (K > 32) {
    __syncwarp();
    for (int k = 32 + lane; k < K; k += 32) {
      const size_t p = (size_t)t * K + k;
      gate[p] = gate[p] / sum;
    }
  }
  if (close_lo <= close_hi) {
    // the token, and every expert whose float32 key is within `near` of the
    // span of the close decisions' keys
    const float lo = close_lo - near, hi = close_hi + near;
    int c = 0;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (j * 32 + lane < N_r && kb[j] >= lo && kb[j] <= hi) ++c;
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == 0) {
      const int slot = atomicAdd(&rl.hdr[0], 1);
      rl.tok[slot] = t;
      rl.start[slot] = t * N_r;
      rl.num[slot] = total;
    }
    int w = t * N_r + incl - c;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int e = j * 32 + lane;
      if (e < N_r) {
        if (kb[j] >= lo && kb[j] <= hi) rl.pair[w++] = t * N_r + e;
        if (logits_out) logits_out[(size_t)t * N_r + e] = xv[j];
      }
    }
  }
}

}  // namespace moe
