// Row-gather pipeline for the per-token kernels that read K routed rows from
// random places in the grouped buffers (the combine of the h'-equation of
// "DeepSeek-V3 技術報告", section 方法 / 2, and its backward).  These kernels
// move whole 16-byte-aligned rows and do a few FMAs per element, so they are
// bound by how many bytes each SM keeps in flight: here four producer warps
// stage every row a step needs into shared memory with bulk asynchronous
// copies (a ring of stages, ~180 KB per SM; producer warp p fills the stages
// of the jobs j with j % 4 == p, spreading the per-copy issue cost that one
// warp alone is bound by), and four consumer warps do the arithmetic from
// shared memory.
//
// A job is (token t, column chunk q of 2 KB, or 1 KB / 512 B when a stage of
// many rows would leave fewer than eight stages).  Tokens go in groups of four, one
// per consumer warp, and a group's jobs are ordered chunk-major, so the four
// warps work side by side and every per-token reduction stays inside one warp
// (no block-wide barrier after the start).  Every wait is bounded (1 s) and
// reported through the device error word.
//
// Row slots of a job, by mode:
//   COMBINE      u_t, ys_j[t] (N_s), y_perm[r_k] (K)            -> h'_t
//   COMBINE_BWD  dh_t, u_t, y_perm[r_k] (K), e_idx(t,k) (K)      -> dy_perm[r_k], d_gate, d_logit
//   UNPERM_BWD   dh_t, dxs_j[t] (N_s), dx_perm[r_k] (K), e_k (K) -> du_t
// Sums are float32 in the same order as the per-warp kernels (residual or
// upstream row, shared rows j ascending, routed rows k ascending, centroid
// terms k ascending).  A slot whose grouped row lies outside [0, n_perm), or
// (backward) whose expert id lies outside [0, N_r), is left out: nothing is
// read for it and it takes no part in any sum.
#include <atomic>

#include "launch.h"
#include "sm100.cuh"

namespace moe {

namespace {

// Bound of the pipeline's stage waits (moe_set_pipeline_wait_limit).
constexpr uint64_t kDefaultWaitNs = 1000000000ull;
std::atomic<uint64_t> g_pipeline_wait_ns{kDefaultWaitNs};

using namespace sm100;

constexpr int kMaxChunk = 2048;              // bytes of a row per job (2048, 1024 or 512)
constexpr int kConsumerWarps = 4;            // one token of a group each
constexpr int kProducers = 4;               // 256 threads: at most 255 registers each
constexpr int kThreads = 32 * (kConsumerWarps + kProducers);
// the stage count is a multiple of kConsumerWarps, hence of kProducers
static_assert(kConsumerWarps % kProducers == 0, "one producer per stage");
constexpr int kSmemBudget = 200 * 1024;
constexpr int kMaxStages = 8;
constexpr int kMaxSlots = 64;              // two per lane of a producer warp
constexpr uint64_t kWaitNs = 1000000000ull;

struct GatherParams {
  const uint8_t* a;          // u (COMBINE) or dh (backward): row t
  const uint8_t* b;          // u (COMBINE_BWD): row t
  const uint8_t* sh;         // shared-expert rows [N_s][T] (ys or dxs)
  int N_s;
  const uint8_t* perm;       // grouped rows (y_perm or dx_perm)
  long long n_perm;          // rows of perm
  const uint8_t* cent;       // centroids E [N_r][d] (backward)
  int N_r;                   // rows of cent (backward)
  const int32_t* inv_row;    // [T, K]
  const int32_t* idx;        // [T, K] (backward), else nullptr
  const float* w;            // gate (COMBINE, COMBINE_BWD) or d_logit (UNPERM_BWD) [T, K]
  int T, K;
  long long row_bytes;
  uint8_t* out;              // h' / dy_perm / du
  float* d_gate;             // COMBINE_BWD outputs
  float* d_logit;
  float* d_logit_perm;
  int chunk;                 // bytes of a row per job
  int stages;                // a multiple of kConsumerWarps (see the ring below)
  uint64_t wait_ns;          // bound of every wait on a stage (the drain keeps kWaitNs)
  int* err;
};

__host__ __device__ inline int slots_of(int mode, int N_s, int K) {
  return mode == GATHER_COMBINE ? 1 + N_s + K : mode == GATHER_COMBINE_BWD ? 2 + 2 * K
                                                                           : 1 + N_s + 2 * K;
}

// Grouped row of slot k of token t, or -1 when the slot is left out: its row
// lies outside [0, n_perm) or, where expert ids are read (backward), its id
// lies outside [0, N_r).
__device__ __forceinline__ int slot_grouped_row(const GatherParams& p, int t, int k) {
  const int r = p.inv_row[(size_t)t * p.K + k];
  if (r < 0 || r >= p.n_perm) return -1;
  if (p.idx) {
    const int e = p.idx[(size_t)t * p.K + k];
    if (e < 0 || e >= p.N_r) return -1;
  }
  return r;
}

// Source row of slot `s` of token t, or nullptr (slot unused or left out).
template <int MODE>
__device__ __forceinline__ const uint8_t* slot_row(const GatherParams& p, int t, int s) {
  const int K = p.K, N_s = p.N_s;
  const size_t rb = (size_t)p.row_bytes;
  if (s == 0) return p.a + (size_t)t * rb;
  if (MODE == GATHER_COMBINE_BWD) {
    if (s == 1) return p.b + (size_t)t * rb;
    s -= 2;
  } else {
    if (s <= N_s) return p.sh + ((size_t)(s - 1) * p.T + t) * rb;
    s -= 1 + N_s;
  }
  if (s < K) {
    const int r = slot_grouped_row(p, t, s);
    return r >= 0 ? p.perm + (size_t)r * rb : nullptr;
  }
  s -= K;
  if (MODE != GATHER_COMBINE && s < K) {
    if (slot_grouped_row(p, t, s) < 0) return nullptr;
    return p.cent + (size_t)p.idx[(size_t)t * K + s] * rb;
  }
  return nullptr;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int MODE, typename E, int KMAX>
__global__ void __launch_bounds__(kThreads, 1) gather_pipe_kernel(const GatherParams p) {
  constexpr int N = Vec<E>::N;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* buf = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  const int K = p.K, N_s = p.N_s, S = p.stages, CH = p.chunk;
  const int R = slots_of(MODE, N_s, K);
  const int stage_bytes = R * CH;
  uint64_t* full = reinterpret_cast<uint64_t*>(buf + (size_t)S * stage_bytes);
  uint64_t* empty = full + S;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + S);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int Q = (int)((p.row_bytes + CH - 1) / CH);
  const int n_groups = (p.T + kConsumerWarps - 1) / kConsumerWarps;

  if (warp >= kConsumerWarps) {
    // ---------------------------------------------------------------- producers
    // Every producer walks the whole ring (stage and phase advance for every
    // job) and arms only its own jobs, so each stage (S is a multiple of
    // kProducers) has a single producer as well as a single consumer.
    const int pw = warp - kConsumerWarps;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    long long armed = 0;                // ring positions passed (every producer's jobs)
    for (int g = blockIdx.x; g < n_groups && ok; g += gridDim.x) {
      // this lane's slots (lane, lane + 32) of the group's four tokens
      const uint8_t* src[kConsumerWarps][2];
      int nvalid[kConsumerWarps];
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const int t = g * kConsumerWarps + w;
        const bool tv = t < p.T;
        src[w][0] = tv && lane < R ? slot_row<MODE>(p, t, lane) : nullptr;
        src[w][1] = tv && lane + 32 < R ? slot_row<MODE>(p, t, lane + 32) : nullptr;
        nvalid[w] = __popc(__ballot_sync(0xffffffffu, src[w][0] != nullptr)) +
                    __popc(__ballot_sync(0xffffffffu, src[w][1] != nullptr));
      }
      for (int q = 0; q < Q && ok; ++q) {
        const uint32_t cb = (uint32_t)min((long long)CH, p.row_bytes - (long long)q * CH);
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          if ((int)(armed % kProducers) != pw) {
            ++armed;
            if (++stage == S) { stage = 0; phase ^= 1; }
            continue;
          }
          bool got = true;
          if (lane == 0) got = mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.wait_ns);
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            if (lane == 0) { *abort_flag = 1; atomicOr(p.err, ERR_GATHER_TIMEOUT); }
            ok = false;
            break;
          }
          if (lane == 0) mbar_arrive_expect_tx(&full[stage], (uint32_t)nvalid[w] * cb);
          __syncwarp();
          uint8_t* dst = buf + (size_t)stage * stage_bytes;
          const size_t off = (size_t)q * CH;
          if (src[w][0]) bulk_load(dst + lane * CH, src[w][0] + off, cb, &full[stage]);
          if (src[w][1]) bulk_load(dst + (lane + 32) * CH, src[w][1] + off, cb, &full[stage]);
          ++armed;
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
    }
    // drain: no copy may still be writing shared memory when the block
    // exits.  Only the last S jobs can have copies in flight, and no later
    // job reused their stages, so each one's full barrier completes with the
    // job's own phase whether or not a consumer took it (after an abort the
    // consumers stop taking jobs).  One deadline bounds the whole drain.
    if (lane == 0) {
      const uint64_t t0 = globaltimer_ns();
      for (long long j = armed > S ? armed - S : 0; j < armed; ++j) {
        if ((int)(j % kProducers) != pw) continue;
        uint64_t* bar = &full[(int)(j % S)];
        const uint32_t par = (uint32_t)((j / S) & 1);
        while (!mbar_try_wait(bar, par) && globaltimer_ns() - t0 <= kWaitNs) {
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- consumers
    // warp w takes token w of every group; in a group its job of chunk q is
    // number 4q + w, so it skips the other warps' jobs in the ring.  S is a
    // multiple of kConsumerWarps, so job n's stage n % S is only ever used by
    // warp n % 4: each stage has one consumer, which takes its jobs in ring
    // order (the one-producer, one-consumer ring: a stage's barrier is never
    // more than one phase away from the job its consumer waits for).
    long long n = warp;                 // ring position of this warp's next job
    for (int g = blockIdx.x; g < n_groups; g += gridDim.x) {
      const int t = g * kConsumerWarps + warp;
      const bool tv = t < p.T;
      int rows[KMAX];
      float wk[KMAX], dg[KMAX], lg[KMAX];
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        rows[k] = -1;
        wk[k] = 0.f;
        dg[k] = 0.f;
        lg[k] = 0.f;
        if (tv && k < K) {
          rows[k] = slot_grouped_row(p, t, k);
          wk[k] = p.w[(size_t)t * K + k];
        }
      }
      bool ok = true;
      for (int q = 0; q < Q; ++q, n += kConsumerWarps) {
        const int stage = (int)(n % S);
        const uint32_t phase = (uint32_t)((n / S) & 1);
        const bool got = mbar_wait_bounded(&full[stage], phase, abort_flag, p.wait_ns);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) { *abort_flag = 1; atomicOr(p.err, ERR_GATHER_TIMEOUT); }
          ok = false;
          break;
        }
        if (tv) {
          const uint8_t* st = buf + (size_t)stage * stage_bytes;
          const long long cb = min((long long)CH, p.row_bytes - (long long)q * CH);
#pragma unroll
          for (int m = 0; m < kMaxChunk / 512; ++m) {
            const int cbyte = m * 512 + lane * 16;
            if (cbyte >= cb) break;
            const size_t gcol = (size_t)q * CH + cbyte;   // byte offset inside a row
            auto row = [&](int slot) {
              return *reinterpret_cast<const uint4*>(st + slot * CH + cbyte);
            };
            float acc[N], tmp[N];
            if (MODE == GATHER_COMBINE) {
              Vec<E>::load(row(0), acc);
              for (int j = 0; j < N_s; ++j) {
                Vec<E>::load(row(1 + j), tmp);
#pragma unroll
                for (int i = 0; i < N; ++i) acc[i] += tmp[i];
              }
#pragma unroll
              for (int k = 0; k < KMAX; ++k) {
                if (k < K && rows[k] >= 0) {
                  Vec<E>::load(row(1 + N_s + k), tmp);
#pragma unroll
                  for (int i = 0; i < N; ++i) acc[i] = fmaf(wk[k], tmp[i], acc[i]);
                }
              }
              *reinterpret_cast<uint4*>(p.out + (size_t)t * p.row_bytes + gcol) =
                  Vec<E>::store(acc);
            } else if (MODE == GATHER_COMBINE_BWD) {
              float fd[N], fu[N];
              Vec<E>::load(row(0), fd);
              Vec<E>::load(row(1), fu);
#pragma unroll
              for (int k = 0; k < KMAX; ++k) {
                if (k < K && rows[k] >= 0) {
                  Vec<E>::load(row(2 + k), tmp);
#pragma unroll
                  for (int i = 0; i < N; ++i) dg[k] = fmaf(fd[i], tmp[i], dg[k]);
#pragma unroll
                  for (int i = 0; i < N; ++i) tmp[i] = wk[k] * fd[i];
                  *reinterpret_cast<uint4*>(p.out + (size_t)rows[k] * p.row_bytes + gcol) =
                      Vec<E>::store(tmp);
                  Vec<E>::load(row(2 + K + k), tmp);
#pragma unroll
                  for (int i = 0; i < N; ++i) lg[k] = fmaf(fu[i], tmp[i], lg[k]);
                }
              }
            } else {
              Vec<E>::load(row(0), acc);
              for (int j = 0; j < N_s; ++j) {
                Vec<E>::load(row(1 + j), tmp);
#pragma unroll
                for (int i = 0; i < N; ++i) acc[i] += tmp[i];
              }
#pragma unroll
              for (int k = 0; k < KMAX; ++k) {
                if (k < K && rows[k] >= 0) {
                  Vec<E>::load(row(1 + N_s + k), tmp);
#pragma unroll
                  for (int i = 0; i < N; ++i) acc[i] += tmp[i];
                }
              }
#pragma unroll
              for (int k = 0; k < KMAX; ++k) {
                if (k < K && rows[k] >= 0) {
                  Vec<E>::load(row(1 + N_s + K + k), tmp);
#pragma unroll
                  for (int i = 0; i < N; ++i) acc[i] = fmaf(wk[k], tmp[i], acc[i]);
                }
              }
              *reinterpret_cast<uint4*>(p.out + (size_t)t * p.row_bytes + gcol) =
                  Vec<E>::store(acc);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
      }
      if (!ok) break;
      if (MODE == GATHER_COMBINE_BWD && tv) {
        // the token's gate and affinity gradients (selection held fixed):
        //   ds_k = (dg_k - sum_j g_j dg_j) / sum_j s_j,  dlogit_k = ds_k s_k (1 - s_k)
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
          if (k < K) {
            dg[k] = warp_sum(dg[k]);
            lg[k] = warp_sum(lg[k]);
          }
        }
        if (lane == 0) {
          // a left-out slot is not part of the selection: no s in the sum,
          // zero gradients
          float S_sum = 0.f, gdg = 0.f, sk[KMAX];
#pragma unroll
          for (int k = 0; k < KMAX; ++k) {
            sk[k] = 0.f;
            if (k < K && rows[k] >= 0) {
              sk[k] = 1.0f / (1.0f + expf(-lg[k]));
              S_sum += sk[k];
              gdg = fmaf(wk[k], dg[k], gdg);
            }
          }
#pragma unroll
          for (int k = 0; k < KMAX; ++k) {
            if (k < K) {
              const bool in = rows[k] >= 0;
              const float ds = (dg[k] - gdg) / S_sum;
              const float dl = in ? ds * sk[k] * (1.0f - sk[k]) : 0.f;
              p.d_gate[(size_t)t * K + k] = in ? dg[k] : 0.f;
              p.d_logit[(size_t)t * K + k] = dl;
              if (in) p.d_logit_perm[rows[k]] = dl;
            }
          }
        }
      }
    }
  }
}

template <int MODE, typename E, int KMAX>
moe_status pipe_launch(const GatherParams& p, size_t smem, int grid, cudaStream_t s) {
  auto kern = gather_pipe_kernel<MODE, E, KMAX>;
  static bool attr_done[kMaxSmemDevices] = {};
  // the attribute is set once per device: always the whole budget
  const moe_status st = ensure_max_smem(reinterpret_cast<const void*>(kern), kSmemBudget,
                                        attr_done, "gather pipeline smem attribute");
  if (st != MOE_OK) return st;
  kern<<<grid, kThreads, smem, s>>>(p);
  return cuda_check(cudaGetLastError(), "gather pipeline launch");
}

template <int MODE, typename E>
moe_status pipe_dispatch(const GatherParams& p, size_t smem, int grid, cudaStream_t s) {
  if (p.K <= 8) return pipe_launch<MODE, E, 8>(p, smem, grid, s);
  return pipe_launch<MODE, E, 16>(p, smem, grid, s);
}

}  // namespace

bool gather_pipe_supported(int mode, int N_s, int K, long long row_bytes) {
  return K >= 1 && K <= 16 && N_s >= 0 && row_bytes > 0 && row_bytes % 16 == 0 &&
         slots_of(mode, N_s, K) <= kMaxSlots;
}

moe_status launch_gather_pipe(int mode, moe_dtype dt, const void* a, const void* b,
                              const void* sh, int N_s, const void* perm, long long n_perm,
                              const void* cent, int N_r, const int32_t* inv_row,
                              const int32_t* idx, const float* w, int T, int K,
                              long long row_bytes, void* out, float* d_gate, float* d_logit,
                              float* d_logit_perm, cudaStream_t s) {
  if (T <= 0) return MOE_OK;
  GatherParams p;
  p.a = static_cast<const uint8_t*>(a);
  p.b = static_cast<const uint8_t*>(b);
  p.sh = static_cast<const uint8_t*>(sh);
  p.N_s = N_s;
  p.perm = static_cast<const uint8_t*>(perm);
  p.n_perm = n_perm;
  p.cent = static_cast<const uint8_t*>(cent);
  p.N_r = N_r;
  p.inv_row = inv_row;
  p.idx = mode == GATHER_COMBINE ? nullptr : idx;
  p.w = w;
  p.T = T;
  p.K = K;
  p.row_bytes = row_bytes;
  p.out = static_cast<uint8_t*>(out);
  p.d_gate = d_gate;
  p.d_logit = d_logit;
  p.d_logit_perm = d_logit_perm;
  p.err = device_error_word();
  if (!p.err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  p.wait_ns = g_pipeline_wait_ns.load(std::memory_order_relaxed);
  // a multiple of kConsumerWarps stages (one consumer warp per stage): the
  // largest chunk that fits kMaxStages of them, else the largest with four
  const int R = slots_of(mode, N_s, K);
  int chunk = 0, stages = 0;
  for (int c = kMaxChunk; c >= 512; c /= 2) {
    int st = (kSmemBudget - 1024) / (R * c) / kConsumerWarps * kConsumerWarps;
    if (st > kMaxStages) st = kMaxStages;
    if (st > stages) { stages = st; chunk = c; }
    if (stages == kMaxStages) break;
  }
  if (stages < kConsumerWarps)
    return fail(MOE_ERR_UNSUPPORTED, "gather pipeline: %d row slots", R);
  const int stage_bytes = R * chunk;
  p.chunk = chunk;
  p.stages = stages;
  const size_t smem = 128 + (size_t)stages * stage_bytes + (size_t)stages * 16 + 16;
  if (smem > (size_t)kSmemBudget) return fail(MOE_ERR_UNSUPPORTED, "gather pipeline: smem");
  const int n_groups = (T + kConsumerWarps - 1) / kConsumerWarps;
  int grid = sm_count();
  if (grid > n_groups) grid = n_groups;
  const bool f32 = dt == MOE_F32;
  switch (mode) {
    case GATHER_COMBINE:
      return f32 ? pipe_dispatch<GATHER_COMBINE, float>(p, smem, grid, s)
                 : pipe_dispatch<GATHER_COMBINE, __nv_bfloat16>(p, smem, grid, s);
    case GATHER_COMBINE_BWD:
      return f32 ? pipe_dispatch<GATHER_COMBINE_BWD, float>(p, smem, grid, s)
                 : pipe_dispatch<GATHER_COMBINE_BWD, __nv_bfloat16>(p, smem, grid, s);
    case GATHER_UNPERM_BWD:
      return f32 ? pipe_dispatch<GATHER_UNPERM_BWD, float>(p, smem, grid, s)
                 : pipe_dispatch<GATHER_UNPERM_BWD, __nv_bfloat16>(p, smem, grid, s);
  }
  return fail(MOE_ERR_INVALID_ARG, "gather pipeline: mode %d", mode);
}

}  // namespace moe

extern "C" moe_status moe_set_pipeline_wait_limit(unsigned long long ns) {
  moe::clear_last_error();
  moe::g_pipeline_wait_ns.store(ns ? (uint64_t)ns : moe::kDefaultWaitNs, std::memory_order_relaxed);
  return MOE_OK;
}
