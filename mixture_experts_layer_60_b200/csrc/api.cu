// extern "C" entry points of libmoe.so (declared in include/moe.h).  Each
// validates its arguments on the host, then enqueues kernels on `stream`.
#include "launch.h"

#include <atomic>

using namespace moe;

namespace {

constexpr int kAbiVersion = 2;

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline bool al16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

std::atomic<float> g_refine_gap{kRouterRefineGap};
std::atomic<float> g_near{kRouterNearBoundary};

int dtype_bytes(moe_dtype dt) {
  switch (dt) {
    case MOE_F32: return 4;
    case MOE_BF16: return 2;
    case MOE_E4M3: return 1;
  }
  return 0;
}

moe_status check_device() { return check_sm100(); }

#define MOE_REQUIRE(cond, status, ...) \
  do {                                 \
    if (!(cond)) return fail(status, __VA_ARGS__); \
  } while (0)

#define MOE_TRY(expr)                 \
  do {                                \
    moe_status _st = (expr);          \
    if (_st != MOE_OK) return _st;    \
  } while (0)

// Router workspace: float32 logits [T, N_r] (the fused router writes only
// the rows of listed tokens), then the tie-break lists: a 2-word header,
// tok/start/num [T] int32 and candidate pairs [T*N_r] int32.
size_t route_ws(int T, int N_r) {
  if (T <= 0 || N_r <= 0) return 0;
  const size_t tn = align_up((size_t)T * N_r * sizeof(float), 256);
  return tn + align_up((size_t)(2 + 3 * (size_t)T) * 4, 256) + tn;
}

RefineLists refine_lists(void* workspace, int T, int N_r) {
  const size_t tn = align_up((size_t)T * N_r * sizeof(float), 256);
  uint8_t* p = static_cast<uint8_t*>(workspace) + tn;
  RefineLists rl;
  rl.hdr = reinterpret_cast<int32_t*>(p);
  rl.tok = rl.hdr + 2;
  rl.start = rl.tok + T;
  rl.num = rl.start + T;
  p += align_up((size_t)(2 + 3 * (size_t)T) * 4, 256);
  rl.pair = reinterpret_cast<int32_t*>(p);
  return rl;
}

size_t ffn_ws(moe_dtype dt, int rows, int I) {
  if (rows <= 0 || I <= 0) return 0;
  switch (dt) {
    case MOE_F32: return align_up((size_t)rows * I * 4, 256);
    case MOE_BF16: return align_up((size_t)rows * I * 2, 256);
    case MOE_E4M3:
      return align_up((size_t)rows * I, 256) + align_up((size_t)rows * (I / 128) * 4, 256);
  }
  return 0;
}

}  // namespace

extern "C" {

int moe_abi_version(void) { return kAbiVersion; }

const char* moe_last_error(void) { return last_error_text(); }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
  }
  return "MOE_STATUS_UNKNOWN";
}

size_t moe_route_workspace_size(int T, int N_r) { return route_ws(T, N_r); }

moe_status moe_set_router_tie_break(float refine_gap, float near) {
  clear_last_error();
  MOE_REQUIRE(refine_gap >= 0.f && near >= 0.f, MOE_ERR_INVALID_ARG,
              "moe_set_router_tie_break: gap %g and near %g must be >= 0", refine_gap, near);
  const bool deflt = refine_gap == 0.f && near == 0.f;
  g_refine_gap.store(deflt ? kRouterRefineGap : refine_gap);
  g_near.store(deflt ? kRouterNearBoundary : near);
  return MOE_OK;
}

}  // extern "C"

namespace moe {
void router_tie_break(float* refine_gap, float* near) {
  *refine_gap = g_refine_gap.load();
  *near = g_near.load();
}
}  // namespace moe

namespace {

moe_status route_impl(const char* who, const void* u, const void* E, moe_dtype dt, const float* b,
                      int T, int d, int N_r, int K, int n_groups, int topk_groups,
                      int32_t* topk_idx, float* topk_gate, int32_t* counts, void* workspace,
                      size_t workspace_bytes, void* stream) {
  clear_last_error();
  MOE_REQUIRE(dt == MOE_F32 || dt == MOE_BF16, MOE_ERR_UNSUPPORTED,
              "%s: dtype must be MOE_F32 or MOE_BF16", who);
  MOE_REQUIRE(T >= 0 && d > 0 && N_r > 0 && K > 0, MOE_ERR_INVALID_ARG,
              "%s: bad sizes T=%d d=%d N_r=%d K=%d", who, T, d, N_r, K);
  MOE_REQUIRE(N_r <= 1024 && K <= N_r, MOE_ERR_UNSUPPORTED,
              "%s: need 1 <= K <= N_r <= 1024 (K=%d N_r=%d)", who, K, N_r);
  MOE_REQUIRE(n_groups >= 1 && n_groups <= 32 && N_r % n_groups == 0 && topk_groups >= 1 &&
                  topk_groups <= n_groups,
              MOE_ERR_INVALID_ARG,
              "%s: need 1 <= topk_groups <= n_groups <= 32 with N_r %% n_groups == 0", who);
  MOE_REQUIRE((long long)topk_groups * (N_r / n_groups) >= K, MOE_ERR_INVALID_ARG,
              "%s: the kept groups hold fewer than K experts", who);
  MOE_REQUIRE(d % 64 == 0, MOE_ERR_UNSUPPORTED, "%s: d=%d must be a multiple of 64", who, d);
  MOE_REQUIRE((long long)d * dtype_bytes(dt) <= 32768, MOE_ERR_UNSUPPORTED,
              "%s: a row of u is at most 32 KB (d=%d)", who, d);
  MOE_REQUIRE((long long)T * N_r <= 0x7fffffffLL, MOE_ERR_UNSUPPORTED,
              "%s: T * N_r must fit in 31 bits (T=%d N_r=%d)", who, T, N_r);
  MOE_REQUIRE(E && b && counts, MOE_ERR_INVALID_ARG, "%s: null pointer", who);
  MOE_REQUIRE(T == 0 || (u && topk_idx && topk_gate && workspace), MOE_ERR_INVALID_ARG,
              "%s: null pointer", who);
  MOE_REQUIRE(workspace_bytes >= route_ws(T, N_r), MOE_ERR_WORKSPACE,
              "%s: workspace %zu < %zu bytes", who, workspace_bytes, route_ws(T, N_r));
  MOE_REQUIRE(T == 0 || reinterpret_cast<uintptr_t>(workspace) % 256 == 0, MOE_ERR_INVALID_ARG,
              "%s: workspace must be 256-byte aligned", who);
  MOE_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  MOE_TRY(cuda_check(cudaMemsetAsync(counts, 0, (size_t)N_r * sizeof(int32_t), s), "zero counts"));
  if (T == 0) return MOE_OK;
  float* logits = static_cast<float*>(workspace);
  const RefineLists rl = refine_lists(workspace, T, N_r);
  MOE_TRY(cuda_check(cudaMemsetAsync(rl.hdr, 0, 2 * sizeof(int32_t), s), "zero tie-break lists"));
  float gap, near;
  router_tie_break(&gap, &near);
  if (router_tc_supported(dt, d, N_r, K, n_groups, topk_groups)) {
    MOE_TRY(launch_router_tc(u, E, b, T, d, N_r, K, n_groups, topk_groups, topk_idx, topk_gate,
                             counts, logits, rl, gap, near, s));
  } else {
    if (dt == MOE_BF16 && N_r % 64 == 0)
      MOE_TRY(launch_tc_gemm(u, E, N_r, nullptr, 1, T, N_r, d, TC_EPI_STORE_F32, logits, s));
    else
      MOE_TRY(launch_logits_simt(u, E, dt, T, d, N_r, logits, s));
    MOE_TRY(launch_topk(logits, b, T, N_r, K, n_groups, topk_groups, topk_idx, topk_gate, counts,
                        rl, gap, near, s));
  }
  return launch_refine(u, E, dt, logits, b, d, N_r, K, n_groups, topk_groups, rl, near, T,
                       topk_idx, topk_gate, counts, s);
}

}  // namespace

extern "C" {

moe_status moe_route(const void* u, const void* E, moe_dtype dt, const float* b, int T, int d,
                     int N_r, int K, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return route_impl("moe_route", u, E, dt, b, T, d, N_r, K, 1, 1, topk_idx, topk_gate, counts,
                    workspace, workspace_bytes, stream);
}

moe_status moe_route_grouped(const void* u, const void* E, moe_dtype dt, const float* b, int T,
                             int d, int N_r, int K, int n_groups, int topk_groups,
                             int32_t* topk_idx, float* topk_gate, int32_t* counts,
                             void* workspace, size_t workspace_bytes, void* stream) {
  return route_impl("moe_route_grouped", u, E, dt, b, T, d, N_r, K, n_groups, topk_groups,
                    topk_idx, topk_gate, counts, workspace, workspace_bytes, stream);
}

size_t moe_permute_workspace_size(int T, int N_r) {
  if (T <= 0 || N_r <= 0) return 0;
  return permute_ws_bytes(T, N_r);
}

}  // extern "C"

namespace moe {

moe_status validate_permute_args(const char* who, const void* u, const float* u_scale,
                                 moe_dtype dt, const int32_t* topk_idx, int T, int d, int N_r,
                                 int K, const void* x_perm, const float* x_scale,
                                 const int32_t* offsets, const int32_t* perm_src,
                                 const int32_t* inv_row, int* elem_bytes) {
  const int eb = dtype_bytes(dt);
  MOE_REQUIRE(eb > 0, MOE_ERR_UNSUPPORTED, "%s: unknown dtype %d", who, (int)dt);
  MOE_REQUIRE(T >= 0 && d > 0 && N_r > 0 && K > 0, MOE_ERR_INVALID_ARG,
              "%s: bad sizes T=%d d=%d N_r=%d K=%d", who, T, d, N_r, K);
  MOE_REQUIRE(N_r <= 1024 && K <= N_r, MOE_ERR_UNSUPPORTED, "%s: need 1 <= K <= N_r <= 1024",
              who);
  MOE_REQUIRE(((size_t)d * eb) % 16 == 0, MOE_ERR_UNSUPPORTED,
              "%s: a row (%d x %d bytes) must be a multiple of 16 bytes", who, d, eb);
  MOE_REQUIRE(offsets, MOE_ERR_INVALID_ARG, "%s: null offsets", who);
  MOE_REQUIRE(T == 0 || (u && topk_idx && x_perm && perm_src && inv_row), MOE_ERR_INVALID_ARG,
              "%s: null pointer", who);
  if (dt == MOE_E4M3) {
    MOE_REQUIRE(d % 128 == 0, MOE_ERR_UNSUPPORTED, "%s: e4m3 needs d %% 128 == 0", who);
    MOE_REQUIRE(T == 0 || (u_scale && x_scale), MOE_ERR_INVALID_ARG,
                "%s: e4m3 needs u_scale and x_scale", who);
  } else {
    MOE_REQUIRE(!u_scale && !x_scale, MOE_ERR_INVALID_ARG, "%s: scales are only for MOE_E4M3",
                who);
  }
  MOE_REQUIRE(reinterpret_cast<uintptr_t>(u) % 16 == 0 &&
                  reinterpret_cast<uintptr_t>(x_perm) % 16 == 0,
              MOE_ERR_INVALID_ARG, "%s: u and x_perm must be 16-byte aligned", who);
  *elem_bytes = eb;
  return MOE_OK;
}

}  // namespace moe

extern "C" {

moe_status moe_permute(const void* u, const float* u_scale, moe_dtype dt, const int32_t* topk_idx,
                       int T, int d, int N_r, int K, void* x_perm, float* x_scale,
                       int32_t* offsets, int32_t* perm_src, int32_t* inv_row, void* workspace,
                       size_t workspace_bytes, void* stream) {
  clear_last_error();
  int eb = 0;
  MOE_TRY(validate_permute_args("moe_permute", u, u_scale, dt, topk_idx, T, d, N_r, K, x_perm,
                                x_scale, offsets, perm_src, inv_row, &eb));
  MOE_REQUIRE(T == 0 || workspace, MOE_ERR_INVALID_ARG, "moe_permute: null workspace");
  MOE_REQUIRE(workspace_bytes >= moe_permute_workspace_size(T, N_r), MOE_ERR_WORKSPACE,
              "moe_permute: workspace %zu < %zu bytes", workspace_bytes,
              moe_permute_workspace_size(T, N_r));
  MOE_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  if (T == 0)
    return cuda_check(cudaMemsetAsync(offsets, 0, (size_t)(N_r + 1) * sizeof(int32_t), s),
                      "zero offsets");
  return launch_permute(u, dt == MOE_E4M3 ? u_scale : nullptr, eb, topk_idx, T, d, N_r, K, x_perm,
                        dt == MOE_E4M3 ? x_scale : nullptr, offsets, perm_src, inv_row, workspace,
                        s);
}

moe_status moe_permute_index(const int32_t* topk_idx, int T, int N_r, int K, int32_t* offsets,
                             int32_t* perm_src, int32_t* inv_row, void* workspace,
                             size_t workspace_bytes, void* stream) {
  clear_last_error();
  const char* who = "moe_permute_index";
  MOE_REQUIRE(T >= 0 && N_r > 0 && K > 0, MOE_ERR_INVALID_ARG, "%s: bad sizes T=%d N_r=%d K=%d",
              who, T, N_r, K);
  MOE_REQUIRE(N_r <= 1024 && K <= N_r, MOE_ERR_UNSUPPORTED, "%s: need 1 <= K <= N_r <= 1024",
              who);
  MOE_REQUIRE(offsets, MOE_ERR_INVALID_ARG, "%s: null offsets", who);
  MOE_REQUIRE(T == 0 || (topk_idx && perm_src && inv_row && workspace), MOE_ERR_INVALID_ARG,
              "%s: null pointer", who);
  MOE_REQUIRE(workspace_bytes >= moe_permute_workspace_size(T, N_r), MOE_ERR_WORKSPACE,
              "%s: workspace %zu < %zu bytes", who, workspace_bytes,
              moe_permute_workspace_size(T, N_r));
  MOE_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  if (T == 0)
    return cuda_check(cudaMemsetAsync(offsets, 0, (size_t)(N_r + 1) * sizeof(int32_t), s),
                      "zero offsets");
  return launch_permute(nullptr, nullptr, 0, topk_idx, T, 0, N_r, K, nullptr, nullptr, offsets,
                        perm_src, inv_row, workspace, s);
}

size_t moe_expert_ffn_workspace_size(moe_dtype dt, int rows, int I) { return ffn_ws(dt, rows, I); }

namespace {

moe_status check_ffn_common(const char* who, const void* x, const int32_t* offsets, int n_groups,
                            int rows, int d, int I, moe_dtype dt, const void* W) {
  MOE_REQUIRE(dtype_bytes(dt) > 0, MOE_ERR_UNSUPPORTED, "%s: unknown dtype", who);
  MOE_REQUIRE(rows >= 0 && d > 0 && I > 0 && n_groups > 0, MOE_ERR_INVALID_ARG,
              "%s: bad sizes rows=%d d=%d I=%d n_groups=%d", who, rows, d, I, n_groups);
  MOE_REQUIRE(n_groups <= 1024, MOE_ERR_UNSUPPORTED, "%s: at most 1024 groups", who);
  MOE_REQUIRE(d % 128 == 0 && I % 128 == 0, MOE_ERR_UNSUPPORTED,
              "%s: d=%d and I=%d must be multiples of 128", who, d, I);
  MOE_REQUIRE(offsets && W, MOE_ERR_INVALID_ARG, "%s: null pointer", who);
  MOE_REQUIRE(rows == 0 || x, MOE_ERR_INVALID_ARG, "%s: null pointer", who);
  return MOE_OK;
}

moe_status run_gate_up(const void* x, const float* x_scale, const int32_t* offsets, int n_groups,
                       int rows, int d, int I, moe_dtype dt, const void* W_gate_up,
                       const float* w_scale_gate_up, void* h, float* h_scale, cudaStream_t s) {
  if (dt == MOE_F32)
    return launch_simt_gemm(x, W_gate_up, 2LL * I * d, offsets, n_groups, rows, I, d, true,
                            MOE_F32, h, MOE_F32, s);
  if (dt == MOE_BF16)
    return launch_ws_gemm(x, W_gate_up, 2 * I, offsets, n_groups, rows, I, d, true, h, s);
  return launch_fp8_gemm(x, x_scale, W_gate_up, w_scale_gate_up, 2 * I, offsets, n_groups, rows,
                         I, d, true, h, h_scale, s);
}

moe_status run_down(const void* h, const float* h_scale, const int32_t* offsets, int n_groups,
                    int rows, int d, int I, moe_dtype dt, const void* W_down,
                    const float* w_scale_down, void* y, cudaStream_t s) {
  if (dt == MOE_F32)
    return launch_simt_gemm(h, W_down, (long long)d * I, offsets, n_groups, rows, d, I, false,
                            MOE_F32, y, MOE_F32, s);
  if (dt == MOE_BF16) {
    if (d % 256 == 0)
      return launch_ws_gemm(h, W_down, d, offsets, n_groups, rows, d, I, false, y, s);
    return launch_tc_gemm(h, W_down, d, offsets, n_groups, rows, d, I, TC_EPI_STORE_BF16, y, s);
  }
  return launch_fp8_gemm(h, h_scale, W_down, w_scale_down, d, offsets, n_groups, rows, d, I,
                         false, y, nullptr, s);
}

moe_status check_scales(const char* who, moe_dtype dt, const void* a, const void* b) {
  if (dt == MOE_E4M3)
    MOE_REQUIRE(a && b, MOE_ERR_INVALID_ARG, "%s: e4m3 needs activation and weight scales", who);
  else
    MOE_REQUIRE(!a && !b, MOE_ERR_INVALID_ARG, "%s: scales are only for MOE_E4M3", who);
  return MOE_OK;
}

}  // namespace

moe_status moe_expert_ffn(const void* x, const float* x_scale, const int32_t* offsets,
                          int n_groups, int rows, int d, int I, moe_dtype dt,
                          const void* W_gate_up, const float* w_scale_gate_up,
                          const void* W_down, const float* w_scale_down, void* y,
                          void* workspace, size_t workspace_bytes, void* stream) {
  clear_last_error();
  MOE_TRY(check_ffn_common("moe_expert_ffn", x, offsets, n_groups, rows, d, I, dt, W_gate_up));
  MOE_REQUIRE(W_down, MOE_ERR_INVALID_ARG, "moe_expert_ffn: null pointer");
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(y && workspace, MOE_ERR_INVALID_ARG, "moe_expert_ffn: null pointer");
  MOE_TRY(check_scales("moe_expert_ffn", dt, x_scale, w_scale_gate_up));
  MOE_TRY(check_scales("moe_expert_ffn", dt, x_scale, w_scale_down));
  MOE_REQUIRE(workspace_bytes >= ffn_ws(dt, rows, I), MOE_ERR_WORKSPACE,
              "moe_expert_ffn: workspace %zu < %zu bytes", workspace_bytes, ffn_ws(dt, rows, I));
  MOE_REQUIRE(reinterpret_cast<uintptr_t>(workspace) % 256 == 0 &&
                  reinterpret_cast<uintptr_t>(y) % 16 == 0,
              MOE_ERR_INVALID_ARG, "moe_expert_ffn: workspace 256-byte and y 16-byte alignment");
  MOE_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  void* h = workspace;
  float* hs = dt == MOE_E4M3
                  ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                             align_up((size_t)rows * I, 256))
                  : nullptr;
  MOE_TRY(run_gate_up(x, x_scale, offsets, n_groups, rows, d, I, dt, W_gate_up, w_scale_gate_up, h,
                      hs, s));
  return run_down(h, hs, offsets, n_groups, rows, d, I, dt, W_down, w_scale_down, y, s);
}

moe_status moe_expert_gate_up(const void* x, const float* x_scale, const int32_t* offsets,
                              int n_groups, int rows, int d, int I, moe_dtype dt,
                              const void* W_gate_up, const float* w_scale_gate_up, void* h,
                              float* h_scale, void* stream) {
  clear_last_error();
  MOE_TRY(check_ffn_common("moe_expert_gate_up", x, offsets, n_groups, rows, d, I, dt, W_gate_up));
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(h, MOE_ERR_INVALID_ARG, "moe_expert_gate_up: null h");
  MOE_TRY(check_scales("moe_expert_gate_up", dt, x_scale, w_scale_gate_up));
  MOE_REQUIRE(dt != MOE_E4M3 || h_scale, MOE_ERR_INVALID_ARG, "moe_expert_gate_up: null h_scale");
  MOE_REQUIRE(dt == MOE_E4M3 || !h_scale, MOE_ERR_INVALID_ARG,
              "moe_expert_gate_up: h_scale is only for MOE_E4M3");
  MOE_REQUIRE(reinterpret_cast<uintptr_t>(h) % 16 == 0, MOE_ERR_INVALID_ARG,
              "moe_expert_gate_up: h must be 16-byte aligned");
  MOE_TRY(check_device());
  return run_gate_up(x, x_scale, offsets, n_groups, rows, d, I, dt, W_gate_up, w_scale_gate_up, h,
                     h_scale, as_stream(stream));
}

moe_status moe_expert_down(const void* h, const float* h_scale, const int32_t* offsets,
                           int n_groups, int rows, int d, int I, moe_dtype dt, const void* W_down,
                           const float* w_scale_down, void* y, void* stream) {
  clear_last_error();
  MOE_TRY(check_ffn_common("moe_expert_down", h, offsets, n_groups, rows, d, I, dt, W_down));
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(y, MOE_ERR_INVALID_ARG, "moe_expert_down: null y");
  MOE_TRY(check_scales("moe_expert_down", dt, h_scale, w_scale_down));
  MOE_REQUIRE(reinterpret_cast<uintptr_t>(y) % 16 == 0 &&
                  reinterpret_cast<uintptr_t>(h) % 16 == 0,
              MOE_ERR_INVALID_ARG, "moe_expert_down: h and y must be 16-byte aligned");
  MOE_TRY(check_device());
  return run_down(h, h_scale, offsets, n_groups, rows, d, I, dt, W_down, w_scale_down, y,
                  as_stream(stream));
}

namespace {

moe_status check_shared_common(const char* who, const int32_t* offsets, int n_groups, int rows,
                               int T, int N_s, int d, int I, const void* W, const void* Ws,
                               const void* out) {
  MOE_REQUIRE(rows >= 0 && T >= 0 && N_s >= 0 && d > 0 && I > 0 && n_groups > 0,
              MOE_ERR_INVALID_ARG, "%s: bad sizes rows=%d T=%d N_s=%d d=%d I=%d n_groups=%d", who,
              rows, T, N_s, d, I, n_groups);
  MOE_REQUIRE(n_groups <= 1024, MOE_ERR_UNSUPPORTED, "%s: at most 1024 groups", who);
  MOE_REQUIRE(d % 256 == 0 && I % 128 == 0, MOE_ERR_UNSUPPORTED,
              "%s: d=%d must be a multiple of 256 and I=%d of 128", who, d, I);
  MOE_REQUIRE((long long)rows + (long long)N_s * T < (1LL << 31), MOE_ERR_UNSUPPORTED,
              "%s: rows + N_s*T must fit in 31 bits", who);
  MOE_REQUIRE(offsets && W && out && (N_s == 0 || Ws), MOE_ERR_INVALID_ARG, "%s: null pointer",
              who);
  MOE_REQUIRE(al16(out), MOE_ERR_INVALID_ARG, "%s: outputs must be 16-byte aligned", who);
  return MOE_OK;
}

}  // namespace

moe_status moe_expert_gate_up_shared(const void* x, const int32_t* offsets, int n_groups,
                                     int rows, const void* u, int T, int N_s, int d, int I,
                                     const void* W_gate_up, const void* Ws_gate_up, void* h,
                                     void* stream) {
  clear_last_error();
  const char* who = "moe_expert_gate_up_shared";
  MOE_TRY(check_shared_common(who, offsets, n_groups, rows, T, N_s, d, I, W_gate_up, Ws_gate_up,
                              h));
  MOE_REQUIRE(rows == 0 || x, MOE_ERR_INVALID_ARG, "%s: null x", who);
  MOE_REQUIRE(N_s == 0 || T == 0 || u, MOE_ERR_INVALID_ARG, "%s: null u", who);
  MOE_REQUIRE(al16(x) && al16(u), MOE_ERR_INVALID_ARG, "%s: x and u must be 16-byte aligned", who);
  if (rows == 0 && (N_s == 0 || T == 0)) return MOE_OK;
  MOE_TRY(check_device());
  WsExtraGroups ex;
  ex.X = u;
  ex.W = Ws_gate_up;
  ex.n_extra = T > 0 ? N_s : 0;
  ex.T = T;
  ex.x_local = true;
  // a routed buffer of no rows still needs a valid tensor map: use u's
  return launch_ws_gemm(rows ? x : u, W_gate_up, 2 * I, offsets, n_groups, rows, I, d, true, h,
                        as_stream(stream), &ex);
}

moe_status moe_expert_down_shared(const void* h, const int32_t* offsets, int n_groups, int rows,
                                  int T, int N_s, int d, int I, const void* W_down,
                                  const void* Ws_down, void* y, void* stream) {
  clear_last_error();
  const char* who = "moe_expert_down_shared";
  MOE_TRY(check_shared_common(who, offsets, n_groups, rows, T, N_s, d, I, W_down, Ws_down, y));
  MOE_REQUIRE(h && al16(h), MOE_ERR_INVALID_ARG, "%s: h null or misaligned", who);
  if (rows == 0 && (N_s == 0 || T == 0)) return MOE_OK;
  MOE_TRY(check_device());
  WsExtraGroups ex;
  ex.X = h;
  ex.W = Ws_down;
  ex.n_extra = T > 0 ? N_s : 0;
  ex.T = T;
  ex.x_local = false;
  return launch_ws_gemm(h, W_down, d, offsets, n_groups, rows, d, I, false, y, as_stream(stream),
                        &ex);
}

moe_status moe_combine(const void* u, const void* y_shared, int N_s, const void* y_perm,
                       const int32_t* inv_row, const float* topk_gate, moe_dtype dt, int T, int d,
                       int K, void* h_out, void* stream) {
  clear_last_error();
  MOE_REQUIRE(dt == MOE_F32 || dt == MOE_BF16, MOE_ERR_UNSUPPORTED,
              "moe_combine: dtype must be MOE_F32 or MOE_BF16");
  MOE_REQUIRE(T >= 0 && d > 0 && K > 0 && N_s >= 0, MOE_ERR_INVALID_ARG,
              "moe_combine: bad sizes T=%d d=%d K=%d N_s=%d", T, d, K, N_s);
  MOE_REQUIRE(((size_t)d * dtype_bytes(dt)) % 16 == 0, MOE_ERR_UNSUPPORTED,
              "moe_combine: a row must be a multiple of 16 bytes");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(u && y_perm && inv_row && topk_gate && h_out && (N_s == 0 || y_shared),
              MOE_ERR_INVALID_ARG, "moe_combine: null pointer");
  MOE_REQUIRE(reinterpret_cast<uintptr_t>(u) % 16 == 0 &&
                  reinterpret_cast<uintptr_t>(y_perm) % 16 == 0 &&
                  reinterpret_cast<uintptr_t>(h_out) % 16 == 0 &&
                  reinterpret_cast<uintptr_t>(y_shared) % 16 == 0,
              MOE_ERR_INVALID_ARG, "moe_combine: rows must be 16-byte aligned");
  MOE_TRY(check_device());
  return launch_combine(u, y_shared, N_s, y_perm, inv_row, topk_gate, dt, T, d, K, h_out,
                        as_stream(stream));
}

moe_status moe_bias_update(float* b, const int32_t* counts, int N_r, int T, int K, float gamma,
                           void* stream) {
  clear_last_error();
  MOE_REQUIRE(b && counts, MOE_ERR_INVALID_ARG, "moe_bias_update: null pointer");
  MOE_REQUIRE(N_r > 0 && T >= 0 && K > 0, MOE_ERR_INVALID_ARG,
              "moe_bias_update: bad sizes N_r=%d T=%d K=%d", N_r, T, K);
  MOE_TRY(check_device());
  return launch_bias_update(b, counts, N_r, T, K, gamma, as_stream(stream));
}

moe_status moe_quantize_1x128(const void* x, int rows, int cols, uint8_t* q, float* scale,
                              void* stream) {
  clear_last_error();
  MOE_REQUIRE(rows >= 0 && cols > 0 && cols % 128 == 0, MOE_ERR_UNSUPPORTED,
              "moe_quantize_1x128: cols=%d must be a positive multiple of 128", cols);
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(x && q && scale, MOE_ERR_INVALID_ARG, "moe_quantize_1x128: null pointer");
  MOE_REQUIRE(reinterpret_cast<uintptr_t>(x) % 16 == 0 && reinterpret_cast<uintptr_t>(q) % 16 == 0,
              MOE_ERR_INVALID_ARG, "moe_quantize_1x128: x and q must be 16-byte aligned");
  MOE_TRY(check_device());
  return launch_quant_1x128(x, rows, cols, q, scale, as_stream(stream));
}

moe_status moe_quantize_128x128(const void* w, int groups, int rows, int cols, uint8_t* q,
                                float* scale, void* stream) {
  clear_last_error();
  MOE_REQUIRE(groups >= 0 && rows > 0 && cols > 0 && rows % 128 == 0 && cols % 128 == 0,
              MOE_ERR_UNSUPPORTED, "moe_quantize_128x128: rows=%d cols=%d must be multiples of 128",
              rows, cols);
  if (groups == 0) return MOE_OK;
  MOE_REQUIRE(w && q && scale, MOE_ERR_INVALID_ARG, "moe_quantize_128x128: null pointer");
  MOE_REQUIRE(reinterpret_cast<uintptr_t>(w) % 16 == 0 && reinterpret_cast<uintptr_t>(q) % 16 == 0,
              MOE_ERR_INVALID_ARG, "moe_quantize_128x128: w and q must be 16-byte aligned");
  MOE_TRY(check_device());
  return launch_quant_128x128(w, groups, rows, cols, q, scale, as_stream(stream));
}

// ---------------------------------------------------------------- backward

namespace {


// Backward workspace.  bf16: dA [rows, 2I] bf16.  e4m3: the FP8 operands of
// the two Dgrads and two Wgrads and their scales (see fp8_bwd_layout).
struct Fp8BwdLayout {
  size_t dy_q, dy_s, dA_q, dA_s, dA_bf, blk, dyT_q, dyT_s, hT_q, hT_s, dAT_q, dAT_s, xT_q, xT_s,
      tail, total;
};
Fp8BwdLayout fp8_bwd_layout(int rows, int d, int I, int G) {
  Fp8BwdLayout L;
  const size_t R = (size_t)rows, nb = (size_t)(rows + 127) / 128 + G;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = align_up(o + bytes, 256); return at; };
  L.dy_q = take(R * d);
  L.dy_s = take(R * (d / 128) * 4);
  L.dA_q = take(R * 2 * I);
  L.dA_s = take(R * (2 * I / 128) * 4);
  L.dA_bf = take(R * 2 * I * 2);
  L.blk = take((size_t)(G + 1) * 4);
  L.dyT_q = take(R * d);
  L.dyT_s = take(nb * d * 4);
  L.hT_q = take(R * I);
  L.hT_s = take(nb * I * 4);
  L.dAT_q = take(R * 2 * I);
  L.dAT_s = take(nb * 2 * I * 4);
  L.xT_q = take(R * d);
  L.xT_s = take(nb * d * 4);
  L.tail = take(wgrad_tail_bytes((size_t)(d > 2 * I ? d : 2 * I), 128, G));   // Wgrad A tails
  L.total = o;
  return L;
}

size_t ffn_bwd_ws(moe_dtype dt, int rows, int d, int I, int G) {
  if (rows <= 0 || I <= 0 || d <= 0 || G <= 0) return 0;
  if (dt == MOE_BF16)   // dA, then the Wgrad A operand's tail blocks
    return align_up((size_t)rows * 2 * I * 2, 256) +
           wgrad_tail_bytes((size_t)(d > 2 * I ? d : 2 * I) * 2, 64, G);
  if (dt == MOE_E4M3) return fp8_bwd_layout(rows, d, I, G).total;
  return 0;
}

moe_status check_rowwise(const char* who, moe_dtype dt, int T, int d, int K) {
  MOE_REQUIRE(dt == MOE_F32 || dt == MOE_BF16, MOE_ERR_UNSUPPORTED,
              "%s: dtype must be MOE_F32 or MOE_BF16", who);
  MOE_REQUIRE(T >= 0 && d > 0 && K > 0, MOE_ERR_INVALID_ARG, "%s: bad sizes T=%d d=%d K=%d", who,
              T, d, K);
  MOE_REQUIRE(K <= 16, MOE_ERR_UNSUPPORTED, "%s: K=%d > 16", who, K);
  MOE_REQUIRE(((size_t)d * dtype_bytes(dt)) % 16 == 0, MOE_ERR_UNSUPPORTED,
              "%s: a row must be a multiple of 16 bytes", who);
  return MOE_OK;
}

}  // namespace

moe_status moe_expert_gate_up_save(const void* x, const float* x_scale, const int32_t* offsets,
                                   int n_groups, int rows, int d, int I, moe_dtype dt,
                                   const void* W_gate_up, const float* w_scale_gate_up, void* h,
                                   float* h_scale, void* a_gu, void* stream) {
  clear_last_error();
  const char* who = "moe_expert_gate_up_save";
  MOE_TRY(check_ffn_common(who, x, offsets, n_groups, rows, d, I, dt, W_gate_up));
  MOE_REQUIRE(dt == MOE_BF16 || dt == MOE_E4M3, MOE_ERR_UNSUPPORTED,
              "%s: MOE_BF16 or MOE_E4M3 only", who);
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(h && a_gu, MOE_ERR_INVALID_ARG, "%s: null pointer", who);
  MOE_TRY(check_scales(who, dt, x_scale, w_scale_gate_up));
  MOE_REQUIRE((dt == MOE_E4M3) == (h_scale != nullptr), MOE_ERR_INVALID_ARG,
              "%s: h_scale is required for MOE_E4M3 and only for it", who);
  MOE_REQUIRE(al16(h) && al16(a_gu) && al16(x), MOE_ERR_INVALID_ARG,
              "%s: x, h and a_gu must be 16-byte aligned", who);
  MOE_TRY(check_device());
  if (dt == MOE_E4M3)
    return launch_fp8_gemm_ex(x, x_scale, W_gate_up, w_scale_gate_up, 2 * I, offsets, n_groups,
                              rows, I, d, F8_SWIGLU_SAVE, false, h, h_scale, a_gu, 2 * I, nullptr,
                              as_stream(stream));
  return launch_ws_gemm_ex(x, W_gate_up, 2 * I, offsets, n_groups, rows, I, d, WS_SWIGLU_SAVE,
                           false, h, I, a_gu, 2 * I, as_stream(stream));
}

moe_status moe_combine_backward(const void* dh_out, const void* u, const void* E,
                                const void* y_perm, const int32_t* inv_row,
                                const int32_t* topk_idx, const float* topk_gate, moe_dtype dt,
                                int T, int d, int K, int N_r, void* dy_perm, float* d_gate,
                                float* d_logit, float* d_logit_perm, void* stream) {
  clear_last_error();
  MOE_TRY(check_rowwise("moe_combine_backward", dt, T, d, K));
  MOE_REQUIRE(N_r > 0, MOE_ERR_INVALID_ARG, "moe_combine_backward: N_r=%d", N_r);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(dh_out && u && E && y_perm && inv_row && topk_idx && topk_gate && dy_perm &&
                  d_gate && d_logit && d_logit_perm,
              MOE_ERR_INVALID_ARG, "moe_combine_backward: null pointer");
  MOE_REQUIRE(al16(dh_out) && al16(u) && al16(E) && al16(y_perm) && al16(dy_perm),
              MOE_ERR_INVALID_ARG, "moe_combine_backward: rows must be 16-byte aligned");
  MOE_TRY(check_device());
  return launch_combine_backward(dh_out, u, E, y_perm, inv_row, topk_idx, topk_gate, dt, T, d, K,
                                 N_r, dy_perm, d_gate, d_logit, d_logit_perm, as_stream(stream));
}

moe_status moe_quantize_128x1_grouped(const void* x, int rows, int cols, const int32_t* offsets,
                                      int n_groups, uint8_t* q, float* scale,
                                      int32_t* block_start, void* stream) {
  clear_last_error();
  MOE_REQUIRE(rows >= 0 && cols > 0 && cols % 128 == 0, MOE_ERR_UNSUPPORTED,
              "moe_quantize_128x1_grouped: cols=%d must be a positive multiple of 128", cols);
  MOE_REQUIRE(n_groups > 0 && n_groups <= 1 << 20, MOE_ERR_INVALID_ARG,
              "moe_quantize_128x1_grouped: n_groups=%d", n_groups);
  MOE_REQUIRE(block_start, MOE_ERR_INVALID_ARG, "moe_quantize_128x1_grouped: null block_start");
  MOE_REQUIRE(rows == 0 || (x && q && scale), MOE_ERR_INVALID_ARG,
              "moe_quantize_128x1_grouped: null pointer");
  MOE_REQUIRE(al16(x) && al16(q) && al16(scale), MOE_ERR_INVALID_ARG,
              "moe_quantize_128x1_grouped: x, q and scale must be 16-byte aligned");
  MOE_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  MOE_TRY(launch_block_table(offsets, offsets ? n_groups : 1, rows, block_start, s));
  return launch_quant_128x1(x, cols, nullptr, false, rows, cols, offsets, n_groups, block_start, q,
                            scale, s);
}

size_t moe_expert_ffn_backward_workspace_size(moe_dtype dt, int rows, int d, int I,
                                              int n_groups) {
  return ffn_bwd_ws(dt, rows, d, I, n_groups);
}

moe_status moe_expert_ffn_backward(const void* x, const int32_t* x_rows, const int32_t* offsets,
                                   int n_groups, int rows, int d, int I, moe_dtype dt,
                                   const void* W_gate_up, const float* w_scale_gate_up,
                                   const void* W_down, const float* w_scale_down,
                                   const void* a_gu, const void* h, const void* dy, void* dx,
                                   void* dW_gate_up, void* dW_down, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  clear_last_error();
  const char* who = "moe_expert_ffn_backward";
  MOE_TRY(check_ffn_common(who, x, offsets, n_groups, rows, d, I, dt, W_gate_up));
  MOE_REQUIRE(dt == MOE_BF16 || dt == MOE_E4M3, MOE_ERR_UNSUPPORTED,
              "%s: MOE_BF16 or MOE_E4M3 only", who);
  MOE_REQUIRE(d % 256 == 0 && I % 256 == 0, MOE_ERR_UNSUPPORTED,
              "%s: d=%d and I=%d must be multiples of 256", who, d, I);
  MOE_REQUIRE(W_down && dW_gate_up && dW_down, MOE_ERR_INVALID_ARG, "%s: null pointer", who);
  MOE_REQUIRE(al16(dW_gate_up) && al16(dW_down), MOE_ERR_INVALID_ARG,
              "%s: weight gradients must be 16-byte aligned", who);
  MOE_TRY(check_scales(who, dt, w_scale_gate_up, w_scale_down));
  MOE_REQUIRE(dt == MOE_E4M3 || !x_rows, MOE_ERR_INVALID_ARG,
              "%s: x_rows is only for MOE_E4M3", who);
  cudaStream_t s = as_stream(stream);
  if (rows == 0) {
    MOE_TRY(check_device());
    const size_t per = (size_t)n_groups * 2 * I * d * 2;
    MOE_TRY(cuda_check(cudaMemsetAsync(dW_gate_up, 0, per, s), "zero dW_gate_up"));
    return cuda_check(cudaMemsetAsync(dW_down, 0, (size_t)n_groups * d * I * 2, s),
                      "zero dW_down");
  }
  MOE_REQUIRE(a_gu && dy && dx && workspace && (dt == MOE_E4M3 || h), MOE_ERR_INVALID_ARG,
              "%s: null pointer", who);
  MOE_REQUIRE(al16(x) && al16(a_gu) && al16(h) && al16(dy) && al16(dx), MOE_ERR_INVALID_ARG,
              "%s: activations must be 16-byte aligned", who);
  MOE_REQUIRE(reinterpret_cast<uintptr_t>(workspace) % 256 == 0, MOE_ERR_INVALID_ARG,
              "%s: workspace must be 256-byte aligned", who);
  const size_t need = ffn_bwd_ws(dt, rows, d, I, n_groups);
  MOE_REQUIRE(workspace_bytes >= need, MOE_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who,
              workspace_bytes, need);
  MOE_TRY(check_device());
  if (dt == MOE_BF16) {
    void* dA = workspace;
    void* tail = static_cast<uint8_t*>(workspace) + align_up((size_t)rows * 2 * I * 2, 256);
    // Wgrad of the down projection needs only dy and h
    MOE_TRY(launch_wgrad_gemm(dy, d, h, I, offsets, n_groups, rows, tail, dW_down, s));
    // Dgrad of the down projection fused with the SwiGLU backward -> dA
    MOE_TRY(launch_ws_gemm_ex(dy, W_down, 0, offsets, n_groups, rows, I, d, WS_DSWIGLU, true, dA,
                              2 * I, const_cast<void*>(a_gu), 2 * I, s));
    // Dgrad of the gate/up projection
    MOE_TRY(launch_ws_gemm_ex(dA, W_gate_up, 0, offsets, n_groups, rows, d, 2 * I, WS_STORE, true,
                              dx, d, nullptr, 0, s));
    // Wgrad of the gate/up projection
    return launch_wgrad_gemm(dA, 2 * I, x, d, offsets, n_groups, rows, tail, dW_gate_up, s);
  }
  // ---- FP8 (E4M3) backward
  const Fp8BwdLayout L = fp8_bwd_layout(rows, d, I, n_groups);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(w + off); };
  int32_t* blk = reinterpret_cast<int32_t*>(w + L.blk);
  const int G = offsets ? n_groups : 1;
  // Dgrad of the down projection (dy quantised 1x128) fused with the SwiGLU
  // backward: dA as bf16 and as E4M3 1x128
  MOE_TRY(launch_quant_1x128(dy, rows, d, w + L.dy_q, f32(L.dy_s), s));
  MOE_TRY(launch_fp8_gemm_ex(w + L.dy_q, f32(L.dy_s), W_down, w_scale_down, 0, offsets, n_groups,
                             rows, I, d, F8_DSWIGLU, true, w + L.dA_q, f32(L.dA_s),
                             const_cast<void*>(a_gu), 2 * I, w + L.dA_bf, s));
  // Dgrad of the gate/up projection
  MOE_TRY(launch_fp8_gemm_ex(w + L.dA_q, f32(L.dA_s), W_gate_up, w_scale_gate_up, 0, offsets,
                             n_groups, rows, d, 2 * I, F8_STORE, true, dx, nullptr, nullptr, 0,
                             nullptr, s));
  // Wgrad operands: 128-row blocks of each group, one scale per column
  MOE_TRY(launch_block_table(offsets, G, rows, blk, s));
  MOE_TRY(launch_quant_128x1(dy, d, nullptr, false, rows, d, offsets, n_groups, blk, w + L.dyT_q,
                             f32(L.dyT_s), s));
  MOE_TRY(launch_quant_128x1(a_gu, 2 * I, nullptr, true, rows, I, offsets, n_groups, blk,
                             w + L.hT_q, f32(L.hT_s), s));
  MOE_TRY(launch_wgrad_fp8(w + L.dyT_q, f32(L.dyT_s), d, w + L.hT_q, f32(L.hT_s), I, offsets,
                           n_groups, rows, blk, w + L.tail, dW_down, s));
  MOE_TRY(launch_quant_128x1(w + L.dA_bf, 2 * I, nullptr, false, rows, 2 * I, offsets, n_groups,
                             blk, w + L.dAT_q, f32(L.dAT_s), s));
  MOE_TRY(launch_quant_128x1(x, d, x_rows, false, rows, d, offsets, n_groups, blk, w + L.xT_q,
                             f32(L.xT_s), s));
  return launch_wgrad_fp8(w + L.dAT_q, f32(L.dAT_s), 2 * I, w + L.xT_q, f32(L.xT_s), d, offsets,
                          n_groups, rows, blk, w + L.tail, dW_gate_up, s);
}

moe_status moe_unpermute_backward(const void* dh_out, const void* dx_shared, int N_s,
                                  const void* dx_perm, const int32_t* inv_row,
                                  const int32_t* topk_idx, const float* d_logit, const void* E,
                                  moe_dtype dt, int T, int d, int K, int N_r, void* du,
                                  void* stream) {
  clear_last_error();
  MOE_TRY(check_rowwise("moe_unpermute_backward", dt, T, d, K));
  MOE_REQUIRE(N_s >= 0 && N_r > 0, MOE_ERR_INVALID_ARG, "moe_unpermute_backward: N_s=%d N_r=%d",
              N_s, N_r);
  MOE_REQUIRE(N_s + 2 * K <= 63, MOE_ERR_UNSUPPORTED,
              "moe_unpermute_backward: N_s + 2K = %d exceeds 63", N_s + 2 * K);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(dh_out && dx_perm && inv_row && topk_idx && d_logit && E && du &&
                  (N_s == 0 || dx_shared),
              MOE_ERR_INVALID_ARG, "moe_unpermute_backward: null pointer");
  MOE_REQUIRE(al16(dh_out) && al16(dx_perm) && al16(E) && al16(du) && al16(dx_shared),
              MOE_ERR_INVALID_ARG, "moe_unpermute_backward: rows must be 16-byte aligned");
  MOE_TRY(check_device());
  return launch_unpermute_backward(dh_out, dx_shared, N_s, dx_perm, inv_row, topk_idx, d_logit, E,
                                   dt, T, d, K, N_r, du, as_stream(stream));
}

moe_status moe_router_weight_grad(const void* x_perm, const int32_t* x_rows,
                                  const float* d_logit_perm, const int32_t* offsets,
                                  moe_dtype dt, int N_r, int d, float* dE, void* stream) {
  clear_last_error();
  MOE_REQUIRE(dt == MOE_F32 || dt == MOE_BF16, MOE_ERR_UNSUPPORTED,
              "moe_router_weight_grad: dtype must be MOE_F32 or MOE_BF16");
  MOE_REQUIRE(N_r > 0 && d > 0, MOE_ERR_INVALID_ARG, "moe_router_weight_grad: bad sizes");
  MOE_REQUIRE(((size_t)d * dtype_bytes(dt)) % 16 == 0, MOE_ERR_UNSUPPORTED,
              "moe_router_weight_grad: a row must be a multiple of 16 bytes");
  MOE_REQUIRE(x_perm && d_logit_perm && offsets && dE, MOE_ERR_INVALID_ARG,
              "moe_router_weight_grad: null pointer");
  MOE_REQUIRE(al16(x_perm) && al16(dE), MOE_ERR_INVALID_ARG,
              "moe_router_weight_grad: x_perm and dE must be 16-byte aligned");
  MOE_TRY(check_device());
  return launch_router_weight_grad(x_perm, x_rows, d_logit_perm, offsets, dt, N_r, d, dE,
                                   as_stream(stream));
}

// ---------------------------------------------------------------- expert parallelism

moe_status moe_ep_plan(const int32_t* counts_all, int W, int rank, int N_r,
                       int32_t* recv_offsets, int32_t* send_base, void* stream) {
  clear_last_error();
  MOE_REQUIRE(W >= 1 && W <= 8 && rank >= 0 && rank < W, MOE_ERR_INVALID_ARG,
              "moe_ep_plan: W=%d (1..8) rank=%d", W, rank);
  MOE_REQUIRE(N_r > 0 && N_r % W == 0, MOE_ERR_INVALID_ARG,
              "moe_ep_plan: N_r=%d must be a positive multiple of W=%d", N_r, W);
  MOE_REQUIRE(counts_all && recv_offsets && send_base, MOE_ERR_INVALID_ARG,
              "moe_ep_plan: null pointer");
  MOE_TRY(check_device());
  return launch_ep_plan(counts_all, W, rank, N_r, recv_offsets, send_base, as_stream(stream));
}

moe_status moe_ep_dispatch(const void* u, moe_dtype dt, int T, int d, int K,
                           const int32_t* topk_idx, const int32_t* inv_row,
                           const int32_t* offsets, const int32_t* send_base, int N_r, int W,
                           int rank, void* const* recv_rows, void* const* recv_tags,
                           long long recv_cap, void* stream) {
  clear_last_error();
  MOE_TRY(check_rowwise("moe_ep_dispatch", dt, T, d, K));
  MOE_REQUIRE(W >= 1 && W <= 8 && rank >= 0 && rank < W && N_r > 0 && N_r % W == 0,
              MOE_ERR_INVALID_ARG, "moe_ep_dispatch: W=%d rank=%d N_r=%d", W, rank, N_r);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(u && topk_idx && inv_row && offsets && send_base && recv_rows && recv_tags,
              MOE_ERR_INVALID_ARG, "moe_ep_dispatch: null pointer");
  for (int i = 0; i < W; ++i)
    MOE_REQUIRE(recv_rows[i] && recv_tags[i] && al16(recv_rows[i]) &&
                    reinterpret_cast<uintptr_t>(recv_tags[i]) % 8 == 0,
                MOE_ERR_INVALID_ARG, "moe_ep_dispatch: rank %d buffers null or misaligned", i);
  MOE_REQUIRE(al16(u), MOE_ERR_INVALID_ARG, "moe_ep_dispatch: u must be 16-byte aligned");
  MOE_REQUIRE(recv_cap >= 0, MOE_ERR_INVALID_ARG, "moe_ep_dispatch: recv_cap");
  MOE_TRY(check_device());
  return launch_ep_dispatch(u, dtype_bytes(dt), T, d, K, topk_idx, inv_row, offsets, send_base,
                            N_r, W, rank, recv_rows, recv_tags, recv_cap, as_stream(stream));
}

moe_status moe_ep_return(const void* y, moe_dtype dt, const void* recv_tags,
                         const int32_t* n_rows, long long recv_cap, int d, int W,
                         void* const* ret_rows, long long ret_cap, void* stream) {
  clear_last_error();
  MOE_TRY(check_rowwise("moe_ep_return", dt, 0, d, 1));
  MOE_REQUIRE(W >= 1 && W <= 8, MOE_ERR_INVALID_ARG, "moe_ep_return: W=%d", W);
  MOE_REQUIRE(recv_cap >= 0 && recv_cap < (1LL << 31) && ret_cap >= 0, MOE_ERR_INVALID_ARG,
              "moe_ep_return: capacities");
  if (recv_cap == 0) return MOE_OK;
  MOE_REQUIRE(y && recv_tags && n_rows && ret_rows, MOE_ERR_INVALID_ARG,
              "moe_ep_return: null pointer");
  for (int i = 0; i < W; ++i)
    MOE_REQUIRE(ret_rows[i] && al16(ret_rows[i]), MOE_ERR_INVALID_ARG,
                "moe_ep_return: rank %d buffer null or misaligned", i);
  MOE_REQUIRE(al16(y), MOE_ERR_INVALID_ARG, "moe_ep_return: y must be 16-byte aligned");
  MOE_TRY(check_device());
  return launch_ep_return(y, dtype_bytes(dt), recv_tags, n_rows, (int)recv_cap, d, W, ret_rows,
                          ret_cap, as_stream(stream));
}

moe_status moe_device_status(int* flags) {
  clear_last_error();
  MOE_REQUIRE(flags, MOE_ERR_INVALID_ARG, "moe_device_status: null pointer");
  *flags = 0;
  MOE_TRY(cuda_check(cudaDeviceSynchronize(), "moe_device_status synchronize"));
  int* word = device_error_word();
  MOE_REQUIRE(word, MOE_ERR_CUDA, "moe_device_status: error word unavailable");
  MOE_TRY(cuda_check(cudaMemcpy(flags, word, sizeof(int), cudaMemcpyDeviceToHost), "read error word"));
  MOE_TRY(cuda_check(cudaMemset(word, 0, sizeof(int)), "clear error word"));
  return *flags ? fail(MOE_ERR_TIMEOUT, "a kernel gave up a bounded wait (flags 0x%x)", *flags)
                : MOE_OK;
}

}  // extern "C"
