"""Python binding of libmoe.so, the B200 DeepSeekMoE layer library.

Argument marshalling only: every function here takes torch tensors that
already live on the GPU, passes their device pointers and sizes to the C ABI
of include/moe.h, and raises MoeError on a non-zero status.  All arithmetic
runs in the library's CUDA kernels.  There is no CPU path: importing works
without a GPU, but every call needs the built library and a B200.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MoeError", "lib", "LIB_PATH", "SYMBOLS",
    "moe_route", "moe_route_grouped", "moe_permute", "moe_permute_noalloc", "moe_expert_ffn", "moe_expert_gate_up", "moe_expert_down", "moe_combine", "moe_bias_update",
    "moe_quantize_1x128", "moe_quantize_128x128", "moe_device_status",
    "moe_set_pipeline_wait_limit", "moe_expert_gate_up_shared", "moe_expert_down_shared",
    "moe_set_router_tie_break",
    "moe_route_workspace_size", "moe_permute_workspace_size", "moe_expert_ffn_workspace_size",
    "moe_expert_gate_up_save", "moe_combine_backward", "moe_expert_ffn_backward",
    "moe_expert_ffn_backward_workspace_size", "moe_unpermute_backward", "moe_router_weight_grad",
    "moe_quantize_128x1_grouped", "moe_ep_plan", "moe_ep_dispatch", "moe_ep_return",
    "moe_permute_index",
]

# MOE_LIBRARY (environment) selects another build of the library, e.g. the
# bounds-checked libmoe_checked.so; default: the in-tree libmoe.so.
LIB_PATH = os.environ.get("MOE_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                         "libmoe.so")

MOE_F32, MOE_BF16, MOE_E4M3 = 0, 1, 2
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT"}

_vp, _i, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float

# name -> (restype, argtypes); mirrors include/moe.h
SYMBOLS = {
    "moe_abi_version": (_i, []),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_status_string": (ctypes.c_char_p, [_i]),
    "moe_route_workspace_size": (_sz, [_i, _i]),
    "moe_route": (_i, [_vp, _vp, _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_route_grouped": (_i, [_vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz,
                               _vp]),
    "moe_permute_workspace_size": (_sz, [_i, _i]),
    "moe_permute": (_i, [_vp, _vp, _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_ffn_workspace_size": (_sz, [_i, _i, _i]),
    "moe_expert_ffn": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                            _vp]),
    "moe_expert_gate_up": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "moe_expert_down": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_combine": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp]),
    "moe_bias_update": (_i, [_vp, _vp, _i, _i, _i, _f, _vp]),
    "moe_quantize_1x128": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "moe_quantize_128x128": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_device_status": (_i, [ctypes.POINTER(_i)]),
    "moe_set_pipeline_wait_limit": (_i, [ctypes.c_ulonglong]),
    "moe_set_router_tie_break": (_i, [_f, _f]),
    "moe_expert_gate_up_shared": (_i, [_vp, _vp, _i, _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_expert_down_shared": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_permute_noalloc": (_i, [_vp, _vp, _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_permute_index": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_gate_up_save": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                                     _vp]),
    "moe_combine_backward": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp,
                                  _vp, _vp, _vp]),
    "moe_expert_ffn_backward_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "moe_expert_ffn_backward": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_unpermute_backward": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp,
                                    _vp]),
    "moe_router_weight_grad": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "moe_quantize_128x1_grouped": (_i, [_vp, _i, _i, _vp, _i, _vp, _vp, _vp, _vp]),
    "moe_ep_plan": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_ep_dispatch": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _i, _i, _i,
                             ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.c_longlong, _vp]),
    "moe_ep_return": (_i, [_vp, _i, _vp, _vp, ctypes.c_longlong, _i, _i, ctypes.POINTER(_vp),
                           ctypes.c_longlong, _vp]),
}


class MoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mixture_experts_layer_60_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SYMBOLS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _check(status: int):
    if status != 0:
        raise MoeError(status, lib().moe_last_error().decode(errors="replace"))


# Tracing: with MOE_NVTX=1 in the environment every call below is wrapped in
# an NVTX range named after the C entry point (visible in ncu / nsys timelines).
_NVTX = os.environ.get("MOE_NVTX", "0") not in ("", "0")


def _traced(fn):
    if not _NVTX:
        return fn
    import functools

    @functools.wraps(fn)
    def wrap(*a, **k):
        torch.cuda.nvtx.range_push(fn.__name__)
        try:
            return fn(*a, **k)
        finally:
            torch.cuda.nvtx.range_pop()
    return wrap


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmoe takes device tensors only")
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors only")
    return t.data_ptr()


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dt(t):
    if t.dtype == torch.float32:
        return MOE_F32
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return MOE_E4M3
    raise ValueError(f"unsupported dtype {t.dtype}")


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


# ------------------------------------------------------------------ sizes

def moe_route_workspace_size(T: int, N_r: int) -> int:
    return lib().moe_route_workspace_size(T, N_r)


def moe_permute_workspace_size(T: int, N_r: int) -> int:
    return lib().moe_permute_workspace_size(T, N_r)


def moe_expert_ffn_workspace_size(dt: int, rows: int, I: int) -> int:
    return lib().moe_expert_ffn_workspace_size(dt, rows, I)


# ------------------------------------------------------------------ calls

def moe_route(u, E, b, K, topk_idx, topk_gate, counts, workspace, stream=None):
    T, d = u.shape
    _check(lib().moe_route(_p(u), _p(E), _dt(u), _p(b), T, d, E.shape[0], K, _p(topk_idx),
                           _p(topk_gate), _p(counts), _p(workspace), _nbytes(workspace),
                           _s(stream)))


def moe_route_grouped(u, E, b, K, n_groups, topk_groups, topk_idx, topk_gate, counts, workspace,
                      stream=None):
    T, d = u.shape
    _check(lib().moe_route_grouped(_p(u), _p(E), _dt(u), _p(b), T, d, E.shape[0], K, n_groups,
                                   topk_groups, _p(topk_idx), _p(topk_gate), _p(counts),
                                   _p(workspace), _nbytes(workspace), _s(stream)))


def moe_permute(u, topk_idx, N_r, x_perm, offsets, perm_src, inv_row, workspace,
                u_scale=None, x_scale=None, stream=None):
    T, d = u.shape
    K = topk_idx.shape[1]
    _check(lib().moe_permute(_p(u), _p(u_scale), _dt(u), _p(topk_idx), T, d, N_r, K, _p(x_perm),
                             _p(x_scale), _p(offsets), _p(perm_src), _p(inv_row), _p(workspace),
                             _nbytes(workspace), _s(stream)))


def moe_permute_noalloc(u, topk_idx, N_r, x_perm, offsets, perm_src, inv_row, u_scale=None,
                        x_scale=None, stream=None):
    """moe_permute without a workspace, for callers that cannot allocate device
    memory: the library keeps a static 1 MiB scratch array per GPU (see
    include/moe.h for the size limit and the rule that overlapping calls race)."""
    T, d = u.shape
    K = topk_idx.shape[1]
    _check(lib().moe_permute_noalloc(_p(u), _p(u_scale), _dt(u), _p(topk_idx), T, d, N_r, K,
                                     _p(x_perm), _p(x_scale), _p(offsets), _p(perm_src),
                                     _p(inv_row), _s(stream)))


def moe_permute_index(topk_idx, N_r, offsets, perm_src, inv_row, workspace, stream=None):
    """The grouping of moe_permute (offsets, perm_src, inv_row) without the row copies."""
    T, K = topk_idx.shape
    _check(lib().moe_permute_index(_p(topk_idx), T, N_r, K, _p(offsets), _p(perm_src),
                                   _p(inv_row), _p(workspace), _nbytes(workspace), _s(stream)))


def moe_expert_ffn(x, offsets, W_gate_up, W_down, y, workspace, x_scale=None,
                   w_scale_gate_up=None, w_scale_down=None, stream=None):
    rows, d = x.shape
    n_groups, two_i, _ = W_gate_up.shape
    _check(lib().moe_expert_ffn(_p(x), _p(x_scale), _p(offsets), n_groups, rows, d, two_i // 2,
                                _dt(x), _p(W_gate_up), _p(w_scale_gate_up), _p(W_down),
                                _p(w_scale_down), _p(y), _p(workspace), _nbytes(workspace),
                                _s(stream)))


def moe_expert_gate_up(x, offsets, W_gate_up, h, x_scale=None, w_scale_gate_up=None,
                       h_scale=None, stream=None):
    rows, d = x.shape
    n_groups, two_i, _ = W_gate_up.shape
    _check(lib().moe_expert_gate_up(_p(x), _p(x_scale), _p(offsets), n_groups, rows, d,
                                    two_i // 2, _dt(x), _p(W_gate_up), _p(w_scale_gate_up), _p(h),
                                    _p(h_scale), _s(stream)))


def moe_expert_down(h, offsets, W_down, y, h_scale=None, w_scale_down=None, stream=None):
    rows, I = h.shape
    n_groups, d, _ = W_down.shape
    _check(lib().moe_expert_down(_p(h), _p(h_scale), _p(offsets), n_groups, rows, d, I, _dt(h),
                                 _p(W_down), _p(w_scale_down), _p(y), _s(stream)))


def moe_expert_gate_up_shared(x, offsets, W_gate_up, u, Ws_gate_up, h, stream=None):
    """Routed gate/up (x [rows, d]) with the shared experts' gate/up of u
    [T, d] as extra groups of one launch: h [rows + N_s*T, I]."""
    rows, d = x.shape
    n_groups, two_i, _ = W_gate_up.shape
    T, N_s = u.shape[0], Ws_gate_up.shape[0]
    _check(lib().moe_expert_gate_up_shared(_p(x), _p(offsets), n_groups, rows, _p(u), T, N_s, d,
                                           two_i // 2, _p(W_gate_up), _p(Ws_gate_up), _p(h),
                                           _s(stream)))


def moe_expert_down_shared(h, offsets, W_down, Ws_down, rows, T, y, stream=None):
    """Routed down projection of h[:rows] and the shared experts' of
    h[rows + j*T + t] in one launch: y [rows + N_s*T, d]."""
    n_groups, d, I = W_down.shape
    N_s = Ws_down.shape[0]
    _check(lib().moe_expert_down_shared(_p(h), _p(offsets), n_groups, rows, T, N_s, d, I,
                                        _p(W_down), _p(Ws_down), _p(y), _s(stream)))


def moe_combine(u, y_shared, y_perm, inv_row, topk_gate, h_out, stream=None):
    T, d = u.shape
    N_s = 0 if y_shared is None else y_shared.shape[0]
    _check(lib().moe_combine(_p(u), _p(y_shared), N_s, _p(y_perm), _p(inv_row), _p(topk_gate),
                             _dt(u), T, d, inv_row.shape[1], _p(h_out), _s(stream)))


def moe_bias_update(b, counts, T, K, gamma=0.001, stream=None):
    _check(lib().moe_bias_update(_p(b), _p(counts), b.shape[0], T, K, gamma, _s(stream)))


def moe_quantize_1x128(x, q, scale, stream=None):
    rows, cols = x.shape
    _check(lib().moe_quantize_1x128(_p(x), rows, cols, _p(q), _p(scale), _s(stream)))


def moe_quantize_128x128(w, q, scale, stream=None):
    groups, rows, cols = w.shape
    _check(lib().moe_quantize_128x128(_p(w), groups, rows, cols, _p(q), _p(scale), _s(stream)))


def moe_set_router_tie_break(refine_gap: float = 0.0, near: float = 0.0):
    """Thresholds of the router's float64 tie-break; (0, 0) restores the defaults."""
    _check(lib().moe_set_router_tie_break(float(refine_gap), float(near)))


def moe_set_pipeline_wait_limit(ns: int = 0):
    """Bound (ns) of the row-gather pipeline's waits; 0 restores the default 1 s."""
    _check(lib().moe_set_pipeline_wait_limit(int(ns)))


def moe_device_status() -> int:
    flags = ctypes.c_int(0)
    st = lib().moe_device_status(ctypes.byref(flags))
    if st not in (0, 5):
        _check(st)
    return flags.value


# ------------------------------------------------------------------ backward

def moe_expert_ffn_backward_workspace_size(dt: int, rows: int, d: int, I: int,
                                           n_groups: int) -> int:
    return lib().moe_expert_ffn_backward_workspace_size(dt, rows, d, I, n_groups)


def moe_expert_gate_up_save(x, offsets, W_gate_up, h, a_gu, x_scale=None, w_scale_gate_up=None,
                            h_scale=None, stream=None):
    rows, d = x.shape
    n_groups, two_i, _ = W_gate_up.shape
    _check(lib().moe_expert_gate_up_save(_p(x), _p(x_scale), _p(offsets), n_groups, rows, d,
                                         two_i // 2, _dt(x), _p(W_gate_up), _p(w_scale_gate_up),
                                         _p(h), _p(h_scale), _p(a_gu), _s(stream)))


def moe_combine_backward(dh_out, u, E, y_perm, inv_row, topk_idx, topk_gate, dy_perm, d_gate,
                         d_logit, d_logit_perm, stream=None):
    T, d = u.shape
    _check(lib().moe_combine_backward(_p(dh_out), _p(u), _p(E), _p(y_perm), _p(inv_row),
                                      _p(topk_idx), _p(topk_gate), _dt(u), T, d,
                                      inv_row.shape[1], E.shape[0], _p(dy_perm), _p(d_gate),
                                      _p(d_logit), _p(d_logit_perm), _s(stream)))


def moe_expert_ffn_backward(x, offsets, W_gate_up, W_down, a_gu, h, dy, dx, dW_gate_up, dW_down,
                            workspace, x_rows=None, w_scale_gate_up=None, w_scale_down=None,
                            stream=None):
    """dt follows the weights: bf16 weights -> MOE_BF16, e4m3 weights (uint8
    with their 128x128 scales) -> MOE_E4M3.  x is bf16 in both cases."""
    rows, d = dy.shape
    n_groups, two_i, _ = W_gate_up.shape
    _check(lib().moe_expert_ffn_backward(_p(x), _p(x_rows), _p(offsets), n_groups, rows, d,
                                         two_i // 2, _dt(W_gate_up), _p(W_gate_up),
                                         _p(w_scale_gate_up), _p(W_down), _p(w_scale_down),
                                         _p(a_gu), _p(h), _p(dy), _p(dx), _p(dW_gate_up),
                                         _p(dW_down), _p(workspace), _nbytes(workspace),
                                         _s(stream)))


def moe_unpermute_backward(dh_out, dx_shared, dx_perm, inv_row, topk_idx, d_logit, E, du,
                           stream=None):
    T, d = dh_out.shape
    N_s = 0 if dx_shared is None else dx_shared.shape[0]
    _check(lib().moe_unpermute_backward(_p(dh_out), _p(dx_shared), N_s, _p(dx_perm), _p(inv_row),
                                        _p(topk_idx), _p(d_logit), _p(E), _dt(dh_out), T, d,
                                        inv_row.shape[1], E.shape[0], _p(du), _s(stream)))


def moe_router_weight_grad(x, d_logit_perm, offsets, dE, x_rows=None, stream=None):
    N_r, d = dE.shape
    _check(lib().moe_router_weight_grad(_p(x), _p(x_rows), _p(d_logit_perm), _p(offsets), _dt(x),
                                        N_r, d, _p(dE), _s(stream)))


def moe_quantize_128x1_grouped(x, offsets, q, scale, block_start, stream=None):
    rows, cols = x.shape
    n_groups = 1 if offsets is None else offsets.shape[0] - 1
    _check(lib().moe_quantize_128x1_grouped(_p(x), rows, cols, _p(offsets), n_groups, _p(q),
                                            _p(scale), _p(block_start), _s(stream)))


# ------------------------------------------------------------------ expert parallelism

def _ptrs(tensors):
    arr = (ctypes.c_void_p * len(tensors))(*[_p(t) for t in tensors])
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)), arr


def moe_ep_plan(counts_all, rank, recv_offsets, send_base, stream=None):
    W, N_r = counts_all.shape
    _check(lib().moe_ep_plan(_p(counts_all), W, rank, N_r, _p(recv_offsets), _p(send_base),
                             _s(stream)))


def moe_ep_dispatch(u, topk_idx, inv_row, offsets, send_base, rank, recv_rows, recv_tags,
                    stream=None):
    """recv_rows / recv_tags: one tensor per rank (this GPU's or a peer's)."""
    T, d = u.shape
    W = len(recv_rows)
    rp, _k1 = _ptrs(recv_rows)
    tp, _k2 = _ptrs(recv_tags)
    _check(lib().moe_ep_dispatch(_p(u), _dt(u), T, d, topk_idx.shape[1], _p(topk_idx),
                                 _p(inv_row), _p(offsets), _p(send_base), send_base.shape[0], W,
                                 rank, rp, tp, recv_rows[0].shape[0], _s(stream)))


def moe_ep_return(y, recv_tags, n_rows, ret_rows, stream=None):
    cap, d = y.shape
    W = len(ret_rows)
    rp, _k = _ptrs(ret_rows)
    _check(lib().moe_ep_return(_p(y), _dt(y), _p(recv_tags), _p(n_rows), cap, d, W, rp,
                               ret_rows[0].shape[0], _s(stream)))


# wrap the public calls for tracing (no-op unless MOE_NVTX is set)
for _name in [n for n in __all__ if n.startswith("moe_") and n in globals()
              and not n.endswith("workspace_size")]:
    globals()[_name] = _traced(globals()[_name])
