"""ctypes binding of the C++ CPU oracle (oracle/moe_ref.cpp).

TEST INFRASTRUCTURE ONLY: the test-suite, the smoke check and the benchmark's
CPU arm use it; the CUDA library never does.  This module only marshals
arrays; every step of the arithmetic is in moe_ref.cpp (plain C++17 loops in
float64, OpenMP across rows or output columns).  Inputs are passed in their
stored form: float32 arrays, or bfloat16 as torch CPU tensors (read as their
raw 16-bit words).

    route(u, E, b, K, n_groups=1, topk_groups=1) -> dict(s, key, idx, gate, counts)
    permute_indices(idx, N_r) -> (offsets, perm_src, inv_row)
    bias_update(b, counts, T, K, gamma=0.001) -> b'
    layer_forward(u, idx, gate, routed, shared, fp8=False) -> h' [T, d] float64
    expert_ffn(x, W_gate_up, W_down, fp8=False) -> y [n, d] float64
    set_threads(n) -> OpenMP threads in force (timing only)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_ref.cpp")
LIB = os.path.join(HERE, "libmoe_ref.so")
GAMMA = 0.001

_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int


def build(force: bool = False) -> str:
    """g++ -O2 -fopenmp, no floating-point contraction (plain IEEE float64)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["g++", "-std=c++17", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               SRC, "-o", LIB]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("building the C++ oracle failed:\n" + r.stderr)
    return LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.ref_route.restype = _I
        L.ref_route.argtypes = [_P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P]
        L.ref_permute.restype = None
        L.ref_permute.argtypes = [_P, _I, _I, _I, _P, _P, _P]
        L.ref_bias_update.restype = None
        L.ref_bias_update.argtypes = [_P, _P, _I, ctypes.c_longlong, _I, ctypes.c_float]
        L.ref_layer_forward.restype = _I
        L.ref_layer_forward.argtypes = [_P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _I, _P, _P, _I, _I,
                                        _P]
        L.ref_set_threads.restype = _I
        L.ref_set_threads.argtypes = [_I]
        L.ref_expert_ffn.restype = None
        L.ref_expert_ffn.argtypes = [_P, _I, _I, _I, _I, _P, _P, _I, _P]
        _lib = L
    return _lib


def _stored(a):
    """(contiguous host array holding the stored values, dt code): float32 -> 0,
    bfloat16 (a torch tensor) -> 1 as raw 16-bit words."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16), 1
            if a.dtype == torch.float32:
                return a.numpy(), 0
            raise TypeError(f"stored dtype {a.dtype} is not float32 or bfloat16")
    except ImportError:
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, 0
    if a.dtype == np.uint16:
        return a, 1
    raise TypeError(f"stored dtype {a.dtype} is not float32 or bfloat16 words")


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_P)


def set_threads(n: int) -> int:
    """OpenMP threads of the following oracle calls (n > 0); returns the count
    in force (n <= 0 only queries it).  Results do not depend on it."""
    return int(lib().ref_set_threads(int(n)))


def route(u, E, b, K, n_groups=1, topk_groups=1):
    ua, dt = _stored(u)
    Ea, dtE = _stored(E)
    if dt != dtE:
        raise TypeError("u and E must have the same stored dtype")
    T, d = ua.shape
    N_r = Ea.shape[0]
    b = np.ascontiguousarray(np.asarray(b, np.float32))
    idx = np.empty((T, K), np.int32)
    gate = np.empty((T, K), np.float32)
    counts = np.empty(N_r, np.int32)
    s = np.empty((T, N_r), np.float32)
    key = np.empty((T, N_r), np.float32)
    rc = lib().ref_route(_ptr(ua), _ptr(Ea), dt, _ptr(b), T, d, N_r, K, n_groups, topk_groups,
                         _ptr(idx), _ptr(gate), _ptr(counts), _ptr(s), _ptr(key))
    if rc != 0:
        raise ValueError("ref_route: bad sizes")
    return {"s": s, "key": key, "idx": idx, "gate": gate, "counts": counts}


def permute_indices(idx, N_r):
    idx = np.ascontiguousarray(np.asarray(idx, np.int32))
    T, K = idx.shape
    offsets = np.empty(N_r + 1, np.int32)
    perm_src = np.full(T * K, -1, np.int32)
    inv_row = np.empty((T, K), np.int32)
    lib().ref_permute(_ptr(idx), T, K, N_r, _ptr(offsets), _ptr(perm_src), _ptr(inv_row))
    return offsets, perm_src, inv_row


def bias_update(b, counts, T, K, gamma=GAMMA):
    out = np.array(b, np.float32, copy=True)
    c = np.ascontiguousarray(np.asarray(counts, np.int32))
    lib().ref_bias_update(_ptr(out), _ptr(c), out.shape[0], int(T), int(K), float(gamma))
    return out


def layer_forward(u, idx, gate, routed, shared, fp8=False):
    """routed[e] / shared[j]: (W_gate_up [2I, d], W_down [d, I]) in the stored
    dtype of u, or None for a routed expert no token selects (routed may be a
    dict).  Returns h' [T, d] float64."""
    ua, dt = _stored(u)
    T, d = ua.shape
    idx = np.ascontiguousarray(np.asarray(idx, np.int32))
    gate = np.ascontiguousarray(np.asarray(gate, np.float32))
    K = idx.shape[1]
    N_r = len(routed)
    keep = []

    def ptrs(seq, n):
        gu = (_P * max(n, 1))()
        dn = (_P * max(n, 1))()
        I = None
        for e in range(n):
            w = seq[e] if not isinstance(seq, dict) else seq.get(e)
            if w is None:
                continue
            a, dta = _stored(w[0])
            c, dtc = _stored(w[1])
            if dta != dt or dtc != dt:
                raise TypeError("weights must have the stored dtype of u")
            keep.extend([a, c])
            gu[e] = a.ctypes.data
            dn[e] = c.ctypes.data
            I = a.shape[0] // 2
        return gu, dn, I

    rgu, rdn, I = ptrs(routed, N_r)
    sgu, sdn, I_s = ptrs(shared, len(shared))
    I = I if I is not None else I_s
    out = np.empty((T, d), np.float64)
    rc = lib().ref_layer_forward(_ptr(ua), dt, T, d, I, _ptr(idx), _ptr(gate), K, rgu, rdn, N_r,
                                 sgu, sdn, len(shared), int(fp8), _ptr(out))
    if rc != 0:
        raise ValueError("ref_layer_forward: a selected expert has no weights")
    return out


def expert_ffn(x, W_gate_up, W_down, fp8=False):
    xa, dt = _stored(x)
    gu, dtg = _stored(W_gate_up)
    dn, dtd = _stored(W_down)
    if not dt == dtg == dtd:
        raise TypeError("x and the weights must share a stored dtype")
    n, d = xa.shape
    I = gu.shape[0] // 2
    y = np.empty((n, d), np.float64)
    lib().ref_expert_ffn(_ptr(xa), dt, n, d, I, _ptr(gu), _ptr(dn), int(fp8), _ptr(y))
    return y
