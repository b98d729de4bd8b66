"""The C-ABI library builds, loads and exports every entry point of
include/moe.h; argument checks answer with a status before any CUDA work.
No GPU is needed: only calls that fail validation are made."""
import ctypes
import os
import re

import pytest

import mixture_experts_layer_60_b200 as moe
from mixture_experts_layer_60_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    moe_build.build()
    return moe.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+)\s*\(", text)))


def test_header_symbols_exported(L):
    names = header_functions()
    assert len(names) >= 14
    raw = ctypes.CDLL(moe.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in moe.h but not exported"
        assert n in moe.SYMBOLS, f"{n} has no binding"


def test_checked_build_exports_the_same_symbols():
    """The bounds-checked variant (-DMOE_CHECK_BOUNDS) builds from the same
    sources and exports every entry point of the header."""
    path = moe_build.build(check_bounds=True)
    assert path.endswith("libmoe_checked.so")
    raw = ctypes.CDLL(path)
    for n in header_functions():
        assert hasattr(raw, n), f"{n} missing from the checked build"


def test_binding_names_match_header():
    assert set(moe.SYMBOLS) == set(header_functions())


def test_abi_version_and_status_strings(L):
    assert L.moe_abi_version() == 2
    assert L.moe_status_string(0) == b"MOE_OK"
    assert L.moe_status_string(3) == b"MOE_ERR_WORKSPACE"


def test_workspace_sizes(L):
    assert L.moe_route_workspace_size(8192, 256) >= 8192 * 256 * 4 + 8193 * 4
    assert L.moe_route_workspace_size(0, 256) == 0
    assert L.moe_permute_workspace_size(8192, 256) >= 2 * 32 * 256 * 4
    assert L.moe_expert_ffn_workspace_size(1, 65536, 2048) == 65536 * 2048 * 2
    assert L.moe_expert_ffn_workspace_size(0, 100, 128) >= 100 * 128 * 4
    fp8 = L.moe_expert_ffn_workspace_size(2, 1000, 256)
    assert fp8 >= 1000 * 256 + 1000 * 2 * 4


def _last(L):
    return L.moe_last_error().decode()


def test_route_argument_errors(L):
    dummy = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    assert L.moe_route(dummy, dummy, 2, dummy, 8, 64, 16, 4, dummy, dummy, dummy, dummy, 4096,
                       None) == 2
    assert "dtype" in _last(L)
    assert L.moe_route(dummy, dummy, 1, dummy, 8, 64, 16, 17, dummy, dummy, dummy, dummy, 4096,
                       None) == 2
    assert L.moe_route(dummy, dummy, 1, dummy, 8, 64, 2000, 4, dummy, dummy, dummy, dummy, 1 << 20,
                       None) == 2
    assert L.moe_route(dummy, dummy, 1, dummy, 8, 96, 16, 4, dummy, dummy, dummy, dummy, 4096,
                       None) == 2
    assert L.moe_route(dummy, None, 1, dummy, 8, 64, 16, 4, dummy, dummy, dummy, dummy, 4096,
                       None) == 1
    assert L.moe_route(dummy, dummy, 1, dummy, -1, 64, 16, 4, dummy, dummy, dummy, dummy, 4096,
                       None) == 1
    assert L.moe_route(dummy, dummy, 1, dummy, 8, 64, 16, 4, dummy, dummy, dummy, dummy, 16,
                       None) == 3
    assert "workspace" in _last(L)


def test_permute_argument_errors(L):
    d = ctypes.c_void_p(256)
    assert L.moe_permute(d, None, 7, d, 8, 64, 16, 4, d, None, d, d, d, d, 1 << 20, None) == 2
    assert L.moe_permute(d, None, 2, d, 8, 64, 16, 4, d, None, d, d, d, d, 1 << 20, None) == 2
    assert L.moe_permute(d, None, 1, d, 8, 64, 16, 4, d, None, None, d, d, d, 1 << 20, None) == 1
    assert L.moe_permute(d, d, 1, d, 8, 64, 16, 4, d, None, d, d, d, d, 1 << 20, None) == 1
    assert L.moe_permute(d, None, 1, d, 8, 64, 16, 4, d, None, d, d, d, d, 8, None) == 3
    assert L.moe_permute(d, None, 1, d, 8, 4, 16, 4, d, None, d, d, d, d, 1 << 20, None) == 2


def test_permute_index_argument_errors(L):
    d = ctypes.c_void_p(256)
    # moe_permute_index(topk_idx, T, N_r, K, offsets, perm_src, inv_row, ws, bytes, stream)
    assert L.moe_permute_index(d, -1, 16, 4, d, d, d, d, 1 << 20, None) == 1     # T < 0
    assert L.moe_permute_index(d, 8, 16, 0, d, d, d, d, 1 << 20, None) == 1      # K = 0
    assert L.moe_permute_index(d, 8, 2048, 4, d, d, d, d, 1 << 20, None) == 2    # N_r > 1024
    assert L.moe_permute_index(d, 8, 16, 17, d, d, d, d, 1 << 20, None) == 2     # K > N_r
    assert L.moe_permute_index(d, 8, 16, 4, None, d, d, d, 1 << 20, None) == 1   # no offsets
    assert L.moe_permute_index(d, 8, 16, 4, d, None, d, d, 1 << 20, None) == 1   # no perm_src
    assert L.moe_permute_index(d, 8, 16, 4, d, d, d, d, 8, None) == 3            # workspace
    assert b"moe_permute_index" in L.moe_last_error()


def test_expert_ffn_argument_errors(L):
    d = ctypes.c_void_p(256)
    assert L.moe_expert_ffn(d, None, d, 4, 100, 192, 128, 1, d, None, d, None, d, d, 1 << 30,
                            None) == 2
    assert L.moe_expert_ffn(d, None, d, 4, 100, 256, 100, 1, d, None, d, None, d, d, 1 << 30,
                            None) == 2
    assert L.moe_expert_ffn(d, None, d, 2000, 100, 256, 128, 1, d, None, d, None, d, d, 1 << 30,
                            None) == 2
    assert L.moe_expert_ffn(d, None, d, 4, 100, 256, 128, 2, d, None, d, None, d, d, 1 << 30,
                            None) == 1
    assert L.moe_expert_ffn(d, d, d, 4, 100, 256, 128, 1, d, None, d, None, d, d, 1 << 30,
                            None) == 1
    assert L.moe_expert_ffn(d, None, d, 4, 100, 256, 128, 1, d, None, d, None, d, d, 64,
                            None) == 3
    assert L.moe_expert_ffn(d, None, None, 4, 100, 256, 128, 1, d, None, d, None, d, d, 1 << 30,
                            None) == 1


def test_combine_bias_quant_argument_errors(L):
    d = ctypes.c_void_p(256)
    assert L.moe_combine(d, d, 1, d, d, d, 2, 8, 64, 4, d, None) == 2
    assert L.moe_combine(d, None, 1, d, d, d, 1, 8, 64, 4, d, None) == 1
    assert L.moe_combine(d, d, 1, d, d, d, 1, 8, 4, 4, d, None) == 2
    assert L.moe_bias_update(None, d, 16, 8, 4, ctypes.c_float(0.001), None) == 1
    assert L.moe_bias_update(d, d, 0, 8, 4, ctypes.c_float(0.001), None) == 1
    assert L.moe_quantize_1x128(d, 4, 100, d, d, None) == 2
    assert L.moe_quantize_1x128(None, 4, 128, d, d, None) == 1
    assert L.moe_quantize_128x128(d, 1, 100, 128, d, d, None) == 2
    assert L.moe_device_status(None) == 1


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "_LIB", None)
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        moe.lib()


def test_backward_argument_errors(L):
    d = ctypes.c_void_p(256)
    # gate/up with saved pre-activations: bf16 or e4m3 (with scales)
    assert L.moe_expert_gate_up_save(d, None, d, 4, 100, 256, 256, 0, d, None, d, None, d,
                                     None) == 2
    assert L.moe_expert_gate_up_save(d, None, d, 4, 100, 256, 256, 1, d, None, None, None, d,
                                     None) == 1
    assert L.moe_expert_gate_up_save(d, None, d, 4, 100, 256, 256, 2, d, None, d, d, d,
                                     None) == 1
    # FFN backward: bf16 or e4m3, d and I multiples of 256, workspace size
    assert L.moe_expert_ffn_backward_workspace_size(1, 1000, 256, 256, 4) >= 1000 * 512 * 2
    assert L.moe_expert_ffn_backward_workspace_size(0, 1000, 256, 256, 4) == 0
    f8 = L.moe_expert_ffn_backward_workspace_size(2, 1000, 256, 256, 4)
    assert f8 >= 1000 * (256 + 512 + 1024 + 256 + 256 + 512 + 256)
    args = lambda dt, dd, I, ws: (d, None, d, 4, 100, dd, I, dt, d, None, d, None, d, d, d, d, d,
                                  d, d, ws, None)
    assert L.moe_expert_ffn_backward(*args(0, 256, 256, 1 << 30)) == 2
    assert L.moe_expert_ffn_backward(*args(1, 256, 128, 1 << 30)) == 2
    assert L.moe_expert_ffn_backward(*args(1, 384, 256, 1 << 30)) == 2
    assert L.moe_expert_ffn_backward(*args(1, 256, 256, 64)) == 3
    assert "workspace" in _last(L)
    assert L.moe_expert_ffn_backward(*args(2, 256, 256, 1 << 30)) == 1   # e4m3 needs scales
    assert L.moe_expert_ffn_backward(d, d, d, 4, 100, 256, 256, 1, d, None, d, None, d, d, d, d,
                                     d, d, d, 1 << 30, None) == 1          # x_rows only for e4m3
    assert L.moe_expert_ffn_backward(d, None, d, 4, 100, 256, 256, 1, d, None, None, None, d, d,
                                     d, d, d, d, d, 1 << 30, None) == 1
    # per-token backward kernels
    assert L.moe_combine_backward(d, d, d, d, d, d, d, 2, 8, 64, 4, 16, d, d, d, d, None) == 2
    assert L.moe_combine_backward(d, d, d, d, d, d, d, 1, 8, 64, 17, 32, d, d, d, d, None) == 2
    assert L.moe_combine_backward(d, d, d, d, d, d, d, 1, 8, 4, 4, 16, d, d, d, d, None) == 2
    assert L.moe_combine_backward(d, d, None, d, d, d, d, 1, 8, 64, 4, 16, d, d, d, d, None) == 1
    assert L.moe_combine_backward(d, d, d, d, d, d, d, 1, 8, 64, 4, 0, d, d, d, d, None) == 1
    assert L.moe_unpermute_backward(d, None, 1, d, d, d, d, d, 1, 8, 64, 4, 16, d, None) == 1
    assert L.moe_unpermute_backward(d, d, 1, d, d, d, d, d, 2, 8, 64, 4, 16, d, None) == 2
    assert L.moe_unpermute_backward(d, d, 1, d, d, d, d, d, 1, 8, 64, 4, 0, d, None) == 1
    # row slots of the gather pipeline: N_s + 2K at most 63
    assert L.moe_unpermute_backward(d, d, 32, d, d, d, d, d, 1, 8, 64, 16, 32, d, None) == 2
    assert L.moe_unpermute_backward(d, d, 31, d, d, d, d, d, 1, 0, 64, 16, 32, d, None) == 0
    assert L.moe_router_weight_grad(d, None, d, d, 2, 16, 64, d, None) == 2
    assert L.moe_router_weight_grad(d, None, d, None, 1, 16, 64, d, None) == 1
    # FP8 Wgrad quantiser
    assert L.moe_quantize_128x1_grouped(d, 100, 100, d, 4, d, d, d, None) == 2
    assert L.moe_quantize_128x1_grouped(d, 100, 128, d, 4, d, d, None, None) == 1


def test_expert_parallel_argument_errors(L):
    d = ctypes.c_void_p(256)
    assert L.moe_ep_plan(d, 9, 0, 16, d, d, None) == 1           # at most 8 ranks
    assert L.moe_ep_plan(d, 3, 0, 16, d, d, None) == 1           # N_r % W
    assert L.moe_ep_plan(d, 2, 2, 16, d, d, None) == 1           # rank < W
    assert L.moe_ep_plan(None, 2, 0, 16, d, d, None) == 1
    two = (ctypes.c_void_p * 2)(256, 256)
    pp = ctypes.cast(two, ctypes.POINTER(ctypes.c_void_p))
    nul = (ctypes.c_void_p * 2)(256, None)
    pn = ctypes.cast(nul, ctypes.POINTER(ctypes.c_void_p))
    assert L.moe_ep_dispatch(d, 2, 8, 64, 4, d, d, d, d, 16, 2, 0, pp, pp, 64, None) == 2  # dtype
    assert L.moe_ep_dispatch(d, 1, 8, 64, 4, d, d, d, d, 16, 2, 0, pn, pp, 64, None) == 1  # null rank buffer
    assert L.moe_ep_dispatch(d, 1, 8, 64, 4, d, d, d, d, 15, 2, 0, pp, pp, 64, None) == 1  # N_r % W
    assert L.moe_ep_return(d, 1, d, d, 64, 64, 9, pp, 64, None) == 1                       # W
    assert L.moe_ep_return(d, 1, d, d, 64, 64, 2, pn, 64, None) == 1


def test_plain_c_program_links_and_calls(L, tmp_path):
    """include/moe.h is a C header: a strict C99 program compiles against it,
    links libmoe.so and calls the host-side entry points (no GPU needed)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_moe.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "moe.h"
int main(void) {
  if (moe_abi_version() <= 0) return 1;
  if (strcmp(moe_status_string(MOE_ERR_WORKSPACE), "MOE_ERR_WORKSPACE") != 0) return 2;
  if (moe_route_workspace_size(0, 256) != 0) return 3;
  if (moe_route_workspace_size(8192, 256) == 0) return 4;
  /* a bad argument answers with a status before any device work */
  if (moe_combine(NULL, NULL, 0, NULL, NULL, NULL, MOE_BF16, 8, 64, 4, NULL, NULL) !=
      MOE_ERR_INVALID_ARG)
    return 5;
  if (moe_last_error()[0] == 0) return 6;
  printf("ok %d\n", moe_abi_version());
  return 0;
}
''')
    exe = tmp_path / "use_moe"
    lib_dir = os.path.dirname(moe.LIB_PATH)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I" + os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L" + lib_dir, "-lmoe", "-Wl,-rpath," + lib_dir],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.startswith("ok"), (r.returncode, r.stdout, r.stderr)
