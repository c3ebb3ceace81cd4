"""CPU checks of the boundary: the C-ABI library builds, loads and exports every symbol the
headers declare; struct layouts agree with the header; host-side validation needs no GPU."""
import ctypes
import subprocess

import pytest

from conditional_sparse_attention_b200 import _lib, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    names = _lib.declared_symbols()
    assert len(names) >= 20
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # and the binding declares a signature for each of them
    assert set(names) <= set(_lib._SIGS), set(names) - set(_lib._SIGS)


def test_workload_generator_library_exports(lib):
    from workload import device
    device.build()
    L = device.lib()
    assert hasattr(L, "odagen_fill_normal_bf16") and hasattr(L, "odagen_fill_kv")


def test_struct_layouts_match_header(lib, tmp_path):
    """sizeof/offsetof from a C compiler reading include/oda.h equal the ctypes mirrors."""
    src = tmp_path / "sz.c"
    src.write_text("""
#include <stdio.h>
#include <stddef.h>
#include "oda.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(oda_config), sizeof(oda_kv_layer),
         sizeof(oda_head_weights), sizeof(oda_state), offsetof(oda_config, theta),
         offsetof(oda_config, deterministic), offsetof(oda_head_weights, out_b),
         offsetof(oda_state, conv_width), sizeof(oda_head_grads), offsetof(oda_head_grads, out_b));
  printf("%d %d\\n", ODA_MAX_BATCH, ODA_MAX_LAYERS);
  return 0;
}
""")
    exe = tmp_path / "sz"
    r = subprocess.run(["gcc", "-I", _lib.INCLUDE, "-I", "/usr/local/cuda/include", str(src),
                        "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()
    got = [int(x) for x in out]
    C = _lib
    want = [ctypes.sizeof(C.OdaConfig), ctypes.sizeof(C.OdaKVLayer), ctypes.sizeof(C.OdaHeadWeights),
            ctypes.sizeof(C.OdaState), C.OdaConfig.theta.offset, C.OdaConfig.deterministic.offset,
            C.OdaHeadWeights.out_b.offset,
            C.OdaState.conv_width.offset, ctypes.sizeof(C.OdaHeadGrads), C.OdaHeadGrads.out_b.offset,
            C.MAX_BATCH, C.MAX_LAYERS]
    assert got == want


def test_host_validation_without_gpu(lib):
    assert lib.oda_version() == 1
    assert lib.oda_status_string(1) == b"ODA_ERR_INVALID_ARG"
    out = ctypes.c_void_p()
    bad = _lib.OdaConfig(1, 16, 5, 128, 16, 10, 4, 2048, 2048, 0.0, 0)
    assert lib.oda_create(ctypes.byref(bad), ctypes.byref(out)) == 2
    assert b"Hkv" in lib.oda_last_error() and not out.value
    bad = _lib.OdaConfig(1, 16, 8, 64, 16, 10, 4, 2048, 2048, 0.0, 0)
    assert lib.oda_create(ctypes.byref(bad), ctypes.byref(out)) == 2
    bad = _lib.OdaConfig(1, 16, 8, 128, 16, 10, 4, 2048, 1000, 0.0, 0)
    assert lib.oda_create(ctypes.byref(bad), ctypes.byref(out)) == 2
    assert lib.oda_create(None, ctypes.byref(out)) == 1
    assert lib.oda_attend_local(None, None, None, None, None, None, None, None, None) == 1
    assert lib.oda_graph_launch(None, None) == 1
    assert lib.oda_destroy(None) == 0


def test_recall_grad_host_validation_without_gpu(lib):
    """oda_recall_grad checks its arguments on the host before any CUDA call: null pointers,
    batch and width limits, and the workspace size, each with its own status."""
    ws = lib.oda_recall_grad_workspace_bytes
    assert ws(0, 2048) == 0
    a, b, c = ws(4, 2048), ws(8, 2048), ws(4, 4096)
    assert 0 < a < b and a < c and a % 256 == 0
    w, g = _lib.OdaHeadWeights(), _lib.OdaHeadGrads()
    args = [ctypes.byref(w), ctypes.byref(g)]
    null6 = [None] * 6
    # null pointers
    assert lib.oda_recall_grad(*args, 4, 2048, *null6, ctypes.c_float(0.0), None, None, None,
                               None, 0, None) == 1
    # non-null dummies: the batch and width checks fail before anything is read
    fake = [ctypes.c_void_p(4096 * (i + 1)) for i in range(6)]
    outs = [ctypes.c_void_p(4096 * (i + 10)) for i in range(3)]
    wsp = ctypes.c_void_p(1 << 20)
    assert lib.oda_recall_grad(*args, 17, 2048, *fake, ctypes.c_float(0.0), *outs, wsp, 1 << 30,
                               None) == 2
    assert lib.oda_recall_grad(*args, 4, 1536, *fake, ctypes.c_float(0.0), *outs, wsp, 1 << 30,
                               None) == 2
    assert lib.oda_recall_grad(*args, 4, 2048, *fake, ctypes.c_float(0.0), *outs, wsp, a - 1,
                               None) == 1
    assert b"workspace" in lib.oda_last_error()
    assert lib.oda_recall_grad(*args, 4, 2048, *fake, ctypes.c_float(-1.0), *outs, wsp, a,
                               None) == 1
    assert b"lambda" in lib.oda_last_error()
