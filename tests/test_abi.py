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
  printf("%zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(oda_config), sizeof(oda_kv_layer),
         sizeof(oda_head_weights), sizeof(oda_state), offsetof(oda_config, theta),
         offsetof(oda_config, deterministic), offsetof(oda_head_weights, out_b),
         offsetof(oda_state, conv_width));
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
            C.OdaState.conv_width.offset, C.MAX_BATCH, C.MAX_LAYERS]
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
