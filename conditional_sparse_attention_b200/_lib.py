"""ctypes view of liboda.so (include/oda.h, include/oda_glue.h).

Loading fails loudly: there is no fallback implementation of any entry point.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "liboda.so")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")

c_int32, c_int64, c_float, c_void_p = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p

ODA_OK = 0
STATUS = {0: "ODA_OK", 1: "ODA_ERR_INVALID_ARG", 2: "ODA_ERR_UNSUPPORTED", 3: "ODA_ERR_CUDA",
          4: "ODA_ERR_DEVICE", 5: "ODA_ERR_STATE"}
DEVERR_PAGE_RANGE = 0x1
DEVERR_POS_RANGE = 0x2
DEVERR_WAIT_TIMEOUT = 0x4
MAX_BATCH = 256
MAX_LAYERS = 64


class OdaConfig(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("n_q_heads", c_int32), ("n_kv_heads", c_int32),
                ("head_dim", c_int32), ("page_size", c_int32), ("max_pages", c_int32),
                ("sinks", c_int32), ("window", c_int32), ("head_in_dim", c_int32),
                ("theta", c_float), ("overlap_layers", c_int32), ("deterministic", c_int32)]


class OdaKVLayer(ctypes.Structure):
    _fields_ = [("k", c_void_p), ("v", c_void_p), ("n_pages", c_int64)]


class OdaKV8Layer(ctypes.Structure):
    _fields_ = [("kv", c_void_p), ("n_pages", c_int64)]


class OdaBBLayer(ctypes.Structure):
    _fields_ = [("attn_norm", c_void_p), ("w_qkv", c_void_p), ("w_o", c_void_p),
                ("mlp_norm", c_void_p), ("w_gate", c_void_p), ("w_up", c_void_p),
                ("w_down", c_void_p), ("ffn", c_int32)]


class OdaHeadWeights(ctypes.Structure):
    _fields_ = [("tower_norm", c_void_p * 3), ("tower_w", c_void_p * 3), ("tower_b", c_void_p * 3),
                ("fuse_w", c_void_p), ("fuse_b", c_void_p), ("ffn_norm", c_void_p * 2),
                ("ffn_gate", c_void_p * 2), ("ffn_up", c_void_p * 2), ("ffn_down", c_void_p * 2),
                ("out_norm", c_void_p), ("out_w", c_void_p), ("out_b", c_void_p)]


class OdaHeadGrads(ctypes.Structure):
    _fields_ = OdaHeadWeights._fields_


class OdaState(ctypes.Structure):
    _fields_ = [("rec", c_void_p), ("conv", c_void_p), ("n_layers", c_int32), ("heads", c_int32),
                ("dk", c_int32), ("dv", c_int32), ("conv_taps", c_int32), ("conv_width", c_int32)]


_P = ctypes.POINTER
_SIGS = {
    "oda_create": ([_P(OdaConfig), _P(c_void_p)], c_int32),
    "oda_destroy": ([c_void_p], c_int32),
    "oda_attend_local": ([c_void_p, _P(OdaKVLayer), c_void_p, c_void_p, c_void_p, c_void_p,
                          c_void_p, c_void_p, c_void_p], c_int32),
    "oda_attend_full_if": ([c_void_p, _P(OdaKVLayer), c_void_p, c_void_p, c_void_p, c_void_p,
                            c_void_p, c_void_p, c_void_p, c_void_p], c_int32),
    "oda_attend_full_if_noalloc": ([_P(OdaConfig), _P(OdaKVLayer), c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p],
                                   c_int32),
    "oda_attend_local_fp8": ([c_void_p, _P(OdaKV8Layer), c_void_p, c_void_p, c_void_p, c_void_p,
                              c_void_p, c_void_p, c_void_p], c_int32),
    "oda_attend_full_if_fp8": ([c_void_p, _P(OdaKV8Layer), c_void_p, c_void_p, c_void_p, c_void_p,
                                c_void_p, c_void_p, c_void_p, c_void_p], c_int32),
    "oda_kv8_pack": ([_P(OdaKVLayer), _P(OdaKV8Layer), c_int32, c_void_p], c_int32),
    "oda_commit_fp8": ([c_void_p, _P(OdaKV8Layer), c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p],
                       c_int32),
    "oda_bb_begin": ([c_void_p, c_void_p, c_void_p, c_void_p], c_int32),
    "oda_bb_qkv": ([c_void_p, _P(OdaBBLayer), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p],
                   c_int32),
    "oda_bb_attn_out": ([c_void_p, _P(OdaBBLayer), c_void_p, c_void_p, c_void_p], c_int32),
    "oda_bb_mlp": ([c_void_p, _P(OdaBBLayer), c_void_p, c_void_p, c_void_p], c_int32),
    "oda_bb_pack_weight": ([c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p], c_int32),
    "oda_bb_post_attention": ([c_void_p, _P(OdaBBLayer), _P(OdaBBLayer), c_void_p, c_void_p, c_void_p,
                               c_void_p, c_void_p, c_void_p, c_void_p], c_int32),
    "oda_bb_final_norm": ([c_void_p, c_void_p, c_void_p, c_void_p, c_void_p], c_int32),
    "oda_bb_lm_head": ([c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                        c_void_p], c_int32),
    "oda_bb_embed": ([c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p], c_int32),
    "oda_index_positions": ([c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_int32, c_void_p,
                             c_void_p], c_int32),
    "oda_recall_score": ([c_void_p, _P(OdaHeadWeights), c_void_p, c_void_p, c_void_p, c_void_p,
                          c_void_p, c_void_p, c_void_p, c_void_p], c_int32),
    "oda_recall_plan": ([c_void_p, _P(c_int32), _P(c_int32), _P(c_int32)], c_int32),
    "oda_recall_grad_workspace_bytes": ([c_int32, c_int32], ctypes.c_size_t),
    "oda_recall_grad": ([_P(OdaHeadWeights), _P(OdaHeadGrads), c_int32, c_int32, c_void_p, c_void_p,
                         c_void_p, c_void_p, c_void_p, c_void_p, ctypes.c_float, c_void_p, c_void_p,
                         c_void_p, c_void_p, ctypes.c_size_t, c_void_p], c_int32),
    "oda_commit": ([c_void_p, _P(OdaKVLayer), c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p], c_int32),
    "oda_snapshot": ([c_void_p, _P(OdaState), _P(OdaState), c_void_p], c_int32),
    "oda_restore": ([c_void_p, c_void_p, _P(OdaState), _P(OdaState), c_void_p], c_int32),
    "oda_cond_begin": ([c_void_p, c_void_p, c_void_p, _P(c_void_p)], c_int32),
    "oda_cond_end": ([c_void_p, c_void_p], c_int32),
    "oda_graph_begin": ([c_void_p], c_int32),
    "oda_graph_end": ([c_void_p, _P(c_void_p)], c_int32),
    "oda_graph_launch": ([c_void_p, c_void_p], c_int32),
    "oda_graph_destroy": ([c_void_p], c_int32),
    "oda_get_error": ([c_void_p, _P(c_int32)], c_int32),
    "oda_clear_error": ([c_void_p, c_void_p], c_int32),
    "oda_probe_wait": ([c_void_p, c_int32, ctypes.c_int64, c_void_p], c_int32),
    "oda_status_string": ([c_int32], ctypes.c_char_p),
    "oda_last_error": ([], ctypes.c_char_p),
    "oda_version": ([], c_int32),
    "oda_glue_hidden": ([c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p],
                        c_int32),
    "oda_glue_gdn": ([c_void_p, _P(OdaState), c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                      c_void_p, c_void_p, c_void_p, c_void_p], c_int32),
    "oda_glue_gdn_step": ([c_void_p, _P(OdaState), _P(OdaState), c_int32, c_void_p, c_void_p,
                           c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p], c_int32),
}

_lib = None


class OdaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def declared_symbols() -> list:
    """Every function declared in include/*.h."""
    names = []
    for f in sorted(os.listdir(INCLUDE)):
        if f.endswith(".h"):
            txt = open(os.path.join(INCLUDE, f)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"\b(oda_[a-z_0-9]+)\s*\(", txt)
    return sorted(set(names))


def load():
    """The loaded library; raises if it is missing (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m conditional_sparse_attention_b200.build` (the CUDA path has no fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def check(status: int) -> None:
    if status != ODA_OK:
        msg = load().oda_last_error().decode(errors="replace")
        raise OdaError(status, msg)
