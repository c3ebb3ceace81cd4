"""Python binding of the ODA C ABI: one function per entry point, same names, argument
marshalling only (torch tensors -> device pointers, torch streams -> cudaStream_t).

Every function raises OdaError on a non-OK status.  Tensors must already live on the device
the context was created on; shapes follow include/oda.h.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import torch

from . import _lib
from ._lib import (OdaBBLayer, OdaConfig, OdaError, OdaHeadGrads, OdaHeadWeights,  # noqa: F401
                   OdaKV8Layer, OdaKVLayer, OdaState, check)

_c = ctypes.c_void_p


def _p(t) -> ctypes.c_void_p:
    if t is None:
        return _c(None)
    if isinstance(t, int):
        return _c(t)
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return _c(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return _c(stream)
    return _c(stream.cuda_stream)


class Context:
    """Owns an oda_ctx*; freed by close() or garbage collection."""

    def __init__(self, handle: ctypes.c_void_p, cfg: OdaConfig):
        self.handle = handle
        self.cfg = cfg

    def close(self):
        if self.handle and self.handle.value:
            _lib.load().oda_destroy(self.handle)
            self.handle = _c(None)

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


def make_config(batch, n_q_heads, n_kv_heads, max_pages, head_in_dim, sinks=4, window=2048,
                theta=0.0, head_dim=128, page_size=16, overlap_layers=False,
                deterministic=False) -> OdaConfig:
    return OdaConfig(batch, n_q_heads, n_kv_heads, head_dim, page_size, max_pages, sinks, window,
                     head_in_dim, theta, 1 if overlap_layers else 0, 1 if deterministic else 0)


def kv_layer(k: torch.Tensor, v: torch.Tensor) -> OdaKVLayer:
    """Pool descriptor: k, v bf16 [n_pages, Hkv, 16, 128]."""
    return OdaKVLayer(k.data_ptr(), v.data_ptr(), int(k.shape[0]))


KV8_BLOCK_BYTES = 4224


def kv8_layer(kv: torch.Tensor) -> OdaKV8Layer:
    """fp8 pool descriptor: kv uint8 [n_pages, Hkv, 4224] (page blocks, see include/oda.h)."""
    return OdaKV8Layer(kv.data_ptr(), int(kv.shape[0]))


def head_weights(P: dict, cls=OdaHeadWeights):
    """Descriptor from a dict of device fp32 tensors named as in include/oda.h."""
    w = cls()
    for i in range(3):
        w.tower_norm[i] = P[f"tower_norm{i}"].data_ptr()
        w.tower_w[i] = P[f"tower_w{i}"].data_ptr()
        w.tower_b[i] = P[f"tower_b{i}"].data_ptr()
    w.fuse_w, w.fuse_b = P["fuse_w"].data_ptr(), P["fuse_b"].data_ptr()
    for j in range(2):
        w.ffn_norm[j] = P[f"ffn_norm{j}"].data_ptr()
        w.ffn_gate[j] = P[f"ffn_gate{j}"].data_ptr()
        w.ffn_up[j] = P[f"ffn_up{j}"].data_ptr()
        w.ffn_down[j] = P[f"ffn_down{j}"].data_ptr()
    w.out_norm, w.out_w, w.out_b = (P["out_norm"].data_ptr(), P["out_w"].data_ptr(),
                                    P["out_b"].data_ptr())
    return w


def head_grads(G: dict) -> OdaHeadGrads:
    """Gradient-buffer descriptor from a dict of device fp32 tensors (names as the weights)."""
    return head_weights(G, OdaHeadGrads)


def state(rec: torch.Tensor, conv: torch.Tensor) -> OdaState:
    """rec fp32 [B, n_layers, heads, dv, dk]; conv fp32 [B, n_layers, taps, width]."""
    _, n, h, dv, dk = rec.shape
    _, n2, taps, width = conv.shape
    assert n == n2
    return OdaState(rec.data_ptr(), conv.data_ptr(), n, h, dk, dv, taps, width)


def oda_create(cfg: OdaConfig) -> Context:
    h = _c()
    check(_lib.load().oda_create(ctypes.byref(cfg), ctypes.byref(h)))
    return Context(h, cfg)


def oda_destroy(ctx: Context) -> None:
    ctx.close()


def oda_attend_local(ctx, layer: OdaKVLayer, page_table, pos, q, k_new, v_new, out, stream=None):
    check(_lib.load().oda_attend_local(ctx.handle, ctypes.byref(layer), _p(page_table), _p(pos),
                                       _p(q), _p(k_new), _p(v_new), _p(out), _s(stream)))


def oda_attend_full_if(ctx, layer: OdaKVLayer, page_table, pos, flag, q, k_new, v_new, out,
                       stream=None):
    check(_lib.load().oda_attend_full_if(ctx.handle, ctypes.byref(layer), _p(page_table), _p(pos),
                                         _p(flag), _p(q), _p(k_new), _p(v_new), _p(out), _s(stream)))


def oda_attend_full_if_noalloc(cfg: OdaConfig, layer: OdaKVLayer, page_table, pos, flag, q, k_new,
                               v_new, out, device_error=None, stream=None):
    """Full-set attention without a context: scratch in the library's static device array."""
    check(_lib.load().oda_attend_full_if_noalloc(ctypes.byref(cfg), ctypes.byref(layer),
                                                 _p(page_table), _p(pos), _p(flag), _p(q),
                                                 _p(k_new), _p(v_new), _p(out), _p(device_error),
                                                 _s(stream)))


def oda_attend_local_fp8(ctx, layer: OdaKV8Layer, page_table, pos, q, k_new, v_new, out,
                         stream=None):
    check(_lib.load().oda_attend_local_fp8(ctx.handle, ctypes.byref(layer), _p(page_table),
                                           _p(pos), _p(q), _p(k_new), _p(v_new), _p(out),
                                           _s(stream)))


def oda_attend_full_if_fp8(ctx, layer: OdaKV8Layer, page_table, pos, flag, q, k_new, v_new, out,
                           stream=None):
    check(_lib.load().oda_attend_full_if_fp8(ctx.handle, ctypes.byref(layer), _p(page_table),
                                             _p(pos), _p(flag), _p(q), _p(k_new), _p(v_new),
                                             _p(out), _s(stream)))


def oda_kv8_pack(src: OdaKVLayer, dst: OdaKV8Layer, n_kv_heads: int, stream=None):
    check(_lib.load().oda_kv8_pack(ctypes.byref(src), ctypes.byref(dst), n_kv_heads, _s(stream)))


def oda_commit_fp8(ctx, layers: Sequence[OdaKV8Layer], page_table, pos, flag, k_stage_local,
                   v_stage_local, k_stage_full, v_stage_full, h_local, h_full, h_prev,
                   stream=None):
    arr = (OdaKV8Layer * len(layers))(*layers)
    check(_lib.load().oda_commit_fp8(ctx.handle, arr, len(layers), _p(page_table), _p(pos),
                                     _p(flag), _p(k_stage_local), _p(v_stage_local),
                                     _p(k_stage_full), _p(v_stage_full), _p(h_local), _p(h_full),
                                     _p(h_prev), _s(stream)))


def oda_index_positions(ctx, mode: int, pos, flag, positions, cap: int, counts, stream=None):
    check(_lib.load().oda_index_positions(ctx.handle, mode, _p(pos), _p(flag), _p(positions), cap,
                                          _p(counts), _s(stream)))


def oda_recall_score(ctx, w: OdaHeadWeights, h_prev, emb, h_loc, sched, score, flag, any_flag,
                     stream=None):
    check(_lib.load().oda_recall_score(ctx.handle, ctypes.byref(w), _p(h_prev), _p(emb), _p(h_loc),
                                       _p(sched), _p(score), _p(flag), _p(any_flag), _s(stream)))


def oda_recall_plan(ctx) -> tuple:
    """(tile, groups, ring) of the fused head launch for this context, or (0, 0, 0) where the
    six phase launches run."""
    t, g, r = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int32(0)
    check(_lib.load().oda_recall_plan(ctx.handle, ctypes.byref(t), ctypes.byref(g), ctypes.byref(r)))
    return t.value, g.value, r.value


def oda_recall_grad_workspace_bytes(batch: int, head_in_dim: int) -> int:
    return int(_lib.load().oda_recall_grad_workspace_bytes(batch, head_in_dim))


def oda_recall_grad(w: OdaHeadWeights, grad: OdaHeadGrads, batch: int, head_in_dim: int, h_prev,
                    emb, h_loc, p_full, p_local, valid, lam: float, loss, q, y, workspace,
                    stream=None):
    check(_lib.load().oda_recall_grad(ctypes.byref(w), ctypes.byref(grad), batch, head_in_dim,
                                      _p(h_prev), _p(emb), _p(h_loc), _p(p_full), _p(p_local),
                                      _p(valid), float(lam), _p(loss), _p(q), _p(y), _p(workspace),
                                      workspace.numel() * workspace.element_size(), _s(stream)))


def oda_commit(ctx, layers: Sequence[OdaKVLayer], page_table, pos, flag, k_stage_local,
               v_stage_local, k_stage_full, v_stage_full, h_local, h_full, h_prev, stream=None):
    arr = (OdaKVLayer * len(layers))(*layers)
    check(_lib.load().oda_commit(ctx.handle, arr, len(layers), _p(page_table), _p(pos), _p(flag),
                                 _p(k_stage_local), _p(v_stage_local), _p(k_stage_full),
                                 _p(v_stage_full), _p(h_local), _p(h_full), _p(h_prev), _s(stream)))


def oda_snapshot(ctx, live: OdaState, snap: OdaState, stream=None):
    check(_lib.load().oda_snapshot(ctx.handle, ctypes.byref(live), ctypes.byref(snap), _s(stream)))


def oda_restore(ctx, flag, snap: OdaState, live: OdaState, stream=None):
    check(_lib.load().oda_restore(ctx.handle, _p(flag), ctypes.byref(snap), ctypes.byref(live),
                                  _s(stream)))


def oda_cond_begin(ctx, stream, any_flag) -> int:
    """Returns the cudaStream_t (as int) on which the conditional body must be issued."""
    body = _c()
    check(_lib.load().oda_cond_begin(ctx.handle, _s(stream), _p(any_flag), ctypes.byref(body)))
    return body.value or 0


def oda_cond_end(ctx, stream):
    check(_lib.load().oda_cond_end(ctx.handle, _s(stream)))


class Graph:
    def __init__(self, handle):
        self.handle = handle

    def launch(self, stream=None):
        check(_lib.load().oda_graph_launch(self.handle, _s(stream)))

    def close(self):
        if self.handle and self.handle.value:
            _lib.load().oda_graph_destroy(self.handle)
            self.handle = _c(None)

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


def oda_graph_begin(stream):
    check(_lib.load().oda_graph_begin(_s(stream)))


def oda_graph_end(stream) -> Graph:
    h = _c()
    check(_lib.load().oda_graph_end(_s(stream), ctypes.byref(h)))
    return Graph(h)


def oda_graph_launch(g: Graph, stream=None):
    g.launch(stream)


def oda_graph_destroy(g: Graph):
    g.close()


def oda_get_error(ctx) -> int:
    """Synchronises the device and returns the sticky device error word (0 if clean)."""
    v = ctypes.c_int32(0)
    st = _lib.load().oda_get_error(ctx.handle, ctypes.byref(v))
    if st not in (0, 4):
        check(st)
    return int(v.value)


def oda_clear_error(ctx, stream=None):
    check(_lib.load().oda_clear_error(ctx.handle, _s(stream)))


def oda_probe_wait(ctx, which: int, limit_ns: int, stream=None):
    check(_lib.load().oda_probe_wait(ctx.handle, which, int(limit_ns), _s(stream)))


def oda_version() -> int:
    return int(_lib.load().oda_version())


def oda_glue_hidden(ctx, emb, terms, n_terms: int, flag, h, stream=None):
    check(_lib.load().oda_glue_hidden(ctx.handle, _p(emb), _p(terms), n_terms, _p(flag), _p(h),
                                      _s(stream)))


def oda_glue_gdn_step(ctx, src: OdaState, dst: OdaState, layer: int, c, v, alpha, beta, taps, flag,
                      o, stream=None):
    check(_lib.load().oda_glue_gdn_step(ctx.handle, ctypes.byref(src), ctypes.byref(dst), layer,
                                        _p(c), _p(v), _p(alpha), _p(beta), _p(taps), _p(flag), _p(o),
                                        _s(stream)))


def oda_glue_gdn(ctx, st: OdaState, layer: int, c, v, alpha, beta, taps, flag, o, stream=None):
    check(_lib.load().oda_glue_gdn(ctx.handle, ctypes.byref(st), layer, _p(c), _p(v), _p(alpha),
                                   _p(beta), _p(taps), _p(flag), _p(o), _s(stream)))


# ------------------------------------------------------------------ synthetic backbone
def bb_layer(attn_norm, w_qkv, w_o, mlp_norm, w_gate, w_up, w_down) -> OdaBBLayer:
    """Layer descriptor from device tensors (norm weights fp32 [D]; projections bf16 or int16
    [out, in]); F is taken from w_gate."""
    return OdaBBLayer(attn_norm.data_ptr(), w_qkv.data_ptr(), w_o.data_ptr(), mlp_norm.data_ptr(),
                      w_gate.data_ptr(), w_up.data_ptr(), w_down.data_ptr(), int(w_gate.shape[0]))


def oda_bb_begin(ctx, emb, x, stream=None):
    check(_lib.load().oda_bb_begin(ctx.handle, _p(emb), _p(x), _s(stream)))


def oda_bb_qkv(ctx, layer: OdaBBLayer, x, q, k_new, v_new, stream=None):
    check(_lib.load().oda_bb_qkv(ctx.handle, ctypes.byref(layer), _p(x), _p(q), _p(k_new), _p(v_new),
                                 _s(stream)))


def oda_bb_attn_out(ctx, layer: OdaBBLayer, o, x, stream=None):
    check(_lib.load().oda_bb_attn_out(ctx.handle, ctypes.byref(layer), _p(o), _p(x), _s(stream)))


def oda_bb_pack_weight(ctx, src, dst, stream=None):
    """dst = src ([rows][cols] bf16, row-major) in the projections' packed layout."""
    rows, cols = src.shape
    if tuple(dst.shape) != (rows, cols) or src.element_size() != 2 or dst.element_size() != 2:
        raise ValueError("bb_pack_weight: src and dst must be bf16 matrices of one shape")
    check(_lib.load().oda_bb_pack_weight(ctx.handle, _p(src), rows, cols, _p(dst), _s(stream)))


def oda_bb_mlp(ctx, layer: OdaBBLayer, x, act, stream=None):
    check(_lib.load().oda_bb_mlp(ctx.handle, ctypes.byref(layer), _p(x), _p(act), _s(stream)))


def oda_bb_post_attention(ctx, layer: OdaBBLayer, next_layer, o, x, act, q=None, k_new=None, v_new=None,
                          stream=None):
    """attn_out(layer) + mlp(layer) + qkv(next_layer) as one cooperative launch; next_layer None
    stops after the MLP."""
    nxt = ctypes.byref(next_layer) if next_layer is not None else None
    check(_lib.load().oda_bb_post_attention(ctx.handle, ctypes.byref(layer), nxt, _p(o), _p(x), _p(act),
                                            _p(q), _p(k_new), _p(v_new), _s(stream)))


def oda_bb_final_norm(ctx, gamma, x, h, stream=None):
    check(_lib.load().oda_bb_final_norm(ctx.handle, _p(gamma), _p(x), _p(h), _s(stream)))


def oda_bb_lm_head(ctx, embed, vocab: int, h, logits, token, next_emb, stream=None):
    check(_lib.load().oda_bb_lm_head(ctx.handle, _p(embed), vocab, _p(h), _p(logits), _p(token),
                                     _p(next_emb), _s(stream)))


def oda_bb_embed(ctx, embed, vocab: int, token, emb, stream=None):
    check(_lib.load().oda_bb_embed(ctx.handle, _p(embed), vocab, _p(token), _p(emb), _s(stream)))
