"""Host-side generation of every seeded input of a decode workload (numpy arrays).

Each function returns the same values the device generator writes for the same key, so
the oracle can rebuild any slice that the CUDA path reads.  bf16 tensors are returned as
uint16 bit patterns; fp32 tensors as float32.

Synthetic stand-in for the frozen backbone (no trained weights exist): at every decode
step, every attention layer receives a seeded query q [B, Hq, 128] and current key/value
k, v [B, Hkv, 128] per branch (local / full); a layer that no attention layer precedes
gets the same draws in both branches, as a real backbone would.  Recurrent (gated-delta)
layers of the hybrid workload receive seeded conv inputs, values and gates the same way.
"""
from __future__ import annotations

import numpy as np

from . import gen
from .configs import CONV_TAPS, CONV_WIDTH, GDN_DIM, GDN_HEADS, PAGE, Workload

Tag = gen.Tag
LOCAL, FULL = 0, 1
TOWER = 1024
FFN = 2048


def _branch_id(wl: Workload, layer: int, branch: int) -> int:
    return 0 if wl.shared_inputs(layer) else branch


# ----------------------------------------------------------------------------- KV cache
def cache_key(wl: Workload, which: str, layer: int, b: int) -> int:
    tag = Tag.K_CACHE if which == "k" else Tag.V_CACHE
    return gen.key(wl.seed, tag, layer, b)


def cache_tokens(wl: Workload, which: str, layer: int, b: int, n_tokens: int,
                 start: int = 0) -> np.ndarray:
    """Prefilled cache of one (layer, sequence): tokens start..start+n-1, [n, Hkv, 128] bf16 bits."""
    per_tok = wl.Hkv * wl.d
    v = gen.normal_bf16(cache_key(wl, which, layer, b), n_tokens * per_tok, start * per_tok)
    return v.reshape(n_tokens, wl.Hkv, wl.d)


def page_table(wl: Workload, max_pages: int) -> np.ndarray:
    """[B, max_pages] int32 physical page ids into a pool of B * max_pages pages."""
    n = wl.B * max_pages
    if wl.shuffle_pages:
        perm = gen.permutation(gen.key(wl.seed, Tag.PAGES), n)
    else:
        perm = np.arange(n, dtype=np.int32)
    return perm.reshape(wl.B, max_pages).astype(np.int32)


# ------------------------------------------------------------------------ per-step inputs
def step_qkv(wl: Workload, step: int, layer: int, branch: int):
    """(q [B,Hq,128], k [B,Hkv,128], v [B,Hkv,128]) bf16 bits of the attention layer with
    backbone index ``layer`` (not its attention ordinal)."""
    br = _branch_id(wl, layer, branch)
    q = gen.normal_bf16(gen.key(wl.seed, Tag.Q, step, layer, br), wl.B * wl.Hq * wl.d)
    k = gen.normal_bf16(gen.key(wl.seed, Tag.K_NEW, step, layer, br), wl.B * wl.Hkv * wl.d)
    v = gen.normal_bf16(gen.key(wl.seed, Tag.V_NEW, step, layer, br), wl.B * wl.Hkv * wl.d)
    return (q.reshape(wl.B, wl.Hq, wl.d), k.reshape(wl.B, wl.Hkv, wl.d),
            v.reshape(wl.B, wl.Hkv, wl.d))


def qkv_keys(wl: Workload, step: int, layer: int, branch: int):
    br = _branch_id(wl, layer, branch)
    return (gen.key(wl.seed, Tag.Q, step, layer, br), gen.key(wl.seed, Tag.K_NEW, step, layer, br),
            gen.key(wl.seed, Tag.V_NEW, step, layer, br))


def emb(wl: Workload, step: int) -> np.ndarray:
    """E(x_t) stand-in: [B, D] fp32 N(0,1)."""
    return gen.normal_f32(gen.key(wl.seed, Tag.EMB, step), wl.B * wl.D).reshape(wl.B, wl.D)


def h_prev0(wl: Workload) -> np.ndarray:
    """Hidden state chosen at the step before the first routed step: [B, D] fp32 N(0,1)."""
    return gen.normal_f32(gen.key(wl.seed, Tag.H_PREV0), wl.B * wl.D).reshape(wl.B, wl.D)


def schedule(wl: Workload, step: int):
    """Scheduled recall flags [B] int32 (Bernoulli(rate_b)), or None for head routing."""
    if wl.routing != "bernoulli":
        return None
    return gen.bernoulli(gen.key(wl.seed, Tag.SCHED, step), wl.B, np.asarray(wl.rates))


# ---------------------------------------------------------------------------- recall head
def head_shapes(D: int) -> list:
    """(name, shape) of every recall-head tensor, in storage order."""
    s = []
    for i in range(3):
        s += [(f"tower_norm{i}", (D,)), (f"tower_w{i}", (TOWER, D)), (f"tower_b{i}", (TOWER,))]
    s += [("fuse_w", (TOWER, 9 * TOWER)), ("fuse_b", (TOWER,))]
    for j in range(2):
        s += [(f"ffn_norm{j}", (TOWER,)), (f"ffn_gate{j}", (FFN, TOWER)),
              (f"ffn_up{j}", (FFN, TOWER)), (f"ffn_down{j}", (TOWER, FFN))]
    s += [("out_norm", (TOWER,)), ("out_w", (TOWER,)), ("out_b", (1,))]
    return s


def head_weights(wl: Workload, perturb: bool = False) -> dict:
    """Recall-head parameters: Xavier-uniform matrices, zero biases, unit norm weights.

    ``perturb`` also draws the norm weights from U(0.5, 1.5) and the biases from
    U(-0.1, 0.1), so that tests exercise every parameter.  out_b is the workload's b_o.
    """
    out = {}
    for idx, (name, shape) in enumerate(head_shapes(wl.D)):
        k = gen.key(wl.seed, Tag.HEAD_W, idx)
        n = int(np.prod(shape))
        if name == "out_b":
            a = np.full(1, wl.head_bias, dtype=np.float32)
            if perturb:
                a = a + gen.uniform_f32(k, 1, -0.1, 0.1)
        elif "norm" in name:
            a = gen.uniform_f32(k, n, 0.5, 1.5) if perturb else np.ones(n, np.float32)
        elif name.endswith("_b") or name.startswith("tower_b") or name == "fuse_b":
            a = gen.uniform_f32(k, n, -0.1, 0.1) if perturb else np.zeros(n, np.float32)
        elif name == "out_w":
            a = gen.xavier_uniform(k, 1, TOWER).reshape(n)
        else:
            a = gen.xavier_uniform(k, shape[0], shape[1])
        out[name] = np.ascontiguousarray(a.reshape(shape), dtype=np.float32)
    return out


def head_param_count(D: int) -> int:
    return int(sum(int(np.prod(s)) for _, s in head_shapes(D)))


# ------------------------------------------------------------------- gated-delta layers
def gdn_step_inputs(wl: Workload, step: int, layer: int, branch: int):
    """Inputs of one recurrent layer: conv input c [B,2048], value v [B,16,128],
    decay alpha [B,16] ~ U(0.9,1), write strength beta [B,16] ~ U(0,1); all fp32."""
    br = _branch_id(wl, layer, branch)
    B = wl.B
    c = gen.normal_f32(gen.key(wl.seed, Tag.GDN_C, step, layer, br), B * CONV_WIDTH)
    v = gen.normal_f32(gen.key(wl.seed, Tag.GDN_V, step, layer, br), B * GDN_HEADS * GDN_DIM)
    a = gen.uniform_f32(gen.key(wl.seed, Tag.GDN_ALPHA, step, layer, br), B * GDN_HEADS, 0.9, 1.0)
    be = gen.uniform_f32(gen.key(wl.seed, Tag.GDN_BETA, step, layer, br), B * GDN_HEADS, 0.0, 1.0)
    return (c.reshape(B, CONV_WIDTH), v.reshape(B, GDN_HEADS, GDN_DIM),
            a.reshape(B, GDN_HEADS), be.reshape(B, GDN_HEADS))


def gdn_taps(wl: Workload, layer: int) -> np.ndarray:
    """Depthwise causal conv taps [4, 2048] fp32 ~ U(-0.5, 0.5)."""
    return gen.uniform_f32(gen.key(wl.seed, Tag.GDN_TAPS, layer), CONV_TAPS * CONV_WIDTH,
                           -0.5, 0.5).reshape(CONV_TAPS, CONV_WIDTH)


def gdn_state0(wl: Workload):
    """Initial recurrent state [B, n_gdn, 16, 128, 128] ~ N(0, 1/128) and conv state
    [B, n_gdn, 4, 2048] ~ N(0, 1), fp32."""
    n = len(wl.gdn_layers)
    B = wl.B
    s = gen.normal_f32(gen.key(wl.seed, Tag.GDN_STATE0), B * n * GDN_HEADS * GDN_DIM * GDN_DIM)
    s = (s * np.float32(1.0 / np.sqrt(GDN_DIM))).astype(np.float32)
    c = gen.normal_f32(gen.key(wl.seed, Tag.GDN_CONV0), B * n * CONV_TAPS * CONV_WIDTH)
    return (s.reshape(B, n, GDN_HEADS, GDN_DIM, GDN_DIM), c.reshape(B, n, CONV_TAPS, CONV_WIDTH))


def n_pages_for(tokens: int) -> int:
    return (tokens + PAGE - 1) // PAGE


# ------------------------------------------------------------ synthetic backbone weights
BB_TENSORS = ("w_qkv", "w_o", "w_gate", "w_up", "w_down")


def bb_shapes(wl: Workload) -> dict:
    """[rows, cols] of each bf16 projection of one layer (row-major [out][in])."""
    D, F = wl.D, wl.ffn
    return {"w_qkv": ((wl.Hq + 2 * wl.Hkv) * wl.d, D), "w_o": (D, wl.Hq * wl.d),
            "w_gate": (F, D), "w_up": (F, D), "w_down": (D, F)}


def bb_log2_scale(fan_in: int) -> int:
    """Weights are N(0,1) times 2^-floor(log2(fan_in) / 2), about 1/sqrt(fan_in) as an exact
    power of two, so the device fill and this generator agree bit for bit."""
    return -(int(np.log2(fan_in)) // 2)


def bb_weight_key(wl: Workload, layer: int, name: str) -> int:
    return gen.key(wl.seed, Tag.BB_W, layer, BB_TENSORS.index(name))


def bb_weight(wl: Workload, layer: int, name: str, rows=None) -> np.ndarray:
    """One projection (bf16 bits [rows, cols]), or rows r0..r1-1 of it if rows = (r0, r1)."""
    R, C = bb_shapes(wl)[name]
    r0, r1 = rows if rows is not None else (0, R)
    v = gen.normal_bf16(bb_weight_key(wl, layer, name), (r1 - r0) * C, r0 * C, bb_log2_scale(C))
    return v.reshape(r1 - r0, C)


def bb_norms(wl: Workload, layer: int) -> tuple:
    """(attention-input norm weight, MLP-input norm weight), fp32 [D] ~ U(0.5, 1.5); layer -1
    gives the final norm's weight in both slots."""
    a = gen.uniform_f32(gen.key(wl.seed, Tag.BB_NORM, layer, 0), wl.D, 0.5, 1.5)
    m = gen.uniform_f32(gen.key(wl.seed, Tag.BB_NORM, layer, 1), wl.D, 0.5, 1.5)
    return a, m


# The embedding table is N(0,1) * 2^-3: with tied N(0,1) rows the token's own row dominates the
# residual stream and greedy decoding of random weights repeats one token; at 1/8 the layers'
# contributions decide the next token.
BB_EMBED_LOG2_SCALE = -3


def bb_embed_key(wl: Workload) -> int:
    return gen.key(wl.seed, Tag.BB_EMBED)


def bb_embed_rows(wl: Workload, tokens) -> np.ndarray:
    """Rows of the embedding table (bf16 bits [len(tokens), D])."""
    out = np.empty((len(tokens), wl.D), np.uint16)
    for i, t in enumerate(tokens):
        out[i] = gen.normal_bf16(bb_embed_key(wl), wl.D, int(t) * wl.D, BB_EMBED_LOG2_SCALE)
    return out


def bb_embed(wl: Workload) -> np.ndarray:
    """The whole embedding table, bf16 bits [vocab, D] (small vocabularies only)."""
    return gen.normal_bf16(bb_embed_key(wl), wl.vocab * wl.D, 0,
                           BB_EMBED_LOG2_SCALE).reshape(wl.vocab, wl.D)


def bb_token0(wl: Workload) -> np.ndarray:
    """First token of each sequence, int32 [B] uniform over the vocabulary."""
    u = gen.uniform_f64(gen.key(wl.seed, Tag.TOKEN0), wl.B)
    return np.minimum((u * wl.vocab).astype(np.int64), wl.vocab - 1).astype(np.int32)
