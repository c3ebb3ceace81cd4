"""Shapes of the five synthetic decode workloads (and scaled-down copies for tests).

Data only: batch, layer layout, head counts, context lengths, step counts, routing mode
and seeds.  The Qwen3-shaped sizes follow the method notes' throughput and quality
setups (Qwen3-1.7B: 16 query / 8 KV heads; Qwen3-8B: 32 / 8 and 36 layers; the hybrid
Qwen3.5-2B: 24 layers of which 6 are softmax attention).
"""
from __future__ import annotations

import dataclasses
import json
import os
from dataclasses import dataclass, field

import numpy as np

from . import gen

PAGE = 16
HEAD_DIM = 128
SINKS = 4
WINDOW = 2048
GDN_HEADS = 16
GDN_DIM = 128
CONV_TAPS = 4
CONV_WIDTH = 2048

_HERE = os.path.dirname(os.path.abspath(__file__))
_CALIB = os.path.join(os.path.dirname(_HERE), "tests", "golden", "head_bias_calibration.json")


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    n_layers: int                 # backbone layers (attention + recurrent)
    attn_layers: tuple            # indices of the softmax-attention layers
    Hq: int
    Hkv: int
    ctx: tuple                    # cached tokens per sequence before the first decode step
    steps: int
    routing: str                  # "head" (gate on the score) or "bernoulli" (scheduled flags)
    rates: tuple = ()             # per-sequence recall rates when routing == "bernoulli"
    head_bias: float = 0.0        # output bias b_o of the recall head
    shuffle_pages: bool = False
    theta: float = 0.0
    sinks: int = SINKS
    window: int = WINDOW
    d: int = HEAD_DIM
    ffn: int = 0                  # synthetic backbone: gated-MLP width (0: no backbone weights)
    vocab: int = 0                # synthetic backbone: vocabulary (tied embedding / LM head)
    note: str = ""

    @property
    def backbone(self) -> bool:
        """True when every layer runs random-weight projections around attention (QKV from the
        residual, o_proj, gated MLP) and each step ends with the LM head."""
        return self.ffn > 0

    @property
    def D(self) -> int:
        """Hidden width = Hq * head_dim (also the recall head's input width)."""
        return self.Hq * self.d

    @property
    def L(self) -> int:
        return len(self.attn_layers)

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def gdn_layers(self) -> tuple:
        return tuple(i for i in range(self.n_layers) if i not in self.attn_layers)

    @property
    def hybrid(self) -> bool:
        return len(self.gdn_layers) > 0

    def shared_inputs(self, layer: int) -> bool:
        """True where both branches see the same layer input: no attention layer precedes it."""
        return layer <= min(self.attn_layers)

    def max_pages(self, extra_steps: int = 0) -> int:
        """Pages per sequence needed for ctx + steps (+ extra) tokens."""
        need = max(self.ctx) + self.steps + extra_steps + 1
        return (need + PAGE - 1) // PAGE

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _uniform_ints(seed: int, tag: int, n: int, lo: int, hi: int) -> tuple:
    u = gen.uniform_f64(gen.key(seed, tag), n)
    return tuple(int(lo + int(x * (hi - lo + 1))) for x in u)


def _uniform_floats(seed: int, tag: int, n: int, lo: float, hi: float) -> tuple:
    u = gen.uniform_f64(gen.key(seed, tag), n)
    return tuple(float(lo + (hi - lo) * x) for x in u)


def calibrated_bias(name: str, default: float = 0.0) -> float:
    """Output bias b_o stored by tests/golden/make_head_bias_calibration.py (oracle-computed)."""
    try:
        with open(_CALIB) as f:
            return float(json.load(f)[name]["b_o"])
    except (OSError, KeyError, ValueError):
        return default


def cfg0() -> Workload:
    return Workload("cfg0_qwen3_1p7b_layer_ctx4k", 1000, B=1, n_layers=1, attn_layers=(0,),
                    Hq=16, Hkv=8, ctx=(4096,), steps=8, routing="head",
                    note="single Qwen3-1.7B-shaped layer, context 4096, recall head routing")


def cfg1() -> Workload:
    return Workload("cfg1_28layer_ctx32k_b8", 1001, B=8, n_layers=28, attn_layers=tuple(range(28)),
                    Hq=16, Hkv=8, ctx=(32768,) * 8, steps=64, routing="head",
                    head_bias=calibrated_bias("cfg1_28layer_ctx32k_b8"),
                    note="28-layer stack, context 32768, head routing calibrated to ~40% recall")


def cfg2() -> Workload:
    return Workload("cfg2_qwen3_8b_ctx128k_b4_r0.125", 1002, B=4, n_layers=36,
                    attn_layers=tuple(range(36)), Hq=32, Hkv=8, ctx=(131072,) * 4, steps=32,
                    routing="bernoulli", rates=(0.125,) * 4,
                    note="Qwen3-8B-shaped attention, context 131072, Bernoulli(0.125) recall")


def cfg3() -> Workload:
    seed = 1003
    B = 32
    return Workload("cfg3_paged_divergent_b32", seed, B=B, n_layers=4, attn_layers=(0, 1, 2, 3),
                    Hq=16, Hkv=8, ctx=_uniform_ints(seed, gen.Tag.CTX, B, 8192, 131072), steps=64,
                    routing="bernoulli", rates=_uniform_floats(seed, gen.Tag.RATE, B, 0.05, 0.5),
                    shuffle_pages=True,
                    note="shuffled 16-token pages, context U[8192,131072], recall rate U[0.05,0.5]")


def cfg4() -> Workload:
    return Workload("cfg4_hybrid_6attn_18gdn_ctx64k_b8", 1004, B=8, n_layers=24,
                    attn_layers=(3, 7, 11, 15, 19, 23), Hq=16, Hkv=8, ctx=(65536,) * 8, steps=32,
                    routing="bernoulli", rates=(0.4,) * 8,
                    note="hybrid: 6 attention + 18 gated-delta layers, snapshot/restore, recall 0.4")


def bb_qwen3_1p7b(ctx: int = 131072, B: int = 1) -> Workload:
    """Whole decode step of a Qwen3-1.7B-shaped model with a synthetic frozen backbone: 28
    layers, hidden 2048 (16 query / 8 KV heads of 128), gated MLP 6144, vocabulary 151936 with
    tied embeddings, random bf16 weights; batch 1 and about 1/8 scheduled full calls as in the
    method notes' throughput setup, the head still run."""
    return Workload(f"bb_qwen3_1p7b_ctx{ctx // 1024}k_b{B}_r0.125", 1005, B=B, n_layers=28,
                    attn_layers=tuple(range(28)), Hq=16, Hkv=8, ctx=(ctx,) * B, steps=32,
                    routing="bernoulli", rates=(0.125,) * B, ffn=6144, vocab=151936,
                    note="synthetic Qwen3-1.7B-shaped backbone, LM head, Bernoulli(0.125) recall")


def cfg2_ctx32k_l2() -> Workload:
    """Profiling case of the 128K workload's kernels: same heads and batch, 2 layers, context
    32768 (1 GiB of cache: larger than L2, small enough for a many-pass profiler capture)."""
    return cfg2().replace(name="cfg2_profile_ctx32k_l2", n_layers=2, attn_layers=(0, 1),
                          ctx=(32768,) * 4, steps=8)


def cfg3_ctx8k_l2() -> Workload:
    """Profiling case of the divergent batch's kernels: the same 32 sequences and heads, 2 layers,
    context 8192 (2.1 GB of cache: larger than L2, small enough for a many-pass profiler capture)."""
    return cfg3().replace(name="cfg3_profile_ctx8k_l2", n_layers=2, attn_layers=(0, 1),
                          ctx=(8192,) * 32, steps=8)


def bb_qwen3_1p7b_l2() -> Workload:
    """Profiling case of the synthetic-backbone step: the same layer shapes, 2 layers, 4K
    context (under 1 GB on the device, so a many-pass profiler capture stays small)."""
    return bb_qwen3_1p7b(ctx=4096).replace(name="bb_qwen3_1p7b_ctx4k_l2", n_layers=2, attn_layers=(0, 1))


ALL = {"cfg0": cfg0, "cfg1": cfg1, "cfg2": cfg2, "cfg3": cfg3, "cfg4": cfg4,
       "cfg2_ctx32k_l2": cfg2_ctx32k_l2, "cfg3_ctx8k_l2": cfg3_ctx8k_l2, "bb": bb_qwen3_1p7b, "bb_l2": bb_qwen3_1p7b_l2}


def get(name: str) -> Workload:
    return ALL[name]()


def scaled(wl: Workload, *, ctx=None, steps=None, n_layers=None, B=None, name=None) -> Workload:
    """A smaller copy of a workload (for oracle-sized parity runs), same structure."""
    kw = {}
    if B is not None and B != wl.B:
        kw["B"] = B
        kw["ctx"] = tuple(wl.ctx[i % len(wl.ctx)] for i in range(B))
        if wl.rates:
            kw["rates"] = tuple(wl.rates[i % len(wl.rates)] for i in range(B))
    if ctx is not None:
        c = kw.get("ctx", wl.ctx)
        if isinstance(ctx, (int, np.integer)):
            kw["ctx"] = (int(ctx),) * len(c)
        else:
            kw["ctx"] = tuple(int(x) for x in ctx)
    if steps is not None:
        kw["steps"] = steps
    if n_layers is not None:
        if wl.hybrid:
            period = wl.n_layers // len(wl.attn_layers)
            kw["n_layers"] = n_layers
            kw["attn_layers"] = tuple(i for i in range(n_layers) if i % period == period - 1)
        else:
            kw["n_layers"] = n_layers
            kw["attn_layers"] = tuple(range(n_layers))
    kw["name"] = name or (wl.name + "_scaled")
    return dataclasses.replace(wl, **kw)
