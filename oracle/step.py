"""One ODA decode step over explicit state, with deep copies and no in-place sharing.

[notes §2.3] (first and third paragraphs, eq. h_t / p_t / C_t):
  1. run the local forward pass (index set S^L in every restricted attention layer);
  2. score it with the recall head; route full iff the score exceeds theta or is non-finite
     (or take the scheduled flag, as in the throughput setup of [notes §3.3], where the head
     still runs but the full calls are scheduled by hand);
  3. the full recompute starts from the SAME pre-step state, not from the local pass's
     scratch state: each layer's current K,V are staged, not written; for hybrid backbones
     the conv and recurrent states are snapshotted before the local pass and restored before
     the retry;
  4. commit: h_t = h_t^{b_t}; C_t = C_{t-1} || Delta C_t^{b_t} - only the chosen branch's
     staged K,V go to the cache (one position per sequence), and the recurrent update kept
     is the chosen branch's; output and cache always come from the same branch.

The synthetic backbone (weights are not available): residual x = E(x_t) + sum over layers of
the layer outputs (attention o reshaped to Hq*128, recurrent o), h = RMSNorm(x) without
weight (eps 1e-6) = the "last-layer normalised hidden" the head reads [notes §2.2].
Per-layer queries and current K/V are the workload's seeded draws (workload/inputs.py).
"""
from __future__ import annotations

import copy
from dataclasses import dataclass, field

import numpy as np

from workload import inputs as wi
from workload.configs import Workload

import functools

from . import backbone as BB
from . import kv_fp8
from .attention import append_current, attend, attend_bits, bf16_to_f64
from .delta import gdn_layer
from .gate import route_full
from .head import recall_head, rmsnorm
from .sets import full_set, local_set

LOCAL, FULL = 0, 1


@dataclass
class OracleState:
    pos: list                      # t per sequence: 1-based position of the token being decoded
    h_prev: np.ndarray             # [B, D] fp64: previous step's chosen final hidden
    k_cache: list                  # [attention layer][b] -> uint16 [t-1, Hkv, 128]
    v_cache: list
    gdn_S: np.ndarray = None       # [B, n_gdn, 16, 128, 128] fp64
    gdn_conv: np.ndarray = None    # [B, n_gdn, 4, 2048] fp64
    kv: str = "bf16"               # "bf16": caches hold bf16 bits; "fp8": caches hold the
                                   # decoded values (fp64) of rows stored as e4m3 + scale
    tokens: np.ndarray = None      # synthetic backbone: the current token x_t of each sequence
    emb: np.ndarray = None         # synthetic backbone: E(x_t) [B, D] fp64


@dataclass
class StepRecord:
    scores: np.ndarray
    flags: np.ndarray
    o: dict = field(default_factory=dict)      # (branch, attention ordinal) -> [B, Hq, 128]
    h: dict = field(default_factory=dict)      # branch -> [B, D]
    staged_k: dict = field(default_factory=dict)   # (branch, ordinal) -> uint16 [B, Hkv, 128]
    staged_v: dict = field(default_factory=dict)
    staged_q: dict = field(default_factory=dict)   # synthetic backbone: (branch, ordinal) -> q bits
    logits: np.ndarray = None      # synthetic backbone: LM head on the committed hidden
    tokens: np.ndarray = None      # synthetic backbone: x_{t+1} (greedy)


def _stored(bits: np.ndarray, kv: str) -> np.ndarray:
    """A cache row block as the cache holds it: bf16 bits, or (fp8) the decoded values of its
    quantised rows (oracle.kv_fp8's format)."""
    if kv == "bf16":
        return bits
    codes, scales = kv_fp8.quantize_rows(bf16_to_f64(bits))
    return kv_fp8.dequantize_rows(codes, scales)


def initial_state(wl: Workload, kv: str = "bf16") -> OracleState:
    """Prefilled caches (ctx_b tokens each), h_{t-1} and recurrent state from the generator.
    kv = "fp8": the prefilled rows are stored quantised (the cache holds their decoded values)."""
    kc, vc = [], []
    for a in range(wl.L):
        kc.append([_stored(wi.cache_tokens(wl, "k", a, b, wl.ctx[b]), kv) for b in range(wl.B)])
        vc.append([_stored(wi.cache_tokens(wl, "v", a, b, wl.ctx[b]), kv) for b in range(wl.B)])
    st = OracleState(pos=[c + 1 for c in wl.ctx], h_prev=wi.h_prev0(wl).astype(np.float64),
                     k_cache=kc, v_cache=vc, kv=kv)
    if wl.backbone:
        st.tokens = wi.bb_token0(wl)
        st.emb = bf16_to_f64(wi.bb_embed_rows(wl, st.tokens))
    if wl.hybrid:
        S, C = wi.gdn_state0(wl)
        st.gdn_S = S.astype(np.float64)
        st.gdn_conv = C.astype(np.float64)
    return st


def snapshot(state: OracleState):
    """Copy of the recurrent and conv state (the part a pass advances in place)."""
    if state.gdn_S is None:
        return None
    return (state.gdn_S.copy(), state.gdn_conv.copy())


def restore(snap, state: OracleState, flags) -> None:
    """Put the snapshotted pre-step state back for the flagged sequences only."""
    if snap is None:
        return
    for b, f in enumerate(flags):
        if f:
            state.gdn_S[b] = snap[0][b]
            state.gdn_conv[b] = snap[1][b]


@functools.lru_cache(maxsize=2)
def backbone_weights(wl: Workload):
    """The synthetic backbone's weights (bf16 bits / fp32 norms) per attention layer, the final
    norm weight and the embedding table, from the seeded generators."""
    layers = []
    for layer in wl.attn_layers:
        w = {name: wi.bb_weight(wl, layer, name) for name in wi.BB_TENSORS}
        w["attn_norm"], w["mlp_norm"] = wi.bb_norms(wl, layer)
        layers.append(w)
    return layers, wi.bb_norms(wl, -1)[0], wi.bb_embed(wl)


def run_backbone_pass(wl: Workload, state: OracleState, branch: int, active, rec: StepRecord):
    """One pass of the synthetic backbone (oracle.backbone) from the pre-step residual E(x_t):
    per layer q/k/v from the residual, attention over S^L or S^F for the sequences in
    ``active``, o_proj and the MLP; returns h = the final norm of the residual."""
    layers, g_final, _ = backbone_weights(wl)
    B, D = wl.B, wl.D
    x = state.emb.copy()
    for a, layer in enumerate(wl.attn_layers):
        w = layers[a]
        q, k, v = BB.attn_in(x, w["attn_norm"], w["w_qkv"], wl.Hq, wl.Hkv)
        rec.staged_q[(branch, a)] = q
        rec.staged_k[(branch, a)] = k
        rec.staged_v[(branch, a)] = v
        o = np.full((B, wl.Hq, wl.d), np.nan)
        for b in active:
            t = state.pos[b]
            S = local_set(t, wl.sinks, wl.window) if branch == LOCAL else full_set(t)
            if state.kv == "bf16":
                o[b] = attend_bits(q[b], state.k_cache[a][b], state.v_cache[a][b], k[b], v[b], S)
            else:
                o[b] = attend(bf16_to_f64(q[b]), append_current(state.k_cache[a][b], bf16_to_f64(k[b])),
                              append_current(state.v_cache[a][b], bf16_to_f64(v[b])), S)
        rec.o[(branch, a)] = o
        x = BB.attn_out(x, o.reshape(B, D), w["w_o"])
        x = BB.mlp(x, w["mlp_norm"], w["w_gate"], w["w_up"], w["w_down"])
    h = np.full((B, D), np.nan)
    for b in active:
        h[b] = BB.rmsnorm(x[b], g_final)
    rec.h[branch] = h
    return h


def run_pass(wl: Workload, state: OracleState, step: int, branch: int, active, rec: StepRecord):
    """One forward pass of the synthetic backbone for the sequences in ``active``.

    Attention layers read the committed cache plus the branch's staged current K,V over
    S^L (local) or S^F (full); recurrent layers advance ``state``'s gdn arrays in place.
    Returns h [B, D] (rows of inactive sequences are NaN).
    """
    if wl.backbone:
        return run_backbone_pass(wl, state, branch, active, rec)
    B, D = wl.B, wl.D
    e = wi.emb(wl, step).astype(np.float64)
    x = e.copy()
    a = 0
    gdn_j = 0
    for layer in range(wl.n_layers):
        if layer in wl.attn_layers:
            q, k, v = wi.step_qkv(wl, step, layer, branch)
            rec.staged_k[(branch, a)] = k
            rec.staged_v[(branch, a)] = v
            o = np.full((B, wl.Hq, wl.d), np.nan)
            for b in active:
                t = state.pos[b]
                S = local_set(t, wl.sinks, wl.window) if branch == LOCAL else full_set(t)
                if state.kv == "bf16":
                    o[b] = attend_bits(q[b], state.k_cache[a][b], state.v_cache[a][b], k[b], v[b], S)
                else:   # stored rows decoded; the current token exactly as this branch computed it
                    o[b] = attend(bf16_to_f64(q[b]),
                                  append_current(state.k_cache[a][b], bf16_to_f64(k[b])),
                                  append_current(state.v_cache[a][b], bf16_to_f64(v[b])), S)
                x[b] += o[b].reshape(D)
            rec.o[(branch, a)] = o
            a += 1
        else:
            c, vv, al, be = wi.gdn_step_inputs(wl, step, layer, branch)
            taps = wi.gdn_taps(wl, layer).astype(np.float64)
            for b in active:
                S_new, conv_new, o = gdn_layer(state.gdn_S[b, gdn_j], state.gdn_conv[b, gdn_j],
                                               c[b].astype(np.float64), vv[b].astype(np.float64),
                                               al[b].astype(np.float64), be[b].astype(np.float64),
                                               taps)
                state.gdn_S[b, gdn_j] = S_new
                state.gdn_conv[b, gdn_j] = conv_new
                x[b] += o
            gdn_j += 1
    h = np.full((B, D), np.nan)
    for b in active:
        h[b] = rmsnorm(x[b])
    rec.h[branch] = h
    return h


def decode_step(wl: Workload, state: OracleState, step: int, head_params: dict,
                sched=None):
    """One routed decode step.  Returns (new_state, StepRecord); ``state`` is not modified."""
    live = copy.deepcopy(state)
    B = wl.B
    snap = snapshot(live)
    rec = StepRecord(scores=np.zeros(B), flags=np.zeros(B, dtype=np.int32))
    h_loc = run_pass(wl, live, step, LOCAL, range(B), rec)
    e = live.emb if wl.backbone else wi.emb(wl, step).astype(np.float64)
    for b in range(B):
        rec.scores[b] = recall_head(head_params, live.h_prev[b], e[b], h_loc[b])
        full = route_full(rec.scores[b], wl.theta) if sched is None else bool(sched[b])
        rec.flags[b] = 1 if full else 0
    flagged = [b for b in range(B) if rec.flags[b]]
    restore(snap, live, rec.flags)
    run_pass(wl, live, step, FULL, flagged, rec)
    commit(wl, live, rec)
    if wl.backbone:
        # [notes §2.3, eq. p_t]: the output distribution once, from the committed hidden h_t
        _, _, E = backbone_weights(wl)
        rec.logits, rec.tokens = BB.lm_head(live.h_prev, E)
        live.tokens = rec.tokens
        live.emb = bf16_to_f64(E[rec.tokens])
    return live, rec


def commit(wl: Workload, state: OracleState, rec: StepRecord) -> None:
    """Append the chosen branch's staged K,V at position t, take its hidden, advance t."""
    for b in range(wl.B):
        br = FULL if rec.flags[b] else LOCAL
        for a in range(wl.L):
            state.k_cache[a][b] = np.concatenate(
                [state.k_cache[a][b], _stored(rec.staged_k[(br, a)][b], state.kv)[None]], axis=0)
            state.v_cache[a][b] = np.concatenate(
                [state.v_cache[a][b], _stored(rec.staged_v[(br, a)][b], state.kv)[None]], axis=0)
        state.h_prev[b] = rec.h[br][b]
        state.pos[b] += 1


def fresh_full_step(wl: Workload, state: OracleState, step: int):
    """Full pass for every sequence from a fresh copy of the pre-step state (no snapshot,
    no local pass): the reference the transactional retry must equal."""
    live = copy.deepcopy(state)
    rec = StepRecord(scores=np.zeros(wl.B), flags=np.ones(wl.B, dtype=np.int32))
    run_pass(wl, live, step, FULL, range(wl.B), rec)
    return live, rec
