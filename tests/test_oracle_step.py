"""Pins of oracle.step: commit invariants, retry-from-pre-step-state, local = full where the
sets coincide, scheduled routing, and the gate's use of the head score."""
import copy

import numpy as np
import pytest

from oracle import step as S
from oracle.gate import route_full
from oracle.sets import full_set, local_set
from workload import configs, inputs


def _small_attn(ctx=(40, 2100), L=2, steps=2, routing="bernoulli", rates=(0.5, 0.5)):
    wl = configs.cfg0().replace(name="t_small", B=len(ctx), n_layers=L,
                                attn_layers=tuple(range(L)), ctx=tuple(ctx), steps=steps,
                                routing=routing, rates=tuple(rates))
    return wl


def _small_head(wl, seed=7):
    return inputs.head_weights(wl, perturb=True)


def _force(wl, flags):
    return np.asarray(flags, dtype=np.int32)


def test_commit_appends_exactly_the_chosen_branch():
    wl = _small_attn(ctx=(40, 2100, 2200), L=2, rates=(0.5,) * 3)
    P = _small_head(wl)
    st0 = S.initial_state(wl)
    flags = [1, 0, 1]
    st1, rec = S.decode_step(wl, st0, 0, P, sched=_force(wl, flags))
    assert rec.flags.tolist() == flags
    for b in range(wl.B):
        br = S.FULL if flags[b] else S.LOCAL
        other = S.LOCAL if flags[b] else S.FULL
        assert st1.pos[b] == st0.pos[b] + 1
        assert np.array_equal(st1.h_prev[b], rec.h[br][b])
        for a in range(wl.L):
            kc0, kc1 = st0.k_cache[a][b], st1.k_cache[a][b]
            assert kc1.shape[0] == kc0.shape[0] + 1
            assert np.array_equal(kc1[:-1], kc0) and np.array_equal(st1.v_cache[a][b][:-1],
                                                                      st0.v_cache[a][b])
            assert np.array_equal(kc1[-1], rec.staged_k[(br, a)][b])
            assert np.array_equal(st1.v_cache[a][b][-1], rec.staged_v[(br, a)][b])
            if a > 0:  # layer 0 inputs are shared; later layers differ between branches
                assert not np.array_equal(kc1[-1], rec.staged_k[(other, a)][b])
    # the input state is untouched
    assert st0.pos == [c + 1 for c in wl.ctx]


def test_local_equals_full_where_sets_coincide():
    wl = _small_attn(ctx=(100, 2051), L=1)
    P = _small_head(wl)
    st = S.initial_state(wl)
    _, rec = S.decode_step(wl, st, 0, P, sched=_force(wl, [1, 1]))
    for b in range(wl.B):
        t = st.pos[b]
        assert local_set(t) == full_set(t)
        assert np.array_equal(rec.o[(S.LOCAL, 0)][b], rec.o[(S.FULL, 0)][b])
        assert np.array_equal(rec.h[S.LOCAL][b], rec.h[S.FULL][b])


def test_local_differs_from_full_beyond_2052():
    wl = _small_attn(ctx=(2200,), L=1)
    P = _small_head(wl)
    _, rec = S.decode_step(wl, S.initial_state(wl), 0, P, sched=_force(wl, [1]))
    assert not np.allclose(rec.o[(S.LOCAL, 0)][0], rec.o[(S.FULL, 0)][0])


def test_gate_routes_on_the_head_score():
    wl = _small_attn(ctx=(30, 60, 90, 120), L=1, routing="head")
    P = _small_head(wl)
    st = S.initial_state(wl)
    _, rec = S.decode_step(wl, st, 0, P)
    assert rec.flags.tolist() == [int(route_full(q)) for q in rec.scores]
    # shifting b_o moves every decision the same way
    hi = dict(P, out_b=P["out_b"] + 100.0)
    lo = dict(P, out_b=P["out_b"] - 100.0)
    assert S.decode_step(wl, st, 0, hi)[1].flags.tolist() == [1] * 4
    assert S.decode_step(wl, st, 0, lo)[1].flags.tolist() == [0] * 4
    nan = dict(P, out_b=np.array([np.nan]))
    assert S.decode_step(wl, st, 0, nan)[1].flags.tolist() == [1] * 4


def _small_hybrid(B=2):
    wl = configs.cfg4()
    return wl.replace(name="t_hybrid", B=B, n_layers=4, attn_layers=(1, 3), ctx=(50,) * B,
                      rates=(0.5,) * B, steps=2)


def test_restore_then_retry_equals_fresh_full_step():
    wl = _small_hybrid(B=2)
    P = _small_head(wl)
    st0 = S.initial_state(wl)
    st1, rec = S.decode_step(wl, st0, 0, P, sched=np.array([1, 0], np.int32))
    fresh, frec = S.fresh_full_step(wl, st0, 0)
    # flagged sequence: the committed state and hidden equal a fresh full step, bit for bit
    assert np.array_equal(st1.gdn_S[0], fresh.gdn_S[0])
    assert np.array_equal(st1.gdn_conv[0], fresh.gdn_conv[0])
    assert np.array_equal(rec.h[S.FULL][0], frec.h[S.FULL][0])
    assert np.array_equal(st1.h_prev[0], frec.h[S.FULL][0])
    # unflagged sequence: advanced exactly once, by the local branch
    wl_local = copy.deepcopy(st0)
    r2 = S.StepRecord(scores=np.zeros(2), flags=np.zeros(2, np.int32))
    S.run_pass(wl, wl_local, 0, S.LOCAL, [1], r2)
    assert np.array_equal(st1.gdn_S[1], wl_local.gdn_S[1])
    assert not np.array_equal(st1.gdn_S[1], st0.gdn_S[1])
    assert np.array_equal(st1.h_prev[1], r2.h[S.LOCAL][1])


def test_without_restore_the_state_would_advance_twice():
    """The failure mode the page warns about: a retry from the local scratch state differs."""
    wl = _small_hybrid(B=1)
    st0 = S.initial_state(wl)
    live = copy.deepcopy(st0)
    r = S.StepRecord(scores=np.zeros(1), flags=np.ones(1, np.int32))
    S.run_pass(wl, live, 0, S.LOCAL, [0], r)
    S.run_pass(wl, live, 0, S.FULL, [0], r)          # no restore in between
    fresh, _ = S.fresh_full_step(wl, st0, 0)
    assert not np.allclose(live.gdn_S[0], fresh.gdn_S[0])


def test_snapshot_restore_masks_by_flag():
    wl = _small_hybrid(B=3)
    st = S.initial_state(wl)
    snap = S.snapshot(st)
    st.gdn_S += 1.0
    st.gdn_conv -= 1.0
    S.restore(snap, st, [1, 0, 1])
    assert np.array_equal(st.gdn_S[0], snap[0][0]) and np.array_equal(st.gdn_S[2], snap[0][2])
    assert np.array_equal(st.gdn_S[1], snap[0][1] + 1.0)
    assert np.array_equal(st.gdn_conv[1], snap[1][1] - 1.0)


def test_multi_step_trajectory_counts():
    wl = _small_attn(ctx=(20, 33), L=1, steps=3)
    P = _small_head(wl)
    st = S.initial_state(wl)
    n_routed = 0
    for s in range(wl.steps):
        st, _ = S.decode_step(wl, st, s, P, sched=inputs.schedule(wl, s))
        n_routed += 1
    assert st.pos == [c + 1 + wl.steps for c in wl.ctx]
    assert [st.k_cache[0][b].shape[0] for b in range(2)] == [c + wl.steps for c in wl.ctx]
    assert n_routed == wl.steps


def test_fp8_cache_commits_the_decoded_quantised_row_and_tracks_bf16():
    """fp8 mode: the commit appends the chosen row as stored (quantised, decoded), the cache's
    older rows are untouched, and every attention output stays within the format's error of the
    bf16-cache step (same inputs, same routing)."""
    from oracle import kv_fp8
    from oracle.attention import bf16_to_f64
    wl = _small_attn(ctx=(40, 2100), L=2, rates=(1.0, 1.0))
    P = _small_head(wl)
    s8 = S.initial_state(wl, kv="fp8")
    s16 = S.initial_state(wl)
    # prefilled rows: every stored row is within e4m3's half step (2^-4 relative) of bf16's
    for a in range(wl.L):
        for b in range(wl.B):
            x = bf16_to_f64(s16.k_cache[a][b])
            d = np.abs(s8.k_cache[a][b] - x)
            assert np.all(d <= 2.0 ** -4 * np.maximum(np.abs(x), np.max(np.abs(x), axis=-1, keepdims=True) / 448 * 2.0 ** -6) + 1e-12)
    n8, rec8 = S.decode_step(wl, s8, 0, P, sched=_force(wl, [1, 0]))
    n16, rec16 = S.decode_step(wl, s16, 0, P, sched=_force(wl, [1, 0]))
    for b, br in ((0, S.FULL), (1, S.LOCAL)):
        for a in range(wl.L):
            row = rec8.staged_k[(br, a)][b]
            c, sc = kv_fp8.quantize_rows(bf16_to_f64(row))
            assert np.array_equal(n8.k_cache[a][b][-1], kv_fp8.dequantize_rows(c, sc))
            assert np.array_equal(n8.k_cache[a][b][:-1], s8.k_cache[a][b])
    for key, o in rec8.o.items():
        for b in range(wl.B):
            if key[0] == S.FULL and b == 1:
                continue
            r = np.linalg.norm(o[b] - rec16.o[key][b]) / np.linalg.norm(rec16.o[key][b])
            assert r < 0.08, (key, b, r)
