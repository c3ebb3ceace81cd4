"""GPU parity at full size for the divergent batch and the hybrid stack, in the launch
configuration bench.py times (one CUDA graph per step with the retry under a conditional node,
layer overlap on).  The oracle checks, from slices it regenerates with the seeded generator:

* divergent batch (32 sequences, contexts U[8K, 128K], shuffled 16-token pages, 4 layers): routing
  equals the schedule, every committed K/V is bit-exact, the local outputs of every layer and
  the recall score for the shortest, the longest and two more sequences, and the full-branch
  output of the shortest and the longest flagged sequences;
* hybrid stack (6 attention + 18 gated-delta layers, context 65536, batch 8): two steps through
  the ping-pong state buffers; for one flagged and one unflagged sequence of the second step the
  whole layer stack (attention outputs, gated-delta outputs, the recall score) and the
  recurrent and conv state after each step (relative L2 1e-5, the fp32 update's bar), and every
  committed K/V bit-exact.
"""
import numpy as np
import pytest
import torch

from helpers import attn_close, build_all, score_close
from oracle.attention import attend_bits
from oracle.delta import gdn_layer
from oracle.head import recall_head, rmsnorm
from oracle.sets import full_set, local_set
from workload import configs, inputs

pytestmark = pytest.mark.gpu
LOCAL, FULL = 0, 1


@pytest.fixture(scope="module", autouse=True)
def _build():
    build_all()


def _rows(wl, a, b, t, which, committed=None):
    """Cached rows (1-based positions < t) of the set as a compact array, in position order:
    prefilled rows regenerated, rows committed by earlier steps from `committed`."""
    S = sorted(p - 1 for p in (local_set(t, wl.sinks, wl.window) if which == LOCAL else full_set(t))
               if p < t)
    pre = [r for r in S if r < wl.ctx[b]]
    ks, vs = [], []
    if pre:
        lo = prev = pre[0]
        for r in pre[1:] + [None]:
            if r is None or r != prev + 1:
                ks.append(inputs.cache_tokens(wl, "k", a, b, prev + 1 - lo, start=lo))
                vs.append(inputs.cache_tokens(wl, "v", a, b, prev + 1 - lo, start=lo))
                lo = r
            prev = r
    for r in S:
        if r >= wl.ctx[b]:
            ks.append(committed[(a, b, r)][0][None])
            vs.append(committed[(a, b, r)][1][None])
    return np.concatenate(ks), np.concatenate(vs)


def _attend(wl, a, b, t, q, k, v, which, committed=None):
    kc, vc = _rows(wl, a, b, t, which, committed)
    return attend_bits(q, kc, vc, k, v, full_set(kc.shape[0] + 1))


def _committed_rows(dec, wl, rows_per_seq):
    pt = dec.page_table.cpu().numpy()
    out = {}
    for a in range(wl.L):
        kp, vp = dec.k_pool[a], dec.v_pool[a]
        for b in range(wl.B):
            for row in rows_per_seq(b):
                page, slot = pt[b, row // 16], row % 16
                out[(a, b, row)] = (kp[page, :, slot].cpu().view(torch.int16).numpy().view(np.uint16),
                                    vp[page, :, slot].cpu().view(torch.int16).numpy().view(np.uint16))
    return out


def test_divergent_batch_full_size():
    from conditional_sparse_attention_b200.engine import OdaDecoder
    wl = configs.cfg3()
    s = next(s for s in range(0, 200) if inputs.schedule(wl, s).sum() >= 4)
    dec = OdaDecoder(wl, capacity_steps=4)
    dec.capture()
    buf = dec.make_step_buffer(s)
    dec.step(buf)
    dec.synchronize()
    flag = dec.flag.cpu().numpy().copy()
    score = dec.score.cpu().numpy().copy()
    o = dec.o.cpu().numpy().copy()
    assert dec.device_error() == 0
    assert dec.pos.cpu().tolist() == [c + 2 for c in wl.ctx]
    got = _committed_rows(dec, wl, lambda b: [wl.ctx[b]])
    head = {k: v.cpu().numpy() for k, v in dec.head_params.items()}
    dec.close()
    del dec
    torch.cuda.empty_cache()

    sched = inputs.schedule(wl, s)
    assert flag.tolist() == sched.tolist()
    staged = {(br, a): inputs.step_qkv(wl, s, layer, br) for br in (LOCAL, FULL)
              for a, layer in enumerate(wl.attn_layers)}
    for a in range(wl.L):
        for b in range(wl.B):
            br = FULL if sched[b] else LOCAL
            gk, gv = got[(a, b, wl.ctx[b])]
            assert np.array_equal(gk, staged[(br, a)][1][b]) and np.array_equal(gv, staged[(br, a)][2][b])
    order = np.argsort(wl.ctx)
    sample = sorted({int(order[0]), int(order[-1]), int(order[len(order) // 3]), int(order[2 * len(order) // 3])})
    e = inputs.emb(wl, s).astype(np.float64)
    hp = inputs.h_prev0(wl).astype(np.float64)
    for b in sample:
        t = wl.ctx[b] + 1
        x = e[b].copy()
        for a, layer in enumerate(wl.attn_layers):
            q, k, v = staged[(LOCAL, a)]
            ref = _attend(wl, a, b, t, q[b], k[b], v[b], LOCAL)
            ok, ma, rel = attn_close(o[LOCAL, layer, b], ref.reshape(-1))
            assert ok, ("local", a, b, t, ma, rel)
            x += ref.reshape(-1)
        q_ref = recall_head(head, hp[b], e[b], rmsnorm(x))
        assert score_close(score[b], q_ref), (b, score[b], q_ref)
    flagged = [b for b in order if sched[b]]
    for b in (int(flagged[0]), int(flagged[-1])):
        t = wl.ctx[b] + 1
        a = 2
        q, k, v = staged[(FULL, a)]
        ref = _attend(wl, a, b, t, q[b], k[b], v[b], FULL)
        ok, ma, rel = attn_close(o[FULL, wl.attn_layers[a], b], ref.reshape(-1))
        assert ok, ("full", b, t, ma, rel)


def _gdn_oracle_pass(wl, step, branch, b, S, C, hp, head, o_gpu, e_b, committed):
    """The whole layer stack of one sequence and branch from state (S, C): compares the attention
    and gated-delta outputs with the GPU's, returns (S', C', h)."""
    x = e_b.copy()
    a = j = 0
    taps = None
    for layer in range(wl.n_layers):
        if layer in wl.attn_layers:
            q, k, v = inputs.step_qkv(wl, step, layer, branch)
            ref = _attend(wl, a, b, wl.ctx[b] + 1 + step_index(wl, step), q[b], k[b], v[b], branch,
                          committed)
            ok, ma, rel = attn_close(o_gpu[branch, layer, b], ref.reshape(-1))
            assert ok, ("attention", step, branch, layer, b, ma, rel)
            x += ref.reshape(-1)
            a += 1
        else:
            c, vv, al, be = inputs.gdn_step_inputs(wl, step, layer, branch)
            taps = inputs.gdn_taps(wl, layer).astype(np.float64)
            S[j], C[j], og = gdn_layer(S[j], C[j], c[b].astype(np.float64), vv[b].astype(np.float64),
                                       al[b].astype(np.float64), be[b].astype(np.float64), taps)
            r = np.linalg.norm(o_gpu[branch, layer, b] - og) / np.linalg.norm(og)
            assert r < 1e-4, ("gated delta output", step, branch, layer, b, r)
            x += og
            j += 1
    return S, C, rmsnorm(x)


_STEP0 = {}


def step_index(wl, step):
    return step - _STEP0[wl.name]


def test_hybrid_stack_full_size_two_steps():
    from conditional_sparse_attention_b200.engine import OdaDecoder
    wl = configs.cfg4()
    # two consecutive steps; in the second one sequence flagged and one not
    s1 = next(s for s in range(1, 200) if 0 < inputs.schedule(wl, s).sum() < wl.B)
    steps = [s1 - 1, s1]
    _STEP0[wl.name] = steps[0]
    dec = OdaDecoder(wl, capacity_steps=4)
    dec.capture()
    recs = []
    for s in steps:
        dec.step(dec.make_step_buffer(s))
        dec.synchronize()
        rec_b, conv_b = dec.live_state()
        recs.append(dict(flag=dec.flag.cpu().numpy().copy(), score=dec.score.cpu().numpy().copy(),
                         o=dec.o.cpu().numpy().copy(), rec=rec_b.cpu().numpy().copy(),
                         conv=conv_b.cpu().numpy().copy()))
    assert dec.device_error() == 0
    got = _committed_rows(dec, wl, lambda b: [wl.ctx[b], wl.ctx[b] + 1])
    head = {k: v.cpu().numpy() for k, v in dec.head_params.items()}
    dec.close()
    del dec
    torch.cuda.empty_cache()

    for j, s in enumerate(steps):
        sched = inputs.schedule(wl, s)
        assert recs[j]["flag"].tolist() == sched.tolist()
        for a, layer in enumerate(wl.attn_layers):
            for b in range(wl.B):
                br = FULL if sched[b] else LOCAL
                _, k, v = inputs.step_qkv(wl, s, layer, br)
                gk, gv = got[(a, b, wl.ctx[b] + j)]
                assert np.array_equal(gk, k[b]) and np.array_equal(gv, v[b]), ("committed KV", a, b, j)
    sched1 = inputs.schedule(wl, steps[1])
    picks = [int(np.flatnonzero(sched1)[0]), int(np.flatnonzero(sched1 == 0)[0])]
    S0, C0 = inputs.gdn_state0(wl)
    hp0 = inputs.h_prev0(wl).astype(np.float64)
    for b in picks:
        S = S0[b].astype(np.float64).copy()
        C = C0[b].astype(np.float64).copy()
        hp = hp0[b]
        for j, s in enumerate(steps):
            e_b = inputs.emb(wl, s).astype(np.float64)[b]
            flagged = bool(inputs.schedule(wl, s)[b])
            SL, CL, hL = _gdn_oracle_pass(wl, s, LOCAL, b, S.copy(), C.copy(), hp, head, recs[j]["o"],
                                          e_b, got)
            q_ref = recall_head(head, hp, e_b, hL)
            assert score_close(recs[j]["score"][b], q_ref), (j, b, recs[j]["score"][b], q_ref)
            if flagged:   # the retry starts from the pre-step state (S, C), not from (SL, CL)
                S, C, h = _gdn_oracle_pass(wl, s, FULL, b, S.copy(), C.copy(), hp, head, recs[j]["o"],
                                           e_b, got)
            else:
                S, C, h = SL, CL, hL
            hp = h
            rs = np.linalg.norm(recs[j]["rec"][b] - S) / np.linalg.norm(S)
            rc = np.linalg.norm(recs[j]["conv"][b] - C) / np.linalg.norm(C)
            assert rs < 1e-5 and rc < 1e-6, ("state", j, b, flagged, rs, rc)
