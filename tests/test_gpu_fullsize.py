"""GPU parity at full size: the 128K-context, 36-layer, batch-4 workload in the launch
configuration bench.py times (one CUDA graph per step, retry under a conditional node, layer
overlap on).  Two routed steps are run; the oracle then checks, from slices it regenerates
with the seeded generator:

  * routing equals the schedule, positions advance by one per step;
  * every committed K/V (36 layers x 4 sequences x 2 steps) is bit-exact;
  * sampled local-branch outputs (several layers and sequences), all 36 local outputs and
    the recall score of one sequence, and a sampled full-branch output of a flagged sequence,
    within the attention / score tolerances.
"""
import numpy as np
import pytest
import torch

from helpers import attn_close, build_all, score_close
from oracle.attention import attend_bits
from oracle.head import recall_head, rmsnorm
from oracle.sets import full_set, local_set
from workload import configs, inputs

pytestmark = pytest.mark.gpu

LOCAL, FULL = 0, 1


@pytest.fixture(scope="module", autouse=True)
def _build():
    build_all()


def _set_rows(wl, a, b, t, committed):
    """The cached rows of (layer a, sequence b) that S^L_t reads, in position order, as compact
    [n, Hkv, 128] arrays: prefilled rows regenerated, committed rows from the oracle's staging.
    (Attention over the set only needs those rows; the current token is appended by the caller.)"""
    rows = sorted(p - 1 for p in local_set(t) if p < t)
    ctx = wl.ctx[b]
    ks, vs = [], []
    pre = [r for r in rows if r < ctx]
    for lo, hi in _runs(pre) if pre else []:
        ks.append(inputs.cache_tokens(wl, "k", a, b, hi - lo, start=lo))
        vs.append(inputs.cache_tokens(wl, "v", a, b, hi - lo, start=lo))
    for r in rows:
        if r >= ctx:
            ks.append(committed[(a, b, r)][0][None])
            vs.append(committed[(a, b, r)][1][None])
    return np.concatenate(ks), np.concatenate(vs)


def _local_out(wl, a, b, t, q, k, v, committed):
    kc, vc = _set_rows(wl, a, b, t, committed)
    return attend_bits(q, kc, vc, k, v, full_set(kc.shape[0] + 1))


def _runs(sorted_rows):
    out = []
    start = prev = sorted_rows[0]
    for r in sorted_rows[1:]:
        if r != prev + 1:
            out.append((start, prev + 1))
            start = r
        prev = r
    out.append((start, prev + 1))
    return out


def test_full_size_two_steps():
    from conditional_sparse_attention_b200.engine import OdaDecoder
    wl = configs.cfg2()
    # two consecutive step indices whose schedule flags at least one sequence in the second
    s1 = next(s for s in range(1, 200) if inputs.schedule(wl, s).any())
    steps = [s1 - 1, s1]
    dec = OdaDecoder(wl, capacity_steps=4)
    dec.capture()
    pos0 = dec.pos.cpu().numpy().copy()
    recs = []
    for s in steps:
        dec.step(dec.make_step_buffer(s))
        dec.synchronize()
        recs.append(dict(flag=dec.flag.cpu().numpy().copy(), score=dec.score.cpu().numpy().copy(),
                         o=dec.o.cpu().numpy().copy()))
    assert dec.device_error() == 0
    assert dec.pos.cpu().numpy().tolist() == (pos0 + 2).tolist()
    pt = dec.page_table.cpu().numpy()
    # committed positions (cache rows ctx and ctx+1) of every layer and sequence
    got_kv = {}
    for a in range(wl.L):
        for b in range(wl.B):
            for j in range(2):
                row = wl.ctx[b] + j
                page, slot = pt[b, row // 16], row % 16
                got_kv[(a, b, row)] = (
                    dec.k_pool[a][page, :, slot].cpu().view(torch.int16).numpy().view(np.uint16),
                    dec.v_pool[a][page, :, slot].cpu().view(torch.int16).numpy().view(np.uint16))
    head = {k: v.cpu().numpy() for k, v in dec.head_params.items()}
    dec.close()
    del dec
    torch.cuda.empty_cache()

    committed = {}
    for j, s in enumerate(steps):
        sched = inputs.schedule(wl, s)
        assert recs[j]["flag"].tolist() == sched.tolist()
        for a, layer in enumerate(wl.attn_layers):
            staged = {br: inputs.step_qkv(wl, s, layer, br) for br in (LOCAL, FULL)}
            for b in range(wl.B):
                br = FULL if sched[b] else LOCAL
                row = wl.ctx[b] + j
                ek, ev = staged[br][1][b], staged[br][2][b]
                gk, gv = got_kv[(a, b, row)]
                assert np.array_equal(gk, ek) and np.array_equal(gv, ev), ("committed KV", a, b, j)
                committed[(a, b, row)] = (ek, ev)

    # one sequence unflagged in the first step: the oracle's own h_{t-1} for the second step is
    # its local hidden of the first step
    b_all = int(np.flatnonzero(inputs.schedule(wl, steps[0]) == 0)[0])
    e0 = inputs.emb(wl, steps[0]).astype(np.float64)[b_all].copy()
    for a, layer in enumerate(wl.attn_layers):
        q, k, v = inputs.step_qkv(wl, steps[0], layer, LOCAL)
        ref = _local_out(wl, a, b_all, wl.ctx[b_all] + 1, q[b_all], k[b_all], v[b_all], committed)
        ok, ma, rel = attn_close(recs[0]["o"][LOCAL, layer, b_all], ref.reshape(-1))
        assert ok, ("local step 1", a, b_all, ma, rel)
        e0 += ref.reshape(-1)
    h_prev_oracle = rmsnorm(e0)

    # second step: sampled local outputs, one sequence's whole local pass and score
    s = steps[1]
    rec = recs[1]
    t = {b: wl.ctx[b] + 2 for b in range(wl.B)}
    h_acc = inputs.emb(wl, s).astype(np.float64)[b_all].copy()
    for a, layer in enumerate(wl.attn_layers):
        q, k, v = inputs.step_qkv(wl, s, layer, LOCAL)
        for b in range(wl.B):
            if b != b_all and a not in (0, 17, 35):
                continue
            ref = _local_out(wl, a, b, t[b], q[b], k[b], v[b], committed)
            ok, ma, rel = attn_close(rec["o"][LOCAL, layer, b], ref.reshape(-1))
            assert ok, ("local", a, b, ma, rel)
            if b == b_all:
                h_acc += ref.reshape(-1)
    h_loc = rmsnorm(h_acc)
    q_ref = recall_head(head, h_prev_oracle, inputs.emb(wl, s).astype(np.float64)[b_all], h_loc)
    assert score_close(rec["score"][b_all], q_ref), (rec["score"][b_all], q_ref)

    # one flagged sequence: full-branch output of a sampled layer over the whole history
    fb = int(np.flatnonzero(rec["flag"])[0])
    a = 7
    layer = wl.attn_layers[a]
    q, k, v = inputs.step_qkv(wl, s, layer, FULL)
    n = t[fb] - 1
    kc = np.empty((n, wl.Hkv, 128), np.uint16)
    vc = np.empty_like(kc)
    kc[:wl.ctx[fb]] = inputs.cache_tokens(wl, "k", a, fb, wl.ctx[fb])
    vc[:wl.ctx[fb]] = inputs.cache_tokens(wl, "v", a, fb, wl.ctx[fb])
    kc[wl.ctx[fb]], vc[wl.ctx[fb]] = committed[(a, fb, wl.ctx[fb])]
    ref = attend_bits(q[fb], kc, vc, k[fb], v[fb], full_set(t[fb]))
    ok, ma, rel = attn_close(rec["o"][FULL, layer, fb], ref.reshape(-1))
    assert ok, ("full", a, fb, ma, rel)
