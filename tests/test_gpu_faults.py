"""GPU: bounded waits give up with an error status, and the context keeps working.

Every spin-wait in the kernels (copy-ring mbarriers, the fused head's grid barrier) is bounded
by the global timer and, when the limit passes, sets ODA_DEVERR_WAIT_TIMEOUT in the context's
error word and returns instead of trapping.  oda_probe_wait runs one such wait, through the
same device helpers, on a target nothing will ever reach (an mbarrier with no arrival, a grid
barrier one CTA above the grid) with a short limit.  No fault, trap or endless loop is involved.
After the timeout is reported and cleared, ordinary calls on the same context must give the
oracle's results.
"""
import numpy as np
import pytest
import torch

from helpers import attn_close, build_all
from oracle.attention import attend_bits
from oracle.sets import full_set, local_set
from workload import configs, device as wdev, inputs

pytestmark = pytest.mark.gpu

TIMEOUT_BIT = 0x4


@pytest.fixture(scope="module", autouse=True)
def _build():
    build_all()


def _attention_setup():
    from conditional_sparse_attention_b200 import oda
    wl = configs.cfg0().replace(name="t_faults", seed=31, B=2, ctx=(3000, 40), steps=2)
    mp = wl.max_pages()
    pt = torch.from_numpy(inputs.page_table(wl, mp)).cuda()
    k = torch.empty((wl.B * mp, wl.Hkv, 16, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    wdev.fill_kv(k, pt, wl.ctx, [inputs.cache_key(wl, "k", 0, b) for b in range(wl.B)], wl.Hkv)
    wdev.fill_kv(v, pt, wl.ctx, [inputs.cache_key(wl, "v", 0, b) for b in range(wl.B)], wl.Hkv)
    q, kn, vn = inputs.step_qkv(wl, 0, 0, 0)
    t = lambda a: torch.from_numpy(a.view(np.int16)).cuda()  # noqa: E731
    pos = torch.tensor([c + 1 for c in wl.ctx], dtype=torch.int32, device="cuda")
    ctx = oda.oda_create(oda.make_config(wl.B, wl.Hq, wl.Hkv, mp, 2048))
    return wl, ctx, oda.kv_layer(k, v), pt, pos, (q, kn, vn), (t(q), t(kn), t(vn)), (k, v)


def _oracle(wl, host_qkv, b, mode):
    q, kn, vn = host_qkv
    t = wl.ctx[b] + 1
    kc = inputs.cache_tokens(wl, "k", 0, b, wl.ctx[b])
    vc = inputs.cache_tokens(wl, "v", 0, b, wl.ctx[b])
    S = local_set(t, wl.sinks, wl.window) if mode == 0 else full_set(t)
    return attend_bits(q[b], kc, vc, kn[b], vn[b], S)


@pytest.mark.parametrize("which", [0, 1])
def test_wait_gives_up_and_context_recovers(which):
    from conditional_sparse_attention_b200 import oda
    wl, ctx, layer, pt, pos, host_qkv, (q, kn, vn), _keep = _attention_setup()
    assert oda.oda_get_error(ctx) == 0
    oda.oda_probe_wait(ctx, which, 100_000)          # 100 us limit
    assert oda.oda_get_error(ctx) & TIMEOUT_BIT
    oda.oda_clear_error(ctx)
    assert oda.oda_get_error(ctx) == 0
    # the context still computes correctly: local and full attention against the oracle
    out = torch.zeros((wl.B, wl.Hq, 128), device="cuda")
    flag = torch.ones(wl.B, dtype=torch.int32, device="cuda")
    for mode in (0, 1):
        if mode == 0:
            oda.oda_attend_local(ctx, layer, pt, pos, q, kn, vn, out)
        else:
            oda.oda_attend_full_if(ctx, layer, pt, pos, flag, q, kn, vn, out)
        torch.cuda.synchronize()
        assert oda.oda_get_error(ctx) == 0
        got = out.cpu().numpy()
        for b in range(wl.B):
            ok, ma, rel = attn_close(got[b], _oracle(wl, host_qkv, b, mode))
            assert ok, (mode, b, ma, rel)
    ctx.close()


def test_probe_wait_refuses_bad_arguments():
    from conditional_sparse_attention_b200 import _lib, oda
    _wl, ctx, *_rest = _attention_setup()
    for which, lim in ((2, 100_000), (0, 10), (1, 5_000_000_000)):
        with pytest.raises(_lib.OdaError) as e:
            oda.oda_probe_wait(ctx, which, lim)
        assert e.value.status == 1
    ctx.close()


def test_grid_barrier_counter_back_to_zero_after_probe():
    """After a grid-barrier timeout, the fused recall head (which uses the same counter) still
    scores correctly: back-to-back scores before and after the probe are bitwise equal."""
    from conditional_sparse_attention_b200 import oda
    wl = configs.cfg0().replace(name="t_faults_head", seed=32, B=2, ctx=(10, 20))
    P = inputs.head_weights(wl, perturb=True)
    dev = torch.device("cuda")
    Pd = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in P.items()}
    w = oda.head_weights(Pd)
    ctx = oda.oda_create(oda.make_config(wl.B, wl.Hq, wl.Hkv, 4, wl.D))
    x = [torch.from_numpy(inputs.emb(wl, i)).to(dev) for i in range(3)]
    score = torch.zeros(wl.B, device=dev)
    flag = torch.zeros(wl.B, dtype=torch.int32, device=dev)
    anyf = torch.zeros(1, dtype=torch.int32, device=dev)
    oda.oda_recall_score(ctx, w, x[0], x[1], x[2], None, score, flag, anyf)
    s0 = score.clone()
    oda.oda_probe_wait(ctx, 1, 50_000)
    assert oda.oda_get_error(ctx) & TIMEOUT_BIT
    oda.oda_clear_error(ctx)
    oda.oda_recall_score(ctx, w, x[0], x[1], x[2], None, score, flag, anyf)
    torch.cuda.synchronize()
    assert oda.oda_get_error(ctx) == 0
    assert torch.equal(score, s0)
    ctx.close()
