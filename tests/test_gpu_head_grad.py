"""GPU parity: oda_recall_grad (labels, Huber loss, recall-head gradient) vs the fp64 oracle.

Tolerances (fp32 arithmetic with dot products of up to 9216 terms, several layers deep):
loss relative 1e-5, labels relative 1e-6, scores as the recall-score tolerance, every gradient
tensor relative L2 2e-4 against the oracle's.
"""
import numpy as np
import pytest
import torch

from helpers import build_all, score_close
from oracle import head_grad
from workload import configs, gen, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    build_all()


def _case(B, D, seed, valid=None, lam=0.01):
    Hq = D // 128
    wl = configs.cfg0().replace(name="t_grad", seed=seed, B=B, Hq=Hq, Hkv=Hq // 2, ctx=(10,) * B)
    P = inputs.head_weights(wl, perturb=True)
    xs = [gen.normal_f32(gen.key(seed, 91, i), B * D).reshape(B, D) for i in range(3)]
    rng = np.random.default_rng(seed)
    p_full = rng.uniform(0.02, 0.98, B).astype(np.float32)
    p_local = rng.uniform(0.02, 0.98, B).astype(np.float32)
    if valid is None:
        valid = (rng.uniform(0, 1, B) < 0.75).astype(np.int32)
        valid[0] = 1
    return P, xs, p_full, p_local, np.asarray(valid, np.int32), lam


def _run_gpu(P, xs, p_full, p_local, valid, lam):
    from conditional_sparse_attention_b200 import oda
    B, D = xs[0].shape
    dev = "cuda"
    Pd = {k: torch.from_numpy(v).to(dev) for k, v in P.items()}
    Gd = {k: torch.full_like(v, float("nan")) for k, v in Pd.items()}   # every entry must be written
    hx = [torch.from_numpy(np.ascontiguousarray(x)).to(dev) for x in xs]
    pf, pl = torch.from_numpy(p_full).to(dev), torch.from_numpy(p_local).to(dev)
    vd = torch.from_numpy(valid).to(dev)
    loss = torch.zeros(1, device=dev)
    q = torch.zeros(B, device=dev)
    y = torch.zeros(B, device=dev)
    ws = torch.empty(oda.oda_recall_grad_workspace_bytes(B, D), dtype=torch.uint8, device=dev)
    oda.oda_recall_grad(oda.head_weights(Pd), oda.head_grads(Gd), B, D, hx[0], hx[1], hx[2], pf, pl,
                        vd, lam, loss, q, y, ws)
    torch.cuda.synchronize()
    return (float(loss.item()), q.cpu().numpy(), y.cpu().numpy(),
            {k: v.cpu().numpy() for k, v in Gd.items()})


def _check(case):
    P, xs, p_full, p_local, valid, lam = case
    loss, q, y, G = _run_gpu(*case)
    # the oracle on the same fp32 probabilities (upcast)
    rl, rq, ry, RG = head_grad.loss_and_grad(P, xs[0], xs[1], xs[2], p_full.astype(np.float64),
                                             p_local.astype(np.float64), valid, lam)
    for b in range(len(q)):
        assert score_close(q[b], rq[b]), (b, q[b], rq[b])
    assert np.allclose(y, ry, rtol=1e-6, atol=1e-7), (y, ry)
    assert loss == pytest.approx(rl, rel=1e-5, abs=1e-7)
    for k, ref in RG.items():
        got = G[k].astype(np.float64)
        assert np.all(np.isfinite(got)), k
        nrm = np.linalg.norm(ref)
        err = np.linalg.norm(got - ref)
        assert err <= 2e-4 * max(nrm, 1e-12), (k, err, nrm)


@pytest.mark.parametrize("B,D,seed", [(3, 2048, 801), (12, 1024, 802), (2, 4096, 803)])
def test_loss_and_gradient_match_oracle(B, D, seed):
    _check(_case(B, D, seed))


def test_gradient_is_bitwise_repeatable():
    case = _case(4, 2048, 804)
    a = _run_gpu(*case)
    b = _run_gpu(*case)
    assert a[0] == b[0] and np.array_equal(a[1], b[1])
    for k in a[3]:
        assert np.array_equal(a[3][k], b[3][k]), k


def test_no_valid_position_gives_zero_loss_and_gradient():
    loss, q, y, G = _run_gpu(*_case(3, 1024, 805, valid=[0, 0, 0]))
    assert loss == 0.0 and not np.any(y)
    for k, g in G.items():
        assert np.all(g == 0.0), k


def test_rejects_unsupported_shapes():
    from conditional_sparse_attention_b200 import oda
    P, xs, pf, pl, valid, lam = _case(2, 1024, 806)
    Pd = {k: torch.from_numpy(v).to("cuda") for k, v in P.items()}
    Gd = {k: torch.empty_like(v) for k, v in Pd.items()}
    t = torch.zeros(64, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")   # too small
    with pytest.raises(oda.OdaError):
        oda.oda_recall_grad(oda.head_weights(Pd), oda.head_grads(Gd), 2, 1024, t, t, t, t, t,
                            t, lam, t, t, t, ws)
    ws = torch.empty(oda.oda_recall_grad_workspace_bytes(17, 1024), dtype=torch.uint8, device="cuda")
    with pytest.raises(oda.OdaError):
        oda.oda_recall_grad(oda.head_weights(Pd), oda.head_grads(Gd), 17, 1024, t, t, t, t, t,
                            t, lam, t, t, t, ws)
