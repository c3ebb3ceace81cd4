"""Pins of the synthetic-backbone oracle (oracle.backbone) against torch's own modules, the bf16
rounding against torch's conversion, and closed-form special cases."""
import numpy as np
import pytest
import torch

from oracle import backbone as BB
from oracle.attention import bf16_to_f64
from workload import gen


def _bits(seed, shape, scale=0):
    return gen.normal_bf16(gen.key(seed, 1), int(np.prod(shape)), 0, scale).reshape(shape)


def test_bf16_rounding_matches_torch():
    """torch rounds fp64 to bf16 through fp32, so the comparison uses fp32-representable values
    (one rounding on both sides); one value above a midpoint by less than fp32 resolves is
    checked by hand."""
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-3, 2000),
                        rng.normal(0, 1e3, 2000)]).astype(np.float32).astype(np.float64)
    # exact ties: values halfway between neighbouring bf16 numbers
    base = bf16_to_f64(gen.normal_bf16(gen.key(3, 1), 2000))
    ties = base + np.ldexp(1.0, np.frexp(base)[1] - 9)
    x = np.concatenate([x, ties, -ties])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(BB.bf16(x), want)
    assert np.array_equal(BB.bf16_bits(BB.bf16(x)),
                          torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    # the midpoint 1.56640625 of the bf16 neighbours 1.5625 and 1.5703125 goes to the even one
    # (1.5625); 2^-40 above it the nearest is the upper neighbour
    mid = 1.56640625
    assert BB.bf16(np.array(mid)) == 1.5625 and BB.bf16(np.array(-mid)) == -1.5625
    assert BB.bf16(np.array(mid + 2.0 ** -40)) == 1.5703125


class TorchLayer(torch.nn.Module):
    """The same stand-in layer built from torch.nn modules in fp64 (independent composition)."""

    def __init__(self, D, F, Hq, Hkv, ga, gm, Wqkv, Wo, Wg, Wu, Wd):
        super().__init__()
        f = lambda b: torch.from_numpy(bf16_to_f64(b))  # noqa: E731
        self.na = torch.nn.RMSNorm(D, eps=1e-6, dtype=torch.float64)
        self.nm = torch.nn.RMSNorm(D, eps=1e-6, dtype=torch.float64)
        self.na.weight.data = torch.from_numpy(ga.astype(np.float64))
        self.nm.weight.data = torch.from_numpy(gm.astype(np.float64))
        self.qkv = torch.nn.Linear(D, Wqkv.shape[0], bias=False, dtype=torch.float64)
        self.o = torch.nn.Linear(Hq * 128, D, bias=False, dtype=torch.float64)
        self.g = torch.nn.Linear(D, F, bias=False, dtype=torch.float64)
        self.u = torch.nn.Linear(D, F, bias=False, dtype=torch.float64)
        self.d = torch.nn.Linear(F, D, bias=False, dtype=torch.float64)
        for mod, w in ((self.qkv, Wqkv), (self.o, Wo), (self.g, Wg), (self.u, Wu), (self.d, Wd)):
            mod.weight.data = f(w)
        self.Hq, self.Hkv = Hq, Hkv

    @staticmethod
    def r(t):
        return t.to(torch.bfloat16).to(torch.float64)

    def forward(self, x, o):
        y = self.r(self.qkv(self.r(self.na(x))))
        x = x + self.o(self.r(o))
        m = self.r(self.nm(x))
        x = x + self.d(self.r(torch.nn.functional.silu(self.g(m)) * self.u(m)))
        return y, x


@pytest.mark.parametrize("B,Hq,Hkv,F", [(1, 4, 2, 1024), (3, 2, 1, 512)])
def test_layer_matches_a_composition_of_torch_modules(B, Hq, Hkv, F):
    D = Hq * 128
    rng = np.random.default_rng(B)
    Wqkv = _bits(11, ((Hq + 2 * Hkv) * 128, D), -5)
    Wo, Wg, Wu = _bits(12, (D, Hq * 128), -5), _bits(13, (F, D), -5), _bits(14, (F, D), -5)
    Wd = _bits(15, (D, F), -5)
    ga, gm = rng.uniform(0.5, 1.5, D), rng.uniform(0.5, 1.5, D)
    x = rng.normal(0, 3, (B, D))
    o = rng.normal(0, 1, (B, Hq * 128))
    q, k, v = BB.attn_in(x, ga, Wqkv, Hq, Hkv)
    x2 = BB.mlp(BB.attn_out(x, o, Wo), gm, Wg, Wu, Wd)
    t = TorchLayer(D, F, Hq, Hkv, ga, gm, Wqkv, Wo, Wg, Wu, Wd)
    with torch.no_grad():
        y_t, x_t = t(torch.from_numpy(x), torch.from_numpy(o))
    got = np.concatenate([bf16_to_f64(q).reshape(B, -1), bf16_to_f64(k).reshape(B, -1),
                          bf16_to_f64(v).reshape(B, -1)], axis=1)
    # the same bf16 values except where summation order moves a value across a rounding edge
    diff = got != y_t.numpy()
    assert diff.mean() < 1e-3
    assert np.allclose(got, y_t.numpy(), rtol=2 ** -7, atol=0)
    assert np.allclose(x2, x_t.numpy(), rtol=1e-6, atol=1e-9)


def test_zero_weights_leave_the_residual_and_zero_qkv():
    B, Hq, Hkv, F = 2, 2, 1, 512
    D = Hq * 128
    z = lambda s: np.zeros(s, np.uint16)  # noqa: E731  (bf16 +0.0)
    x = np.random.default_rng(4).normal(0, 1, (B, D))
    q, k, v = BB.attn_in(x, np.ones(D), z(((Hq + 2 * Hkv) * 128, D)), Hq, Hkv)
    assert not q.any() and not k.any() and not v.any()
    o = np.ones((B, Hq * 128))
    assert np.array_equal(BB.attn_out(x, o, z((D, Hq * 128))), x)
    assert np.array_equal(BB.mlp(x, np.ones(D), z((F, D)), z((F, D)), z((D, F))), x)


def test_rmsnorm_and_silu_closed_forms():
    x = np.array([[3.0, -4.0]])
    assert np.allclose(BB.rmsnorm(x, [1.0, 2.0]), [[3 / np.sqrt(12.5 + 1e-6), -8 / np.sqrt(12.5 + 1e-6)]])
    assert BB.silu(np.array(0.0)) == 0.0
    assert np.isclose(BB.silu(np.array(2.0)), 2.0 / (1.0 + np.exp(-2.0)))


def test_identity_projection_passes_the_normalised_input_through():
    """W_qkv = [I; I; 0] with unit norm weights: q = k-heads = bf16(RMSNorm(x))."""
    Hq = Hkv = 1
    D = 128
    I = np.eye(D)
    W = np.concatenate([I, I, np.zeros((D, D))])
    Wb = BB.bf16_bits(W)
    x = np.random.default_rng(5).normal(0, 2, (2, D))
    q, k, v = BB.attn_in(x, np.ones(D), Wb, Hq, Hkv)
    n = BB.bf16(BB.rmsnorm(x, np.ones(D)))
    assert np.array_equal(bf16_to_f64(q)[:, 0], n) and np.array_equal(bf16_to_f64(k)[:, 0], n)
    assert not v.any()


def test_lm_head_argmax_takes_the_smallest_index_on_ties():
    E = BB.bf16_bits(np.array([[1.0, 0.0], [2.0, 0.0], [2.0, 0.0], [-5.0, 0.0]]))
    logits, tok = BB.lm_head(np.array([[1.0, 7.0], [-1.0, 0.0]]), E)
    assert np.array_equal(logits, [[1.0, 2.0, 2.0, -5.0], [-1.0, -2.0, -2.0, 5.0]])
    assert tok.tolist() == [1, 3]
