"""GPU: the allocation-free full-set attention (oda_attend_full_if_noalloc) against the
context-based entry point.

Some callers cannot allocate device memory: a plugin inside a host framework that only lends
it buffers, or a latency-critical loop where cudaMalloc's implicit synchronisation is not
acceptable.  For them the library keeps the split-KV scratch in a static device array; this
checks that two calls in a row through that array give the same outputs as the ordinary
entry point (within the attention tolerance), leave unflagged rows alone, and that a shape too
large for the array is refused before anything is launched.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import attn_close, build_all
from workload import configs, device as wdev, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    build_all()


def _setup(ctx_lens, Hq=32, Hkv=8, seed=99):
    from conditional_sparse_attention_b200 import oda
    wl = configs.cfg0().replace(name="t_noalloc", seed=seed, B=len(ctx_lens), n_layers=1,
                                attn_layers=(0,), Hq=Hq, Hkv=Hkv, ctx=tuple(ctx_lens), steps=2,
                                shuffle_pages=True)
    mp = wl.max_pages()
    pt = torch.from_numpy(inputs.page_table(wl, mp)).cuda()
    k = torch.full((wl.B * mp, Hkv, 16, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    v = torch.full_like(k, float("nan"))
    wdev.fill_kv(k, pt, wl.ctx, [inputs.cache_key(wl, "k", 0, b) for b in range(wl.B)], Hkv)
    wdev.fill_kv(v, pt, wl.ctx, [inputs.cache_key(wl, "v", 0, b) for b in range(wl.B)], Hkv)
    q, kn, vn = inputs.step_qkv(wl, 0, 0, 0)
    t = lambda a: torch.from_numpy(a.view(np.int16)).cuda()  # noqa: E731
    pos = torch.tensor([c + 1 for c in wl.ctx], dtype=torch.int32, device="cuda")
    cfg = oda.make_config(wl.B, Hq, Hkv, mp, max(512, wl.D))
    return wl, cfg, oda.kv_layer(k, v), pt, pos, t(q), t(kn), t(vn), (k, v)


def test_noalloc_matches_context_entry_point_twice():
    from conditional_sparse_attention_b200 import oda
    ctx_lens = [0, 17, 2052, 2053, 4096, 9000, 30000, 700]
    wl, cfg, layer, pt, pos, q, kn, vn, _keep = _setup(ctx_lens)
    flag = torch.tensor([1, 0, 1, 1, 0, 1, 1, 1], dtype=torch.int32, device="cuda")
    ref = torch.full((wl.B, wl.Hq, 128), 5.0, device="cuda")
    c = oda.oda_create(cfg)
    oda.oda_attend_full_if(c, layer, pt, pos, flag, q, kn, vn, ref)
    torch.cuda.synchronize()
    assert oda.oda_get_error(c) == 0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(2):
        out = torch.full((wl.B, wl.Hq, 128), 5.0, device="cuda")
        oda.oda_attend_full_if_noalloc(cfg, layer, pt, pos, flag, q, kn, vn, out, err)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
    assert int(err.item()) == 0
    r = ref.cpu().numpy()
    for out in outs:
        for b in range(wl.B):
            if flag[b]:
                ok, ma, rel = attn_close(out[b], r[b])
                assert ok, (b, ma, rel)
            else:
                assert np.all(out[b] == 5.0), f"unflagged row {b} was written"


def test_noalloc_bit_identical_in_deterministic_mode():
    """With deterministic = 1 both entry points launch the same grid with the same page
    pattern, so their outputs agree bit for bit (on two calls in a row)."""
    from conditional_sparse_attention_b200 import oda
    ctx_lens = [60000, 900, 2053, 4097, 33]
    wl, cfg, layer, pt, pos, q, kn, vn, _keep = _setup(ctx_lens, seed=101)
    cfg.deterministic = 1
    flag = torch.ones(wl.B, dtype=torch.int32, device="cuda")
    ref = torch.zeros((wl.B, wl.Hq, 128), device="cuda")
    c = oda.oda_create(cfg)
    oda.oda_attend_full_if(c, layer, pt, pos, flag, q, kn, vn, ref)
    torch.cuda.synchronize()
    assert oda.oda_get_error(c) == 0
    for _ in range(2):
        out = torch.zeros_like(ref)
        oda.oda_attend_full_if_noalloc(cfg, layer, pt, pos, flag, q, kn, vn, out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    c.close()


def test_noalloc_refuses_invalid_config_fields():
    from conditional_sparse_attention_b200 import _lib, oda
    wl, cfg, layer, pt, pos, q, kn, vn, _keep = _setup([100, 200])
    out = torch.zeros((2, 32, 128), device="cuda")
    flag = torch.ones(2, dtype=torch.int32, device="cuda")
    for field, val in (("deterministic", 2), ("sinks", -1), ("window", 0)):
        bad = oda.make_config(2, 32, 8, cfg.max_pages, 4096)
        setattr(bad, field, val)
        with pytest.raises(_lib.OdaError):
            oda.oda_attend_full_if_noalloc(bad, layer, pt, pos, flag, q, kn, vn, out)


def test_noalloc_refuses_shapes_beyond_its_scratch():
    from conditional_sparse_attention_b200 import _lib, oda
    wl, cfg, layer, pt, pos, q, kn, vn, _keep = _setup([100, 200])
    big = oda.make_config(256, 64, 8, 4, 8192)   # (SMs + 256*8) * 8 * 520 bytes > 4 MiB
    out = torch.zeros((2, 32, 128), device="cuda")
    flag = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(_lib.OdaError) as e:
        oda.oda_attend_full_if_noalloc(big, layer, pt, pos, flag, q, kn, vn, out)
    assert e.value.status == 2 and b"scratch" in _lib.load().oda_last_error()
