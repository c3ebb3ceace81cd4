"""GPU: commit and snapshot/restore are bit-exact data movement; generator twin is bit-exact."""
import numpy as np
import pytest
import torch

from helpers import build_all, logical_cache
from workload import configs, device as wdev, gen, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    build_all()


def test_device_generator_is_bit_identical():
    k = gen.key(123, 4, 5)
    x = torch.zeros(100003, dtype=torch.int16, device="cuda")
    wdev.fill_normal_bf16(x, k, start=777)
    assert np.array_equal(x.cpu().numpy().view(np.uint16), gen.normal_bf16(k, 100003, start=777))
    wl = configs.cfg3().replace(B=3, ctx=(33, 1000, 16))
    mp = wl.max_pages()
    pt = torch.from_numpy(inputs.page_table(wl, mp)).cuda()
    pool = torch.zeros((3 * mp, wl.Hkv, 16, 128), dtype=torch.int16, device="cuda")
    wdev.fill_kv(pool, pt, wl.ctx, [inputs.cache_key(wl, "k", 2, b) for b in range(3)], wl.Hkv)
    host = pool.cpu().numpy().view(np.uint16)
    for b in range(3):
        assert np.array_equal(logical_cache(host, pt.cpu().numpy(), b, wl.ctx[b]),
                              inputs.cache_tokens(wl, "k", 2, b, wl.ctx[b]))


def test_commit_writes_exactly_the_chosen_branch():
    from conditional_sparse_attention_b200 import oda
    wl = configs.cfg3().replace(B=5, n_layers=3, attn_layers=(0, 1, 2), ctx=(0, 15, 16, 2100, 77))
    B, L, Hkv, D = wl.B, wl.L, wl.Hkv, wl.D
    mp = wl.max_pages()
    pt_np = inputs.page_table(wl, mp)
    pt = torch.from_numpy(pt_np).cuda()
    pools_k = [torch.zeros((B * mp, Hkv, 16, 128), dtype=torch.int16, device="cuda") for _ in range(L)]
    pools_v = [torch.zeros_like(p) for p in pools_k]
    for a in range(L):
        wdev.fill_kv(pools_k[a], pt, wl.ctx, [inputs.cache_key(wl, "k", a, b) for b in range(B)], Hkv)
        wdev.fill_kv(pools_v[a], pt, wl.ctx, [inputs.cache_key(wl, "v", a, b) for b in range(B)], Hkv)
    before_k = [p.cpu().numpy().copy() for p in pools_k]
    stage = {}
    for br in (0, 1):
        for which in ("k", "v"):
            arr = gen.normal_bf16(gen.key(9, br, ord(which)), L * B * Hkv * 128).reshape(L, B, Hkv, 128)
            stage[(br, which)] = arr
    st = {k: torch.from_numpy(v.view(np.int16)).cuda() for k, v in stage.items()}
    hL = torch.randn(B, D, device="cuda")
    hF = torch.randn(B, D, device="cuda")
    h_prev = torch.zeros(B, D, device="cuda")
    pos = torch.tensor([c + 1 for c in wl.ctx], dtype=torch.int32, device="cuda")
    flags = np.array([1, 0, 1, 0, 1], np.int32)
    c = oda.oda_create(oda.make_config(B, wl.Hq, Hkv, mp, D))
    layers = [oda.kv_layer(pools_k[a], pools_v[a]) for a in range(L)]
    oda.oda_commit(c, layers, pt, pos, torch.from_numpy(flags).cuda(), st[(0, "k")], st[(0, "v")],
                   st[(1, "k")], st[(1, "v")], hL, hF, h_prev)
    torch.cuda.synchronize()
    assert oda.oda_get_error(c) == 0
    assert pos.cpu().tolist() == [x + 2 for x in wl.ctx]
    hp = h_prev.cpu().numpy()
    for b in range(B):
        ref = (hF if flags[b] else hL)[b].cpu().numpy()
        assert np.array_equal(hp[b], ref)
    for a in range(L):
        after = pools_k[a].cpu().numpy().view(np.uint16)
        afterv = pools_v[a].cpu().numpy().view(np.uint16)
        changed = np.argwhere(np.any(after != before_k[a].view(np.uint16), axis=(2, 3)))
        for b in range(B):
            t = wl.ctx[b] + 1
            br = 1 if flags[b] else 0
            lk = logical_cache(after, pt_np, b, t)
            lv = logical_cache(afterv, pt_np, b, t)
            assert np.array_equal(lk[t - 1], stage[(br, "k")][a, b])
            assert np.array_equal(lv[t - 1], stage[(br, "v")][a, b])
            assert np.array_equal(lk[:t - 1], inputs.cache_tokens(wl, "k", a, b, t - 1))
        # exactly one (page, head-block) slot per sequence changed per head
        assert len({tuple(x) for x in changed}) <= B * Hkv


def test_snapshot_restore_bit_exact():
    from conditional_sparse_attention_b200 import oda
    B, n = 4, 3
    rec = torch.randn(B, n, 16, 128, 128, device="cuda")
    conv = torch.randn(B, n, 4, 2048, device="cuda")
    rec0, conv0 = rec.clone(), conv.clone()
    rs, cs = torch.zeros_like(rec), torch.zeros_like(conv)
    c = oda.oda_create(oda.make_config(B, 16, 8, 4, 2048))
    live, snap = oda.state(rec, conv), oda.state(rs, cs)
    oda.oda_snapshot(c, live, snap)
    torch.cuda.synchronize()
    assert torch.equal(rs, rec0) and torch.equal(cs, conv0)
    rec.add_(1.0)
    conv.mul_(-2.0)
    flags = torch.tensor([1, 0, 0, 1], dtype=torch.int32, device="cuda")
    oda.oda_restore(c, flags, snap, live)
    torch.cuda.synchronize()
    for b in range(B):
        if flags[b]:
            assert torch.equal(rec[b], rec0[b]) and torch.equal(conv[b], conv0[b])
        else:
            assert torch.equal(rec[b], rec0[b] + 1.0) and torch.equal(conv[b], conv0[b] * -2.0)
