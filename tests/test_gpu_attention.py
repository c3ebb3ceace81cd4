"""GPU parity: oda_attend_local / oda_attend_full_if / oda_index_positions vs the oracle.

Same seeded inputs on both sides (workload generators); the oracle computes each output
directly from the set definition in fp64.  Context lengths cover empty caches, page edges,
the sink/window overlap around t = 2052..2064, and ragged tails; page tables are shuffled.
"""
import numpy as np
import pytest
import torch

from helpers import ATTN_MAX_ABS, ATTN_REL_L2, attn_close, build_all
from oracle.attention import attend_bits
from oracle.sets import full_set, local_set
from workload import configs, device as wdev, gen, inputs

pytestmark = pytest.mark.gpu

EDGE_CTX = [0, 1, 3, 4, 5, 15, 16, 17, 100, 2047, 2048, 2050, 2051, 2052, 2053, 2058, 2062,
            2063, 2064, 2065, 2100, 4095, 4096, 5000]


@pytest.fixture(scope="module", autouse=True)
def _build():
    build_all()


def _wl(ctx, Hq=16, Hkv=8, seed=77, shuffle=True, steps=2):
    return configs.cfg0().replace(name="t_attn", seed=seed, B=len(ctx), n_layers=1,
                                  attn_layers=(0,), Hq=Hq, Hkv=Hkv, ctx=tuple(ctx), steps=steps,
                                  shuffle_pages=shuffle)


class Setup:
    def __init__(self, wl, extra_pool_pages=0, deterministic=False):
        from conditional_sparse_attention_b200 import oda
        self.oda = oda
        self.wl = wl
        dev = torch.device("cuda")
        self.max_pages = wl.max_pages()
        self.pt_np = inputs.page_table(wl, self.max_pages)
        self.pt = torch.from_numpy(self.pt_np).to(dev)
        n_pool = wl.B * self.max_pages + extra_pool_pages
        # slots outside every sequence's cache hold NaN: they must never reach an output
        self.k = torch.full((n_pool, wl.Hkv, 16, 128), float("nan"), dtype=torch.bfloat16, device=dev)
        self.v = torch.full_like(self.k, float("inf"))
        wdev.fill_kv(self.k, self.pt, wl.ctx, [inputs.cache_key(wl, "k", 0, b) for b in range(wl.B)], wl.Hkv)
        wdev.fill_kv(self.v, self.pt, wl.ctx, [inputs.cache_key(wl, "v", 0, b) for b in range(wl.B)], wl.Hkv)
        self.layer = oda.kv_layer(self.k, self.v)
        q, kn, vn = inputs.step_qkv(wl, 0, 0, 0)
        self.q_np, self.kn_np, self.vn_np = q, kn, vn
        self.q = torch.from_numpy(q.view(np.int16)).to(dev)
        self.kn = torch.from_numpy(kn.view(np.int16)).to(dev)
        self.vn = torch.from_numpy(vn.view(np.int16)).to(dev)
        self.pos = torch.tensor([c + 1 for c in wl.ctx], dtype=torch.int32, device=dev)
        cfg = oda.make_config(wl.B, wl.Hq, wl.Hkv, self.max_pages, max(512, wl.D), wl.sinks, wl.window,
                              deterministic=deterministic)
        self.ctx = oda.oda_create(cfg)

    def oracle(self, b, mode):
        wl = self.wl
        t = wl.ctx[b] + 1
        kc = inputs.cache_tokens(wl, "k", 0, b, wl.ctx[b])
        vc = inputs.cache_tokens(wl, "v", 0, b, wl.ctx[b])
        S = local_set(t, wl.sinks, wl.window) if mode == 0 else full_set(t)
        return attend_bits(self.q_np[b], kc, vc, self.kn_np[b], self.vn_np[b], S)


@pytest.mark.parametrize("Hq,Hkv", [(16, 8), (32, 8), (8, 1), (4, 4), (24, 8)])
def test_local_matches_oracle(Hq, Hkv):
    s = Setup(_wl(EDGE_CTX, Hq, Hkv))
    out = torch.full((s.wl.B, Hq, 128), 7.0, device="cuda")
    s.oda.oda_attend_local(s.ctx, s.layer, s.pt, s.pos, s.q, s.kn, s.vn, out)
    torch.cuda.synchronize()
    assert s.oda.oda_get_error(s.ctx) == 0
    got = out.cpu().numpy()
    for b in range(s.wl.B):
        ok, ma, rel = attn_close(got[b], s.oracle(b, 0))
        assert ok, f"b={b} ctx={s.wl.ctx[b]} max_abs={ma:.3g} rel_l2={rel:.3g}"


@pytest.mark.parametrize("ctx,Hq,Hkv", [([40000], 16, 8), ([65536], 32, 8), ([5000, 70000], 8, 4),
                                        ([3000], 8, 1), ([2052, 17], 16, 4)])
def test_local_small_batches_large_clusters(ctx, Hq, Hkv):
    """Few (sequence, KV head) pairs give the largest clusters (8 CTAs, each rank's partial pushed
    into rank 0's inbox); the cluster size is cut where the inbox would not fit (g = 8)."""
    s = Setup(_wl(ctx, Hq, Hkv, seed=80))
    out = torch.full((s.wl.B, Hq, 128), 7.0, device="cuda")
    s.oda.oda_attend_local(s.ctx, s.layer, s.pt, s.pos, s.q, s.kn, s.vn, out)
    torch.cuda.synchronize()
    assert s.oda.oda_get_error(s.ctx) == 0
    got = out.cpu().numpy()
    for b in range(s.wl.B):
        ok, ma, rel = attn_close(got[b], s.oracle(b, 0))
        assert ok, f"b={b} ctx={ctx[b]} max_abs={ma:.3g} rel_l2={rel:.3g}"


@pytest.mark.parametrize("Hq,Hkv", [(16, 8), (32, 8), (8, 1), (4, 4), (24, 8)])
def test_full_if_matches_oracle_and_skips_unflagged(Hq, Hkv):
    ctx = [0, 17, 2052, 2053, 2064, 4096, 5000, 9000, 16, 3333]
    s = Setup(_wl(ctx, Hq, Hkv, seed=78))
    flags = np.array([1, 0, 1, 1, 0, 1, 1, 1, 1, 0], np.int32)
    flag = torch.from_numpy(flags).cuda()
    out = torch.full((s.wl.B, Hq, 128), 7.0, device="cuda")
    s.oda.oda_attend_full_if(s.ctx, s.layer, s.pt, s.pos, flag, s.q, s.kn, s.vn, out)
    torch.cuda.synchronize()
    assert s.oda.oda_get_error(s.ctx) == 0
    got = out.cpu().numpy()
    for b in range(s.wl.B):
        if flags[b]:
            ok, ma, rel = attn_close(got[b], s.oracle(b, 1))
            assert ok, f"b={b} ctx={ctx[b]} max_abs={ma:.3g} rel_l2={rel:.3g}"
        else:
            assert np.all(got[b] == 7.0), f"unflagged b={b} was written"


def test_local_equals_full_where_sets_coincide():
    ctx = [0, 5, 1000, 2051]
    s = Setup(_wl(ctx, seed=79))
    o1 = torch.zeros((4, 16, 128), device="cuda")
    o2 = torch.zeros_like(o1)
    s.oda.oda_attend_local(s.ctx, s.layer, s.pt, s.pos, s.q, s.kn, s.vn, o1)
    s.oda.oda_attend_full_if(s.ctx, s.layer, s.pt, s.pos, torch.ones(4, dtype=torch.int32, device="cuda"),
                             s.q, s.kn, s.vn, o2)
    torch.cuda.synchronize()
    # same set, same pages: identical except for the split schedule, within the bar
    for b in range(4):
        ok, ma, rel = attn_close(o1[b].cpu().numpy(), o2[b].cpu().numpy())
        assert ok, (b, ma, rel)


def test_index_sets_bit_exact():
    ctx = EDGE_CTX + [131072]
    wl = _wl(ctx, seed=80)
    from conditional_sparse_attention_b200 import oda
    max_pages = wl.max_pages()
    cfg = oda.make_config(wl.B, 16, 8, max_pages, 2048)
    c = oda.oda_create(cfg)
    pos = torch.tensor([x + 1 for x in ctx], dtype=torch.int32, device="cuda")
    flags = np.array([(i % 3) != 1 for i in range(len(ctx))], np.int32)
    flag = torch.from_numpy(flags).cuda()
    cap = 131073 + 8
    positions = torch.zeros((wl.B, cap), dtype=torch.int32, device="cuda")
    counts = torch.zeros(wl.B, dtype=torch.int32, device="cuda")
    for mode in (0, 1):
        oda.oda_index_positions(c, mode, pos, flag, positions, cap, counts)
        torch.cuda.synchronize()
        P, C = positions.cpu().numpy(), counts.cpu().numpy()
        for b, x in enumerate(ctx):
            t = x + 1
            if mode == 1 and not flags[b]:
                assert C[b] == 0
                continue
            ref = local_set(t) if mode == 0 else full_set(t)
            got = P[b, :C[b]].tolist()
            assert len(got) == len(set(got)), "a position was visited twice"
            assert set(got) == ref, (mode, b, t)
            assert got[-1] == t  # the staged current token comes last


def test_bad_page_entry_sets_error_word():
    ctx = [40, 3000]
    s = Setup(_wl(ctx, seed=81, shuffle=False))
    pt_bad = s.pt.clone()
    pt_bad[1, 100] = s.k.shape[0] + 5   # beyond the pool
    pt_bad[0, 1] = -1
    out = torch.zeros((2, 16, 128), device="cuda")
    s.oda.oda_attend_full_if(s.ctx, s.layer, pt_bad, s.pos, torch.ones(2, dtype=torch.int32, device="cuda"),
                             s.q, s.kn, s.vn, out)
    err = s.oda.oda_get_error(s.ctx)
    assert err & 0x1
    assert np.isfinite(out.cpu().numpy()).all()
    s.oda.oda_clear_error(s.ctx)
    assert s.oda.oda_get_error(s.ctx) == 0
    # position beyond the table's capacity: no output written, error flagged
    pos_bad = s.pos.clone()
    pos_bad[0] = s.max_pages * 16 + 2
    out.fill_(3.0)
    s.oda.oda_attend_local(s.ctx, s.layer, s.pt, pos_bad, s.q, s.kn, s.vn, out)
    assert s.oda.oda_get_error(s.ctx) & 0x2
    assert np.all(out[0].cpu().numpy() == 3.0)


def test_invalid_arguments_rejected_on_host():
    from conditional_sparse_attention_b200 import oda
    from conditional_sparse_attention_b200._lib import OdaError
    with pytest.raises(OdaError):
        oda.oda_create(oda.make_config(1, 16, 5, 10, 2048))        # Hq % Hkv != 0
    with pytest.raises(OdaError):
        oda.oda_create(oda.make_config(1, 16, 8, 10, 2048, head_dim=64))
    s = Setup(_wl([10], seed=82))
    with pytest.raises(OdaError):
        s.oda.oda_attend_local(s.ctx, s.layer, s.pt, s.pos, s.q, s.kn, s.vn, None)


@pytest.mark.parametrize("ctx,Hq,Hkv", [
    # many short sequences: fewer units than CTAs, CTAs spanning several (sequence, head) pairs
    ([int(x) for x in np.random.default_rng(5).integers(0, 300, 40)], 16, 8),
    # one long sequence and one KV head: every CTA claims chunks of the same (b, h)
    ([50000], 8, 1),
    # lengths spread over two orders of magnitude with every sequence flagged
    ([70000, 900, 33, 20000, 4097, 1, 131072 - 3000], 32, 8),
])
def test_full_set_chunk_claims_cover_every_page(ctx, Hq, Hkv):
    s = Setup(_wl(ctx, Hq, Hkv, seed=83))
    flag = torch.ones(len(ctx), dtype=torch.int32, device="cuda")
    out = torch.full((s.wl.B, Hq, 128), 7.0, device="cuda")
    for rep in range(2):   # the second launch runs on counters reset by the first
        s.oda.oda_attend_full_if(s.ctx, s.layer, s.pt, s.pos, flag, s.q, s.kn, s.vn, out)
        torch.cuda.synchronize()
        assert s.oda.oda_get_error(s.ctx) == 0
        got = out.cpu().numpy()
        for b in range(s.wl.B):
            ok, ma, rel = attn_close(got[b], s.oracle(b, 1))
            assert ok, f"rep={rep} b={b} ctx={ctx[b]} max_abs={ma:.3g} rel_l2={rel:.3g}"


def test_full_set_fixed_pattern_is_bitwise_repeatable():
    """deterministic = 1: the pages of each (sequence, head) go to the CTAs in a fixed pattern,
    so repeated launches give identical bits (and match the oracle within tolerance)."""
    ctx = [60000, 900, 20000, 4097, 33, 131072 - 3000]
    s = Setup(_wl(ctx, 32, 8, seed=84), deterministic=True)
    flag = torch.ones(len(ctx), dtype=torch.int32, device="cuda")
    outs = []
    for rep in range(3):
        out = torch.full((s.wl.B, 32, 128), 7.0, device="cuda")
        s.oda.oda_attend_full_if(s.ctx, s.layer, s.pt, s.pos, flag, s.q, s.kn, s.vn, out)
        torch.cuda.synchronize()
        assert s.oda.oda_get_error(s.ctx) == 0
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
    for b in range(s.wl.B):
        ok, ma, rel = attn_close(outs[0][b], s.oracle(b, 1))
        assert ok, f"b={b} ctx={ctx[b]} max_abs={ma:.3g} rel_l2={rel:.3g}"


def test_context_with_smaller_group_keeps_earlier_context_working():
    """The full-set kernel's shared-memory limit is one setting per process: creating a context
    with g = 1 after one with g = 8 must not break the g = 8 context's launches."""
    from conditional_sparse_attention_b200 import oda
    ctx = [3000, 131]
    s8 = Setup(_wl(ctx, 64, 8, seed=85))           # g = 8: the largest shared-memory need
    c1 = oda.oda_create(oda.make_config(2, 4, 4, s8.max_pages, 512))   # g = 1, created later
    flag = torch.ones(2, dtype=torch.int32, device="cuda")
    out = torch.full((2, 64, 128), 7.0, device="cuda")
    s8.oda.oda_attend_full_if(s8.ctx, s8.layer, s8.pt, s8.pos, flag, s8.q, s8.kn, s8.vn, out)
    torch.cuda.synchronize()
    assert s8.oda.oda_get_error(s8.ctx) == 0
    got = out.cpu().numpy()
    for b in range(2):
        ok, ma, rel = attn_close(got[b], s8.oracle(b, 1))
        assert ok, (b, ma, rel)
    c1.close()
