"""GPU parity of the fp8 (e4m3) KV page path against the oracle.

* oda_kv8_pack and oda_commit_fp8 write codes and scales bit-exact to the oracle's quantiser
  (oracle.kv_fp8.quantize_rows), read back here with a decoder of the block layout written from
  its description in include/oda.h (not from the kernels).
* oda_attend_local_fp8 / oda_attend_full_if_fp8 match oracle.kv_fp8.attend_quantized (attention
  over the decoded cache plus the exact bf16 current token) within the attention tolerance, at
  the edge contexts, for every GQA group size, with pools whose unused slots are NaN codes.
"""
import numpy as np
import pytest
import torch

from helpers import attn_close, build_all, decode_kv8_block as decode_block
from oracle import kv_fp8
from oracle.attention import bf16_to_f64
from oracle.sets import full_set, local_set
from workload import configs, device as wdev, inputs

pytestmark = pytest.mark.gpu

BLOCK = 4224
EDGE_CTX = [0, 1, 3, 4, 5, 15, 16, 17, 100, 2047, 2048, 2050, 2051, 2052, 2053, 2058, 2062,
            2063, 2064, 2065, 2100, 4095, 4096, 5000]


@pytest.fixture(scope="module", autouse=True)
def _build():
    build_all()


def _wl(ctx, Hq=16, Hkv=8, seed=177, shuffle=True):
    return configs.cfg0().replace(name="t_kv8", seed=seed, B=len(ctx), n_layers=1,
                                  attn_layers=(0,), Hq=Hq, Hkv=Hkv, ctx=tuple(ctx), steps=2,
                                  shuffle_pages=shuffle)


class Setup8:
    """bf16 pools (NaN outside every sequence) packed into an fp8 pool; step-0 q and staging."""

    def __init__(self, wl, deterministic=False):
        from conditional_sparse_attention_b200 import oda
        self.oda, self.wl = oda, wl
        dev = torch.device("cuda")
        self.max_pages = wl.max_pages()
        self.pt_np = inputs.page_table(wl, self.max_pages)
        self.pt = torch.from_numpy(self.pt_np).to(dev)
        n_pool = wl.B * self.max_pages
        self.k = torch.full((n_pool, wl.Hkv, 16, 128), float("nan"), dtype=torch.bfloat16, device=dev)
        self.v = torch.full_like(self.k, float("nan"))
        wdev.fill_kv(self.k, self.pt, wl.ctx, [inputs.cache_key(wl, "k", 0, b) for b in range(wl.B)], wl.Hkv)
        wdev.fill_kv(self.v, self.pt, wl.ctx, [inputs.cache_key(wl, "v", 0, b) for b in range(wl.B)], wl.Hkv)
        self.kv8 = torch.zeros((n_pool, wl.Hkv, BLOCK), dtype=torch.uint8, device=dev)
        self.layer8 = oda.kv8_layer(self.kv8)
        oda.oda_kv8_pack(oda.kv_layer(self.k, self.v), self.layer8, wl.Hkv)
        q, kn, vn = inputs.step_qkv(wl, 0, 0, 0)
        self.q_np, self.kn_np, self.vn_np = q, kn, vn
        self.q = torch.from_numpy(q.view(np.int16)).to(dev)
        self.kn = torch.from_numpy(kn.view(np.int16)).to(dev)
        self.vn = torch.from_numpy(vn.view(np.int16)).to(dev)
        self.pos = torch.tensor([c + 1 for c in wl.ctx], dtype=torch.int32, device=dev)
        cfg = oda.make_config(wl.B, wl.Hq, wl.Hkv, self.max_pages, max(512, wl.D), wl.sinks,
                              wl.window, deterministic=deterministic)
        self.ctx = oda.oda_create(cfg)

    def oracle(self, b, mode):
        wl = self.wl
        t = wl.ctx[b] + 1
        kc = inputs.cache_tokens(wl, "k", 0, b, wl.ctx[b])
        vc = inputs.cache_tokens(wl, "v", 0, b, wl.ctx[b])
        S = local_set(t, wl.sinks, wl.window) if mode == 0 else full_set(t)
        return kv_fp8.attend_quantized(self.q_np[b], kc, vc, self.kn_np[b], self.vn_np[b], S)


def test_pack_is_bit_exact_to_the_oracle_quantiser():
    wl = _wl([37, 2053, 300], seed=170)
    s = Setup8(wl)
    torch.cuda.synchronize()
    pool = s.kv8.cpu().numpy()
    for b in range(wl.B):
        n = wl.ctx[b]
        kb = inputs.cache_tokens(wl, "k", 0, b, n)
        vb = inputs.cache_tokens(wl, "v", 0, b, n)
        kc, ks = kv_fp8.quantize_rows(bf16_to_f64(kb))
        vc, vs = kv_fp8.quantize_rows(bf16_to_f64(vb))
        for tok in range(n):
            phys = s.pt_np[b, tok // 16]
            for h in range(wl.Hkv):
                K, V, sk, sv = decode_block(pool[phys, h])
                j = tok % 16
                assert np.array_equal(K[j], kc[tok, h]), (b, tok, h, "K codes")
                assert np.array_equal(V[j], vc[tok, h]), (b, tok, h, "V codes")
                assert sk[j] == ks[tok, h] and sv[j] == vs[tok, h], (b, tok, h, "scales")


@pytest.mark.parametrize("Hq,Hkv", [(16, 8), (32, 8), (8, 1), (4, 4), (24, 8), (64, 8)])
def test_local_fp8_matches_oracle(Hq, Hkv):
    s = Setup8(_wl(EDGE_CTX, Hq, Hkv))
    out = torch.full((s.wl.B, Hq, 128), 7.0, device="cuda")
    s.oda.oda_attend_local_fp8(s.ctx, s.layer8, s.pt, s.pos, s.q, s.kn, s.vn, out)
    torch.cuda.synchronize()
    assert s.oda.oda_get_error(s.ctx) == 0
    got = out.cpu().numpy()
    for b in range(s.wl.B):
        ok, ma, rel = attn_close(got[b], s.oracle(b, 0))
        assert ok, f"b={b} ctx={s.wl.ctx[b]} max_abs={ma:.3g} rel_l2={rel:.3g}"


@pytest.mark.parametrize("Hq,Hkv", [(16, 8), (32, 8), (8, 1), (4, 4), (24, 8), (64, 8)])
def test_full_fp8_matches_oracle_and_skips_unflagged(Hq, Hkv):
    ctx = [0, 17, 2052, 2053, 2064, 4096, 5000, 9000, 16, 3333]
    s = Setup8(_wl(ctx, Hq, Hkv, seed=178))
    flags = np.array([1, 0, 1, 1, 0, 1, 1, 1, 1, 0], np.int32)
    flag = torch.from_numpy(flags).cuda()
    out = torch.full((s.wl.B, Hq, 128), 7.0, device="cuda")
    for rep in range(2):
        s.oda.oda_attend_full_if_fp8(s.ctx, s.layer8, s.pt, s.pos, flag, s.q, s.kn, s.vn, out)
        torch.cuda.synchronize()
        assert s.oda.oda_get_error(s.ctx) == 0
        got = out.cpu().numpy()
        for b in range(s.wl.B):
            if flags[b]:
                ok, ma, rel = attn_close(got[b], s.oracle(b, 1))
                assert ok, f"rep={rep} b={b} ctx={ctx[b]} max_abs={ma:.3g} rel_l2={rel:.3g}"
            else:
                assert np.all(got[b] == 7.0), f"unflagged b={b} was written"


def test_full_fp8_long_contexts_and_deterministic_replays():
    ctx = [50000, 900, 131072 - 3000, 33]
    s = Setup8(_wl(ctx, 32, 8, seed=179), deterministic=True)
    flag = torch.ones(len(ctx), dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(2):
        out = torch.zeros((s.wl.B, 32, 128), device="cuda")
        s.oda.oda_attend_full_if_fp8(s.ctx, s.layer8, s.pt, s.pos, flag, s.q, s.kn, s.vn, out)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
    assert s.oda.oda_get_error(s.ctx) == 0
    assert np.array_equal(outs[0], outs[1])
    for b in range(s.wl.B):
        ok, ma, rel = attn_close(outs[0][b], s.oracle(b, 1))
        assert ok, f"b={b} ctx={ctx[b]} max_abs={ma:.3g} rel_l2={rel:.3g}"


def test_fp8_local_equals_full_where_sets_coincide_and_tracks_bf16():
    """Same set -> same value (within the bar); and the format's error against the bf16 cache
    stays at the e4m3 level (a few percent relative)."""
    from oracle.attention import attend_bits
    ctx = [5, 1000, 2051]
    s = Setup8(_wl(ctx, seed=180))
    o1 = torch.zeros((3, 16, 128), device="cuda")
    o2 = torch.zeros_like(o1)
    s.oda.oda_attend_local_fp8(s.ctx, s.layer8, s.pt, s.pos, s.q, s.kn, s.vn, o1)
    s.oda.oda_attend_full_if_fp8(s.ctx, s.layer8, s.pt, s.pos, torch.ones(3, dtype=torch.int32, device="cuda"),
                                 s.q, s.kn, s.vn, o2)
    torch.cuda.synchronize()
    for b in range(3):
        ok, ma, rel = attn_close(o1[b].cpu().numpy(), o2[b].cpu().numpy())
        assert ok, (b, ma, rel)
        t = ctx[b] + 1
        ref16 = attend_bits(s.q_np[b], inputs.cache_tokens(s.wl, "k", 0, b, ctx[b]),
                            inputs.cache_tokens(s.wl, "v", 0, b, ctx[b]), s.kn_np[b], s.vn_np[b],
                            full_set(t))
        r = np.linalg.norm(o2[b].cpu().numpy() - ref16) / np.linalg.norm(ref16)
        assert r < 0.08, (b, r)


def test_commit_fp8_writes_the_chosen_branch_bit_exact():
    from conditional_sparse_attention_b200 import oda
    ctx = [40, 2047, 16]
    wl = _wl(ctx, seed=181)
    s = Setup8(wl)
    L, B, Hkv, D = 2, wl.B, wl.Hkv, wl.D
    dev = torch.device("cuda")
    pools = [s.kv8, s.kv8.clone()]
    layers = [oda.kv8_layer(p) for p in pools]
    before = [p.cpu().numpy() for p in pools]
    st = {}
    for name in ("kl", "vl", "kf", "vf"):
        tag = {"kl": 11, "vl": 12, "kf": 13, "vf": 14}[name]
        from workload import gen
        st[name] = gen.normal_bf16(gen.key(wl.seed, 900 + tag), L * B * Hkv * 128).reshape(L, B, Hkv, 128)
    tt = {k: torch.from_numpy(v.view(np.int16)).to(dev) for k, v in st.items()}
    h_l = torch.randn(B, D, device=dev)
    h_f = torch.randn(B, D, device=dev)
    h_prev = torch.zeros(B, D, device=dev)
    flag = torch.tensor([1, 0, 1], dtype=torch.int32, device=dev)
    pos = s.pos.clone()
    oda.oda_commit_fp8(s.ctx, layers, s.pt, pos, flag, tt["kl"], tt["vl"], tt["kf"], tt["vf"],
                       h_l, h_f, h_prev)
    torch.cuda.synchronize()
    assert s.oda.oda_get_error(s.ctx) == 0
    assert pos.cpu().tolist() == [c + 2 for c in ctx]
    assert torch.equal(h_prev[0], h_f[0]) and torch.equal(h_prev[1], h_l[1]) and torch.equal(h_prev[2], h_f[2])
    for l in range(L):
        after = pools[l].cpu().numpy()
        changed = np.zeros(after.shape[:2], bool)
        for b in range(B):
            t = ctx[b] + 1
            phys, j = s.pt_np[b, (t - 1) // 16], (t - 1) % 16
            changed[phys] = True
            br = "f" if flag[b] else "l"
            kc, ks = kv_fp8.quantize_rows(bf16_to_f64(st["k" + br][l, b]))
            vc, vs = kv_fp8.quantize_rows(bf16_to_f64(st["v" + br][l, b]))
            for h in range(Hkv):
                K, V, sk, sv = decode_block(after[phys, h])
                K0, V0, sk0, sv0 = decode_block(before[l][phys, h])
                assert np.array_equal(K[j], kc[h]) and np.array_equal(V[j], vc[h])
                assert sk[j] == ks[h] and sv[j] == vs[h]
                other = [i for i in range(16) if i != j]
                assert np.array_equal(K[other], K0[other]) and np.array_equal(V[other], V0[other])
                assert np.array_equal(sk[other], sk0[other], equal_nan=True)
                assert np.array_equal(sv[other], sv0[other], equal_nan=True)
        # no other page was touched
        assert np.array_equal(after[~changed], before[l][~changed])
