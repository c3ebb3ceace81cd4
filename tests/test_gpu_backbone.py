"""GPU parity of the synthetic-backbone calls (include/oda_backbone.h) and of whole decode
steps of the synthetic model against the oracle (oracle.backbone, oracle.step).

The stand-in's definition rounds projection inputs, q/k/v and the MLP activation to bf16; the GPU
takes those roundings from fp32 values and the oracle from fp64 ones, so a value within an fp32
rounding error of a bf16 midpoint can land one bf16 step apart.  bf16 outputs are therefore
compared as: equal except for at most 0.5% of the elements, and those within one bf16 step; fp32
outputs within relative L2 1e-4 (projections) or the attention tolerance (attention outputs).
Greedy tokens are compared where the oracle's two largest logits differ by more than 1e-3.
Along a trajectory the two residual streams (fp32 here, fp64 in the oracle) drift apart by the
roundings of every layer.  So the kernels are checked teacher-forced - every attention output
against the oracle on the GPU's own q/k/v and committed cache, the recall score on the GPU's own
inputs - and the independent oracle trajectory within a drift bound; the cache must hold exactly
the GPU's own committed rows.
"""
import numpy as np
import pytest
import torch

from helpers import TIE_BAND, attn_close, build_all, logical_cache, packed_index, score_close
from oracle import backbone as BB
from oracle import step as OS
from oracle.attention import bf16_to_f64
from oracle.head import recall_head
from workload import configs, device as wdev, gen, inputs

pytestmark = pytest.mark.gpu
TOKEN_TIE = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _build():
    build_all()


def _bits_t(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _packed_t(ctx, a):
    """Row-major bf16 bits (numpy) -> a packed device matrix (via oda_bb_pack_weight)."""
    from conditional_sparse_attention_b200 import oda
    src = _bits_t(a)
    dst = torch.empty_like(src)
    oda.oda_bb_pack_weight(ctx, src, dst)
    return dst


def bf16_close(got_bits, ref_bits, frac=5e-3):
    g, r = bf16_to_f64(got_bits), bf16_to_f64(ref_bits)
    diff = g != r
    step = np.abs(r) * 2.0 ** -7 + 1e-30
    return diff.mean() <= frac and np.all(np.abs(g - r)[diff] <= step[diff] * 1.01)


def rel_l2(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-30))


def _wl(B=3, Hq=4, Hkv=2, F=1024, V=2000, seed=300):
    return configs.bb_qwen3_1p7b().replace(name=f"t_bb_{B}_{Hq}_{F}", seed=seed, B=B, n_layers=1,
                                           attn_layers=(0,), Hq=Hq, Hkv=Hkv, ctx=(10,) * B,
                                           ffn=F, vocab=V, rates=(0.5,) * B)


class Layer:
    def __init__(self, wl):
        from conditional_sparse_attention_b200 import oda
        self.oda = oda
        self.wl = wl
        self.w = {n: inputs.bb_weight(wl, 0, n) for n in inputs.BB_TENSORS}
        self.ga, self.gm = inputs.bb_norms(wl, 0)
        self.ctx = oda.oda_create(oda.make_config(wl.B, wl.Hq, wl.Hkv, 8, max(512, wl.D)))
        d = {n: _packed_t(self.ctx, v) for n, v in self.w.items()}
        self.d = d
        self.tga, self.tgm = torch.from_numpy(self.ga).cuda(), torch.from_numpy(self.gm).cuda()
        self.layer = oda.bb_layer(self.tga, d["w_qkv"], d["w_o"], self.tgm, d["w_gate"], d["w_up"],
                                  d["w_down"])


@pytest.mark.parametrize("B,Hq,Hkv,F", [(1, 4, 2, 1024), (3, 4, 2, 1536), (8, 8, 2, 512),
                                        (1, 16, 8, 6144)])
def test_projections_match_oracle(B, Hq, Hkv, F):
    wl = _wl(B, Hq, Hkv, F)
    L = Layer(wl)
    oda, D = L.oda, wl.D
    rng = np.random.default_rng(B + F)
    x = rng.normal(0, 2, (B, D)).astype(np.float32)
    o = rng.normal(0, 1, (B, D)).astype(np.float32)
    tx = torch.from_numpy(x).cuda()
    q = torch.zeros((B, Hq, 128), dtype=torch.int16, device="cuda")
    k = torch.zeros((B, Hkv, 128), dtype=torch.int16, device="cuda")
    v = torch.zeros_like(k)
    oda.oda_bb_qkv(L.ctx, L.layer, tx, q, k, v)
    x1 = tx.clone()
    oda.oda_bb_attn_out(L.ctx, L.layer, torch.from_numpy(o).cuda(), x1)
    x2 = tx.clone()
    act = torch.zeros((B, F), dtype=torch.bfloat16, device="cuda")
    oda.oda_bb_mlp(L.ctx, L.layer, x2, act)
    h = torch.zeros_like(tx)
    oda.oda_bb_final_norm(L.ctx, L.tgm, tx, h)
    torch.cuda.synchronize()
    assert oda.oda_get_error(L.ctx) == 0
    rq, rk, rv = BB.attn_in(x.astype(np.float64), L.ga, L.w["w_qkv"], Hq, Hkv)
    u16 = lambda t: t.cpu().numpy().view(np.uint16)  # noqa: E731
    assert bf16_close(u16(q), rq) and bf16_close(u16(k), rk) and bf16_close(u16(v), rv)
    assert rel_l2(x1.cpu().numpy(), BB.attn_out(x, o, L.w["w_o"])) < 1e-5
    ref2 = BB.mlp(x.astype(np.float64), L.gm, L.w["w_gate"], L.w["w_up"], L.w["w_down"])
    assert rel_l2(x2.cpu().numpy() - x, ref2 - x) < 1e-3
    assert rel_l2(h.cpu().numpy(), BB.rmsnorm(x.astype(np.float64), L.gm)) < 1e-6
    L.ctx.close()


@pytest.mark.parametrize("B,V", [(1, 2000), (5, 4096), (8, 151936)])
def test_lm_head_matches_oracle(B, V):
    wl = _wl(B, 16, 8, 512, V, seed=301)
    from conditional_sparse_attention_b200 import oda
    D = wl.D
    ctx = oda.oda_create(oda.make_config(B, wl.Hq, wl.Hkv, 8, D))
    E = inputs.bb_embed(wl)
    rowmajor = torch.empty((V, D), dtype=torch.int16, device="cuda")
    wdev.fill_normal_bf16(rowmajor, inputs.bb_embed_key(wl), 0, inputs.BB_EMBED_LOG2_SCALE)
    assert np.array_equal(rowmajor.cpu().numpy().view(np.uint16), E)
    tE = torch.empty_like(rowmajor)
    oda.oda_bb_pack_weight(ctx, rowmajor, tE)
    del rowmajor
    rng = np.random.default_rng(V)
    h = rng.normal(0, 1, (B, D)).astype(np.float32)
    logits = torch.zeros((B, V), device="cuda")
    tok = torch.zeros(B, dtype=torch.int32, device="cuda")
    emb = torch.zeros((B, D), device="cuda")
    oda.oda_bb_lm_head(ctx, tE, V, torch.from_numpy(h).cuda(), logits, tok, emb)
    torch.cuda.synchronize()
    ref, rtok = BB.lm_head(h.astype(np.float64), E)
    assert rel_l2(logits.cpu().numpy(), ref) < 1e-5
    top2 = np.sort(ref, axis=1)[:, -2:]
    for b in range(B):
        if top2[b, 1] - top2[b, 0] > TOKEN_TIE:
            assert tok[b].item() == rtok[b]
        assert np.array_equal(emb[b].cpu().numpy(), bf16_to_f64(E[tok[b].item()]).astype(np.float32))
    # embedding lookup alone, with an out-of-range token taken as 0
    t2 = torch.tensor([3, V + 7, 0, 1, 2, 3, 4, 5][:B], dtype=torch.int32, device="cuda")
    oda.oda_bb_embed(ctx, tE, V, t2, emb)
    torch.cuda.synchronize()
    want = [3, 0, 0, 1, 2, 3, 4, 5][:B]
    assert t2.cpu().tolist() == want
    assert np.array_equal(emb.cpu().numpy(), bf16_to_f64(E[want]).astype(np.float32))
    ctx.close()


def _small_model(kv="bf16", seed=2005):
    return configs.bb_qwen3_1p7b().replace(name=f"t_bb_traj_{kv}", seed=seed, B=2, n_layers=2,
                                           attn_layers=(0, 1), Hq=4, Hkv=2, ctx=(100, 3000),
                                           steps=4, rates=(0.5, 0.5), ffn=1024, vocab=2000)


# Drift bound of the independent trajectory: every layer re-rounds four bf16 vectors from an fp32
# stream (the oracle from fp64), each rounding moving ~2^-9 of an element when it flips; over the
# two layers and four steps here the outputs stay within 1e-2 relative L2.
DRIFT = 1e-2


@pytest.mark.parametrize("kv,graph", [("bf16", True), ("bf16", False), ("fp8", True)])
def test_backbone_trajectory_matches_oracle(kv, graph):
    from conditional_sparse_attention_b200.engine import OdaDecoder
    from oracle.attention import attend_bits
    from oracle.kv_fp8 import attend_quantized
    from oracle.sets import full_set, local_set
    wl = _small_model(kv)
    dec = OdaDecoder(wl, perturb_head=True, kv_format=kv)
    P = {k: v.cpu().numpy() for k, v in dec.head_params.items()}
    if graph:
        dec.capture()
    st = OS.initial_state(wl, kv=kv)
    assert dec.token.cpu().tolist() == st.tokens.tolist()
    # the GPU's own committed rows per (layer, sequence): the cache the kernels read
    own_k = [[inputs.cache_tokens(wl, "k", a, b, wl.ctx[b]) for b in range(wl.B)] for a in range(wl.L)]
    own_v = [[inputs.cache_tokens(wl, "v", a, b, wl.ctx[b]) for b in range(wl.B)] for a in range(wl.L)]
    u16 = lambda t: t.cpu().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    for s in range(wl.steps):
        sched = inputs.schedule(wl, s)
        # the head is teacher-forced: scored by the oracle on the GPU's own inputs
        hp = dec.h_prev.cpu().numpy().astype(np.float64)
        em = dec.emb.cpu().numpy().astype(np.float64)
        pos = dec.pos.cpu().numpy().copy()
        dec.step(dec.make_step_buffer(s))
        dec.synchronize()
        st, rec = OS.decode_step(wl, st, s, P, sched=sched)
        flags = dec.flag.cpu().numpy()
        assert flags.tolist() == rec.flags.tolist(), s
        sc = dec.score.cpu().numpy()
        hl = dec.h[0].cpu().numpy().astype(np.float64)
        for b in range(wl.B):
            ref = recall_head(P, hp[b], em[b], hl[b])
            assert score_close(sc[b], ref), (s, b, sc[b], ref)
        o = dec.o.cpu().numpy()
        q_all, k_all, v_all = u16(dec.bb_q), u16(dec.bb_k), u16(dec.bb_v)
        for a in range(wl.L):
            for br in (0, 1):
                rows = [b for b in range(wl.B) if br == 0 or flags[b]]
                for b in rows:
                    t = int(pos[b])
                    S = local_set(t, wl.sinks, wl.window) if br == 0 else full_set(t)
                    # kernel parity: the oracle attends with the GPU's own q/k/v and cache
                    args = (q_all[br, a, b], own_k[a][b], own_v[a][b], k_all[br, a, b], v_all[br, a, b], S)
                    ref = attend_bits(*args) if kv == "bf16" else attend_quantized(*args)
                    ok, ma, rel = attn_close(o[br, a, b], ref.reshape(-1))
                    assert ok, ("teacher-forced", s, a, br, b, ma, rel)
                    # drift of the independent trajectory
                    r = rel_l2(o[br, a, b], rec.o[(br, a)][b].reshape(-1))
                    assert r < DRIFT, ("drift", s, a, br, b, r)
                if a == 0 and rows:   # from the exact embedding: equal up to rounding edges
                    assert bf16_close(k_all[br, a][rows], rec.staged_k[(br, a)][rows]), (s, br, "k")
        for b in range(wl.B):
            br = 1 if flags[b] else 0
            for a in range(wl.L):
                own_k[a][b] = np.concatenate([own_k[a][b], k_all[br, a, b][None]])
                own_v[a][b] = np.concatenate([own_v[a][b], v_all[br, a, b][None]])
            assert rel_l2(hl[b], rec.h[0][b]) < DRIFT, (s, b)
        top2 = np.sort(rec.logits, axis=1)[:, -2:]
        tok = dec.token.cpu().numpy()
        if np.any(top2[:, 1] - top2[:, 0] <= TOKEN_TIE):
            pytest.skip(f"near-tie of the greedy token at step {s}; trajectories may part")
        assert tok.tolist() == rec.tokens.tolist(), (s, tok, rec.tokens)
        assert dec.pos.cpu().tolist() == st.pos
    assert dec.device_error() == 0
    # the commit wrote the GPU's own chosen-branch rows into the cache, bit for bit (bf16)
    if kv == "bf16":
        pt = dec.page_table.cpu().numpy()
        for a in range(wl.L):
            kp = dec.k_pool[a].cpu().view(torch.int16).numpy().view(np.uint16)
            vp = dec.v_pool[a].cpu().view(torch.int16).numpy().view(np.uint16)
            for b in range(wl.B):
                n = wl.ctx[b] + wl.steps
                assert np.array_equal(logical_cache(kp, pt, b, n), own_k[a][b])
                assert np.array_equal(logical_cache(vp, pt, b, n), own_v[a][b])
    dec.close()


@pytest.mark.parametrize("B,Hq,Hkv,F,with_next", [(1, 4, 2, 1024, True), (3, 4, 2, 1536, True),
                                                  (8, 8, 2, 512, False), (4, 16, 8, 6144, True),
                                                  (8, 16, 8, 6144, False)])
def test_post_attention_equals_separate_calls(B, Hq, Hkv, F, with_next):
    """oda_bb_post_attention does the arithmetic of oda_bb_attn_out, oda_bb_mlp and oda_bb_qkv (of
    the next layer) in the same order, so its outputs equal theirs bit for bit; the separate calls
    are the ones checked against the oracle above."""
    from conditional_sparse_attention_b200 import oda
    wl = _wl(B, Hq, Hkv, F).replace(n_layers=2, attn_layers=(0, 1))
    D = wl.D
    ctx = oda.oda_create(oda.make_config(B, Hq, Hkv, 8, D))
    layers, keep = [], []
    for a in range(2):
        w = {}
        for n, (R, C) in inputs.bb_shapes(wl).items():
            rowmajor = torch.empty((R, C), dtype=torch.bfloat16, device="cuda")
            wdev.fill_normal_bf16(rowmajor, inputs.bb_weight_key(wl, a, n), 0, inputs.bb_log2_scale(C))
            w[n] = torch.empty_like(rowmajor)
            oda.oda_bb_pack_weight(ctx, rowmajor, w[n])
        ga, gm = (torch.from_numpy(g).cuda() for g in inputs.bb_norms(wl, a))
        keep += [w, ga, gm]
        layers.append(oda.bb_layer(ga, w["w_qkv"], w["w_o"], gm, w["w_gate"], w["w_up"], w["w_down"]))
    rng = np.random.default_rng(F + B)
    x0 = torch.from_numpy(rng.normal(0, 2, (B, D)).astype(np.float32)).cuda()
    o = torch.from_numpy(rng.normal(0, 1, (B, D)).astype(np.float32)).cuda()

    def outputs():
        return (torch.zeros((B, Hq, 128), dtype=torch.int16, device="cuda"),
                torch.zeros((B, Hkv, 128), dtype=torch.int16, device="cuda"),
                torch.zeros((B, Hkv, 128), dtype=torch.int16, device="cuda"),
                torch.zeros((B, F), dtype=torch.bfloat16, device="cuda"))

    x1 = x0.clone()
    q1, k1, v1, act1 = outputs()
    oda.oda_bb_attn_out(ctx, layers[0], o, x1)
    oda.oda_bb_mlp(ctx, layers[0], x1, act1)
    if with_next:
        oda.oda_bb_qkv(ctx, layers[1], x1, q1, k1, v1)
    for rep in range(3):   # repeated launches: the barrier counters return to zero
        x2 = x0.clone()
        q2, k2, v2, act2 = outputs()
        if with_next:
            oda.oda_bb_post_attention(ctx, layers[0], layers[1], o, x2, act2, q2, k2, v2)
        else:
            oda.oda_bb_post_attention(ctx, layers[0], None, o, x2, act2)
        torch.cuda.synchronize()
        assert oda.oda_get_error(ctx) == 0
        assert torch.equal(x1, x2), rep
        assert torch.equal(act1, act2), rep
        assert torch.equal(q1, q2) and torch.equal(k1, k2) and torch.equal(v1, v2), rep
    with pytest.raises(oda.OdaError):   # the next layer's outputs are required
        oda.oda_bb_post_attention(ctx, layers[0], layers[1], o, x2, act2)
    ctx.close()


@pytest.mark.parametrize("graph", [True, False])
def test_backbone_fused_step_equals_separate_launches(graph):
    """A whole-model trajectory with the fused post-attention launch equals the one with the
    separate projection launches, bit for bit (same kernels' arithmetic, fewer launches)."""
    from conditional_sparse_attention_b200.engine import OdaDecoder
    wl = _small_model("bf16", seed=2011).replace(n_layers=3, attn_layers=(0, 1, 2))
    runs = []
    for fused in (True, False):
        dec = OdaDecoder(wl, perturb_head=True, bb_fused=fused)
        if graph:
            dec.capture()
        out = []
        for s in range(wl.steps):
            dec.step(dec.make_step_buffer(s))
            dec.synchronize()
            out.append((dec.token.cpu().clone(), dec.h_prev.cpu().clone(), dec.o.cpu().clone(),
                        dec.flag.cpu().clone()))
        assert dec.device_error() == 0
        runs.append(out)
        dec.close()
    for s, (a, b) in enumerate(zip(*runs)):
        for ta, tb in zip(a, b):
            assert torch.equal(ta, tb), s


@pytest.mark.parametrize("rows,cols", [(16, 512), (48, 1536), (4096, 2048), (2048, 6144)])
def test_pack_weight_layout(rows, cols):
    """oda_bb_pack_weight moves every element to the offset the header's formula gives, bit for
    bit; bad shapes, aliasing and misalignment are rejected."""
    from conditional_sparse_attention_b200 import oda
    ctx = oda.oda_create(oda.make_config(1, 4, 2, 8, 512))
    rng = np.random.default_rng(rows + cols)
    a = rng.integers(0, 2**16, (rows, cols), dtype=np.uint16)
    got = _packed_t(ctx, a).cpu().numpy().view(np.uint16).reshape(-1)
    want = np.empty(rows * cols, dtype=np.uint16)
    want[packed_index(rows, cols).reshape(-1)] = a.reshape(-1)
    assert np.array_equal(got, want)
    t = torch.zeros((32, 1024), dtype=torch.bfloat16, device="cuda")
    for src, dst in [(t[:24], torch.zeros((24, 1024), dtype=torch.bfloat16, device="cuda")),
                     (t[:, :768], torch.zeros((32, 768), dtype=torch.bfloat16, device="cuda")),
                     (t, t)]:
        with pytest.raises(oda.OdaError):
            oda.oda_bb_pack_weight(ctx, src.contiguous() if src is not t else src, dst)
    flat = torch.zeros(32 * 1024 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(oda.OdaError):   # 2 bytes off 16-byte alignment
        oda.oda_bb_pack_weight(ctx, flat[1:1 + 32 * 1024].view(32, 1024), torch.zeros_like(t))
    ctx.close()
