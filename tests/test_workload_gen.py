"""Host generator checks: determinism, slice consistency, bf16 rounding vs torch, N(0,1) moments."""
import numpy as np
import torch

from workload import configs, gen, inputs


def test_stream_slices_are_consistent():
    k = gen.key(5, 1, 2, 3)
    full = gen.raw_u64(k, 1000)
    assert np.array_equal(full[300:700], gen.raw_u64(k, 400, start=300))
    assert np.array_equal(gen.normal_bf16(k, 1000)[10:20], gen.normal_bf16(k, 10, start=10))
    assert gen.key(5, 1, 2, 3) != gen.key(5, 1, 3, 2) != gen.key(6, 1, 2, 3)


def test_mix64_matches_python_ints():
    z = np.array([0, 1, 2**63 + 12345, 2**64 - 1], dtype=np.uint64)
    ref = [gen._mix64_int(int(x)) for x in z]
    assert [int(x) for x in gen.mix64(z)] == ref


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.00390625, 1.01171875, -2.0, 0.0, 3.0e38], np.float32)])
    ours = gen.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_normal_table_and_moments():
    t = gen.bf16_bits_to_f32(gen.normal_bf16_table())
    assert np.all(np.diff(t) >= 0) and np.array_equal(t, -t[::-1])
    v = gen.bf16_bits_to_f32(gen.normal_bf16(gen.key(1, 2), 1 << 20)).astype(np.float64)
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1.0) < 0.01
    f = gen.normal_f32(gen.key(3), 1 << 18).astype(np.float64)
    assert abs(f.mean()) < 0.01 and abs(f.std() - 1.0) < 0.01


def test_workload_shapes_and_page_tables():
    wl = configs.cfg3()
    assert len(wl.ctx) == 32 and all(8192 <= c <= 131072 for c in wl.ctx)
    assert all(0.05 <= r <= 0.5 for r in wl.rates)
    mp = wl.max_pages()
    pt = inputs.page_table(wl, mp)
    assert sorted(pt.reshape(-1).tolist()) == list(range(wl.B * mp))
    assert not np.array_equal(pt.reshape(-1), np.arange(wl.B * mp))
    wl2 = configs.cfg2()
    assert wl2.D == 4096 and wl2.g == 4 and wl2.L == 36
    assert configs.cfg4().gdn_layers == tuple(i for i in range(24) if i % 4 != 3)
    q, k, v = inputs.step_qkv(wl2.replace(B=1), 0, 0, 0)
    q1, k1, v1 = inputs.step_qkv(wl2.replace(B=1), 0, 0, 1)
    assert np.array_equal(q, q1)  # layer 0: both branches see the same input
    q2, _, _ = inputs.step_qkv(wl2.replace(B=1), 0, 1, 1)
    q3, _, _ = inputs.step_qkv(wl2.replace(B=1), 0, 1, 0)
    assert not np.array_equal(q2, q3)
