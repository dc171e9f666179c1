"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test fixes one part of what the method computes to something outside the
oracle itself: a mathematical identity (the transform pair preserves q.k), a
textbook routine (softmax attention, a full sort), a library conversion
(numpy float16, torch bfloat16), exact round trips, hand-worked examples
under tests/golden, and properties that hold for any input.
"""
import json
import math
import os

import numpy as np
import pytest

from bit_kv_cache_dqk_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantizer_examples.json")


def textbook_attention(q, k, v, scale):
    """softmax(q k^T * scale) v in fp64; q [h][d], k/v [L][d]."""
    s = (q @ k.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


# ------------------------------------------------------------------ formats
def test_f16_rounding_matches_numpy(oracle_mod):
    rng = np.random.default_rng(0)
    x = rng.standard_normal(30000) * 10.0 ** rng.uniform(-9, 4.8, 30000)
    x = x[np.abs(x) < 65504]
    # include exact ties at several binades
    ties = np.array([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2.0 ** -25, 3 * 2.0 ** -25,
                     1024 + 0.5, 2048 + 1.0, -(1 + 2.0 ** -11)])
    x = np.concatenate([x, ties])
    ours = np.array([oracle_mod.f64_to_f16_bits(v) for v in x], dtype=np.uint16)
    assert np.array_equal(ours, x.astype(np.float16).view(np.uint16))
    back = np.array([oracle_mod.f16_bits_to_f64(h) for h in ours])
    assert np.array_equal(back, x.astype(np.float16).astype(np.float64))


def test_f16_saturates_beyond_range(oracle_mod):
    for v, bits in [(65504.0, 0x7BFF), (70000.0, 0x7BFF), (-1e9, 0xFBFF), (65519.9, 0x7BFF)]:
        assert oracle_mod.f64_to_f16_bits(v) == bits


def test_bf16_rounding_matches_torch(oracle_mod):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(30000) * 10.0 ** rng.uniform(-40, 30, 30000)).astype(np.float32)
    ours = np.array([oracle_mod.f32_to_bf16_bits(v) for v in x], dtype=np.uint16)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_golden_f16_examples(oracle_mod):
    g = json.load(open(GOLDEN))
    for v, bits in g["f16_round"][0]["cases"]:
        assert oracle_mod.f64_to_f16_bits(v) == bits, v


# ------------------------------------------------------------------ transform pair
@pytest.mark.parametrize("name", ["tiny", "long"])
def test_transform_pair_preserves_dot_products(oracle_mod, name):
    """Sparsity 0, quantization off: (T_Q q).(T_K k) equals q.k (fp64, 1e-10)."""
    w = I.CONFIGS[name].with_(hkv=2, hq=4 if name == "long" else 2)
    _, _, tk64, tq64 = I.transforms(w)
    rng = np.random.default_rng(5)
    L = 64
    k = rng.standard_normal((L, w.hkv, w.d))
    v = rng.standard_normal((L, w.hkv, w.d))
    q = rng.standard_normal((w.hq, w.d))
    _, scores = oracle_mod.decode_dense(tk64, tq64, k, v, q, pct=0, want_scores=True)
    G = w.hq // w.hkv
    for h in range(w.hq):
        direct = k[:, h // G, :] @ q[h] / math.sqrt(w.d)
        assert np.max(np.abs(scores[h] - direct)) <= 1e-10 * max(1.0, np.abs(direct).max())


def test_quant_off_is_textbook_attention(oracle_mod):
    w = I.CONFIGS["long"].with_(hkv=2, hq=8)
    _, _, tk64, tq64 = I.transforms(w)
    rng = np.random.default_rng(6)
    L = 300
    k = rng.standard_normal((L, 2, w.d)) * 2
    v = rng.standard_normal((L, 2, w.d))
    q = rng.standard_normal((8, w.d))
    out = oracle_mod.decode_dense(tk64, tq64, k, v, q, pct=0)
    for h in range(8):
        ref = textbook_attention(q[h:h + 1], k[:, h // 4], v[:, h // 4], 1 / math.sqrt(w.d))[0]
        assert np.max(np.abs(out[h] - ref)) <= 1e-10 * max(1.0, np.abs(ref).max())


def test_dense_ones_values_sum_to_one(oracle_mod):
    """Softmax rows sum to 1: with v = 1 everywhere the output is exactly 1."""
    rng = np.random.default_rng(7)
    d, L = 64, 500
    t = np.eye(d)
    k = rng.standard_normal((L, 1, d)) * 3
    q = rng.standard_normal((3, d))
    out = oracle_mod.decode_dense(t, t, k, np.ones((L, 1, d)), q, pct=40)
    assert np.max(np.abs(out - 1.0)) <= 1e-12


def test_transform_f32_contract(oracle_mod):
    """fp32 transform = fp64 sum of exact products rounded once; identity is exact."""
    rng = np.random.default_rng(8)
    d = 128
    t = rng.standard_normal((d, d)).astype(np.float32)
    x = rng.standard_normal(d).astype(np.float32)
    y = oracle_mod.transform_f32(t, x)
    ref = np.array([math.fsum(float(t[c, i]) * float(x[i]) for i in range(d)) for c in range(d)])
    # the sequential fp64 sum differs from the exact sum by far less than an fp32 ulp
    assert np.max(np.abs(y.astype(np.float64) - ref) / np.maximum(np.abs(ref), 1e-30)) < 2 ** -23
    assert np.array_equal(oracle_mod.transform_f32(np.eye(d, dtype=np.float32), x), x)


# ------------------------------------------------------------------ quantizer
def test_golden_quantizer_groups(oracle_mod):
    g = json.load(open(GOLDEN))
    for case in g["groups"]:
        x = np.array(case["x"] * 2, dtype=np.float32)     # d = 64: two identical groups
        codes, scale, mn, ch0 = oracle_mod.quantize_vec(x, case["protect_ch0"])
        assert list(codes[:32]) == case["codes"], case["name"]
        assert int(scale[0]) == case["scale_bits"] and int(mn[0]) == case["min_bits"], case["name"]
        if case["protect_ch0"]:
            assert ch0 == case["ch0_bits"]
            # group 1 holds channel 32 = x[0] (not protected) -> its range includes 100
            assert int(scale[1]) != case["scale_bits"]


def _f16(v):
    return np.float16(v)


def test_int2_grid_round_trip(oracle_mod):
    """Values already on an INT2 grid (fp16 min and power-of-two scale, codes 0
    and 3 both present) come back with the same codes, scale and min."""
    rng = np.random.default_rng(9)
    for trial in range(300):
        d = 128 if trial % 2 else 64
        ng = d // 32
        scale = 2.0 ** rng.integers(-6, 4, size=ng)
        mn = np.array([float(_f16(v)) for v in rng.standard_normal(ng) * 4])
        codes = rng.integers(0, 4, size=d).astype(np.uint8)
        protect = bool(trial % 3 == 0)
        for g in range(ng):
            lo = 32 * g + (1 if (g == 0 and protect) else 0)
            codes[lo], codes[lo + 1] = 0, 3
        x = (mn[np.arange(d) // 32] + codes * scale[np.arange(d) // 32]).astype(np.float32)
        assert np.array_equal(x.astype(np.float64), mn[np.arange(d) // 32] + codes * scale[np.arange(d) // 32])
        if protect:
            x[0] = np.float32(rng.standard_normal() * 50)
            codes[0] = 0
        c2, s2, m2, ch0 = oracle_mod.quantize_vec(x, protect)
        assert np.array_equal(c2, codes)
        assert np.array_equal(s2, scale.astype(np.float16).view(np.uint16))
        assert np.array_equal(m2, mn.astype(np.float16).view(np.uint16))
        if protect:
            assert ch0 == oracle_mod.f32_to_bf16_bits(x[0])


def test_quantizer_error_bound(oracle_mod):
    """|x - x^| <= scale/2 + |mn - min_h| + 1.5 ulp(scale) for every channel."""
    rng = np.random.default_rng(10)
    for trial in range(200):
        d = 128
        x = (rng.standard_t(3, size=d) * 10.0 ** rng.uniform(-2, 2)).astype(np.float32)
        codes, scale, mn, _ = oracle_mod.quantize_vec(x, False)
        for g in range(4):
            s = float(scale.view(np.float16)[g])
            m = float(mn.view(np.float16)[g])
            xs = x[32 * g:32 * g + 32].astype(np.float64)
            ulp = float(np.spacing(np.float16(s)))
            xh = m + codes[32 * g:32 * g + 32] * s
            bound = s / 2 + abs(xs.min() - m) + 1.5 * ulp + 1e-12 * np.abs(xs).max()
            assert np.all(np.abs(xs - xh) <= bound)
            assert codes.max() <= 3


def test_scale_zero_group(oracle_mod):
    x = np.full(64, -2.75, dtype=np.float32)
    codes, scale, mn, _ = oracle_mod.quantize_vec(x, False)
    assert not codes.any() and not scale.any()
    assert np.all(mn.view(np.float16) == np.float16(-2.75))


# ------------------------------------------------------------------ selection
def test_golden_selection_and_n_keep(oracle_mod):
    g = json.load(open(GOLDEN))
    for case in g["selection"]:
        q = np.array(case["q"])
        assert list(oracle_mod.select(np.abs(q), case["keep"])) == case["sel"], case["why"]
    for d, pct, keep in g["n_keep"][0]["cases"]:
        assert oracle_mod.n_keep(d, pct) == keep


def _brute_select(absq, keep):
    order = sorted(range(1, len(absq)), key=lambda c: (-absq[c], c))
    return sorted([0] + order[:keep - 1])


def test_selection_matches_exhaustive_sort(oracle_mod):
    rng = np.random.default_rng(11)
    for trial in range(3000):
        d = [64, 128, 37][trial % 3]
        kind = trial % 5
        if kind == 0:
            a = np.abs(rng.standard_normal(d))
        elif kind == 1:
            a = np.abs(rng.integers(-3, 4, size=d)).astype(np.float64)     # many ties
        elif kind == 2:
            a = np.zeros(d)                                               # all equal
        elif kind == 3:
            a = np.abs(np.float32(rng.standard_normal(d)).astype(np.float16)).astype(np.float64)
        else:
            a = np.abs(np.where(rng.random(d) < 0.5, 0.0, -0.0))          # +-0
        keep = int(rng.integers(1, d + 1))
        assert list(oracle_mod.select(a, keep)) == _brute_select(list(a), keep)


def test_qprep_selection_uses_fp32_magnitudes(oracle_mod):
    rng = np.random.default_rng(12)
    d = 128
    t = rng.standard_normal((d, d)).astype(np.float32) * 0.1 + np.eye(d, dtype=np.float32)
    for _ in range(20):
        q = rng.standard_normal(d).astype(np.float32)
        qp, sel = oracle_mod.qprep(t, q, 40)
        assert np.array_equal(qp, oracle_mod.transform_f32(t, q))
        assert list(sel) == _brute_select(list(np.abs(qp.astype(np.float64))), 77)


# ------------------------------------------------------------------ quantized decode
def _small_seq(oracle_mod, L=200, hkv=2, hq=8, d=128, seed=13, v_ch0=False, identity=False):
    rng = np.random.default_rng(seed)
    if identity:
        t_k = np.tile(np.eye(d, dtype=np.float32), (hkv, 1, 1))
    else:
        t_k = (np.eye(d) + 0.05 * rng.standard_normal((hkv, d, d))).astype(np.float32)
    t_q = np.stack([np.linalg.inv(t.astype(np.float64)).T for t in t_k]).astype(np.float32)
    k = rng.standard_normal((L, hkv, d)).astype(np.float32) * 2
    v = rng.standard_normal((L, hkv, d)).astype(np.float32)
    q = rng.standard_normal((hq, d)).astype(np.float32)
    cache = oracle_mod.append(t_k, k, v, v_ch0=v_ch0)
    return cache, q, t_k, t_q


@pytest.mark.parametrize("v_ch0", [False, True])
def test_quantized_decode_is_attention_over_dequantized_cache(oracle_mod, v_ch0):
    """With T_K = I and sparsity 0 the decode is plain softmax attention over the
    dequantized rows (dequantized here, in numpy, from the stored fields)."""
    cache, q, t_k, t_q = _small_seq(oracle_mod, identity=True, v_ch0=v_ch0)
    out, sel, qp = oracle_mod.decode_seq(cache, q, t_q, hq=8, pct=0, v_ch0=v_ch0)
    kh, vh = oracle_mod.dequant(cache, v_ch0=v_ch0)
    for h in range(8):
        ref = textbook_attention(qp[h:h + 1].astype(np.float64), kh[:, h // 4], vh[:, h // 4],
                                 1 / math.sqrt(128))[0]
        assert np.max(np.abs(out[h] - ref)) <= 1e-12
    assert np.array_equal(qp, q)            # T_Q = I^T = I exactly


def test_pruned_decode_matches_masked_attention(oracle_mod):
    """At 40 % sparsity the scores use only the selected channels."""
    cache, q, t_k, t_q = _small_seq(oracle_mod, seed=14)
    out, sel, qp = oracle_mod.decode_seq(cache, q, t_q, hq=8, pct=40)
    kh, vh = oracle_mod.dequant(cache)
    for h in range(8):
        qm = np.zeros(128)
        qm[sel[h]] = qp[h, sel[h]]
        ref = textbook_attention(qm[None], kh[:, h // 4], vh[:, h // 4], 1 / math.sqrt(128))[0]
        assert np.max(np.abs(out[h] - ref)) <= 1e-12
        assert list(sel[h]) == _brute_select(list(np.abs(qp[h].astype(np.float64))), 77)


def test_single_token_returns_its_value(oracle_mod):
    cache, q, t_k, t_q = _small_seq(oracle_mod, L=1, seed=15)
    out, _, _ = oracle_mod.decode_seq(cache, q, t_q, hq=8, pct=40)
    _, vh = oracle_mod.dequant(cache)
    for h in range(8):
        assert np.array_equal(out[h], vh[0, h // 4])


def test_zero_query_averages_values(oracle_mod):
    cache, q, t_k, t_q = _small_seq(oracle_mod, L=77, seed=16)
    out, _, _ = oracle_mod.decode_seq(cache, np.zeros_like(q), t_q, hq=8, pct=40)
    _, vh = oracle_mod.dequant(cache)
    for h in range(8):
        assert np.max(np.abs(out[h] - vh[:, h // 4].mean(axis=0))) <= 1e-12


def test_gqa_equals_separate_mha_runs(oracle_mod):
    """G = 4 query heads over one kv head == four single-head runs."""
    cache, q, t_k, t_q = _small_seq(oracle_mod, hkv=1, hq=4, seed=17)
    out, sel, _ = oracle_mod.decode_seq(cache, q, t_q, hq=4, pct=40)
    for h in range(4):
        o1, s1, _ = oracle_mod.decode_seq(cache, q[h:h + 1], t_q, hq=1, pct=40)
        assert np.array_equal(o1[0], out[h]) and np.array_equal(s1[0], sel[h])


def test_thread_count_does_not_change_results(oracle_mod):
    cache, q, t_k, t_q = _small_seq(oracle_mod, hkv=2, hq=8, seed=18)
    a = oracle_mod.decode_seq(cache, q, t_q, hq=8, pct=40, threads=1)
    b = oracle_mod.decode_seq(cache, q, t_q, hq=8, pct=40, threads=8)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_append_is_per_row_transform_then_quantize(oracle_mod):
    rng = np.random.default_rng(19)
    d, hkv = 64, 2
    t_k = rng.standard_normal((hkv, d, d)).astype(np.float32) * 0.2
    k = rng.standard_normal((5, hkv, d)).astype(np.float32)
    v = rng.standard_normal((5, hkv, d)).astype(np.float32)
    c = oracle_mod.append(t_k, k, v)
    for t in range(5):
        for j in range(hkv):
            kp = oracle_mod.transform_f32(t_k[j], k[t, j])
            codes, s, m, ch0 = oracle_mod.quantize_vec(kp, True)
            assert np.array_equal(c["kcodes"][t, j], codes) and c["kch0"][t, j] == ch0
            codes, s, m, _ = oracle_mod.quantize_vec(v[t, j], False)
            assert np.array_equal(c["vcodes"][t, j], codes) and np.array_equal(c["vscale"][t, j], s)


# ------------------------------------------------- one (scale, min) group per token
def test_one_group_grid_round_trip(oracle_mod):
    """group_size = d: values on one INT2 grid over the whole row (channel 0
    protected or not) come back with the same codes, scale and min."""
    rng = np.random.default_rng(21)
    for trial in range(200):
        d = 128 if trial % 2 else 64
        scale = 2.0 ** int(rng.integers(-6, 4))
        mn = float(_f16(rng.standard_normal() * 4))
        codes = rng.integers(0, 4, size=d).astype(np.uint8)
        protect = bool(trial % 3 == 0)
        codes[1], codes[2] = 0, 3
        x = (mn + codes * scale).astype(np.float32)
        if protect:
            x[0] = np.float32(rng.standard_normal() * 50)
            codes[0] = 0
        c2, s2, m2, ch0 = oracle_mod.quantize_vec(x, protect, gs=d)
        assert s2.shape == (1,) and m2.shape == (1,)
        assert np.array_equal(c2, codes)
        assert s2[0] == np.float16(scale).view(np.uint16) and m2[0] == np.float16(mn).view(np.uint16)


def test_one_group_equals_per_group_when_ranges_agree(oracle_mod):
    """When every 32-channel group spans the same [min, max], the per-group and
    the per-token quantizers must give the same codes, scales and mins."""
    rng = np.random.default_rng(22)
    for trial in range(100):
        d = 128
        x = rng.uniform(-1.0, 1.0, size=d).astype(np.float32)
        lo, hi = np.float32(-1.5), np.float32(2.25)
        for g in range(4):
            x[32 * g + 3], x[32 * g + 17] = lo, hi
        protect = bool(trial % 2)
        c32, s32, m32, ch32 = oracle_mod.quantize_vec(x, protect)
        c1, s1, m1, ch1 = oracle_mod.quantize_vec(x, protect, gs=d)
        assert np.array_equal(c32, c1) and ch32 == ch1
        assert np.all(s32 == s1[0]) and np.all(m32 == m1[0])


def test_one_group_decode_is_attention_over_dequantized_cache(oracle_mod):
    rng = np.random.default_rng(23)
    L, hkv, d = 40, 2, 128
    k = rng.standard_normal((L, hkv, d)).astype(np.float32)
    v = rng.standard_normal((L, hkv, d)).astype(np.float32)
    eye = np.broadcast_to(np.eye(d, dtype=np.float32), (hkv, d, d)).copy()
    cache = oracle_mod.append(eye, k, v, gs=d)
    assert cache["kscale"].shape == (L, hkv, 1)
    q = rng.standard_normal((4, d)).astype(np.float32)
    out, sel, qp = oracle_mod.decode_seq(cache, q, eye, hq=4, pct=0)
    kh, vh = oracle_mod.dequant(cache)
    for h in range(4):
        ref = textbook_attention(qp[h:h + 1].astype(np.float64), kh[:, h // 2], vh[:, h // 2], 1 / math.sqrt(d))[0]
        assert np.max(np.abs(out[h] - ref)) <= 1e-12
