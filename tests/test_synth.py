"""The seeded input generators (CPU): distribution, determinism, slicing, rounding."""

import json
import math
import os

import numpy as np
import pytest
import torch

from synth import workloads as sw


def test_normal_moments():
    x = sw.normal_f64(sw.stream_key(123, 1), 0, 2_000_000)
    assert abs(x.mean()) < 0.004
    assert abs(x.var() - 1.0) < 0.005
    kurt = np.mean((x - x.mean()) ** 4) / x.var() ** 2
    assert abs(kurt - 3.0) < 0.05


def test_series_against_numpy():
    u = np.random.default_rng(0).random(200_000)
    u = np.where(u == 0, 0.5, u)
    rel = np.max(np.abs(sw._log_series(u) - np.log(u)) / np.abs(np.log(u)))
    assert rel < 2e-15
    c, s = sw._sincos_turn(u)
    assert np.max(np.abs(c - np.cos(2 * np.pi * u))) < 3e-15
    assert np.max(np.abs(s - np.sin(2 * np.pi * u))) < 3e-15


def test_counter_based_slicing():
    key = sw.stream_key(7, 2)
    whole = sw.normal_f64(key, 0, 1001)
    for a, n in ((0, 10), (1, 9), (500, 501), (999, 2)):
        assert np.array_equal(sw.normal_f64(key, a, n), whole[a:a + n])
    assert not np.array_equal(sw.normal_f64(sw.stream_key(7, 3), 0, 10), whole[:10])


def test_generate_matches_slices():
    r = sw.RECIPES["tiny_rbf_sink_causal_f32"]
    w = sw.generate(r)
    for t in ("q", "k", "v"):
        for h in range(r.H):
            assert np.array_equal(sw.as_f64(r, w[t][0, h]), sw.tensor_slice_f64(r, t, 0, h))
    assert w["sink"].tolist() == [0.0, 1.0]
    assert w["bias"] is None


def test_bf16_round_to_nearest_even():
    one = 1.0
    cases = {
        one: 0x3F80,
        one + 2.0 ** -8: 0x3F80,             # tie -> even (down)
        one + 3 * 2.0 ** -8: 0x3F82,         # tie -> even (up)
        one + 2.0 ** -8 + 2.0 ** -30: 0x3F81,  # just above the tie
        -2.5: 0xC020,
        0.0: 0x0000,
    }
    got = sw.bf16_round_bits(np.array(list(cases)))
    assert got.tolist() == list(cases.values())
    x = np.random.default_rng(1).standard_normal(100_000).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(sw.bf16_round_bits(x), ref)
    assert np.array_equal(sw.bf16_bits_to_f64(ref),
                          torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_logit_variance_golden(golden_dir):
    """Var(q.k) = d_k for iid N(0,1) entries; ~1 after scaling by 1/sqrt(d_k)."""
    with open(os.path.join(golden_dir, "logit_variance_dk512.json")) as f:
        g = json.load(f)
    d = g["d_k"]
    n = 4000
    q = sw.normal_f64(sw.stream_key(11, 1), 0, n * d).reshape(n, d)
    k = sw.normal_f64(sw.stream_key(11, 2), 0, n * d).reshape(n, d)
    dots = np.einsum("ne,ne->n", q, k)
    tol = 0.1  # ~4.5 standard errors of a 4000-sample variance
    assert abs(dots.var() / d - 1.0) < tol
    assert abs((dots / math.sqrt(d)).var() - 1.0) < tol
    assert abs(g["unscaled_variance"] / d - 1.0) < tol and abs(g["scaled_variance"] - 1.0) < tol


def test_bias_recipe():
    r = sw.Recipe("b", N=1, Hq=1, H=1, L=300, S=300, E=64, Ev=64, dtype="f32", mode="dot",
                  scale=1.0, mask_kind="none", bias="random10", seed=2)
    b = sw.bias_matrix(r)
    assert b.dtype == np.float32 and set(np.unique(b).tolist()) <= {0.0, -np.inf}
    assert np.all(np.diag(b) == 0.0)
    frac = np.mean(np.isinf(b))
    assert 0.09 < frac < 0.11


def test_register_workload_structure():
    r = sw.RECIPES["rbf_registers_4k_bf16"]
    k = sw.tensor_slice_f64(r, "k", 1, 5)
    v = sw.tensor_slice_f64(r, "v", 1, 5)
    assert np.all(k[: r.registers] == 0) and np.all(v[: r.registers] == 0)
    assert np.all(np.abs(k[r.registers:]).sum(axis=1) > 0)
    # lognormal key factors: log of key norms spreads well beyond a plain N(0,1) row
    norms = np.linalg.norm(k[r.registers:] - sw.sinusoidal_table(r.S - r.registers, r.E), axis=1)
    assert np.std(np.log(norms)) > 0.8


def test_recipe_table():
    names = list(sw.RECIPES)
    assert len(names) == 6
    for r in sw.RECIPES.values():
        assert r.Hq % r.H == 0 and r.E in (64, 128) and r.Ev in (64, 128)


def test_key_index_set_is_a_random_subset():
    """Each (n, KV head) list holds n_sel distinct positions in [0, S), not sorted,
    differs across heads, and repeats cyclically when n_sel > S."""
    import dataclasses
    base = sw.RECIPES["tiny_rbf_sink_causal_f32"]
    r = dataclasses.replace(base, N=2, H=3, Hq=3, S=500, n_sel=37)
    a, b = sw.key_index_set(r), sw.key_index_set(r)
    assert a.shape == (2, 3, 37) and a.dtype == np.int32 and np.array_equal(a, b)
    for n in range(2):
        for h in range(3):
            lst = a[n, h]
            assert len(set(lst.tolist())) == 37 and lst.min() >= 0 and lst.max() < 500
            assert not np.all(np.diff(lst) > 0)
    assert not np.array_equal(a[0, 0], a[0, 1])
    big = sw.key_index_set(dataclasses.replace(r, S=10, n_sel=25))
    assert np.array_equal(big[0, 0, :10], big[0, 0, 10:20])
    assert sorted(big[0, 0, :10].tolist()) == list(range(10))
    assert sw.key_index_set(base) is None


def test_pack_mask_bits_layout():
    """Bit j % 32 of word j // 32 of row i is keep[i, j]; bits past S are zero."""
    rng = np.random.default_rng(3)
    for L, S in ((3, 1), (4, 31), (2, 32), (5, 77), (1, 128)):
        keep = rng.random((L, S)) < 0.5
        w = sw.pack_mask_bits(keep)
        assert w.dtype == np.uint32 and w.shape == (L, (S + 31) // 32)
        for i in range(L):
            for j in range((S + 31) // 32 * 32):
                bit = (int(w[i, j // 32]) >> (j % 32)) & 1
                assert bit == (int(keep[i, j]) if j < S else 0), (L, S, i, j)


def test_keep_matrix_matches_random10_bias_and_padding_ranges():
    import dataclasses
    base = sw.RECIPES["tiny_rbf_sink_causal_f32"]
    r = dataclasses.replace(base, bias="random10", keep_mask="random10", L=50, S=70)
    keep, bias = sw.keep_matrix(r), sw.bias_matrix(r)
    assert np.array_equal(keep, bias == 0.0)
    p = dataclasses.replace(base, N=64, S=1000, pad_left=0.25, pad_right=0.1)
    ks, ke = sw.kv_ranges(p)
    assert ks.min() >= 0 and ks.max() < 250 and ke.min() > 900 and ke.max() <= 1000 and len(set(ks)) > 10
    assert sw.kv_ranges(base) == (None, None)


def test_mixed_bias_blocks():
    """The mixed bias: -inf where random10 puts it, finite values in [-2, 2) on the odd
    128 x 128 blocks, exact zeros elsewhere; the diagonal is never -inf."""
    r = sw.Recipe("mixed", N=1, Hq=1, H=1, L=300, S=520, E=64, Ev=64, dtype="bf16", mode="dot", scale=0.125,
                  mask_kind="none", bias="mixed", seed=9)
    b = sw.bias_matrix(r)
    import dataclasses
    base = sw.bias_matrix(dataclasses.replace(r, name="r10", bias="random10"))
    assert np.array_equal(np.isneginf(b), np.isneginf(base))
    odd = ((np.arange(r.L)[:, None] // 128) + (np.arange(r.S)[None, :] // 128)) % 2 == 1
    fin = np.isfinite(b)
    assert np.all(b[fin & ~odd] == 0.0)
    vals = b[fin & odd]
    assert vals.size > 0 and vals.min() >= -2.0 and vals.max() < 2.0 and np.count_nonzero(vals) == vals.size
    assert np.all(np.isfinite(np.diagonal(b)))
    assert np.array_equal(b, sw.bias_matrix(r))
