"""Pins of the float64 oracle: each check compares the oracle with something
other than itself (a value a page prints, a closed form, an invariant, a
library routine the definition reduces to, or pure-Python brute force).

Each ``check_*`` raises AssertionError on a mismatch.  ``test_oracle_pins.py``
runs them against the oracle; ``test_oracle_mutations.py`` plants plausible
mistakes in the oracle and shows that some check catches each one.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F
from torch.nn.attention.bias import causal_lower_right

from oracle import attention as orc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# ----------------------------------------------------------------------------
# the dot-product path reduces to a library routine: torch SDPA in float64
# ----------------------------------------------------------------------------

def check_dot_matches_sdpa(seed=0):
    rng = np.random.default_rng(seed)
    cases = [
        # N, Hq, H, L, S, E, Ev, mask
        (2, 4, 4, 9, 9, 8, 6, "none"),
        (1, 4, 2, 7, 13, 8, 8, "causal"),      # L != S: bottom-right alignment
        (2, 6, 2, 11, 11, 16, 4, "causal"),    # GQA g = 3
        (1, 2, 1, 5, 12, 4, 4, "bias"),
    ]
    for N, Hq, H, L, S, E, Ev, mask in cases:
        q, k, v = _rand(rng, N, Hq, L, E), _rand(rng, N, H, S, E), _rand(rng, N, H, S, Ev)
        scale = 0.37
        bias = None
        kw = {}
        if mask == "causal":
            kw["attn_mask"] = causal_lower_right(L, S)
        elif mask == "bias":
            b = np.where(rng.random((L, S)) < 0.3, -np.inf, 0.0)
            b[:, -1] = 0.0  # keep each row non-empty
            bias = b
            kw["attn_mask"] = torch.from_numpy(b)
        ref = F.scaled_dot_product_attention(
            torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
            scale=scale, enable_gqa=(Hq != H), **kw).numpy()
        out, _ = orc.attention_forward(q, k, v, scale=scale, mode="dot",
                                       mask_kind="causal" if mask == "causal" else "none",
                                       bias=bias)
        err = np.max(np.abs(out - ref))
        assert err < 1e-12, (mask, err)


# ----------------------------------------------------------------------------
# brute force with pure-Python loops on tiny inputs (every mode, mask, sink)
# ----------------------------------------------------------------------------

def _brute_row(qi, i, K, V, L, scale, mode, sink, mask_kind, window, brow):
    S = len(K)
    ip = i + (S - L)
    zs, vs = [], []
    for j in range(S):
        if mask_kind == "causal" and j > ip:
            continue
        if mask_kind == "window" and not (0 <= ip - j < window):
            continue
        if mode == "dot":
            z = scale * math.fsum(a * b for a, b in zip(qi, K[j]))
        else:
            z = -scale * math.fsum((a - b) ** 2 for a, b in zip(qi, K[j])) \
                + scale * math.fsum(a * a for a in qi)
        if brow is not None:
            z += brow[j]
        if z == -math.inf:
            continue
        zs.append(z)
        vs.append(V[j])
    cands = zs + ([sink] if sink is not None else [])
    if not cands:
        return [0.0] * len(V[0]), -math.inf
    M = max(cands)
    ws = [math.exp(z - M) for z in zs]
    D = math.fsum(ws) + (math.exp(sink - M) if sink is not None else 0.0)
    out = [math.fsum(w * vj[d] for w, vj in zip(ws, vs)) / D for d in range(len(V[0]))]
    return out, M + math.log(D)


def check_brute_force(seed=1):
    rng = np.random.default_rng(seed)
    for mode in ("dot", "rbf"):
        for mask_kind, window in (("none", 0), ("causal", 0), ("window", 2), ("window", 1)):
            for sink in (None, 0.3, -2.0):
                for L, S in ((4, 4), (2, 5), (5, 3)):
                    E, Ev = 3, 2
                    q, k, v = _rand(rng, 1, 2, L, E), _rand(rng, 1, 1, S, E), _rand(rng, 1, 1, S, Ev)
                    bias = np.where(rng.random((L, S)) < 0.2, -np.inf, 0.0)
                    sk = None if sink is None else np.array([sink, sink + 0.5])
                    out, lse = orc.attention_forward(q, k, v, scale=0.6, mode=mode, sink=sk,
                                                     mask_kind=mask_kind, window=window, bias=bias)
                    for hq in range(2):
                        s = None if sk is None else float(sk[hq])
                        for i in range(L):
                            bo, bl = _brute_row(list(q[0, hq, i]), i, k[0, 0].tolist(), v[0, 0].tolist(),
                                                L, 0.6, mode, s, mask_kind, window, bias[i].tolist())
                            assert np.allclose(out[0, hq, i], bo, rtol=0, atol=1e-12), (mode, mask_kind, sink)
                            if bl == -math.inf:
                                assert lse[0, hq, i] == -np.inf
                            else:
                                assert abs(lse[0, hq, i] - bl) < 1e-12, (mode, mask_kind, sink)


# ----------------------------------------------------------------------------
# RBF: the expansion identity, and the two temperature limits
# ----------------------------------------------------------------------------

def check_rbf_expansion(seed=2):
    """Direct -scale*||q-k||^2 (+ scale*||q||^2 frame) equals the expanded
    2*scale*q.k - scale*||k||^2 (the expansion -||q||^2 - ||k||^2 + 2 q.k with
    the query norm dropped by shift invariance)."""
    rng = np.random.default_rng(seed)
    q, k = _rand(rng, 7, 16) * 3, _rand(rng, 11, 16) * 2
    scale = 0.125
    z = orc.logits(q, k, scale, "rbf")
    expanded = scale * (2.0 * np.einsum("re,se->rs", q, k) - np.einsum("se,se->s", k, k)[None, :])
    rel = np.max(np.abs(z - expanded)) / np.max(np.abs(expanded))
    assert rel < 1e-12, rel


def check_rbf_limits(seed=3):
    rng = np.random.default_rng(seed)
    L, S, E, Ev = 6, 9, 5, 4
    q, k, v = _rand(rng, 1, 1, L, E), _rand(rng, 1, 1, S, E), _rand(rng, 1, 1, S, Ev)
    for mask_kind in ("none", "causal"):
        vis = orc.visible(np.arange(L), S, L, mask_kind)
        # scale -> 0: uniform over visible keys -> mean of visible value rows
        out, _ = orc.attention_forward(q, k, v, scale=1e-13, mode="rbf", mask_kind=mask_kind)
        for i in range(L):
            mean = v[0, 0][vis[i]].mean(axis=0)
            assert np.allclose(out[0, 0, i], mean, atol=1e-9)
        # scale -> inf: one-hot on the nearest visible key (brute-force argmin)
        out, _ = orc.attention_forward(q, k, v, scale=1e4, mode="rbf", mask_kind=mask_kind)
        for i in range(L):
            best, bj = math.inf, -1
            for j in range(S):
                if not vis[i, j]:
                    continue
                d = sum((a - b) ** 2 for a, b in zip(q[0, 0, i], k[0, 0, j]))
                if d < best:
                    best, bj = d, j
            assert np.allclose(out[0, 0, i], v[0, 0, bj], atol=1e-9)


def check_dot_limits(seed=4):
    """scale -> 0: weights uniform over visible keys, lse = ln(n_vis) (ln(n_vis + e^s) with a sink)."""
    rng = np.random.default_rng(seed)
    L, S, E, Ev = 5, 8, 4, 3
    q, k, v = _rand(rng, 1, 1, L, E), _rand(rng, 1, 1, S, E), _rand(rng, 1, 1, S, Ev)
    for sink in (None, 0.7):
        sk = None if sink is None else np.array([sink])
        out, lse = orc.attention_forward(q, k, v, scale=1e-15, mode="dot", mask_kind="causal", sink=sk)
        for i in range(L):
            nvis = i + (S - L) + 1
            extra = 0.0 if sink is None else math.exp(sink)
            assert abs(lse[0, 0, i] - math.log(nvis + extra)) < 1e-12
            mean = v[0, 0, :nvis].mean(axis=0) * nvis / (nvis + extra)
            assert np.allclose(out[0, 0, i], mean, atol=1e-12)


def check_uniform_entropy_golden():
    """Golden: n = 24 tokens, temperature -> inf: mean row entropy ln 24 = 3.178."""
    g = _golden("uniform_entropy_n24.json")
    n = g["n"]
    rng = np.random.default_rng(5)
    x = _rand(rng, n, 2)
    rows = np.arange(n)
    _, _, alpha, _ = orc.attend_rows(x, rows, x, x, n, scale=1e-12, mode="dot", return_weights=True)
    ent = float(np.mean(-np.sum(alpha * np.log(alpha), axis=1)))
    assert round(ent, g["decimals"]) == g["entropy"], ent


# ----------------------------------------------------------------------------
# sink
# ----------------------------------------------------------------------------

def check_sink_limit(seed=6):
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, 1, 2, 6, 4), _rand(rng, 1, 1, 6, 4), _rand(rng, 1, 1, 6, 3)
    for mode in ("dot", "rbf"):
        ref, rl = orc.attention_forward(q, k, v, scale=0.5, mode=mode, mask_kind="causal")
        for s in (-np.inf, -1e30):
            out, lse = orc.attention_forward(q, k, v, scale=0.5, mode=mode, mask_kind="causal",
                                             sink=np.array([s, s]))
            assert np.array_equal(out, ref) and np.array_equal(lse, rl), (mode, s)


def check_sink_mass(seed=7):
    """Weights sum to 1 - p_sink, p_sink = e^{s - lse}; out = (1 - p_sink) * out_without_sink."""
    rng = np.random.default_rng(seed)
    L, S = 5, 7
    q, k, v = _rand(rng, L, 4), _rand(rng, S, 4), _rand(rng, S, 3)
    rows = np.arange(L)
    for mode in ("dot", "rbf"):
        for s in (-1.0, 0.0, 2.5):
            out, lse, alpha, ps = orc.attend_rows(q, rows, k, v, L, scale=0.4, mode=mode, sink=s,
                                                  mask_kind="causal", return_weights=True)
            base, _ = orc.attend_rows(q, rows, k, v, L, scale=0.4, mode=mode, mask_kind="causal")
            assert np.all(alpha >= 0)
            assert np.allclose(alpha.sum(axis=1), 1.0 - ps, atol=1e-14)
            assert np.allclose(ps, np.exp(s - lse), atol=1e-14)
            assert np.allclose(out, (1.0 - ps)[:, None] * base, atol=1e-13)


def check_zero_sink_equivalence(seed=8):
    """R zero K/V rows prepended (and visible to every query) equal no registers
    plus a sink logit ln R: a zero key has logit exactly 0 in both score modes,
    i.e. adding e^0 = 1 to the denominator per register (page 'Attention Sink'
    §3.3 zero sink; register tokens of the RBF page)."""
    rng = np.random.default_rng(seed)
    L, E, Ev = 6, 5, 4
    for R in (1, 4):
        for mode in ("dot", "rbf"):
            for mask_kind in ("none", "causal"):
                q = _rand(rng, 1, 2, L, E)
                k, v = _rand(rng, 1, 1, L, E), _rand(rng, 1, 1, L, Ev)
                kr = np.concatenate([np.zeros((1, 1, R, E)), k], axis=2)
                vr = np.concatenate([np.zeros((1, 1, R, Ev)), v], axis=2)
                with_regs, _ = orc.attention_forward(q, kr, vr, scale=0.3, mode=mode, mask_kind=mask_kind)
                sinked, _ = orc.attention_forward(q, k, v, scale=0.3, mode=mode, mask_kind=mask_kind,
                                                  sink=np.full(2, math.log(R)))
                assert np.allclose(with_regs, sinked, atol=1e-13), (R, mode, mask_kind)


# ----------------------------------------------------------------------------
# convexity, masks, structure
# ----------------------------------------------------------------------------

def check_convexity(seed=9):
    rng = np.random.default_rng(seed)
    L, S = 8, 8
    q, k, v = _rand(rng, L, 6) * 2, _rand(rng, S, 6), _rand(rng, S, 5)
    rows = np.arange(L)
    for mode in ("dot", "rbf"):
        for mask_kind, w in (("none", 0), ("causal", 0), ("window", 3)):
            out, _, alpha, _ = orc.attend_rows(q, rows, k, v, L, scale=0.9, mode=mode,
                                               mask_kind=mask_kind, window=w, return_weights=True)
            vis = orc.visible(rows, S, L, mask_kind, w)
            assert np.all(alpha >= 0) and np.all(alpha[~vis] == 0)
            assert np.allclose(alpha.sum(axis=1), 1.0, atol=1e-14)
            for i in range(L):
                vv = v[vis[i]]
                assert np.all(out[i] >= vv.min(axis=0) - 1e-14)
                assert np.all(out[i] <= vv.max(axis=0) + 1e-14)


def check_causal_alignment_golden():
    g = _golden("causal_alignment_L1_S6.json")
    L, S = g["L"], g["S"]
    br = orc.visible(np.array([0]), S, L, "causal")[0]
    assert br.tolist() == g["bottom_right_row"]
    # the top-left alignment is the same rule with the offset S - L taken as 0
    tl = orc.visible(np.array([0]), S, S, "causal")[0]
    assert tl.tolist() == g["top_left_row"]
    assert causal_lower_right(L, S)._materialize().tolist()[0] == g["bottom_right_row"]


def check_fully_masked_rows(seed=10):
    """A row whose keys are all masked gives out = 0 (as SDPA returns), lse = -inf;
    with a sink, out = 0 and lse = s."""
    rng = np.random.default_rng(seed)
    L, S = 4, 5
    q, k, v = _rand(rng, 1, 1, L, 3), _rand(rng, 1, 1, S, 3), _rand(rng, 1, 1, S, 2)
    bias = np.zeros((L, S))
    bias[2, :] = -np.inf
    out, lse = orc.attention_forward(q, k, v, scale=0.5, bias=bias)
    ref = F.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
                                         attn_mask=torch.from_numpy(bias), scale=0.5).numpy()
    assert np.all(out[0, 0, 2] == 0.0) and lse[0, 0, 2] == -np.inf
    assert np.max(np.abs(out - ref)) < 1e-12
    out, lse = orc.attention_forward(q, k, v, scale=0.5, bias=bias, sink=np.array([0.25]))
    assert np.all(out[0, 0, 2] == 0.0) and lse[0, 0, 2] == 0.25
    # L > S with causal: rows i < L - S see no key
    q2 = _rand(rng, 1, 1, 6, 3)
    out, lse = orc.attention_forward(q2, k[:, :, :3], v[:, :, :3], scale=0.5, mask_kind="causal")
    assert np.all(out[0, 0, :3] == 0.0) and np.all(lse[0, 0, :3] == -np.inf)
    assert np.all(np.isfinite(lse[0, 0, 3:]))


def check_window_semantics(seed=11):
    rng = np.random.default_rng(seed)
    L, S = 7, 10
    q, k, v = _rand(rng, 1, 1, L, 4), _rand(rng, 1, 1, S, 4), _rand(rng, 1, 1, S, 3)
    # W = 1: each query sees only its own aligned key i' = i + S - L
    out, _ = orc.attention_forward(q, k, v, scale=0.8, mask_kind="window", window=1)
    for i in range(L):
        assert np.array_equal(out[0, 0, i], v[0, 0, i + S - L])
    # W >= S: identical to causal
    a, la = orc.attention_forward(q, k, v, scale=0.8, mask_kind="window", window=S)
    b, lb = orc.attention_forward(q, k, v, scale=0.8, mask_kind="causal")
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    # exactly min(W, i'+1) keys visible
    for W in (2, 3, 5):
        vis = orc.visible(np.arange(L), S, L, "window", W)
        for i in range(L):
            assert vis[i].sum() == min(W, i + S - L + 1)


def check_permutation_equivariance(seed=12):
    rng = np.random.default_rng(seed)
    L, S = 6, 9
    q, k, v = _rand(rng, 1, 1, L, 4), _rand(rng, 1, 1, S, 4), _rand(rng, 1, 1, S, 3)
    for mode in ("dot", "rbf"):
        base, bl = orc.attention_forward(q, k, v, scale=0.7, mode=mode)
        pk = rng.permutation(S)
        o, l_ = orc.attention_forward(q, k[:, :, pk], v[:, :, pk], scale=0.7, mode=mode)
        assert np.allclose(o, base, atol=1e-13) and np.allclose(l_, bl, atol=1e-13)
        pq = rng.permutation(L)
        o, l_ = orc.attention_forward(q[:, :, pq], k, v, scale=0.7, mode=mode)
        assert np.allclose(o, base[:, :, pq], atol=1e-13) and np.allclose(l_, bl[:, :, pq], atol=1e-13)


def check_gqa_repeat(seed=13):
    rng = np.random.default_rng(seed)
    N, Hq, H, L, S = 2, 6, 2, 5, 7
    q, k, v = _rand(rng, N, Hq, L, 4), _rand(rng, N, H, S, 4), _rand(rng, N, H, S, 3)
    sink = rng.standard_normal(Hq)
    for mode in ("dot", "rbf"):
        a, la = orc.attention_forward(q, k, v, scale=0.5, mode=mode, mask_kind="causal", sink=sink)
        kr, vr = np.repeat(k, Hq // H, axis=1), np.repeat(v, Hq // H, axis=1)
        b, lb = orc.attention_forward(q, kr, vr, scale=0.5, mode=mode, mask_kind="causal", sink=sink)
        assert np.array_equal(a, b) and np.array_equal(la, lb)


def check_magnitude_bullying(seed=20):
    """Page "Dot-Product Attention을 거리 기반 RBF-Attention으로 교체한 실험기", section
    details: under the dot product a key of large magnitude takes the softmax even
    when it is poorly aligned, and under RBF, which scores by Euclidean distance, a
    key's weight goes to zero as its magnitude grows.  One key (index 0) is put in a
    random direction u with norm g*sqrt(E) among 63 keys of lognormal size.  As g
    grows, its dot-product weight on the queries with q.u > 1 rises toward 1 and its
    RBF weight on every query falls toward 0; no query's RBF argmax is that key."""
    rng = np.random.default_rng(seed)
    E, S, L = 16, 64, 256
    q = _rand(rng, L, E)
    k = _rand(rng, S, E) * np.exp(0.5 * _rand(rng, S, 1))
    u = _rand(rng, E)
    u /= np.linalg.norm(u)
    v = _rand(rng, S, 4)
    rows = np.arange(L)
    aligned = q @ u > 1.0
    assert aligned.sum() >= 20
    dot_mass, rbf_max = [], []
    for g in (1.0, 2.0, 4.0, 8.0):
        kk = k.copy()
        kk[0] = g * math.sqrt(E) * u
        a_dot = orc.attend_rows(q, rows, kk, v, L, scale=0.25, mode="dot", return_weights=True)[2]
        a_rbf = orc.attend_rows(q, rows, kk, v, L, scale=0.25, mode="rbf", return_weights=True)[2]
        dot_mass.append(a_dot[aligned, 0].mean())
        rbf_max.append(a_rbf[:, 0].max())
        if g >= 4.0:
            assert not np.any(a_rbf.argmax(axis=1) == 0)
    assert all(a < b for a, b in zip(dot_mass, dot_mass[1:])), dot_mass
    assert all(a > b for a, b in zip(rbf_max, rbf_max[1:])), rbf_max
    assert dot_mass[-1] > 0.95 and rbf_max[-1] < 1e-15, (dot_mass, rbf_max)


def check_streaming_mask(seed=14):
    """StreamingLLM mask: keep = 0 is the sliding window, keep >= i'+1 is causal,
    the visible count is |{j < keep} u {i'-W < j <= i'}|, and a decode query over
    the whole cache equals plain attention over the compacted cache (the kept
    first tokens followed by the last W tokens)."""
    rng = np.random.default_rng(seed)
    L, S = 6, 20
    for W, keep in ((3, 0), (4, 2), (5, 7), (20, 1)):
        vis = orc.visible(np.arange(L), S, L, "streaming", W, keep)
        if keep == 0:
            assert np.array_equal(vis, orc.visible(np.arange(L), S, L, "window", W))
        for i in range(L):
            ip = i + S - L
            want = {j for j in range(S) if j <= ip and (j < keep or ip - j < W)}
            assert set(np.nonzero(vis[i])[0].tolist()) == want
    assert np.array_equal(orc.visible(np.arange(L), S, L, "streaming", 2, S),
                          orc.visible(np.arange(L), S, L, "causal"))
    for mode in ("dot", "rbf"):
        for W, keep in ((5, 3), (1, 4), (7, 0)):
            q = _rand(rng, 1, 2, 1, 4)
            k, v = _rand(rng, 1, 1, S, 4), _rand(rng, 1, 1, S, 3)
            sink = np.array([0.3, -0.7])
            full, lf = orc.attention_forward(q, k, v, scale=0.6, mode=mode, sink=sink, mask_kind="streaming",
                                             window=W, keep=keep)
            idx = list(range(keep)) + list(range(S - W, S))
            comp, lc = orc.attention_forward(q, k[:, :, idx], v[:, :, idx], scale=0.6, mode=mode, sink=sink)
            assert np.allclose(full, comp, atol=1e-13) and np.allclose(lf, lc, atol=1e-13), (mode, W, keep)


def check_index_set(seed=15):
    """Exact attention over a key list: the full list in order is the dense
    forward; a subset equals the dense forward with -inf added off the subset;
    list order does not matter; a key listed twice equals the dense forward with
    ln 2 added to its logit; entries outside [0, S) select nothing; one selected
    key gives its value row and its own logit as lse (closed form)."""
    rng = np.random.default_rng(seed)
    N, H, Hq, L, S, E, Ev = 2, 2, 4, 3, 40, 5, 4
    q, k, v = _rand(rng, N, Hq, L, E), _rand(rng, N, H, S, E), _rand(rng, N, H, S, Ev)
    sink = rng.standard_normal(Hq)
    bias = np.where(rng.random((L, S)) < 0.1, -np.inf, 0.0)
    scale = 0.45
    for mk, W in (("none", 0), ("causal", 0), ("window", 9)):
        full = np.broadcast_to(np.arange(S), (N, H, S))
        a = orc.attention_over_index_set(q, k, v, full, scale=scale, sink=sink, mask_kind=mk, window=W, bias=bias)
        b = orc.attention_forward(q, k, v, scale=scale, sink=sink, mask_kind=mk, window=W, bias=bias)
        assert np.allclose(a[0], b[0], atol=1e-13) and np.allclose(a[1], b[1], atol=1e-13), mk
        # subsets with the last cached keys included (visible to every row under the masks)
        idx = np.stack([np.stack([rng.permutation(S - 1)[:11] for _ in range(H)]) for _ in range(N)])
        idx[..., 0] = S - 1  # distinct from the rest, which come from 0..S-2
        dup = idx.copy()
        dup[..., 1] = dup[..., 0]  # key S-1 listed twice
        for lst, extra in ((idx, 0.0), (dup, math.log(2.0))):
            got_o, got_l = orc.attention_over_index_set(q, k, v, lst, scale=scale, sink=sink, mask_kind=mk,
                                                        window=W, bias=bias)
            for n in range(N):
                for hq in range(Hq):
                    kvh = hq // (Hq // H)
                    add = np.full(S, -np.inf)
                    add[np.unique(lst[n, kvh])] = 0.0
                    add[S - 1] += extra
                    brow = bias + add[None, :]
                    ref_o, ref_l = orc.attend_rows(q[n, hq], np.arange(L), k[n, kvh], v[n, kvh], L, scale=scale,
                                                   sink=float(sink[hq]), mask_kind=mk, window=W, bias_rows=brow)
                    assert np.allclose(got_o[n, hq], ref_o, atol=1e-13), (mk, n, hq, extra)
                    assert np.allclose(got_l[n, hq], ref_l, atol=1e-13), (mk, n, hq, extra)
        perm = idx[..., rng.permutation(idx.shape[-1])]
        p_o, p_l = orc.attention_over_index_set(q, k, v, perm, scale=scale, sink=sink, mask_kind=mk, window=W)
        i_o, i_l = orc.attention_over_index_set(q, k, v, idx, scale=scale, sink=sink, mask_kind=mk, window=W)
        assert np.allclose(p_o, i_o, atol=1e-13) and np.allclose(p_l, i_l, atol=1e-13)
    # entries outside [0, S) select nothing
    pad = np.concatenate([np.full((N, H, 3), -1), idx, np.full((N, H, 2), S), np.full((N, H, 1), S + 7)], axis=-1)
    a = orc.attention_over_index_set(q, k, v, pad, scale=scale, sink=sink)
    b = orc.attention_over_index_set(q, k, v, idx, scale=scale, sink=sink)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    none = np.full((N, H, 4), -3)
    o0, l0 = orc.attention_over_index_set(q, k, v, none, scale=scale)
    assert np.all(o0 == 0.0) and np.all(l0 == -np.inf)
    o1, l1 = orc.attention_over_index_set(q, k, v, none, scale=scale, sink=sink)
    assert np.all(o1 == 0.0) and np.allclose(l1, np.broadcast_to(sink[None, :, None], l1.shape))
    # one selected key: out = its value row, lse = its logit (closed form, no softmax code involved)
    one = np.full((N, H, 1), 17)
    o, l = orc.attention_over_index_set(q, k, v, one, scale=scale)
    for n in range(N):
        for hq in range(Hq):
            kvh = hq // (Hq // H)
            assert np.allclose(o[n, hq], np.broadcast_to(v[n, kvh, 17], (L, Ev)), atol=1e-15)
            z = scale * sum(q[n, hq, :, e] * k[n, kvh, 17, e] for e in range(E))
            assert np.allclose(l[n, hq], z, atol=1e-13)


def check_padding_and_keep_mask(seed=16):
    """Keep mask and key padding: a keep mask equals the 0/-inf bias; key ranges
    equal the keep mask built from them; a left-padded input with kv_start = pad
    gives the unpadded input's output on the real tokens (the page's left-padding
    check), whatever the padding holds; left-padded start rows under a causal mask
    see no key (out 0, lse -inf; with a sink lse = s); kv_end = m equals keys and
    values cut to m."""
    rng = np.random.default_rng(seed)
    N, H, Hq, E, Ev = 2, 2, 4, 6, 5
    sink = rng.standard_normal(Hq)
    # keep mask == additive 0/-inf bias
    L, S = 7, 23
    q, k, v = _rand(rng, N, Hq, L, E), _rand(rng, N, H, S, E), _rand(rng, N, H, S, Ev)
    keep = rng.random((L, S)) < 0.6
    for mk in ("none", "causal"):
        a = orc.attention_forward(q, k, v, scale=0.4, sink=sink, mask_kind=mk, mask_keep=keep)
        b = orc.attention_forward(q, k, v, scale=0.4, sink=sink, mask_kind=mk, bias=np.where(keep, 0.0, -np.inf))
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]), mk
    # key ranges == the keep mask of the same range (per batch)
    ks, ke = np.array([3, 0]), np.array([19, 11])
    r1 = orc.attention_forward(q, k, v, scale=0.4, sink=sink, kv_start=ks, kv_end=ke)
    for n in range(N):
        km = np.zeros((L, S), dtype=bool)
        km[:, ks[n]:ke[n]] = True
        r2 = orc.attention_forward(q[n:n + 1], k[n:n + 1], v[n:n + 1], scale=0.4, sink=sink, mask_keep=km)
        assert np.array_equal(r1[0][n:n + 1], r2[0]) and np.array_equal(r1[1][n:n + 1], r2[1])
    # left padding: the real tokens' outputs do not depend on the padding
    L0, P = 9, 5
    q0, k0, v0 = _rand(rng, N, Hq, L0, E), _rand(rng, N, H, L0, E), _rand(rng, N, H, L0, Ev)
    pad = lambda x: np.concatenate([100.0 * _rand(rng, *x.shape[:2], P, x.shape[3]), x], axis=2)  # noqa: E731
    qp, kp, vp = pad(q0), pad(k0), pad(v0)
    for mk in ("none", "causal"):
        ref = orc.attention_forward(q0, k0, v0, scale=0.4, sink=sink, mask_kind=mk)
        got = orc.attention_forward(qp, kp, vp, scale=0.4, sink=sink, mask_kind=mk, kv_start=np.full(N, P))
        assert np.allclose(got[0][:, :, P:], ref[0], atol=1e-13) and np.allclose(got[1][:, :, P:], ref[1], atol=1e-13)
        if mk == "causal":
            # start rows see only padding
            nos = orc.attention_forward(qp, kp, vp, scale=0.4, mask_kind=mk, kv_start=np.full(N, P))
            assert np.all(nos[0][:, :, :P] == 0.0) and np.all(nos[1][:, :, :P] == -np.inf)
            assert np.all(got[0][:, :, :P] == 0.0)
            assert np.allclose(got[1][:, :, :P], np.broadcast_to(sink[None, :, None], (N, Hq, P)))
    # right padding: kv_end = m equals cutting K and V to m keys (no position-dependent mask)
    m = 15
    cut = orc.attention_forward(q, k[:, :, :m], v[:, :, :m], scale=0.4, sink=sink)
    end = orc.attention_forward(q, k, v, scale=0.4, sink=sink, kv_end=np.full(N, m))
    assert np.allclose(end[0], cut[0], atol=1e-13) and np.allclose(end[1], cut[1], atol=1e-13)


def check_backward_finite_differences(seed=17):
    """Every gradient of attention_backward against central differences of the
    forward (loss = sum(out * W)), for both score modes, three mask kinds, with
    and without a sink, under GQA: the differences involve none of the backward's
    formulas."""
    rng = np.random.default_rng(seed)
    N, Hq, H, L, S, E, Ev = 2, 2, 1, 4, 6, 3, 2
    h = 1e-6
    for mode in ("dot", "rbf"):
        for mk, W in (("none", 0), ("causal", 0), ("window", 3)):
            for with_sink in (False, True):
                q, k, v = _rand(rng, N, Hq, L, E), _rand(rng, N, H, S, E), _rand(rng, N, H, S, Ev)
                Wt = _rand(rng, N, Hq, L, Ev)
                sink = rng.standard_normal(Hq) if with_sink else None
                kw = dict(scale=0.7, mode=mode, mask_kind=mk, window=W)

                def loss(q_, k_, v_, s_):
                    o, _ = orc.attention_forward(q_, k_, v_, sink=s_, **kw)
                    return float(np.sum(o * Wt))

                dq, dk, dv, ds = orc.attention_backward(q, k, v, Wt, sink=sink, **kw)
                for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
                    it = np.nditer(arr, flags=["multi_index"])
                    for _ in it:
                        idx = it.multi_index
                        a, b = arr.copy(), arr.copy()
                        a[idx] += h
                        b[idx] -= h
                        args_a = {"q": (a, k, v), "k": (q, a, v), "v": (q, k, a)}[name]
                        args_b = {"q": (b, k, v), "k": (q, b, v), "v": (q, k, b)}[name]
                        fd = (loss(*args_a, sink) - loss(*args_b, sink)) / (2 * h)
                        assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (mode, mk, with_sink, name, idx,
                                                                                 fd, grad[idx])
                if with_sink:
                    for hh in range(Hq):
                        sa, sb = sink.copy(), sink.copy()
                        sa[hh] += h
                        sb[hh] -= h
                        fd = (loss(q, k, v, sa) - loss(q, k, v, sb)) / (2 * h)
                        assert abs(fd - ds[hh]) <= 1e-6 * max(1.0, abs(fd)), (mode, mk, "sink", hh)
                else:
                    assert np.all(ds == 0.0)


def check_backward_finite_differences_masks(seed=19):
    """The gradients under the streaming mask, and under keep bits with key padding,
    against central differences of the forward with the same mask (GQA, a sink)."""
    rng = np.random.default_rng(seed)
    N, Hq, H, L, S, E, Ev = 2, 2, 1, 5, 8, 3, 2
    h = 1e-6
    keep_m = rng.random((L, S)) < 0.7
    cfgs = [dict(mask_kind="streaming", window=3, keep=2),
            dict(mask_kind="causal", mask_keep=keep_m, kv_start=np.array([1, 0]), kv_end=np.array([8, 6]))]
    for mode in ("dot", "rbf"):
        for cfg in cfgs:
            q, k, v = _rand(rng, N, Hq, L, E), _rand(rng, N, H, S, E), _rand(rng, N, H, S, Ev)
            Wt = _rand(rng, N, Hq, L, Ev)
            sink = rng.standard_normal(Hq)
            kw = dict(scale=0.6, mode=mode, **cfg)

            def loss(q_, k_, v_, s_):
                o, _ = orc.attention_forward(q_, k_, v_, sink=s_, **kw)
                return float(np.sum(o * Wt))

            dq, dk, dv, ds = orc.attention_backward(q, k, v, Wt, sink=sink, **kw)
            for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
                it = np.nditer(arr, flags=["multi_index"])
                for _ in it:
                    idx = it.multi_index
                    a, b = arr.copy(), arr.copy()
                    a[idx] += h
                    b[idx] -= h
                    args_a = {"q": (a, k, v), "k": (q, a, v), "v": (q, k, a)}[name]
                    args_b = {"q": (b, k, v), "k": (q, b, v), "v": (q, k, b)}[name]
                    fd = (loss(*args_a, sink) - loss(*args_b, sink)) / (2 * h)
                    assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (mode, cfg["mask_kind"], name, idx)
            for hh in range(Hq):
                sa, sb = sink.copy(), sink.copy()
                sa[hh] += h
                sb[hh] -= h
                fd = (loss(q, k, v, sa) - loss(q, k, v, sb)) / (2 * h)
                assert abs(fd - ds[hh]) <= 1e-6 * max(1.0, abs(fd)), (mode, cfg["mask_kind"], "sink")


def check_backward_matches_sdpa_autograd(seed=18):
    """Dot mode without a sink: the gradients equal PyTorch's SDPA autograd in
    float64 (no mask, bottom-right causal, and an additive 0/-inf bias)."""
    rng = np.random.default_rng(seed)
    N, H, L, S, E, Ev = 2, 3, 5, 9, 4, 6
    q, k, v = _rand(rng, N, H, L, E), _rand(rng, N, H, S, E), _rand(rng, N, H, S, Ev)
    dout = _rand(rng, N, H, L, Ev)
    bias = np.where(rng.random((L, S)) < 0.2, -np.inf, 0.0)
    bias[:, -1] = 0.0
    for mk, mask in (("none", None), ("causal", causal_lower_right(L, S)), ("bias", bias)):
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        am = torch.tensor(mask) if mk == "bias" else mask
        out = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=am, scale=0.5)
        out.backward(torch.tensor(dout))
        dq, dk, dv, _ = orc.attention_backward(q, k, v, dout, scale=0.5, mask_kind="causal" if mk == "causal" else "none",
                                               bias=bias if mk == "bias" else None)
        for got, want in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            assert np.allclose(got, want.numpy(), atol=1e-12), mk


ALL_CHECKS = [
    check_dot_matches_sdpa, check_brute_force, check_rbf_expansion, check_rbf_limits,
    check_dot_limits, check_uniform_entropy_golden, check_sink_limit, check_sink_mass,
    check_zero_sink_equivalence, check_convexity, check_causal_alignment_golden,
    check_fully_masked_rows, check_window_semantics, check_permutation_equivariance,
    check_gqa_repeat, check_magnitude_bullying, check_streaming_mask, check_index_set, check_padding_and_keep_mask,
    check_backward_finite_differences, check_backward_finite_differences_masks, check_backward_matches_sdpa_autograd,
]
