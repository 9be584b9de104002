"""Plant plausible mistakes in the oracle (on the CPU) and show a pin catches each."""

import numpy as np
import pytest

import oracle_pins as pins
from oracle import attention as orc

_real_logits = orc.logits
_real_visible = orc.visible
_real_softmax = orc.softmax_with_sink


def _rbf_direct_frame(q_rows, k, scale, mode, key_block=512):
    z = _real_logits(q_rows, k, scale, mode, key_block)
    if mode == "rbf":  # drop the +scale*||q||^2 frame term
        z = z - scale * np.einsum("re,re->r", q_rows, q_rows)[:, None]
    return z


def _rbf_sign_flip(q_rows, k, scale, mode, key_block=512):
    z = _real_logits(q_rows, k, scale, mode, key_block)
    if mode == "rbf":
        qn = scale * np.einsum("re,re->r", q_rows, q_rows)[:, None]
        z = -(z - qn) + qn
    return z


def _rbf_without_key_norm(q_rows, k, scale, mode, key_block=512):
    if mode == "rbf":  # the dot product's logit 2*scale*q.k with no -scale*||k||^2 penalty
        return 2.0 * scale * (np.asarray(q_rows) @ np.asarray(k).T)
    return _real_logits(q_rows, k, scale, mode, key_block)


def _dot_scale_dropped(q_rows, k, scale, mode, key_block=512):
    if mode == "dot":
        return q_rows @ k.T
    return _real_logits(q_rows, k, scale, mode, key_block)


def _top_left(rows, S, L, mask_kind, window=0, keep=0):
    return _real_visible(rows, S, S, mask_kind, window, keep)


def _window_off_by_one(rows, S, L, mask_kind, window=0, keep=0):
    if mask_kind in ("window", "streaming"):
        rows = np.asarray(rows)
        d = rows[:, None] + (S - L) - np.arange(S)[None, :]
        return (d >= 0) & ((d <= window) | (np.arange(S)[None, :] < keep))
    return _real_visible(rows, S, L, mask_kind, window, keep)


def _streaming_keep_ignored(rows, S, L, mask_kind, window=0, keep=0):
    if mask_kind == "streaming":
        return _real_visible(rows, S, L, "window", window)
    return _real_visible(rows, S, L, mask_kind, window, keep)


def _sink_in_values(z, vis, sink):
    alpha, ps, lse = _real_softmax(z, vis, sink)
    if sink is not None and alpha.shape[1]:
        alpha = alpha.copy()
        alpha[:, 0] += ps  # sink mass leaks into the first value row
    return alpha, ps, lse


def _lse_without_sink(z, vis, sink):
    alpha, ps, lse = _real_softmax(z, vis, sink)
    _, _, lse0 = _real_softmax(z, vis, None)
    return alpha, ps, lse0 if sink is not None else lse


_real_select = orc.select_keys
_real_visible_at = orc.visible_at


def _select_unique(sel, S):
    return np.unique(_real_select(sel, S))  # drops repeated listings


def _select_clipped(sel, S):
    return np.clip(np.asarray(sel, dtype=np.int64), 0, S - 1)  # clips padding instead of dropping it


def _visible_at_list_position(rows, positions, S, L, mask_kind, window=0):
    return _real_visible(rows, S, L, mask_kind, window)[:, np.arange(len(positions))]


def _select_ignored(sel, S):
    return np.arange(S)  # attends over the whole cache


_real_padded_visible = orc.padded_visible


def _padding_range_ignored(vis, keep_rows=None, kv_range=None):
    return _real_padded_visible(vis, keep_rows, None)


def _keep_mask_inverted(vis, keep_rows=None, kv_range=None):
    inv = None if keep_rows is None else ~np.asarray(keep_rows, dtype=bool)
    return _real_padded_visible(vis, inv, kv_range)


def _padding_end_inclusive(vis, keep_rows=None, kv_range=None):
    wide = None if kv_range is None else (kv_range[0], kv_range[1] + 1)
    return _real_padded_visible(vis, keep_rows, wide)


_real_score_grads = orc.score_input_grads


def _softmax_grad_no_D(P, dP, D):
    return P * dP  # drops the -D_i term


def _rbf_grad_without_norm_term(dS, q_rows, k, scale, mode):
    if mode == "rbf":
        return 2.0 * scale * dS @ k, 2.0 * scale * dS.T @ q_rows  # drops -k_j sum_i dS_ij
    return _real_score_grads(dS, q_rows, k, scale, mode)


def _dot_grad_unscaled(dS, q_rows, k, scale, mode):
    if mode == "dot":
        return dS @ k, dS.T @ q_rows
    return _real_score_grads(dS, q_rows, k, scale, mode)


def _sink_grad_sign(p_sink, D):
    return float(np.sum(p_sink * D))


MUTATIONS = [
    ("softmax_grad", _softmax_grad_no_D, pins.check_backward_finite_differences),
    ("softmax_grad", _softmax_grad_no_D, pins.check_backward_matches_sdpa_autograd),
    ("score_input_grads", _rbf_grad_without_norm_term, pins.check_backward_finite_differences),
    ("score_input_grads", _dot_grad_unscaled, pins.check_backward_matches_sdpa_autograd),
    ("sink_grad", _sink_grad_sign, pins.check_backward_finite_differences),
    ("padded_visible", _padding_range_ignored, pins.check_padding_and_keep_mask),
    ("padded_visible", _keep_mask_inverted, pins.check_padding_and_keep_mask),
    ("padded_visible", _padding_end_inclusive, pins.check_padding_and_keep_mask),
    ("select_keys", _select_unique, pins.check_index_set),
    ("select_keys", _select_clipped, pins.check_index_set),
    ("select_keys", _select_ignored, pins.check_index_set),
    ("visible_at", _visible_at_list_position, pins.check_index_set),
    ("logits", _rbf_direct_frame, pins.check_zero_sink_equivalence),
    ("logits", _rbf_direct_frame, pins.check_rbf_expansion),
    ("logits", _rbf_sign_flip, pins.check_rbf_limits),
    ("logits", _rbf_sign_flip, pins.check_magnitude_bullying),
    ("logits", _rbf_without_key_norm, pins.check_magnitude_bullying),
    ("logits", _dot_scale_dropped, pins.check_dot_matches_sdpa),
    ("visible", _top_left, pins.check_causal_alignment_golden),
    ("visible", _top_left, pins.check_dot_matches_sdpa),
    ("visible", _window_off_by_one, pins.check_window_semantics),
    ("visible", _window_off_by_one, pins.check_streaming_mask),
    ("visible", _streaming_keep_ignored, pins.check_streaming_mask),
    ("softmax_with_sink", _sink_in_values, pins.check_sink_mass),
    ("softmax_with_sink", _lse_without_sink, pins.check_brute_force),
]


@pytest.mark.parametrize("attr,bad,check", MUTATIONS,
                         ids=[f"{a}:{b.__name__}->{c.__name__}" for a, b, c in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, attr, bad, check):
    monkeypatch.setattr(orc, attr, bad)
    with pytest.raises(AssertionError):
        check()


def test_gqa_head_map_mistake_is_caught(monkeypatch):
    """Reading KV head hq % H instead of hq // (Hq/H) is caught by the SDPA pin."""
    real_forward = orc.attention_forward

    def forward_modulo(q, k, v, **kw):
        q = np.asarray(q)
        Hq, H = q.shape[1], k.shape[1]
        perm = [hq % H for hq in range(Hq)]
        # emulate the wrong map by handing each query head the KV head hq % H
        kk = np.asarray(k)[:, perm]
        vv = np.asarray(v)[:, perm]
        return real_forward(q, kk, vv, **kw)

    monkeypatch.setattr(orc, "attention_forward", forward_modulo)
    with pytest.raises(AssertionError):
        pins.check_dot_matches_sdpa()


@pytest.mark.parametrize("dropped", ["keep", "mask_keep", "kv_start", "kv_end"])
def test_backward_mask_argument_dropped_is_caught(monkeypatch, dropped):
    """A backward that ignores one of the streaming mask's kept keys, the keep bits or
    the key padding (while the forward honours it) is caught by the finite-difference
    pin of the masked gradients."""
    real_backward = orc.attention_backward

    def backward_without(*args, **kw):
        kw.pop(dropped, None)
        return real_backward(*args, **kw)

    monkeypatch.setattr(orc, "attention_backward", backward_without)
    with pytest.raises(AssertionError):
        pins.check_backward_finite_differences_masks()
