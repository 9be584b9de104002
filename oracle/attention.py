"""Float64 CPU oracle of the fused attention forward  out = softmax(z + B) V.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library and the library never calls it.

It is the plain definition, written out in float64 per (batch, query head),
in blocks of query rows so that memory stays bounded:

* Score (page "어텐션 메커니즘" §2; page "SDPA란 무엇인가" §1, the
  softmax(QK^T/sqrt(E) + B)V formula and its four steps):
    dot  z_ij = scale * <q_i, k_j>
    rbf  z_ij = -scale * ||q_i - k_j||^2 + scale * ||q_i||^2
  The RBF distance is computed directly, element by element (page
  "Dot-Product Attention을 거리 기반 RBF-Attention으로 교체한 실험기",
  섹션별 상세: distance attention, torch.cdist form).  The + scale*||q_i||^2
  term fixes the logit frame to the expanded form 2*scale*<q,k> -
  scale*||k||^2 that the same page derives by shift invariance; it cancels in
  any softmax without a sink and only matters when a sink logit competes.
* Mask (page "SDPA란 무엇인가" §1 bias B in {0, -inf}; §4 trap 3 causal
  alignment; page "어텐션 메커니즘" §5 causal mask, §6 sliding window):
  with the bottom-right alignment i' = i + (S - L),
    causal  key j visible iff j <= i'
    window  key j visible iff 0 <= i' - j < W   (W keys, self included)
  and an additive bias B[i, j] (0 or -inf) composes with either.
* StreamingLLM mask (page "Attention Sink" §3.2: keep the first tokens'
  KV plus a rolling window of recent tokens): with R kept initial tokens,
    streaming  key j visible iff j <= i'  and  (j < R  or  i' - j < W)
* Grouped-query attention (page "SDPA란 무엇인가" §5): query head hq reads
  KV head hq // (Hq // H).
* Sink (page "Attention Sink" §4.2, §5.2-5.4): a per-query-head logit s_h
  enters the softmax denominator and not the value sum.  With A the visible
  keys:  M = max(max_{j in A} z_j, s),  D = e^{s-M} + sum_{j in A} e^{z_j-M},
  out = sum_{j in A} e^{z_j-M} v_j / D,  lse = M + ln D.
* A row with no visible key and no sink gives out = 0 and lse = -inf (page
  "SDPA란 무엇인가" §4: SDPA returns 0 instead of NaN for a fully masked row).
* Boolean keep mask and key padding (page "SDPA란 무엇인가" §1: B is 0 or
  -inf; §4 trap 1: a boolean attn_mask marks with True the pairs that take
  part, the opposite of key_padding_mask; the left-padding check: with the
  mask passed, padded and unpadded inputs give the same output for the real
  tokens): key j is visible to row i only where keep[i, j] is True and, for
  batch n, kv_start[n] <= j < kv_end[n].  Both compose with every mask kind.
* Backward (page "Attention Sink" §4.2 and §5: the sinks and register tokens
  are learned parameters, so training needs gradients of q, k, v and the sink
  logit; page "Dot-Product Attention을 거리 기반 RBF-Attention으로 교체한
  실험기": the RBF model is trained): the chain rule through the definitions
  above, written out in ``attention_backward``.
* Exact attention over a selected key subset (page "기술 요약: SOCKET - 희소
  어텐션을 위한 SOft Collision Kernel EsTimator", 방법론, 핵심 메커니즘 step 4:
  the top-k keys are picked, then exact attention runs on that subset): the
  softmax and the value sum run over the listed keys of the KV head only, with
  the mask taken at each key's original position.  One list per (batch, KV
  head), shared by the group's query heads; entries outside [0, S) select
  nothing; a repeated entry counts once per listing.

Two readings are decisions that the pages leave open.  One is the window width
(W keys, self included).  The other is lse with a sink (ln of the full
denominator, sink term included).  For both, parity is unpinned beyond
internal consistency: the pins check only that each is applied the same way
everywhere (W = 1 keeps the own key, W >= S is causal, p_sink = e^(s - lse)).
"""

from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def visible(rows: np.ndarray, S: int, L: int, mask_kind: str, window: int = 0, keep: int = 0) -> np.ndarray:
    """Boolean (R, S) visibility of keys 0..S-1 for query positions ``rows``.

    Bottom-right alignment: query i sits at key position i' = i + (S - L).
    ``keep`` is the number of initial tokens the streaming mask keeps.
    """
    rows = np.asarray(rows, dtype=np.int64)
    ip = rows[:, None] + (S - L)
    j = np.arange(S, dtype=np.int64)[None, :]
    if mask_kind == "none":
        return np.ones((rows.size, S), dtype=bool)
    if mask_kind == "causal":
        return j <= ip
    if mask_kind == "window":
        if window < 1:
            raise ValueError("window must be >= 1")
        d = ip - j
        return (d >= 0) & (d < window)
    if mask_kind == "streaming":
        if window < 1 or keep < 0:
            raise ValueError("streaming mask needs window >= 1 and keep >= 0")
        d = ip - j
        return (d >= 0) & ((j < keep) | (d < window))
    raise ValueError(f"unknown mask kind {mask_kind!r}")


def logits(q_rows: np.ndarray, k: np.ndarray, scale: float, mode: str, key_block: int = 512) -> np.ndarray:
    """Unmasked logits z (R, S) in float64."""
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    if mode == "dot":
        return scale * (q_rows @ k.T)
    if mode == "rbf":
        R, S = q_rows.shape[0], k.shape[0]
        d2 = np.empty((R, S), dtype=np.float64)
        # direct squared distance, sum over e of (q_e - k_e)^2
        for j0 in range(0, S, key_block):
            diff = q_rows[:, None, :] - k[None, j0:j0 + key_block, :]
            d2[:, j0:j0 + key_block] = np.einsum("rse,rse->rs", diff, diff)
        qn = np.einsum("re,re->r", q_rows, q_rows)
        return -scale * d2 + scale * qn[:, None]
    raise ValueError(f"unknown mode {mode!r}")


def softmax_with_sink(z: np.ndarray, vis: np.ndarray, sink: float | None):
    """Weights alpha (R, S), sink probability (R,), lse (R,) from masked logits.

    ``z`` already carries the additive bias; ``vis`` marks keys the mask kind
    leaves visible.  Keys with z = -inf (from the bias) get weight 0.
    """
    zm = np.where(vis, z, NEG_INF)
    s = NEG_INF if sink is None else float(sink)
    M = np.maximum(np.max(zm, axis=1, initial=NEG_INF), s)
    finite = np.isfinite(M)
    Ms = np.where(finite, M, 0.0)
    e = np.where(np.isfinite(zm), np.exp(zm - Ms[:, None]), 0.0)
    es = np.exp(s - Ms) if np.isfinite(s) else np.zeros_like(Ms)
    D = es + e.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        alpha = np.where(finite[:, None], e / np.where(finite, D, 1.0)[:, None], 0.0)
        p_sink = np.where(finite, es / np.where(finite, D, 1.0), 0.0)
        lse = np.where(finite, Ms + np.log(np.where(finite, D, 1.0)), NEG_INF)
    return alpha, p_sink, lse


def padded_visible(vis: np.ndarray, keep_rows=None, kv_range=None) -> np.ndarray:
    """Narrow a visibility matrix (R, S) by a boolean keep matrix (R, S) and a key range (start, end)."""
    if keep_rows is not None:
        vis = vis & np.asarray(keep_rows, dtype=bool)
    if kv_range is not None:
        j = np.arange(vis.shape[1])[None, :]
        vis = vis & (j >= kv_range[0]) & (j < kv_range[1])
    return vis


def attend_rows(q_rows, rows, k, v, L, *, scale, mode="dot", sink=None, mask_kind="none",
                window=0, bias_rows=None, return_weights=False, keep=0, keep_rows=None, kv_range=None):
    """Attention of query rows ``q_rows`` (R, E) at positions ``rows`` against one KV head.

    k (S, E), v (S, Ev), bias_rows (R, S) or None, keep_rows (R, S) bool or
    None, kv_range (start, end) or None.  Returns out (R, Ev) and lse (R,)
    (and the weights and sink probability when asked).
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    S = k.shape[0]
    z = logits(q_rows, k, scale, mode)
    if bias_rows is not None:
        z = z + np.asarray(bias_rows, dtype=np.float64)
    vis = padded_visible(visible(rows, S, L, mask_kind, window, keep), keep_rows, kv_range)
    alpha, p_sink, lse = softmax_with_sink(z, vis, sink)
    out = alpha @ v
    if return_weights:
        return out, lse, alpha, p_sink
    return out, lse


def attention_forward(q, k, v, *, scale, mode="dot", sink=None, mask_kind="none", window=0,
                      bias=None, row_block=128, keep=0, mask_keep=None, kv_start=None, kv_end=None):
    """Whole forward: q (N,Hq,L,E), k (N,H,S,E), v (N,H,S,Ev) float64.

    sink: per-query-head logits (Hq,) or None.  bias: (L, S) or None.
    mask_keep: (L, S) bool or None.  kv_start, kv_end: (N,) ints or None
    (0 and S).  Returns out (N,Hq,L,Ev) and lse (N,Hq,L).
    """
    q = np.asarray(q, dtype=np.float64)
    N, Hq, L, _ = q.shape
    H = k.shape[1]
    if Hq % H:
        raise ValueError("Hq must be a multiple of H")
    g = Hq // H
    Ev = v.shape[3]
    out = np.zeros((N, Hq, L, Ev), dtype=np.float64)
    lse = np.zeros((N, Hq, L), dtype=np.float64)
    for n in range(N):
        for hq in range(Hq):
            kvh = hq // g
            s = None if sink is None else float(sink[hq])
            for i0 in range(0, L, row_block):
                rows = np.arange(i0, min(L, i0 + row_block))
                b = None if bias is None else np.asarray(bias)[rows]
                kr = None if mask_keep is None else np.asarray(mask_keep, dtype=bool)[rows]
                rng = None
                if kv_start is not None or kv_end is not None:
                    rng = (0 if kv_start is None else int(kv_start[n]),
                           k.shape[2] if kv_end is None else int(kv_end[n]))
                o, l = attend_rows(q[n, hq, rows], rows, k[n, kvh], v[n, kvh], L, scale=scale,
                                   mode=mode, sink=s, mask_kind=mask_kind, window=window,
                                   bias_rows=b, keep=keep, keep_rows=kr, kv_range=rng)
                out[n, hq, rows] = o
                lse[n, hq, rows] = l
    return out, lse


def select_keys(sel: np.ndarray, S: int) -> np.ndarray:
    """The entries of a key list that name a cached key (0 <= j < S), in list order."""
    sel = np.asarray(sel, dtype=np.int64)
    return sel[(sel >= 0) & (sel < S)]


def visible_at(rows, positions, S: int, L: int, mask_kind: str, window: int = 0) -> np.ndarray:
    """Visibility (R, len(positions)) of keys at the given original positions."""
    return visible(rows, S, L, mask_kind, window)[:, np.asarray(positions, dtype=np.int64)]


def attention_over_index_set(q, k, v, key_idx, *, scale, sink=None, mask_kind="none", window=0, bias=None):
    """Exact attention of every query row over the keys listed for its KV head.

    q (N,Hq,L,E), k (N,H,S,E), v (N,H,S,Ev), key_idx (N,H,K) integer key
    positions.  sink: (Hq,) or None; bias: (L, S) or None, read at the original
    positions.  Returns out (N,Hq,L,Ev) and lse (N,Hq,L).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, Hq, L, _ = q.shape
    H, S = k.shape[1], k.shape[2]
    if Hq % H:
        raise ValueError("Hq must be a multiple of H")
    g = Hq // H
    out = np.zeros((N, Hq, L, v.shape[3]), dtype=np.float64)
    lse = np.zeros((N, Hq, L), dtype=np.float64)
    rows = np.arange(L)
    for n in range(N):
        for hq in range(Hq):
            kvh = hq // g
            pos = select_keys(np.asarray(key_idx)[n, kvh], S)
            z = logits(q[n, hq], k[n, kvh][pos], scale, "dot")
            if bias is not None:
                z = z + np.asarray(bias, dtype=np.float64)[:, pos]
            vis = visible_at(rows, pos, S, L, mask_kind, window)
            alpha, _, l = softmax_with_sink(z, vis, None if sink is None else float(sink[hq]))
            out[n, hq] = alpha @ v[n, kvh][pos]
            lse[n, hq] = l
    return out, lse


def softmax_grad(P: np.ndarray, dP: np.ndarray, D: np.ndarray) -> np.ndarray:
    """dS_ij = P_ij (dP_ij - D_i): the gradient through the row softmax."""
    return P * (dP - D[:, None])


def score_input_grads(dS: np.ndarray, q_rows: np.ndarray, k: np.ndarray, scale: float, mode: str):
    """(dq, dk) of one head from the logit gradients dS (R, S)."""
    if mode == "dot":
        return scale * dS @ k, scale * dS.T @ q_rows
    return 2.0 * scale * dS @ k, 2.0 * scale * (dS.T @ q_rows - k * dS.sum(axis=0)[:, None])


def sink_grad(p_sink: np.ndarray, D: np.ndarray) -> float:
    """d loss / d s for one head: -sum_i p_i D_i."""
    return -float(np.sum(p_sink * D))


def attention_backward(q, k, v, dout, *, scale, mode="dot", sink=None, mask_kind="none", window=0, bias=None,
                       keep=0, mask_keep=None, kv_start=None, kv_end=None):
    """Gradients of the forward with respect to q, k, v and the sink logits.

    The chain rule through the definitions above, in float64 and in this order
    (row i, key j of one (batch, query head); P and D from the forward):
      P_ij  = exp(z_ij - lse_i) on visible keys, 0 elsewhere
      D_i   = sum_e dout_ie * out_ie
      dV_j += sum_i P_ij dout_i                       (summed over the KV group)
      dP_ij = dout_i . v_j
      dS_ij = P_ij (dP_ij - D_i)
      dot:  dQ_i = scale sum_j dS_ij k_j,   dK_j += scale sum_i dS_ij q_i
      rbf:  z_ij = 2 scale q_i.k_j - scale |k_j|^2 (the logit frame above), so
            dQ_i = 2 scale sum_j dS_ij k_j,  dK_j += 2 scale (sum_i dS_ij q_i - k_j sum_i dS_ij)
      sink: the sink's share p_i = exp(s - lse_i) gives d out_i / d s = -p_i out_i,
            so dsink_h = -sum_i p_i D_i (summed over batch and rows).
    q, k, v, dout float64 arrays as in attention_forward; masks and padding as
    there.  Returns dq, dk, dv (shapes of q, k, v) and dsink (Hq,) (zeros
    without a sink).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    N, Hq, L, _ = q.shape
    H, S = k.shape[1], k.shape[2]
    g = Hq // H
    out, lse = attention_forward(q, k, v, scale=scale, mode=mode, sink=sink, mask_kind=mask_kind, window=window,
                                 bias=bias, keep=keep, mask_keep=mask_keep, kv_start=kv_start, kv_end=kv_end)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dsink = np.zeros(Hq, dtype=np.float64)
    rows = np.arange(L)
    vis_kind = visible(rows, S, L, mask_kind, window, keep)
    for n in range(N):
        rng = None
        if kv_start is not None or kv_end is not None:
            rng = (0 if kv_start is None else int(kv_start[n]), S if kv_end is None else int(kv_end[n]))
        vis = padded_visible(vis_kind, mask_keep, rng)
        for hq in range(Hq):
            kvh = hq // g
            z = logits(q[n, hq], k[n, kvh], scale, mode)
            if bias is not None:
                z = z + np.asarray(bias, dtype=np.float64)
            l = lse[n, hq][:, None]
            live = np.isfinite(l)
            P = np.where(vis & np.isfinite(z) & live, np.exp(np.where(live, z - l, 0.0)), 0.0)
            D = np.einsum("ie,ie->i", dout[n, hq], out[n, hq])
            dv[n, kvh] += P.T @ dout[n, hq]
            dP = dout[n, hq] @ v[n, kvh].T
            dS = softmax_grad(P, dP, D)
            gq, gk = score_input_grads(dS, q[n, hq], k[n, kvh], scale, mode)
            dq[n, hq] = gq
            dk[n, kvh] += gk
            if sink is not None:
                ps = np.where(live[:, 0], np.exp(float(sink[hq]) - np.where(live[:, 0], lse[n, hq], 0.0)), 0.0)
                dsink[hq] += sink_grad(ps, D)
    return dq, dk, dv, dsink
