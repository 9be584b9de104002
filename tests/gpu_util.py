"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the float64 oracle on the same seeded inputs, and compare."""

from __future__ import annotations

import math

import numpy as np
import torch

import attention_tiled_attn_b200 as attn
from oracle import attention as orc
from synth import gpu as sgpu
from synth import workloads as sw

# tolerances (fp32: exact-fp32 path; bf16: tensor cores with fp32 accumulation)
F32_ABS = 1e-5
F32_LSE = 1e-5
BF16_ABS = 2e-2
BF16_REL_L2 = 5e-3
BF16_LSE = 1e-3

def api_mode(r: sw.Recipe) -> str:
    return r.mode  # "dot" or "rbf"; a sink applies whenever sink logits are passed


def run_gpu(r: sw.Recipe, t: dict):
    if r.n_sel > 0:
        out, lse = attn.attn_decode_indexed(t["q"], t["k"], t["v"], t["key_idx"], scale=r.scale, sink=t["sink"],
                                            mask_kind=r.mask_kind, window=r.window, bias=t["bias"])
        torch.cuda.synchronize()
        return out, lse
    out, lse = attn.attn_fwd(t["q"], t["k"], t["v"], scale=r.scale, mode=api_mode(r), sink=t["sink"],
                             mask_kind=r.mask_kind, window=r.window, bias=t["bias"], keep_first=r.keep,
                             mask_bits=t.get("mask_bits"), kv_start=t.get("kv_start"), kv_end=t.get("kv_end"))
    torch.cuda.synchronize()
    return out, lse


def out_to_f64(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy().astype(np.float64)


def oracle_rows(r: sw.Recipe, n: int, hq: int, rows, host: dict | None = None):
    """Oracle out (R, Ev) and lse (R,) for query rows of (n, hq), from host-regenerated inputs."""
    rows = np.asarray(rows, dtype=np.int64)
    kvh = hq // r.group
    if r.n_sel > 0:
        # the index-set oracle on this query head alone (one KV head, all L rows), then the rows asked for
        q = sw.tensor_slice_f64(r, "q", n, hq)[None, None]
        k = sw.tensor_slice_f64(r, "k", n, kvh)[None, None]
        v = sw.tensor_slice_f64(r, "v", n, kvh)[None, None]
        idx = (host["key_idx"] if host is not None else sw.key_index_set(r))[n, kvh][None, None]
        sink = sw.sink_logits(r)
        bias = sw.bias_matrix(r)
        o, l = orc.attention_over_index_set(q, k, v, idx, scale=r.scale,
                                            sink=None if sink is None else sink[hq:hq + 1].astype(np.float64),
                                            mask_kind=r.mask_kind, window=r.window,
                                            bias=None if bias is None else bias.astype(np.float64))
        return o[0, 0, rows], l[0, 0, rows]
    if host is not None:
        q = sw.as_f64(r, host["q"][n, hq])
        k = sw.as_f64(r, host["k"][n, kvh])
        v = sw.as_f64(r, host["v"][n, kvh])
    else:
        q = sw.tensor_slice_f64(r, "q", n, hq)
        k = sw.tensor_slice_f64(r, "k", n, kvh)
        v = sw.tensor_slice_f64(r, "v", n, kvh)
    sink = sw.sink_logits(r)
    bias = sw.bias_matrix(r)
    s = None if sink is None else float(sink[hq])
    b = None if bias is None else bias[rows].astype(np.float64)
    km = sw.keep_matrix(r)
    ks, ke = sw.kv_ranges(r)
    rng = None if ks is None else (int(ks[n]), int(ke[n]))
    return orc.attend_rows(q[rows], rows, k, v, r.L, scale=r.scale, mode=r.mode, sink=s,
                           mask_kind=r.mask_kind, window=r.window, bias_rows=b, keep=r.keep,
                           keep_rows=None if km is None else km[rows], kv_range=rng)


def compare(r: sw.Recipe, got_out, got_lse, ref_out, ref_lse, what=""):
    got_out = np.asarray(got_out, dtype=np.float64)
    got_lse = np.asarray(got_lse, dtype=np.float64)
    dead = ~np.isfinite(ref_lse)
    assert np.array_equal(~np.isfinite(got_lse), dead), f"{what}: -inf lse rows differ"
    if dead.any():
        assert np.all(got_out[dead] == 0.0), f"{what}: fully masked rows must be 0"
        assert np.all(got_lse[dead] == -np.inf)
    live = ~dead
    err = np.abs(got_out - ref_out)
    lse_err = np.abs(got_lse[live] - ref_lse[live]) if live.any() else np.zeros(1)
    if r.dtype == "f32":
        assert err.max() <= F32_ABS, f"{what}: max abs {err.max():.3e}"
        assert lse_err.max() <= F32_LSE, f"{what}: lse {lse_err.max():.3e}"
    else:
        assert err.max() <= BF16_ABS, f"{what}: max abs {err.max():.3e}"
        nrm = np.linalg.norm(ref_out)
        if nrm > 0:
            rel = np.linalg.norm(got_out - ref_out) / nrm
            assert rel <= BF16_REL_L2, f"{what}: rel L2 {rel:.3e}"
        assert lse_err.max() <= BF16_LSE, f"{what}: lse {lse_err.max():.3e}"
    return float(err.max()), float(lse_err.max())


def small_recipe(name, **kw) -> sw.Recipe:
    base = dict(N=1, Hq=2, H=2, L=64, S=64, E=64, Ev=64, dtype="bf16", mode="dot", scale=0.125,
                mask_kind="none", window=0, sink="none", bias="none", seed=100)
    base.update(kw)
    return sw.Recipe(name, **base)


def run_and_check_full(r: sw.Recipe, key_idx: np.ndarray | None = None):
    """Whole-tensor comparison for small recipes (key_idx overrides the recipe's key lists)."""
    host = sw.generate(r)
    t = {k: sgpu.to_device(host[k], r) for k in ("q", "k", "v")}
    t["sink"] = None if host["sink"] is None else torch.from_numpy(host["sink"]).cuda()
    t["bias"] = None if host["bias"] is None else torch.from_numpy(host["bias"]).cuda()
    if r.n_sel > 0:
        idx = host["key_idx"] if key_idx is None else key_idx
        t["key_idx"] = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
        out, lse = run_gpu(r, t)
        ref_out, ref_lse = orc.attention_over_index_set(
            sw.as_f64(r, host["q"]), sw.as_f64(r, host["k"]), sw.as_f64(r, host["v"]), idx, scale=r.scale,
            sink=None if host["sink"] is None else host["sink"].astype(np.float64), mask_kind=r.mask_kind,
            window=r.window, bias=None if host["bias"] is None else host["bias"].astype(np.float64))
        return compare(r, out_to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, r.name)
    if host["keep"] is not None:
        t["mask_bits"] = torch.from_numpy(sw.pack_mask_bits(host["keep"]).view(np.int32)).cuda()
    if host["kv_start"] is not None:
        t["kv_start"] = torch.from_numpy(host["kv_start"]).cuda()
        t["kv_end"] = torch.from_numpy(host["kv_end"]).cuda()
    out, lse = run_gpu(r, t)
    ref_out, ref_lse = orc.attention_forward(
        sw.as_f64(r, host["q"]), sw.as_f64(r, host["k"]), sw.as_f64(r, host["v"]), scale=r.scale, mode=r.mode,
        sink=None if host["sink"] is None else host["sink"].astype(np.float64), mask_kind=r.mask_kind,
        window=r.window, bias=None if host["bias"] is None else host["bias"].astype(np.float64), keep=r.keep,
        mask_keep=host["keep"], kv_start=host["kv_start"], kv_end=host["kv_end"])
    return compare(r, out_to_f64(out), lse.cpu().numpy(), ref_out, ref_lse, r.name)


def sample_rows(L: int, rng, count=24):
    fixed = {0, L - 1, min(127, L - 1), min(128, L - 1), L // 2}
    extra = set(rng.integers(0, L, size=count).tolist())
    return np.array(sorted(fixed | extra))
