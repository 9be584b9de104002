"""Backward (attn_bwd) on the GPU against the float64 oracle's attention_backward.

Inputs are the seeded bf16 draws of synth.workloads; the oracle widens the same
bits to float64 and runs its own forward, so it shares nothing with the CUDA
path but the inputs.  dout is a second seeded bf16 draw.

Tolerance (bf16 operands, fp32 accumulation): the kernel rounds P and dS to bf16
before the tensor-core products (relative error 2^-9 each) and reads D from the
bf16 forward output (2^-9); each gradient element sums O(S) or O(L) such terms
of mixed sign, so its error is a few 2^-9 (2e-3) relative to the gradient's
scale.  Measured on a B200 over the cases below and the three full-size
workloads, the largest errors were 4.2e-3 relative L2 and 4.3e-3 * max |ref|
max abs for dq, dk and dv, and 1.02e-2 relative L2 for dsink (a vector of one
sum per head, whose terms cancel).  The bar keeps about twice that: relative L2
and max abs / max |ref| <= 1e-2 for dq, dk, dv and <= 2e-2 for dsink.
"""

import dataclasses

import numpy as np
import pytest
import torch

import attention_tiled_attn_b200 as attn
from oracle import attention as orc
from synth import gpu as sgpu
from synth import workloads as sw

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS_FRAC = 1e-2
DSINK_REL_L2 = 2e-2
DSINK_MAX_ABS_FRAC = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda_ready():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from attention_tiled_attn_b200 import build as b
    b.build()
    sgpu.build()
    yield
    assert attn.device_status() == 0, "a kernel recorded a bounded-wait timeout"


def R(name, **kw):
    base = dict(N=1, Hq=2, H=2, L=64, S=64, E=64, Ev=64, dtype="bf16", mode="dot", scale=0.125,
                mask_kind="none", window=0, sink="none", bias="none", seed=200)
    base.update(kw)
    return sw.Recipe(name, **base)


CASES = [
    R("b_dot_causal_300_e128_g2", L=300, S=300, E=128, Ev=128, Hq=4, H=2, mask_kind="causal"),
    R("b_rbf_causal_257_sink", L=257, S=257, mode="rbf", mask_kind="causal", sink="fixed", sink_values=(0.0, 1.0)),
    R("b_dot_window100_515_g3_sink", L=515, S=515, Ev=128, Hq=6, H=2, mask_kind="window", window=100,
      sink="normal"),
    R("b_dot_none_L200_S600_g4_e128_ev64", L=200, S=600, E=128, Ev=64, Hq=8, H=2),
    R("b_dot_causal_L1_S1000_g4_decode", L=1, S=1000, E=128, Ev=128, Hq=8, H=2, mask_kind="causal", sink="normal",
      scale=0.0884),
    R("b_rbf_window64_L130_S700_e64_ev128", L=130, S=700, Ev=128, mode="rbf", mask_kind="window", window=64,
      scale=0.05),
    R("b_rbf_registers_260", L=260, S=260, mode="rbf", mask_kind="causal", registers=4, key_lognormal=True,
      sinusoid_pe=True, sink="normal"),
    R("b_dot_causal_33_g16", L=33, S=33, Hq=16, H=1, mask_kind="causal"),
    R("b_dot_none_600_n2", L=600, S=600, N=2, E=128, Ev=128, Hq=2, H=1, sink="normal", scale=0.0884),
    # the streaming mask, keep bits and key padding of attn_fwd_streaming / attn_fwd_padded
    R("b_stream_w100_keep4_600_g2", L=600, S=600, Hq=4, H=2, mask_kind="streaming", window=100, keep=4,
      sink="normal"),
    R("b_rbf_stream_w64_keep130_400", L=400, S=400, mode="rbf", mask_kind="streaming", window=64, keep=130,
      scale=0.05),
    R("b_keep_bits_causal_300_e128", L=300, S=300, E=128, Ev=128, Hq=4, H=2, mask_kind="causal",
      keep_mask="random10", sink="normal"),
    R("b_left_pad_causal_500_n3", L=500, S=500, N=3, mask_kind="causal", pad_left=0.5),
    R("b_rbf_window_keep_both_pads_450", L=450, S=450, N=2, mode="rbf", mask_kind="window", window=100,
      keep_mask="random10", pad_left=0.3, pad_right=0.3, scale=0.05),
    R("b_keep_right_pad_L200_S700", L=200, S=700, N=2, keep_mask="random10", pad_right=0.5, Ev=128),
    # every key tile walks exactly one, two or three 64-query tiles (pipeline fill and drain with
    # the dK of a tile issued out of order)
    R("b_dot_none_64_one_tile_e128", L=64, S=64, E=128, Ev=128, Hq=1, H=1),
    R("b_dot_none_128_two_tiles_e128", L=128, S=128, E=128, Ev=128, Hq=1, H=1),
    R("b_dot_none_192_three_tiles_e128", L=192, S=192, E=128, Ev=128, Hq=1, H=1),
    R("b_rbf_none_160_three_tiles_ragged", L=160, S=160, mode="rbf", Hq=1, H=1, scale=0.05),
]


def _dout(r, seed=77):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((r.N, r.Hq, r.L, r.Ev))
    return sw.bf16_round_bits(x)


def _check(name, got, ref):
    got = np.asarray(got, dtype=np.float64)
    nrm = np.linalg.norm(ref)
    err = np.abs(got - ref)
    scale = max(np.abs(ref).max(), 1e-30)
    sink = name.endswith("dsink")
    rel_bar, abs_bar = (DSINK_REL_L2, DSINK_MAX_ABS_FRAC) if sink else (REL_L2, MAX_ABS_FRAC)
    if nrm > 0:
        rel = np.linalg.norm(got - ref) / nrm
        assert rel <= rel_bar, f"{name}: rel L2 {rel:.3e}"
    assert err.max() <= abs_bar * scale, f"{name}: max abs {err.max():.3e} vs scale {scale:.3e}"
    return float(err.max() / scale)


def run_case(r):
    host = sw.generate(r)
    t = {x: sgpu.to_device(host[x], r) for x in ("q", "k", "v")}
    sink = None if host["sink"] is None else torch.from_numpy(host["sink"]).cuda()
    km = host["keep"]
    masks = dict(keep_first=r.keep,
                 mask_bits=None if km is None else torch.from_numpy(sw.pack_mask_bits(km).view(np.int32)).cuda(),
                 kv_start=None if host["kv_start"] is None else torch.from_numpy(host["kv_start"]).cuda(),
                 kv_end=None if host["kv_end"] is None else torch.from_numpy(host["kv_end"]).cuda())
    out, lse = attn.attn_fwd(t["q"], t["k"], t["v"], scale=r.scale, mode=r.mode, sink=sink, mask_kind=r.mask_kind,
                             window=r.window, **masks)
    dout_bits = _dout(r)
    dout = sgpu.to_device(dout_bits, r)
    dq, dk, dv, dsink = attn.attn_bwd(t["q"], t["k"], t["v"], out, lse, dout, scale=r.scale, mode=r.mode, sink=sink,
                                      mask_kind=r.mask_kind, window=r.window, **masks)
    torch.cuda.synchronize()
    q64, k64, v64 = (sw.as_f64(r, host[x]) for x in ("q", "k", "v"))
    rq, rk, rv, rs = orc.attention_backward(q64, k64, v64, sw.bf16_bits_to_f64(dout_bits), scale=r.scale,
                                            mode=r.mode,
                                            sink=None if host["sink"] is None else host["sink"].astype(np.float64),
                                            mask_kind=r.mask_kind, window=r.window, keep=r.keep, mask_keep=km,
                                            kv_start=host["kv_start"], kv_end=host["kv_end"])
    pairs = {"dq": (dq.cpu().numpy(), rq), "dk": (dk.cpu().numpy(), rk), "dv": (dv.cpu().numpy(), rv)}
    if sink is not None:
        pairs["dsink"] = (dsink.cpu().numpy(), rs)
    else:
        assert dsink is None
    res = {g: _errors(got, ref) for g, (got, ref) in pairs.items()}
    print(f"{r.name}: " + ", ".join(f"{g} rel L2 {e[0]:.2e} max abs/max|ref| {e[1]:.2e}" for g, e in res.items()))
    for g, (got, ref) in pairs.items():
        _check(f"{r.name} {g}", got, ref)
    return res


@pytest.mark.parametrize("r", CASES, ids=lambda r: r.name)
def test_backward_matches_oracle(r):
    run_case(r)


def test_backward_repeat_calls_are_deterministic_up_to_dq_order():
    """dk, dv and dsink are written once per key tile and are bit-identical across
    calls; dq sums tiles in an unordered way and agrees to float32 rounding."""
    r = dataclasses.replace(CASES[0], name="det")
    host = sw.generate(r)
    t = {x: sgpu.to_device(host[x], r) for x in ("q", "k", "v")}
    out, lse = attn.attn_fwd(t["q"], t["k"], t["v"], scale=r.scale, mask_kind=r.mask_kind)
    dout = sgpu.to_device(_dout(r), r)
    a = attn.attn_bwd(t["q"], t["k"], t["v"], out, lse, dout, scale=r.scale, mask_kind=r.mask_kind)
    b = attn.attn_bwd(t["q"], t["k"], t["v"], out, lse, dout, scale=r.scale, mask_kind=r.mask_kind)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert torch.allclose(a[0], b[0], rtol=1e-5, atol=1e-6)


def test_backward_with_sink_but_no_dsink_output():
    """Through the C entry point: sink logits given, dsink NULL. The call succeeds, writes dq, dk, dv
    (equal to the call that also returns dsink) and touches no dsink memory."""
    r = dataclasses.replace(CASES[2], name="no_dsink")
    host = sw.generate(r)
    t = {x: sgpu.to_device(host[x], r) for x in ("q", "k", "v")}
    sink = torch.from_numpy(host["sink"]).cuda()
    out, lse = attn.attn_fwd(t["q"], t["k"], t["v"], scale=r.scale, sink=sink, mask_kind=r.mask_kind,
                             window=r.window)
    dout = sgpu.to_device(_dout(r), r)
    ref = attn.attn_bwd(t["q"], t["k"], t["v"], out, lse, dout, scale=r.scale, sink=sink, mask_kind=r.mask_kind,
                        window=r.window)
    dq, dk, dv = (torch.empty_like(x) for x in ref[:3])
    st = attn.attn_bwd_raw(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), out.data_ptr(),
                           dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), None,
                           r.N, r.Hq, r.H, r.L, r.S, r.E, r.Ev, r.scale, 0, sink.data_ptr(), 2, r.window,
                           torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
    assert torch.allclose(dq, ref[0], rtol=1e-5, atol=1e-6)


# ---------------------------------------------------------------------------
# the benchmark's three backward workloads at full size
# ---------------------------------------------------------------------------

BWD_FULL = ["dot_causal_2k_bf16", "rbf_registers_4k_bf16", "sink_gqa_window_16k_bf16"]


def _dout_slice_host(r, n, hq):
    """dout[n, hq] as the device generator draws it for the benchmark (its own stream of the
    counter-based generator, bf16), regenerated on the host and widened to float64."""
    key = sw.stream_key(r.seed, sw.STREAM_DOUT)
    x = sw.normal_f64(key, ((n * r.Hq + hq) * r.L) * r.Ev, r.L * r.Ev).reshape(r.L, r.Ev)
    return sw.bf16_bits_to_f64(sw.bf16_round_bits(x))


def _errors(got, ref):
    """(relative L2 error, max abs error / max |ref|) of one gradient tensor."""
    got = np.asarray(got, dtype=np.float64)
    scale = max(np.abs(ref).max(), 1e-30)
    nrm = np.linalg.norm(ref)
    rel = float(np.linalg.norm(got - ref) / nrm) if nrm > 0 else 0.0
    return rel, float(np.abs(got - ref).max() / scale)


@pytest.mark.parametrize("name", BWD_FULL)
def test_backward_full_size(name):
    """The whole workload's backward on the GPU, in the benchmark's launch configuration
    (forward out and lse, dout from the generator's own stream); the oracle backward of the
    last (batch, KV head) slice -- all query heads of the group, every row and key -- gives dq
    of those heads, dk and dv of that KV head (the last key tile and the window edge included)
    and, with one batch, dsink of the group's heads."""
    r = sw.RECIPES[name]
    t = sgpu.generate_on_device(r)
    out, lse = attn.attn_fwd(t["q"], t["k"], t["v"], scale=r.scale, mode=r.mode, sink=t["sink"],
                             mask_kind=r.mask_kind, window=r.window)
    dout = torch.empty_like(out)
    sgpu.normal_into(dout, sw.stream_key(r.seed, sw.STREAM_DOUT))
    dq, dk, dv, dsink = attn.attn_bwd(t["q"], t["k"], t["v"], out, lse, dout, scale=r.scale, mode=r.mode,
                                      sink=t["sink"], mask_kind=r.mask_kind, window=r.window)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    n, kvh = r.N - 1, r.H - 1
    heads = list(range(kvh * r.group, (kvh + 1) * r.group))
    got_dq = dq[n, heads].cpu().numpy()
    got_dk = dk[n, kvh].cpu().numpy()
    got_dv = dv[n, kvh].cpu().numpy()
    got_ds = None if dsink is None else dsink[heads].cpu().numpy()
    del t, out, lse, dout, dq, dk, dv, dsink
    torch.cuda.empty_cache()
    q = np.stack([sw.tensor_slice_f64(r, "q", n, hq) for hq in heads])[None]
    k = sw.tensor_slice_f64(r, "k", n, kvh)[None, None]
    v = sw.tensor_slice_f64(r, "v", n, kvh)[None, None]
    do = np.stack([_dout_slice_host(r, n, hq) for hq in heads])[None]
    s = sw.sink_logits(r)
    rq, rk, rv, rs = orc.attention_backward(q, k, v, do, scale=r.scale, mode=r.mode,
                                            sink=None if s is None else s[heads].astype(np.float64),
                                            mask_kind=r.mask_kind, window=r.window)
    report = {}
    for g, (got, ref) in {"dq": (got_dq, rq[0]), "dk": (got_dk, rk[0, 0]), "dv": (got_dv, rv[0, 0])}.items():
        report[g] = _errors(got, ref)
        _check(f"{name} {g}", got, ref)
    if got_ds is not None and r.N == 1:
        # the kernel sums dsink over the batch; with one batch the slice's heads are complete
        report["dsink"] = _errors(got_ds, rs)
        _check(f"{name} dsink", got_ds, rs)
    print(f"{name} backward (n={n}, kv head {kvh}): " +
          ", ".join(f"{g} rel L2 {e[0]:.2e} max abs/max|ref| {e[1]:.2e}" for g, e in report.items()))
