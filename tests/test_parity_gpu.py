"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs.  Small cases compare every element; the reference
workloads, and every variant of them that the benchmark times, run at full
size in the benchmark's launch configuration and are compared on sampled
rows."""

import dataclasses

import numpy as np
import pytest
import torch

import attention_tiled_attn_b200 as attn
from synth import gpu as sgpu
from synth import workloads as sw

import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda_ready():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from attention_tiled_attn_b200 import build as b
    b.build()
    sgpu.build()
    yield
    assert attn.device_status() == 0, "a kernel recorded a bounded-wait timeout"


R = gu.small_recipe

PREFILL_CASES = [
    R("p_dot_none_128", L=128, S=128),
    R("p_dot_causal_300_e128_g2", L=300, S=300, E=128, Ev=128, Hq=4, H=2, mask_kind="causal"),
    R("p_rbf_causal_257_sink", L=257, S=257, mode="rbf", mask_kind="causal", sink="fixed",
      sink_values=(0.0, 1.0)),
    R("p_dot_window100_515_g3_sink", L=515, S=515, Ev=128, Hq=6, H=2, mask_kind="window", window=100,
      sink="normal"),
    R("p_dot_causal_L200_S600_g4", L=200, S=600, E=128, Ev=64, Hq=8, H=2, mask_kind="causal"),
    R("p_dot_causal_L300_S100_empty_rows", L=300, S=100, mask_kind="causal"),
    R("p_dot_bias10_192", L=192, S=192, Hq=1, H=1, bias="random10"),
    R("p_rbf_window64_400_g2_bias", L=400, S=400, Hq=4, H=2, mode="rbf", mask_kind="window", window=64,
      bias="random10"),
    R("p_rbf_registers_260", L=260, S=260, mode="rbf", mask_kind="causal", registers=4, key_lognormal=True,
      sinusoid_pe=True, sink="normal"),
    R("p_dot_L17_S1", L=17, S=1),
    R("p_dot_causal_33_g16", L=33, S=33, Hq=16, H=1, mask_kind="causal"),
    R("p_rbf_none_L128_S1000_e128", L=128, S=1000, E=128, Ev=128, mode="rbf", scale=0.05),
    R("p_dot_window1_130", L=130, S=130, mask_kind="window", window=1),
    R("p_dot_none_600_g2_e128_sink", L=600, S=600, E=128, Ev=128, Hq=4, H=2, N=2, sink="normal",
      scale=0.0884),
    # streaming mask: kept initial keys plus a window; key tiles in between are skipped
    R("p_stream_keep4_w64_600_g2_sink", L=600, S=600, Hq=4, H=2, mask_kind="streaming", window=64, keep=4,
      sink="normal"),
    R("p_rbf_stream_keep130_w100_700_bias", L=700, S=700, E=128, Ev=128, mode="rbf", mask_kind="streaming",
      window=100, keep=130, bias="random10", scale=0.05),
    R("p_stream_keep0_w50_300", L=300, S=300, mask_kind="streaming", window=50, keep=0),
    R("p_stream_keep_all_300", L=300, S=300, Hq=4, H=1, mask_kind="streaming", window=20, keep=1000),
    R("p_stream_L200_S900_keep16_w128_e128", L=200, S=900, E=128, Ev=128, Hq=6, H=2, mask_kind="streaming",
      window=128, keep=16, sink="normal", scale=0.0884),
    R("p_stream_w1_keep1_520", L=520, S=520, mask_kind="streaming", window=1, keep=1),
    R("p_stream_keep256_w128_1100", L=1100, S=1100, N=2, mask_kind="streaming", window=128, keep=256),
    # a float bias is turned into keep bits before the kernel; blocks holding finite
    # nonzero entries are flagged and add the bias values themselves
    R("p_dot_bias_mixed_causal_300_e128_g2", L=300, S=300, E=128, Ev=128, Hq=4, H=2, mask_kind="causal",
      bias="mixed", sink="normal", scale=0.0884),
    R("p_rbf_bias_mixed_window_L260_S401", L=260, S=401, Hq=2, H=1, mode="rbf", mask_kind="window", window=200,
      bias="mixed", scale=0.05),
    R("p_dot_bias_mixed_none_L130_S257_sink", L=130, S=257, bias="mixed", sink="normal"),
]

FP32_CASES = [
    R("f_dot_bias_130_e128", L=130, S=130, E=128, Ev=128, dtype="f32", bias="random10"),
    R("f_rbf_window50_sink_g3", L=150, S=170, Hq=3, H=1, dtype="f32", mode="rbf", mask_kind="window", window=50,
      sink="normal"),
    R("f_dot_causal_70_g2_ev128", L=70, S=70, Ev=128, Hq=2, H=1, dtype="f32", mask_kind="causal"),
    R("f_dot_causal_L1_S6", L=1, S=6, dtype="f32", mask_kind="causal"),
    R("f_dot_causal_L40_S10_empty", L=40, S=10, dtype="f32", mask_kind="causal", sink="fixed",
      sink_values=(0.5, -0.5)),
    R("f_stream_keep5_w40_300_sink", L=300, S=300, Hq=4, H=2, dtype="f32", mask_kind="streaming", window=40,
      keep=5, sink="normal"),
    R("f_rbf_stream_keep70_w30_L100_S400", L=100, S=400, dtype="f32", mode="rbf", mask_kind="streaming",
      window=30, keep=70, bias="random10"),
]

DECODE_CASES = [
    R("d_L1_g4_S1000_sink", L=1, S=1000, E=128, Ev=128, N=2, Hq=12, H=3, sink="normal", scale=0.0884),
    R("d_L1_g1_S5000_causal", L=1, S=5000, N=3, Hq=1, H=1, mask_kind="causal"),
    R("d_L4_g4_S777_causal_sink", L=4, S=777, Hq=8, H=2, mask_kind="causal", sink="normal"),
    R("d_L2_g2_S300_window_bias", L=2, S=300, Hq=2, H=1, mask_kind="window", window=50, bias="random10"),
    R("d_L1_g8_S64", L=1, S=64, Hq=8, H=1),
    R("d_L1_S1", L=1, S=1, Hq=2, H=2),
    R("d_L3_g5_S129_e128_ev64", L=3, S=129, E=128, Ev=64, Hq=5, H=1),
    R("d_many_units", L=1, S=200, N=40, Hq=16, H=8, sink="normal"),
    R("d_L2_causal_S1_empty_row", L=2, S=1, Hq=2, H=2, mask_kind="causal"),
    R("d_stream_L1_S5000_keep4_w1000_g4", L=1, S=5000, Hq=8, H=2, mask_kind="streaming", window=1000, keep=4,
      sink="normal"),
    R("d_stream_L3_S800_keep70_w100_g2_bias", L=3, S=800, Hq=4, H=2, mask_kind="streaming", window=100, keep=70,
      bias="random10"),
    R("d_stream_L1_S300_keep200_w150_overlap", L=1, S=300, mask_kind="streaming", window=150, keep=200),
    R("d_stream_L2_S50_keep0_w10", L=2, S=50, mask_kind="streaming", window=10, keep=0),
    R("d_stream_many_units", L=1, S=3000, N=40, Hq=16, H=8, E=128, Ev=128, mask_kind="streaming", window=256,
      keep=4, scale=0.0884),
    # units of one 64-key chunk: a CTA's range holds whole units with a single chunk, so one of the two
    # consumer groups has no chunk of the unit and merges its empty state; two-chunk units with a
    # ragged second chunk split between CTAs at odd offsets
    R("d_single_chunk_units_E128", L=1, S=64, N=40, Hq=32, H=8, E=128, Ev=128, sink="normal", scale=0.0884),
    R("d_two_chunk_ragged_units_E128", L=1, S=100, N=37, Hq=16, H=4, E=128, Ev=128, mode="rbf", scale=0.05),
    # the RBF score on the split-key path (key norms from the staged chunk)
    R("d_rbf_L1_g4_S1000_sink", L=1, S=1000, E=128, Ev=128, N=2, Hq=8, H=2, mode="rbf", sink="normal",
      scale=0.0884),
    R("d_rbf_L4_g4_S777_causal_sink", L=4, S=777, Hq=8, H=2, mode="rbf", mask_kind="causal", sink="normal",
      scale=0.05),
    R("d_rbf_L2_S300_window_bias", L=2, S=300, Hq=2, H=1, mode="rbf", mask_kind="window", window=50,
      bias="random10"),
    R("d_rbf_lognormal_keys_L3_S400_e64_ev128", L=3, S=400, Hq=3, H=1, Ev=128, mode="rbf", mask_kind="causal",
      key_lognormal=True, sink="normal"),
    R("d_rbf_stream_L1_S5000_keep4_w1000_g4", L=1, S=5000, Hq=8, H=2, mode="rbf", mask_kind="streaming",
      window=1000, keep=4, sink="normal", scale=0.05),
    # one unit over every CTA: more than 32 partials per unit for the combine
    R("d_rbf_one_unit_S19200_e128_ev64", L=1, S=19200, Hq=4, H=1, E=128, Ev=64, mode="rbf", sink="normal",
      scale=0.05),
    R("d_one_unit_L3_S20000_g5", L=3, S=20000, Hq=5, H=1, mask_kind="causal", sink="normal"),
]


# packed keep bits and per-batch key padding (attn_fwd_padded), on every path
PADDED_CASES = [
    R("pd_keep_causal_300_g2_e128", L=300, S=300, E=128, Ev=128, Hq=4, H=2, mask_kind="causal",
      keep_mask="random10", sink="normal"),
    R("pd_left_pad_causal_600", L=600, S=600, N=3, mask_kind="causal", pad_left=0.5),
    R("pd_right_pad_none_500_e128", L=500, S=500, N=2, E=128, Ev=128, pad_right=0.4, sink="normal"),
    R("pd_rbf_window_keep_both_pads_700", L=700, S=700, N=2, mode="rbf", mask_kind="window", window=100,
      keep_mask="random10", pad_left=0.3, pad_right=0.3),
    R("pd_keep_none_L200_S1000", L=200, S=1000, keep_mask="random10", pad_left=0.2),
    R("pd_keep_S130_ragged_words", L=130, S=130, Hq=6, H=2, keep_mask="random10", mask_kind="causal"),
    R("f_pd_keep_left_causal_f32", L=150, S=170, Hq=3, H=1, dtype="f32", mask_kind="causal", keep_mask="random10",
      pad_left=0.4, sink="normal"),
    R("f_pd_right_window_rbf_f32", L=100, S=300, N=2, dtype="f32", mode="rbf", mask_kind="window", window=60,
      pad_right=0.5),
    R("d_pd_keep_L2_S777", L=2, S=777, Hq=4, H=2, keep_mask="random10", sink="normal"),
    R("d_pd_left_L1_S5000", L=1, S=5000, N=4, Hq=8, H=2, E=128, Ev=128, pad_left=0.5, scale=0.0884),
    R("d_pd_right_L4_g4_causal", L=4, S=900, N=3, Hq=8, H=2, mask_kind="causal", pad_right=0.6, keep_mask="random10"),
    R("d_pd_rbf_keep_left_L2_S777", L=2, S=777, Hq=4, H=2, mode="rbf", keep_mask="random10", pad_left=0.3,
      sink="normal", scale=0.05),
]


@pytest.mark.parametrize("r", PADDED_CASES, ids=lambda r: r.name)
def test_padded_small(r):
    gu.run_and_check_full(r)


def test_padded_start_beyond_end_masks_everything():
    """kv_start >= kv_end leaves the batch no key: out 0, lse -inf (or the sink)."""
    for sink in ("none", "normal"):
        r = R("pd_empty", L=130, S=130, N=2, Hq=2, H=2, sink=sink, pad_left=0.9)
        host = sw.generate(r)
        t = {x: sgpu.to_device(host[x], r) for x in ("q", "k", "v")}
        t["sink"] = None if host["sink"] is None else torch.from_numpy(host["sink"]).cuda()
        t["bias"] = None
        t["kv_start"] = torch.tensor([120, 7], dtype=torch.int32, device="cuda")
        t["kv_end"] = torch.tensor([60, 7], dtype=torch.int32, device="cuda")
        out, lse = gu.run_gpu(r, t)
        assert torch.all(out == 0)
        want = float("-inf") if host["sink"] is None else None
        for hq in range(r.Hq):
            col = lse[:, hq].cpu().numpy()
            exp = want if want is not None else float(host["sink"][hq])
            assert np.all(col == exp) if want is not None else np.allclose(col, exp, atol=1e-6)


# exact decode over a listed key subset (a top-k selection's output)
INDEXED_CASES = [
    R("ix_L1_g4_S1000_sel100_sink", L=1, S=1000, E=128, Ev=128, N=2, Hq=8, H=2, n_sel=100, sink="normal",
      scale=0.0884),
    R("ix_L1_S5000_sel333_e64", L=1, S=5000, N=1, Hq=2, H=2, n_sel=333),
    R("ix_L4_g4_S300_sel50_causal", L=4, S=300, Hq=8, H=2, n_sel=50, mask_kind="causal", sink="normal"),
    R("ix_L2_g2_S300_sel90_window_bias", L=2, S=300, Hq=2, H=1, n_sel=90, mask_kind="window", window=50,
      bias="random10"),
    R("ix_sel1", L=1, S=200, Hq=4, H=4, n_sel=1),
    R("ix_sel_over_S_repeats", L=1, S=50, Hq=2, H=1, n_sel=130, sink="normal"),
    R("ix_many_units", L=1, S=2000, N=40, Hq=16, H=8, E=128, Ev=128, n_sel=70, scale=0.0884),
    R("ix_e64_ev128_g16", L=1, S=700, Hq=16, H=1, E=64, Ev=128, n_sel=200),
    R("ix_e128_ev64_L3_g5", L=3, S=400, Hq=5, H=1, E=128, Ev=64, n_sel=129, mask_kind="causal"),
]


@pytest.mark.parametrize("r", INDEXED_CASES, ids=lambda r: r.name)
def test_decode_indexed_small(r):
    gu.run_and_check_full(r)


def test_decode_indexed_padding_and_duplicates():
    """-1 and >= S entries select nothing; a listed duplicate counts twice; an all-padding list gives
    out = 0 and lse = -inf (lse = sink with a sink)."""
    r = R("ix_pad", L=2, S=300, Hq=4, H=2, n_sel=40, sink="normal")
    idx = sw.key_index_set(r).copy()
    idx[0, 0, :5] = -1
    idx[0, 1, 7] = 300
    idx[1 % r.N, 1, 9] = 10**6
    idx[0, 0, 20] = idx[0, 0, 21]
    gu.run_and_check_full(r, idx)
    for sink in ("none", "normal"):
        r0 = R("ix_all_pad", L=1, S=100, Hq=2, H=2, n_sel=70, sink=sink)
        gu.run_and_check_full(r0, np.full((r0.N, r0.H, 70), -1, dtype=np.int32))


@pytest.mark.parametrize("r", PREFILL_CASES, ids=lambda r: r.name)
def test_prefill_bf16_small(r):
    gu.run_and_check_full(r)


@pytest.mark.parametrize("r", FP32_CASES, ids=lambda r: r.name)
def test_fp32_small(r):
    gu.run_and_check_full(r)


@pytest.mark.parametrize("r", DECODE_CASES, ids=lambda r: r.name)
def test_decode_bf16_small(r):
    assert (r.Hq // r.H) * r.L <= 16
    gu.run_and_check_full(r)


def test_tiny_reference_workload_fp32():
    gu.run_and_check_full(sw.RECIPES["tiny_rbf_sink_causal_f32"])


def test_output_canaries():
    """Nothing is written past the end of out and lse."""
    r = R("canary", L=300, S=300, E=128, Ev=128, Hq=4, H=2, mask_kind="causal", sink="normal")
    host = sw.generate(r)
    q, k, v = (sgpu.to_device(host[x], r) for x in ("q", "k", "v"))
    sink = torch.from_numpy(host["sink"]).cuda()
    for shape_l in (r.L, 1):
        qq = q[:, :, :shape_l].contiguous()
        n_out = r.N * r.Hq * shape_l * r.Ev
        n_lse = r.N * r.Hq * shape_l
        obuf = torch.full((n_out + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
        lbuf = torch.full((n_lse + 4096,), 7.0, dtype=torch.float32, device="cuda")
        out = obuf[:n_out].view(r.N, r.Hq, shape_l, r.Ev)
        lse = lbuf[:n_lse].view(r.N, r.Hq, shape_l)
        attn.attn_fwd(qq, k, v, scale=r.scale, sink=sink, mask_kind="causal", out=out, lse=lse)
        torch.cuda.synchronize()
        assert torch.all(obuf[n_out:] == 7.0) and torch.all(lbuf[n_lse:] == 7.0)


def test_repeat_calls_are_deterministic():
    r = R("det", L=256, S=256, Hq=4, H=2, mask_kind="causal", sink="normal")
    host = sw.generate(r)
    t = {x: sgpu.to_device(host[x], r) for x in ("q", "k", "v")}
    t["sink"], t["bias"] = torch.from_numpy(host["sink"]).cuda(), None
    a, la = gu.run_gpu(r, t)
    b, lb = gu.run_gpu(r, t)
    assert torch.equal(a, b) and torch.equal(la, lb)


# ---------------------------------------------------------------------------
# the reference workloads at full size, sampled rows
# ---------------------------------------------------------------------------

FULL = ["dot_causal_2k_bf16", "dot_bias10_2k_f32", "rbf_registers_4k_bf16", "sink_gqa_window_16k_bf16",
        "decode_sink_gqa_128k_bf16"]


def test_decode_indexed_full_size_top_k_33x():
    """The long-context decode workload (N=32, 32 query / 8 KV heads, S=131072, E=128) over a
    33x-sparse selection (3971 keys per KV head, as the benchmark times it), sampled units against
    the oracle."""
    r = dataclasses.replace(sw.RECIPES["decode_sink_gqa_128k_bf16"], name="decode_top_k_33x", n_sel=131072 // 33)
    t = sgpu.generate_on_device(r)
    out, lse = gu.run_gpu(r, t)
    assert torch.isfinite(out.float()).all()
    host = {"key_idx": sw.key_index_set(r)}
    for n, hq in ((0, 0), (r.N - 1, r.Hq - 1), (17, 13)):
        ref_out, ref_lse = gu.oracle_rows(r, n, hq, [0], host)
        gu.compare(r, gu.out_to_f64(out[n, hq, [0]]), lse[n, hq, [0]].cpu().numpy(), ref_out, ref_lse,
                   f"top-k n={n} hq={hq}")
    del t, out, lse
    torch.cuda.empty_cache()


def _variant(base: str, label: str, **kw):
    r = dataclasses.replace(sw.RECIPES[base], name=f"{base}:{label}", **kw)
    return pytest.param(r, id=r.name)


# the benchmark's extra lines: controls and mask variants of the reference workloads, same shapes and data
FULL_VARIANTS = [
    _variant("dot_causal_2k_bf16", "steady_state_noncausal_8k", N=1, L=8192, S=8192, mask_kind="none"),
    _variant("dot_causal_2k_bf16", "keep_bits_random10", keep_mask="random10"),
    _variant("dot_causal_2k_bf16", "bias_random10", bias="random10"),
    _variant("dot_causal_2k_bf16", "left_pad_upto50", pad_left=0.5),
    _variant("rbf_registers_4k_bf16", "dot_control", mode="dot"),
    _variant("sink_gqa_window_16k_bf16", "no_sink_control", sink="none"),
    _variant("sink_gqa_window_16k_bf16", "streaming_keep4", mask_kind="streaming", keep=4),
    _variant("decode_sink_gqa_128k_bf16", "no_sink_control", sink="none"),
    _variant("decode_sink_gqa_128k_bf16", "streaming_keep4_w4096", mask_kind="streaming", window=4096, keep=4),
    _variant("decode_sink_gqa_128k_bf16", "rbf", mode="rbf"),
    _variant("decode_sink_gqa_128k_bf16", "batch1", N=1),
    _variant("dot_causal_2k_bf16", "bias_mixed", bias="mixed"),
]


@pytest.mark.parametrize("name", FULL)
def test_reference_workload_full_size(name):
    check_full_size(sw.RECIPES[name])


@pytest.mark.parametrize("r", FULL_VARIANTS)
def test_bench_variant_full_size(r):
    check_full_size(r)


def check_full_size(r: sw.Recipe):
    """The whole workload on the GPU; sampled rows of three (n, hq) units (two for decode) against the oracle."""
    name = r.name
    t = sgpu.generate_on_device(r)
    out, lse = gu.run_gpu(r, t)
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(sum(map(ord, name)))
    units = [(0, 0), (r.N - 1, r.Hq - 1), (int(rng.integers(r.N)), int(rng.integers(r.Hq)))]
    if r.L == 1:
        units = units[:2]
    for n, hq in units:
        rows = gu.sample_rows(r.L, rng, count=12 if r.L > 1 else 0)
        ref_out, ref_lse = gu.oracle_rows(r, n, hq, rows)
        got = gu.out_to_f64(out[n, hq, rows])
        got_lse = lse[n, hq, rows].cpu().numpy()
        gu.compare(r, got, got_lse, ref_out, ref_lse, f"{name} n={n} hq={hq}")
    del t, out, lse
    torch.cuda.empty_cache()
