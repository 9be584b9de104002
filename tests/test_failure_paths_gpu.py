"""Failure paths on the GPU without faulting or hanging it.

* A bounded wait that runs out: a kernel waits on a barrier nothing arrives at,
  gives up after a short cycle limit and records the timeout; the host reads
  ATTN_ERR_DEVICE_TIMEOUT once through attn_device_status, and the context
  stays usable (a forward call afterwards matches the oracle).
* A workspace allocation that fails: with the next allocation made to fail,
  a decode call and a prefill call with a float bias return ATTN_ERR_WORKSPACE
  and write nothing; the next call allocates and succeeds.
"""

import numpy as np
import pytest
import torch

import attention_tiled_attn_b200 as attn
from synth import gpu as sgpu
from synth import workloads as sw

import gpu_util as gu

pytestmark = pytest.mark.gpu

ATTN_ERR_WORKSPACE = -12
ATTN_ERR_DEVICE_TIMEOUT = -14


@pytest.fixture(scope="module", autouse=True)
def _cuda_ready():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from attention_tiled_attn_b200 import build as b
    b.build()
    sgpu.build()
    yield
    attn.inject_workspace_failures(0)
    assert attn.device_status() == 0


def test_bounded_wait_timeout_is_reported_and_the_context_survives():
    assert attn.device_status() == 0
    assert attn.inject_wait_timeout(20000) == 0
    assert attn.device_status() == ATTN_ERR_DEVICE_TIMEOUT
    assert attn.device_status() == 0  # read-and-clear
    assert attn.inject_wait_timeout(0) == -2
    gu.run_and_check_full(gu.small_recipe("after_timeout", L=200, S=200, Hq=4, H=2, mask_kind="causal",
                                          sink="normal"))
    assert attn.device_status() == 0


def _fill_nan(t):
    t.fill_(float("nan"))
    return t


@pytest.mark.parametrize("kind", ["decode", "prefill_bias"])
def test_failed_workspace_allocation_launches_nothing(kind):
    if kind == "decode":
        r = gu.small_recipe("ws_decode", L=1, S=3000, N=2, Hq=8, H=2, E=128, Ev=128, sink="normal", scale=0.0884)
    else:
        r = gu.small_recipe("ws_bias", L=300, S=300, Hq=2, H=2, mask_kind="causal", bias="random10")
    host = sw.generate(r)
    t = {x: sgpu.to_device(host[x], r) for x in ("q", "k", "v")}
    sink = None if host["sink"] is None else torch.from_numpy(host["sink"]).cuda()
    bias = None if host["bias"] is None else torch.from_numpy(host["bias"]).cuda()
    out = _fill_nan(torch.empty((r.N, r.Hq, r.L, r.Ev), dtype=torch.bfloat16, device="cuda"))
    lse = _fill_nan(torch.empty((r.N, r.Hq, r.L), dtype=torch.float32, device="cuda"))
    stream = torch.cuda.current_stream().cuda_stream
    ptr = lambda x: None if x is None else x.data_ptr()  # noqa: E731
    call = lambda: attn.attn_fwd_raw(  # noqa: E731
        ptr(t["q"]), ptr(t["k"]), ptr(t["v"]), ptr(out), ptr(lse), r.N, r.Hq, r.H, r.L, r.S, r.E, r.Ev, r.scale,
        attn.MODES[r.mode], ptr(sink), attn.MASKS[r.mask_kind], r.window, ptr(bias), 0, stream)
    torch.cuda.synchronize()
    attn.release_workspace()
    assert attn.inject_workspace_failures(1) == 0
    assert call() == ATTN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(out.float()).all() and torch.isnan(lse).all(), "a failed call wrote output"
    assert call() == 0  # the injection is used up: this call allocates
    torch.cuda.synchronize()
    ref = gu.oracle_rows(r, 0, 0, np.arange(r.L), host)
    gu.compare(r, gu.out_to_f64(out[0, 0]), lse[0, 0].cpu().numpy(), *ref, what=kind)
    assert attn.device_status() == 0
