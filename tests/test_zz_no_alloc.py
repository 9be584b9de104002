"""The allocation-free decode entry point against the regular one.

attn_decode_fwd_noalloc serves callers that may not allocate device memory
while they run (services that reserve all GPU memory at start-up, host
frameworks whose allocator owns the device): it runs the decode kernels on a
fixed scratch array compiled into the library.  Here it is called through the
C ABI twice in a row and each result is compared with attn_fwd's on the same
inputs, within the bf16 tolerances of the other parity tests.  The file is
named so that pytest collects it last, and it sets up everything it needs so
that it also passes alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

import attention_tiled_attn_b200 as attn
from attention_tiled_attn_b200 import build as attn_build
from synth import gpu as sgpu
from synth import workloads as sw

pytestmark = pytest.mark.gpu

BF16_ABS, BF16_REL_L2, BF16_LSE = 2e-2, 5e-3, 1e-3

CASES = [
    sw.Recipe("na_L1_g4_S1000_sink", N=2, Hq=8, H=2, L=1, S=1000, E=128, Ev=128, dtype="bf16", mode="dot",
              scale=0.0884, mask_kind="none", sink="normal", seed=21),
    sw.Recipe("na_L4_g4_S777_causal_bias", N=1, Hq=8, H=2, L=4, S=777, E=64, Ev=64, dtype="bf16", mode="dot",
              scale=0.125, mask_kind="causal", bias="random10", seed=22),
    sw.Recipe("na_L1_S131072_e128", N=2, Hq=32, H=8, L=1, S=131072, E=128, Ev=128, dtype="bf16", mode="dot",
              scale=0.0884, mask_kind="none", sink="normal", seed=23),
]


def _ptr(t):
    return None if t is None else t.data_ptr()


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required")
    attn_build.build()
    sgpu.build()
    return attn.load_library()


def _inputs(r):
    t = sgpu.generate_on_device(r)
    return t


@pytest.mark.parametrize("r", CASES, ids=lambda r: r.name)
def test_noalloc_matches_attn_fwd_twice(lib, r):
    t = _inputs(r)
    ref_out, ref_lse = attn.attn_fwd(t["q"], t["k"], t["v"], scale=r.scale, mode=r.mode, sink=t["sink"],
                                     mask_kind=r.mask_kind, window=r.window, bias=t["bias"])
    torch.cuda.synchronize()
    ref = ref_out.float()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = attn.attn_decode_fwd_noalloc_raw(
            _ptr(t["q"]), _ptr(t["k"]), _ptr(t["v"]), _ptr(out), _ptr(lse), r.N, r.Hq, r.H, r.L, r.S, r.E, r.Ev,
            r.scale, attn.MODES[r.mode], _ptr(t["sink"]), attn.MASKS[r.mask_kind], r.window, _ptr(t["bias"]),
            stream)
        assert st == 0, attn.status_string(st)
        torch.cuda.synchronize()
        got = out.float()
        err = (got - ref).abs().max().item()
        rel = ((got - ref).norm() / ref.norm()).item()
        finite = torch.isfinite(ref_lse)
        assert torch.equal(torch.isfinite(lse), finite)
        lerr = (lse[finite] - ref_lse[finite]).abs().max().item() if finite.any() else 0.0
        assert err <= BF16_ABS and rel <= BF16_REL_L2 and lerr <= BF16_LSE, (call, err, rel, lerr)
    assert attn.device_status() == 0


def _pool_reserved_bytes(dev: int) -> int:
    """Bytes the device's default stream-ordered pool (the one cudaMallocAsync draws on) holds."""
    from cuda.bindings import driver as drv
    err, pool = drv.cuDeviceGetDefaultMemPool(dev)
    assert err == drv.CUresult.CUDA_SUCCESS, err
    err, val = drv.cuMemPoolGetAttribute(pool, drv.CUmemPool_attribute.CU_MEMPOOL_ATTR_RESERVED_MEM_CURRENT)
    assert err == drv.CUresult.CUDA_SUCCESS, err
    return int(val)


def test_noalloc_call_takes_no_device_memory(lib):
    """With the library's own workspace released, a call after the first (which loads the
    library's device code and the fixed array into the context) changes neither the device's
    free memory nor what its default stream-ordered pool holds."""
    r = CASES[0]
    t = _inputs(r)
    out = torch.empty((r.N, r.Hq, r.L, r.Ev), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((r.N, r.Hq, r.L), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    dev = torch.cuda.current_device()

    def call():
        st = attn.attn_decode_fwd_noalloc_raw(
            _ptr(t["q"]), _ptr(t["k"]), _ptr(t["v"]), _ptr(out), _ptr(lse), r.N, r.Hq, r.H, r.L, r.S, r.E, r.Ev,
            r.scale, attn.MODES[r.mode], _ptr(t["sink"]), attn.MASKS[r.mask_kind], r.window, _ptr(t["bias"]),
            stream)
        assert st == 0, attn.status_string(st)
        torch.cuda.synchronize()

    attn.release_workspace()
    call()
    free0, _ = torch.cuda.mem_get_info()
    pool0 = _pool_reserved_bytes(dev)
    call()
    free1, _ = torch.cuda.mem_get_info()
    pool1 = _pool_reserved_bytes(dev)
    assert free1 == free0, (free0, free1)
    assert pool1 == pool0, (pool0, pool1)


def test_noalloc_rejects_oversized_and_non_decode_calls(lib):
    P = 0x10000  # aligned placeholder addresses: both calls are rejected before any launch
    # 2048 (batch, KV head) units of a 64-key cache need more partial slots than the fixed area holds
    st = attn.attn_decode_fwd_noalloc_raw(P, P, P, P, P, 512, 4, 4, 1, 64, 128, 128, 0.1, 0, None, 0, 0, None,
                                          None)
    assert st == -16, attn.status_string(st)
    assert "scratch" in attn.status_string(st)
    # a prefill-shaped call is not served by this entry point
    st = attn.attn_decode_fwd_noalloc_raw(P, P, P, P, P, 1, 2, 2, 300, 300, 64, 64, 0.1, 0, None, 0, 0, None, None)
    assert st == -17, attn.status_string(st)
    assert attn.decode_noalloc_scratch_bytes() == 8 << 20
