"""The GPU copy of the input generator draws the same bits as the host copy."""

import numpy as np
import pytest
import torch

from synth import gpu as sgpu
from synth import workloads as sw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float64, torch.float32, torch.bfloat16])
@pytest.mark.parametrize("start,count", [(0, 1000), (1, 999), (123457, 4097), (10**9, 33)])
def test_device_draws_match_host(dtype, start, count):
    sgpu.build()
    key = sw.stream_key(5, 2)
    x = torch.empty(count, dtype=dtype, device="cuda")
    sgpu.normal_into(x, key, start)
    host = sw.normal_f64(key, start, count)
    if dtype == torch.float64:
        assert np.array_equal(x.cpu().numpy(), host)
    elif dtype == torch.float32:
        assert np.array_equal(x.cpu().numpy(), host.astype(np.float32))
    else:
        assert np.array_equal(x.view(torch.int16).cpu().numpy().view(np.uint16), sw.bf16_round_bits(host))


def test_device_workload_matches_host_slices():
    r = sw.RECIPES["dot_causal_2k_bf16"]
    t = sgpu.generate_on_device(r)
    for name, (n, h) in (("q", (3, 15)), ("k", (0, 0)), ("v", (2, 7))):
        got = t[name][n, h].view(torch.int16).cpu().numpy().view(np.uint16)
        want = sw.bf16_round_bits(sw._slice_values_f64(r, name, n, h))
        assert np.array_equal(got, want)
