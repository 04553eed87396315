"""GPU-side error paths: argument checks that return a status, empty inputs,
and failure detection of a bounded device wait (a barrier nothing completes
times out, records the error, and the context stays usable)."""
import numpy as np
import pytest
import torch

import workloads
from gpu_common import gpu_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sage():
    import quantized_attention_08_b200 as s
    s.load_library()
    return s


def test_wait_timeout_is_reported_and_context_survives(sage):
    st, _ = sage.sage_get_device_error()
    assert st == sage.SAGE_OK
    sage.sage_selftest_wait_timeout(50_000_000)  # 50 ms
    st, word = sage.sage_get_device_error()
    assert st == sage.SAGE_ERR_DEVICE_TIMEOUT
    assert word & 1 and (word >> 8) & 0xFF == 0xEE
    # cleared after reading, and the GPU still computes correct results
    st, _ = sage.sage_get_device_error()
    assert st == sage.SAGE_OK
    w = workloads.get("small_b_n256_d64")
    q, k, v = workloads.generate(w)
    o = gpu_forward(sage, q, k, v, causal=True, sm_scale=w.scale, variant="B")
    assert np.array_equal(o[0, 0, 0], v[0, 0, 0])


def test_empty_inputs_are_noops(sage):
    q = torch.empty(0, 2, 128, 64, dtype=torch.float16, device="cuda")
    o = sage.sage_attn_fwd(q, q, q)
    assert o.shape == q.shape
    q = torch.empty(1, 2, 0, 64, dtype=torch.float16, device="cuda")
    sage.sage_attn_fwd(q, q, q, variant="8+8")


def test_bad_arguments_raise(sage):
    q = torch.zeros(1, 2, 128, 96, dtype=torch.float16, device="cuda")
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd(q, q, q)
    assert e.value.status == 2
    q = torch.zeros(1, 3, 128, 64, dtype=torch.float16, device="cuda")
    k = torch.zeros(1, 2, 128, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd(q, k, k)
    assert e.value.status == 2
    base = torch.zeros(2 * 128 * 64 + 8, dtype=torch.float16, device="cuda")
    mis = base[4:4 + 2 * 128 * 64].view(1, 2, 128, 64)  # 8-byte offset
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd(mis, mis, mis)
    assert e.value.status == 3
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    ok = torch.zeros(1, 2, 128, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd_ws(ok, ok, ok, ws)
    assert e.value.status == 7
