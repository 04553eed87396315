"""GPU parity of the 8+8 variant with the narrowed operand ranges P_r = 56,
V_r = 9 (the SageAttention2++ review's Eq. (2) / Table 2 pair): the same
criteria as the other variants against the oracle's 8+8 mirror run with
those ranges."""
import numpy as np
import pytest

import oracle
import workloads
from gpu_common import compare_attention

pytestmark = pytest.mark.gpu

VAR = "8+8-r56"


@pytest.fixture(scope="module")
def sage():
    import quantized_attention_08_b200 as s
    s.load_library()
    return s


def _accuracy(out):
    assert out["cossim"] >= 0.998, out
    # like 8+8, the relative L1 of E4M3 operands is a property of the method:
    # the kernel must match its mirror's
    assert out["rel_l1"] <= 1.1 * out["mirror_rel_l1"] + 1e-3, out


def test_small(sage):
    _accuracy(compare_attention(sage, workloads.get("small_b_n256_d64"), VAR))


@pytest.mark.parametrize("kw", [dict(N=300, H=4, H_kv=2), dict(N=333, causal=True, d=128),
                                dict(N=129, H=2, H_kv=1, causal=True)],
                         ids=["ragged_gqa", "ragged_causal_d128", "tail_causal_gqa"])
def test_shapes(sage, kw):
    w = workloads.get("small_b_n256_d64").with_(seed=500 + kw["N"], **kw)
    _accuracy(compare_attention(sage, w, VAR))


@pytest.mark.parametrize("name,blocks", [("llm_8p8_b2_h16_n4096_d128", [0, 13, 31]),
                                         ("prefill_gqa_causal_h32_kv8_n8192_d128", [0, 1, 40, 63]),
                                         ("video_dit_h24_n32768_d128", [0, 255])])
def test_full_size_sampled(sage, name, blocks):
    _accuracy(compare_attention(sage, workloads.get(name), VAR, q_blocks=blocks))


def test_r56_differs_from_448(sage):
    """The narrowed ranges reach the kernel: its output is not the 8+8 one."""
    import torch
    from gpu_common import gpu_forward
    w = workloads.get("small_b_n256_d64")
    q, k, v = workloads.generate(w)
    a = gpu_forward(sage, q, k, v, causal=False, sm_scale=w.scale, variant="8+8")
    b = gpu_forward(sage, q, k, v, causal=False, sm_scale=w.scale, variant=VAR)
    assert np.abs(a.astype(np.float64) - b.astype(np.float64)).max() > 0
