"""GPU parity of the pre-pass: bit-exact q_hat, k_hat, delta_q, delta_k,
mean_k, v_hat and delta_v against the oracle on every workload shape,
including ragged sequences and degenerate blocks."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sage():
    import quantized_attention_08_b200 as s
    s.load_library()
    return s


def _bits(x):
    return np.ascontiguousarray(x).view(np.uint32)


def check_prepass(sage, q, k, v, sm_scale, with_v=True):
    tq, tk, tv = to_dev(q, k, v)
    qh, kh, dq, dk, mk = sage.sage_smooth_quant_qk(tq, tk, sm_scale)
    torch.cuda.synchronize()
    eq, edq = oracle.quant_q(q, sm_scale)
    ekh, edk, emk = oracle.smooth_quant_k(k)
    assert np.array_equal(_bits(mk.cpu().numpy()), _bits(emk)), "mean_k"
    assert np.array_equal(_bits(dq.cpu().numpy()), _bits(edq)), "delta_q"
    assert np.array_equal(_bits(dk.cpu().numpy()), _bits(edk)), "delta_k"
    assert np.array_equal(qh.cpu().numpy(), eq), "q_hat"
    assert np.array_equal(kh.cpu().numpy(), ekh), "k_hat"
    if with_v:
        vh, dv = sage.sage_quant_v_fp8(tv, 448.0)
        torch.cuda.synchronize()
        evh, edv = oracle.quant_v_fp8(v, 448.0)
        assert np.array_equal(_bits(dv.cpu().numpy()), _bits(edv)), "delta_v"
        assert np.array_equal(vh.cpu().numpy(), evh), "v_hat"
        vh9, dv9 = sage.sage_quant_v_fp8(tv, 9.0)
        evh9, edv9 = oracle.quant_v_fp8(v, 9.0)
        assert np.array_equal(_bits(dv9.cpu().numpy()), _bits(edv9)), "delta_v (V_r=9)"
        assert np.array_equal(vh9.cpu().numpy(), evh9), "v_hat (V_r=9)"
        # the combined three-launch pre-pass gives the same bits
        cq, ck, cdq, cdk, cmk, cvh, cdv = sage.sage_smooth_quant_qkv(tq, tk, tv, sm_scale, 448.0)
        for got, exp in ((cq, eq), (ck, ekh), (cvh, evh)):
            assert np.array_equal(got.cpu().numpy(), exp)
        for got, exp in ((cdq, edq), (cdk, edk), (cmk, emk), (cdv, edv)):
            assert np.array_equal(_bits(got.cpu().numpy()), _bits(exp))


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_prepass_bit_exact_workloads(sage, name):
    w = workloads.get(name)
    q, k, v = workloads.generate(w)
    check_prepass(sage, q, k, v, w.scale)


@pytest.mark.parametrize("N,d", [(1, 64), (127, 128), (129, 64), (300, 128), (1000, 64)])
def test_prepass_bit_exact_ragged(sage, N, d):
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=2, H=4, H_kv=2, N=N, d=d, seed=N + d)
    q, k, v = workloads.generate(w)
    check_prepass(sage, q, k, v, 1.0 / np.sqrt(d))


def test_prepass_sweep_points(sage):
    for w in workloads.sweep_workloads()[::5]:
        w = w.with_(B=min(w.B, 2))
        q, k, v = workloads.generate(w)
        check_prepass(sage, q, k, v, w.scale)


def test_prepass_degenerate_blocks(sage):
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 2, 384, 64)).astype(np.float16)
    q[:, :, 128:256] = 0                      # all-zero Q block -> delta 0, codes 0
    k = np.broadcast_to(rng.standard_normal((1, 2, 1, 64)).astype(np.float16), (1, 2, 384, 64)).copy()
    v = rng.standard_normal((1, 2, 384, 64)).astype(np.float16)
    v[..., 5] = 0                             # zero V column -> delta_v 0
    v[..., 7] = 60000.0                       # large magnitudes
    v[0, 0, 3, :] = -0.0                      # signed zeros keep their E4M3 sign bit
    k[0, 1, :, 3] = -65504.0                  # extreme fp16 values in the exact mean
    check_prepass(sage, q, k, v, 0.125)
