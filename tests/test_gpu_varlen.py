"""GPU parity of packed variable-length batches (sequences of different
lengths along the token axis, [H, T, d], cu_seqlens on the device) against
the oracle's per-sequence mirror.

  * the pre-pass is bit-exact, sequence by sequence, against the oracle's
    quantizers applied to that sequence alone;
  * the output meets criterion (b) against the oracle's varlen mirror (same
    tolerance and ambiguity slack as the fixed-length tests);
  * a batch of equal lengths equals the fixed-length entry point bit for bit;
  * lengths of the SageAttention review's Table 7 models (N = 17776,
    N = 1105) mixed with short and empty sequences."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import EPS_P, M_MAX_NATURAL, MAX_SLACK_FRACTION, TOL_B, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sage():
    import quantized_attention_08_b200 as s
    s.load_library()
    return s


def packed_inputs(lens, H, Hk, d, seed):
    """Seeded packed q [H,T,d], k, v [H_kv,T,d] with the 8+8 LLM workload's
    recipe, each sequence drawn as its own B=1 workload (so sequences differ
    in their K bias)."""
    qs, ks, vs = [], [], []
    for i, n in enumerate(lens):
        w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=1, H=H, H_kv=Hk, N=max(n, 1), d=d,
                                                            seed=seed + i)
        q, k, v = workloads.generate(w)
        qs.append(q[0, :, :n]), ks.append(k[0, :, :n]), vs.append(v[0, :, :n])
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return (np.ascontiguousarray(np.concatenate(qs, axis=1)), np.ascontiguousarray(np.concatenate(ks, axis=1)),
            np.ascontiguousarray(np.concatenate(vs, axis=1)), cu)


@pytest.mark.parametrize("d", [64, 128])
def test_prepass_bit_exact_per_sequence(sage, d):
    lens = [300, 0, 129, 1, 513]
    q, k, v, cu = packed_inputs(lens, 4, 2, d, seed=40 + d)
    tq, tk, tv, tcu = to_dev(q, k, v, cu)
    scale = 1.0 / np.sqrt(d)
    qh, kh, dq, dk, mk, vh, dv = sage.sage_smooth_quant_qkv_varlen(tq, tk, tcu, max(lens), v=tv,
                                                                   sm_scale=scale)
    qh, kh, dq, dk, mk, vh, dv = (t.cpu().numpy() for t in (qh, kh, dq, dk, mk, vh, dv))
    for b, (a, e) in enumerate(zip(cu[:-1], cu[1:])):
        if a == e:
            assert np.all(mk[b] == 0) and np.all(dv[b] == 0)
            continue
        nb = (e - a + 127) // 128
        oq, odq = oracle.quant_q(q[None, :, a:e], scale)
        ok_, odk, omk = oracle.smooth_quant_k(k[None, :, a:e])
        ov, odv = oracle.quant_v_fp8(v[None, :, a:e])
        assert np.array_equal(qh[:, a:e], oq[0])
        assert np.array_equal(kh[:, a:e], ok_[0])
        assert np.array_equal(vh[:, a:e], ov[0])
        assert np.array_equal(dq[b, :, :nb].view(np.uint32), odq[0].view(np.uint32))
        assert np.array_equal(dk[b, :, :nb].view(np.uint32), odk[0].view(np.uint32))
        assert np.array_equal(mk[b].view(np.uint32), omk[0].view(np.uint32))
        assert np.array_equal(dv[b].view(np.uint32), odv[0].view(np.uint32))


def check_varlen(sage, lens, H, Hk, d, causal, variant, seed, q_blocks=None):
    q, k, v, cu = packed_inputs(lens, H, Hk, d, seed)
    tq, tk, tv, tcu = to_dev(q, k, v, cu)
    o = sage.sage_attn_fwd_varlen(tq, tk, tv, tcu, max(lens), causal=causal, variant=variant)
    st, word = sage.sage_get_device_error()
    assert st == 0, f"device error word {word:#x}"
    o = o.cpu().numpy()
    mirror, inter = oracle.sage_attention_varlen(q, k, v, cu, causal=causal, variant=variant,
                                                 q_blocks=q_blocks, ambiguity=EPS_P)
    rows = np.zeros(q.shape[1], bool)
    for b, (a, e) in enumerate(zip(cu[:-1], cu[1:])):
        if q_blocks is None:
            rows[a:e] = True
        elif b in q_blocks:
            for qb in q_blocks[b]:
                rows[a + qb * 128:min(e, a + qb * 128 + 128)] = True
    assert np.all(np.isfinite(o[:, rows]))
    err = np.abs(o[:, rows].astype(np.float64) - mirror[:, rows].astype(np.float64))
    slack = inter["slack"][:, rows]
    assert float(np.abs(inter["m"][:, rows]).max(initial=0.0)) <= M_MAX_NATURAL
    assert np.all(err <= TOL_B + slack), float(err.max())
    assert (err > TOL_B).mean() <= MAX_SLACK_FRACTION
    return o, mirror


@pytest.mark.parametrize("variant", ["B", "8+8"])
@pytest.mark.parametrize("causal", [False, True])
def test_mixed_lengths_small(sage, variant, causal):
    check_varlen(sage, [300, 1, 0, 129, 385], 4, 2, 64, causal, variant, seed=70)


@pytest.mark.parametrize("variant", ["B", "8+8"])
def test_table7_lengths_sampled(sage, variant):
    """N = 17776 (CogVideoX) and N = 1105 (Unidiffuser) of the review's
    Table 7, with a 129-token sequence; sampled q blocks of each against all
    of its keys."""
    lens = [17776, 1105, 129]
    blocks = {0: [0, 69, 138], 1: [0, 8], 2: [0, 1]}
    check_varlen(sage, lens, 2, 1, 128, False, variant, seed=90, q_blocks=blocks)


@pytest.mark.parametrize("variant", ["B", "8+8"])
@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_equal_fixed_length_path(sage, variant, causal):
    B, H, Hk, N, d = 3, 4, 2, 200, 128
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=B, H=H, H_kv=Hk, N=N, d=d, seed=33)
    q, k, v = workloads.generate(w)
    tq, tk, tv = to_dev(q, k, v)
    o_fix = sage.sage_attn_fwd(tq, tk, tv, causal=causal, variant=variant)
    pk = lambda x: torch.from_numpy(np.ascontiguousarray(  # noqa: E731
        x.transpose(1, 0, 2, 3).reshape(x.shape[1], B * N, d))).cuda()
    cu = torch.arange(0, B * N + 1, N, dtype=torch.int32, device="cuda")
    o_var = sage.sage_attn_fwd_varlen(pk(q), pk(k), pk(v), cu, N, causal=causal, variant=variant)
    o_var = o_var.reshape(H, B, N, d).permute(1, 0, 2, 3)
    assert torch.equal(o_fix, o_var)
