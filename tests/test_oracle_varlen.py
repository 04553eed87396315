"""Pins of the oracle's variable-length batch (sequences packed along the
token axis, [H, T, d]): each sequence is an independent problem.

  * a batch of equal lengths equals the fixed-length batch [B, H, N, d]
    (catches a wrong offset, a transposed layout or a shared statistic);
  * a sequence's output does not depend on the other sequences' tokens --
    not even through mean(K) or delta_V, which a smoothing over the whole
    packed batch would share;
  * empty sequences and ragged lengths are allowed."""
import numpy as np
import pytest

import oracle
import workloads


def _packed(q, k, v):
    """[B, H, N, d] -> [H, B*N, d] (sequence b at tokens b*N .. b*N+N-1)."""
    B, H, N, d = q.shape
    f = lambda x: np.ascontiguousarray(x.transpose(1, 0, 2, 3).reshape(x.shape[1], B * N, d))  # noqa: E731
    return f(q), f(k), f(v)


@pytest.mark.parametrize("variant", ["B", "8+8"])
@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_equal_the_fixed_length_batch(variant, causal):
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=3, H=4, H_kv=2, N=200, d=64,
                                                        causal=causal, seed=31)
    q, k, v = workloads.generate(w)
    o_fix, _ = oracle.sage_attention(q, k, v, causal=causal, sm_scale=w.scale, variant=variant)
    qp, kp, vp = _packed(q, k, v)
    cu = np.arange(0, 3 * 200 + 1, 200, dtype=np.int32)
    o_var, _ = oracle.sage_attention_varlen(qp, kp, vp, cu, causal=causal, sm_scale=w.scale,
                                            variant=variant)
    for b in range(3):
        assert np.array_equal(o_var[:, b * 200:(b + 1) * 200], o_fix[b])


@pytest.mark.parametrize("variant", ["B", "8+8"])
def test_sequences_are_independent(variant):
    rng = np.random.default_rng(7)
    H, Hk, d = 2, 1, 64
    lens = [129, 0, 300, 1]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q = rng.standard_normal((H, T, d)).astype(np.float16)
    k = (rng.standard_normal((Hk, T, d)) + 3.0).astype(np.float16)
    v = rng.standard_normal((Hk, T, d)).astype(np.float16)
    o, inter = oracle.sage_attention_varlen(q, k, v, cu, causal=True, variant=variant)
    # each sequence alone
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        if a == b:
            assert inter["per_sequence"][s] is None
            continue
        o1, i1 = oracle.sage_attention(q[None, :, a:b], k[None, :, a:b], v[None, :, a:b],
                                       causal=True, variant=variant)
        assert np.array_equal(o[:, a:b], o1[0])
        assert np.array_equal(inter["per_sequence"][s]["mean_k"], oracle.mean_k(k[None, :, a:b]))
    # scaling the other sequences' K and V leaves sequence 2 unchanged
    k2, v2 = k.copy(), v.copy()
    k2[:, :129] *= np.float16(4)
    v2[:, 429:] *= np.float16(8)
    o2, _ = oracle.sage_attention_varlen(q, k2, v2, cu, causal=True, variant=variant)
    assert np.array_equal(o2[:, 129:429], o[:, 129:429])
    assert not np.array_equal(o2[:, :129], o[:, :129])
