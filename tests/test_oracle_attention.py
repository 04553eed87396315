"""Pins for the oracle's attention (CPU only).

The truth (mode R) is checked against pure-Python loops and against torch's
fp64 scaled_dot_product_attention (a library routine); the online tiled
mirror is pinned to R through exact special cases (identity quantizers,
random per-block scales), the Smooth-K shift invariance, closed-form
special cases and the invariants the pages state."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float16)


def _brute(q, k, v, causal, scale):
    B, H, N, d = q.shape
    Hk = k.shape[1]
    out = np.zeros(q.shape)
    for b in range(B):
        for h in range(H):
            hk = h * Hk // H
            for r in range(N):
                s = [scale * sum(float(q[b, h, r, c]) * float(k[b, hk, t, c]) for c in range(d))
                     for t in range(N)]
                keys = [t for t in range(N) if not causal or t <= r]
                mx = max(s[t] for t in keys)
                w = {t: math.exp(s[t] - mx) for t in keys}
                z = sum(w.values())
                for c in range(d):
                    out[b, h, r, c] = sum(w[t] * float(v[b, hk, t, c]) for t in keys) / z
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_reference_matches_pure_python(causal):
    q, k, v = _rand((1, 2, 6, 3), 1), _rand((1, 1, 6, 3), 2, 2.0), _rand((1, 1, 6, 3), 3)
    r = oracle.attention_reference(q, k, v, causal=causal, sm_scale=0.7)
    assert np.allclose(r, _brute(q, k, v, causal, 0.7), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_reference_matches_torch_sdpa_fp64(causal):
    q, k, v = _rand((2, 4, 200, 64), 4), _rand((2, 2, 200, 64), 5, 3.0), _rand((2, 2, 200, 64), 6)
    r = oracle.attention_reference(q, k, v, causal=causal, sm_scale=0.125)
    tq = torch.from_numpy(q.astype(np.float64))
    tk = torch.from_numpy(k.astype(np.float64)).repeat_interleave(2, dim=1)
    tv = torch.from_numpy(v.astype(np.float64)).repeat_interleave(2, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.125)
    assert np.allclose(r, ref.numpy(), rtol=0, atol=1e-12)


def test_smooth_k_shift_invariance_small():
    w = workloads.get("small_b_n256_d64")
    q, k, v = workloads.generate(w)
    r = oracle.attention_reference(q, k, v, causal=False, sm_scale=w.scale)
    rs = oracle.attention_reference(q, k, v, causal=False, sm_scale=w.scale, smooth_k=True)
    assert np.abs(r - rs).max() <= 1e-12


def test_smooth_k_shift_invariance_sampled_rows_causal_gqa():
    w = workloads.get("prefill_gqa_causal_h32_kv8_n8192_d128").with_(H=4, H_kv=1, N=1024)
    q, k, v = workloads.generate(w)
    blocks = [0, 3, 7]
    r = oracle.attention_reference(q, k, v, causal=True, sm_scale=w.scale, q_blocks=blocks)
    rs = oracle.attention_reference(q, k, v, causal=True, sm_scale=w.scale, q_blocks=blocks, smooth_k=True)
    assert np.abs(r - rs).max() <= 1e-12


def _nb(N):
    return (N + 127) // 128


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 300, 513])
def test_online_tiling_exact_equals_reference(causal, N):
    """Identity quantizers and fp64 S: Algorithm 1 must reproduce the
    textbook softmax exactly (up to fp64 rounding), whatever the tiling."""
    q, k, v = _rand((1, 4, N, 32), 10 + N), _rand((1, 2, N, 32), 20 + N, 2.0), _rand((1, 2, N, 32), 30 + N)
    scale = 0.2
    r = oracle.attention_reference(q, k, v, causal=causal, sm_scale=scale)
    ones_q = np.ones((1, 4, _nb(N)))
    ones_k = np.ones((1, 2, _nb(N)))
    o = oracle.attention_online(q.astype(np.float64) * scale, k.astype(np.float64), ones_q, ones_k,
                                v.astype(np.float64), causal=causal, operand="exact",
                                s_fp32=False, out_fp16=False)
    assert np.abs(o - r).max() <= 1e-12


def test_online_uses_the_right_block_scales():
    """Random per-block scales folded into the operands must cancel exactly:
    a wrong q- or kv-block index in the dequantization would not cancel."""
    N = 400
    q, k, v = _rand((1, 2, N, 16), 1), _rand((1, 1, N, 16), 2), _rand((1, 1, N, 16), 3)
    rng = np.random.default_rng(9)
    sq = rng.uniform(0.5, 4, (1, 2, _nb(N)))
    sk = rng.uniform(0.5, 4, (1, 1, _nb(N)))
    rq = np.repeat(sq, 128, axis=2)[:, :, :N, None]
    rk = np.repeat(sk, 128, axis=2)[:, :, :N, None]
    for causal in (False, True):
        r = oracle.attention_reference(q, k, v, causal=causal, sm_scale=0.3)
        o = oracle.attention_online(q.astype(np.float64) * 0.3 / rq, k.astype(np.float64) / rk, sq, sk,
                                    v.astype(np.float64), causal=causal, operand="exact",
                                    s_fp32=False, out_fp16=False)
        assert np.abs(o - r).max() <= 1e-12


@pytest.mark.parametrize("variant", ["B", "8+8"])
def test_causal_row0_is_v0(variant):
    w = workloads.get("prefill_gqa_causal_h32_kv8_n8192_d128").with_(H=2, H_kv=1, N=256)
    q, k, v = workloads.generate(w)
    o, inter = oracle.sage_attention(q, k, v, causal=True, variant=variant)
    if variant == "B":
        assert np.array_equal(o[0, :, 0], np.broadcast_to(v[0, 0, 0], o[0, :, 0].shape))
    else:
        deq = oracle.e4m3_decode(inter["v_hat"][0, 0, 0]) * inter["delta_v"][0, 0]
        assert np.abs(o[0, :, 0].astype(np.float64) - deq).max() <= np.abs(deq).max() * 2.0 ** -10


@pytest.mark.parametrize("variant", ["B", "8+8"])
def test_zero_q_gives_column_mean(variant):
    N = 300
    q = np.zeros((1, 1, N, 64), np.float16)
    _, k, v = workloads.generate(workloads.get("small_b_n256_d64").with_(N=N, H=1, H_kv=1))
    o, inter = oracle.sage_attention(q, k, v, causal=False, variant=variant)
    assert np.all(inter["delta_q"] == 0)
    if variant == "B":
        mean = v.astype(np.float64).mean(axis=2)
    else:
        mean = (oracle.e4m3_decode(inter["v_hat"]) * inter["delta_v"][:, :, None, :]).mean(axis=2)
    assert np.array_equal(o[0, 0], np.broadcast_to(oracle.fp16_rne(mean[0, 0]), o[0, 0].shape))


def test_identical_keys_smooth_to_zero():
    N = 256
    q, _, v = workloads.generate(workloads.get("small_b_n256_d64"))
    k = np.broadcast_to(_rand((1, 2, 1, 64), 4, 5.0), (1, 2, N, 64)).copy()
    o, inter = oracle.sage_attention(q, k, v, causal=False, variant="B")
    assert np.all(inter["k_hat"] == 0) and np.all(inter["delta_k"] == 0)
    mean = v.astype(np.float64).mean(axis=2)
    assert np.array_equal(o, np.broadcast_to(oracle.fp16_rne(mean)[:, :, None, :], o.shape))


def test_rowmax_p_tilde_invariant():
    """max P~ <= 1 in every tile, and == 1 where the running max moved
    (always in a row's first tile): the static P~ scale of the pages."""
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=1, H=2, H_kv=2, N=640)
    q, k, v = workloads.generate(w)
    qh, dq = oracle.quant_q(q, w.scale)
    kh, dk, _ = oracle.smooth_quant_k(k)
    for causal in (False, True):
        _, st = oracle.attention_online(qh, kh, dq, dk, v, causal=causal, operand="fp16",
                                        return_stats=True)
        for j, pmax, moved in st["tiles"]:
            assert np.all(pmax <= 1.0)
            assert np.all(pmax[moved] == 1.0)
            if j == 0:
                assert np.all(moved)


def _golden(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].split()
        if line:
            out.setdefault(line[0], []).append(line[1:])
    return out


def test_fp16_accumulator_bound_against_page_values():
    g = _golden("sa2pp_fp16_accumulator.txt")
    n = int(g["products_per_mma"][0][0])
    assert oracle.FP16_MAX == float(g["fp16_max"][0][0])
    assert oracle.f16acc_product_limit(n) == float(g["product_limit"][0][0])
    p, vv = map(float, g["example_p_v"][0])
    assert oracle.f16acc_bound_ok(p, vv, n)
    fits = {}
    for p_r, v_r, who in g["table2_pair"]:
        fits[(float(p_r), float(v_r))] = oracle.f16acc_bound_ok(float(p_r), float(v_r), n)
    assert fits == {(448.0, 448.0): False, (112.0, 4.5): True, (56.0, 9.0): True}
    # a 128-wide kv tile summed in one FP16 accumulator: (56, 9) still fits
    assert oracle.f16acc_bound_ok(56.0, 9.0, 128) and not oracle.f16acc_bound_ok(112.0, 9.0, 128)
    # all of 448, 112, 56, 9 and 4.5 are exact E4M3 values
    for x in (448.0, 112.0, 56.0, 9.0, 4.5):
        assert oracle.e4m3_round(np.array([x]))[0] == x


def test_static_scales_golden():
    g = _golden("sa1_static_scales.txt")
    assert float(g["e4m3_max"][0][0]) == oracle.E4M3_MAX
    x = np.random.default_rng(1).standard_normal((1, 1, 128, 64)).astype(np.float32)
    xh, _ = oracle.quant_blocks(x)
    assert np.abs(xh.astype(int)).max() == int(g["int8_qmax"][0][0])


def test_f16acc_simulation_flags_overflow_only_for_wide_ranges():
    """Adversarial tile: every key identical and every V at its column max,
    so all P_hat = P_r and all V_hat = V_r."""
    N, d = 128, 64
    q = np.zeros((1, 1, N, d), np.float16)
    k = np.zeros((1, 1, N, d), np.float16)
    v = np.full((1, 1, N, d), 1.0, np.float16)
    _, inter = oracle.sage_attention(q, k, v, causal=False, variant="8+8", v_r=448.0, p_r=448.0,
                                     simulate_f16acc=True)
    assert inter["f16acc_overflow"]
    o, inter = oracle.sage_attention(q, k, v, causal=False, variant="8+8", v_r=9.0, p_r=56.0,
                                     simulate_f16acc=True)
    assert not inter["f16acc_overflow"]
    assert np.all(o == 1.0)


def test_metric_definitions():
    a = np.random.default_rng(0).standard_normal(1000)
    assert oracle.cossim(a, a) == pytest.approx(1.0)
    assert oracle.cossim(3 * a, a) == pytest.approx(1.0)
    assert oracle.cossim(-a, a) == pytest.approx(-1.0)
    assert oracle.rel_l1(a, a) == 0.0
    assert oracle.rel_l1(1.1 * a, a) == pytest.approx(0.1)
    assert oracle.rmse(a + 0.5, a) == pytest.approx(0.5)


@pytest.mark.parametrize("variant", ["B", "8+8"])
def test_quantized_mirror_accuracy_small(variant):
    """Context, not a pin: the accuracy level of the method on the small
    workload (the pages' Table 2 reports CosSim 99.99% / L1 0.0116 for
    INT8+FP16 and 99.94% / 0.0345 for INT8+E4M3 on real layers)."""
    w = workloads.get("small_b_n256_d64")
    q, k, v = workloads.generate(w)
    o, _ = oracle.sage_attention(q, k, v, causal=False, variant=variant)
    r = oracle.attention_reference(q, k, v, causal=False, sm_scale=w.scale)
    assert oracle.cossim(o, r) >= 0.998
    if variant == "B":
        assert oracle.rel_l1(o, r) <= 0.02
    else:
        assert oracle.rel_l1(o, r) <= 0.05


@pytest.mark.parametrize("variant", ["B", "8+8"])
def test_ambiguity_slack_bounds_the_flips(variant):
    """The slack is zero without a band, and bounds the change of the output
    when every ambiguous operand code takes its other value."""
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=1, H=2, H_kv=1, N=700, causal=True)
    q, k, v = workloads.generate(w)
    o0, i0 = oracle.sage_attention(q, k, v, causal=True, variant=variant, ambiguity=0.0,
                                   simulate_f16acc=False)
    assert "slack" not in i0
    eps = 2.0 ** -9   # wide band, so that many codes are ambiguous
    o1, i1 = oracle.sage_attention(q, k, v, causal=True, variant=variant, ambiguity=eps)
    assert np.array_equal(o0, o1)
    slack = i1["slack"]
    assert np.all(slack >= 0) and slack.max() > 0
    of, _ = oracle.sage_attention(q, k, v, causal=True, variant=variant, ambiguity=eps,
                                  flip_ambiguous=True)
    diff = np.abs(of.astype(np.float64) - o0.astype(np.float64))
    # both outputs are rounded to fp16: half an ulp each, at most one ulp of the larger
    big = np.maximum(np.abs(o0), np.abs(of)).astype(np.float16)
    ulp = np.spacing(big).astype(np.float64)
    assert np.all(diff <= slack + ulp)
    assert diff.max() > 0
