"""GPU parity of the whole forward pass against the oracle.

(b) max |O_gpu - O_mirror| <= 2e-3 element by element (the quantized mirror
    follows Algorithm 1 step by step on the same inputs);
(c) cosine similarity >= 0.998 against fp64 attention; relative L1 <= 0.02
    wherever the method itself (the mirror, no GPU involved) meets it.  8+8
    on unit-variance data, and variant B on the video-DiT inputs, sit above
    0.02 in the mirror already; there the GPU must match the mirror's own
    relative L1 within 10%.
Small cases compare every output; full-size workloads compare sampled q
blocks (each computed by the oracle against all keys)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import EPS_P, compare_attention, gpu_forward, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sage():
    import quantized_attention_08_b200 as s
    s.load_library()
    return s


def _truth_checks(r, variant):
    assert r["cossim"] >= 0.998, r
    # Rel-L1 <= 0.02 where the method itself (the quantized mirror, no GPU)
    # meets it; where it does not (8+8 on unit-variance data; variant B on
    # the video-DiT inputs, mirror 0.022), the GPU is held to the mirror's
    # own value within 10%
    assert r["rel_l1"] <= max(0.02, 1.1 * r["mirror_rel_l1"] + 1e-3), r
    if variant == "B" and r["mirror_rel_l1"] <= 0.02:
        assert r["rel_l1"] <= 0.02, r


@pytest.mark.parametrize("variant", ["B", "8+8"])
def test_small_workload(sage, variant):
    w = workloads.get("small_b_n256_d64")
    _truth_checks(compare_attention(sage, w, variant), variant)


CASES = [
    # (H, H_kv, N, d, causal)
    (2, 2, 128, 64, False),
    (2, 2, 128, 128, True),
    (4, 2, 300, 128, False),
    (4, 2, 300, 128, True),
    (4, 1, 129, 64, True),
    (2, 2, 1000, 64, False),
    (3, 3, 640, 128, True),
    (2, 1, 1, 64, False),
    (2, 1, 1, 128, True),
    (2, 2, 385, 64, True),
]


@pytest.mark.parametrize("variant", ["B", "8+8"])
@pytest.mark.parametrize("H,Hk,N,d,causal", CASES)
def test_ragged_gqa_causal(sage, variant, H, Hk, N, d, causal):
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(
        B=2, H=H, H_kv=Hk, N=N, d=d, causal=causal, seed=N * 7 + d + H)
    compare_attention(sage, w, variant, check_truth=False)


@pytest.mark.parametrize("variant", ["B", "8+8"])
def test_quantized_entry_point_on_oracle_operands(sage, variant):
    """sage_attn_fwd_quantized fed the oracle's own quantized operands."""
    w = workloads.get("prefill_gqa_causal_h32_kv8_n8192_d128").with_(H=4, H_kv=2, N=700)
    q, k, v = workloads.generate(w)
    qh, dq = oracle.quant_q(q, w.scale)
    kh, dk, _ = oracle.smooth_quant_k(k)
    if variant == "B":
        vop, dv, vin = v, None, v
        mirror = oracle.attention_online(qh, kh, dq, dk, v, causal=True, operand="fp16",
                                         ambiguity=EPS_P)
    else:
        vin, dv = oracle.quant_v_fp8(v)
        mirror = oracle.attention_online(qh, kh, dq, dk, oracle.e4m3_decode(vin), causal=True,
                                         operand="e4m3", dv=dv, ambiguity=EPS_P)
    tqh, tkh, tdq, tdk, tv = to_dev(qh, kh, dq, dk, vin)
    tdv = to_dev(dv)[0] if dv is not None else None
    o = sage.sage_attn_fwd_quantized(tqh, tkh, tdq, tdk, tv, tdv, causal=True, variant=variant)
    o = o.cpu().numpy()
    mirror, slack = mirror[0], mirror[1]["slack"]
    assert np.all(np.abs(o.astype(np.float64) - mirror.astype(np.float64)) <= 2e-3 + slack)


@pytest.mark.parametrize("variant", ["B", "8+8"])
def test_degenerate_inputs(sage, variant):
    """Q = 0 (uniform weights: column mean of V) and identical keys."""
    N = 300
    w = workloads.get("small_b_n256_d64").with_(N=N)
    _, k, v = workloads.generate(w)
    q = np.zeros((1, 2, N, 64), np.float16)
    compare_attention(sage, w, variant, inputs=(q, k, v), check_truth=False)
    q2, _, _ = workloads.generate(w)
    k2 = np.broadcast_to(k[:, :, :1], k.shape).copy()
    compare_attention(sage, w, variant, inputs=(q2, k2, v), check_truth=False)


def test_causal_first_row_equals_first_value_row(sage):
    w = workloads.get("prefill_gqa_causal_h32_kv8_n8192_d128").with_(H=4, H_kv=2, N=256)
    q, k, v = workloads.generate(w)
    o = gpu_forward(sage, q, k, v, causal=True, sm_scale=w.scale, variant="B")
    for h in range(4):
        assert np.array_equal(o[0, h, 0], v[0, h // 2, 0])


def test_workspace_and_host_entry_points_agree(sage):
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=1, H=4, H_kv=2, N=513)
    q, k, v = workloads.generate(w)
    tq, tk, tv = to_dev(q, k, v)
    for variant in ("B", "8+8"):
        o1 = sage.sage_attn_fwd(tq, tk, tv, causal=False, variant=variant)
        nbytes = sage.sage_attn_workspace_bytes(1, 4, 2, 513, 128, variant)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        o2 = sage.sage_attn_fwd_ws(tq, tk, tv, ws, causal=False, variant=variant)
        hq, hk, hv = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
        ho = torch.empty(hq.shape, dtype=torch.float16).pin_memory()
        sage.sage_attn_fwd_host(hq, hk, hv, ho, causal=False, variant=variant)
        assert torch.equal(o1, o2)
        assert torch.equal(o1.cpu(), ho)


@pytest.mark.parametrize("shape", [(2, 8, 2, 333, True), (3, 6, 3, 200, False), (1, 24, 24, 130, False)],
                         ids=["gqa_causal_4units", "9units_5chunks_early_break", "24units"])
def test_host_pipeline_equals_device_path(sage, shape):
    """sage_attn_fwd_host splits the (batch, kv head) units into chunks whose
    copies overlap the kernels; the output is sage_attn_fwd's, bit for bit."""
    B, H, Hk, N, causal = shape
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=B, H=H, H_kv=Hk, N=N, d=64,
                                                        causal=causal, seed=900 + N)
    q, k, v = workloads.generate(w)
    tq, tk, tv = to_dev(q, k, v)
    hq, hk, hv = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    for variant in ("B", "8+8", "8+8-r56"):
        o1 = sage.sage_attn_fwd(tq, tk, tv, causal=causal, variant=variant)
        ho = torch.empty(hq.shape, dtype=torch.float16).pin_memory()
        sage.sage_attn_fwd_host(hq, hk, hv, ho, causal=causal, variant=variant)
        assert torch.equal(o1.cpu(), ho), variant
    # pageable host memory works too
    ho = torch.empty(q.shape, dtype=torch.float16)
    sage.sage_attn_fwd_host(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), ho,
                            causal=causal, variant="8+8")
    assert torch.equal(sage.sage_attn_fwd(tq, tk, tv, causal=causal, variant="8+8").cpu(), ho)


def test_host_path_concurrent_calls(sage):
    """Two host threads call sage_attn_fwd_host at once on the same device:
    one uses the device's cached side streams, the other its own; both
    outputs equal the device path's, call after call."""
    import threading
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=2, H=4, H_kv=2, N=700, seed=61)
    q, k, v = workloads.generate(w)
    tq, tk, tv = to_dev(q, k, v)
    ref = sage.sage_attn_fwd(tq, tk, tv, causal=False, variant="8+8").cpu()
    hq, hk, hv = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    outs = [torch.empty(hq.shape, dtype=torch.float16).pin_memory() for _ in range(2)]
    errors = []

    def run(i):
        try:
            torch.cuda.set_device(0)
            for _ in range(6):
                outs[i].zero_()
                sage.sage_attn_fwd_host(hq, hk, hv, outs[i], causal=False, variant="8+8")
                if not torch.equal(outs[i], ref):
                    errors.append(i)
        except Exception as ex:  # surfaced below
            errors.append(repr(ex))

    threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads)
    assert not errors, errors


def test_repeated_calls_are_deterministic(sage):
    w = workloads.get("prefill_gqa_causal_h32_kv8_n8192_d128").with_(H=8, H_kv=2, N=2048)
    q, k, v = workloads.generate(w)
    a = gpu_forward(sage, q, k, v, causal=True, sm_scale=w.scale, variant="8+8")
    b = gpu_forward(sage, q, k, v, causal=True, sm_scale=w.scale, variant="8+8")
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- full-size workloads
# q blocks sampled per workload (each computed by the oracle against all
# keys) and the variants run there: the workload's own, and variant B on the
# video-DiT shape too (the path the bench also times there).
SAMPLED = {
    "llm_8p8_b2_h16_n4096_d128": ([0, 13, 31], ("8+8",)),
    "prefill_gqa_causal_h32_kv8_n8192_d128": ([0, 1, 40, 63], ("B", "8+8")),
    "video_dit_h24_n32768_d128": ([0, 101, 255], ("8+8", "B")),
}


@pytest.mark.parametrize("name", list(SAMPLED))
def test_full_size_workloads_sampled(sage, name):
    w = workloads.get(name)
    inputs = workloads.generate(w)
    blocks, variants = SAMPLED[name]
    for variant in variants:
        r = compare_attention(sage, w, variant, q_blocks=blocks, inputs=inputs)
        _truth_checks(r, variant)


@pytest.mark.parametrize("idx", [0, 3, 9, 13, 18, 23])
def test_sweep_points_sampled(sage, idx):
    w = workloads.sweep_workloads()[idx]
    w = w.with_(B=min(w.B, 4))
    nqb = (w.N + 127) // 128
    inputs = workloads.generate(w)
    for variant in w.variants:
        compare_attention(sage, w, variant, q_blocks=[0, nqb // 2, nqb - 1], inputs=inputs)
