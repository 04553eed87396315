"""Helpers shared by the GPU parity tests (inputs come from `workloads`,
expected values from `oracle`; the CUDA path is reached only through the
C-ABI binding)."""
import json
import os

import numpy as np
import torch

import oracle
import workloads

TOL_B = 2e-3  # max |O_gpu - O_mirror| on fp16 outputs of unit-variance data

# Relative bound on how far the kernel's fp32 P~ may sit from the oracle's:
# the kernel forms x = acc*c + bias with c = fl(fl(dq*log2 e)*dk) (two fp32
# roundings and one fused multiply-add, |x| up to ~100) and evaluates 2^x with
# ex2.approx.ftz.f32 (relative error below 2^-22); the oracle rounds
# S = fl(fl(acc)*fl(dq*dk)) and takes exp(S - m) in fp64.  Together these stay
# well below 2^-14.  An operand code (fp16 or E4M3 of P~) whose exact value
# lies within this band of a rounding midpoint may legitimately go either
# way; the oracle reports the effect of every such element as slack.
EPS_P = 2.0 ** -14


def to_dev(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


def rows_of(N, q_blocks):
    if q_blocks is None:
        return np.arange(N)
    return np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in q_blocks])


def gpu_forward(sage, q, k, v, *, causal, sm_scale, variant):
    tq, tk, tv = to_dev(q, k, v)
    o = sage.sage_attn_fwd(tq, tk, tv, causal=causal, sm_scale=sm_scale, variant=variant)
    st, word = sage.sage_get_device_error()
    assert st == 0, f"device error word {word:#x}"
    return o.cpu().numpy()


def compare_attention(sage, w, variant, q_blocks=None, inputs=None, check_truth=True):
    """Run the GPU forward and the oracle on the same inputs; assert
    criterion (b) against the quantized mirror and report criterion (c)
    against fp64 attention.  Returns a dict of the measured numbers."""
    q, k, v = inputs if inputs is not None else workloads.generate(w)
    o_gpu = gpu_forward(sage, q, k, v, causal=w.causal, sm_scale=w.scale, variant=variant)
    rows = rows_of(w.N, q_blocks)
    o_gpu = o_gpu[:, :, rows]
    # the narrowed 8+8 ranges (P_r = 56, V_r = 9) are the oracle's 8+8 with those ranges
    ranges = dict(variant="8+8", v_r=9.0, p_r=56.0) if variant == "8+8-r56" else dict(variant=variant)
    mirror, inter = oracle.sage_attention(q, k, v, causal=w.causal, sm_scale=w.scale,
                                          q_blocks=q_blocks, ambiguity=EPS_P, **ranges)
    slack = inter["slack"]
    assert np.all(np.isfinite(o_gpu))
    err = np.abs(o_gpu.astype(np.float64) - mirror.astype(np.float64))
    out = {"max_err_vs_mirror": float(err.max()), "max_slack": float(slack.max()),
           "max_excess": float((err - slack).max())}
    if check_truth:
        ref = oracle.attention_reference(q, k, v, causal=w.causal, sm_scale=w.scale,
                                         q_blocks=q_blocks)
        out["cossim"] = oracle.cossim(o_gpu, ref)
        out["rel_l1"] = oracle.rel_l1(o_gpu, ref)
        out["mirror_rel_l1"] = oracle.rel_l1(mirror, ref)
    log = os.environ.get("SAGE_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"workload": w.name, "variant": variant, "B": w.B, "H": w.H,
                                "H_kv": w.H_kv, "N": w.N, "d": w.d, "causal": w.causal,
                                "q_blocks": q_blocks, **out}) + "\n")
    # criterion (b): within 2e-3 of the mirror, plus the effect of the
    # operand codes that are ambiguous at the kernel's exp precision
    assert np.all(err <= TOL_B + slack), out
    return out
