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

# Relative bound EPS_P on how far the kernel's fp32 P~ may sit from the
# oracle's, for the elements whose operand code can be non-zero (exponent
# e = (acc - acc_max) * dq * dk * log2 e >= -25 in log2 units).  With m the
# row max of S in log2 units and every fp32 operation rounded once:
#   kernel: c = fl(fl(dq * fl(log2 e)) * dk) is within 3 * 2^-24 of its exact
#     value; x = fl(acc * c + bias) with bias = -fl(acc_max * c) (8+8: plus
#     log2 P_r, rounded once) differs from e by at most
#     2^-24 * (3|e| + |m| + |x| + |m| + 9);  p = 2^x by ex2.approx.f32 or
#     the FMA-pipe polynomial, each within 2^-21.9 relative;
#   oracle: S = fl(acc * fl(dq * dk)), m_o = max S, p = fl32(exp(S - m_o)):
#     at most 2^-24 * (2|e| + 2|m|) in the exponent and 2^-24 in the result.
# Relative difference <= ln2 * 2^-24 * (5|e| + 4|m| + |x| + 9) + 2^-21.9 + 2^-24,
# with |e|, |x| <= 25: <= 2^-16 whenever |m| <= 50 (log2 units), i.e. a max
# logit below 35 in natural units -- compare_attention checks that bound on
# the oracle's row maxima.  An operand code (fp16 or E4M3 of P~) whose exact
# value lies within this band of a rounding midpoint may legitimately go
# either way; the oracle reports the effect of every such element as slack.
EPS_P = 2.0 ** -16
M_MAX_NATURAL = 35.0  # largest |row max of S| for which EPS_P holds
# criterion (b) may lean on the slack for at most this fraction of outputs
MAX_SLACK_FRACTION = 1e-4


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
    m_max = float(np.abs(inter["m"]).max())
    assert np.all(np.isfinite(o_gpu))
    err = np.abs(o_gpu.astype(np.float64) - mirror.astype(np.float64))
    over = err > TOL_B
    out = {"max_err_vs_mirror": float(err.max()), "max_slack": float(slack.max()),
           "slack_p999": float(np.quantile(slack, 0.999)), "max_excess": float((err - slack).max()),
           "n_over_tol": int(over.sum()), "frac_over_tol": float(over.mean()),
           "max_row_max_natural": m_max, "eps_p_log2": float(np.log2(EPS_P))}
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
    # the derivation of EPS_P assumes row maxima below M_MAX_NATURAL
    assert m_max <= M_MAX_NATURAL, out
    # criterion (b): within 2e-3 of the mirror, plus the effect of the
    # operand codes that are ambiguous at the kernel's exp precision ...
    assert np.all(err <= TOL_B + slack), out
    # ... which only a vanishing fraction of the outputs may need
    assert over.mean() <= MAX_SLACK_FRACTION, out
    return out
