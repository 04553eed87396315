"""Helpers shared by the GPU parity tests (inputs come from `workloads`,
expected values from `oracle`; the CUDA path is reached only through the
C-ABI binding)."""
import numpy as np
import torch

import oracle
import workloads

TOL_B = 2e-3  # max |O_gpu - O_mirror| on fp16 outputs of unit-variance data


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
    mirror, _ = oracle.sage_attention(q, k, v, causal=w.causal, sm_scale=w.scale,
                                      variant=variant, q_blocks=q_blocks)
    assert np.all(np.isfinite(o_gpu))
    err = np.abs(o_gpu.astype(np.float64) - mirror.astype(np.float64))
    out = {"max_err_vs_mirror": float(err.max())}
    if check_truth:
        ref = oracle.attention_reference(q, k, v, causal=w.causal, sm_scale=w.scale,
                                         q_blocks=q_blocks)
        out["cossim"] = oracle.cossim(o_gpu, ref)
        out["rel_l1"] = oracle.rel_l1(o_gpu, ref)
        out["mirror_rel_l1"] = oracle.rel_l1(mirror, ref)
    assert out["max_err_vs_mirror"] <= TOL_B, out
    return out
