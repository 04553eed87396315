"""Pin of the quantized mirror (the oracle's Algorithm 1 with quantized
operands) against an element-by-element pure-Python restatement of the same
steps on tiny inputs, using PyTorch's fp16 / float8_e4m3fn casts (library
routines) for the operand rounding.  A transposed block scale, a wrong
tile order, a dropped rescale or a wrong operand scale would show up."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

F32 = np.float32


def _f16(x: float) -> float:
    return float(torch.tensor(x, dtype=torch.float32).to(torch.float16).item())


def _e4m3(x: float) -> float:
    # saturating E4M3 of an fp32 value (|x| <= 448 here by construction)
    return float(torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).float().item())


def loops_attention(qh, kh, dq, dk, vop, dv, causal, operand, p_r):
    B, H, N, d = qh.shape
    Hk = kh.shape[1]
    out = np.zeros((B, H, N, d))
    for b in range(B):
        for h in range(H):
            hk = h * Hk // H
            for r in range(N):
                i = r // 128
                m, l = -math.inf, 0.0
                o = [0.0] * d
                for j in range((N + 127) // 128):
                    if causal and j > i:
                        break
                    keys = [t for t in range(j * 128, min(N, j * 128 + 128)) if not (causal and t > r)]
                    sc = F32(F32(dq[b, h, i]) * F32(dk[b, hk, j]))
                    S = []
                    for t in keys:
                        acc = sum(int(qh[b, h, r, c]) * int(kh[b, hk, t, c]) for c in range(d))
                        S.append(float(F32(F32(acc) * sc)))
                    m_new = max(m, max(S))
                    alpha = 0.0 if m == -math.inf else math.exp(m - m_new)
                    P = [float(F32(math.exp(s - m_new))) for s in S]
                    l = alpha * l + sum(P)
                    if operand == "fp16":
                        pop = [_f16(p) for p in P]
                    else:
                        pop = [_e4m3(float(F32(F32(p) * F32(p_r)))) for p in P]
                    for c in range(d):
                        o[c] = alpha * o[c] + sum(pop[n] * float(vop[b, hk, t, c])
                                                  for n, t in enumerate(keys))
                    m = m_new
                for c in range(d):
                    scale = (float(dv[b, hk, c]) / (p_r * l)) if operand == "e4m3" else 1.0 / l
                    out[b, h, r, c] = _f16(o[c] * scale)
    return out


@pytest.mark.parametrize("variant,p_r,v_r", [("B", 448.0, 448.0), ("8+8", 448.0, 448.0),
                                             ("8+8", 56.0, 9.0)])
@pytest.mark.parametrize("causal", [False, True])
def test_mirror_equals_python_loops(variant, p_r, v_r, causal):
    w = workloads.get("small_b_n256_d64").with_(B=1, H=2, H_kv=1, N=130, d=8, k_n_out=2,
                                                seed=61 + int(causal))
    q, k, v = workloads.generate(w)
    mirror, inter = oracle.sage_attention(q, k, v, causal=causal, sm_scale=w.scale,
                                          variant=variant, v_r=v_r, p_r=p_r)
    if variant == "B":
        vop, dv, operand = v.astype(np.float64), None, "fp16"
    else:
        vop = oracle.e4m3_decode(inter["v_hat"])
        dv, operand = inter["delta_v"], "e4m3"
    got = loops_attention(inter["q_hat"], inter["k_hat"], inter["delta_q"], inter["delta_k"],
                          vop, dv, causal, operand, p_r)
    m64 = mirror.astype(np.float64)
    # same arithmetic up to the order of fp64 sums: equal, or one fp16 ulp apart
    ulp = np.spacing(np.abs(m64).astype(np.float16)).astype(np.float64)
    diff = np.abs(got - m64)
    assert np.all(diff <= ulp), float(diff.max())
    assert (diff == 0).mean() > 0.99
