"""Seeded synthetic inputs for the quantized-attention hot path.

This module is shared by the CPU oracle's tests and by the CUDA path's
tests and benchmark.  It holds no arithmetic of the method itself: it only
draws random fp16 tensors with the shapes and value distributions of the
workloads (LLM prefill and video-DiT attention shapes), so both sides see
the same bytes.

Recipe (identical for every workload):
  * generator: numpy.random.default_rng(seed)  (PCG64), float32 draws,
    sums formed in float32, one cast to fp16 (round-to-nearest-even) at the end;
  * draw order: Q base [B,H,N,d]; Q per-channel bias [B,H,1,d] (if any);
    K base [B,Hkv,N,d]; K per-channel bias [B,Hkv,1,d]; then for every
    (b, h_kv) in row-major order the outlier channels
    (choice(d, n_out, replace=False)) and, for signed outliers, their signs
    (choice([-1, 1], n_out)); finally V [B,Hkv,N,d];
  * "bias drawn N(0, v)" means variance v (sigma = sqrt(v)); the bias is one
    vector per head, shared by every token of that head (the channel-wise
    outliers of K described in the SageAttention paper, Figure 4 / Section
    "Smooth K").
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "sweep_workloads", "generate", "get"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    H_kv: int
    N: int
    d: int
    causal: bool
    variants: tuple          # ("B",), ("8+8",) or both
    seed: int
    q_bias_var: float = 0.0  # 0 -> no Q bias drawn
    k_bias_var: float = 0.0
    k_n_out: int = 0         # number of outlier channels added to the K bias
    k_out_mag: float = 0.0
    k_out_signed: bool = False
    v_var: float = 1.0
    sm_scale: Optional[float] = None  # None -> 1/sqrt(d)

    @property
    def scale(self) -> float:
        return self.sm_scale if self.sm_scale is not None else 1.0 / math.sqrt(self.d)

    @property
    def ops(self) -> float:
        """4*B*H*N^2*d, halved for causal (the throughput numerator)."""
        o = 4.0 * self.B * self.H * self.N * self.N * self.d
        return o / 2 if self.causal else o

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the target: a small case, an 8+8 LLM-ish case,
# an LLM-prefill GQA causal case, a video-DiT long-sequence case, and a sweep.
WORKLOADS = {
    "small_b_n256_d64": Workload(
        "small_b_n256_d64", B=1, H=2, H_kv=2, N=256, d=64, causal=False,
        variants=("B",), seed=0, k_bias_var=4.0, k_n_out=4, k_out_mag=20.0),
    "llm_8p8_b2_h16_n4096_d128": Workload(
        "llm_8p8_b2_h16_n4096_d128", B=2, H=16, H_kv=16, N=4096, d=128,
        causal=False, variants=("8+8",), seed=1, q_bias_var=1.0,
        k_bias_var=4.0, k_n_out=8, k_out_mag=30.0),
    "prefill_gqa_causal_h32_kv8_n8192_d128": Workload(
        "prefill_gqa_causal_h32_kv8_n8192_d128", B=1, H=32, H_kv=8, N=8192,
        d=128, causal=True, variants=("B", "8+8"), seed=2, k_bias_var=3.0,
        v_var=0.5, sm_scale=1.0 / math.sqrt(128.0)),
    "video_dit_h24_n32768_d128": Workload(
        "video_dit_h24_n32768_d128", B=1, H=24, H_kv=24, N=32768, d=128,
        causal=False, variants=("8+8",), seed=3, q_bias_var=2.0,
        k_bias_var=6.0, k_n_out=16, k_out_mag=40.0, k_out_signed=True),
}


def sweep_workloads():
    """d in {64,128} x N in {1K..32K} x {non-causal, causal}; B*N = 65536, H = 16.

    Seed = 100 + (d_i*6 + N_i)*2 + causal_i; K bias generator as in the
    8+8 LLM workload (bias variance 4, 8 outlier channels at +30, Q bias
    variance 1)."""
    out = []
    for di, d in enumerate((64, 128)):
        for ni, n in enumerate((1024, 2048, 4096, 8192, 16384, 32768)):
            for ci, causal in enumerate((False, True)):
                idx = (di * 6 + ni) * 2 + ci
                out.append(Workload(
                    f"sweep_d{d}_n{n}_{'causal' if causal else 'full'}",
                    B=65536 // n, H=16, H_kv=16, N=n, d=d, causal=causal,
                    variants=("B", "8+8"), seed=100 + idx, q_bias_var=1.0,
                    k_bias_var=4.0, k_n_out=8, k_out_mag=30.0))
    return out


def get(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    for w in sweep_workloads():
        if w.name == name:
            return w
    raise KeyError(name)


def generate(w: Workload):
    """Return (q, k, v) as numpy float16 arrays, [B,H,N,d] / [B,Hkv,N,d]."""
    rng = np.random.default_rng(w.seed)
    f32 = np.float32
    q = rng.standard_normal((w.B, w.H, w.N, w.d), dtype=f32)
    if w.q_bias_var > 0:
        qb = rng.standard_normal((w.B, w.H, 1, w.d), dtype=f32) * f32(math.sqrt(w.q_bias_var))
        q += qb
    k = rng.standard_normal((w.B, w.H_kv, w.N, w.d), dtype=f32)
    kb = rng.standard_normal((w.B, w.H_kv, 1, w.d), dtype=f32)
    if w.k_bias_var > 0:
        kb *= f32(math.sqrt(w.k_bias_var))
    else:
        kb[...] = 0
    if w.k_n_out > 0:
        for b in range(w.B):
            for h in range(w.H_kv):
                ch = rng.choice(w.d, w.k_n_out, replace=False)
                if w.k_out_signed:
                    sg = rng.choice(np.array([-1, 1]), w.k_n_out).astype(f32)
                else:
                    sg = np.ones(w.k_n_out, dtype=f32)
                kb[b, h, 0, ch] += sg * f32(w.k_out_mag)
    k += kb
    v = rng.standard_normal((w.B, w.H_kv, w.N, w.d), dtype=f32)
    if w.v_var != 1.0:
        v *= f32(math.sqrt(w.v_var))
    return q.astype(np.float16), k.astype(np.float16), v.astype(np.float16)


def rope_tables(N: int, d: int, base: float = 10000.0):
    """cos / sin tables [N, d/2] (float32) of the usual rotary frequencies:
    angle(t, i) = t * base^(-2i/d), evaluated in float64, rounded once."""
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    ang = np.arange(N, dtype=np.float64)[:, None] * theta[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)

