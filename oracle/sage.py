"""Plain, slow, CPU oracle of SageAttention-style quantized attention.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
bench's CPU-baseline / reference legs may import this module; the product
path (the C-ABI library and its Python binding) never does, and shares no
code, table or helper with it.

Sources (web pages describing the method):
  [SA1]  "SageAttention: Accurate 8-Bit Attention for Plug-and-Play
         Inference Acceleration" (detailed review page): Algorithm 1
         (SAGEAttn-B), Eq. 4-5 (quantized attention), Eq. 6 (Smooth K and
         its shift-invariance proof), "Problem Formulation" assumptions
         (max P~ = 1 gives a static P~ scale), "关键实现细节" item 1
         (1/sqrt(d) folded into the quantization of Q).
  [SA2++] "SageAttention2++: A More Efficient Implementation of
         SageAttention2" (review page): "核心公式" (delta_Q, delta_K,
         delta_P, delta_V formulas; Eq. (1) FP16-accumulator bound; Eq. (2)
         narrowed ranges P_r, V_r), Table 2 ((P_r, V_r) pairs).

Readings where the pages leave a step open (each one is listed in the
design notes of the repository):
  * block sizes b_q = b_kv = 128 tokens; the last block of a ragged
    sequence is short;
  * mean(K) is an exact sum (each fp16 value is an integer multiple of
    2^-24), converted to fp64, divided by N in fp64, rounded once to fp32;
  * smoothed K = fp32(k) - mean_fp32 (one fp32 subtraction);
  * x_Q = fp32(q) * fp32(sm_scale);
  * delta = absmax / 127 and a_hat = round_half_even(x / delta), both fp32
    IEEE divisions, clamped to [-127, 127]; an all-zero block has delta 0
    and a_hat 0;
  * delta_P is static, 1/P_r (P_r = 448 for 8+8): P_hat = e4m3(P~ * P_r);
    delta_V = colmax|V| / V_r per (batch, kv head, channel);
  * P~ = exp(S - m_new) evaluated in fp64 and rounded to fp32; the running
    row sum l adds this fp32 P~ before the operand rounding;
  * GQA: query head h reads kv head floor(h * H_kv / H);
  * causal mask is square and top-left aligned (key t visible to query r
    iff t <= r);
  * rotary embedding (when used): rotate-half pairing with caller cos/sin
    tables [N, d/2], fp32 products and sum, rounded to fp16, then the
    pre-pass unchanged; the narrowed 8+8 ranges use P_r = 56, V_r = 9.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

from .codecs import e4m3_decode, e4m3_encode, e4m3_round, fp16_rne, FP16_MAX

BLOCK = 128
F32 = np.float32


# --------------------------------------------------------------------------
# Pre-pass: Smooth K ([SA1] Eq. 6, Algorithm 1 step 1) and the per-block
# quantizer psi ([SA1] Algorithm 1 step 2; [SA2++] delta_Q / delta_K).
# --------------------------------------------------------------------------

def mean_k(k: np.ndarray) -> np.ndarray:
    """mean(K) = (1/N) * sum_t K[t, :] per (batch, kv head, channel) ([SA1] Eq. 6).

    The sum is exact: every fp16 value times 2^24 is an integer, summed in
    int64.  The integer sum is converted to fp64 (round to nearest), scaled
    by 2^-24, divided by N in fp64 and rounded once to fp32."""
    B, Hk, N, d = k.shape
    if N == 0:
        return np.zeros((B, Hk, d), dtype=F32)
    ki = (k.astype(np.float64) * 2.0 ** 24).astype(np.int64)
    s = ki.sum(axis=2, dtype=np.int64)
    return ((s.astype(np.float64) * 2.0 ** -24) / float(N)).astype(F32)


def quant_blocks(x: np.ndarray, block: int = BLOCK):
    """psi: per-block symmetric INT8 quantizer over blocks of `block` tokens.

    x: fp32 [..., N, d].  Returns (x_hat int8 [..., N, d], delta fp32
    [..., ceil(N/block)]) with delta = max|x_blk| / 127 and
    x_hat = round_half_even(x / delta) ([SA2++] delta_Q = max|Q|/127,
    Q_hat = ⌈Q/delta_Q⌋)."""
    assert x.dtype == F32
    *lead, N, d = x.shape
    nb = (N + block - 1) // block
    xh = np.zeros(x.shape, dtype=np.int8)
    delta = np.zeros((*lead, nb), dtype=F32)
    for bi in range(nb):
        sl = slice(bi * block, min(N, (bi + 1) * block))
        blk = x[..., sl, :]
        absmax = np.abs(blk).max(axis=(-2, -1)).astype(F32)
        dl = (absmax / F32(127.0)).astype(F32)
        delta[..., bi] = dl
        dlb = dl[..., None, None]
        safe = np.where(dlb == 0, F32(1.0), dlb).astype(F32)
        with np.errstate(invalid="ignore", divide="ignore"):
            r = np.rint((blk / safe).astype(F32))
        r = np.clip(r, -127, 127)
        r = np.where(dlb == 0, 0, r)
        xh[..., sl, :] = r.astype(np.int8)
    return xh, delta


def quant_q(q: np.ndarray, sm_scale: float):
    """psi_Q(Q * sm_scale): the softmax scale is folded into the
    quantization of Q ([SA1] Algorithm 1 step 2 and implementation detail 1)."""
    x = (q.astype(F32) * F32(sm_scale)).astype(F32)
    return quant_blocks(x)


def smooth_quant_k(k: np.ndarray):
    """phi_K = psi_K o gamma: subtract mean(K) then quantize per block.
    Returns (k_hat int8, delta_k fp32, mean_k fp32)."""
    mk = mean_k(k)
    x = (k.astype(F32) - mk[:, :, None, :]).astype(F32)
    kh, dk = quant_blocks(x)
    return kh, dk, mk


def quant_v_fp8(v: np.ndarray, v_r: float = 448.0):
    """8+8 V quantizer ([SA2++] delta_V = colmax(|V|)/448, Eq. (2) with a
    general V_r): delta_V per (batch, kv head, channel) over all tokens,
    V_hat = e4m3_rne_satfinite(fp32(v) / delta_V).
    Returns (v_hat uint8 codes, same layout as v; delta_v fp32 [B,Hkv,d])."""
    vf = v.astype(F32)
    B, Hk, N, d = v.shape
    if N == 0:
        return np.zeros(v.shape, np.uint8), np.zeros((B, Hk, d), F32)
    colmax = np.abs(vf).max(axis=2).astype(F32)
    dv = (colmax / F32(v_r)).astype(F32)
    safe = np.where(dv == 0, F32(1.0), dv).astype(F32)
    y = (vf / safe[:, :, None, :]).astype(F32)
    codes = e4m3_encode(y)
    codes = np.where(dv[:, :, None, :] == 0, np.uint8(0), codes).astype(np.uint8)
    return codes, dv


# --------------------------------------------------------------------------
# Rotary position embedding before the quantizers ([SA1] implementation
# detail 1: Q and K are rotated and quantized in one pass; the SageAttention
# summary page: a kernel fusing RoPE with quantization).
# --------------------------------------------------------------------------

def rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotary embedding of fp16 x [..., N, d] in the rotate-half pairing:
    channel i < d/2 pairs with i + d/2, and at token t with c = cos[t, i],
    s = sin[t, i] (fp32 tables [N, d/2]):
        y[i]       = x[i] * c - x[i + d/2] * s
        y[i + d/2] = x[i + d/2] * c + x[i] * s
    Each product is rounded to fp32, then the sum, then the result to fp16
    (the value a separate rotary pass would write back in fp16); the fused
    pre-pass reproduces exactly this."""
    d = x.shape[-1]
    h = d // 2
    assert cos.shape == (x.shape[-2], h) and sin.shape == cos.shape
    xf = x.astype(F32)
    c = cos.astype(F32)
    s = sin.astype(F32)
    x1, x2 = xf[..., :h], xf[..., h:]
    y1 = ((x1 * c).astype(F32) - (x2 * s).astype(F32)).astype(F32)
    y2 = ((x2 * c).astype(F32) + (x1 * s).astype(F32)).astype(F32)
    return fp16_rne(np.concatenate([y1, y2], axis=-1).astype(np.float64))


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _kv_head(h: int, H: int, Hk: int) -> int:
    return (h * Hk) // H


def _rows_from_blocks(N: int, q_blocks: Optional[Sequence[int]]) -> np.ndarray:
    if q_blocks is None:
        return np.arange(N)
    parts = [np.arange(b * BLOCK, min(N, (b + 1) * BLOCK)) for b in q_blocks]
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def attention_reference(q, k, v, *, causal: bool, sm_scale: float,
                        q_blocks: Optional[Sequence[int]] = None,
                        smooth_k: bool = False) -> np.ndarray:
    """Full-precision truth: O = softmax(sm_scale * Q K^T [+ causal mask]) V in
    fp64 on the fp16 inputs (mode R).  With smooth_k, K is replaced by
    K - mean(K) computed in fp64 (mode R_s; equal to R by [SA1] Eq. 6).
    Returns float64 [B, H, rows, d] for the rows of the selected q blocks."""
    B, H, N, d = q.shape
    Hk = k.shape[1]
    rows = _rows_from_blocks(N, q_blocks)
    out = np.zeros((B, H, len(rows), d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            hk = _kv_head(h, H, Hk)
            Q = q[b, h, rows].astype(np.float64)
            K = k[b, hk].astype(np.float64)
            if smooth_k:
                K = K - K.mean(axis=0, keepdims=True)
            V = v[b, hk].astype(np.float64)
            S = sm_scale * (Q @ K.T)
            if causal:
                S = np.where(np.arange(N)[None, :] > rows[:, None], -np.inf, S)
            S = S - S.max(axis=1, keepdims=True)
            P = np.exp(S)
            out[b, h] = (P @ V) / P.sum(axis=1, keepdims=True)
    return out


def attention_online(qh, kh, dq, dk, vop, *, causal: bool, operand: str,
                     p_r: float = 448.0, dv=None,
                     q_blocks: Optional[Sequence[int]] = None,
                     s_fp32: bool = True, simulate_f16acc: bool = False,
                     return_stats: bool = False, out_fp16: bool = True,
                     ambiguity: float = 0.0, flip_ambiguous: bool = False):
    """Tiled attention with online softmax, following [SA1] Algorithm 1
    steps 3-9 and Eq. 4-5.

    qh [B,H,N,d], kh [B,Hkv,N,d]: quantized operands (int8 codes, or any
    real values for the exactness checks); dq [B,H,nb], dk [B,Hkv,nb]: the
    per-block scales; vop [B,Hkv,N,d]: the V operand as real values (the
    fp16 V for SAGEAttn-B, the decoded E4M3 V_hat for 8+8).

    operand: how the fp32 P~ becomes the P~V operand --
      "fp16"  SAGEAttn-B (P~ rounded to fp16),
      "e4m3"  8+8 (P_hat = e4m3(fp32(P~ * P_r)); output multiplied by
              delta_V[c] / P_r),
      "exact" no rounding (for checks).
    s_fp32: S = fp32(acc) * fp32(dq*dk) as in the kernel; False keeps fp64.
    simulate_f16acc: round every per-tile partial P_hat V_hat to fp16
    (the FP16 accumulator of [SA2++], flushed per tile).
    ambiguity: relative band eps.  The operand code of an fp32 P~ is
    decided by floating point; an implementation whose P~ differs from this
    one by at most a factor (1 +- eps) may legitimately pick the neighbouring
    code when P~ (times P_r) lies within that band of a rounding midpoint.
    For every such ambiguous element the difference between the two codes,
    times |V operand|, is accumulated (with the same online rescaling as O)
    into a per-output slack; the function then also returns that slack,
    scaled like O, and each row's final running max m (the row max of S).  flip_ambiguous: use the other code for every ambiguous
    element (checks that the slack bounds the effect).
    Each q block walks its kv tiles in ascending order; with causal only
    tiles j <= i, masking keys t > r on the diagonal tile."""
    B, H, N, d = qh.shape
    Hk = kh.shape[1]
    nkv = (N + BLOCK - 1) // BLOCK
    rows = _rows_from_blocks(N, q_blocks)
    rblk = rows // BLOCK
    out = np.zeros((B, H, len(rows), d), dtype=np.float64)
    slack = np.zeros((B, H, len(rows), d), dtype=np.float64)
    m_final = np.zeros((B, H, len(rows)), dtype=np.float64)
    stats = []
    f16acc_overflow = False
    for b in range(B):
        for h in range(H):
            hk = _kv_head(h, H, Hk)
            Qf = qh[b, h, rows].astype(np.float64)
            Kf = kh[b, hk].astype(np.float64)
            Vf = vop[b, hk].astype(np.float64)
            m = np.full(len(rows), -np.inf, dtype=F32 if s_fp32 else np.float64)
            l = np.zeros(len(rows), dtype=np.float64)
            O = np.zeros((len(rows), d), dtype=np.float64)
            SL = np.zeros((len(rows), d), dtype=np.float64)
            for j in range(nkv):
                act = (rblk >= j) if causal else np.ones(len(rows), bool)
                if not act.any():
                    break
                ia = np.nonzero(act)[0]
                cols = np.arange(j * BLOCK, min(N, (j + 1) * BLOCK))
                acc = Qf[ia] @ Kf[cols].T          # exact for integer operands
                if s_fp32:
                    sc = (dq[b, h, rblk[ia]].astype(F32) * F32(dk[b, hk, j])).astype(F32)
                    S = (acc.astype(F32) * sc[:, None]).astype(F32)
                else:
                    sc = dq[b, h, rblk[ia]].astype(np.float64) * float(dk[b, hk, j])
                    S = acc * sc[:, None]
                if causal:
                    ninf = F32(-np.inf) if s_fp32 else -np.inf
                    S = np.where(cols[None, :] > rows[ia][:, None], ninf, S)
                m_old = m[ia]
                m_new = np.maximum(m_old, S.max(axis=1))
                P = np.exp(S.astype(np.float64) - m_new.astype(np.float64)[:, None])
                if s_fp32:
                    P = P.astype(F32)
                with np.errstate(invalid="ignore"):
                    alpha = np.exp(m_old.astype(np.float64) - m_new.astype(np.float64))
                alpha = np.where(np.isneginf(m_old), 0.0, alpha)
                if return_stats:
                    stats.append((j, P.max(axis=1).astype(np.float64), m_new > m_old))
                l[ia] = alpha * l[ia] + P.astype(np.float64).sum(axis=1)
                if operand == "fp16":
                    pop = fp16_rne(P.astype(F32)).astype(np.float64)
                    rnd = lambda z: fp16_rne(z).astype(np.float64)  # noqa: E731
                    zv = P.astype(np.float64)
                elif operand == "e4m3":
                    pop = e4m3_decode(e4m3_encode((P.astype(F32) * F32(p_r)).astype(F32)))
                    rnd = e4m3_round
                    zv = P.astype(np.float64) * float(p_r)
                elif operand == "exact":
                    pop = P.astype(np.float64)
                    rnd, zv = None, None
                else:
                    raise ValueError(operand)
                if ambiguity > 0 and rnd is not None:
                    lo = rnd(zv * (1.0 - ambiguity))
                    hi = rnd(zv * (1.0 + ambiguity))
                    amb = lo != hi
                    dp = np.where(amb, hi - lo, 0.0)
                    if flip_ambiguous:
                        pop = np.where(amb, np.where(pop == lo, hi, lo), pop)
                    SL[ia] = alpha[:, None] * SL[ia] + dp @ np.abs(Vf[cols])
                part = pop @ Vf[cols]
                if simulate_f16acc:
                    if np.abs(part).max(initial=0.0) > FP16_MAX:
                        f16acc_overflow = True
                    part = fp16_rne(part).astype(np.float64)
                O[ia] = alpha[:, None] * O[ia] + part
                m[ia] = m_new
            if operand == "e4m3":
                scale = dv[b, hk][None, :].astype(np.float64) / (float(p_r) * l[:, None])
            else:
                scale = 1.0 / l[:, None]
            out[b, h] = O * scale
            slack[b, h] = SL * scale
            m_final[b, h] = m
    if out_fp16:
        out = fp16_rne(out)
    if return_stats or simulate_f16acc or ambiguity > 0:
        return out, {"tiles": stats, "f16acc_overflow": f16acc_overflow, "slack": slack,
                     "m": m_final}
    return out


def sage_attention(q, k, v, *, causal: bool, sm_scale: Optional[float] = None,
                   variant: str = "B", v_r: float = 448.0, p_r: float = 448.0,
                   q_blocks: Optional[Sequence[int]] = None,
                   simulate_f16acc: bool = False, ambiguity: float = 0.0,
                   flip_ambiguous: bool = False):
    """Quantized mirror (mode QO) of the whole forward pass: Smooth K,
    per-block INT8 Q/K, then Algorithm 1 with the fp16 (variant "B") or
    E4M3 (variant "8+8") P~V.  Returns (O fp16 [B,H,rows,d], intermediates)."""
    d = q.shape[-1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    qh, dq = quant_q(q, sm_scale)
    kh, dk, mk = smooth_quant_k(k)
    inter = {"q_hat": qh, "delta_q": dq, "k_hat": kh, "delta_k": dk, "mean_k": mk}
    extra = dict(q_blocks=q_blocks, ambiguity=ambiguity, flip_ambiguous=flip_ambiguous)
    if variant == "B":
        o = attention_online(qh, kh, dq, dk, v, causal=causal, operand="fp16", **extra)
    elif variant == "8+8":
        vh, dv = quant_v_fp8(v, v_r)
        inter.update(v_hat=vh, delta_v=dv)
        o = attention_online(qh, kh, dq, dk, e4m3_decode(vh), causal=causal,
                             operand="e4m3", p_r=p_r, dv=dv,
                             simulate_f16acc=simulate_f16acc, **extra)
    else:
        raise ValueError(variant)
    if isinstance(o, tuple):
        o, st = o
        inter["f16acc_overflow"] = st["f16acc_overflow"]
        inter["slack"] = st["slack"]
        inter["m"] = st["m"]
    return o, inter


def sage_attention_varlen(q, k, v, cu_seqlens, *, causal: bool, sm_scale: Optional[float] = None,
                          variant: str = "B", v_r: float = 448.0, p_r: float = 448.0,
                          q_blocks: Optional[dict] = None, ambiguity: float = 0.0):
    """A batch of sequences of different lengths packed along the token axis
    (the SageAttention review's Table 7 runs models whose sequence lengths
    are not multiples of the block size, e.g. N = 17776 and N = 1105).

    q [H, T, d], k and v [H_kv, T, d]; sequence s holds tokens
    cu_seqlens[s] .. cu_seqlens[s+1] - 1 of every head.  Every sequence is its
    own attention problem: its own mean(K), its own 128-token blocks counted
    from its first token, its own delta_V -- sage_attention on each slice.
    q_blocks: optional {s: [q block indices of sequence s]} to restrict the
    output rows (sequences not in the dict are skipped when it is given).
    Returns (O fp16 [H, T, d] -- rows not computed are zero --, list of the
    per-sequence intermediates, None for an empty or skipped sequence)."""
    cu = [int(x) for x in cu_seqlens]
    assert cu[0] == 0 and all(b >= a for a, b in zip(cu, cu[1:])) and cu[-1] == q.shape[1]
    out = np.zeros(q.shape, np.float16)
    slack = np.zeros(q.shape, np.float64)
    m = np.zeros(q.shape[:2], np.float64)
    inters = []
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b == a or (q_blocks is not None and s not in q_blocks):
            inters.append(None)
            continue
        blocks = None if q_blocks is None else q_blocks[s]
        o_s, inter = sage_attention(q[None, :, a:b], k[None, :, a:b], v[None, :, a:b],
                                    causal=causal, sm_scale=sm_scale, variant=variant, v_r=v_r,
                                    p_r=p_r, q_blocks=blocks, ambiguity=ambiguity)
        rows = _rows_from_blocks(b - a, blocks)
        out[:, a + rows] = o_s[0]
        if "slack" in inter:
            slack[:, a + rows] = inter["slack"][0]
            m[:, a + rows] = inter["m"][0]
        inters.append(inter)
    return out, {"per_sequence": inters, "slack": slack, "m": m}


# --------------------------------------------------------------------------
# FP16-accumulator bound ([SA2++] Eq. (1)-(2))
# --------------------------------------------------------------------------

def f16acc_product_limit(n: int) -> float:
    """Largest P_r * V_r such that n products of magnitude <= P_r*V_r cannot
    overflow an fp16 accumulator: floor(65504 / n)  ([SA2++] Eq. (1):
    |32 * p * v| <= 65504, i.e. P_r * V_r <= 2047 for n = 32)."""
    return float(math.floor(FP16_MAX / n))


def f16acc_bound_ok(p_r: float, v_r: float, n: int) -> bool:
    """n * P_r * V_r <= 65504: with P~ <= 1 (so |P_hat| <= P_r) and
    |V_hat| <= V_r no partial sum of n products can leave the fp16 range."""
    return n * p_r * v_r <= FP16_MAX


# --------------------------------------------------------------------------
# Accuracy metrics named in [SA1] Table 2 (CosSim, Relative L1, RMSE)
# --------------------------------------------------------------------------

def cossim(o, r) -> float:
    o = np.asarray(o, np.float64).ravel()
    r = np.asarray(r, np.float64).ravel()
    return float(o @ r / (np.linalg.norm(o) * np.linalg.norm(r)))


def rel_l1(o, r) -> float:
    o = np.asarray(o, np.float64)
    r = np.asarray(r, np.float64)
    return float(np.abs(o - r).sum() / np.abs(r).sum())


def rmse(o, r) -> float:
    o = np.asarray(o, np.float64)
    r = np.asarray(r, np.float64)
    return float(np.sqrt(np.mean((o - r) ** 2)))
