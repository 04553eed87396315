"""sage_smooth_quant_qk_noalloc: the pre-pass of Q and K without any device
allocation inside the call (its partial sums go to a static 4 MiB array in
the library).  Its results must equal those of sage_smooth_quant_qk bit for
bit, on consecutive calls that reuse the same static scratch.

This file is named so that pytest collects it last: it has to pass both on
its own and after every other test has run in the same process."""
import ctypes

import numpy as np
import pytest
import torch

import workloads

MAX_PARTIALS = 1 << 19  # entries of the static scratch (int64)


def _partials(B, H_kv, N, d):
    return B * H_kv * ((N + 255) // 256) * d


def test_oversized_call_is_rejected_before_any_cuda_call():
    """Sizes beyond the static scratch return SAGE_ERR_UNSUPPORTED with a
    detail message; the check needs no GPU (the pointers are never used)."""
    from quantized_attention_08_b200 import build
    build.build()
    import quantized_attention_08_b200 as pkg
    lib = pkg.load_library()
    fake = ctypes.c_void_p(1 << 20)
    B, H, H_kv, N, d = 1, 32, 32, 32768 + 1, 128  # one chunk past the limit
    assert _partials(B, H_kv, N, d) > MAX_PARTIALS
    st = lib.sage_smooth_quant_qk_noalloc(fake, fake, B, H, H_kv, N, d, 0.088, fake, fake, fake,
                                          fake, fake, None)
    assert st == 2
    assert "static scratch" in pkg.sage_last_error_detail()
    # empty inputs are a no-op, as for the allocating entry point
    assert lib.sage_smooth_quant_qk_noalloc(None, None, 0, H, H_kv, N, d, 0.088, None, None, None,
                                            None, None, None) == 0


def _outputs(B, H, H_kv, N, d, dev="cuda"):
    nb = (N + 127) // 128
    return (torch.empty(B, H, N, d, dtype=torch.int8, device=dev),
            torch.empty(B, H_kv, N, d, dtype=torch.int8, device=dev),
            torch.empty(B, H, nb, dtype=torch.float32, device=dev),
            torch.empty(B, H_kv, nb, dtype=torch.float32, device=dev),
            torch.empty(B, H_kv, d, dtype=torch.float32, device=dev))


def _poisoned(B, H, H_kv, N, d):
    outs = _outputs(B, H, H_kv, N, d)
    for t in outs:
        t.view(torch.uint8).fill_(0xA5)
    return outs


def _inputs(case):
    if isinstance(case, str):
        w = workloads.get(case)
        q, k, _ = workloads.generate(w)
        return (torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(), w.scale)
    B, H, H_kv, N, d, seed = case
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn(B, H, N, d, generator=g, device="cuda").half()
    k = (torch.randn(B, H_kv, N, d, generator=g, device="cuda") +
         3.0 * torch.randn(B, H_kv, 1, d, generator=g, device="cuda")).half()
    return q, k, 1.0 / d ** 0.5


def _same_bits(a, b, name):
    assert a.shape == b.shape, name
    va, vb = a.view(torch.uint8), b.view(torch.uint8)
    n_diff = int((va != vb).sum())
    assert n_diff == 0, f"{name}: {n_diff} bytes differ"


# small workload, an LLM-prefill shape, a ragged GQA shape, and one that fills
# the static scratch exactly (B*H_kv*ceil(N/256)*d == 2^19)
CASES = ["small_b_n256_d64", "llm_8p8_b2_h16_n4096_d128",
         (3, 4, 2, 1000, 128, 11), (1, 64, 64, 32768, 64, 12)]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: c if isinstance(c, str) else
                         "B{}_H{}_Hkv{}_N{}_d{}".format(*c[:5]))
def test_noalloc_matches_allocating_entry_point_on_two_calls_in_a_row(case):
    import quantized_attention_08_b200 as sage
    q, k, scale = _inputs(case)
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    assert _partials(B, H_kv, N, d) <= MAX_PARTIALS
    ref = sage.sage_smooth_quant_qk(q, k, sm_scale=scale)
    first = sage.sage_smooth_quant_qk_noalloc(q, k, _poisoned(B, H, H_kv, N, d), sm_scale=scale)
    second = sage.sage_smooth_quant_qk_noalloc(q, k, _poisoned(B, H, H_kv, N, d), sm_scale=scale)
    torch.cuda.synchronize()
    names = ("q_hat", "k_hat", "delta_q", "delta_k", "mean_k")
    for call, outs in (("first", first), ("second", second)):
        for n, a, b in zip(names, ref, outs):
            _same_bits(a, b, f"{call} call, {n}")


@pytest.mark.gpu
def test_noalloc_after_a_larger_call_reads_no_stale_scratch():
    """A large call fills more of the static array than the small call that
    follows it; the small call's results must not depend on what is left."""
    import quantized_attention_08_b200 as sage
    big_q, big_k, big_s = _inputs((2, 16, 8, 8192, 128, 21))
    small_q, small_k, small_s = _inputs((1, 4, 4, 700, 128, 22))
    ref = sage.sage_smooth_quant_qk(small_q, small_k, sm_scale=small_s)
    B, H, N, d = big_q.shape
    sage.sage_smooth_quant_qk_noalloc(big_q, big_k, _outputs(B, H, big_k.shape[1], N, d),
                                      sm_scale=big_s)
    B, H, N, d = small_q.shape
    got = sage.sage_smooth_quant_qk_noalloc(small_q, small_k,
                                            _poisoned(B, H, small_k.shape[1], N, d),
                                            sm_scale=small_s)
    torch.cuda.synchronize()
    for n, a, b in zip(("q_hat", "k_hat", "delta_q", "delta_k", "mean_k"), ref, got):
        _same_bits(a, b, n)


@pytest.mark.gpu
def test_noalloc_draws_nothing_from_the_stream_ordered_pool():
    """The allocating entry point raises the default memory pool's high-water
    mark; the allocation-free one leaves it where it was."""
    rt = pytest.importorskip("cuda.bindings.runtime")
    drv = pytest.importorskip("cuda.bindings.driver")
    import quantized_attention_08_b200 as sage
    q, k, scale = _inputs((2, 8, 4, 4096, 128, 31))
    B, H, N, d = q.shape
    outs = _outputs(B, H, k.shape[1], N, d)
    torch.cuda.synchronize()
    err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
    assert err == rt.cudaError_t.cudaSuccess

    def used(attr):
        e, v = rt.cudaMemPoolGetAttribute(pool, attr)
        assert e == rt.cudaError_t.cudaSuccess
        return int(v)

    def reset_high():
        e, = rt.cudaMemPoolSetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh,
                                        drv.cuuint64_t(0))
        assert e == rt.cudaError_t.cudaSuccess

    cur = used(rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemCurrent)
    # positive control: the allocating entry point shows up in the pool
    reset_high()
    sage.sage_smooth_quant_qk(q, k, sm_scale=scale, out=outs)
    torch.cuda.synchronize()
    assert used(rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh) > cur
    reset_high()
    for _ in range(2):
        sage.sage_smooth_quant_qk_noalloc(q, k, outs, sm_scale=scale)
    torch.cuda.synchronize()
    assert used(rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh) == cur
    assert np.isfinite(outs[4].cpu().numpy()).all()
