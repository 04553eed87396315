"""CPU checks of the C-ABI library: it builds, loads without a GPU, and
exports every function declared in include/sage.h; host-side argument
checks that return before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sage.h")


@pytest.fixture(scope="module")
def lib():
    from quantized_attention_08_b200 import build
    build.build()
    import quantized_attention_08_b200 as pkg
    return pkg.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+(sage_[a-z0-9_]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("sage_smooth_quant_qk", "sage_quant_v_fp8", "sage_attn_fwd",
              "sage_attn_fwd_quantized", "sage_get_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol():
    import quantized_attention_08_b200 as pkg
    for name in declared_functions():
        assert name in pkg._SIGS, name
        assert callable(getattr(pkg, name)), name


def test_status_strings_and_version(lib):
    import quantized_attention_08_b200 as pkg
    assert pkg.sage_status_string(0) == "ok"
    assert "aligned" in pkg.sage_status_string(3)
    assert re.match(r"\d+\.\d+\.\d+", pkg.sage_version())
    assert pkg.sage_v_hat_layout() == 0


def test_host_argument_checks_need_no_gpu(lib):
    """Shape / variant / scale errors are reported before any CUDA call."""
    f = lib.sage_attn_fwd
    fake = ctypes.c_void_p(1 << 20)
    # d = 96 unsupported
    assert f(fake, fake, fake, fake, 1, 2, 2, 128, 96, 0, 0.1, 0, None) == 2
    # H not a multiple of H_kv
    assert f(fake, fake, fake, fake, 1, 3, 2, 128, 64, 0, 0.1, 0, None) == 2
    # unknown variant
    assert f(fake, fake, fake, fake, 1, 2, 2, 128, 64, 0, 0.1, 7, None) == 2
    # sm_scale <= 0, NaN
    assert f(fake, fake, fake, fake, 1, 2, 2, 128, 64, 0, 0.0, 0, None) == 1
    assert f(fake, fake, fake, fake, 1, 2, 2, 128, 64, 0, float("nan"), 0, None) == 1
    # negative size, bad causal flag
    assert f(fake, fake, fake, fake, 1, 2, 2, -1, 64, 0, 0.1, 0, None) == 1
    assert f(fake, fake, fake, fake, 1, 2, 2, 128, 64, 2, 0.1, 0, None) == 1
    # null pointer
    assert f(None, fake, fake, fake, 1, 2, 2, 128, 64, 0, 0.1, 0, None) == 1
    # misaligned
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert f(odd, fake, fake, fake, 1, 2, 2, 128, 64, 0, 0.1, 0, None) == 3
    # empty problems are a no-op
    assert f(None, None, None, None, 0, 2, 2, 128, 64, 0, 0.1, 0, None) == 0
    assert f(None, None, None, None, 1, 2, 2, 0, 64, 0, 0.1, 0, None) == 0
    # V range of the fp8 quantizer
    g = lib.sage_quant_v_fp8
    assert g(fake, 1, 2, 128, 64, 500.0, fake, fake, None) == 1
    assert g(fake, 1, 2, 128, 64, 0.0, fake, fake, None) == 1
    # rotary pre-pass: tables are required and 16-byte aligned
    r = lib.sage_smooth_quant_qkv_rope
    args = lambda cs, sn: (fake, fake, None, cs, sn, 1, 2, 2, 128, 64, 0.125, 448.0,
                           fake, fake, None, fake, fake, fake, None, None)
    assert r(*args(None, fake)) == 1
    assert r(*args(fake, None)) == 1
    assert r(*args(odd, fake)) == 3
    assert r(*args(fake, fake)[:5], 1, 2, 2, 128, 96, *args(fake, fake)[10:]) == 2


def test_varlen_and_host_argument_checks_need_no_gpu(lib):
    """The packed-batch and host-buffer entry points reject bad arguments
    before any CUDA call (status codes of include/sage.h: 1 invalid,
    2 unsupported, 3 misaligned), and an empty batch is a no-op."""
    fake = ctypes.c_void_p(1 << 20)
    cu = ctypes.c_void_p(1 << 16)
    f = lib.sage_attn_fwd_varlen
    # (q, k, v, o, cu_seqlens, B, max_seqlen, T, H, H_kv, d, causal, sm_scale, variant, stream)
    ok = [fake, fake, fake, fake, cu, 2, 128, 200, 2, 2, 64, 0, 0.125, 1, None]

    def call(**kw):
        a = list(ok)
        for i, key in enumerate(("q", "k", "v", "o", "cu", "B", "max_seqlen", "T", "H", "H_kv", "d",
                                 "causal", "sm_scale", "variant")):
            if key in kw:
                a[i] = kw[key]
        return f(*a)

    assert call(cu=None) == 1                                  # no offsets for a non-empty batch
    assert call(cu=ctypes.c_void_p((1 << 16) + 2)) == 3        # offsets not 4-byte aligned
    assert call(T=-1) == 1
    assert call(T=(1 << 30) + 1) == 2                          # row coordinates are 32-bit
    assert call(d=96) == 2
    assert call(variant=7) == 2
    assert call(causal=2) == 1
    assert call(sm_scale=0.0) == 1
    assert call(q=None) == 1
    assert call(o=ctypes.c_void_p((1 << 20) + 8)) == 3
    assert call(B=0, cu=None) == 0                             # empty batch
    assert call(T=0, cu=None) == 0
    h = lib.sage_attn_fwd_host
    # (q, k, v, o, B, H, H_kv, N, d, causal, sm_scale, variant, stream)
    assert h(None, fake, fake, fake, 1, 2, 2, 128, 64, 0, 0.125, 1, None) == 1
    assert h(fake, fake, fake, fake, 1, 2, 2, 128, 96, 0, 0.125, 1, None) == 2
    assert h(fake, fake, fake, fake, 1, 2, 2, 128, 64, 0, -1.0, 1, None) == 1
    assert h(None, None, None, None, 0, 2, 2, 128, 64, 0, 0.125, 1, None) == 0


def test_size_limits_are_rejected_before_any_cuda_call(lib):
    """The documented limits: B*H <= 65535 (grid.y) and N <= 2^24 (32-bit
    TMA coordinates); one past each is SAGE_ERR_UNSUPPORTED.  (Only calls
    that the host checks reject are made: the pointers are fake.)"""
    f = lib.sage_attn_fwd
    fake = ctypes.c_void_p(1 << 20)
    assert f(fake, fake, fake, fake, 1, 65536, 65536, 128, 64, 0, 0.1, 0, None) == 2
    assert f(fake, fake, fake, fake, 2, 32768, 32768, 128, 64, 0, 0.1, 0, None) == 2
    assert f(fake, fake, fake, fake, 1, 2, 2, (1 << 24) + 1, 64, 0, 0.1, 0, None) == 2
    q = lib.sage_smooth_quant_qk
    assert q(fake, fake, 1, 2, 2, (1 << 24) + 1, 128, 0.1, fake, fake, fake, fake, fake, None) == 2
    assert lib.sage_attn_workspace_bytes(1, 65536, 65536, 128, 64, 0) == 0


def test_workspace_size_is_consistent(lib):
    import quantized_attention_08_b200 as pkg
    a = pkg.sage_attn_workspace_bytes(1, 32, 8, 8192, 128, "B")
    b = pkg.sage_attn_workspace_bytes(1, 32, 8, 8192, 128, "8+8")
    # q_hat + k_hat at least, and 8+8 adds v_hat
    assert a >= 32 * 8192 * 128 + 8 * 8192 * 128
    assert b >= a + 8 * 8192 * 128
    assert pkg.sage_attn_workspace_bytes(0, 32, 8, 8192, 128, "B") == 0
    assert pkg.sage_attn_workspace_bytes(1, 32, 8, 8192, 96, "B") == 0
