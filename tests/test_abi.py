"""C-ABI checks that need no GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

from entmax_sm_attention_b200 import binding as eb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "entmax_attn.h")


@pytest.fixture(scope="module")
def lib():
    from entmax_sm_attention_b200 import build

    build.build()
    return eb.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(entmax_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(eb.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", eb.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def _desc(**kw):
    base = dict(B=1, H=2, L=300, d=64, alpha=1.5, scale=0.125, causal=0, window=-1, kv_len=None,
                dtype=eb.ENTMAX_BF16, max_sweeps=0, wait_limit_us=0, alibi_slopes=None, selftest=0, mask64=0)
    base.update(kw)
    return eb.AttnDesc(base["B"], base["H"], base["L"], base["d"], base["alpha"], base["scale"], base["causal"],
                       base["window"], base["kv_len"], base["dtype"], base["max_sweeps"], base["wait_limit_us"],
                       base["alibi_slopes"], base["selftest"], base["mask64"])


def test_workspace_bytes_valid_and_invalid(lib):
    n = lib.entmax_attn_workspace_bytes(ctypes.byref(_desc()))
    assert n > 0 and n % 256 == 0
    # grows with L
    assert lib.entmax_attn_workspace_bytes(ctypes.byref(_desc(L=4096))) > n
    for bad in (dict(B=0), dict(L=0), dict(d=32), dict(alpha=1.0), dict(alpha=17.0), dict(scale=0.0), dict(causal=2),
                dict(max_sweeps=-1), dict(max_sweeps=65), dict(L=eb.ENTMAX_MAX_L + 1), dict(dtype=7),
                dict(wait_limit_us=-1), dict(selftest=2), dict(mask64=2)):
        assert lib.entmax_attn_workspace_bytes(ctypes.byref(_desc(**bad))) == 0, bad


@pytest.mark.parametrize("bad,code", [
    (dict(d=128), eb.ENTMAX_EUNSUPPORTED),
    (dict(alpha=17.0), eb.ENTMAX_EUNSUPPORTED),
    (dict(alpha=1.0), eb.ENTMAX_EINVAL),
    (dict(alpha=0.5), eb.ENTMAX_EINVAL),
    (dict(alpha=1.25, dtype=eb.ENTMAX_FP32), eb.ENTMAX_EUNSUPPORTED),
    (dict(alibi_slopes=1 << 20, dtype=eb.ENTMAX_FP32), eb.ENTMAX_EUNSUPPORTED),
    (dict(dtype=9), eb.ENTMAX_EINVAL),
    (dict(L=eb.ENTMAX_MAX_L + 128), eb.ENTMAX_EUNSUPPORTED),
    (dict(B=-1), eb.ENTMAX_EINVAL),
    (dict(scale=float("nan")), eb.ENTMAX_EINVAL),
    (dict(max_sweeps=100), eb.ENTMAX_EINVAL),
    (dict(wait_limit_us=-5), eb.ENTMAX_EINVAL),
    (dict(selftest=3), eb.ENTMAX_EINVAL),
    (dict(mask64=-1), eb.ENTMAX_EINVAL),
])
def test_forward_rejects_on_host(lib, bad, code):
    d = _desc(**bad)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails before any launch
    rc = lib.entmax_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, fake, None)
    assert rc == code


def test_null_and_misaligned_pointers_rejected(lib):
    d = _desc()
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert lib.entmax_attn_fwd(ctypes.byref(d), None, good, good, good, good, good, None) == eb.ENTMAX_EINVAL
    assert lib.entmax_attn_fwd(ctypes.byref(d), odd, good, good, good, good, good, None) == eb.ENTMAX_EINVAL
    ws_odd = ctypes.c_void_p((1 << 20) + 128)   # workspace must be 256-byte aligned
    assert lib.entmax_attn_fwd(ctypes.byref(d), good, good, good, good, good, ws_odd, None) == eb.ENTMAX_EINVAL
    assert lib.entmax_attn_bwd(ctypes.byref(d), good, good, good, odd, good, good, good, good, good,
                               None) == eb.ENTMAX_EINVAL
    assert lib.entmax_attn_fwd(None, good, good, good, good, good, good, None) == eb.ENTMAX_EINVAL


def test_rows_rejects_on_host(lib):
    p = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    f15 = ctypes.c_float(1.5)
    assert lib.entmax_rows(p, 4, 0, 4, f15, p, p, None, None) == eb.ENTMAX_EINVAL   # n = 0
    assert lib.entmax_rows(p, 4, 8, 6, f15, p, p, None, None) == eb.ENTMAX_EINVAL   # ld % 4
    assert lib.entmax_rows(p, 4, 8, 4, f15, p, p, None, None) == eb.ENTMAX_EINVAL   # ld < n
    assert lib.entmax_rows(p, 4, 8, 8, ctypes.c_float(1.2), p, p, None, None) == eb.ENTMAX_EUNSUPPORTED
    assert lib.entmax_rows(p, -1, 8, 8, f15, p, p, None, None) == eb.ENTMAX_EINVAL
    assert lib.entmax_rows(p, 4, 8, 8, f15, p, p, odd, None) == eb.ENTMAX_EINVAL     # misaligned status
    assert lib.entmax_rows(p, 0, 8, 8, f15, p, p, None, None) == eb.ENTMAX_OK      # empty: no-op


def test_general_alpha_accepted(lib):
    """Any 1 < alpha <= 16 is a valid bf16 attention problem (run-time alpha variant)."""
    for a in (1.01, 1.25, 1.75, 3.0, 16.0):
        assert lib.entmax_attn_workspace_bytes(ctypes.byref(_desc(alpha=a))) > 0, a


def test_desc_layout_matches_header():
    """The ctypes mirror has the header's field order (checked by offsets of the tail)."""
    assert eb.AttnDesc.alibi_slopes.offset % 8 == 0
    assert eb.AttnDesc.selftest.offset > eb.AttnDesc.alibi_slopes.offset


def test_block_mask64_needs_a_mask64_forward(lib):
    """entmax_attn_block_mask64 rejects a descriptor without mask64 before touching memory."""
    good = ctypes.c_void_p(1 << 20)
    assert lib.entmax_attn_block_mask64(ctypes.byref(_desc()), good, good, None) == eb.ENTMAX_EINVAL
    assert lib.entmax_attn_block_mask64(ctypes.byref(_desc(mask64=1)), good, None, None) == eb.ENTMAX_EINVAL
