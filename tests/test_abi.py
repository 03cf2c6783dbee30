"""The C-ABI library without a GPU: it loads, exports every declared entry
point, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

from gqa_prefix_suffix_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dm05_suffix_attn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dm05_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from gqa_prefix_suffix_b200 import build
    build.build()
    return bd.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(bd.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", bd.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (dm05_[a-z_0-9]+)$", out, flags=re.M))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)


def test_status_strings(lib):
    for st in (0, -1, -2, -3, -4, -5, -6):
        assert bd.dm05_status_string(st).startswith("DM05_")
    assert "unknown" in bd.dm05_status_string(99)


FAKE = 0x7f0000001000  # 16-byte aligned, never dereferenced: checks fail first


def call(**kw):
    a = dict(q=FAKE, k_prefix=FAKE, v_prefix=FAKE, prefix_valid_len=None, prefix_mask=None,
             k_suffix=FAKE, v_suffix=FAKE, out=FAKE, lse=None, B=1, Hq=8, Hkv=4, P=1024, S=50, D=256,
             stream=None)
    a.update(kw)
    return bd.dm05_suffix_attn(a["q"], a["k_prefix"], a["v_prefix"], a["prefix_valid_len"],
                               a["prefix_mask"], a["k_suffix"], a["v_suffix"], a["out"], a["lse"],
                               a["B"], a["Hq"], a["Hkv"], a["P"], a["S"], a["D"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), bd.DM05_ERR_NULL),
    (dict(k_suffix=None), bd.DM05_ERR_NULL),
    (dict(v_suffix=None), bd.DM05_ERR_NULL),
    (dict(out=None), bd.DM05_ERR_NULL),
    (dict(k_prefix=None), bd.DM05_ERR_NULL),
    (dict(v_prefix=None), bd.DM05_ERR_NULL),
    (dict(B=0), bd.DM05_ERR_SHAPE),
    (dict(S=0), bd.DM05_ERR_SHAPE),
    (dict(P=-1), bd.DM05_ERR_SHAPE),
    (dict(Hq=6), bd.DM05_ERR_SHAPE),
    (dict(Hkv=0), bd.DM05_ERR_SHAPE),
    (dict(P=(1 << 24) + 1), bd.DM05_ERR_SHAPE),
    (dict(D=128), bd.DM05_ERR_UNSUPPORTED),
    (dict(S=65), bd.DM05_ERR_UNSUPPORTED),        # G*S = 130 > 128
    (dict(Hkv=8, S=129), bd.DM05_ERR_UNSUPPORTED),
    (dict(q=FAKE + 8), bd.DM05_ERR_ALIGN),
    (dict(k_prefix=FAKE + 2), bd.DM05_ERR_ALIGN),
    (dict(v_suffix=FAKE + 4), bd.DM05_ERR_ALIGN),
    (dict(out=FAKE + 8), bd.DM05_ERR_ALIGN),
    (dict(lse=FAKE + 2), bd.DM05_ERR_ALIGN),
])
def test_host_checks_reject(lib, kw, status):
    assert call(**kw) == status


def test_prefix_pointers_optional_when_p_is_zero(lib):
    # P == 0 accepts NULL prefix pointers: the checks pass, so the call gets
    # as far as CUDA, which is absent here (or it launches on a GPU machine: not
    # in this CPU test).
    import torch
    if torch.cuda.is_available():
        pytest.skip("would launch on a GPU")
    assert call(P=0, k_prefix=None, v_prefix=None) == bd.DM05_ERR_CUDA


def test_workspace_bytes(lib):
    assert bd.dm05_suffix_attn_workspace_bytes(1, 8, 4, 1024, 50, 256) > 0
    assert bd.dm05_suffix_attn_workspace_bytes(1, 8, 4, 1024, 50, 128) == 0
    assert bd.dm05_suffix_attn_workspace_bytes(0, 8, 4, 1024, 50, 256) == 0


def test_split_override_values(lib):
    for v in range(0, 17):
        assert bd.dm05_set_split_override(v) == bd.DM05_OK
    for v in (17, 32, -1):
        assert bd.dm05_set_split_override(v) == bd.DM05_ERR_SHAPE
    assert bd.dm05_set_split_override(0) == bd.DM05_OK


def test_row_block_override_values(lib):
    for v in range(0, 17):
        assert bd.dm05_set_row_block_override(v) == bd.DM05_OK
    for v in (17, 32, -1):
        assert bd.dm05_set_row_block_override(v) == bd.DM05_ERR_SHAPE
    assert bd.dm05_set_row_block_override(0) == bd.DM05_OK


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(bd, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(bd, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        bd.lib()


def call_host(**kw):
    a = dict(q=FAKE, k_prefix=FAKE, v_prefix=FAKE, prefix_valid_len=None, prefix_mask=None,
             k_suffix=FAKE, v_suffix=FAKE, out=FAKE, lse=None, B=1, Hq=8, Hkv=4, P=1024, S=50, D=256,
             stream=None)
    a.update(kw)
    return bd.dm05_suffix_attn_host(a["q"], a["k_prefix"], a["v_prefix"], a["prefix_valid_len"],
                                    a["prefix_mask"], a["k_suffix"], a["v_suffix"], a["out"], a["lse"],
                                    a["B"], a["Hq"], a["Hkv"], a["P"], a["S"], a["D"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), bd.DM05_ERR_NULL),
    (dict(out=None), bd.DM05_ERR_NULL),
    (dict(v_prefix=None), bd.DM05_ERR_NULL),
    (dict(B=0), bd.DM05_ERR_SHAPE),
    (dict(Hq=6), bd.DM05_ERR_SHAPE),
    (dict(D=128), bd.DM05_ERR_UNSUPPORTED),
    (dict(S=65), bd.DM05_ERR_UNSUPPORTED),
])
def test_host_entry_checks_reject(lib, kw, status):
    # the host-buffer entry point checks its arguments before any CUDA call
    assert call_host(**kw) == status


def test_host_entry_takes_unaligned_host_buffers(lib):
    # host addresses need no alignment: an odd address passes the checks and
    # the call reaches CUDA (absent here)
    import torch
    if torch.cuda.is_available():
        pytest.skip("would copy from fake host addresses on a GPU")
    assert call_host(q=FAKE + 2, out=FAKE + 6, lse=FAKE + 1) == bd.DM05_ERR_CUDA


def expected_copy_bytes(valid_len, has_mask, want_lse, B, Hq, Hkv, P, S, D):
    """Bytes the host entry point moves, counted tensor by tensor: Q and the
    suffix K/V whole, the prefix K/V rows below the clamped valid length, the
    valid-length and mask arrays when given; O (and the LSE) back."""
    row = D * 2
    rows = [P] * B if valid_len is None else [min(max(int(v), 0), P) for v in valid_len]
    h2d = B * Hq * S * row                      # q
    h2d += 2 * B * Hkv * S * row                # k_suffix, v_suffix
    h2d += sum(2 * Hkv * n * row for n in rows)  # k_prefix, v_prefix rows in range
    h2d += 0 if valid_len is None else 4 * B
    h2d += B * P if has_mask else 0
    d2h = B * Hq * S * row + (B * Hq * S * 4 if want_lse else 0)
    return h2d, d2h


@pytest.mark.parametrize("valid_len,has_mask,want_lse,B,P,S", [
    (None, False, True, 1, 1024, 50),
    ([900], False, True, 1, 1024, 50),
    ([900], True, False, 1, 1024, 50),
    ([0], False, True, 1, 576, 10),
    ([-5, 2000, 700, 1024], True, True, 4, 1024, 50),   # clamped both ways
    (None, False, False, 2, 0, 10),
])
def test_host_copy_bytes(lib, valid_len, has_mask, want_lse, B, P, S):
    arr = None
    if valid_len is not None:
        arr = (ctypes.c_int32 * B)(*valid_len)
    rc, h2d, d2h = bd.dm05_suffix_attn_host_copy_bytes(
        None if arr is None else ctypes.addressof(arr), has_mask, want_lse, B, 8, 4, P, S, 256)
    assert rc == bd.DM05_OK
    assert (h2d, d2h) == expected_copy_bytes(valid_len, has_mask, want_lse, B, 8, 4, P, S, 256)


def test_host_copy_bytes_checks_sizes(lib):
    assert bd.dm05_suffix_attn_host_copy_bytes(None, 0, 1, 1, 8, 4, 1024, 50, 128)[0] == bd.DM05_ERR_UNSUPPORTED
    assert bd.dm05_suffix_attn_host_copy_bytes(None, 0, 1, 0, 8, 4, 1024, 50, 256)[0] == bd.DM05_ERR_SHAPE


def test_selftest_wait_timeout_checks_its_limit(lib):
    for bad in (0, -1, 2001):
        assert bd.dm05_selftest_wait_timeout(bad, None) == bd.DM05_ERR_SHAPE
    import torch
    if not torch.cuda.is_available():
        assert bd.dm05_selftest_wait_timeout(10, None) == bd.DM05_ERR_CUDA  # no device here


def _host_inputs(B=1, Hq=8, Hkv=4, P=64, S=10, D=256):
    import torch
    bf = torch.bfloat16
    return dict(q=torch.zeros(B, Hq, S, D, dtype=bf), k_prefix=torch.zeros(B, Hkv, P, D, dtype=bf),
                v_prefix=torch.zeros(B, Hkv, P, D, dtype=bf), k_suffix=torch.zeros(B, Hkv, S, D, dtype=bf),
                v_suffix=torch.zeros(B, Hkv, S, D, dtype=bf))


def _bad_host_argument(case):
    """One argument of a suffix_attn_host call made wrong, by name."""
    import torch
    return {
        "q": dict(q=torch.zeros(1, 8, 10, 256)),                                   # fp32
        "k_prefix": dict(k_prefix=torch.zeros(1, 4, 32, 256, dtype=torch.bfloat16)),  # P mismatch
        "v_suffix": dict(v_suffix=torch.zeros(1, 4, 256, 10, dtype=torch.bfloat16).transpose(2, 3)),
        "prefix_valid_len": dict(prefix_valid_len=torch.zeros(1, dtype=torch.int64)),
        "prefix_mask": dict(prefix_mask=torch.ones(1, 63, dtype=torch.uint8)),
        "out": dict(out=torch.zeros(1, 8, 10, 128, dtype=torch.bfloat16)),
        "lse": dict(lse=torch.zeros(1, 8, 10, dtype=torch.float64)),
    }[case]


@pytest.mark.parametrize("what", ["q", "k_prefix", "v_suffix", "prefix_valid_len", "prefix_mask", "out", "lse"])
def test_host_binding_rejects_bad_tensors(lib, what):
    # the binding checks CPU tensors before it calls the library
    a = _host_inputs()
    a.update(_bad_host_argument(what))
    q, kp, vp, ks, vs = a.pop("q"), a.pop("k_prefix"), a.pop("v_prefix"), a.pop("k_suffix"), a.pop("v_suffix")
    with pytest.raises(ValueError, match=what):
        bd.suffix_attn_host(q, kp, vp, ks, vs, **a)
