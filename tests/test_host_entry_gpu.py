"""The host-buffer entry point (dm05_suffix_attn_host) on the GPU.

It copies the inputs in, runs the same kernel with the same work
decomposition as dm05_suffix_attn, and copies the result back, so its output
must equal the device entry point's bit for bit; a few cases are also held
to the fp64 oracle directly.  Prefix rows past the valid length are not
copied, so NaN there on the host, and stale data left in the staging buffer
by an earlier call, must not reach the result.
"""
import numpy as np
import pytest
import torch

from gqa_prefix_suffix_b200 import binding as bd
from gqa_prefix_suffix_b200 import inputs as gen

from test_parity_gpu import check_close, ref, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gqa_prefix_suffix_b200 import build
    build.build()
    bd.lib()
    yield


def run_host(inp, pinned=True, with_lse=True, stream=None):
    h = inp.tensors()
    if pinned:
        h = {k: (None if v is None else v.pin_memory()) for k, v in h.items()}
    out, lse = bd.suffix_attn_host(h["q"], h["k_prefix"], h["v_prefix"], h["k_suffix"], h["v_suffix"],
                                   prefix_valid_len=h["prefix_valid_len"], prefix_mask=h["prefix_mask"],
                                   want_lse=with_lse, stream=stream)
    if stream is None:
        torch.cuda.current_stream().synchronize()
    else:
        stream.synchronize()
    rc, word = bd.dm05_get_error_word(None if stream is None else stream.cuda_stream)
    assert rc == 0
    return out, lse, word


def same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.int16), b.contiguous().view(torch.int16))


CASES = [
    # name, B, Hq, Hkv, P, S, valid_len (None | list | "rand"), mask_frac
    ("base_shape", 1, 8, 4, 1024, 50, [900], 0.0),
    ("libero_shape", 1, 8, 4, 576, 10, [512], 0.0),
    ("no_valid_len", 2, 8, 4, 200, 20, None, 0.0),
    ("whole_buckets", 3, 8, 4, 130, 16, [130, 130, 130], 0.1),
    ("mixed_runs", 5, 8, 4, 257, 30, [257, 0, 257, 257, 100], 0.1),
    ("ragged_batch", 8, 8, 4, 640, 50, "rand", 0.1),
    ("no_prefix", 2, 8, 4, 0, 10, None, 0.0),
]


def make_case(name, B, Hq, Hkv, P, S, valid, mask_frac, seed=31):
    kw = {}
    if valid == "rand":
        kw["valid_range"] = (0, P)
    elif valid is not None:
        kw["valid_len"] = valid
    return gen.make_inputs(B, Hq, Hkv, P, S, 256, seed + len(name), mask_frac=mask_frac, name=name, **kw)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_host_entry_equals_device_entry(case):
    inp = make_case(*case)
    o_h, l_h, _ = run_host(inp)
    o_d, l_d, _ = run_gpu(inp)
    assert same_bits(o_h, o_d), case[0]
    assert torch.equal(l_h, l_d), case[0]


@pytest.mark.parametrize("case", [CASES[0], CASES[5]], ids=[CASES[0][0], CASES[5][0]])
def test_host_entry_against_oracle(case):
    inp = make_case(*case)
    o_ref, l_ref = ref(inp)
    out, lse, _ = run_host(inp)
    check_close(out, lse, o_ref, l_ref, f"host entry {case[0]}")


def test_host_rows_past_valid_len_are_not_copied():
    # a first call fills the staging buffer with finite rows; the second
    # copies fewer rows and has NaN past each valid length on the host
    full = gen.make_inputs(2, 8, 4, 300, 20, 256, 41, valid_len=[300, 300])
    run_host(full)
    inp = gen.make_inputs(2, 8, 4, 300, 20, 256, 42, valid_len=[170, 3], mask_frac=0.1)
    o_ref, l_ref = ref(inp)
    for b, vl in enumerate((170, 3)):
        inp.k_prefix[b, :, vl:] = float("nan")
        inp.v_prefix[b, :, vl:] = float("nan")
    out, lse, _ = run_host(inp)
    assert torch.isfinite(out.float()).all()
    check_close(out, lse, o_ref, l_ref, "host entry, NaN past valid_len")


def test_host_valid_len_out_of_range_is_clamped_and_flagged():
    inp = gen.make_inputs(2, 8, 4, 128, 10, 256, 43, valid_len=[-5, 500])
    out, lse, word = run_host(inp)
    assert word & bd.DM05_EW_VALID_LEN_CLAMPED
    o_ref, l_ref = ref(inp)
    check_close(out, lse, o_ref, l_ref, "host entry, clamped")


def test_host_entry_pageable_and_no_lse():
    inp = make_case(*CASES[0])
    o_p, l_p, _ = run_host(inp, pinned=False, with_lse=False)
    assert l_p is None
    o_d, _, _ = run_gpu(inp)
    assert same_bits(o_p, o_d)


def test_host_entry_staging_grows_and_shrinks():
    small = make_case(*CASES[1])
    big = make_case(*CASES[5])
    s = torch.cuda.Stream()
    results = []
    for inp in (small, big, small, big):
        o, l, _ = run_host(inp, stream=s)
        results.append((o, l))
    assert same_bits(results[0][0], results[2][0]) and torch.equal(results[0][1], results[2][1])
    assert same_bits(results[1][0], results[3][0]) and torch.equal(results[1][1], results[3][1])
    o_d, l_d, _ = run_gpu(big)
    assert same_bits(results[3][0], o_d)


def test_host_entry_refuses_capture():
    inp = make_case(*CASES[1])
    h = {k: (None if v is None else v.pin_memory()) for k, v in inp.tensors().items()}
    out = torch.empty((1, 8, 10, 256), dtype=torch.bfloat16).pin_memory()
    s = torch.cuda.Stream()
    x = torch.zeros(16, device="cuda")
    g = torch.cuda.CUDAGraph()
    ptr = lambda t: None if t is None else t.data_ptr()
    with torch.cuda.graph(g, stream=s):
        x.add_(1.0)
        rc = bd.dm05_suffix_attn_host(ptr(h["q"]), ptr(h["k_prefix"]), ptr(h["v_prefix"]),
                                      ptr(h["prefix_valid_len"]), None, ptr(h["k_suffix"]), ptr(h["v_suffix"]),
                                      ptr(out), None, 1, 8, 4, 576, 10, 256, s.cuda_stream)
    assert rc == bd.DM05_ERR_UNSUPPORTED
    g.replay()
    torch.cuda.synchronize()
    assert float(x[0]) == 1.0
    del g


def test_host_copy_bytes_match_the_copies():
    inp = make_case(*CASES[5])
    vl = inp.prefix_valid_len
    rc, h2d, d2h = bd.dm05_suffix_attn_host_copy_bytes(vl.data_ptr(), True, True, inp.B, 8, 4, inp.P, inp.S, 256)
    assert rc == 0
    rows = np.clip(vl.numpy(), 0, inp.P)
    kv = int(rows.sum()) * 4 * 2 * 512
    assert h2d == inp.q.numel() * 2 + inp.k_suffix.numel() * 4 + kv + 4 * inp.B + inp.prefix_mask.numel()
    assert d2h == inp.q.numel() * 2 + inp.B * 8 * inp.S * 4


def pinned_view(shape, dtype, offset, pad=256, fill=0xA5):
    """A contiguous view at byte `offset` inside a larger page-locked buffer
    filled with a guard pattern; returns (view, whole buffer)."""
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((offset + n + pad,), fill, dtype=torch.uint8).pin_memory()
    return buf[offset:offset + n].view(dtype).view(shape), buf


@pytest.mark.parametrize("out_off,lse_off,pin_lse", [
    (16, 4, True),      # device writes O and the LSE straight into the views
    (48, 12, True),
    (8, 4, True),       # O not 16-byte aligned: staging and a copy back
    (16, 4, False),     # LSE pageable: staging and a copy back for both
])
def test_host_entry_output_buffers(out_off, lse_off, pin_lse):
    inp = make_case(*CASES[5])
    B, Hq, S = inp.B, inp.Hq, inp.S
    h = {k: (None if v is None else v.pin_memory()) for k, v in inp.tensors().items()}
    out, out_buf = pinned_view((B, Hq, S, 256), torch.bfloat16, out_off)
    if pin_lse:
        lse, lse_buf = pinned_view((B, Hq, S), torch.float32, lse_off)
    else:
        lse_buf = torch.full((lse_off + B * Hq * S * 4 + 256,), 0xA5, dtype=torch.uint8)
        lse = lse_buf[lse_off:lse_off + B * Hq * S * 4].view(torch.float32).view(B, Hq, S)
    bd.suffix_attn_host(h["q"], h["k_prefix"], h["v_prefix"], h["k_suffix"], h["v_suffix"],
                        prefix_valid_len=h["prefix_valid_len"], prefix_mask=h["prefix_mask"], out=out, lse=lse)
    torch.cuda.synchronize()
    o_d, l_d, _ = run_gpu(inp)
    assert same_bits(out, o_d)
    assert torch.equal(lse, l_d)
    n_out = out.numel() * 2
    assert (out_buf[:out_off] == 0xA5).all() and (out_buf[out_off + n_out:] == 0xA5).all()
    n_lse = lse.numel() * 4
    assert (lse_buf[:lse_off] == 0xA5).all() and (lse_buf[lse_off + n_lse:] == 0xA5).all()


def test_release_then_call_again():
    # dm05_release frees the staging buffers and workspaces; the next calls
    # (host and device entry points) allocate them again
    inp = make_case(*CASES[0])
    o1, l1, _ = run_host(inp)
    torch.cuda.synchronize()
    bd.dm05_release()
    o2, l2, _ = run_host(inp)
    o3, l3, _ = run_gpu(inp)
    assert same_bits(o1, o2) and torch.equal(l1, l2)
    assert same_bits(o2, o3) and torch.equal(l2, l3)
