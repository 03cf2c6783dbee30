"""The allocation-free entry point against the allocating one.

dm05_suffix_attn_noalloc serves callers that must not allocate device memory
(for example a serving process that has reserved nearly all of HBM for its
KV cache, or a real-time control loop that cannot take cudaMalloc's implicit
synchronisation).  Its scratch, the kernel's error word and the partial
results of split calls, lives in one fixed 8 MiB array inside the library;
when a split's partials would not fit, the call uses fewer CTAs per
(sample, KV head).  This file is collected last on purpose: a run that stops
at the first failure has then already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
from gqa_prefix_suffix_b200 import binding as bd
from gqa_prefix_suffix_b200 import inputs as gen
from parity import check_close

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, LSE_ABS = 1e-2, 1e-3, 1e-3


def _ptr(t):
    return None if t is None else t.data_ptr()


@pytest.mark.parametrize("workload", ["base_chunk", "batched_mask"])
def test_noalloc_matches_allocating_entry_point(workload):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gqa_prefix_suffix_b200 import build
    build.build()
    d = gen.WORKLOADS[workload]().to("cuda")
    B, Hq, Hkv, P, S, D = d.B, d.Hq, d.Hkv, d.P, d.S, d.D
    stream = torch.cuda.current_stream().cuda_stream

    want_out, want_lse = bd.suffix_attn(d.q, d.k_prefix, d.v_prefix, d.k_suffix, d.v_suffix,
                                        prefix_valid_len=d.prefix_valid_len, prefix_mask=d.prefix_mask)
    torch.cuda.synchronize()

    for call in range(2):  # the first call does the per-device set-up, the second reuses it
        out = torch.full((B, Hq, S, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device="cuda")
        rc = bd.dm05_suffix_attn_noalloc(_ptr(d.q), _ptr(d.k_prefix), _ptr(d.v_prefix), _ptr(d.prefix_valid_len),
                                         _ptr(d.prefix_mask), _ptr(d.k_suffix), _ptr(d.v_suffix), _ptr(out),
                                         _ptr(lse), B, Hq, Hkv, P, S, D, stream)
        assert rc == bd.DM05_OK, bd.dm05_status_string(rc)
        torch.cuda.synchronize()
        err = (out.float() - want_out.float()).abs()
        assert bool(torch.isfinite(out.float()).all()), f"call {call}: non-finite output"
        assert float(err.max()) <= MAX_ABS, f"call {call}: max err {float(err.max())}"
        assert float(err.mean()) <= MEAN_ABS, f"call {call}: mean err {float(err.mean())}"
        lerr = (lse - want_lse).abs()
        assert float(lerr.max()) <= LSE_ABS, f"call {call}: lse err {float(lerr.max())}"


def test_noalloc_rejects_bad_arguments_before_launch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fake = 0x7f0000001000
    args = [fake, fake, fake, None, None, fake, fake, fake, None]
    assert bd.dm05_suffix_attn_noalloc(*args, 1, 8, 4, 1024, 50, 128, None) == bd.DM05_ERR_UNSUPPORTED
    assert bd.dm05_suffix_attn_noalloc(*args, 0, 8, 4, 1024, 50, 256, None) == bd.DM05_ERR_SHAPE
    bad = list(args)
    bad[0] = None
    assert bd.dm05_suffix_attn_noalloc(*bad, 1, 8, 4, 1024, 50, 256, None) == bd.DM05_ERR_NULL
    # the base-model chunk's split plan fits the fixed scratch array (8 MiB), so the
    # allocation-free call runs the same decomposition as the allocating one
    rc, splits, _, row_blocks = bd.dm05_suffix_attn_plan(1, 8, 4, 1024, 50, 256)
    assert rc == bd.DM05_OK
    sq = -(-50 // row_blocks)
    need = 256 + (4 * row_blocks * splits * 2 * sq * 1040 if splits > 1 else 0)
    np.testing.assert_equal(need <= 8 << 20, True)


PART_ROW_BYTES = 256 * 4 + 16   # one partial row: 256 fp32 of O and a float4 of statistics
SCRATCH_BYTES = 8 << 20


def _partial_bytes(units, splits, row_blocks, G, S):
    sq = -(-S // row_blocks)
    return units * row_blocks * splits * G * sq * PART_ROW_BYTES if splits > 1 else 0


def _call_noalloc(d, out, lse, stream):
    return bd.dm05_suffix_attn_noalloc(_ptr(d.q), _ptr(d.k_prefix), _ptr(d.v_prefix), _ptr(d.prefix_valid_len),
                                       _ptr(d.prefix_mask), _ptr(d.k_suffix), _ptr(d.v_suffix), _ptr(out),
                                       _ptr(lse), d.B, d.Hq, d.Hkv, d.P, d.S, d.D, stream)


@pytest.mark.parametrize("B", [2, 32])
def test_noalloc_uses_fewer_ctas_when_partials_do_not_fit(B):
    # With 16 CTAs per (sample, KV head) the partial results of B = 2 (about
    # 13 MB) or B = 32 (about 213 MB) do not fit the 8 MiB array: the call
    # halves the split count until they do (to 8 for B = 2, to 1 for B = 32)
    # and must still give the allocating entry point's result.
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inp = gen.make_inputs(B, 8, 4, 1024, 50, 256, 4100 + B, valid_range=(576, 1024), mask_frac=0.1,
                          peak_frac=0.01, peak_mult=4.0)
    d = inp.to("cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert bd.dm05_set_split_override(16) == bd.DM05_OK
    try:
        rc, splits, _, row_blocks = bd.dm05_suffix_attn_plan(B, 8, 4, 1024, 50, 256)
        assert rc == bd.DM05_OK and splits == 16
        assert _partial_bytes(B * 4, splits, row_blocks, 2, 50) > SCRATCH_BYTES - 256
        # the allocating call runs 16 splits, this one fewer: the two round
        # differently, so each is held to the oracle with the shared parity bar
        o_ref, l_ref = oracle.inputs_call(inp, nthreads=min(8, oracle.max_threads()))
        for call in range(2):
            out = torch.full((B, 8, 50, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
            lse = torch.full((B, 8, 50), float("nan"), dtype=torch.float32, device="cuda")
            assert _call_noalloc(d, out, lse, stream) == bd.DM05_OK
            torch.cuda.synchronize()
            rc, word = bd.dm05_get_error_word(stream)
            assert rc == bd.DM05_OK and word == 0, hex(word)
            assert bool(torch.isfinite(out.float()).all()), f"call {call}: non-finite output"
            check_close(out.cpu(), lse.cpu(), o_ref, l_ref, f"noalloc B={B} call {call}")
    finally:
        bd.dm05_set_split_override(0)


def test_noalloc_error_bits_are_readable():
    # A prefix_valid_len outside [0, P] is clamped and flagged in the fixed
    # array's error word; dm05_get_error_word returns the flag and clears it.
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inp = gen.make_inputs(2, 8, 4, 128, 10, 256, 4200, valid_len=[-3, 999])
    d = inp.to("cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert bd.dm05_get_error_word(stream)[0] == bd.DM05_OK  # clears earlier bits
    out = torch.empty((2, 8, 10, 256), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 8, 10), dtype=torch.float32, device="cuda")
    assert _call_noalloc(d, out, lse, stream) == bd.DM05_OK
    rc, word = bd.dm05_get_error_word(stream)
    assert rc == bd.DM05_OK and word & bd.DM05_EW_VALID_LEN_CLAMPED, hex(word)
    rc, word = bd.dm05_get_error_word(stream)
    assert rc == bd.DM05_OK and word == 0, "the bits must be cleared by the read"
    want_out, want_lse = bd.suffix_attn(d.q, d.k_prefix, d.v_prefix, d.k_suffix, d.v_suffix,
                                        prefix_valid_len=d.prefix_valid_len)
    torch.cuda.synchronize()
    assert float((out.float() - want_out.float()).abs().max()) <= MAX_ABS
    assert float((lse - want_lse).abs().max()) <= LSE_ABS
