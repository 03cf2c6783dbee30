"""The allocation-free entry point against the allocating one.

dm05_suffix_attn_noalloc serves callers that must not allocate device memory
(for example a serving process that has reserved nearly all of HBM for its
KV cache, or a real-time control loop that cannot take cudaMalloc's implicit
synchronisation).  It keeps its only scratch, the kernel's error word, in a
fixed array inside the library.  This file is collected last on purpose: a
run that stops at the first failure has then already run every other test.
"""
import numpy as np
import pytest
import torch

from gqa_prefix_suffix_b200 import binding as bd
from gqa_prefix_suffix_b200 import inputs as gen

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
