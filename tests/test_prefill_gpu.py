"""Prefix-prefill attention under the prefix-causal mask (the CUDA path
through dm05_prefix_prefill_attn) against the fp64 oracle, element by element
on the rows below each sample's valid length, with the tolerance stated in
parity.py.  Rows at or past the valid length must be left untouched."""
import numpy as np
import pytest
import torch

import oracle
from gqa_prefix_suffix_b200 import binding as bd
from gqa_prefix_suffix_b200 import inputs as gen
from parity import check_close

pytestmark = pytest.mark.gpu

SENTINEL = -3.0


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gqa_prefix_suffix_b200 import build
    build.build()
    bd.lib()
    yield
    bd.dm05_set_split_override(0)


def run_prefill(inp, splits=0):
    d = inp.to("cuda")
    out = torch.full((d.B, d.Hq, d.P, d.D), SENTINEL, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((d.B, d.Hq, d.P), SENTINEL, dtype=torch.float32, device="cuda")
    assert bd.dm05_set_split_override(splits) == 0
    try:
        bd.prefix_prefill_attn(d.q, d.k, d.v, valid_len=d.valid_len, out=out, lse=lse)
        torch.cuda.synchronize()
    finally:
        bd.dm05_set_split_override(0)
    rc, word = bd.dm05_get_error_word(None)
    assert rc == 0
    return out.cpu(), lse.cpu(), word


def check_prefill(inp, out, lse, what):
    o_ref, l_ref = oracle.prefix_causal_attn(inp.q, inp.k, inp.v, inp.valid_len, inp.B, inp.Hq, inp.Hkv, inp.P,
                                             inp.D, nthreads=min(8, oracle.max_threads()))
    for b in range(inp.B):
        vl = inp.P if inp.valid_len is None else max(0, min(inp.P, int(inp.valid_len[b])))
        if vl > 0:
            # few keys in the first rows: the mean bound follows the rounding floor there
            check_close(out[b:b + 1, :, :vl], lse[b:b + 1, :, :vl], o_ref[b:b + 1, :, :vl], l_ref[b:b + 1, :, :vl],
                        f"{what} sample {b} (valid {vl})", keys=1)
        assert bool((out[b, :, vl:].float() == SENTINEL).all()), f"{what}: padding rows of sample {b} written"
        assert bool((lse[b, :, vl:] == SENTINEL).all()), f"{what}: padding lse of sample {b} written"


SHAPES = [
    # name, B, Hq, Hkv, P, valid (None | list)
    ("p1", 1, 8, 4, 1, None),
    ("p7_g2", 2, 8, 4, 7, [7, 3]),
    ("p63", 1, 8, 4, 63, [63]),
    ("p64", 1, 8, 4, 64, None),
    ("p65", 2, 8, 4, 65, [65, 64]),
    ("p127_g1", 1, 4, 4, 127, [100]),
    ("p200_g4", 2, 8, 2, 200, [200, 129]),
    ("p150_g8", 1, 8, 1, 150, [150]),
    ("p300_zero", 2, 8, 4, 300, [0, 300]),
    ("p333_rand", 3, 8, 4, 333, "rand"),
]


@pytest.mark.parametrize("case", SHAPES, ids=[c[0] for c in SHAPES])
def test_prefill_shapes(case):
    name, B, Hq, Hkv, P, valid = case
    kw = {"valid_range": (0, P)} if valid == "rand" else {"valid_len": valid}
    inp = gen.make_prefill_inputs(B, Hq, Hkv, P, 256, 600 + P + B, name=name, **kw)
    out, lse, word = run_prefill(inp)
    assert word == 0
    check_prefill(inp, out, lse, name)


@pytest.mark.parametrize("splits", [1, 2, 4, 8, 16])
def test_prefill_every_split_count(splits):
    inp = gen.make_prefill_inputs(1, 8, 4, 640, 256, 700, valid_len=600)
    out, lse, word = run_prefill(inp, splits=splits)
    assert word == 0
    check_prefill(inp, out, lse, f"splits={splits}")


def test_prefill_rows_past_valid_len_are_never_read():
    inp = gen.make_prefill_inputs(2, 8, 4, 256, 256, 701, valid_len=[200, 77])
    want = run_prefill(inp)
    for b, vl in enumerate((200, 77)):
        inp.k[b, :, vl:] = float("nan")
        inp.v[b, :, vl:] = float("nan")
        inp.q[b, :, vl:] = float("nan")
    out, lse, _ = run_prefill(inp)
    check_prefill(inp, out, lse, "nan padding")
    assert torch.equal(out.view(torch.int16), want[0].view(torch.int16))


def test_prefill_valid_len_clamped_and_flagged():
    inp = gen.make_prefill_inputs(2, 8, 4, 96, 256, 702, valid_len=[-4, 1000])
    out, lse, word = run_prefill(inp)
    assert word & bd.DM05_EW_VALID_LEN_CLAMPED
    check_prefill(inp, out, lse, "clamped")


def test_prefill_base_prefix():
    inp = gen.prefill_base()
    out, lse, word = run_prefill(inp)
    assert word == 0
    check_prefill(inp, out, lse, inp.name)


def test_prefill_history_prefix():
    inp = gen.prefill_history()
    out, lse, word = run_prefill(inp)
    assert word == 0
    check_prefill(inp, out, lse, inp.name)


def test_prefill_then_suffix_on_the_same_cache():
    # the prefill's K/V are the cache the suffix call reads next: both calls
    # on one stream, the suffix one checked against the oracle
    pre = gen.prefill_base()
    suf = gen.make_inputs(1, 8, 4, 1024, 50, 256, 703, valid_len=900, prefix=(pre.k, pre.v))
    dp, ds = pre.to("cuda"), suf.to("cuda")
    out_p, _ = bd.prefix_prefill_attn(dp.q, dp.k, dp.v, valid_len=dp.valid_len)
    out_s, lse_s = bd.suffix_attn(ds.q, dp.k, dp.v, ds.k_suffix, ds.v_suffix, prefix_valid_len=ds.prefix_valid_len)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.inputs_call(suf, nthreads=8)
    check_close(out_s.cpu(), lse_s.cpu(), o_ref, l_ref, "suffix after prefill")


def test_prefill_rejects_bad_arguments():
    fake = 0x7f0000001000
    a = [fake, fake, fake, None, fake, None]
    assert bd.dm05_prefix_prefill_attn(*a, 1, 8, 4, 64, 128, None) == bd.DM05_ERR_UNSUPPORTED
    assert bd.dm05_prefix_prefill_attn(*a, 1, 8, 4, 0, 256, None) == bd.DM05_ERR_SHAPE
    assert bd.dm05_prefix_prefill_attn(*a, 1, 6, 4, 64, 256, None) == bd.DM05_ERR_SHAPE
    assert bd.dm05_prefix_prefill_attn(*a, 1, 32, 1, 64, 256, None) == bd.DM05_ERR_UNSUPPORTED
    b = list(a)
    b[0] = fake + 8
    assert bd.dm05_prefix_prefill_attn(*b, 1, 8, 4, 64, 256, None) == bd.DM05_ERR_ALIGN
    b = list(a)
    b[2] = None
    assert bd.dm05_prefix_prefill_attn(*b, 1, 8, 4, 64, 256, None) == bd.DM05_ERR_NULL
