"""The suffix prologue (QKV projection + QK-Norm + RoPE, dm05_suffix_qkv_prologue)
against the fp64 oracle, element by element.

Tolerance: outputs are rounded once to bf16 from fp32 arithmetic (the
projection accumulates in fp32 over H products of bf16 values; the norm, the
angle reduction and the rotation add errors far below the rounding), so
every element is held to twice the bf16 rounding of its exact value plus a
small absolute floor: |out - y| <= 2^-8 |y| + 2e-3.  The mean error is held to
1.5x the mean error of the correctly rounded result (the normalised queries
and keys have |y| ~ 1, where correct rounding alone costs ~1e-3 on average),
and never more than 2e-3."""
import numpy as np
import pytest
import torch

import oracle
from gqa_prefix_suffix_b200 import binding as bd
from gqa_prefix_suffix_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gqa_prefix_suffix_b200 import build
    build.build()
    bd.lib()


def run_and_check(inp, what):
    d = inp.to("cuda")
    q, k, v = bd.suffix_qkv_prologue(d.x, d.w, d.qw, d.kw, d.pos, inp.B, inp.S, inp.Hq, inp.Hkv, inp.D)
    torch.cuda.synchronize()
    rc, word = bd.dm05_get_error_word(None)
    assert rc == 0 and word == 0, hex(word)
    want = oracle.qkv_prologue(inp.x, inp.w, inp.qw, inp.kw, inp.pos, inp.B, inp.S, inp.H, inp.Hq, inp.Hkv,
                               inp.D, nthreads=min(8, oracle.max_threads()))
    for got, ref, name in zip((q, k, v), want, "qkv"):
        g = got.float().cpu().double().numpy()
        err = np.abs(g - ref)
        bound = 2.0 ** -8 * np.abs(ref) + 2e-3
        assert (err <= bound).all(), (f"{what} {name}: {int((err > bound).sum())} elements over the bound, "
                                      f"max err {err.max():.4g} at |y|={np.abs(ref).flat[err.argmax()]:.3g}")
        floor = np.abs(torch.from_numpy(ref).to(torch.bfloat16).double().numpy() - ref).mean()
        assert err.mean() <= min(2e-3, 1.5 * floor), f"{what} {name}: mean err {err.mean():.3g}, floor {floor:.3g}"
        print(f"[{what} {name}] max err {err.max():.3g}, mean {err.mean():.3g} (rounding floor {floor:.3g})")
    return q, k, v


CASES = [
    # B, S, H, Hq, Hkv, positions start
    (1, 1, 1024, 8, 4, 0),
    (1, 10, 1024, 8, 4, 512),
    (3, 7, 1024, 8, 4, [5, 600, 2047]),
    (1, 65, 1024, 8, 4, 100),          # two 64-token tiles would be needed: one 128-token tile
    (2, 100, 1024, 8, 4, [0, 1900]),   # two 128-token tiles, the second ragged
    (1, 50, 64, 8, 4, 900),            # one K chunk
    (1, 50, 2048, 4, 4, 900),          # one query head per key head
    (1, 16, 1024, 8, 1, 7),            # one key head
    (1, 20, 768, 8, 4, 300),           # three 256-column groups (four-chunk stages, ring not wrapped)
    (2, 30, 1280, 8, 4, [11, 3000]),   # five groups: the three-stage ring wraps
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}_S{c[1]}_H{c[2]}_q{c[3]}kv{c[4]}" for c in CASES])
def test_prologue_shapes(case):
    B, S, H, Hq, Hkv, p0 = case
    inp = gen.make_prologue_inputs(B, S, 6100 + B * 31 + S, H=H, Hq=Hq, Hkv=Hkv, pos0=p0)
    run_and_check(inp, f"B={B} S={S} H={H}")


def test_prologue_base_chunk():
    run_and_check(gen.prologue_base(), "base chunk")


def test_prologue_batched():
    run_and_check(gen.prologue_batched(), "batched")


def test_prologue_feeds_the_suffix_attention():
    # the prologue's outputs are the suffix attention's q / k_suffix / v_suffix,
    # read straight from where the prologue wrote them
    pro = gen.prologue_base()
    att = gen.make_inputs(1, 8, 4, 1024, 50, 256, 6200, valid_len=900)
    dp, da = pro.to("cuda"), att.to("cuda")
    q, k, v = bd.suffix_qkv_prologue(dp.x, dp.w, dp.qw, dp.kw, dp.pos, 1, 50)
    out, lse = bd.suffix_attn(q, da.k_prefix, da.v_prefix, k, v, prefix_valid_len=da.prefix_valid_len)
    torch.cuda.synchronize()
    att.q, att.k_suffix, att.v_suffix = q.cpu(), k.cpu(), v.cpu()
    o_ref, l_ref = oracle.inputs_call(att, nthreads=8)
    from parity import check_close
    check_close(out.cpu(), lse.cpu(), o_ref, l_ref, "attention after the prologue")


def test_prologue_rejects_bad_arguments():
    fake = 0x7f0000001000
    a = [fake] * 8
    assert bd.dm05_suffix_qkv_prologue(*a, 1, 50, 1024, 8, 4, 128, 1e-6, 1e4, None) == bd.DM05_ERR_UNSUPPORTED
    assert bd.dm05_suffix_qkv_prologue(*a, 1, 50, 1000, 8, 4, 256, 1e-6, 1e4, None) == bd.DM05_ERR_UNSUPPORTED
    assert bd.dm05_suffix_qkv_prologue(*a, 0, 50, 1024, 8, 4, 256, 1e-6, 1e4, None) == bd.DM05_ERR_SHAPE
    assert bd.dm05_suffix_qkv_prologue(*a, 1, 50, 1024, 8, 4, 256, 0.0, 1e4, None) == bd.DM05_ERR_SHAPE
    b = list(a)
    b[0] = fake + 2
    assert bd.dm05_suffix_qkv_prologue(*b, 1, 50, 1024, 8, 4, 256, 1e-6, 1e4, None) == bd.DM05_ERR_ALIGN
    b = list(a)
    b[4] = None
    assert bd.dm05_suffix_qkv_prologue(*b, 1, 50, 1024, 8, 4, 256, 1e-6, 1e4, None) == bd.DM05_ERR_NULL
