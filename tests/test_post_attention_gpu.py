"""The post-attention block (dm05_post_attention: output projection + residual,
Adarms, GEGLU, MLP down + gated residual) against the fp64 oracle, element by
element.

Tolerance: the kernels accumulate in fp32, but the two GEMM inputs built on
the way (u, the Adarms output, and m, the GEGLU output) are rounded to bf16
before their projections (the tensor cores' input type), and out is rounded
once to bf16.  The rounding of u and m perturbs each projection by about
2^-9 of its terms' size, spread over their K terms; at the workloads' scale
(every projection O(1)) this stays below the output rounding.  Bound: every
element |out - ref| <= 2^-7 |ref| + 1e-2, and the mean error at most twice the
mean error of the correctly rounded result plus 1e-3."""
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
    out = bd.post_attention(d.attn, d.h, d.scale, d.shift, d.gate, d.wo, d.wgu, d.wd)
    torch.cuda.synchronize()
    rc, word = bd.dm05_get_error_word(None)
    assert rc == 0 and word == 0, hex(word)
    ref = oracle.post_attention(inp.attn, inp.h, inp.scale, inp.shift, inp.gate, inp.wo, inp.wgu, inp.wd, inp.B,
                                inp.S, inp.Hq, inp.D, inp.Hd, inp.F, nthreads=min(16, oracle.max_threads()))
    g = out.float().cpu().double().numpy()
    err = np.abs(g - ref)
    floor = np.abs(torch.from_numpy(ref).to(torch.bfloat16).double().numpy() - ref).mean()
    bound = 2.0 ** -7 * np.abs(ref) + 1e-2
    print(f"[{what}] max err {err.max():.4g}, mean {err.mean():.4g} (rounding floor {floor:.4g}), "
          f"max |ref| {np.abs(ref).max():.3g}")
    assert (err <= bound).all(), f"{what}: {int((err > bound).sum())} elements over the bound, max {err.max():.4g}"
    assert err.mean() <= 2.0 * floor + 1e-3, f"{what}: mean err {err.mean():.4g}"


CASES = [
    # B, S, Hq, D, Hd, F
    (1, 1, 2, 64, 128, 64),
    (2, 7, 2, 128, 256, 320),
    (1, 50, 8, 256, 1024, 4096),
    (3, 70, 4, 64, 256, 512),       # S > 64: two token tiles per sample
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}_S{c[1]}_Hq{c[2]}_D{c[3]}_Hd{c[4]}_F{c[5]}" for c in CASES])
def test_post_attention_shapes(case):
    B, S, Hq, D, Hd, F = case
    inp = gen.make_post_inputs(B, S, 8100 + B * 7 + S, Hq=Hq, D=D, Hd=Hd, F=F)
    run_and_check(inp, f"B={B} S={S} Hd={Hd} F={F}")


def test_post_attention_batched():
    run_and_check(gen.post_batched(), "batched B=32")


def test_post_attention_is_deterministic():
    d = gen.post_base().to("cuda")
    a = bd.post_attention(d.attn, d.h, d.scale, d.shift, d.gate, d.wo, d.wgu, d.wd)
    b = bd.post_attention(d.attn, d.h, d.scale, d.shift, d.gate, d.wo, d.wgu, d.wd)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_post_attention_rejects_bad_arguments():
    fake = 0x7f0000001000
    a = [fake] * 9
    assert bd.dm05_post_attention(*a, 1, 50, 8, 256, 1000, 4096, 1e-6, None) == bd.DM05_ERR_UNSUPPORTED
    assert bd.dm05_post_attention(*a, 1, 50, 8, 100, 1024, 4096, 1e-6, None) == bd.DM05_ERR_UNSUPPORTED
    assert bd.dm05_post_attention(*a, 0, 50, 8, 256, 1024, 4096, 1e-6, None) == bd.DM05_ERR_SHAPE
    b = list(a)
    b[0] = fake + 8
    assert bd.dm05_post_attention(*b, 1, 50, 8, 256, 1024, 4096, 1e-6, None) == bd.DM05_ERR_ALIGN
    b = list(a)
    b[5] = None
    assert bd.dm05_post_attention(*b, 1, 50, 8, 256, 1024, 4096, 1e-6, None) == bd.DM05_ERR_NULL
