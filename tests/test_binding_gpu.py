"""The CUDA-tensor front end (binding.suffix_attn) checks every tensor,
outputs included, before it calls the library: an output buffer that is too
small, strided, of the wrong type or on another device would otherwise be
overrun by the kernel."""
import pytest
import torch

from gqa_prefix_suffix_b200 import binding as bd

pytestmark = pytest.mark.gpu


def _inputs(B=1, Hq=8, Hkv=4, P=64, S=10, D=256):
    bf = torch.bfloat16
    dev = "cuda"
    return dict(q=torch.zeros(B, Hq, S, D, dtype=bf, device=dev),
                k_prefix=torch.zeros(B, Hkv, P, D, dtype=bf, device=dev),
                v_prefix=torch.zeros(B, Hkv, P, D, dtype=bf, device=dev),
                k_suffix=torch.zeros(B, Hkv, S, D, dtype=bf, device=dev),
                v_suffix=torch.zeros(B, Hkv, S, D, dtype=bf, device=dev))


def _bad(case):
    dev = "cuda"
    return {
        "out": dict(out=torch.zeros(1, 8, 10, 128, dtype=torch.bfloat16, device=dev)),             # too small
        "out ": dict(out=torch.zeros(1, 8, 256, 10, dtype=torch.bfloat16, device=dev).transpose(2, 3)),  # strided
        "lse": dict(lse=torch.zeros(1, 8, 10, dtype=torch.float64, device=dev)),                    # wrong dtype
        "lse ": dict(lse=torch.zeros(1, 8, 9, dtype=torch.float32, device=dev)),                    # too small
        "out  ": dict(out=torch.zeros(1, 8, 10, 256, dtype=torch.bfloat16)),                        # on the host
        "prefix_valid_len": dict(prefix_valid_len=torch.zeros(1, dtype=torch.int64, device=dev)),   # wrong dtype
        "prefix_valid_len ": dict(prefix_valid_len=torch.zeros(2, dtype=torch.int32, device=dev)),  # B + 1 values
        "prefix_mask": dict(prefix_mask=torch.ones(1, 63, dtype=torch.uint8, device=dev)),
    }[case]


@pytest.mark.parametrize("what", ["out", "out ", "out  ", "lse", "lse ", "prefix_valid_len", "prefix_valid_len ",
                                  "prefix_mask"])
def test_device_binding_rejects_bad_tensors(what):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    a = _inputs()
    a.update(_bad(what))
    q, kp, vp, ks, vs = a.pop("q"), a.pop("k_prefix"), a.pop("v_prefix"), a.pop("k_suffix"), a.pop("v_suffix")
    with pytest.raises(ValueError, match=what.strip()):
        bd.suffix_attn(q, kp, vp, ks, vs, **a)


def test_device_binding_rejects_a_strided_valid_len():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    a = _inputs(B=2)
    vl = torch.zeros(4, dtype=torch.int32, device="cuda")[::2]   # 2 values, stride 2
    with pytest.raises(ValueError, match="prefix_valid_len"):
        bd.suffix_attn(a["q"], a["k_prefix"], a["v_prefix"], a["k_suffix"], a["v_suffix"], prefix_valid_len=vl)
