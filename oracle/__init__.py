"""fp64 CPU oracle for the DM0.5 action-expert (suffix) attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library in
``gqa_prefix_suffix_b200`` never imports it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, double precision); this module
only compiles it with gcc and marshals numpy arrays through ctypes.  What it
computes and the readings it takes are stated in the header of ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_default = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB, extra_flags=()) -> str:
    """Compile oracle.c into a shared library (gcc -O2, OpenMP, no fast-math)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", "-std=c11", *extra_flags, src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _bits(a) -> np.ndarray:
    """bf16 data as a contiguous uint16 bit-pattern array.

    Accepts a numpy uint16 array (already bit patterns) or a torch bfloat16
    tensor on the CPU."""
    if isinstance(a, np.ndarray):
        if a.dtype != np.uint16:
            raise TypeError("numpy inputs must be uint16 bf16 bit patterns")
        return np.ascontiguousarray(a)
    import torch  # local: the oracle itself needs only numpy
    if a.dtype != torch.bfloat16:
        raise TypeError("torch inputs must be bfloat16")
    return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes front end of one compiled copy of oracle.c."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        p = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_suffix_attn_range.argtypes = [p] * 9 + [i] * 6 + [i, i, i]
        lib.oracle_suffix_attn_range.restype = i
        lib.oracle_suffix_attn_rows.argtypes = [p] * 9 + [i] * 6 + [i, i, ctypes.c_long, ctypes.c_long, i]
        lib.oracle_suffix_attn_rows.restype = i
        lib.oracle_suffix_attn.argtypes = [p] * 9 + [i] * 6 + [i]
        lib.oracle_suffix_attn.restype = i
        lib.oracle_merge_parts.argtypes = [p, p, i, ctypes.c_long, i, p, p]
        lib.oracle_merge_parts.restype = i
        lib.oracle_prefix_causal_attn.argtypes = [p] * 6 + [i] * 6
        lib.oracle_prefix_causal_attn.restype = i
        lib.oracle_qkv_prologue.argtypes = [p] * 5 + [ctypes.c_double] * 2 + [p] * 3 + [i] * 7
        lib.oracle_qkv_prologue.restype = i
        lib.oracle_post_attention.argtypes = [p] * 8 + [ctypes.c_double, p] + [i] * 7
        lib.oracle_post_attention.restype = i
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = i
        self.lib = lib
        self.path = lib_path

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def suffix_attn(self, q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix,
                    v_suffix, B, Hq, Hkv, P, S, D, key_range=None, nthreads: int = 1,
                    row_range=None):
        """Return (out float64 [B,Hq,S,D], lse float64 [B,Hq,S]).

        key_range=(lo, hi) restricts the keys to the index-space slice [lo, hi)
        where [0, P) are prefix positions and [P, P+S) suffix positions.
        row_range=(lo, hi) computes only the flat query rows (b*Hq + h)*S + i
        in [lo, hi); the other rows of the result are left at zero."""
        qb, kpb, vpb = _bits(q), _bits(k_prefix), _bits(v_prefix)
        ksb, vsb = _bits(k_suffix), _bits(v_suffix)
        if qb.size != B * Hq * S * D or ksb.size != B * Hkv * S * D or vsb.size != B * Hkv * S * D:
            raise ValueError("q/k_suffix/v_suffix size does not match the dims")
        if kpb.size != B * Hkv * P * D or vpb.size != B * Hkv * P * D:
            raise ValueError("k_prefix/v_prefix size does not match the dims")
        vl = None
        if prefix_valid_len is not None:
            vl = np.ascontiguousarray(np.asarray(prefix_valid_len, dtype=np.int32).reshape(B))
        mk = None
        if prefix_mask is not None:
            mk = np.ascontiguousarray(np.asarray(prefix_mask, dtype=np.uint8).reshape(B, P))
        out = np.zeros((B, Hq, S, D), dtype=np.float64)
        lse = np.zeros((B, Hq, S), dtype=np.float64)
        lo, hi = (0, P + S) if key_range is None else key_range
        rlo, rhi = (0, B * Hq * S) if row_range is None else row_range
        rc = self.lib.oracle_suffix_attn_rows(
            _ptr(qb), _ptr(kpb), _ptr(vpb), _ptr(vl), _ptr(mk), _ptr(ksb), _ptr(vsb),
            _ptr(out), _ptr(lse), B, Hq, Hkv, P, S, D, int(lo), int(hi), int(rlo), int(rhi),
            int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle_suffix_attn_rows failed with status {rc}")
        return out, lse

    def merge_parts(self, o_parts, lse_parts):
        """Combine partial results over disjoint key sets (log-sum-exp identity).

        o_parts [n, rows, D] float64, lse_parts [n, rows] -> (out [rows, D], lse [rows])."""
        o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
        lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
        n, rows, D = o_parts.shape
        out = np.zeros((rows, D), dtype=np.float64)
        lse = np.zeros((rows,), dtype=np.float64)
        rc = self.lib.oracle_merge_parts(_ptr(o_parts), _ptr(lse_parts), n, rows, D,
                                         _ptr(out), _ptr(lse))
        if rc != 0:
            raise ValueError(f"oracle_merge_parts failed with status {rc}")
        return out, lse

    def prefix_causal_attn(self, q, k, v, valid_len, B, Hq, Hkv, P, D, nthreads: int = 1, fill=0.0):
        """Prefix-prefill attention under the prefix-causal mask.

        q [B,Hq,P,D], k/v [B,Hkv,P,D] (bf16 tensors or uint16 bit patterns),
        valid_len int32 [B] or None.  Returns (out float64 [B,Hq,P,D], lse
        float64 [B,Hq,P]); rows at or past a sample's valid length are not
        computed and keep the value `fill`."""
        qb, kb, vb = _bits(q), _bits(k), _bits(v)
        if qb.size != B * Hq * P * D or kb.size != B * Hkv * P * D or vb.size != B * Hkv * P * D:
            raise ValueError("q/k/v size does not match the dims")
        vl = None
        if valid_len is not None:
            vl = np.ascontiguousarray(np.asarray(valid_len, dtype=np.int32).reshape(B))
        out = np.full((B, Hq, P, D), fill, dtype=np.float64)
        lse = np.full((B, Hq, P), fill, dtype=np.float64)
        rc = self.lib.oracle_prefix_causal_attn(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(vl), _ptr(out), _ptr(lse),
                                                B, Hq, Hkv, P, D, int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle_prefix_causal_attn failed with status {rc}")
        return out, lse

    def qkv_prologue(self, x, w, qw, kw, pos, B, S, H, Hq, Hkv, D, eps=1e-6, theta=10000.0, nthreads: int = 1):
        """QKV projection + QK-Norm + RoPE of the suffix tokens.

        x [B*S, H], w [(Hq+2Hkv)*D, H], qw/kw [D] (bf16 tensors or uint16 bit
        patterns), pos int32 [B*S].  Returns float64 (q [B,Hq,S,D],
        k [B,Hkv,S,D], v [B,Hkv,S,D])."""
        xb, wb, qwb, kwb = _bits(x), _bits(w), _bits(qw), _bits(kw)
        if xb.size != B * S * H or wb.size != (Hq + 2 * Hkv) * D * H or qwb.size != D or kwb.size != D:
            raise ValueError("x/w/qw/kw size does not match the dims")
        pb = np.ascontiguousarray(np.asarray(pos, dtype=np.int32).reshape(B * S))
        q = np.zeros((B, Hq, S, D), dtype=np.float64)
        k = np.zeros((B, Hkv, S, D), dtype=np.float64)
        v = np.zeros((B, Hkv, S, D), dtype=np.float64)
        rc = self.lib.oracle_qkv_prologue(_ptr(xb), _ptr(wb), _ptr(qwb), _ptr(kwb), _ptr(pb), float(eps),
                                          float(theta), _ptr(q), _ptr(k), _ptr(v), B, S, H, Hq, Hkv, D,
                                          int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle_qkv_prologue failed with status {rc}")
        return q, k, v

    def post_attention(self, attn, h, scale, shift, gate, wo, wgu, wd, B, S, Hq, D, Hd, F, eps=1e-6,
                       nthreads: int = 1):
        """Output projection + residual, Adarms, GEGLU, MLP down and gated
        residual.  attn [B,Hq,S,D], h [B*S,Hd], scale/shift/gate [B,Hd],
        wo [Hd,Hq*D], wgu [2F,Hd], wd [Hd,F] (bf16 tensors or uint16 bit
        patterns).  Returns float64 out [B*S, Hd]."""
        arrs = [_bits(a) for a in (attn, h, scale, shift, gate, wo, wgu, wd)]
        sizes = [B * Hq * S * D, B * S * Hd, B * Hd, B * Hd, B * Hd, Hd * Hq * D, 2 * F * Hd, Hd * F]
        if any(a.size != n for a, n in zip(arrs, sizes)):
            raise ValueError("an input's size does not match the dims")
        out = np.zeros((B * S, Hd), dtype=np.float64)
        rc = self.lib.oracle_post_attention(*[_ptr(a) for a in arrs], float(eps), _ptr(out), B, S, Hq, D, Hd, F,
                                            int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle_post_attention failed with status {rc}")
        return out

    def inputs_call(self, inp, nthreads: int = 1, key_range=None, row_range=None):
        """Run on an object with the attributes of a SuffixAttnInputs."""
        return self.suffix_attn(inp.q, inp.k_prefix, inp.v_prefix, inp.prefix_valid_len,
                                inp.prefix_mask, inp.k_suffix, inp.v_suffix,
                                inp.B, inp.Hq, inp.Hkv, inp.P, inp.S, inp.D,
                                key_range=key_range, nthreads=nthreads, row_range=row_range)


def default() -> Oracle:
    """The oracle built from oracle.c next to this file (compiled on demand)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def max_threads() -> int:
    return default().max_threads()


def suffix_attn(*args, **kwargs):
    """Oracle.suffix_attn on the default build."""
    return default().suffix_attn(*args, **kwargs)


def merge_parts(o_parts, lse_parts):
    """Oracle.merge_parts on the default build."""
    return default().merge_parts(o_parts, lse_parts)


def post_attention(*args, **kwargs):
    """Oracle.post_attention on the default build."""
    return default().post_attention(*args, **kwargs)


def qkv_prologue(*args, **kwargs):
    """Oracle.qkv_prologue on the default build."""
    return default().qkv_prologue(*args, **kwargs)


def prefix_causal_attn(*args, **kwargs):
    """Oracle.prefix_causal_attn on the default build."""
    return default().prefix_causal_attn(*args, **kwargs)


def inputs_call(inp, nthreads: int = 1, key_range=None, row_range=None):
    """Oracle.inputs_call on the default build."""
    return default().inputs_call(inp, nthreads=nthreads, key_range=key_range, row_range=row_range)
