"""ctypes binding of the C ABI in include/dm05_suffix_attn.h.

Argument marshalling only: every step of the attention runs in the CUDA
library.  If the library is missing the import of the entry points fails
loudly; there is no other implementation behind these names.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdm05_suffix_attn.so")

DM05_OK = 0
DM05_ERR_NULL = -1
DM05_ERR_SHAPE = -2
DM05_ERR_UNSUPPORTED = -3
DM05_ERR_ALIGN = -4
DM05_ERR_WORKSPACE = -5
DM05_ERR_CUDA = -6
DM05_EW_VALID_LEN_CLAMPED = 0x1
DM05_EW_WAIT_TIMEOUT = 0x2
DM05_EW_BAD_SPLIT = 0x4

DM05_FLAG_PREFIX_STATIC = 0x1

EXPORTS = ("dm05_suffix_attn", "dm05_suffix_attn_ex", "dm05_suffix_attn_workspace_bytes", "dm05_suffix_attn_reserve",
           "dm05_suffix_attn_plan", "dm05_set_split_override", "dm05_set_row_block_override",
           "dm05_get_error_word",
           "dm05_status_string", "dm05_release", "dm05_suffix_attn_noalloc", "dm05_suffix_attn_host",
           "dm05_suffix_attn_host_copy_bytes", "dm05_selftest_wait_timeout", "dm05_prefix_prefill_attn",
           "dm05_prefix_prefill_reserve", "dm05_prefix_prefill_plan", "dm05_suffix_qkv_prologue",
           "dm05_suffix_attn_steps_create", "dm05_suffix_attn_steps_launch", "dm05_suffix_attn_steps_destroy",
           "dm05_post_attention", "dm05_post_attention_reserve")

_lock = threading.Lock()
_lib = None


class Dm05Step(ctypes.Structure):
    """dm05_step: one call's own tensors (device addresses)."""
    _fields_ = [("q", ctypes.c_void_p), ("k_suffix", ctypes.c_void_p), ("v_suffix", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p)]


class Dm05Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {dm05_status_string(status)} ({status})" if what else
                         f"{dm05_status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m gqa_prefix_suffix_b200.build` (nvcc, sm_100a)")
            L = ctypes.CDLL(LIB_PATH)
            p, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            L.dm05_suffix_attn.argtypes = [p] * 9 + [i] * 6 + [p]
            L.dm05_suffix_attn.restype = i
            L.dm05_suffix_attn_ex.argtypes = [p] * 9 + [i] * 6 + [ctypes.c_uint, p]
            L.dm05_suffix_attn_ex.restype = i
            L.dm05_suffix_attn_workspace_bytes.argtypes = [i] * 6
            L.dm05_suffix_attn_workspace_bytes.restype = sz
            L.dm05_suffix_attn_reserve.argtypes = [i] * 6 + [p]
            L.dm05_suffix_attn_reserve.restype = i
            L.dm05_suffix_attn_plan.argtypes = [i] * 6 + [ctypes.POINTER(i)] * 3
            L.dm05_suffix_attn_plan.restype = i
            L.dm05_set_split_override.argtypes = [i]
            L.dm05_set_split_override.restype = i
            L.dm05_set_row_block_override.argtypes = [i]
            L.dm05_set_row_block_override.restype = i
            L.dm05_get_error_word.argtypes = [p, ctypes.POINTER(ctypes.c_uint32)]
            L.dm05_get_error_word.restype = i
            L.dm05_status_string.argtypes = [i]
            L.dm05_status_string.restype = ctypes.c_char_p
            L.dm05_release.argtypes = []
            L.dm05_release.restype = None
            L.dm05_suffix_attn_noalloc.argtypes = [p] * 9 + [i] * 6 + [p]
            L.dm05_suffix_attn_noalloc.restype = i
            L.dm05_suffix_attn_host.argtypes = [p] * 9 + [i] * 6 + [p]
            L.dm05_suffix_attn_host.restype = i
            L.dm05_suffix_attn_host_copy_bytes.argtypes = [p] + [i] * 8 + [ctypes.POINTER(sz)] * 2
            L.dm05_suffix_attn_host_copy_bytes.restype = i
            L.dm05_selftest_wait_timeout.argtypes = [i, p]
            L.dm05_selftest_wait_timeout.restype = i
            L.dm05_prefix_prefill_attn.argtypes = [p] * 6 + [i] * 5 + [p]
            L.dm05_prefix_prefill_attn.restype = i
            L.dm05_prefix_prefill_reserve.argtypes = [i] * 5 + [p]
            L.dm05_prefix_prefill_reserve.restype = i
            L.dm05_prefix_prefill_plan.argtypes = [i] * 5 + [ctypes.POINTER(i)] * 3
            L.dm05_prefix_prefill_plan.restype = i
            L.dm05_suffix_qkv_prologue.argtypes = [p] * 8 + [i] * 6 + [ctypes.c_float] * 2 + [p]
            L.dm05_suffix_qkv_prologue.restype = i
            L.dm05_suffix_attn_steps_create.argtypes = [ctypes.POINTER(Dm05Step), i] + [p] * 4 + [i] * 6 + \
                [ctypes.c_uint, ctypes.POINTER(p)]
            L.dm05_suffix_attn_steps_create.restype = i
            L.dm05_suffix_attn_steps_launch.argtypes = [p, p]
            L.dm05_suffix_attn_steps_launch.restype = i
            L.dm05_suffix_attn_steps_destroy.argtypes = [p]
            L.dm05_suffix_attn_steps_destroy.restype = i
            L.dm05_post_attention.argtypes = [p] * 9 + [i] * 6 + [ctypes.c_float, p]
            L.dm05_post_attention.restype = i
            L.dm05_post_attention_reserve.argtypes = [i] * 6 + [p]
            L.dm05_post_attention_reserve.restype = i
            _lib = L
    return _lib


# ---- the C entry points, same names, integer pointers ------------------------

def dm05_suffix_attn(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix, v_suffix,
                     out, lse, B, Hq, Hkv, P, S, D, stream) -> int:
    return lib().dm05_suffix_attn(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix,
                                  v_suffix, out, lse, B, Hq, Hkv, P, S, D, stream)


def dm05_suffix_attn_ex(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix, v_suffix,
                        out, lse, B, Hq, Hkv, P, S, D, flags, stream) -> int:
    """dm05_suffix_attn with option flags (DM05_FLAG_PREFIX_STATIC)."""
    return lib().dm05_suffix_attn_ex(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix,
                                     v_suffix, out, lse, B, Hq, Hkv, P, S, D, flags, stream)


def dm05_suffix_attn_noalloc(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix, v_suffix,
                             out, lse, B, Hq, Hkv, P, S, D, stream) -> int:
    """The allocation-free entry point (for callers that must not allocate
    device memory); same arguments as dm05_suffix_attn."""
    return lib().dm05_suffix_attn_noalloc(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix,
                                          v_suffix, out, lse, B, Hq, Hkv, P, S, D, stream)


def dm05_suffix_attn_host(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix, v_suffix,
                          out, lse, B, Hq, Hkv, P, S, D, stream) -> int:
    """The host-buffer entry point: every pointer is a host address."""
    return lib().dm05_suffix_attn_host(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix,
                                       v_suffix, out, lse, B, Hq, Hkv, P, S, D, stream)


def dm05_suffix_attn_host_copy_bytes(prefix_valid_len, has_prefix_mask, want_lse, B, Hq, Hkv, P, S, D):
    """Returns (status, host-to-device bytes, device-to-host bytes) of one
    dm05_suffix_attn_host call; prefix_valid_len is a host address or None."""
    h, d = ctypes.c_size_t(0), ctypes.c_size_t(0)
    rc = lib().dm05_suffix_attn_host_copy_bytes(prefix_valid_len, int(bool(has_prefix_mask)), int(bool(want_lse)),
                                                B, Hq, Hkv, P, S, D, ctypes.byref(h), ctypes.byref(d))
    return rc, int(h.value), int(d.value)


def dm05_prefix_prefill_attn(q, k, v, valid_len, out, lse, B, Hq, Hkv, P, D, stream) -> int:
    """The prefix-prefill attention under the prefix-causal mask."""
    return lib().dm05_prefix_prefill_attn(q, k, v, valid_len, out, lse, B, Hq, Hkv, P, D, stream)


def dm05_prefix_prefill_reserve(B, Hq, Hkv, P, D, stream) -> int:
    return lib().dm05_prefix_prefill_reserve(B, Hq, Hkv, P, D, stream)


def dm05_prefix_prefill_plan(B, Hq, Hkv, P, D):
    """Returns (status, splits_per_head, query_block, row_blocks)."""
    sp, qb, rb = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    rc = lib().dm05_prefix_prefill_plan(B, Hq, Hkv, P, D, ctypes.byref(sp), ctypes.byref(qb), ctypes.byref(rb))
    return rc, sp.value, qb.value, rb.value


def dm05_suffix_qkv_prologue(x, w, q_norm_w, k_norm_w, positions, q, k, v, B, S, H, Hq, Hkv, D, eps, theta,
                             stream) -> int:
    """QKV projection + QK-Norm + RoPE of the suffix tokens."""
    return lib().dm05_suffix_qkv_prologue(x, w, q_norm_w, k_norm_w, positions, q, k, v, B, S, H, Hq, Hkv, D,
                                          float(eps), float(theta), stream)


def dm05_suffix_attn_steps_create(steps, k_prefix, v_prefix, prefix_valid_len, prefix_mask, B, Hq, Hkv, P, S, D,
                                  flags=0):
    """steps: a list of (q, k_suffix, v_suffix, out, lse) device addresses.
    Returns (status, handle)."""
    arr = (Dm05Step * len(steps))(*[Dm05Step(*st) for st in steps])
    h = ctypes.c_void_p(0)
    rc = lib().dm05_suffix_attn_steps_create(arr, len(steps), k_prefix, v_prefix, prefix_valid_len, prefix_mask,
                                             B, Hq, Hkv, P, S, D, flags, ctypes.byref(h))
    return rc, h.value


def dm05_suffix_attn_steps_launch(handle, stream) -> int:
    return lib().dm05_suffix_attn_steps_launch(handle, stream)


def dm05_suffix_attn_steps_destroy(handle) -> int:
    return lib().dm05_suffix_attn_steps_destroy(handle)


def dm05_post_attention(attn, h, scale, shift, gate, wo, wgu, wd, out, B, S, Hq, D, Hd, F, eps, stream) -> int:
    """Output projection + residual, Adarms, GEGLU, MLP down + gated residual."""
    return lib().dm05_post_attention(attn, h, scale, shift, gate, wo, wgu, wd, out, B, S, Hq, D, Hd, F,
                                     float(eps), stream)


def dm05_post_attention_reserve(B, S, Hq, D, Hd, F, stream) -> int:
    return lib().dm05_post_attention_reserve(B, S, Hq, D, Hd, F, stream)


def post_attention(attn, h, scale, shift, gate, wo, wgu, wd, eps=1e-6, out=None, stream=None):
    """The post-attention block on CUDA torch tensors; returns out [B*S, Hd] bf16."""
    import torch
    B, Hq, S, D = attn.shape
    Hd = h.shape[1]
    F = wgu.shape[0] // 2
    for name, t, shape in (("attn", attn, (B, Hq, S, D)), ("h", h, (B * S, Hd)), ("scale", scale, (B, Hd)),
                           ("shift", shift, (B, Hd)), ("gate", gate, (B, Hd)), ("wo", wo, (Hd, Hq * D)),
                           ("wgu", wgu, (2 * F, Hd)), ("wd", wd, (Hd, F))):
        if (not t.is_cuda or t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous()
                or t.device != attn.device):
            raise ValueError(f"{name} must be a contiguous CUDA bfloat16 tensor {list(shape)} on {attn.device}")
    if out is None:
        out = torch.empty((B * S, Hd), dtype=torch.bfloat16, device=attn.device)
    if (not out.is_cuda or out.dtype != torch.bfloat16 or tuple(out.shape) != (B * S, Hd) or not out.is_contiguous()):
        raise ValueError(f"out must be a contiguous CUDA bfloat16 tensor {[B * S, Hd]}")
    rc = dm05_post_attention(attn.data_ptr(), h.data_ptr(), scale.data_ptr(), shift.data_ptr(), gate.data_ptr(),
                             wo.data_ptr(), wgu.data_ptr(), wd.data_ptr(), out.data_ptr(), B, S, Hq, D, Hd, F, eps,
                             _stream_handle(stream))
    if rc != DM05_OK:
        raise Dm05Error(rc, "dm05_post_attention")
    return out


def dm05_suffix_attn_workspace_bytes(B, Hq, Hkv, P, S, D) -> int:
    return int(lib().dm05_suffix_attn_workspace_bytes(B, Hq, Hkv, P, S, D))


def dm05_suffix_attn_reserve(B, Hq, Hkv, P, S, D, stream) -> int:
    return lib().dm05_suffix_attn_reserve(B, Hq, Hkv, P, S, D, stream)


def dm05_suffix_attn_plan(B, Hq, Hkv, P, S, D):
    """Returns (status, splits_per_head, tile_rows, row_blocks)."""
    sp, tr, rb = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    rc = lib().dm05_suffix_attn_plan(B, Hq, Hkv, P, S, D, ctypes.byref(sp), ctypes.byref(tr), ctypes.byref(rb))
    return rc, sp.value, tr.value, rb.value


def dm05_set_split_override(splits_per_head: int) -> int:
    return lib().dm05_set_split_override(splits_per_head)


def dm05_set_row_block_override(row_blocks: int) -> int:
    return lib().dm05_set_row_block_override(row_blocks)


def dm05_selftest_wait_timeout(limit_ms: int, stream) -> int:
    """Launches the bounded-wait self-test (a wait that must run out)."""
    return lib().dm05_selftest_wait_timeout(limit_ms, stream)


def dm05_get_error_word(stream):
    """Returns (status, error bits); synchronises the stream and clears the bits."""
    w = ctypes.c_uint32(0)
    rc = lib().dm05_get_error_word(stream, ctypes.byref(w))
    return rc, int(w.value)


def dm05_status_string(status: int) -> str:
    return lib().dm05_status_string(status).decode()


def dm05_release() -> None:
    lib().dm05_release()


# ---- torch front end (marshalling only) -------------------------------------

def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def suffix_attn(q, k_prefix, v_prefix, k_suffix, v_suffix, prefix_valid_len=None, prefix_mask=None,
                out=None, lse=None, want_lse: bool = True, stream=None, prefix_static: bool = False):
    """Suffix attention on CUDA torch tensors; returns (out, lse or None).

    q [B,Hq,S,D] bf16; k_prefix/v_prefix [B,Hkv,P,D] bf16; k_suffix/v_suffix
    [B,Hkv,S,D] bf16; prefix_valid_len int32 [B] or None; prefix_mask uint8
    [B,P] or None.  out (bf16 [B,Hq,S,D]) and lse (fp32 [B,Hq,S]) are
    allocated when not given."""
    import torch
    B, Hq, S, D = q.shape
    Hkv, P = k_prefix.shape[1], k_prefix.shape[2]
    for name, t, dt in (("q", q, torch.bfloat16), ("k_prefix", k_prefix, torch.bfloat16),
                        ("v_prefix", v_prefix, torch.bfloat16), ("k_suffix", k_suffix, torch.bfloat16),
                        ("v_suffix", v_suffix, torch.bfloat16)):
        if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor")
    if tuple(k_prefix.shape) != (B, Hkv, P, D) or tuple(v_prefix.shape) != (B, Hkv, P, D):
        raise ValueError("k_prefix/v_prefix must be [B,Hkv,P,D]")
    if tuple(k_suffix.shape) != (B, Hkv, S, D) or tuple(v_suffix.shape) != (B, Hkv, S, D):
        raise ValueError("k_suffix/v_suffix must be [B,Hkv,S,D]")
    if prefix_valid_len is not None:
        if (not prefix_valid_len.is_cuda or prefix_valid_len.dtype != torch.int32 or prefix_valid_len.numel() != B
                or not prefix_valid_len.is_contiguous()):
            raise ValueError("prefix_valid_len must be a contiguous CUDA int32 tensor of B values")
    if prefix_mask is not None:
        if (not prefix_mask.is_cuda or prefix_mask.dtype != torch.uint8 or tuple(prefix_mask.shape) != (B, P)
                or not prefix_mask.is_contiguous()):
            raise ValueError("prefix_mask must be a contiguous CUDA uint8 tensor [B,P]")
    if out is None:
        out = torch.empty((B, Hq, S, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    # the library writes B*Hq*S rows through these pointers: a smaller or
    # strided buffer would be overrun
    for name, t, shape, dt in (("out", out, (B, Hq, S, D), torch.bfloat16), ("lse", lse, (B, Hq, S), torch.float32)):
        if t is not None and (not t.is_cuda or t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor {list(shape)}")
    for name, t in (("k_prefix", k_prefix), ("v_prefix", v_prefix), ("k_suffix", k_suffix), ("v_suffix", v_suffix),
                    ("prefix_valid_len", prefix_valid_len), ("prefix_mask", prefix_mask), ("out", out), ("lse", lse)):
        if t is not None and t.device != q.device:
            raise ValueError(f"{name} must be on {q.device} like q")
    ptr = lambda t: None if t is None else t.data_ptr()
    rc = dm05_suffix_attn_ex(ptr(q), ptr(k_prefix), ptr(v_prefix), ptr(prefix_valid_len), ptr(prefix_mask),
                             ptr(k_suffix), ptr(v_suffix), ptr(out), ptr(lse), B, Hq, Hkv, P, S, D,
                             DM05_FLAG_PREFIX_STATIC if prefix_static else 0, _stream_handle(stream))
    if rc != DM05_OK:
        raise Dm05Error(rc, "dm05_suffix_attn")
    return out, lse


def suffix_attn_host(q, k_prefix, v_prefix, k_suffix, v_suffix, prefix_valid_len=None, prefix_mask=None,
                     out=None, lse=None, want_lse: bool = True, stream=None):
    """Suffix attention on CPU torch tensors (page-locked for asynchronous
    copies) through dm05_suffix_attn_host; returns (out, lse or None), host
    tensors that hold the result once `stream` has passed the call.

    Shapes and dtypes are those of suffix_attn; every tensor, out and lse
    included, must be a contiguous CPU tensor."""
    import torch
    B, Hq, S, D = q.shape
    Hkv, P = k_prefix.shape[1], k_prefix.shape[2]
    for name, t, dt in (("q", q, torch.bfloat16), ("k_prefix", k_prefix, torch.bfloat16),
                        ("v_prefix", v_prefix, torch.bfloat16), ("k_suffix", k_suffix, torch.bfloat16),
                        ("v_suffix", v_suffix, torch.bfloat16)):
        if t.is_cuda or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU {dt} tensor")
    if tuple(k_prefix.shape) != (B, Hkv, P, D) or tuple(v_prefix.shape) != (B, Hkv, P, D):
        raise ValueError("k_prefix/v_prefix must be [B,Hkv,P,D]")
    if tuple(k_suffix.shape) != (B, Hkv, S, D) or tuple(v_suffix.shape) != (B, Hkv, S, D):
        raise ValueError("k_suffix/v_suffix must be [B,Hkv,S,D]")
    if prefix_valid_len is not None and (prefix_valid_len.is_cuda or prefix_valid_len.dtype != torch.int32
                                         or prefix_valid_len.numel() != B or not prefix_valid_len.is_contiguous()):
        raise ValueError("prefix_valid_len must be a contiguous CPU int32 tensor of B values")
    if prefix_mask is not None and (prefix_mask.is_cuda or prefix_mask.dtype != torch.uint8
                                    or tuple(prefix_mask.shape) != (B, P) or not prefix_mask.is_contiguous()):
        raise ValueError("prefix_mask must be a contiguous CPU uint8 tensor [B,P]")
    pin = q.is_pinned()
    if out is None:
        out = torch.empty((B, Hq, S, D), dtype=torch.bfloat16, pin_memory=pin)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, pin_memory=pin)
    for name, t, shape, dt in (("out", out, (B, Hq, S, D), torch.bfloat16), ("lse", lse, (B, Hq, S), torch.float32)):
        if t is not None and (t.is_cuda or t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CPU {dt} tensor {list(shape)}")
    ptr = lambda t: None if t is None else t.data_ptr()
    rc = dm05_suffix_attn_host(ptr(q), ptr(k_prefix), ptr(v_prefix), ptr(prefix_valid_len), ptr(prefix_mask),
                               ptr(k_suffix), ptr(v_suffix), ptr(out), ptr(lse), B, Hq, Hkv, P, S, D,
                               _stream_handle(stream))
    if rc != DM05_OK:
        raise Dm05Error(rc, "dm05_suffix_attn_host")
    return out, lse


def prefix_prefill_attn(q, k, v, valid_len=None, out=None, lse=None, want_lse: bool = True, stream=None):
    """Prefix-prefill attention on CUDA torch tensors; returns (out, lse or None).

    q [B,Hq,P,D] bf16; k/v [B,Hkv,P,D] bf16; valid_len int32 [B] or None.
    Rows at or past a sample's valid length are not written (a fresh out /
    lse is allocated uninitialised when not given)."""
    import torch
    B, Hq, P, D = q.shape
    Hkv = k.shape[1]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bfloat16 tensor")
    if tuple(k.shape) != (B, Hkv, P, D) or tuple(v.shape) != (B, Hkv, P, D):
        raise ValueError("k/v must be [B,Hkv,P,D]")
    if valid_len is not None and (not valid_len.is_cuda or valid_len.dtype != torch.int32 or valid_len.numel() != B
                                  or not valid_len.is_contiguous()):
        raise ValueError("valid_len must be a contiguous CUDA int32 tensor of B values")
    if out is None:
        out = torch.empty((B, Hq, P, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, P), dtype=torch.float32, device=q.device)
    for name, t, shape, dt in (("out", out, (B, Hq, P, D), torch.bfloat16), ("lse", lse, (B, Hq, P), torch.float32)):
        if t is not None and (not t.is_cuda or t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor {list(shape)}")
    for name, t in (("k", k), ("v", v), ("valid_len", valid_len), ("out", out), ("lse", lse)):
        if t is not None and t.device != q.device:
            raise ValueError(f"{name} must be on {q.device} like q")
    ptr = lambda t: None if t is None else t.data_ptr()
    rc = dm05_prefix_prefill_attn(ptr(q), ptr(k), ptr(v), ptr(valid_len), ptr(out), ptr(lse), B, Hq, Hkv, P, D,
                                  _stream_handle(stream))
    if rc != DM05_OK:
        raise Dm05Error(rc, "dm05_prefix_prefill_attn")
    return out, lse


def suffix_qkv_prologue(x, w, q_norm_w, k_norm_w, positions, B, S, Hq=8, Hkv=4, D=256, eps=1e-6, theta=10000.0,
                        q=None, k=None, v=None, stream=None):
    """QKV projection + QK-Norm + RoPE on CUDA torch tensors; returns (q, k, v)
    in the suffix attention's layout.  x [B*S, H] bf16, w [(Hq+2Hkv)*D, H]
    bf16, norm weights [D] bf16, positions int32 [B*S]."""
    import torch
    H = x.shape[1]
    for name, t, shape, dt in (("x", x, (B * S, H), torch.bfloat16), ("w", w, ((Hq + 2 * Hkv) * D, H), torch.bfloat16),
                               ("q_norm_w", q_norm_w, (D,), torch.bfloat16), ("k_norm_w", k_norm_w, (D,), torch.bfloat16),
                               ("positions", positions, (B * S,), torch.int32)):
        if not t.is_cuda or t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous() or t.device != x.device:
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor {list(shape)} on {x.device}")
    if q is None:
        q = torch.empty((B, Hq, S, D), dtype=torch.bfloat16, device=x.device)
    if k is None:
        k = torch.empty((B, Hkv, S, D), dtype=torch.bfloat16, device=x.device)
    if v is None:
        v = torch.empty((B, Hkv, S, D), dtype=torch.bfloat16, device=x.device)
    for name, t, shape in (("q", q, (B, Hq, S, D)), ("k", k, (B, Hkv, S, D)), ("v", v, (B, Hkv, S, D))):
        if not t.is_cuda or t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bfloat16 tensor {list(shape)}")
    rc = dm05_suffix_qkv_prologue(x.data_ptr(), w.data_ptr(), q_norm_w.data_ptr(), k_norm_w.data_ptr(),
                                  positions.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(), B, S, H, Hq, Hkv, D,
                                  eps, theta, _stream_handle(stream))
    if rc != DM05_OK:
        raise Dm05Error(rc, "dm05_suffix_qkv_prologue")
    return q, k, v


def reserve_for(q, k_prefix, stream=None) -> None:
    """dm05_suffix_attn_reserve for the sizes of these tensors (call before graph capture)."""
    B, Hq, S, D = q.shape
    rc = dm05_suffix_attn_reserve(B, Hq, k_prefix.shape[1], k_prefix.shape[2], S, D, _stream_handle(stream))
    if rc != DM05_OK:
        raise Dm05Error(rc, "dm05_suffix_attn_reserve")
