"""Thin ctypes binding over ``libattn_b200.so`` (C ABI in ``include/attn.h``).

Argument marshalling only: tensors are checked for dtype/device/contiguity, their data pointers and
the current CUDA stream are passed to the C entry points, and a non-zero status becomes an
``AttnError``. PyTorch supplies device memory and streams; every step of the attention itself runs
in the library's kernels. There is no fallback: if the library is missing the call fails.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_NAME = "libattn_b200.so"
library_path = os.path.join(_PKG, LIB_NAME)

ATTN_OK = 0
STATUS_NAMES = {
    0: "ATTN_OK", -1: "ATTN_ERR_NULL", -2: "ATTN_ERR_SHAPE", -3: "ATTN_ERR_GQA", -4: "ATTN_ERR_HEADDIM",
    -5: "ATTN_ERR_ALIGN", -6: "ATTN_ERR_CAUSAL_SQ_GT_SKV", -7: "ATTN_ERR_ARCH", -8: "ATTN_ERR_WORKSPACE",
    -9: "ATTN_ERR_LAUNCH", -10: "ATTN_ERR_DEVICE_TIMEOUT", -11: "ATTN_ERR_SCALE", -12: "ATTN_ERR_CUDA",
    -13: "ATTN_ERR_SCRATCH_LIMIT",
}
EXPORTED = ("attn_fwd", "attn_fwd_ex", "attn_fwd_host", "attn_fwd_strided", "attn_decode_ctas", "attn_status_string", "attn_version",
            "attn_device_status", "attn_decode_noalloc", "attn_decode_paged", "attn_prefill_paged", "attn_bwd", "attn_decode_fp8", "attn_prefill_fp8",
            "attn_decode_paged_fp8", "attn_lse_merge")

_lock = threading.Lock()
_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def load_library(path: str | None = None):
    """Load the library once. Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or library_path
        if not os.path.exists(p):
            raise RuntimeError(f"{LIB_NAME} is not built (expected at {p}); "
                               "run `python -m causal_attention_attn_b200.build`")
        lib = ctypes.CDLL(p)
        i, f, vp = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        lib.attn_fwd.restype = i
        lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
        lib.attn_fwd_ex.restype = i
        lib.attn_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp]
        lib.attn_fwd_host.restype = i
        lib.attn_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
        ll3 = ctypes.POINTER(ctypes.c_longlong)
        lib.attn_fwd_strided.restype = i
        lib.attn_fwd_strided.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, ll3, ll3, ll3, ll3, f, i, vp]
        lib.attn_decode_ctas.restype = i
        lib.attn_decode_ctas.argtypes = [i, i, i, i, i]
        lib.attn_status_string.restype = ctypes.c_char_p
        lib.attn_status_string.argtypes = [i]
        lib.attn_version.restype = i
        lib.attn_version.argtypes = []
        lib.attn_device_status.restype = i
        lib.attn_device_status.argtypes = [vp]
        lib.attn_decode_noalloc.restype = i
        lib.attn_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
        lib.attn_decode_paged.restype = i
        lib.attn_bwd.restype = i
        lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
        lib.attn_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp]
        lib.attn_prefill_paged.restype = i
        lib.attn_prefill_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, i, vp]
        lib.attn_decode_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
        lib.attn_prefill_fp8.restype = i
        lib.attn_prefill_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
        lib.attn_decode_paged_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp]
        lib.attn_lse_merge.restype = i
        lib.attn_lse_merge.argtypes = [vp, vp, vp, vp, vp, ctypes.c_longlong, i, vp]
        if path is None:
            _lib = lib
        return lib


def status_string(status: int) -> str:
    return load_library().attn_status_string(int(status)).decode()


def _check(status: int):
    if status != ATTN_OK:
        raise AttnError(status, status_string(status))


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check_tensor(name, t, dtype, ndim):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_rows(name, t, dtype):
    """A [batch, head, row, dim] tensor in any layout whose last (dim) axis is contiguous."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if t.dim() != 4:
        raise ValueError(f"{name} must have 4 dims, got {tuple(t.shape)}")
    if t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name} must have a contiguous last (head-dim) axis")


def _strides3(t):
    """(batch, head, row) element strides of a [B, H, S, D] view; an axis of extent 1 gets D
    (its stride is never used, and the library wants a multiple of 8)."""
    D = int(t.shape[-1])
    return tuple(int(t.stride(i)) if t.shape[i] > 1 else D for i in range(3))


def attn_fwd_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, Hq: int, Hkv: int,
                 Sq: int, Skv: int, D: int, scale: float, causal: bool, stream: int = 0,
                 decode_ctas: int = 0) -> int:
    """Call the C entry point with raw pointers; returns the status code (no exception)."""
    lib = load_library()
    if decode_ctas:
        return lib.attn_fwd_ex(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, Hq, Hkv, Sq, Skv, D, float(scale),
                               int(causal), int(decode_ctas), stream)
    return lib.attn_fwd(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, Hq, Hkv, Sq, Skv, D, float(scale), int(causal),
                        stream)


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None, causal: bool = True,
             out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None,
             decode_ctas: int = 0):
    """Fused causal attention forward on the GPU.

    q: [B, Hq, Sq, D], k/v: [B, Hkv, Skv, D], bf16, on one CUDA device, each either contiguous or any
    view with a contiguous last axis (e.g. a token-major [B, S, H, D] tensor passed as
    ``x.transpose(1, 2)``); views go through ``attn_fwd_strided``. ``out`` (shape of q) may be such a
    view too. Returns (o [B, Hq, Sq, D] bf16, lse [B, Hq, Sq] fp32, contiguous). ``scale``
    defaults to 1/sqrt(D).
    """
    _check_rows("q", q, torch.bfloat16)
    _check_rows("k", k, torch.bfloat16)
    _check_rows("v", v, torch.bfloat16)
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Skv, Dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or Dk != D:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    else:
        _check_rows("out", out, torch.bfloat16)
        if out.shape != q.shape:
            raise ValueError("out must have the shape of q")
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    else:
        _check_tensor("lse", lse, torch.float32, 3)
        if tuple(lse.shape) != (B, Hq, Sq):
            raise ValueError("lse must be [B, Hq, Sq]")
    strided = not all(t.is_contiguous() for t in (q, k, v, out))
    with torch.cuda.device(q.device):
        if strided:
            arr = [(ctypes.c_longlong * 3)(*_strides3(t)) for t in (q, k, v, out)]
            rc = load_library().attn_fwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                                 lse.data_ptr(), B, Hq, Hkv, Sq, Skv, D, *arr, float(scale),
                                                 int(causal), _stream_handle(stream))
        else:
            rc = attn_fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv,
                              Sq, Skv, D, scale, causal, _stream_handle(stream), decode_ctas)
    _check(rc)
    return out, lse


def attn_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
                  causal: bool = True, device="cuda", stream=None, out_host=None, lse_host=None, dev_bufs=None):
    """End-to-end call on HOST tensors through ``attn_fwd_host``: the library copies q, k, v in,
    runs the attention and copies o and lse out, slice by slice, with the copies of one slice
    overlapping the attention of the next (so pinned inputs and outputs matter: pageable memory
    works but does not overlap).

    ``dev_bufs`` optionally supplies the device staging tensors (q, k, v, o, lse) so that a loop of
    calls does not allocate. Returns host (o, lse); the call synchronises on the stream before
    returning.
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu" or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a bf16 host tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [batch, head, row, dim] tensor")
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Hkv, Skv, D) or tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"k {tuple(k.shape)} / v {tuple(v.shape)} do not match q {tuple(q.shape)}")
    if scale is None:
        scale = D ** -0.5
    stream = stream or torch.cuda.current_stream(device)
    if dev_bufs is None:
        dev_bufs = (torch.empty(q.shape, dtype=torch.bfloat16, device=device),
                    torch.empty(k.shape, dtype=torch.bfloat16, device=device),
                    torch.empty(v.shape, dtype=torch.bfloat16, device=device),
                    torch.empty(q.shape, dtype=torch.bfloat16, device=device),
                    torch.empty((B, Hq, Sq), dtype=torch.float32, device=device))
    qd, kd, vd, od, ld = dev_bufs
    if out_host is None:
        out_host = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    if lse_host is None:
        lse_host = torch.empty((B, Hq, Sq), dtype=torch.float32, pin_memory=True)
    for name, t in (("out_host", out_host), ("lse_host", lse_host)):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor")
    rc = load_library().attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out_host.data_ptr(),
                                      lse_host.data_ptr(), qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                                      ld.data_ptr(), B, Hq, Hkv, Sq, Skv, D, float(scale), int(bool(causal)),
                                      _stream_handle(stream))
    _check(rc)
    stream.synchronize()
    return out_host, lse_host


def attn_decode_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
                        out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Single-token decode through ``attn_decode_noalloc``: the library allocates nothing (its
    scratch is a fixed device array). For callers that must not have the library call cudaMalloc.
    ``out`` and ``lse`` should be passed by such callers; when omitted they are created here with
    torch. q: [B, Hq, 1, D]; k/v: [B, Hkv, Skv, D]. Returns (o, lse)."""
    _check_tensor("q", q, torch.bfloat16, 4)
    _check_tensor("k", k, torch.bfloat16, 4)
    _check_tensor("v", v, torch.bfloat16, 4)
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Skv, Dk = k.shape
    if Sq != 1 or tuple(v.shape) != tuple(k.shape) or Bk != B or Dk != D:
        raise ValueError(f"expected q [B,Hq,1,D] and k, v [B,Hkv,Skv,D]; got {tuple(q.shape)}, {tuple(k.shape)}")
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, 4)
    _check_tensor("lse", lse, torch.float32, 3)
    with torch.cuda.device(q.device):
        rc = load_library().attn_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                                lse.data_ptr(), B, Hq, Hkv, Skv, D, float(scale),
                                                _stream_handle(stream))
    _check(rc)
    return out, lse


def attn_decode_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, block_table: torch.Tensor,
                      seq_lens: torch.Tensor, max_seq_len: int, scale: float | None = None,
                      out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None,
                      decode_ctas: int = 0):
    """Single-token decode over a paged, variable-length KV cache through ``attn_decode_paged``.
    q: [B, Hq, 1, 128] bf16; k_pages, v_pages: [num_pages, Hkv, page_size, 128] bf16;
    block_table: int32 [B, pages_per_seq]; seq_lens: int32 [B] (all on the GPU); max_seq_len: a
    host-side bound of the lengths. Returns (o [B, Hq, 1, 128], lse [B, Hq, 1])."""
    _check_tensor("q", q, torch.bfloat16, 4)
    _check_tensor("k_pages", k_pages, torch.bfloat16, 4)
    _check_tensor("v_pages", v_pages, torch.bfloat16, 4)
    _check_tensor("block_table", block_table, torch.int32, 2)
    _check_tensor("seq_lens", seq_lens, torch.int32, 1)
    B, Hq, Sq, D = q.shape
    num_pages, Hkv, page_size, Dk = k_pages.shape
    if Sq != 1 or tuple(v_pages.shape) != tuple(k_pages.shape) or Dk != D:
        raise ValueError(f"expected q [B,Hq,1,D] and k, v pages [P,Hkv,page,D]; got {tuple(q.shape)}, "
                         f"{tuple(k_pages.shape)}")
    if block_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("block_table and seq_lens need one row / entry per batch element")
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, 4)
    _check_tensor("lse", lse, torch.float32, 3)
    with torch.cuda.device(q.device):
        rc = load_library().attn_decode_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                              block_table.data_ptr(), seq_lens.data_ptr(), out.data_ptr(),
                                              lse.data_ptr(), B, Hq, Hkv, num_pages, page_size,
                                              int(block_table.shape[1]), int(max_seq_len), float(scale),
                                              int(decode_ctas), _stream_handle(stream))
    _check(rc)
    return out, lse


def attn_prefill_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, block_table: torch.Tensor,
                       seq_lens: torch.Tensor, max_seq_len: int, scale: float | None = None, causal: bool = True,
                       out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Chunked prefill over a paged, variable-length KV cache through ``attn_prefill_paged``:
    sequence b's Sq new queries attend to its first seq_lens[b] cached keys, the causal mask aligned
    to the last Sq of them. q: [B, Hq, Sq, 128] bf16; k_pages, v_pages: [num_pages, Hkv, page_size,
    128] bf16; block_table int32 [B, pages_per_seq]; seq_lens int32 [B] (all on the GPU).
    Returns (o [B, Hq, Sq, 128], lse [B, Hq, Sq])."""
    _check_tensor("q", q, torch.bfloat16, 4)
    _check_tensor("k_pages", k_pages, torch.bfloat16, 4)
    _check_tensor("v_pages", v_pages, torch.bfloat16, 4)
    _check_tensor("block_table", block_table, torch.int32, 2)
    _check_tensor("seq_lens", seq_lens, torch.int32, 1)
    B, Hq, Sq, D = q.shape
    num_pages, Hkv, page_size, Dk = k_pages.shape
    if tuple(v_pages.shape) != tuple(k_pages.shape) or Dk != D:
        raise ValueError(f"expected q [B,Hq,Sq,D] and k, v pages [P,Hkv,page,D]; got {tuple(q.shape)}, "
                         f"{tuple(k_pages.shape)}")
    if block_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("block_table and seq_lens need one row / entry per batch element")
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, 4)
    _check_tensor("lse", lse, torch.float32, 3)
    with torch.cuda.device(q.device):
        rc = load_library().attn_prefill_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                               block_table.data_ptr(), seq_lens.data_ptr(), out.data_ptr(),
                                               lse.data_ptr(), B, Hq, Hkv, Sq, num_pages, page_size,
                                               int(block_table.shape[1]), int(max_seq_len), float(scale),
                                               int(bool(causal)), _stream_handle(stream))
    _check(rc)
    return out, lse


def _as_codes(name, t):
    """e4m3 codes: a uint8 tensor, or a float8_e4m3fn tensor viewed as its bytes."""
    if isinstance(t, torch.Tensor) and t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    _check_tensor(name, t, torch.uint8, 4)
    return t


def attn_decode_fp8(q: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor, k_scale: torch.Tensor,
                    v_scale: torch.Tensor, scale: float | None = None, out: torch.Tensor | None = None,
                    lse: torch.Tensor | None = None, stream=None, decode_ctas: int = 0):
    """Single-token decode over an e4m3 K/V cache through ``attn_decode_fp8``.
    q: [B, Hq, 1, 128] bf16; k8, v8: [B, Hkv, Skv, 128] e4m3 codes (uint8 or float8_e4m3fn);
    k_scale, v_scale: fp32 [Hkv, 128] (value = code * coefficient). Returns (o, lse)."""
    _check_tensor("q", q, torch.bfloat16, 4)
    k8, v8 = _as_codes("k8", k8), _as_codes("v8", v8)
    _check_tensor("k_scale", k_scale, torch.float32, 2)
    _check_tensor("v_scale", v_scale, torch.float32, 2)
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Skv, Dk = k8.shape
    if Sq != 1 or tuple(v8.shape) != tuple(k8.shape) or Bk != B or Dk != D \
            or tuple(k_scale.shape) != (Hkv, D) or tuple(v_scale.shape) != (Hkv, D):
        raise ValueError("expected q [B,Hq,1,D], k8, v8 [B,Hkv,Skv,D] and scales [Hkv,D]")
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, 4)
    _check_tensor("lse", lse, torch.float32, 3)
    with torch.cuda.device(q.device):
        rc = load_library().attn_decode_fp8(q.data_ptr(), k8.data_ptr(), v8.data_ptr(), k_scale.data_ptr(),
                                            v_scale.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Skv, D,
                                            float(scale), int(decode_ctas), _stream_handle(stream))
    _check(rc)
    return out, lse


def attn_prefill_fp8(q: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor, k_scale: torch.Tensor,
                     v_scale: torch.Tensor, scale: float | None = None, causal: bool = True,
                     out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Attention of Sq queries over an e4m3 K/V cache through ``attn_prefill_fp8`` (the causal mask
    aligned to the last Sq keys). q: [B, Hq, Sq, 128] bf16; k8, v8: [B, Hkv, Skv, 128] e4m3 codes
    (uint8 or float8_e4m3fn); k_scale, v_scale: fp32 [Hkv, 128]. Returns (o, lse)."""
    _check_tensor("q", q, torch.bfloat16, 4)
    k8, v8 = _as_codes("k8", k8), _as_codes("v8", v8)
    _check_tensor("k_scale", k_scale, torch.float32, 2)
    _check_tensor("v_scale", v_scale, torch.float32, 2)
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Skv, Dk = k8.shape
    if tuple(v8.shape) != tuple(k8.shape) or Bk != B or Dk != D \
            or tuple(k_scale.shape) != (Hkv, D) or tuple(v_scale.shape) != (Hkv, D):
        raise ValueError("expected q [B,Hq,Sq,D], k8, v8 [B,Hkv,Skv,D] and scales [Hkv,D]")
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, 4)
    _check_tensor("lse", lse, torch.float32, 3)
    with torch.cuda.device(q.device):
        rc = load_library().attn_prefill_fp8(q.data_ptr(), k8.data_ptr(), v8.data_ptr(), k_scale.data_ptr(),
                                             v_scale.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Sq, Skv,
                                             D, float(scale), int(bool(causal)), _stream_handle(stream))
    _check(rc)
    return out, lse


def attn_decode_paged_fp8(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, k_scale: torch.Tensor,
                          v_scale: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int,
                          scale: float | None = None, out: torch.Tensor | None = None,
                          lse: torch.Tensor | None = None, stream=None, decode_ctas: int = 0):
    """attn_decode_paged over e4m3 pages: k_pages, v_pages [num_pages, Hkv, page_size, 128] e4m3
    codes; k_scale, v_scale fp32 [Hkv, 128]; the rest as :func:`attn_decode_paged`."""
    _check_tensor("q", q, torch.bfloat16, 4)
    k_pages, v_pages = _as_codes("k_pages", k_pages), _as_codes("v_pages", v_pages)
    _check_tensor("k_scale", k_scale, torch.float32, 2)
    _check_tensor("v_scale", v_scale, torch.float32, 2)
    _check_tensor("block_table", block_table, torch.int32, 2)
    _check_tensor("seq_lens", seq_lens, torch.int32, 1)
    B, Hq, Sq, D = q.shape
    num_pages, Hkv, page_size, Dk = k_pages.shape
    if Sq != 1 or tuple(v_pages.shape) != tuple(k_pages.shape) or Dk != D \
            or tuple(k_scale.shape) != (Hkv, D) or tuple(v_scale.shape) != (Hkv, D):
        raise ValueError("expected q [B,Hq,1,D], pages [P,Hkv,page,D] and scales [Hkv,D]")
    if block_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("block_table and seq_lens need one row / entry per batch element")
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, 4)
    _check_tensor("lse", lse, torch.float32, 3)
    with torch.cuda.device(q.device):
        rc = load_library().attn_decode_paged_fp8(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                                  k_scale.data_ptr(), v_scale.data_ptr(), block_table.data_ptr(),
                                                  seq_lens.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv,
                                                  num_pages, page_size, int(block_table.shape[1]), int(max_seq_len),
                                                  float(scale), int(decode_ctas), _stream_handle(stream))
    _check(rc)
    return out, lse


def attn_lse_merge(o_acc: torch.Tensor, lse_acc: torch.Tensor, o_part: torch.Tensor, lse_part: torch.Tensor,
                   out: torch.Tensor | None = None, stream=None):
    """Merge one attention result over a block of keys (o_part bf16 [..., D], lse_part fp32 [...])
    into a running result (o_acc fp32, lse_acc fp32, same shapes; updated in place) through
    ``attn_lse_merge``. ``out`` (bf16, shape of o_part) optionally receives the merged O."""
    _check_tensor("o_part", o_part, torch.bfloat16, o_part.dim())
    _check_tensor("o_acc", o_acc, torch.float32, o_part.dim())
    _check_tensor("lse_part", lse_part, torch.float32, o_part.dim() - 1)
    _check_tensor("lse_acc", lse_acc, torch.float32, o_part.dim() - 1)
    if o_acc.shape != o_part.shape or lse_acc.shape != lse_part.shape or tuple(lse_part.shape) != tuple(o_part.shape[:-1]):
        raise ValueError("o_acc, o_part [..., D] and lse_acc, lse_part [...] must agree")
    if out is not None:
        _check_tensor("out", out, torch.bfloat16, o_part.dim())
        if out.shape != o_part.shape:
            raise ValueError("out must have the shape of o_part")
    D = int(o_part.shape[-1])
    rows = o_part.numel() // D if D else 0
    with torch.cuda.device(o_part.device):
        rc = load_library().attn_lse_merge(o_acc.data_ptr(), lse_acc.data_ptr(), o_part.data_ptr(), lse_part.data_ptr(),
                                           out.data_ptr() if out is not None else None, rows, D,
                                           _stream_handle(stream))
    _check(rc)
    return o_acc, lse_acc


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
             dout: torch.Tensor, scale: float | None = None, causal: bool = True, dq: torch.Tensor | None = None,
             dk: torch.Tensor | None = None, dv: torch.Tensor | None = None, stream=None):
    """Backward pass through ``attn_bwd``: gradients for q, k, v given dout = dL/do, the forward's
    inputs and its outputs o and lse. Head dim 128. Returns (dq, dk, dv), bf16."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_tensor(name, t, torch.bfloat16, 4)
    _check_tensor("lse", lse, torch.float32, 3)
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Skv, Dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or Dk != D or tuple(o.shape) != tuple(q.shape) \
            or tuple(dout.shape) != tuple(q.shape) or tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("shapes of q, k, v, o, lse, dout disagree")
    if scale is None:
        scale = D ** -0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    with torch.cuda.device(q.device):
        rc = load_library().attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                     lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Sq, Skv, D,
                                     float(scale), int(bool(causal)), _stream_handle(stream))
    _check(rc)
    return dq, dk, dv


def decode_ctas(B: int, Hq: int, Hkv: int, Skv: int, D: int) -> int:
    """Number of CTAs attn_fwd launches for a decode of this shape on the current device."""
    rc = load_library().attn_decode_ctas(B, Hq, Hkv, Skv, D)
    if rc < 0:
        _check(rc)
    return rc


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word: 0 or ATTN_ERR_DEVICE_TIMEOUT."""
    return load_library().attn_device_status(_stream_handle(stream))


def version() -> int:
    return load_library().attn_version()
