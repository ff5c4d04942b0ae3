"""CPU oracle for causal scaled-dot-product attention (fp64, plain three-pass softmax).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA product (``causal_attention_attn_b200``) never
imports it, and this package imports nothing from the product: the two share no code.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over rows); this module only
compiles it with gcc and marshals arrays through ctypes. What it computes, with its sources:

* scores ``s_j = scale * q_i . k_j`` -- "05 · Tích vô hướng, Softmax và toán của Attention", §1 and
  "Vì sao chia cho √128";
* causal mask aligned to the last ``Sq`` key columns (key ``j`` visible to query ``i`` iff
  ``j <= i + Skv - Sq``) -- "第11节：Attention 实现（Flash vs Fallback）", §3;
* softmax in three passes (max, denominator, result) and ``LSE = m + ln l`` -- "AI Infra 入门：
  RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层优化", §3;
* masked keys get weight exactly zero -- "Bộ 06 · Bên trong model", Q2;
* an FP8 (e4m3) K/V cache with one fp32 coefficient per (kv head, channel), dequantised before the
  plain definition -- "MLA 矩阵乘法吸收的数值稳定性治理", §五 (FP8 storage, higher-precision
  accumulation) and §二.1 (per-channel scaling).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle_attn.so")

_lock = threading.Lock()
_lib = None


def compile_oracle(src: str = _SRC, out: str = _LIB_PATH, extra_flags: tuple = ()) -> str:
    """Compile ``src`` into a shared library at ``out`` with gcc (-O2, OpenMP). Returns ``out``."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def build() -> str:
    """Build the oracle library if it is missing or older than its source."""
    if not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_oracle()
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    fn = lib.oracle_attn
    fn.restype = ctypes.c_int
    fn.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # q k v (bf16 bits)
        ctypes.c_void_p, ctypes.c_void_p,  # o lse (fp64)
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_float, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
    ]
    bwd = lib.oracle_attn_bwd
    bwd.restype = ctypes.c_int
    bwd.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # q k v dout (bf16 bits)
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # dq dk dv (fp64)
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_float, ctypes.c_int, ctypes.c_int,
    ]
    fp8 = lib.oracle_attn_fp8kv
    fp8.restype = ctypes.c_int
    fp8.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # q (bf16 bits), k8, v8 (e4m3 codes)
        ctypes.c_void_p, ctypes.c_void_p,  # k_scale, v_scale (fp32 [Hkv, D])
        ctypes.c_void_p, ctypes.c_void_p,  # o lse (fp64)
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_float, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
    ]
    dec = lib.oracle_decode_e4m3
    dec.restype = None
    dec.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
    return lib


def load(path: str | None = None):
    """Load (and build if needed) the oracle library. ``path`` loads another build (tests)."""
    global _lib
    if path is not None:
        return _bind(path)
    with _lock:
        if _lib is None:
            _lib = _bind(build())
        return _lib


def _as_bf16_bits(x) -> np.ndarray:
    """Accept a torch bf16 tensor or a numpy uint16 array of bf16 bit patterns."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must be uint16 arrays of bf16 bit patterns")
        return np.ascontiguousarray(x)
    import torch  # plain CPU tensors only: the oracle reads host memory

    if not isinstance(x, torch.Tensor) or x.dtype != torch.bfloat16:
        raise TypeError("inputs must be torch.bfloat16 tensors or uint16 numpy arrays")
    return x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def attention(q, k, v, scale: float, causal: bool, rows=None, threads: int | None = None, lib=None):
    """Oracle attention.

    q: [B, Hq, Sq, D], k/v: [B, Hkv, Skv, D] in bf16 (torch) or bf16 bits (numpy uint16).
    ``scale`` is rounded to fp32 (the value the GPU receives) before use.
    ``rows``: optional 1-D array of flat row ids ``(b * Hq + h) * Sq + i``.
    Returns ``(o, lse)`` as float64 numpy arrays: with ``rows=None`` o is [B, Hq, Sq, D] and lse
    [B, Hq, Sq]; otherwise o is [len(rows), D] and lse [len(rows)].
    """
    qb, kb, vb = _as_bf16_bits(q), _as_bf16_bits(k), _as_bf16_bits(v)
    if qb.ndim != 4 or kb.ndim != 4 or vb.shape != kb.shape:
        raise ValueError("expected q [B,Hq,Sq,D] and k, v [B,Hkv,Skv,D]")
    B, Hq, Sq, D = qb.shape
    Bk, Hkv, Skv, Dk = kb.shape
    if Bk != B or Dk != D:
        raise ValueError("q and k/v disagree on batch or head dim")
    if rows is None:
        n_rows = B * Hq * Sq
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        n_rows = int(rows_arr.shape[0])
    o = np.empty((n_rows, D), dtype=np.float64)
    lse = np.empty((n_rows,), dtype=np.float64)
    lib = lib if lib is not None else load()
    rc = lib.oracle_attn(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, o.ctypes.data, lse.ctypes.data,
        B, Hq, Hkv, Sq, Skv, D, ctypes.c_float(scale), int(bool(causal)),
        rows_arr.ctypes.data if rows_arr is not None else None, n_rows, int(threads or 0),
    )
    if rc != 0:
        raise ValueError(f"oracle_attn rejected its arguments (code {rc})")
    if rows is None:
        return o.reshape(B, Hq, Sq, D), lse.reshape(B, Hq, Sq)
    return o, lse


def attention_bwd(q, k, v, dout, scale: float, causal: bool, threads: int | None = None, lib=None):
    """Oracle backward pass: the gradients of a loss L with respect to q, k, v, given dO = dL/dO.

    q, dout: [B, Hq, Sq, D]; k, v: [B, Hkv, Skv, D]; bf16 (torch) or bf16 bits (numpy uint16).
    Returns ``(dq, dk, dv)`` as float64 numpy arrays of the input shapes.
    """
    qb, kb, vb, ob = _as_bf16_bits(q), _as_bf16_bits(k), _as_bf16_bits(v), _as_bf16_bits(dout)
    if qb.ndim != 4 or kb.ndim != 4 or vb.shape != kb.shape or ob.shape != qb.shape:
        raise ValueError("expected q, dout [B,Hq,Sq,D] and k, v [B,Hkv,Skv,D]")
    B, Hq, Sq, D = qb.shape
    Bk, Hkv, Skv, Dk = kb.shape
    if Bk != B or Dk != D:
        raise ValueError("q and k/v disagree on batch or head dim")
    dq = np.empty((B, Hq, Sq, D), dtype=np.float64)
    dk = np.empty((B, Hkv, Skv, D), dtype=np.float64)
    dv = np.empty((B, Hkv, Skv, D), dtype=np.float64)
    lib = lib if lib is not None else load()
    rc = lib.oracle_attn_bwd(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, ob.ctypes.data, dq.ctypes.data,
                             dk.ctypes.data, dv.ctypes.data, B, Hq, Hkv, Sq, Skv, D, ctypes.c_float(scale),
                             int(bool(causal)), int(threads or 0))
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd rejected its arguments (code {rc})")
    return dq, dk, dv



def _as_u8(x) -> np.ndarray:
    """Accept a torch uint8 / float8_e4m3fn tensor or a numpy uint8 array of e4m3 codes."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint8:
            raise TypeError("numpy fp8 inputs must be uint8 arrays of e4m3 codes")
        return np.ascontiguousarray(x)
    import torch

    if not isinstance(x, torch.Tensor) or x.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError("fp8 inputs must be torch uint8 / float8_e4m3fn tensors or uint8 numpy arrays")
    return x.detach().to("cpu").contiguous().view(torch.uint8).numpy()


def _as_f32(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.float32)
    return x.detach().to("cpu").contiguous().float().numpy()


def decode_e4m3(codes, lib=None) -> np.ndarray:
    """The oracle's e4m3 decoder applied to an array of codes (float64 result, same shape)."""
    c = _as_u8(codes)
    out = np.empty(c.shape, dtype=np.float64)
    lib = lib if lib is not None else load()
    lib.oracle_decode_e4m3(c.ctypes.data, out.ctypes.data, int(c.size))
    return out


def attention_fp8kv(q, k8, v8, k_scale, v_scale, scale: float, causal: bool, rows=None,
                    threads: int | None = None, lib=None):
    """Oracle attention over an e4m3 K/V cache: k = e4m3(k8) * k_scale[kv head, channel], likewise v.

    q: [B, Hq, Sq, D] bf16; k8/v8: [B, Hkv, Skv, D] e4m3 codes; k_scale/v_scale: [Hkv, D] fp32.
    Returns ``(o, lse)`` as :func:`attention` does.
    """
    qb, kb, vb = _as_bf16_bits(q), _as_u8(k8), _as_u8(v8)
    ks, vs = _as_f32(k_scale), _as_f32(v_scale)
    if qb.ndim != 4 or kb.ndim != 4 or vb.shape != kb.shape:
        raise ValueError("expected q [B,Hq,Sq,D] and k8, v8 [B,Hkv,Skv,D]")
    B, Hq, Sq, D = qb.shape
    Bk, Hkv, Skv, Dk = kb.shape
    if Bk != B or Dk != D or ks.shape != (Hkv, D) or vs.shape != (Hkv, D):
        raise ValueError("q, k8/v8 and the scales [Hkv, D] disagree")
    if rows is None:
        n_rows = B * Hq * Sq
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        n_rows = int(rows_arr.shape[0])
    o = np.empty((n_rows, D), dtype=np.float64)
    lse = np.empty((n_rows,), dtype=np.float64)
    lib = lib if lib is not None else load()
    rc = lib.oracle_attn_fp8kv(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, ks.ctypes.data, vs.ctypes.data,
        o.ctypes.data, lse.ctypes.data, B, Hq, Hkv, Sq, Skv, D, ctypes.c_float(scale), int(bool(causal)),
        rows_arr.ctypes.data if rows_arr is not None else None, n_rows, int(threads or 0),
    )
    if rc != 0:
        raise ValueError(f"oracle_attn_fp8kv rejected its arguments (code {rc})")
    if rows is None:
        return o.reshape(B, Hq, Sq, D), lse.reshape(B, Hq, Sq)
    return o, lse
