"""Oracle: plain fp64 CPU restatement of block-causal attention with cross-step
prefix K/V reuse, and of OFP8 E4M3 round-to-nearest-even encoding.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline / reference leg import this package.  It shares no code
with the CUDA library and imports nothing from it.

The arithmetic lives in ``bca_oracle.c`` (compiled with gcc, no fast-math, OpenMP
over (row, head) pairs).  This module only builds and loads it and marshals
arrays.  Inputs are bf16 bit patterns (numpy uint16) or e4m3 codes (uint8);
torch bf16 / uint8 CPU tensors are accepted and viewed as such.

Sources (cited by page title and section):
  "Qwen-Image-2.1 + vLLM-Omni day-0", "Serving architecture: the cross-step
  prefix KV cache"; "Qwen/Qwen-Image-2.1" (vLLM recipe), "Prefix KV cache";
  OCP OFP8 specification, E4M3; "SGLang-Diffusion stöder Qwen-Image-2.1 på dag
  noll", "Siffrorna, och vad de inte säger" (the Q/K norm between the projection of
  the target rows and the attention).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bca_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libbca_oracle.so")
_lock = threading.Lock()
_lib = None

KIND_BF16 = 0
KIND_E4M3 = 1


def build(force: bool = False) -> str:
    """Compile bca_oracle.c into libbca_oracle.so (gcc -O2 -fopenmp, IEEE math)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.bca_oracle_bf16_to_f64.restype = ctypes.c_double
        lib.bca_oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.bca_oracle_e4m3_decode.restype = ctypes.c_double
        lib.bca_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.bca_oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.bca_oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.bca_oracle_e4m3_encode_n.restype = None
        lib.bca_oracle_e4m3_encode_n.argtypes = [P, i64, P]
        lib.bca_oracle_absmax_scale.restype = ctypes.c_float
        lib.bca_oracle_absmax_scale.argtypes = [P, i64, i64, i64]
        lib.bca_oracle_quantize_prefix.restype = None
        lib.bca_oracle_quantize_prefix.argtypes = [P, i64, i64, i64, i64, i64, P, P]
        lib.bca_oracle_prefill.restype = ctypes.c_int
        lib.bca_oracle_prefill.argtypes = [P, P, P, i64, i64, i64, P, ctypes.c_int,
                                           ctypes.c_double, P, i64, P, ctypes.c_int]
        lib.bca_oracle_cached_step.restype = ctypes.c_int
        lib.bca_oracle_cached_step.argtypes = [P, P, P, i64, i64, i64, P, ctypes.c_int, P,
                                               P, ctypes.c_int, P, i64, i64, ctypes.c_double,
                                               P, i64, P, ctypes.c_int, P, P]
        lib.bca_oracle_rms_norm.restype = None
        lib.bca_oracle_rms_norm.argtypes = [P, i64, i64, P, ctypes.c_double, P]
        lib.bca_oracle_rope.restype = None
        lib.bca_oracle_rope.argtypes = [P, i64, i64, i64, P, P, P]
        lib.bca_oracle_qkv_project.restype = ctypes.c_int
        lib.bca_oracle_qkv_project.argtypes = [P, i64, i64, P, i64, i64, P, P, P, P,
                                               ctypes.c_double, P, i64, P, P, P, ctypes.c_int]
        lib.bca_oracle_max_threads.restype = ctypes.c_int
        lib.bca_oracle_max_threads.argtypes = []
        _lib = lib
        return lib


def _bits16(x) -> np.ndarray:
    """bf16 bit patterns as a C-contiguous uint16 array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16, x.dtype
            x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, x.dtype
    return x


def _bytes8(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous().view(torch.uint8).numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint8, x.dtype
    return x


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return int(_load().bca_oracle_max_threads())


def bf16_to_f64(bits: int) -> float:
    return float(_load().bca_oracle_bf16_to_f64(int(bits)))


def e4m3_decode(code: int) -> float:
    return float(_load().bca_oracle_e4m3_decode(int(code)))


def e4m3_encode(x: float) -> int:
    """Encode one binary32 value (x is first rounded to float32)."""
    return int(_load().bca_oracle_e4m3_encode(float(np.float32(x))))


def e4m3_encode_array(x: np.ndarray) -> np.ndarray:
    flat = np.ascontiguousarray(np.asarray(x, dtype=np.float32).ravel())
    out = np.empty(flat.shape, dtype=np.uint8)
    _load().bca_oracle_e4m3_encode_n(_ptr(flat), flat.size, _ptr(out))
    return out.reshape(np.shape(x))


def absmax_scale(x_bits, n_rows: int, row_stride: int, d: int, offset: int = 0) -> float:
    a = _bits16(x_bits).ravel()
    return float(_load().bca_oracle_absmax_scale(
        ctypes.c_void_p(a.ctypes.data + 2 * offset), n_rows, row_stride, d))


def quantize_prefix(x, P: int, cap: int | None = None):
    """Quantise rows [0, P) of a [tokens, H, d] bf16 tensor into ([H, cap, d] e4m3
    codes, [H] fp32 scales).  Rows [P, cap) of the returned cache are 0."""
    a = _bits16(x)
    assert a.ndim == 3
    _, H, d = a.shape
    cap = P if cap is None else cap
    codes = np.zeros((H, cap, d), dtype=np.uint8)
    scales = np.zeros((H,), dtype=np.float32)
    _load().bca_oracle_quantize_prefix(_ptr(a), P, H, d, H * d, cap, _ptr(codes), _ptr(scales))
    return codes, scales


def prefill(q, k, v, block_offsets, scale: float, rows=None, nthreads: int = 0) -> np.ndarray:
    """Block-causal attention of [S, H, d] bf16 inputs; returns fp64 [n_rows, H, d]."""
    qb, kb, vb = _bits16(q), _bits16(k), _bits16(v)
    S, H, d = qb.shape
    assert kb.shape == qb.shape and vb.shape == qb.shape
    off = np.ascontiguousarray(block_offsets, dtype=np.int32)
    rws = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = S if rws is None else len(rws)
    out = np.empty((n, H, d), dtype=np.float64)
    rc = _load().bca_oracle_prefill(_ptr(qb), _ptr(kb), _ptr(vb), S, H, d, _ptr(off),
                                    len(off) - 1, float(scale),
                                    None if rws is None else _ptr(rws), n, _ptr(out),
                                    int(nthreads))
    if rc != 0:
        raise ValueError("oracle prefill: bad arguments")
    return out


def cached_step(q_t, k_t, v_t, k_cache, v_cache, P: int, scale: float, k_kind=KIND_BF16,
                v_kind=KIND_BF16, k_scale=None, v_scale=None, rows=None,
                nthreads: int = 0, q8=None) -> np.ndarray:
    """Target rows [T, H, d] over [cache rows 0..P-1 ; own rows 0..T-1].
    Caches are [H, cap, d]: bf16 bits (kind 0) or e4m3 codes (kind 1) with [H] scales.
    q8 = (codes [H, T, d] uint8, scales [H] fp32): the e4m3-Q reading -- the scores
    against the cached keys use the dequantised Q codes (quantize_prefix(q_t, T)
    gives them), those against the own keys the bf16 Q."""
    qb, kb, vb = _bits16(q_t), _bits16(k_t), _bits16(v_t)
    T, H, d = qb.shape
    kc = _bits16(k_cache) if k_kind == KIND_BF16 else _bytes8(k_cache)
    vc = _bits16(v_cache) if v_kind == KIND_BF16 else _bytes8(v_cache)
    assert kc.shape[0] == H and kc.shape[2] == d and vc.shape == kc.shape
    cap = kc.shape[1]
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    rws = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = T if rws is None else len(rws)
    out = np.empty((n, H, d), dtype=np.float64)
    qc = qs = None
    if q8 is not None:
        qc = np.ascontiguousarray(q8[0], dtype=np.uint8)
        qs = np.ascontiguousarray(q8[1], dtype=np.float32)
        assert qc.shape == (H, T, d) and qs.shape == (H,)
    rc = _load().bca_oracle_cached_step(
        _ptr(qb), _ptr(kb), _ptr(vb), T, H, d, _ptr(kc), int(k_kind),
        None if ks is None else _ptr(ks), _ptr(vc), int(v_kind),
        None if vs is None else _ptr(vs), int(P), int(cap), float(scale),
        None if rws is None else _ptr(rws), n, _ptr(out), int(nthreads),
        None if qc is None else _ptr(qc), None if qs is None else _ptr(qs))
    if rc != 0:
        raise ValueError("oracle cached_step: bad arguments")
    return out


def rms_norm(x, gamma, eps: float) -> np.ndarray:
    """x: [..., d] bf16 (bits or tensor); gamma: [d] fp32.  fp64 result, same shape."""
    xb = _bits16(x)
    d = xb.shape[-1]
    g = np.ascontiguousarray(gamma, dtype=np.float32)
    assert g.shape == (d,)
    y = np.empty(xb.shape, dtype=np.float64)
    _load().bca_oracle_rms_norm(_ptr(xb), xb.size // d, d, _ptr(g), float(eps), _ptr(y))
    return y


def rope(y, cos_t, sin_t) -> np.ndarray:
    """y: [rows, H, d] fp64; cos_t, sin_t: [rows, d/2] fp32.  Pair (2i, 2i+1) of row t
    turned by the angle whose cos/sin are cos_t[t, i], sin_t[t, i]."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    rows, H, d = y.shape
    c = np.ascontiguousarray(cos_t, dtype=np.float32)
    s = np.ascontiguousarray(sin_t, dtype=np.float32)
    assert c.shape == (rows, d // 2) and s.shape == c.shape
    out = np.empty_like(y)
    _load().bca_oracle_rope(_ptr(y), rows, H, d, _ptr(c), _ptr(s), _ptr(out))
    return out


def qk_norm_rope(x, gamma, cos_t, sin_t, eps: float) -> np.ndarray:
    """rope(rms_norm(x)) for x [rows, H, d] bf16: the exact (fp64) values."""
    return rope(rms_norm(x, gamma, eps), cos_t, sin_t)


def qkv_project(x, w, gamma_q, gamma_k, cos_t, sin_t, eps: float, heads: int, rows=None,
                nthreads: int = 0):
    """x [T, D] bf16 rows, w [3*heads*d, D] bf16 (torch Linear layout: Q heads, K
    heads, V heads) -> (q, k, v), each fp64 [n_rows, heads, d]: the projection
    y = x w^T, then rope(rms_norm(.)) of every Q and K head vector; V as projected.
    gamma_*: [d] fp32; cos_t, sin_t: [T, d/2] fp32."""
    xb, wb = _bits16(x), _bits16(w)
    T, D = xb.shape
    N, D2 = wb.shape
    assert D2 == D and N % (3 * heads) == 0
    d = N // (3 * heads)
    gq = np.ascontiguousarray(gamma_q, dtype=np.float32)
    gk = np.ascontiguousarray(gamma_k, dtype=np.float32)
    c = np.ascontiguousarray(cos_t, dtype=np.float32)
    s = np.ascontiguousarray(sin_t, dtype=np.float32)
    assert gq.shape == (d,) and gk.shape == (d,) and c.shape == (T, d // 2) and s.shape == c.shape
    rws = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = T if rws is None else len(rws)
    q = np.empty((n, heads, d), dtype=np.float64)
    k = np.empty_like(q)
    v = np.empty_like(q)
    rc = _load().bca_oracle_qkv_project(_ptr(xb), T, D, _ptr(wb), heads, d, _ptr(gq), _ptr(gk),
                                        _ptr(c), _ptr(s), float(eps),
                                        None if rws is None else _ptr(rws), n, _ptr(q), _ptr(k),
                                        _ptr(v), int(nthreads))
    if rc != 0:
        raise ValueError("oracle qkv_project: bad arguments")
    return q, k, v
