"""ctypes front end of the CPU oracle (``gad_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline arm of ``bench.py`` use this module.  The CUDA library never imports
it, and it imports nothing from the CUDA library.

The oracle follows the task page "Gated attention decode
(muse_attention_decode)", section "What to compute", evaluated literally in
double precision (see the header comment of ``gad_oracle.c`` for the readings
taken where the page is silent).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gad_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libgad_oracle.so")

HQ, HKV, D = 16, 2, 64   # the page's per-GPU shapes ("heads tp8")
QKV_COLS = 2304


def qkv_cols(hq: int, hkv: int) -> int:
    """Columns of one qkv row: q (hq heads) | k (hkv) | v (hkv) | gate (hq), 64 each."""
    return (2 * hq + 2 * hkv) * D


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE double, no FMA contraction)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
             "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.gado_e4m3_decode.restype = ctypes.c_double
        L.gado_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.gado_e4m3_encode.restype = ctypes.c_uint8
        L.gado_e4m3_encode.argtypes = [ctypes.c_float]
        L.gado_bf16_decode.restype = ctypes.c_double
        L.gado_bf16_decode.argtypes = [ctypes.c_uint16]
        L.gado_bf16_encode.restype = ctypes.c_uint16
        L.gado_bf16_encode.argtypes = [ctypes.c_double]
        dp = ctypes.POINTER(ctypes.c_double)
        L.gado_rmsnorm.restype = None
        L.gado_rmsnorm.argtypes = [dp, dp, ctypes.c_int, ctypes.c_double]
        L.gado_rope_neox.restype = None
        L.gado_rope_neox.argtypes = [dp, ctypes.c_int, ctypes.c_double, ctypes.c_double]
        vp = ctypes.c_void_p
        L.gado_attn_decode.restype = ctypes.c_int
        L.gado_attn_decode.argtypes = [
            vp, vp, vp, vp, vp, vp, ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp,
            ctypes.c_int]
        L.gado_oproj.restype = ctypes.c_int
        L.gado_oproj.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, ctypes.c_int]
        L.gado_attn_decode_heads.restype = ctypes.c_int
        L.gado_attn_decode_heads.argtypes = [
            vp, vp, vp, vp, vp, vp, ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, vp, vp, vp, vp, ctypes.c_int]
    return _lib


# ----------------------------------------------------------------------------
# Scalar primitives (exposed for the pins)
# ----------------------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    return lib().gado_e4m3_decode(int(code) & 0xFF)


def e4m3_encode(x: float) -> int:
    """float32 -> E4M3 code, round to nearest even, saturating to +-448."""
    return int(lib().gado_e4m3_encode(float(np.float32(x))))


def bf16_decode(bits: int) -> float:
    return lib().gado_bf16_decode(int(bits) & 0xFFFF)


def bf16_encode(x: float) -> int:
    return int(lib().gado_bf16_encode(float(x)))


def rmsnorm(x, eps: float = 1e-6) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    dp = ctypes.POINTER(ctypes.c_double)
    lib().gado_rmsnorm(x.ctypes.data_as(dp), y.ctypes.data_as(dp), x.size, eps)
    return y


def rope_neox(u, pos: float, theta: float = 10000.0) -> np.ndarray:
    u = np.array(u, dtype=np.float64, copy=True)
    lib().gado_rope_neox(u.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), u.size, float(pos),
                         float(theta))
    return u


# ----------------------------------------------------------------------------
# The whole step
# ----------------------------------------------------------------------------

@dataclass
class OracleResult:
    out: np.ndarray        # uint16 bf16 bits [T, 64 hq]
    out_exact: np.ndarray  # float64 [T, 64 hq], before bf16 rounding
    attn: np.ndarray       # float64 [T, 64 hq], a before the output norm
    k_cache: np.ndarray    # uint8, after this step's writes
    v_cache: np.ndarray


def _np(x, dtype):
    if hasattr(x, "detach"):  # a torch CPU tensor
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=dtype)


def attn_decode(qkv_bits, positions, page_table, cache_loc, k_cache, v_cache, k_scale: float,
                v_scale: float, page_size: int, window: int, use_rope: bool, want=None,
                nthreads: int | None = None, hq: int = HQ, hkv: int = HKV) -> OracleResult:
    """Run the oracle on host arrays.  The caches are copied, not mutated.

    qkv_bits: uint16 [T, qkv_cols(hq, hkv)] (bf16 bit patterns); positions,
    cache_loc: int64 [T]; page_table: int32 [B, max_pages]; caches: uint8
    [..., 64 hkv] (any leading shape).  want: optional bool [T, hq] selecting
    the (token, head) outputs to compute; outputs not computed are left as 0.
    """
    qkv = _np(qkv_bits, np.uint16).reshape(-1, qkv_cols(hq, hkv))
    pos = _np(positions, np.int64).reshape(-1)
    pt = _np(page_table, np.int32)
    B, max_pages = pt.shape
    cl = _np(cache_loc, np.int64).reshape(-1)
    kc = np.array(_np(k_cache, np.uint8).reshape(-1, hkv * D), copy=True)
    vc = np.array(_np(v_cache, np.uint8).reshape(-1, hkv * D), copy=True)
    T = qkv.shape[0]
    assert T % B == 0 and pos.size == T and cl.size == T
    L = T // B
    want_arr = None
    if want is not None:
        want_arr = np.ascontiguousarray(np.asarray(want, dtype=bool).reshape(T, hq), dtype=np.uint8)
    out = np.zeros((T, hq * D), np.uint16)
    out_exact = np.zeros((T, hq * D), np.float64)
    attn = np.zeros((T, hq * D), np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    vp = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
    st = lib().gado_attn_decode_heads(
        vp(qkv), vp(pos), vp(pt), vp(cl), vp(kc), vp(vc), float(k_scale), float(v_scale), B, L,
        int(hq), int(hkv), max_pages, kc.shape[0], int(page_size), int(window),
        int(bool(use_rope)), vp(want_arr), vp(out), vp(out_exact), vp(attn), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle gado_attn_decode failed with status {st}")
    return OracleResult(out, out_exact, attn, kc, vc)


def oproj(out_bits, o_bits, nthreads: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """The output projection a = out @ o^T (bf16 in, double sum, one bf16
    rounding).  out_bits: uint16 [T, K]; o_bits: uint16 [N, K].  Returns
    (a bits uint16 [T, N], a before rounding float64 [T, N])."""
    x = _np(out_bits, np.uint16)
    w = _np(o_bits, np.uint16)
    T, K = x.shape
    N, K2 = w.shape
    assert K == K2
    a = np.zeros((T, N), np.uint16)
    a_exact = np.zeros((T, N), np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    vp = lambda arr: arr.ctypes.data_as(ctypes.c_void_p)
    st = lib().gado_oproj(vp(x), vp(w), T, K, N, vp(a), vp(a_exact), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle gado_oproj failed with status {st}")
    return a, a_exact


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64 (a shift into float32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
