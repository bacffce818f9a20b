"""Python binding of libgad_attn.so (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; this module
only checks torch tensors' dtypes and layouts, allocates the output and the
workspace with torch when the caller does not pass them, and forwards raw
device pointers and the current CUDA stream to the C ABI (include/gad_attn.h).

Importing it fails loudly when the library has not been built: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgad_attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run `python -m paged_fp8_gated_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)
_vp = ctypes.c_void_p
_lib.gad_attn_workspace_bytes.restype = ctypes.c_size_t
_lib.gad_attn_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
_lib.gad_attn_decode.restype = ctypes.c_int
_lib.gad_attn_decode.argtypes = [
    _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,            # qkv .. v_scale
    ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,  # B, L, max_pages, num_rows
    ctypes.c_int, ctypes.c_int, ctypes.c_int,               # page_size, window, use_rope
    _vp, _vp, ctypes.c_size_t, _vp]                         # out, workspace, bytes, stream
_lib.gad_attn_workspace_bytes_heads.restype = ctypes.c_size_t
_lib.gad_attn_workspace_bytes_heads.argtypes = [ctypes.c_int] * 4
_lib.gad_attn_decode_heads.restype = ctypes.c_int
_lib.gad_attn_decode_heads.argtypes = (list(_lib.gad_attn_decode.argtypes[:11])
                                       + [ctypes.c_int, ctypes.c_int]  # hq, hkv
                                       + list(_lib.gad_attn_decode.argtypes[11:]))
_lib.gad_attn_decode_heads_timed.restype = ctypes.c_int
_lib.gad_attn_decode_heads_timed.argtypes = list(_lib.gad_attn_decode_heads.argtypes) + [_vp]
_lib.gad_attn_prefill.restype = ctypes.c_int
_lib.gad_attn_prefill.argtypes = list(_lib.gad_attn_decode.argtypes)
_lib.gad_attn_prefill_workspace_bytes.restype = ctypes.c_size_t
_lib.gad_attn_prefill_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
_lib.gad_attn_prefill_timed.restype = ctypes.c_int
_lib.gad_attn_prefill_timed.argtypes = list(_lib.gad_attn_decode.argtypes) + [_vp]
_lib.gad_oproj.restype = ctypes.c_int
_lib.gad_oproj.argtypes = [_vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp]
_lib.gad_attn_decode_oproj.restype = ctypes.c_int
_lib.gad_attn_decode_oproj.argtypes = (list(_lib.gad_attn_decode.argtypes[:19])
                                       + [_vp, ctypes.c_int, _vp, _vp])  # o_weight, hidden, a, stream
_lib.gad_attn_decode_timed.restype = ctypes.c_int
_lib.gad_attn_decode_timed.argtypes = list(_lib.gad_attn_decode.argtypes) + [_vp]
_lib.gad_attn_decode_noalloc.restype = ctypes.c_int
_lib.gad_attn_decode_noalloc.argtypes = list(_lib.gad_attn_decode.argtypes[:17]) + [_vp]
_lib.gad_attn_step_status.restype = ctypes.c_int
_lib.gad_attn_step_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_int), _vp]
_lib.gad_oproj_status.restype = ctypes.c_int
_lib.gad_oproj_status.argtypes = [ctypes.POINTER(ctypes.c_int), _vp]


class GadTensor(ctypes.Structure):
    """gad_tensor: data pointer, element type code, rank, extents, strides (elements)."""
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


_GT = ctypes.POINTER(GadTensor)
_lib.gad_attn_set_workspace.restype = ctypes.c_int
_lib.gad_attn_set_workspace.argtypes = [_vp, ctypes.c_size_t]
_lib.gad_attn_workspace_bytes_t.restype = ctypes.c_size_t
_lib.gad_attn_workspace_bytes_t.argtypes = [ctypes.c_int] * 5
_lib.gad_attn_decode_t.restype = ctypes.c_int
_lib.gad_attn_decode_t.argtypes = [_GT] * 9 + [ctypes.c_int] * 3 + [_GT, _vp]
_lib.gad_last_error.restype = ctypes.c_char_p
_lib.gad_last_error.argtypes = []
_lib.gad_status_string.restype = ctypes.c_char_p
_lib.gad_status_string.argtypes = [ctypes.c_int]

HQ, HKV, D = 16, 2, 64
QKV_COLS, OUT_COLS, ROW_BYTES = 2304, 1024, 128
MAX_L, MAX_PREFILL_L = 8, 65536
HIDDEN = 8192

EXPORTED = ("gad_attn_decode", "gad_attn_decode_heads", "gad_attn_decode_timed",
            "gad_attn_decode_heads_timed", "gad_attn_prefill", "gad_attn_prefill_timed",
            "gad_attn_prefill_workspace_bytes", "gad_oproj", "gad_attn_decode_oproj",
            "gad_attn_decode_noalloc", "gad_attn_workspace_bytes",
            "gad_attn_workspace_bytes_heads", "gad_last_error", "gad_status_string",
            "gad_attn_step_status", "gad_oproj_status", "gad_attn_set_workspace",
            "gad_attn_workspace_bytes_t", "gad_attn_decode_t")
# gad_dtype codes (include/gad_attn.h)
DTYPE_BF16, DTYPE_E4M3, DTYPE_U8, DTYPE_I32, DTYPE_I64, DTYPE_F32 = 1, 2, 3, 4, 5, 6
_DTYPE_CODES = {torch.bfloat16: DTYPE_BF16, torch.uint8: DTYPE_U8, torch.int32: DTYPE_I32,
                torch.int64: DTYPE_I64, torch.float32: DTYPE_F32}
if hasattr(torch, "float8_e4m3fn"):
    _DTYPE_CODES[torch.float8_e4m3fn] = DTYPE_E4M3
NOALLOC_SCRATCH_BYTES = 16 << 20


class GadError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.gad_last_error().decode(errors="replace")
        name = _lib.gad_status_string(status).decode()
        super().__init__(f"{where}: {name} ({status}): {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    return _lib


def workspace_bytes(B: int, L: int, hq: int = HQ, hkv: int = HKV) -> int:
    """Workspace of one step; blocks longer than MAX_L tokens go to the prefill
    entry point (16 and 2 heads)."""
    if L > MAX_L and (hq, hkv) == (HQ, HKV):
        n = _lib.gad_attn_prefill_workspace_bytes(int(B), int(L))
    elif (hq, hkv) == (HQ, HKV):
        n = _lib.gad_attn_workspace_bytes(int(B), int(L))
    else:
        n = _lib.gad_attn_workspace_bytes_heads(int(B), int(L), int(hq), int(hkv))
    if n == 0:
        raise GadError(-2, "gad_attn_workspace_bytes")
    return int(n)


def alloc_workspace(B: int, L: int, device=None, hq: int = HQ, hkv: int = HKV) -> torch.Tensor:
    """Caller-owned scratch for gad_attn_decode (256-byte aligned by torch's allocator)."""
    return torch.empty(workspace_bytes(B, L, hq, hkv), dtype=torch.uint8,
                       device=device or "cuda")


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def attn_decode(qkv: torch.Tensor, positions: torch.Tensor, seq_lens: torch.Tensor | None,
                page_table: torch.Tensor, cache_loc: torch.Tensor, k_cache: torch.Tensor,
                v_cache: torch.Tensor, k_scale: torch.Tensor, v_scale: torch.Tensor,
                page_size: int, window: int, use_rope: bool, L: int = 1,
                out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                stream: torch.cuda.Stream | None = None,
                events: list | None = None, hq: int = HQ, hkv: int = HKV) -> torch.Tensor:
    """One decode step (L = 1), verify block (L <= 8) or prefill block (L up to
    MAX_PREFILL_L, through gad_attn_prefill, 16 and 2 heads); returns out bf16
    [B, L, 64 hq].

    Shapes: qkv bf16 [B*L, 64 (2 hq + 2 hkv)]; positions, cache_loc int64 [B*L];
    seq_lens int32 [B] (optional); page_table int32 [B, max_pages]; k_cache / v_cache
    uint8 [num_pages, page_size, hkv, 64] (mutated in the rows cache_loc); k_scale /
    v_scale float32 [1] on the device.  hq, hkv: head counts (16, 2 by default; other
    counts go through gad_attn_decode_heads).  With ``events`` (four torch.cuda.Event
    with timing), the profiling entry point records them around the three kernels.
    """
    _need(qkv, "qkv", torch.bfloat16, 2)
    _need(positions, "positions", torch.int64, 1)
    _need(page_table, "page_table", torch.int32, 2)
    _need(cache_loc, "cache_loc", torch.int64, 1)
    _need(k_cache, "k_cache", torch.uint8)
    _need(v_cache, "v_cache", torch.uint8)
    _need(k_scale, "k_scale", torch.float32)
    _need(v_scale, "v_scale", torch.float32)
    if seq_lens is not None:
        _need(seq_lens, "seq_lens", torch.int32, 1)
    B, max_pages = page_table.shape
    T = qkv.shape[0]
    qkv_cols, out_cols, row_bytes = (2 * hq + 2 * hkv) * D, hq * D, hkv * D
    if qkv.shape[1] != qkv_cols or T != B * L:
        raise ValueError(f"qkv must be [B*L={B * L}, {qkv_cols}], got {tuple(qkv.shape)}")
    if positions.numel() != T or cache_loc.numel() != T:
        raise ValueError("positions and cache_loc need one entry per token")
    if k_cache.shape != v_cache.shape or k_cache.numel() % row_bytes:
        raise ValueError(f"k_cache and v_cache must have the same shape, {row_bytes} bytes per row")
    num_rows = k_cache.numel() // row_bytes
    if out is None:
        out = torch.empty(B, L, out_cols, dtype=torch.bfloat16, device=qkv.device)
    else:
        _need(out, "out", torch.bfloat16)
        if out.numel() != T * out_cols:
            raise ValueError(f"out must hold B*L*{out_cols} values")
    if workspace is None:
        workspace = alloc_workspace(B, L, qkv.device, hq, hkv)
    else:
        _need(workspace, "workspace", torch.uint8)
    s = (stream or torch.cuda.current_stream(qkv.device)).cuda_stream
    head = (_ptr(qkv), _ptr(positions), _ptr(seq_lens), _ptr(page_table), _ptr(cache_loc),
            _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), int(B), int(L))
    tail = (int(max_pages), int(num_rows), int(page_size), int(window), int(bool(use_rope)),
            _ptr(out), _ptr(workspace), int(workspace.numel()), ctypes.c_void_p(s))
    args = head + tail
    tp8 = (hq, hkv) == (HQ, HKV)
    prefill = L > MAX_L
    if prefill and not tp8:
        raise ValueError(f"blocks longer than {MAX_L} tokens take 16 query and 2 KV heads")
    if events is None:
        if prefill:
            st = _lib.gad_attn_prefill(*args)
        else:
            st = _lib.gad_attn_decode(*args) if tp8 else \
                _lib.gad_attn_decode_heads(*head, int(hq), int(hkv), *tail)
    else:
        if len(events) != 4:
            raise ValueError("events must hold four torch.cuda.Event")
        for ev in events:   # materialise the underlying cudaEvent_t
            if ev.cuda_event == 0:
                ev.record()
        arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(ev.cuda_event) for ev in events])
        if prefill:
            st = _lib.gad_attn_prefill_timed(*args, arr)
        else:
            st = _lib.gad_attn_decode_timed(*args, arr) if tp8 else \
                _lib.gad_attn_decode_heads_timed(*head, int(hq), int(hkv), *tail, arr)
    if st != 0:
        raise GadError(st, "gad_attn_prefill" if prefill else "gad_attn_decode")
    return out


def attn_decode_noalloc(qkv: torch.Tensor, positions: torch.Tensor,
                        seq_lens: torch.Tensor | None, page_table: torch.Tensor,
                        cache_loc: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                        k_scale: torch.Tensor, v_scale: torch.Tensor, page_size: int, window: int,
                        use_rope: bool, L: int = 1, out: torch.Tensor | None = None,
                        stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """The step through gad_attn_decode_noalloc: no workspace argument, the library's
    built-in 16 MiB device scratch is used instead (for callers that cannot allocate
    device memory themselves).  Calls on one device must not overlap on the GPU."""
    for t, n, dt in ((qkv, "qkv", torch.bfloat16), (positions, "positions", torch.int64),
                     (page_table, "page_table", torch.int32), (cache_loc, "cache_loc", torch.int64),
                     (k_cache, "k_cache", torch.uint8), (v_cache, "v_cache", torch.uint8),
                     (k_scale, "k_scale", torch.float32), (v_scale, "v_scale", torch.float32)):
        _need(t, n, dt)
    B, max_pages = page_table.shape
    T = qkv.shape[0]
    if qkv.shape[1] != QKV_COLS or T != B * L:
        raise ValueError(f"qkv must be [B*L={B * L}, {QKV_COLS}], got {tuple(qkv.shape)}")
    if positions.numel() != T or cache_loc.numel() != T:
        raise ValueError("positions and cache_loc need one entry per token")
    if k_cache.shape != v_cache.shape or k_cache.numel() % ROW_BYTES:
        raise ValueError(f"k_cache and v_cache must have the same shape, {ROW_BYTES} bytes per row")
    num_rows = k_cache.numel() // ROW_BYTES
    if out is None:
        out = torch.empty(B, L, OUT_COLS, dtype=torch.bfloat16, device=qkv.device)
    else:
        _need(out, "out", torch.bfloat16)
        if out.numel() != T * OUT_COLS:
            raise ValueError(f"out must hold B*L*{OUT_COLS} values")
    s = (stream or torch.cuda.current_stream(qkv.device)).cuda_stream
    st = _lib.gad_attn_decode_noalloc(
        _ptr(qkv), _ptr(positions), _ptr(seq_lens), _ptr(page_table), _ptr(cache_loc),
        _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), int(B), int(L),
        int(max_pages), int(num_rows), int(page_size), int(window), int(bool(use_rope)),
        _ptr(out), ctypes.c_void_p(s))
    if st != 0:
        raise GadError(st, "gad_attn_decode_noalloc")
    return out


def oproj(out: torch.Tensor, o_weight: torch.Tensor, a: torch.Tensor | None = None,
          stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """a = out @ o_weight^T through gad_oproj: out bf16 [T, K], o_weight bf16 [N, K]
    (both CUDA, contiguous); returns a bf16 [T, N]."""
    _need(out, "out", torch.bfloat16)
    _need(o_weight, "o_weight", torch.bfloat16, 2)
    K = out.shape[-1]
    T = out.numel() // K
    N = o_weight.shape[0]
    if o_weight.shape[1] != K:
        raise ValueError(f"o_weight must be [N, {K}], got {tuple(o_weight.shape)}")
    if a is None:
        a = torch.empty(T, N, dtype=torch.bfloat16, device=out.device)
    else:
        _need(a, "a", torch.bfloat16)
        if a.numel() != T * N:
            raise ValueError(f"a must hold {T}x{N} values")
    s = (stream or torch.cuda.current_stream(out.device)).cuda_stream
    st = _lib.gad_oproj(_ptr(out), _ptr(o_weight), _ptr(a), int(T), int(K), int(N), ctypes.c_void_p(s))
    if st != 0:
        raise GadError(st, "gad_oproj")
    return a


def attn_decode_oproj(qkv, positions, seq_lens, page_table, cache_loc, k_cache, v_cache, k_scale,
                      v_scale, page_size: int, window: int, use_rope: bool, o_weight: torch.Tensor,
                      L: int = 1, out: torch.Tensor | None = None, a: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None,
                      stream: torch.cuda.Stream | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """The step and its output projection in one call (gad_attn_decode_oproj);
    returns (out bf16 [B, L, 1024], a bf16 [B * L, hidden])."""
    for t, n, dt in ((qkv, "qkv", torch.bfloat16), (positions, "positions", torch.int64),
                     (page_table, "page_table", torch.int32), (cache_loc, "cache_loc", torch.int64),
                     (k_cache, "k_cache", torch.uint8), (v_cache, "v_cache", torch.uint8),
                     (k_scale, "k_scale", torch.float32), (v_scale, "v_scale", torch.float32)):
        _need(t, n, dt)
    _need(o_weight, "o_weight", torch.bfloat16, 2)
    B, max_pages = page_table.shape
    T = qkv.shape[0]
    if qkv.shape[1] != QKV_COLS or T != B * L:
        raise ValueError(f"qkv must be [B*L={B * L}, {QKV_COLS}], got {tuple(qkv.shape)}")
    hidden = o_weight.shape[0]
    num_rows = k_cache.numel() // ROW_BYTES
    if out is None:
        out = torch.empty(B, L, OUT_COLS, dtype=torch.bfloat16, device=qkv.device)
    if a is None:
        a = torch.empty(T, hidden, dtype=torch.bfloat16, device=qkv.device)
    if workspace is None:
        n = _lib.gad_attn_prefill_workspace_bytes(int(B), int(L))
        if n == 0:
            raise GadError(-2, "gad_attn_prefill_workspace_bytes")
        workspace = torch.empty(int(n), dtype=torch.uint8, device=qkv.device)
    s = (stream or torch.cuda.current_stream(qkv.device)).cuda_stream
    st = _lib.gad_attn_decode_oproj(
        _ptr(qkv), _ptr(positions), _ptr(seq_lens), _ptr(page_table), _ptr(cache_loc), _ptr(k_cache),
        _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), int(B), int(L), int(max_pages), int(num_rows),
        int(page_size), int(window), int(bool(use_rope)), _ptr(out), _ptr(workspace),
        int(workspace.numel()), _ptr(o_weight), int(hidden), _ptr(a), ctypes.c_void_p(s))
    if st != 0:
        raise GadError(st, "gad_attn_decode_oproj")
    return out, a


def raw_call(**kw) -> int:
    """Call the C entry point with raw values (for boundary tests); returns the status."""
    args = [kw.get(k) for k in ("qkv", "positions", "seq_lens", "page_table", "cache_loc",
                                "k_cache", "v_cache", "k_scale", "v_scale")]
    args = [a if (a is None or isinstance(a, ctypes.c_void_p)) else ctypes.c_void_p(a) for a in args]
    args += [kw.get("B", 1), kw.get("L", 1)]
    rest = [kw.get("max_pages", 1), kw.get("num_rows", 1), kw.get("page_size", 1),
            kw.get("window", 0), kw.get("use_rope", 0), kw.get("out"), kw.get("workspace"),
            kw.get("workspace_bytes", 0), kw.get("stream")]
    if kw.get("prefill"):           # through gad_attn_prefill
        return _lib.gad_attn_prefill(*args, *rest)
    if "hq" in kw or "hkv" in kw:   # through gad_attn_decode_heads
        return _lib.gad_attn_decode_heads(*args, kw.get("hq", HQ), kw.get("hkv", HKV), *rest)
    return _lib.gad_attn_decode(*args, *rest)


def last_error() -> str:
    return _lib.gad_last_error().decode(errors="replace")


# ---------------------------------------------------------------------------
# Status words and the tensor-descriptor form
# ---------------------------------------------------------------------------

def step_status(workspace: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> int:
    """GAD_STATUS_* bits of the last step run with `workspace` (None: the
    allocation-free entry point's built-in scratch); waits for `stream`."""
    st = ctypes.c_int(-1)
    dev = workspace.device if workspace is not None else torch.device("cuda", torch.cuda.current_device())
    s = stream or torch.cuda.current_stream(dev)
    rc = _lib.gad_attn_step_status(_ptr(workspace), ctypes.byref(st), ctypes.c_void_p(s.cuda_stream))
    if rc != 0:
        raise GadError(rc, "gad_attn_step_status")
    s.synchronize()
    return int(st.value)


def oproj_status(stream: torch.cuda.Stream | None = None) -> int:
    """GAD_STATUS_* bits of the standalone projections since the last read (then cleared)."""
    st = ctypes.c_int(-1)
    s = stream or torch.cuda.current_stream()
    rc = _lib.gad_oproj_status(ctypes.byref(st), ctypes.c_void_p(s.cuda_stream))
    if rc != 0:
        raise GadError(rc, "gad_oproj_status")
    s.synchronize()
    return int(st.value)


def tensor_desc(t: torch.Tensor | None, dtype: int | None = None, data: int | None = None,
                shape=None, stride=None) -> GadTensor | None:
    """gad_tensor for a torch tensor (its pointer, element type, extents and
    strides); the keyword overrides let tests describe malformed tensors."""
    if t is None and data is None:
        return None
    d = GadTensor()
    d.data = data if data is not None else t.data_ptr()
    d.dtype = dtype if dtype is not None else _DTYPE_CODES.get(t.dtype, 0)
    shp = list(shape if shape is not None else t.shape)
    std = list(stride if stride is not None else t.stride())
    d.ndim = len(shp)
    for i in range(min(4, len(shp))):
        d.shape[i] = int(shp[i])
        d.stride[i] = int(std[i])
    return d


def set_workspace(workspace: torch.Tensor | None) -> None:
    """Register (None: unregister) the scratch gad_attn_decode_t uses on the current device."""
    rc = _lib.gad_attn_set_workspace(_ptr(workspace), 0 if workspace is None else int(workspace.numel()))
    if rc != 0:
        raise GadError(rc, "gad_attn_set_workspace")


def workspace_bytes_t(B: int, L: int, max_pages: int, page_size: int, window: int) -> int:
    n = _lib.gad_attn_workspace_bytes_t(int(B), int(L), int(max_pages), int(page_size), int(window))
    if n == 0:
        raise GadError(-2, "gad_attn_workspace_bytes_t")
    return int(n)


def raw_call_t(descs: dict, page_size: int = 1, window: int = 0, use_rope: int = 0, stream=None) -> int:
    """gad_attn_decode_t on prepared descriptors (missing names pass NULL); returns the status."""
    names = ("qkv", "positions", "seq_lens", "page_table", "cache_loc", "k_cache", "v_cache",
             "k_scale", "v_scale")
    ptrs = [ctypes.byref(descs[n]) if descs.get(n) is not None else None for n in names]
    out = descs.get("out")
    return _lib.gad_attn_decode_t(*ptrs, int(page_size), int(window), int(use_rope),
                                  ctypes.byref(out) if out is not None else None, stream)


def attn_decode_t(qkv, positions, seq_lens, page_table, cache_loc, k_cache, v_cache, k_scale, v_scale,
                  page_size: int, window: int, use_rope: bool, out: torch.Tensor,
                  stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """The step through the descriptor entry point (scratch from set_workspace):
    the tensors are described as they are; the library checks them."""
    descs = dict(qkv=tensor_desc(qkv), positions=tensor_desc(positions), seq_lens=tensor_desc(seq_lens),
                 page_table=tensor_desc(page_table), cache_loc=tensor_desc(cache_loc),
                 k_cache=tensor_desc(k_cache), v_cache=tensor_desc(v_cache), k_scale=tensor_desc(k_scale),
                 v_scale=tensor_desc(v_scale), out=tensor_desc(out))
    s = (stream or torch.cuda.current_stream(out.device)).cuda_stream
    rc = raw_call_t(descs, page_size, window, int(bool(use_rope)), ctypes.c_void_p(s))
    if rc != 0:
        raise GadError(rc, "gad_attn_decode_t")
    return out
