"""The C-ABI library loads, exports every function include/gad_attn.h declares,
and rejects bad arguments on the host before touching a GPU (no GPU needed:
every call here fails validation before any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gad_attn.h")


@pytest.fixture(scope="module")
def lib():
    from paged_fp8_gated_b200 import build
    build.build()
    from paged_fp8_gated_b200 import binding
    return binding


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(gad_[A-Za-z0-9_]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gad_attn_decode", "gad_attn_workspace_bytes", "gad_last_error", "gad_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    for n in declared_functions():
        assert hasattr(so, n), n
    assert set(lib.EXPORTED) <= set(declared_functions())


def test_status_strings(lib):
    so = lib.lib()
    assert so.gad_status_string(0) == b"GAD_OK"
    assert so.gad_status_string(-4) == b"GAD_ERR_UNSUPPORTED"


FAKE = 0x10000  # never dereferenced: validation fails before any device work


def _ok_args(**over):
    a = dict(qkv=FAKE, positions=FAKE, seq_lens=None, page_table=FAKE, cache_loc=FAKE,
             k_cache=FAKE, v_cache=FAKE, k_scale=FAKE, v_scale=FAKE, B=2, L=1, max_pages=8,
             num_rows=64, page_size=1, window=0, use_rope=0, out=FAKE, workspace=FAKE,
             workspace_bytes=1 << 20, stream=None)
    a.update(over)
    return a


@pytest.mark.parametrize("over,status", [
    (dict(qkv=None), -1),
    (dict(out=None), -1),
    (dict(k_scale=None), -1),
    (dict(workspace=None), -5),
    (dict(B=0), -2),
    (dict(B=5000), -2),
    (dict(L=0), -2),
    (dict(L=9), -2),
    (dict(max_pages=0), -2),
    (dict(page_size=16), -4),
    (dict(page_size=64, num_rows=100), -2),
    (dict(num_rows=0), -2),
    (dict(window=-1), -4),
    (dict(qkv=FAKE + 8), -3),
    (dict(k_cache=FAKE + 4), -3),
    (dict(positions=FAKE + 4), -3),
    (dict(workspace=FAKE + 16), -3),
])
def test_argument_checks_fail_before_launch(lib, over, status):
    assert lib.raw_call(**_ok_args(**over)) == status
    assert lib.last_error()


@pytest.mark.parametrize("over,status", [
    (dict(hq=16, hkv=4), -4),             # 4 query heads per KV head
    (dict(hq=24, hkv=3), -4),             # odd KV-head count
    (dict(hq=0, hkv=0), -4),
    (dict(hq=8, hkv=1), -4),
    (dict(hq=128, hkv=16, B=513), -2),    # 513 requests x 8 head groups > 4096 list items
    (dict(hq=128, hkv=16, qkv=FAKE + 8), -3),   # valid heads reach the later checks
    (dict(hq=128, hkv=16, qkv=None), -1),
])
def test_heads_argument_checks(lib, over, status):
    assert lib.raw_call(**_ok_args(**over)) == status
    assert lib.last_error()


@pytest.mark.parametrize("over,status", [
    (dict(L=9), -2),                           # the decode entry point stops at 8 tokens
    (dict(L=9, prefill=True, qkv=FAKE + 8), -3),   # the prefill one takes them
    (dict(L=65537, prefill=True), -2),
    (dict(B=5, L=16384, prefill=True), -2),    # 5 x 512 chunks x 2 KV heads > 4096 items
    (dict(B=2, L=16384, prefill=True, qkv=None), -1),
])
def test_prefill_argument_checks(lib, over, status):
    assert lib.raw_call(**_ok_args(**over)) == status
    assert lib.last_error()


def test_prefill_workspace_query_limits(lib):
    so = lib.lib()
    assert so.gad_attn_prefill_workspace_bytes(5, 16384) == 0
    assert "items" in lib.last_error()
    assert so.gad_attn_prefill_workspace_bytes(1, 0) == 0


def test_heads_workspace_query_rejects_bad_heads(lib):
    so = lib.lib()
    assert so.gad_attn_workspace_bytes_heads(4, 1, 16, 4) == 0
    assert "hq=16" in lib.last_error()
    assert so.gad_attn_workspace_bytes_heads(600, 8, 128, 16) == 0


@pytest.mark.parametrize("T,K,N,out,status", [
    (0, 1024, 8192, FAKE, -2),
    (4, 1000, 8192, FAKE, -2),     # K not a multiple of 64
    (4, 1024, 8000, FAKE, -2),     # N not a multiple of 128
    (4, 1024, 8192, None, -1),
    (4, 1024, 8192, FAKE + 8, -3),
])
def test_oproj_argument_checks(lib, T, K, N, out, status):
    so = lib.lib()
    args = [None if out is None else ctypes.c_void_p(out), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE),
            T, K, N, None]
    assert so.gad_oproj(*args) == status
    assert lib.last_error()


@pytest.mark.parametrize("over,hidden,o_weight,a,status", [
    (dict(), 100, FAKE, FAKE, -2),            # hidden not a multiple of 128
    (dict(), 8192, None, FAKE, -1),
    (dict(), 8192, FAKE, None, -1),
    (dict(out=FAKE + 8), 8192, FAKE, FAKE, -3),
    (dict(L=0), 8192, FAKE, FAKE, -2),
    (dict(L=65537), 8192, FAKE, FAKE, -2),
    (dict(B=0), 8192, FAKE, FAKE, -2),
])
def test_decode_oproj_argument_checks(lib, over, hidden, o_weight, a, status):
    # the step with its projection chained: the projection's own checks run
    # first, on the host, before any launch
    so = lib.lib()
    args = _ok_args(**over)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    st = so.gad_attn_decode_oproj(
        vp(args["qkv"]), vp(args["positions"]), vp(args["seq_lens"]), vp(args["page_table"]),
        vp(args["cache_loc"]), vp(args["k_cache"]), vp(args["v_cache"]), vp(args["k_scale"]),
        vp(args["v_scale"]), args["B"], args["L"], args["max_pages"], args["num_rows"], args["page_size"],
        args["window"], args["use_rope"], vp(args["out"]), vp(args["workspace"]), args["workspace_bytes"],
        vp(o_weight), hidden, vp(a), None)
    assert st == status
    assert lib.last_error()


def test_binding_rejects_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 2304, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lib.attn_decode(x, torch.zeros(1, dtype=torch.int64), None,
                        torch.zeros(1, 4, dtype=torch.int32), torch.zeros(1, dtype=torch.int64),
                        torch.zeros(4, 1, 2, 64, dtype=torch.uint8),
                        torch.zeros(4, 1, 2, 64, dtype=torch.uint8), torch.ones(1), torch.ones(1),
                        1, 0, False)
