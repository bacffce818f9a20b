"""Child process of test_wait_giveup_gpu.py: runs steps on the short-wait build
of the library, in which every pipeline wait inside the kernels gives up as
soon as its phase has not completed at the first probe, and prints one JSON
line with each step's status word.  It loads only that build (not the package binding),
so the production library is never in this process.

After the steps that gave up, a single-token step (whose kernel has no
bounded waits) runs in the same context and is checked against the oracle:
the context stays usable after a kernel has given up.
"""
import ctypes
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from paged_fp8_gated_b200 import build  # noqa: E402
from paged_fp8_gated_b200 import workloads as W  # noqa: E402
from tests import helpers as H  # noqa: E402

vp = ctypes.c_void_p
lib = ctypes.CDLL(build.SHORT_WAIT_LIB)
STEP_ARGS = [vp] * 9 + [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                        ctypes.c_int, vp, vp, ctypes.c_size_t, vp]
for name in ("gad_attn_decode", "gad_attn_prefill"):
    getattr(lib, name).restype = ctypes.c_int
    getattr(lib, name).argtypes = STEP_ARGS
lib.gad_attn_prefill_workspace_bytes.restype = ctypes.c_size_t
lib.gad_attn_prefill_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
lib.gad_attn_decode_oproj.restype = ctypes.c_int
lib.gad_attn_decode_oproj.argtypes = STEP_ARGS[:19] + [vp, ctypes.c_int, vp, vp]
lib.gad_oproj.restype = ctypes.c_int
lib.gad_oproj.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
lib.gad_attn_step_status.restype = ctypes.c_int
lib.gad_attn_step_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int), vp]
lib.gad_oproj_status.restype = ctypes.c_int
lib.gad_oproj_status.argtypes = [ctypes.POINTER(ctypes.c_int), vp]
lib.gad_last_error.restype = ctypes.c_char_p

dev = torch.device("cuda", 0)
p = lambda t: vp(t.data_ptr())


def step_args(d, inp, out, ws):
    B, L = inp["B"], inp["L"]
    num_rows = d["k_cache"].numel() // 128
    return [p(d["qkv"]), p(d["positions"]), p(d["seq_lens"]), p(d["page_table"]), p(d["cache_loc"]),
            p(d["k_cache"]), p(d["v_cache"]), p(d["k_scale_t"]), p(d["v_scale_t"]), B, L,
            d["page_table"].shape[1], num_rows, inp["page_size"], inp["window"], int(inp["use_rope"]),
            p(out), p(ws), ws.numel()]


def status_of(ws):
    st = ctypes.c_int(-1)
    assert lib.gad_attn_step_status(p(ws), ctypes.byref(st), None) == 0
    torch.cuda.synchronize()
    return int(st.value)


def run(spec, oproj=False):
    inp = W.make_inputs(spec)
    d = H.to_device(inp, dev)
    B, L = inp["B"], inp["L"]
    out = torch.empty(B, L, 1024, dtype=torch.bfloat16, device=dev)
    ws = torch.full((int(lib.gad_attn_prefill_workspace_bytes(B, L)),), 0x5A, dtype=torch.uint8, device=dev)
    if oproj:
        w = W.oproj_weight().to(dev)
        a = torch.empty(B * L, w.shape[0], dtype=torch.bfloat16, device=dev)
        rc = lib.gad_attn_decode_oproj(*step_args(d, inp, out, ws), p(w), w.shape[0], p(a), None)
    else:
        fn = lib.gad_attn_prefill if L > 8 else lib.gad_attn_decode
        rc = fn(*step_args(d, inp, out, ws), None)
    assert rc == 0, (rc, lib.gad_last_error())
    torch.cuda.synchronize()
    return status_of(ws), inp, out


res = {}
res["verify"], _, _ = run(W.Spec("gu_verify", B=3, L=8, seq_lens=[100, 2000, 5000], seed=501))
res["prefill"], _, _ = run(W.Spec("gu_prefill", B=2, L=40, seq_lens=[0, 900], window=256, use_rope=True,
                                  seed=502))
res["decode_oproj"], _, _ = run(W.Spec("gu_dec_oproj", B=4, L=1, seq_lens=[10, 300, 900, 3000], seed=503),
                                oproj=True)
# the standalone projection reports into its own word, cleared on read
x = W.oproj_input(32, seed=504).to(dev)
w = W.oproj_weight().to(dev)
a = torch.empty(32, w.shape[0], dtype=torch.bfloat16, device=dev)
assert lib.gad_oproj(p(x), p(w), p(a), 32, 1024, w.shape[0], None) == 0
st = ctypes.c_int(-1)
assert lib.gad_oproj_status(ctypes.byref(st), None) == 0
torch.cuda.synchronize()
res["oproj"] = int(st.value)
assert lib.gad_oproj_status(ctypes.byref(st), None) == 0
torch.cuda.synchronize()
res["oproj_after_read"] = int(st.value)
# the context still works: a single-token step (no bounded waits) is correct
status, inp, out = run(W.Spec("gu_after", B=3, L=1, seq_lens=[5, 700, 2500], seed=505))
res["after_status"] = status
bits = out.view(torch.int16).reshape(-1, 1024).cpu().numpy().astype(np.uint16)
res["after_ok"] = H.compare(bits, H.run_oracle(inp))["ok"]
print(json.dumps(res), flush=True)
