"""The allocation-free entry point, gad_attn_decode_noalloc.

It exists for callers that cannot give the library device scratch memory (a
framework whose memory pool owns every device allocation, a plugin that may not
call cudaMalloc because it can synchronise the device or is refused during a
graph capture, a C host with no device allocator).  It keeps its scratch in a
fixed 16 MiB device array inside the library.  These tests call it through the
C ABI twice in a row and compare with the workspace entry point on the same
inputs; they need nothing from any other test, so they pass alone in a fresh
process as well as after the rest of the suite (this file is collected last).
"""
import numpy as np
import pytest
import torch

from paged_fp8_gated_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

CASES = [
    W.Spec("noalloc_decode_mixed", B=5, L=1, ctx_range=(10, 6000), page_size=1, seed=301),
    W.Spec("noalloc_verify_sliding_p64", B=3, L=8, seq_lens=[40, 1500, 5000], window=2048,
           use_rope=True, page_size=64, kv_scale=1 / 64, gate_std=2.0, seed=302),
]


def _noalloc(d, inp):
    from paged_fp8_gated_b200 import binding
    o = binding.attn_decode_noalloc(d["qkv"], d["positions"], d["seq_lens"], d["page_table"],
                                    d["cache_loc"], d["k_cache"], d["v_cache"], d["k_scale_t"],
                                    d["v_scale_t"], inp["page_size"], inp["window"],
                                    inp["use_rope"], L=inp["L"])
    torch.cuda.synchronize()
    return o.view(torch.int16).reshape(-1, 1024).cpu().numpy().astype(np.uint16)


@pytest.mark.parametrize("spec", CASES, ids=lambda s: s.name)
def test_noalloc_matches_workspace_entry_on_two_calls(spec, cuda_dev):
    inp = W.make_inputs(spec)
    ref_out, ref_k, ref_v = H.run_gpu(inp)          # gad_attn_decode with a caller workspace
    d = H.to_device(inp)
    # The same kernels run on the same tile list (the grid depends only on the
    # shapes), so the two entry points agree bit for bit; the shared scratch
    # keeps the last call's bytes, so the second call must not depend on them.
    for _ in range(2):
        got = _noalloc(d, inp)
        assert np.array_equal(got, ref_out)
    assert np.array_equal(d["k_cache"].reshape(-1, 128).cpu().numpy(), ref_k)
    assert np.array_equal(d["v_cache"].reshape(-1, 128).cpu().numpy(), ref_v)
    # and both are within the tolerance of the oracle
    ref = H.run_oracle(inp)
    st = H.compare(got, ref)
    assert st["ok"], st
    assert np.array_equal(ref_k, ref.k_cache) and np.array_equal(ref_v, ref.v_cache)


def test_noalloc_after_a_larger_step(cuda_dev):
    """A large verify step first fills much more of the shared scratch; a
    smaller decode step after it must not read its leftovers.  The workspace
    entry point, given a workspace full of poison bytes, is the reference."""
    from paged_fp8_gated_b200 import binding
    big = W.make_inputs(W.Spec("noalloc_big", B=32, L=8, ctx_range=(100, 3000), seed=303))
    _noalloc(H.to_device(big), big)
    small = W.make_inputs(W.Spec("noalloc_small", B=3, L=1, seq_lens=[5, 700, 2500], seed=304))
    ws = binding.alloc_workspace(3, 1)
    ws.fill_(0xC3)
    ref_out, _, _ = H.run_gpu(small, workspace=ws)
    d = H.to_device(small)
    assert np.array_equal(_noalloc(d, small), ref_out)


def test_noalloc_rejects_steps_larger_than_its_scratch(cuda_dev):
    from paged_fp8_gated_b200 import binding
    B, L = 1024, 8                                   # needs far more than 16 MiB of scratch
    assert binding.workspace_bytes(B, L) > binding.NOALLOC_SCRATCH_BYTES
    dev = "cuda"
    qkv = torch.zeros(B * L, 2304, dtype=torch.bfloat16, device=dev)
    pos = torch.zeros(B * L, dtype=torch.int64, device=dev)
    pt = torch.zeros(B, 4, dtype=torch.int32, device=dev)
    kc = torch.zeros(4, 1, 2, 64, dtype=torch.uint8, device=dev)
    vc = torch.zeros_like(kc)
    sc = torch.ones(1, dtype=torch.float32, device=dev)
    out = torch.full((B, L, 1024), 7.0, dtype=torch.bfloat16, device=dev)
    with pytest.raises(binding.GadError) as ei:
        binding.attn_decode_noalloc(qkv, pos, None, pt, pos, kc, vc, sc, sc, 1, 0, False, L=L,
                                    out=out)
    assert ei.value.status == -5 and "scratch" in str(ei.value)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())                  # nothing was launched
