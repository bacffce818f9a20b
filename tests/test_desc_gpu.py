"""The tensor-descriptor entry point (gad_attn_decode_t) runs the same step as
the plain-pointer one: the same kernels on the same tile list, so outputs and
cache bytes agree bit for bit.  Shapes come from the descriptors (B, L and the
head counts from out and qkv), the scratch from gad_attn_set_workspace."""
import numpy as np
import pytest
import torch

from paged_fp8_gated_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

CASES = [
    W.Spec("desc_verify_sliding_p64", B=3, L=8, seq_lens=[40, 1500, 5000], window=2048, use_rope=True,
           page_size=64, kv_scale=1 / 64, gate_std=2.0, seed=601),
    W.Spec("desc_decode_full_p1", B=5, L=1, ctx_range=(10, 6000), seed=602),
    W.Spec("desc_heads_dp", B=2, L=8, seq_lens=[37, 3000], page_size=64, seed=603, hq=W.DP_HQ, hkv=W.DP_HKV),
    W.Spec("desc_prefill_L40", B=2, L=40, seq_lens=[0, 900], window=256, use_rope=True, seed=604),
]


@pytest.mark.parametrize("spec", CASES, ids=lambda s: s.name)
def test_descriptor_form_matches_pointer_form(spec, cuda_dev):
    from paged_fp8_gated_b200 import binding
    inp = W.make_inputs(spec)
    hq, hkv = H.heads(inp)
    ref_out, ref_k, ref_v = H.run_gpu(inp)
    d = H.to_device(inp)
    B, L = inp["B"], inp["L"]
    ps = inp["page_size"]
    kc = d["k_cache"].view(-1, ps, hkv, 64)
    vc = d["v_cache"].view(-1, ps, hkv, 64)
    out = torch.empty(B, L, 64 * hq, dtype=torch.bfloat16, device="cuda")
    ws = binding.alloc_workspace(B, L, "cuda", hq, hkv)
    if (hq, hkv) == (16, 2):
        assert binding.workspace_bytes_t(B, L, d["page_table"].shape[1], ps, inp["window"]) == ws.numel()
    binding.set_workspace(ws)
    try:
        binding.attn_decode_t(d["qkv"], d["positions"], d["seq_lens"], d["page_table"], d["cache_loc"], kc, vc,
                              d["k_scale_t"], d["v_scale_t"], ps, inp["window"], inp["use_rope"], out)
        torch.cuda.synchronize()
        assert binding.step_status(ws) == 0
    finally:
        binding.set_workspace(None)
    got = out.view(torch.int16).reshape(B * L, 64 * hq).cpu().numpy().astype(np.uint16)
    assert np.array_equal(got, ref_out)
    assert np.array_equal(d["k_cache"].reshape(-1, 64 * hkv).cpu().numpy(), ref_k)
    assert np.array_equal(d["v_cache"].reshape(-1, 64 * hkv).cpu().numpy(), ref_v)


def test_descriptor_form_needs_registered_scratch(cuda_dev):
    from paged_fp8_gated_b200 import binding
    inp = W.make_inputs(CASES[1])
    d = H.to_device(inp)
    out = torch.full((5, 1, 1024), 3.0, dtype=torch.bfloat16, device="cuda")
    binding.set_workspace(None)
    with pytest.raises(binding.GadError) as ei:
        binding.attn_decode_t(d["qkv"], d["positions"], d["seq_lens"], d["page_table"], d["cache_loc"],
                              d["k_cache"], d["v_cache"], d["k_scale_t"], d["v_scale_t"], 1, 0, False, out)
    assert ei.value.status == -5
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
