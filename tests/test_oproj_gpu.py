"""The output projection a = out @ o^T (gad_oproj, gad_attn_decode_oproj)
against the CPU oracle.

Bound on a (derived from the arithmetic): the kernel sums the K products in
fp32 and rounds once to bf16, the oracle sums in double and rounds once, so
|a_gpu - a_exact| <= 2^-8 |a_exact| (the bf16 rounding) + 1e-5 (|out| @ |o|^T)
(fp32 accumulation over K = 1024 terms, 2^-24 per step, with room).  In the
fused path the step's own output error propagates linearly:
+ |out_gpu - out_oracle| @ |o|^T.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_fp8_gated_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().astype(np.uint16)


def _check_a(a_gpu_bits, a_exact, x_abs_bound):
    got = O.bf16_bits_to_float(a_gpu_bits)
    err = np.abs(got - a_exact)
    bound = 2.0 ** -8 * np.abs(a_exact) + 1e-5 * x_abs_bound + 1e-30
    worst = float((err / bound).max())
    assert np.isfinite(got).all()
    assert worst <= 1.0, f"worst error / bound {worst:.3f}"
    return worst


@pytest.mark.parametrize("T", [1, 5, 16, 32, 100, 128, 256, 300, 1000])
def test_oproj_matches_oracle(T, cuda_dev):
    x = W.oproj_input(T, seed=100 + T)
    w = W.oproj_weight()
    a = torch.empty(T, w.shape[0], dtype=torch.bfloat16, device="cuda")
    from paged_fp8_gated_b200 import binding
    binding.oproj(x.cuda(), w.cuda(), a)
    torch.cuda.synchronize()
    a_bits, a_exact = O.oproj(_bits(x), _bits(w))
    xa = np.abs(O.bf16_bits_to_float(_bits(x))) @ np.abs(O.bf16_bits_to_float(_bits(w))).T
    _check_a(_bits(a), a_exact, xa)
    # almost every element rounds to the oracle's own bf16 value
    assert (_bits(a) == a_bits).mean() > 0.99


@pytest.mark.parametrize("K,N", [(64, 128), (128, 256), (192, 128), (1024, 384)])
def test_oproj_small_shapes(K, N, cuda_dev):
    from paged_fp8_gated_b200 import binding
    g = torch.Generator().manual_seed(K + N)
    x = torch.randn(37, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    a = binding.oproj(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    _, a_exact = O.oproj(_bits(x), _bits(w))
    xa = np.abs(O.bf16_bits_to_float(_bits(x))) @ np.abs(O.bf16_bits_to_float(_bits(w))).T
    _check_a(_bits(a), a_exact, xa)


S = W.Spec


@pytest.mark.parametrize("spec", [
    S("fused_decode_p64", B=4, ctx=3000, page_size=64, seed=160),
    S("fused_verify_p1", B=3, L=8, ctx_range=(500, 4000), seed=161),
    S("fused_prefill_L40", B=2, L=40, seq_lens=[0, 900], window=256, use_rope=True, seed=162),
], ids=lambda s: s.name)
def test_attn_decode_oproj_fused(spec, cuda_dev):
    from paged_fp8_gated_b200 import binding
    inp = W.make_inputs(spec)
    d = H.to_device(inp)
    w = W.oproj_weight(seed=9)
    out, a = binding.attn_decode_oproj(d["qkv"], d["positions"], d["seq_lens"], d["page_table"],
                                       d["cache_loc"], d["k_cache"], d["v_cache"], d["k_scale_t"],
                                       d["v_scale_t"], inp["page_size"], inp["window"],
                                       inp["use_rope"], w.cuda(), L=inp["L"])
    torch.cuda.synchronize()
    T = inp["B"] * inp["L"]
    out_bits = _bits(out).reshape(T, 1024)
    ref = H.run_oracle(inp)
    st = H.compare(out_bits, ref)
    assert st["ok"], st
    # the projection of the step's output, against the oracle's own output projected
    _, a_exact = O.oproj(ref.out, _bits(w))
    wabs = np.abs(O.bf16_bits_to_float(_bits(w))).T
    dout = np.abs(O.bf16_bits_to_float(out_bits) - O.bf16_bits_to_float(ref.out))
    xa = np.abs(O.bf16_bits_to_float(ref.out)) @ wabs
    got = O.bf16_bits_to_float(_bits(a))
    bound = 2.0 ** -8 * np.abs(a_exact) + 1e-5 * xa + dout @ wabs + 1e-30
    assert float((np.abs(got - a_exact) / bound).max()) <= 1.0
    # and bit for bit what the standalone projection gives on the same output
    a2 = binding.oproj(out.reshape(T, 1024), w.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_bits(a2), _bits(a))
