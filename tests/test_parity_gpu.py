"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Cache bytes written by the step: bit-exact everywhere (the whole cache is
compared, so rows the step must not touch are checked too).  Output: max
|gpu - oracle| <= 2e-2 + 2e-2 |oracle| element-wise, on every output for the
small cases and on sampled (token, head) outputs at the full workload sizes.
"""
import numpy as np
import pytest
import torch

from paged_fp8_gated_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

S = W.Spec

SMALL = [
    # the page's gating shapes (section "Shapes"), shrunk only where noted
    S("b1_ctx10_sliding", B=1, ctx=10, window=2048, use_rope=True, page_size=64, seed=101),
    S("b3_ctx2047_sliding", B=3, ctx=2047, window=2048, use_rope=True, page_size=64, seed=102),
    S("b5_ctx5000_sliding_v8_p1", B=5, L=8, ctx=5000, window=2048, use_rope=True, seed=103),
    S("b4_ctx3000_full", B=4, ctx=3000, page_size=64, seed=104),
    S("b8_ctx8192_full_mixed", B=8, ctx_range=(1, 8192), page_size=64, seed=105),
    S("b3_ctx4000_sliding_v8_p1_s64", B=3, L=8, ctx=4000, window=2048, use_rope=True,
      kv_scale=1 / 64, seed=106),
    S("b2_ctx9000_full_s64", B=2, ctx=9000, page_size=64, kv_scale=1 / 64, seed=107),
    S("b4_ctx6000_sliding_v8_p64", B=4, L=8, ctx=6000, window=2048, use_rope=True,
      page_size=64, seed=108),
    S("b4_ctx6000_sliding_v8_soft_p1", B=4, L=8, ctx=6000, window=2048, use_rope=True, seed=153),
    S("b4_ctx6000_full_v8_edges", B=4, L=8, ctx=6000, page_size=64, dist="edges", seed=150),
    S("b4_ctx80k_full_mixed_soft", B=4, ctx_range=(1, 80000), page_size=64, seed=151),
    S("b4_ctx80k_full_mixed_coherent_p1", B=4, ctx_range=(1, 80000), dist="coherent", seed=152),
    # edge cases
    S("ctx0_and_1", B=3, seq_lens=[0, 1, 2], seed=110),
    S("ctx0_verify", B=2, L=8, seq_lens=[0, 3], seed=111),
    S("window1", B=2, seq_lens=[0, 500], window=1, use_rope=True, seed=112),
    S("window_gt_ctx", B=2, L=8, seq_lens=[30, 700], window=5000, use_rope=True, seed=113),
    S("ragged_pages", B=4, seq_lens=[63, 64, 65, 127], page_size=64, seed=114),
    S("ragged_pages_v8", B=4, L=8, seq_lens=[56, 57, 63, 120], page_size=64, seed=115),
    S("L3_block", B=3, L=3, seq_lens=[100, 1000, 64], seed=116),
    S("many_requests", B=40, ctx_range=(0, 3000), seed=117),
    # more list items than the verify kernel's deeper ring leaves table room
    # for: its shallow configuration (three raw stages)
    S("many_items_v8_shallow_ring", B=1800, L=8, ctx_range=(0, 100), seed=162),
    S("many_requests_v8_sliding", B=40, L=8, ctx_range=(0, 5000), window=256, use_rope=True,
      seed=118),
    S("gate_std2_s64", B=2, L=8, ctx=1500, page_size=64, kv_scale=1 / 64, gate_std=2.0, seed=119),
    S("spare_pages", B=2, seq_lens=[333, 777], page_size=64, spare_pages=5, seed=120),
    # 16 and 17 single-token requests: the combine kernel's one-wave form and
    # its 256-thread form
    S("b16_decode_mixed", B=16, ctx_range=(0, 20000), seed=147),
    S("b17_decode_mixed", B=17, ctx_range=(0, 20000), seed=148),
    # many requests
    S("b1100_decode_p1", B=1100, ctx_range=(0, 300), seed=123),
    S("b1100_decode_p64_sliding", B=1100, ctx_range=(0, 400), window=100, use_rope=True,
      page_size=64, seed=124),
    # the page's stress distributions (section "Correctness")
    S("coherent_full", B=4, ctx=6000, dist="coherent", seed=125),
    S("coherent_full_v8_p64", B=2, L=8, ctx=20000, page_size=64, dist="coherent", seed=126),
    S("coherent_sliding_rope", B=3, L=8, ctx=5000, window=2048, use_rope=True, dist="coherent",
      seed=127),
    S("edges_sliding", B=4, ctx=6000, window=2048, dist="edges", seed=128),
    S("edges_sliding_v8", B=4, L=8, ctx=6000, window=2048, dist="edges", seed=129),
    S("edges_sliding_v8_p64_s64", B=3, L=8, ctx=4000, window=2048, page_size=64,
      kv_scale=1 / 64, dist="edges", seed=130),
]


# "heads dp" (128 query heads over 16 KV heads on one GPU): the page's three
# gating shapes, then edge cases of the head-group split.
DP = dict(hq=W.DP_HQ, hkv=W.DP_HKV)
SMALL_DP = [
    W.named("dp8_full_mixed"),
    W.named("dp2_full_v8_soft"),
    W.named("dp2_full_v8_coherent"),
    S("dp_sliding_p1", B=3, ctx_range=(0, 4000), window=2048, use_rope=True, seed=140, **DP),
    S("dp_sliding_v8_s64", B=2, L=8, seq_lens=[37, 3000], window=2048, use_rope=True,
      page_size=64, kv_scale=1 / 64, gate_std=2.0, seed=141, **DP),
    S("dp_ctx0_and_ragged_v3", B=3, L=3, seq_lens=[0, 63, 130], page_size=64, seed=142, **DP),
    S("dp_edges_sliding", B=2, L=8, ctx=3000, window=2048, dist="edges", seed=143, **DP),
    # 2 requests x 8 groups = 16 items (the combine's one-wave form)
    S("dp_b2_decode", B=2, seq_lens=[700, 4000], page_size=64, seed=146, **DP),
    # 512 requests x 8 groups = 4096 list items, the most one call takes
    S("dp_b512_most_items", B=512, ctx_range=(0, 40), seed=144, **DP),
    # 256 requests x 8 groups = 2048 verify items: the shallow ring at page size 64
    S("dp_b256_v8_shallow_ring", B=256, L=8, ctx_range=(0, 40), page_size=64, seed=161, **DP),
]


def _check(inp, want=None, label=""):
    gpu_out, gpu_k, gpu_v = H.run_gpu(inp)
    ref = H.run_oracle(inp, want=want)
    assert np.array_equal(gpu_k, ref.k_cache), f"{label}: k cache bytes differ"
    assert np.array_equal(gpu_v, ref.v_cache), f"{label}: v cache bytes differ"
    st = H.compare(gpu_out, ref, want)
    assert st["ok"], f"{label}: {st}"
    return st


@pytest.mark.parametrize("spec", SMALL, ids=lambda s: s.name)
def test_small_full_compare(spec, cuda_dev):
    _check(W.make_inputs(spec), label=spec.name)


@pytest.mark.parametrize("spec", SMALL_DP, ids=lambda s: s.name)
def test_heads_dp_compare(spec, cuda_dev):
    _check(W.make_inputs(spec), label=spec.name)


def test_heads_dp_equals_eight_tp8_steps(cuda_dev):
    """The library's 128/16-head step against eight of its own 16/2-head steps
    on the column slices.  Cache bytes must match bit for bit; outputs to about
    one bf16 rounding step (4e-3 absolute, for elements near zero after the
    output norm), since the tile list (and with it where the key ranges are
    split between CTAs, i.e. the fp32 summation order) differs."""
    inp = W.make_inputs(S("dp_vs_tp8", B=3, L=8, seq_lens=[5, 700, 2100], window=2048,
                          use_rope=True, seed=145, **DP))
    out_dp, k_dp, v_dp = H.run_gpu(inp)
    hq, hkv = W.DP_HQ, W.DP_HKV
    qkv = inp["qkv"]
    ks, vs, gs = 64 * hq, 64 * (hq + hkv), 64 * (hq + 2 * hkv)
    kc = inp["k_cache"].reshape(-1, hkv, 64)
    vc = inp["v_cache"].reshape(-1, hkv, 64)
    for c in range(hkv // 2):
        sub = dict(inp)
        sub["hq"], sub["hkv"] = 16, 2
        sub["qkv"] = torch.cat([qkv[:, 1024 * c:1024 * (c + 1)], qkv[:, ks + 128 * c:ks + 128 * (c + 1)],
                                qkv[:, vs + 128 * c:vs + 128 * (c + 1)],
                                qkv[:, gs + 1024 * c:gs + 1024 * (c + 1)]], dim=1).contiguous()
        sub["k_cache"] = kc[:, 2 * c:2 * c + 2].contiguous()
        sub["v_cache"] = vc[:, 2 * c:2 * c + 2].contiguous()
        out_tp, k_tp, v_tp = H.run_gpu(sub)
        a = H.O.bf16_bits_to_float(out_dp[:, 1024 * c:1024 * (c + 1)])
        b = H.O.bf16_bits_to_float(out_tp)
        err = np.abs(a - b)
        assert (err <= 4e-3 + 2.0 ** -7 * np.abs(b)).all(), (c, float(err.max()))
        assert np.array_equal(k_dp[:, 128 * c:128 * (c + 1)], k_tp), c
        assert np.array_equal(v_dp[:, 128 * c:128 * (c + 1)], v_tp), c


# Prefill blocks (gad_attn_prefill): the prefill page's five gating tests,
# ragged chunk edges, then its scored shapes on sampled heads.
SMALL_PREFILL = [
    S("pf_b1_ctx0_sliding_q300", B=1, L=300, ctx=0, window=2048, use_rope=True, seed=150),
    S("pf_b1_ctx3000_full_q753", B=1, L=753, ctx=3000, seed=151),
    S("pf_b2_ctx2500_sliding_q753", B=2, L=753, ctx=2500, window=2048, use_rope=True, seed=152),
    # "dist outliers", the one test on 64-token pages
    S("pf_b3_ctx5000_full_q200_outliers_p64", B=3, L=200, ctx=5000, page_size=64,
      dist="outliers", seed=153),
    S("pf_L9_ragged", B=3, L=9, seq_lens=[0, 70, 1000], page_size=64, seed=155),
    S("pf_L13_window_edge", B=2, L=13, seq_lens=[2040, 5000], window=2048, use_rope=True,
      seed=156),
    S("pf_L100_window_small", B=2, L=100, seq_lens=[10, 300], window=64, use_rope=True,
      seed=157),
]


@pytest.mark.parametrize("spec", SMALL_PREFILL, ids=lambda s: s.name)
def test_prefill_compare(spec, cuda_dev):
    _check(W.make_inputs(spec), label=spec.name)


def test_prefill_q4096_sliding_sampled(cuda_dev):
    # "batch 1, ctx 4096, layer sliding, q_len 4096, page 1"
    inp = W.make_inputs(S("pf_b1_ctx4096_sliding_q4096", B=1, L=4096, ctx=4096, window=2048,
                          use_rope=True, seed=154))
    _check(inp, want=H.sample_want(4096, 512, seed=5), label="q4096")


PREFILL_FULL = {"prefill1_full": 96, "prefill4_sliding": 96, "prefill16k_ctx0_full": 64,
                "prefill16k_ctx64k_full": 48}


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(PREFILL_FULL))
def test_prefill_named_sampled(name, cuda_dev):
    inp = W.make_inputs(W.named(name))
    T = inp["B"] * inp["L"]
    _check(inp, want=H.sample_want(T, PREFILL_FULL[name], seed=6), label=name)


def test_verify_full_ctx100k(cuda_dev):
    # "batch 2, ctx 100000, heads tp8, layer full, q_len 8, page 1"
    _check(W.make_inputs(S("b2_ctx100k_full_v8", B=2, L=8, ctx=100000, seed=121)))


def test_long_ctx_1m_sampled(cuda_dev):
    # "batch 1, ctx 1048576, heads tp8, layer full, q_len 8": sampled heads
    inp = W.make_inputs(S("b1_ctx1m_full_v8", B=1, L=8, ctx=1048576, page_size=64, seed=122))
    _check(inp, want=H.sample_want(8, 6, seed=1))


FULL = ["pr1", "decode1_sliding", "decode1_full", "decode32_full", "decode32_sliding",
        "verify16_sliding", "verify16_full", "paged_full", "paged_sliding",
        # the rest of the page's twelve scored loads
        "decode16_full", "decode16_sliding", "verify1_full", "verify1_sliding",
        "verify32_full", "verify32_sliding"]
SAMPLED = {"verify16_full": 24, "paged_full": 32, "decode16_full": 24,
           "verify1_full": 24, "verify32_full": 24, "verify32_sliding": 48}


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_named_workloads(name, cuda_dev):
    inp = W.make_inputs(W.named(name))
    T = inp["B"] * inp["L"]
    want = H.sample_want(T, SAMPLED[name], seed=3) if name in SAMPLED else None
    _check(inp, want=want, label=name)


def test_page_size_1_and_64_agree_bitwise(cuda_dev):
    inp64 = W.make_inputs(S("p64", B=3, L=8, seq_lens=[70, 5, 700], page_size=64, seed=130))
    pt64 = inp64["page_table"].numpy()
    kc64 = inp64["k_cache"].reshape(-1, 128).numpy()
    vc64 = inp64["v_cache"].reshape(-1, 128).numpy()
    pos = inp64["positions"].numpy()
    B, L = 3, 8
    total = pos.reshape(B, L)[:, -1] + 1
    perm = np.random.default_rng(5).permutation(int(total.sum()))
    maxp = int((total.max() + 3) // 4 * 4)
    pt1 = np.zeros((B, maxp), np.int32)
    kc1 = np.zeros((perm.size, 128), np.uint8)
    vc1 = np.zeros_like(kc1)
    off = 0
    for b in range(B):
        for i in range(int(total[b])):
            src = pt64[b, i // 64] * 64 + i % 64
            pt1[b, i] = perm[off + i]
            kc1[perm[off + i]] = kc64[src]
            vc1[perm[off + i]] = vc64[src]
        off += int(total[b])
    inp1 = dict(inp64)
    inp1.update(page_size=1, page_table=torch.from_numpy(pt1),
                cache_loc=torch.from_numpy(pt1[np.repeat(np.arange(B), L), pos].astype(np.int64)),
                k_cache=torch.from_numpy(kc1).view(-1, 1, 2, 64),
                v_cache=torch.from_numpy(vc1).view(-1, 1, 2, 64))
    o64, _, _ = H.run_gpu(inp64)
    o1, _, _ = H.run_gpu(inp1)
    assert np.array_equal(o64, o1)


def test_repeatable_and_workspace_reuse(cuda_dev):
    from paged_fp8_gated_b200 import binding
    inp = W.make_inputs(S("rep", B=6, L=8, ctx_range=(100, 4000), seed=131))
    ws = binding.alloc_workspace(6, 8)
    ws.fill_(0xAB)                         # contents on entry must not matter
    a = H.run_gpu(inp, workspace=ws)
    b = H.run_gpu(inp, workspace=ws)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_graph_capture_replay_matches_eager(cuda_dev):
    from paged_fp8_gated_b200 import binding
    inp = W.make_inputs(S("graph", B=4, ctx_range=(500, 9000), seed=132))
    d = H.to_device(inp)
    k0, v0 = d["k_cache"].clone(), d["v_cache"].clone()
    ws = binding.alloc_workspace(4, 1)
    out = torch.empty(4, 1, 1024, dtype=torch.bfloat16, device="cuda")
    args = (d["qkv"], d["positions"], d["seq_lens"], d["page_table"], d["cache_loc"],
            d["k_cache"], d["v_cache"], d["k_scale_t"], d["v_scale_t"], 1, 0, False)
    binding.attn_decode(*args, L=1, out=out, workspace=ws)
    eager = out.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        binding.attn_decode(*args, L=1, out=out, workspace=ws)  # warm up on the side stream
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            binding.attn_decode(*args, L=1, out=out, workspace=ws)
    torch.cuda.synchronize()
    out.zero_()
    d["k_cache"].copy_(k0)
    d["v_cache"].copy_(v0)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
