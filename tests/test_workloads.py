"""The seeded input generators hold the contract both the oracle and the CUDA
path rely on (task page "Gated attention decode (muse_attention_decode)",
sections "What to compute" and "Shapes"): positions follow the cached
lengths, each token's cache row is the row of its position under the page
table, requests own disjoint pages, and the named distributions have the
structure their names promise.  CPU only, small sizes."""
import numpy as np
import pytest
import torch

from paged_fp8_gated_b200 import workloads as W


def _e4m3_values(codes: torch.Tensor) -> torch.Tensor:
    return codes.view(torch.float8_e4m3fn).float()


@pytest.mark.parametrize("ps,L,permute", [(1, 1, True), (1, 8, True), (64, 8, True), (64, 1, False)])
def test_positions_rows_and_pages_follow_the_contract(ps, L, permute):
    spec = W.Spec("c", B=5, L=L, seq_lens=[0, 1, 63, 64, 300], page_size=ps, permute=permute, seed=3)
    inp = W.make_inputs(spec)
    B, T = spec.B, spec.B * L
    seq = inp["seq_lens"].numpy().astype(np.int64)
    pos = inp["positions"].numpy()
    pt = inp["page_table"].numpy()
    cl = inp["cache_loc"].numpy()
    n_pages = inp["k_cache"].shape[0]
    assert pt.shape[1] % 4 == 0                      # 16-byte page-table row pitch
    pages_used = []
    for b in range(B):
        n = (seq[b] + L + ps - 1) // ps
        pages_used.append(pt[b, :n])
        for j in range(L):
            t = b * L + j
            assert pos[t] == seq[b] + j
            assert cl[t] == pt[b, pos[t] // ps] * ps + pos[t] % ps
    allp = np.concatenate(pages_used)
    assert len(np.unique(allp)) == len(allp)         # requests own disjoint pages
    assert allp.min() >= 0 and allp.max() < n_pages
    assert len(np.unique(cl)) == T                   # no two tokens write one row
    if not permute:
        assert np.array_equal(allp, np.arange(len(allp)))


def test_layouts_and_head_counts():
    inp = W.make_inputs(W.Spec("dp", B=2, L=8, ctx=100, hq=128, hkv=16, page_size=64, seed=4))
    assert inp["qkv"].shape == (16, W.qkv_cols(128, 16)) == (16, 18432)
    assert inp["qkv"].dtype == torch.bfloat16
    assert inp["k_cache"].shape[1:] == (64, 16, 64) and inp["k_cache"].dtype == torch.uint8
    assert inp["positions"].dtype == torch.int64 and inp["cache_loc"].dtype == torch.int64
    assert inp["page_table"].dtype == torch.int32 and inp["seq_lens"].dtype == torch.int32
    assert W.qkv_cols(16, 2) == W.QKV_COLS == 2304 and W.GATE_OFF == 1280


def test_deterministic_in_the_spec():
    a = W.make_inputs(W.Spec("x", B=3, L=8, ctx_range=(10, 500), seed=9))
    b = W.make_inputs(W.Spec("x", B=3, L=8, ctx_range=(10, 500), seed=9))
    c = W.make_inputs(W.Spec("x", B=3, L=8, ctx_range=(10, 500), seed=10))
    for k in ("qkv", "positions", "page_table", "cache_loc", "k_cache", "v_cache"):
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["qkv"], c["qkv"])


def test_cache_prefill_scales_and_gate_std():
    s = 1 / 64
    inp = W.make_inputs(W.Spec("s", B=2, ctx=4000, kv_scale=s, gate_std=2.0, seed=5))
    k = _e4m3_values(inp["k_cache"]).reshape(-1, 64) * s
    v = _e4m3_values(inp["v_cache"]).reshape(-1, 64) * s
    krms = k.pow(2).mean(-1).sqrt()
    assert abs(float(krms.mean()) - 1.0) < 0.03        # unit-RMS keys, stored / scale
    assert abs(float(v.std()) - 1.0) < 0.03            # N(0, 1) values
    gate = inp["qkv"].float()[:, W.GATE_OFF:]
    assert abs(float(gate.std()) - 2.0) < 0.15
    q = inp["qkv"].float()[:, :W.GATE_OFF]
    assert abs(float(q.std()) - 1.0) < 0.1


def test_coherent_keys_share_a_direction():
    inp = W.make_inputs(W.Spec("co", B=1, ctx=3000, dist="coherent", seed=6))
    k = _e4m3_values(inp["k_cache"]).reshape(-1, 2, 64)
    for g in range(2):
        kg = torch.nn.functional.normalize(k[:, g], dim=-1)
        mean_dir = torch.nn.functional.normalize(kg.mean(0), dim=0)
        assert float((kg @ mean_dir).mean()) > 0.8
    # plain draws do not
    k0 = _e4m3_values(W.make_inputs(W.Spec("n", B=1, ctx=3000, seed=6))["k_cache"]).reshape(-1, 2, 64)
    kg = torch.nn.functional.normalize(k0[:, 0], dim=-1)
    assert float((kg @ torch.nn.functional.normalize(kg.mean(0), dim=0)).mean()) < 0.2


def test_edges_put_the_query_direction_at_the_window_edges():
    W_ = 64
    inp = W.make_inputs(W.Spec("e", B=2, ctx=500, window=W_, dist="edges", seed=7))
    pos = inp["positions"].numpy()
    pt = inp["page_table"].numpy()
    k = _e4m3_values(inp["k_cache"]).reshape(-1, 2, 64)
    q = inp["qkv"].float()[:, :16 * 64].view(-1, 2, 8, 64).mean(2)
    for t in range(2):
        for key in (pos[t] - W_ + 1, pos[t] - W_):          # oldest inside, newest outside
            row = int(pt[t, key])
            for g in range(2):
                cos = torch.nn.functional.cosine_similarity(k[row, g], q[t, g], dim=0)
                assert float(cos) > 0.95
                assert float(k[row, g].pow(2).mean().sqrt()) > 2.5   # scaled-up key


def test_edges_on_a_full_layer_mark_the_oldest_and_newest_cached_keys():
    inp = W.make_inputs(W.Spec("ef", B=3, ctx=700, dist="edges", seed=17))
    pt = inp["page_table"].numpy()
    seq = inp["seq_lens"].numpy()
    k = _e4m3_values(inp["k_cache"]).reshape(-1, 2, 64)
    q = inp["qkv"].float()[:, :16 * 64].view(-1, 2, 8, 64).mean(2)
    rms = k.pow(2).mean(-1).sqrt()                       # [rows, 2]
    for b in range(3):
        for key in (0, int(seq[b]) - 1):
            row = int(pt[b, key])
            assert float(rms[row].min()) > 2.5
            for g in range(2):
                assert float(torch.nn.functional.cosine_similarity(k[row, g], q[b, g], dim=0)) > 0.95
    # every other row keeps the plain unit-RMS draw
    marked = {int(pt[b, key]) for b in range(3) for key in (0, int(seq[b]) - 1)}
    others = [r for r in range(k.shape[0]) if r not in marked]
    assert float(rms[others].max()) < 2.0


def test_outlier_channels_carry_sixteen_times_the_scale():
    inp = W.make_inputs(W.Spec("o", B=1, L=8, ctx=2000, dist="outliers", seed=8))
    k = _e4m3_values(inp["k_cache"]).reshape(-1, 2, 64).abs().mean(0)   # [2, 64]
    for g in range(2):
        top2 = torch.topk(k[g], 3).values
        assert float(top2[1] / top2[2]) > 4.0        # two channels stand far above the rest


def test_keys_attended_closed_forms():
    inp = W.make_inputs(W.Spec("k", B=3, L=8, seq_lens=[0, 100, 5000], seed=1))
    assert W.keys_attended(inp) == (0 + 8) + (100 + 8) + (5000 + 8)
    inp = W.make_inputs(W.Spec("k", B=3, L=8, seq_lens=[0, 100, 5000], window=64, seed=1))
    # the union of the block's windows: first token's lo to the last position
    assert W.keys_attended(inp) == 8 + (64 + 7) + (64 + 7)
    inp = W.make_inputs(W.Spec("k", B=1, L=1, seq_lens=[10], window=2048, seed=1))
    assert W.keys_attended(inp) == 11


def test_the_page_load_table_shapes():
    # decode and verify at B = 1, 16, 32; sliding layers: window 2,048 with RoPE;
    # full layers: whole context, no RoPE; page size 1; contexts up to 80,000
    seen = set()
    for load, layer, name in W.LOAD_SET:
        s = W.named(name)
        kind, b = load.split()
        assert s.B == int(b) and s.L == (1 if kind == "decode" else 8)
        assert s.page_size == 1
        if layer == "sliding":   # "dist soft": the plain draw
            assert s.window == 2048 and s.use_rope and s.dist == "normal"
        else:                    # "dist coherent"
            assert s.window == 0 and not s.use_rope and s.dist == "coherent"
        hi = s.ctx if s.ctx is not None else s.ctx_range[1]
        assert hi == 80000
        seen.add((load, layer))
    assert len(seen) == 12
