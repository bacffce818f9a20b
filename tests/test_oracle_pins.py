"""Pins for the CPU oracle: each check rests on something other than the
oracle itself (a closed form, a library routine, an invariant of the
mathematics, or a number printed on the task page), so that a dropped term,
a wrong sign or index, or a transposed operand in the oracle fails here.

Page: "Gated attention decode (muse_attention_decode)", sections "What to
compute", "Shapes" and the load table.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_fp8_gated_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore")

HQ, HKV, D = 16, 2, 64


# ----------------------------------------------------------------------------
# E4M3 codec (OCP FP8 E4M3: bias 7, max 448, no Inf, NaN = S.1111.111)
# ----------------------------------------------------------------------------

def _torch_e4m3_value(code: int) -> float:
    return float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float())


def test_e4m3_decode_matches_torch_and_closed_form():
    for c in range(256):
        v = O.e4m3_decode(c)
        t = _torch_e4m3_value(c)
        if (c & 0x7F) == 0x7F:
            assert math.isnan(v) and math.isnan(t)
            continue
        assert v == t, (c, v, t)
        assert math.copysign(1.0, v) == math.copysign(1.0, t)
    # closed forms of the format
    assert O.e4m3_decode(0x01) == 2.0 ** -9          # smallest subnormal
    assert O.e4m3_decode(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert O.e4m3_decode(0x08) == 2.0 ** -6          # smallest normal
    assert O.e4m3_decode(0x38) == 1.0                # exponent field 7 = bias
    assert O.e4m3_decode(0x7E) == 448.0              # 1.75 * 2^8
    assert O.e4m3_decode(0xFE) == -448.0


def test_e4m3_encode_roundtrip_all_finite_codes():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert O.e4m3_encode(O.e4m3_decode(c)) == c, hex(c)


def test_e4m3_encode_ties_to_even_and_saturates():
    finite = sorted({O.e4m3_decode(c) for c in range(0x7F)})  # non-negative values
    for a, b in zip(finite[:-1], finite[1:]):
        mid = (a + b) / 2
        assert np.float32(mid) == mid                # exactly representable in float32
        ca, cb = O.e4m3_encode(a), O.e4m3_encode(b)
        even = ca if (ca & 1) == 0 else cb
        assert O.e4m3_encode(mid) == even, (a, b)
        assert O.e4m3_encode(-mid) == (even | 0x80)
        # just off the midpoint goes to the nearer side
        assert O.e4m3_encode(np.nextafter(np.float32(mid), np.float32(0))) == ca
        assert O.e4m3_encode(np.nextafter(np.float32(mid), np.float32(1e9))) == cb
    for x in (448.0, 449.0, 463.9, 464.0, 500.0, 1e6, float("inf")):
        assert O.e4m3_encode(x) == 0x7E
        assert O.e4m3_encode(-x) == 0xFE
    assert O.e4m3_encode(float("nan")) & 0x7F == 0x7F
    assert O.e4m3_encode(-0.0) == 0x80
    assert O.e4m3_encode(2.0 ** -10) == 0x00          # half the smallest subnormal: tie to 0
    assert O.e4m3_encode(3 * 2.0 ** -11) == 0x01


def test_e4m3_encode_matches_torch_cast_in_range():
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (0.01, 1.0, 30.0, 150.0)])
    x = x.clamp(-447.0, 447.0)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.e4m3_encode(float(v)) for v in x.numpy()], dtype=np.uint8)
    assert (got == ref).all()


# ----------------------------------------------------------------------------
# bf16
# ----------------------------------------------------------------------------

def test_bf16_codec_matches_torch():
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-30, 1e-3, 1.0, 1e3, 1e30)])
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([O.bf16_encode(float(v)) for v in x.numpy()], dtype=np.uint16)
    assert (got == ref).all()
    for bits in (0x0000, 0x3F80, 0xBF80, 0x0001, 0x7F7F):
        assert O.bf16_decode(bits) == float(torch.tensor([bits], dtype=torch.int32)
                                            .to(torch.int16).view(torch.bfloat16).float())
    # ties to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7
    assert O.bf16_encode(1.0 + 2.0 ** -8) == 0x3F80
    assert O.bf16_encode(1.0 + 3 * 2.0 ** -8) == 0x3F82


# ----------------------------------------------------------------------------
# rmsnorm and RoPE
# ----------------------------------------------------------------------------

def test_rmsnorm_unit_rms_and_eps():
    rng = np.random.default_rng(0)
    for _ in range(20):
        x = rng.normal(size=64) * rng.uniform(0.1, 10)
        y = O.rmsnorm(x)
        ms = np.mean(x * x)
        assert np.sqrt(np.mean(y * y)) == pytest.approx(math.sqrt(ms / (ms + 1e-6)), rel=1e-12)
        assert np.all(np.sign(y) == np.sign(x))
    # eps = 1e-6 decides this case: x = 1e-3 * ones has mean square 1e-6
    y = O.rmsnorm(np.full(64, 1e-3))
    assert y == pytest.approx(np.full(64, 1e-3 / math.sqrt(2e-6)), rel=1e-14)


def test_rope_identity_at_zero_and_closed_form():
    rng = np.random.default_rng(1)
    u = rng.normal(size=64)
    assert np.array_equal(O.rope_neox(u, 0.0), u)
    # unit vector on dim i rotates into dim i+32 by angle p * 10000^(-2i/64)
    for i, p in ((0, 1.0), (1, 1.0), (5, 37.0), (31, 80000.0)):
        e = np.zeros(64)
        e[i] = 1.0
        r = O.rope_neox(e, p)
        ang = p * 10000.0 ** (-i / 32.0)
        assert r[i] == pytest.approx(math.cos(ang), abs=1e-12)
        assert r[i + 32] == pytest.approx(math.sin(ang), abs=1e-12)
        assert np.count_nonzero(np.abs(r) > 1e-15) <= 2
        e2 = np.zeros(64)
        e2[i + 32] = 1.0
        r2 = O.rope_neox(e2, p)
        assert r2[i] == pytest.approx(-math.sin(ang), abs=1e-12)
        assert r2[i + 32] == pytest.approx(math.cos(ang), abs=1e-12)


def test_rope_norm_and_relative_position():
    rng = np.random.default_rng(2)
    q, k = rng.normal(size=64), rng.normal(size=64)
    for p in (3.0, 2047.0, 80000.0):
        assert np.linalg.norm(O.rope_neox(q, p)) == pytest.approx(np.linalg.norm(q), rel=1e-13)
    for (pq, pk, d) in ((10.0, 3.0, 5.0), (80000.0, 78000.0, 17.0), (4.0, 4.0, 1000.0)):
        a = np.dot(O.rope_neox(q, pq), O.rope_neox(k, pk))
        b = np.dot(O.rope_neox(q, pq + d), O.rope_neox(k, pk + d))
        assert a == pytest.approx(b, abs=1e-9)


# ----------------------------------------------------------------------------
# Whole step on hand-built tiny inputs
# ----------------------------------------------------------------------------

def _bf16_bits(x) -> np.ndarray:
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy() \
        .astype(np.uint16)


def _codes(x) -> np.ndarray:
    return torch.tensor(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _values(codes) -> np.ndarray:
    return torch.tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _tiny(seq_len, L=1, window=0, rope=False, kv_scale=1.0, seed=0, n_rows=None):
    """One request, identity page table with page size 1."""
    rng = np.random.default_rng(seed)
    T = L
    total = seq_len + L
    rows = n_rows or total
    qkv = rng.normal(size=(T, 2304)).astype(np.float32)
    kc = _codes(rng.normal(size=(rows, 2, 64)) / kv_scale)
    vc = _codes(rng.normal(size=(rows, 2, 64)) / kv_scale)
    pt = np.arange(((total + 3) // 4) * 4, dtype=np.int32)[None, :]
    pos = np.arange(seq_len, seq_len + L, dtype=np.int64)
    return dict(qkv=qkv, kc=kc, vc=vc, pt=pt, pos=pos, cl=pos.copy(), window=window, rope=rope,
                s=kv_scale)


def _run(c, ps=1, want=None):
    return O.attn_decode(_bf16_bits(c["qkv"]), c["pos"], c["pt"], c["cl"], c["kc"], c["vc"],
                         c["s"], c["s"], ps, c["window"], c["rope"], want=want, nthreads=2)


@pytest.mark.parametrize("scale", [1.0, 1 / 64])
def test_single_key_returns_its_value(scale):
    # seq_len 0: the only key is the token's own (quantised) entry, so a = dequant(v).
    c = _tiny(0, kv_scale=scale, seed=4)
    r = _run(c)
    v = _bf16_bits(c["qkv"][0, 1152:1280]).astype(np.uint32) << 16
    v = v.view(np.float32).astype(np.float64)
    expect_codes = _codes(v / scale)
    assert np.array_equal(r.v_cache[0], expect_codes)
    a_expect = _values(expect_codes) * scale
    for h in range(HQ):
        g = h // 8
        assert np.array_equal(r.attn[0, h * 64:(h + 1) * 64], a_expect[g * 64:(g + 1) * 64])


def test_identical_keys_give_mean_value():
    c = _tiny(37, seed=5)
    c["qkv"][:, 1024:1152] = 1.0          # k = ones -> rmsnorm ~ ones -> E4M3 1.0 (0x38)
    c["kc"][:] = 0x38                     # every cached key is the same vector
    r = _run(c)
    assert (r.k_cache[37] == 0x38).all()
    vals = _values(r.v_cache[:38])        # all 38 keys, including the new one
    for h in range(HQ):
        g = h // 8
        assert np.allclose(r.attn[0, h * 64:(h + 1) * 64], vals[:, g * 64:(g + 1) * 64].mean(0),
                           rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("scale", [1.0, 1 / 64])
def test_two_keys_closed_form_logit_scale(scale):
    # q = ones -> q_norm = 5.473 / sqrt(1 + 1e-6) per dim.  Key 0 = x0 * ones (cached),
    # key 1 = ones (new).  s_i = 5.473 * 64 * k_i / (8 * sqrt(1 + 1e-6)).
    c = _tiny(1, kv_scale=scale, seed=6)
    c["qkv"][:, 0:1024] = 1.0
    c["qkv"][:, 1024:1152] = 1.0
    x0 = 0.8125                            # an E4M3 value: 1.625 * 2^-1
    c["kc"][0] = _codes(np.full((2, 64), x0 / scale))
    r = _run(c)
    qn = 5.473 / math.sqrt(1 + 1e-6)
    k1 = _values(r.k_cache[1, 0:1])[0] * scale
    assert k1 == 1.0
    s0 = qn * 64 * x0 / 8
    s1 = qn * 64 * k1 / 8
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    V = _values(r.v_cache[:2]) * scale
    for h in (0, 7, 8, 15):
        g = h // 8
        expect = w0 * V[0, g * 64:(g + 1) * 64] + (1 - w0) * V[1, g * 64:(g + 1) * 64]
        assert np.allclose(r.attn[0, h * 64:(h + 1) * 64], expect, rtol=1e-12, atol=1e-14)


def test_query_head_reads_kv_head_h_div_8():
    # KV head 0 makes key 0 win, KV head 1 makes key 1 win; values differ per key.
    c = _tiny(1, seed=8)
    c["qkv"][:, 0:1024] = 1.0
    c["qkv"][:, 1024:1088] = -1.0          # new key, kv head 0: -ones (loses)
    c["qkv"][:, 1088:1152] = 1.0           # new key, kv head 1: +ones (wins)
    c["kc"][0] = 0x38                      # cached key = +1.0 on both heads
    c["kc"][0, 1] = 0xB8                   # ... except kv head 1 = -1.0
    c["vc"][0] = 0x38                      # cached value = +1 on both heads
    c["qkv"][:, 1152:1280] = -2.0          # new value = -2 on both heads
    r = _run(c)
    for h in range(HQ):
        a = r.attn[0, h * 64:(h + 1) * 64]
        if h < 8:
            assert np.all(a > 0.99)        # key 0 (value +1) dominates
        else:
            assert np.all(a < -1.99)       # key 1 (value -2) dominates


def test_new_cache_rows_are_quantised_normed_keys():
    c = _tiny(20, L=8, seed=9)
    r = _run(c)
    kraw = (_bf16_bits(c["qkv"][:, 1024:1152]).astype(np.uint32) << 16).view(np.float32)
    vraw = (_bf16_bits(c["qkv"][:, 1152:1280]).astype(np.uint32) << 16).view(np.float32)
    for t in range(8):
        row = c["cl"][t]
        for g in range(2):
            k = kraw[t, g * 64:(g + 1) * 64].astype(np.float64)
            kn = k / np.sqrt(np.mean(k * k) + 1e-6)
            assert np.array_equal(r.k_cache[row, g * 64:(g + 1) * 64], _codes(kn.astype(np.float32)))
        assert np.array_equal(r.v_cache[row], _codes(vraw[t]))
    # rows this step does not own are untouched
    assert np.array_equal(r.k_cache[:20], c["kc"][:20].reshape(20, 128))


# ----------------------------------------------------------------------------
# RoPE inside the step ("What to compute": the rotation comes after the
# QK-norm and before the cache write, at each token's own position)
# ----------------------------------------------------------------------------

def _rotate_np(u, p):
    """NeoX half-split rotation written out from its definition: pairs
    (i, i + 32) turn by the angle p * 10000^(-i/32)."""
    u = np.asarray(u, np.float64)
    ang = float(p) * 10000.0 ** (-np.arange(32) / 32.0)
    c, s = np.cos(ang), np.sin(ang)
    return np.concatenate([u[:32] * c - u[32:] * s, u[32:] * c + u[:32] * s])


@pytest.mark.parametrize("scale", [1.0, 1 / 64])
def test_new_cache_rows_are_quantised_rotated_keys(scale):
    # the step writes E4M3(rotate(rmsnorm(k), positions[t]) / scale): rotated
    # before the quantisation, by the token's own position
    c = _tiny(1000, L=8, rope=True, kv_scale=scale, seed=90)
    r = _run(c)
    kraw = (_bf16_bits(c["qkv"][:, 1024:1152]).astype(np.uint32) << 16).view(np.float32)
    for t in range(8):
        p = int(c["pos"][t])
        row = c["cl"][t]
        for g in range(2):
            k = kraw[t, g * 64:(g + 1) * 64].astype(np.float64)
            kn = k / np.sqrt(np.mean(k * k) + 1e-6)
            expect = _codes((_rotate_np(kn, p) / scale).astype(np.float32))
            assert np.array_equal(r.k_cache[row, g * 64:(g + 1) * 64], expect), (t, g)
            # an unrotated key would differ (the positions are far from 0)
            assert not np.array_equal(expect, _codes((kn / scale).astype(np.float32)))


@pytest.mark.parametrize("aligned", [False, True])
def test_rope_in_step_closed_form_logits(aligned):
    """Every query is the unit vector e_1, so after the QK-norm and the x5.473
    it is qn * e_1 (qn = 5.473 / sqrt(1/64 + 1e-6)), and rotated at position p
    it is qn * (cos(p f) e_1 + sin(p f) e_33) with f = 10000^(-1/32).  Cached
    key 0 is a * e_1 and cached key 1 is a * e_33 (stored as they are: cached
    keys were rotated when they were written), so their logits are
    qn * a * cos(p f) / 8 and qn * a * sin(p f) / 8.  The block's new keys are
    either e_5 (orthogonal to every rotated query: logit 0) or e_1 (rotated at
    the writing token's position p_t, so the logit of token j is
    qn * (cos(p_j f) K_1 + sin(p_j f) K_33) / 8 with K the dequantised codes of
    kn * cos(p_t f) and kn * sin(p_t f)).  Two tokens at positions 2 and 3
    fix that each token's q turns by its own position."""
    S, L = 2, 2
    c = _tiny(S, L=L, rope=True, seed=91)
    a = 8.0 if aligned else 0.25           # both are E4M3 values
    c["qkv"][:, 0:1024] = 0.0
    for h in range(16):
        c["qkv"][:, 64 * h + 1] = 1.0      # q_h = e_1
    c["qkv"][:, 1024:1152] = 0.0
    j_new = 1 if aligned else 5
    c["qkv"][:, 1024 + j_new] = 1.0        # k (both KV heads) = e_1 or e_5
    c["qkv"][:, 1088 + j_new] = 1.0
    c["qkv"][:, 1152:1280] = 0.5           # new values 0.5 (an E4M3 value)
    c["kc"][:] = 0
    c["kc"][0, :, 1] = _codes([a])[0]
    c["kc"][1, :, 33] = _codes([a])[0]
    c["vc"][:] = 0
    c["vc"][0] = 0x38                      # +1
    c["vc"][1] = 0xB8                      # -1
    r = _run(c)
    qn = 5.473 / math.sqrt(1.0 / 64 + 1e-6)
    kn = 1.0 / math.sqrt(1.0 / 64 + 1e-6)
    f = 10000.0 ** (-1.0 / 32.0)
    new_k = []                             # (K_1, K_33) of each new key, dequantised
    for t in range(L):
        pt_ = S + t
        if aligned:
            k1, k33 = _values(_codes(np.array([kn * math.cos(pt_ * f), kn * math.sin(pt_ * f)],
                                              np.float32)))
        else:
            k1 = k33 = 0.0
        new_k.append((float(k1), float(k33)))
    for j in range(L):
        p = S + j
        cs, sn = math.cos(p * f), math.sin(p * f)
        logits = [qn * a * cs / 8, qn * a * sn / 8]
        vals = [1.0, -1.0]
        for t in range(j + 1):             # causal in the block
            logits.append(qn * (cs * new_k[t][0] + sn * new_k[t][1]) / 8)
            vals.append(0.5)
        m = max(logits)
        w = np.exp(np.array(logits) - m)
        expect = float(np.dot(w, vals) / w.sum())
        for h in range(16):
            got = r.attn[j, 64 * h:64 * h + 64]
            assert np.allclose(got, expect, rtol=1e-12, atol=1e-15), (j, h, got[0], expect)


def test_window_equals_truncated_full_attention():
    # sliding window W (no rope, so positions only set ranges) over 40 cached keys
    # == full attention over a cache that holds only the last W-1 cached keys.
    W, S = 9, 40
    c = _tiny(S, window=W, seed=10)
    r = _run(c)
    keep = np.arange(S - (W - 1), S)       # the cached keys inside the window
    c2 = dict(c)
    c2["window"] = 0
    c2["kc"] = np.concatenate([c["kc"][keep], c["kc"][S:S + 1]])
    c2["vc"] = np.concatenate([c["vc"][keep], c["vc"][S:S + 1]])
    c2["pt"] = np.arange(12, dtype=np.int32)[None, :]
    c2["pos"] = np.array([W - 1], np.int64)
    c2["cl"] = c2["pos"].copy()
    r2 = _run(c2)
    assert np.array_equal(r.attn, r2.attn)
    assert np.array_equal(r.out, r2.out)
    # and it differs from full attention over all 41 keys
    c3 = dict(c)
    c3["window"] = 0
    assert not np.array_equal(_run(c3).attn, r.attn)


def test_window_bounds_with_verify_block():
    # token j at p = S + j attends p-W < i <= p: check each token against a
    # single-token call at the same position with the block's earlier rows written.
    W, S, L = 6, 30, 8
    c = _tiny(S, L=L, window=W, rope=True, seed=11)
    r = _run(c)
    kc, vc = c["kc"].copy(), c["vc"].copy()
    for j in range(L):
        cj = dict(c)
        cj["qkv"] = c["qkv"][j:j + 1]
        cj["pos"] = c["pos"][j:j + 1]
        cj["cl"] = c["cl"][j:j + 1]
        cj["kc"], cj["vc"] = kc, vc
        rj = _run(cj)
        assert np.array_equal(rj.out[0], r.out[j])
        assert np.array_equal(rj.attn[0], r.attn[j])
        kc, vc = rj.k_cache.reshape(kc.shape), rj.v_cache.reshape(vc.shape)
    assert np.array_equal(kc.reshape(-1, 128), r.k_cache)


@pytest.mark.parametrize("S,L,W", [(0, 40, 0), (30, 40, 16), (5, 37, 7)])
def test_prefill_block_is_sequential_single_token_steps(S, L, W):
    # The prefill page's attention over a block of L > 8 new tokens is causal in
    # the block: token j (position S + j) sees the cached keys and the block's
    # keys up to itself, inside the window when there is one.  So the block
    # equals L single-token steps run one after another, each appending its own
    # row first ("Prefill layer (muse_prefill_layer)", "What to compute").
    c = _tiny(S, L=L, window=W, rope=W > 0, seed=40 + S + L)
    r = _run(c)
    kc, vc = c["kc"].copy(), c["vc"].copy()
    for j in range(L):
        cj = dict(c)
        cj["qkv"] = c["qkv"][j:j + 1]
        cj["pos"] = c["pos"][j:j + 1]
        cj["cl"] = c["cl"][j:j + 1]
        cj["kc"], cj["vc"] = kc, vc
        rj = _run(cj)
        assert np.array_equal(rj.out[0], r.out[j])
        assert np.array_equal(rj.attn[0], r.attn[j])
        kc, vc = rj.k_cache.reshape(kc.shape), rj.v_cache.reshape(vc.shape)
    assert np.array_equal(kc.reshape(-1, 128), r.k_cache)
    assert np.array_equal(vc.reshape(-1, 128), r.v_cache)
    # the block's first token at position 0 sees only its own key: its
    # attention output is exactly its own dequantised value row
    if S == 0:
        for h in range(16):
            g = h // 8
            v0 = _values(r.v_cache[0, 64 * g:64 * g + 64]) * c["s"]
            assert np.array_equal(r.attn[0, 64 * h:64 * h + 64], v0)


def test_page_size_1_and_64_layouts_agree():
    inp = W.make_inputs(W.Spec("t", B=3, L=8, seq_lens=[70, 5, 200], page_size=64,
                               kv_scale=1 / 64, seed=12))
    pt64 = inp["page_table"].numpy()
    kc64 = inp["k_cache"].numpy().reshape(-1, 128)
    vc64 = inp["v_cache"].numpy().reshape(-1, 128)
    args = dict(k_scale=inp["k_scale"], v_scale=inp["v_scale"], window=0, use_rope=False)
    qkv = inp["qkv"].view(torch.int16).numpy().astype(np.uint16)
    pos = inp["positions"].numpy()
    r64 = O.attn_decode(qkv, pos, pt64, inp["cache_loc"], kc64, vc64, page_size=64, **args)
    # the same logical keys laid out one per row, rows shuffled
    B = 3
    total = pos.reshape(B, 8)[:, -1] + 1
    rng = np.random.default_rng(0)
    perm = rng.permutation(int(total.sum()))
    pt1 = np.zeros((B, int(total.max())), np.int32)
    kc1 = np.zeros((perm.size, 128), np.uint8)
    vc1 = np.zeros_like(kc1)
    off = 0
    for b in range(B):
        for i in range(int(total[b])):
            src = pt64[b, i // 64] * 64 + i % 64
            dst = perm[off + i]
            pt1[b, i] = dst
            kc1[dst] = kc64[src]
            vc1[dst] = vc64[src]
        off += int(total[b])
    cl1 = pt1[np.repeat(np.arange(B), 8), pos]
    r1 = O.attn_decode(qkv, pos, pt1, cl1, kc1, vc1, page_size=1, **args)
    assert np.array_equal(r1.out, r64.out)
    assert np.array_equal(r1.attn, r64.attn)


def test_zero_gate_halves_the_normed_output():
    c = _tiny(50, seed=13)
    c["qkv"][:, 1280:] = 0.0
    r = _run(c)
    y2 = 2.0 * r.out_exact[0].reshape(16, 64)
    a = r.attn[0].reshape(16, 64)
    ms = (a * a).mean(1)
    # 2 * out has RMS sqrt(ms / (ms + eps)) per head and the sign of a
    assert np.allclose(np.sqrt((y2 * y2).mean(1)), np.sqrt(ms / (ms + 1e-6)), rtol=1e-12)
    assert np.all(np.sign(y2) == np.sign(a))
    # large positive gates pass the normed value through, large negative ones close it
    c["qkv"][:, 1280:] = 30.0
    assert np.allclose(_run(c).out_exact, r.out_exact * 2, rtol=1e-12)


def test_output_is_bf16_of_exact():
    c = _tiny(64, seed=14)
    r = _run(c)
    ref = torch.tensor(r.out_exact.astype(np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().astype(np.uint16)
    # double -> bf16 in one rounding vs double -> float -> bf16: equal except at
    # float-level ties, which random data does not hit
    assert np.array_equal(ref, r.out)


def test_want_mask_computes_only_selected_heads():
    c = _tiny(64, L=2, seed=15)
    full = _run(c)
    want = np.zeros((2, 16), bool)
    want[1, 3] = want[0, 15] = True
    part = _run(c, want=want)
    assert np.array_equal(part.out[1, 192:256], full.out[1, 192:256])
    assert np.array_equal(part.out[0, 960:1024], full.out[0, 960:1024])
    assert not part.out[0, :960].any()


# ----------------------------------------------------------------------------
# "heads dp": every head of the layer on one GPU (128 query, 16 KV heads)
# ----------------------------------------------------------------------------

DP_HQ, DP_HKV = 128, 16


def _dp_tiny(seq_len, L=1, window=0, rope=False, seed=0):
    rng = np.random.default_rng(seed)
    total = seq_len + L
    qkv = rng.normal(size=(L, O.qkv_cols(DP_HQ, DP_HKV))).astype(np.float32)
    kc = _codes(rng.normal(size=(total, DP_HKV, 64)))
    vc = _codes(rng.normal(size=(total, DP_HKV, 64)))
    pt = np.arange(((total + 3) // 4) * 4, dtype=np.int32)[None, :]
    pos = np.arange(seq_len, seq_len + L, dtype=np.int64)
    return dict(qkv=qkv, kc=kc, vc=vc, pt=pt, pos=pos, cl=pos.copy(), window=window, rope=rope,
                s=1.0)


def _dp_run(c):
    return O.attn_decode(_bf16_bits(c["qkv"]), c["pos"], c["pt"], c["cl"], c["kc"], c["vc"],
                         c["s"], c["s"], 1, c["window"], c["rope"], nthreads=2, hq=DP_HQ,
                         hkv=DP_HKV)


@pytest.mark.parametrize("L,window,rope", [(1, 0, False), (8, 0, False), (8, 16, True)])
def test_heads_dp_step_is_eight_tp8_steps(L, window, rope):
    """Query heads 8k..8k+7 only ever meet KV head k, so a step over 128/16
    heads must equal eight 16/2-head steps on the matching column slices:
    q and gate columns 1024 g.. (16 heads), k and v columns 128 g.. (2 heads)
    of their own sections, cache bytes 128 g.. of each row."""
    c = _dp_tiny(29, L=L, window=window, rope=rope, seed=21)
    dp = _dp_run(c)
    q_sec, k_sec = 0, DP_HQ * 64
    v_sec, g_sec = k_sec + DP_HKV * 64, k_sec + 2 * DP_HKV * 64
    for g in range(DP_HKV // 2):
        sub = dict(c)
        sub["qkv"] = np.concatenate(
            [c["qkv"][:, q_sec + 1024 * g:q_sec + 1024 * (g + 1)],
             c["qkv"][:, k_sec + 128 * g:k_sec + 128 * (g + 1)],
             c["qkv"][:, v_sec + 128 * g:v_sec + 128 * (g + 1)],
             c["qkv"][:, g_sec + 1024 * g:g_sec + 1024 * (g + 1)]], axis=1)
        sub["kc"] = np.ascontiguousarray(c["kc"][:, 2 * g:2 * g + 2])
        sub["vc"] = np.ascontiguousarray(c["vc"][:, 2 * g:2 * g + 2])
        tp = _run(sub)
        assert np.array_equal(dp.out[:, 1024 * g:1024 * (g + 1)], tp.out)
        assert np.array_equal(dp.k_cache[:, 128 * g:128 * (g + 1)], tp.k_cache)
        assert np.array_equal(dp.v_cache[:, 128 * g:128 * (g + 1)], tp.v_cache)


def test_heads_dp_query_head_reads_kv_head_h_div_8():
    """Two keys per KV head: for even KV heads the cached key wins, for odd
    ones the new key; the winning value is +-(k+1)/4 on KV head k (exact in
    E4M3 and bf16), so each query head's a names the KV head it read."""
    c = _dp_tiny(1, seed=22)
    ks, vs = DP_HQ * 64, DP_HQ * 64 + DP_HKV * 64
    c["qkv"][:, 0:ks] = 1.0                                   # q = ones on every head
    for k in range(DP_HKV):
        sign = 1.0 if k % 2 else -1.0                         # new key +ones wins on odd heads
        c["qkv"][:, ks + 64 * k:ks + 64 * (k + 1)] = sign
        c["kc"][0, k] = 0xB8 if k % 2 else 0x38               # cached key: the other sign
        c["vc"][0, k] = _codes(np.full(64, (k + 1) / 4))      # cached value +(k+1)/4
        c["qkv"][:, vs + 64 * k:vs + 64 * (k + 1)] = -(k + 1) / 4  # new value -(k+1)/4
    r = _dp_run(c)
    for h in range(DP_HQ):
        k = h // 8
        want = -(k + 1) / 4 if k % 2 else (k + 1) / 4
        assert np.allclose(r.attn[0, 64 * h:64 * (h + 1)], want, rtol=1e-12, atol=0), h


def test_heads_dp_gate_columns():
    """A gate of -inf-like size on one query head zeroes that head's output
    alone; the gate section starts at column 64 (hq + 2 hkv) = 10240."""
    c = _dp_tiny(5, seed=23)
    gs = (DP_HQ + 2 * DP_HKV) * 64
    c["qkv"][:, gs + 64 * 77:gs + 64 * 78] = -200.0
    r = _dp_run(c)
    vals = O.bf16_bits_to_float(r.out[0]).reshape(DP_HQ, 64)
    assert (vals[77] == 0).all()                              # +-0 after bf16 rounding
    others = np.delete(vals, 77, axis=0)
    assert (others != 0).sum(axis=1).min() > 32


# ----------------------------------------------------------------------------
# Output projection a = out @ o^T (decoder-layer pages, "What to compute")
# ----------------------------------------------------------------------------

def test_oproj_matches_numpy_matmul():
    """Against numpy's float64 matmul of the decoded bf16 values (a library
    routine, not the oracle's loop), and bf16 of that."""
    rng = np.random.default_rng(31)
    x = _bf16_bits(rng.normal(size=(5, 96)))
    w = _bf16_bits(rng.normal(size=(40, 96)) / 10)
    a, a_exact = O.oproj(x, w, nthreads=3)
    ref = O.bf16_bits_to_float(x) @ O.bf16_bits_to_float(w).T
    assert np.allclose(a_exact, ref, rtol=1e-12, atol=1e-13)
    assert np.array_equal(a, np.array([[O.bf16_encode(v) for v in row] for row in a_exact], np.uint16))


def test_oproj_selection_rows_copy_inputs():
    """Row n of o selects input column n % K (scaled by 2^-j, exact in bf16):
    a[t][n] = out[t][n % K] * 2^-(n % 3), bit for bit."""
    rng = np.random.default_rng(32)
    K, N = 64, 160
    x = _bf16_bits(rng.normal(size=(3, K)))
    wf = np.zeros((N, K), np.float32)
    for n in range(N):
        wf[n, n % K] = 2.0 ** -(n % 3)
    a, _ = O.oproj(x, _bf16_bits(wf), nthreads=2)
    xv = O.bf16_bits_to_float(x)
    want = np.stack([xv[:, n % K] * 2.0 ** -(n % 3) for n in range(N)], axis=1)
    assert np.array_equal(O.bf16_bits_to_float(a), want)


def test_oproj_sign_and_transpose():
    """Negating o negates a; swapping two rows of o swaps the two columns of a
    (a wrong operand order or a transposed weight fails one of these)."""
    rng = np.random.default_rng(33)
    x = _bf16_bits(rng.normal(size=(4, 32)))
    wf = rng.normal(size=(24, 32)).astype(np.float32)
    _, e0 = O.oproj(x, _bf16_bits(wf))
    _, e1 = O.oproj(x, _bf16_bits(-wf))
    assert np.array_equal(e1, -e0)
    ws = wf.copy()
    ws[[3, 17]] = ws[[17, 3]]
    _, e2 = O.oproj(x, _bf16_bits(ws))
    assert np.array_equal(e2[:, [3, 17]], e0[:, [17, 3]])
    # a non-square case where out @ o (no transpose) would not even be defined
    assert e0.shape == (4, 24)


# ----------------------------------------------------------------------------
# The page's own numbers: the floor column of the load table
# ----------------------------------------------------------------------------

def test_floor_table_matches_256_bytes_per_key():
    """The page's floors are bytes / 4.8 TB/s; for one request at ctx 80,000
    on a full layer that is 80,001 keys x 256 bytes (k and v, 2 heads x 64 E4M3
    codes each) -> 4.3 us, and a sliding layer's 2,048 keys -> 0.1 us."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "floors.txt")
    rows = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        load, layer, qlen, floor_us = [s.strip() for s in line.split("|")]
        rows[(load, layer, int(qlen))] = float(floor_us)
    bpk = 2 * HKV * D                      # bytes per key: K and V rows
    full1 = 80001 * bpk / 4.8e12 * 1e6
    assert round(full1, 1) == rows[("decode 1", "full", 1)]
    slide1 = 2048 * bpk / 4.8e12 * 1e6
    assert round(slide1, 1) == rows[("decode 1", "sliding", 1)]
    assert round(80008 * bpk / 4.8e12 * 1e6, 1) == rows[("verify 1", "full", 8)]
