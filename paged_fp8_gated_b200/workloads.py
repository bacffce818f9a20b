"""Seeded synthetic inputs for one attention step (decode or verify block).

This module only draws random inputs with the shapes, value distributions and
paging structure of the loads on the task page "Gated attention decode
(muse_attention_decode)" (sections "Shapes" and the load table).  It holds
none of the attention arithmetic: the pre-existing cache contents are shaped
with torch's own normalisation and float8 cast, which are distribution
recipes, not steps of the method.  Both the CUDA path and the oracle consume
what it returns.

Layouts (all torch CPU tensors), for hq query and hkv KV heads (16 and 2 on
the page's "heads tp8" shapes, 128 and 16 on its "heads dp" ones):
  qkv        bf16  [T, 64 (2 hq + 2 hkv)]  q | k | v | gate, T = B*L
  positions  int64 [T]        seq_lens[b] + j for token t = b*L + j
  seq_lens   int32 [B]        tokens cached before this step
  page_table int32 [B, max_pages]
  cache_loc  int64 [T]        cache row (page*page_size + slot) of token t
  k_cache    uint8 [num_pages, page_size, hkv, 64]   E4M3 codes
  v_cache    uint8 [num_pages, page_size, hkv, 64]
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

HQ, HKV, D = 16, 2, 64                    # "heads tp8": per GPU of eight
DP_HQ, DP_HKV = 8 * HQ, 8 * HKV           # "heads dp": all heads on one GPU
QKV_COLS = HQ * D + 2 * HKV * D + HQ * D  # 2304
GATE_OFF = HQ * D + 2 * HKV * D           # 1280
ROW_BYTES = HKV * D                       # 128


def qkv_cols(hq: int, hkv: int) -> int:
    return (2 * hq + 2 * hkv) * D


@dataclass
class Spec:
    """One synthetic step.  ``seq_lens`` may be a list, or None with ``ctx``
    (all requests at ``ctx``) or ``ctx_range`` (uniform integers, inclusive)."""
    name: str
    B: int
    L: int = 1
    ctx: int | None = None
    ctx_range: tuple[int, int] | None = None
    seq_lens: list[int] | None = None
    window: int = 0            # > 0: sliding window; 0: full attention
    use_rope: bool = False
    page_size: int = 1
    permute: bool = True       # shuffle page ids over the pool
    kv_scale: float = 1.0
    gate_std: float = 1.0
    seed: int = 0
    spare_pages: int = 0       # unused pages in the pool
    dist: str = "normal"       # "normal", "coherent", "edges" or "outliers" (see make_inputs)
    hq: int = HQ               # query heads
    hkv: int = HKV             # key/value heads
    extra: dict = field(default_factory=dict)


def _unit_rms(x: torch.Tensor) -> torch.Tensor:
    return x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + 1e-6)


def _to_e4m3_codes(x: torch.Tensor) -> torch.Tensor:
    return x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def resolve_seq_lens(spec: Spec, gen: torch.Generator) -> np.ndarray:
    if spec.seq_lens is not None:
        s = np.asarray(spec.seq_lens, dtype=np.int64)
    elif spec.ctx_range is not None:
        lo, hi = spec.ctx_range
        s = torch.randint(lo, hi + 1, (spec.B,), generator=gen).numpy().astype(np.int64)
    else:
        s = np.full(spec.B, int(spec.ctx), dtype=np.int64)
    assert s.shape == (spec.B,) and (s >= 0).all()
    return s


def make_inputs(spec: Spec) -> dict:
    """Draw one step's inputs.  Deterministic in ``spec`` (including its seed)."""
    gen = torch.Generator().manual_seed(int(spec.seed))
    B, L, ps = spec.B, spec.L, spec.page_size
    hq, hkv = spec.hq, spec.hkv
    T = B * L
    seq = resolve_seq_lens(spec, gen)
    total = seq + L                                   # keys per request after the append
    pages_per_req = (total + ps - 1) // ps
    n_pages = int(pages_per_req.sum()) + int(spec.spare_pages)
    max_pages = int(pages_per_req.max())
    max_pages = (max_pages + 3) // 4 * 4              # 16-byte row pitch for the page table

    if spec.permute:
        pool = torch.randperm(n_pages, generator=gen).numpy().astype(np.int64)
    else:
        pool = np.arange(n_pages, dtype=np.int64)
    page_table = np.zeros((B, max_pages), dtype=np.int32)
    off = 0
    for b in range(B):
        n = int(pages_per_req[b])
        page_table[b, :n] = pool[off:off + n]
        off += n

    positions = (seq[:, None] + np.arange(L)[None, :]).reshape(-1).astype(np.int64)
    b_of_t = np.repeat(np.arange(B), L)
    cache_loc = (page_table[b_of_t, positions // ps].astype(np.int64) * ps + positions % ps)

    qkv = torch.randn(T, qkv_cols(hq, hkv), generator=gen)
    if spec.gate_std != 1.0:
        qkv[:, (hq + 2 * hkv) * D:] *= spec.gate_std
    outlier_dims = None
    if spec.dist == "outliers":
        # Two channels per KV head carry 16x the scale in q and k (and in the
        # cached keys below), so after the QK-norm those channels dominate the
        # directions and the scores reach several tens: sharp attention.
        outlier_dims = torch.stack([torch.randperm(D, generator=gen)[:2] for _ in range(hkv)])
        grp = hq // hkv
        for g in range(hkv):
            for c in outlier_dims[g].tolist():
                qkv[:, [(g * grp + h) * D + c for h in range(grp)]] *= 16.0
                qkv[:, hq * D + g * D + c] *= 16.0
    qkv = qkv.to(torch.bfloat16)

    # Pre-existing cache: K = E4M3(unit-RMS N(0,1) / scale), V = E4M3(N(0,1) / scale),
    # drawn for every slot of the pool (including the rows this step overwrites).
    rows = n_pages * ps
    k_cache = torch.empty(rows, hkv, D, dtype=torch.uint8)
    v_cache = torch.empty(rows, hkv, D, dtype=torch.uint8)
    chunk = 1 << 20
    inv = 1.0 / float(spec.kv_scale)
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        kx = torch.randn(r1 - r0, hkv, D, generator=gen)
        if outlier_dims is not None:
            for g in range(hkv):
                kx[:, g, outlier_dims[g]] *= 16.0
        kx = _unit_rms(kx)
        vx = torch.randn(r1 - r0, hkv, D, generator=gen)
        k_cache[r0:r1] = _to_e4m3_codes(kx * inv)
        v_cache[r0:r1] = _to_e4m3_codes(vx * inv)

    if spec.dist == "coherent":
        # Keys of each KV head share a direction (so attention spreads over many
        # keys) and values share one too: the page's "dist coherent" loads.
        u = _unit_rms(torch.randn(1, hkv, D, generator=gen))
        vdir = torch.randn(1, hkv, D, generator=gen)
        for r0 in range(0, rows, chunk):
            r1 = min(rows, r0 + chunk)
            kx = _unit_rms(u + 0.35 * torch.randn(r1 - r0, hkv, D, generator=gen))
            vx = vdir + 0.5 * torch.randn(r1 - r0, hkv, D, generator=gen)
            k_cache[r0:r1] = _to_e4m3_codes(kx * inv)
            v_cache[r0:r1] = _to_e4m3_codes(vx * inv)
    elif spec.dist == "edges":
        # Large-logit keys at the window's edges: for every token, the oldest key
        # inside its window and the newest key just outside it copy the token's
        # raw query direction (mean over the KV head's 8 query heads), scaled up.
        # On a full layer the range's edges are its oldest key (0) and its newest
        # cached key.  Meant for layers without RoPE, where that raw direction is
        # the one the scores see; a range off by one key changes the output.
        qraw = qkv.float()[:, :hq * D].view(T, hkv, hq // hkv, D).mean(2)  # [T, hkv, 64]
        for t in range(T):
            b = t // L
            if spec.window > 0:
                edge_keys = (int(positions[t]) - spec.window + 1, int(positions[t]) - spec.window)
            else:
                edge_keys = (0, int(seq[b]) - 1)
            for key in edge_keys:
                if 0 <= key < int(seq[b]):   # cached keys only
                    row = int(page_table[b, key // ps]) * ps + key % ps
                    kdir = _unit_rms(qraw[t])
                    k_cache[row] = _to_e4m3_codes(kdir * (3.0 * inv))
    elif spec.dist not in ("normal", "outliers"):
        raise ValueError(f"unknown dist {spec.dist!r}")

    return dict(
        name=spec.name,
        B=B, L=L, hq=hq, hkv=hkv, page_size=ps, window=int(spec.window),
        use_rope=bool(spec.use_rope),
        k_scale=float(spec.kv_scale), v_scale=float(spec.kv_scale),
        qkv=qkv,
        positions=torch.from_numpy(positions),
        seq_lens=torch.from_numpy(seq.astype(np.int32)),
        page_table=torch.from_numpy(page_table),
        cache_loc=torch.from_numpy(cache_loc),
        k_cache=k_cache.view(n_pages, ps, hkv, D),
        v_cache=v_cache.view(n_pages, ps, hkv, D),
    )


def oproj_weight(seed: int = 7, hidden: int = 8192, k: int = HQ * D) -> torch.Tensor:
    """The decoder layer's output-projection weight o [hidden, k] as seeded
    synthetic bf16 values N(0, 1/k) (the usual fan-in scale; no trained weights
    are available)."""
    gen = torch.Generator().manual_seed(int(seed))
    return (torch.randn(hidden, k, generator=gen) / k ** 0.5).to(torch.bfloat16)


def oproj_input(T: int, seed: int = 8, k: int = HQ * D) -> torch.Tensor:
    """A stand-in for the attention step's output [T, k]: bf16 rows shaped
    like rmsnorm(a) * sigmoid(gate) (unit-RMS rows times sigmoids of N(0,1))."""
    gen = torch.Generator().manual_seed(int(seed))
    x = _unit_rms(torch.randn(T, k // D, D, generator=gen))
    g = torch.sigmoid(torch.randn(T, k // D, D, generator=gen))
    return (x * g).reshape(T, k).to(torch.bfloat16)


def keys_attended(inp: dict) -> int:
    """Distinct cache rows the step reads: sum over requests of the union of
    its tokens' key ranges (full: p_last + 1; sliding: at most W + L - 1)."""
    pos = inp["positions"].numpy().reshape(inp["B"], inp["L"])
    last = pos[:, -1]
    first = pos[:, 0]
    W = inp["window"]
    lo = np.maximum(0, first - W + 1) if W > 0 else np.zeros_like(first)
    return int((last - lo + 1).sum())


# ----------------------------------------------------------------------------
# The page's loads (section "Shapes" and the load table), at the sizes used here
# ----------------------------------------------------------------------------

def named(name: str, seed: int = 0) -> Spec:
    """The standard synthetic steps.  Seed 0 for all, mixed with a per-step offset."""
    specs = {
        # one request, 4096 cached keys + 1 new, full attention, identity pages
        "pr1": Spec("pr1", B=1, L=1, ctx=4096, permute=False, seed=seed),
        # one request at 80,000 cached keys, sliding (window 2048, RoPE) or full
        "decode1_sliding": Spec("decode1_sliding", B=1, L=1, ctx=80000, window=2048,
                                use_rope=True, seed=seed + 11),
        "decode1_full": Spec("decode1_full", B=1, L=1, ctx=80000, dist="coherent", seed=seed + 12),
        # 32 requests, contexts uniform in [40000, 80000], permuted page-1 table
        "decode32_full": Spec("decode32_full", B=32, L=1, ctx_range=(40000, 80000),
                              dist="coherent", seed=seed + 2),
        "decode32_sliding": Spec("decode32_sliding", B=32, L=1, ctx_range=(40000, 80000),
                                 window=2048, use_rope=True, seed=seed + 21),
        # diagnostics for the gather pattern: same step with sequential rows, or 64-key pages
        "decode32_full_seq": Spec("decode32_full_seq", B=32, L=1, ctx_range=(40000, 80000),
                                  permute=False, dist="coherent", seed=seed + 2),
        "decode32_full_p64": Spec("decode32_full_p64", B=32, L=1, ctx_range=(40000, 80000),
                                  page_size=64, dist="coherent", seed=seed + 2),
        # the page's load table (section "Shapes"): decode and verify at B = 1, 16,
        # 32, sliding and full; requests of B > 1 loads draw contexts uniformly
        # from [40000, 80000] like decode32_full; full layers "dist coherent",
        # sliding layers "dist soft" (the plain draw), as the table gives them
        "decode16_full": Spec("decode16_full", B=16, L=1, ctx_range=(40000, 80000), dist="coherent",
                              seed=seed + 51),
        "decode16_sliding": Spec("decode16_sliding", B=16, L=1, ctx_range=(40000, 80000),
                                 window=2048, use_rope=True, seed=seed + 52),
        "verify1_full": Spec("verify1_full", B=1, L=8, ctx=80000, dist="coherent", seed=seed + 53),
        "verify1_sliding": Spec("verify1_sliding", B=1, L=8, ctx=80000, window=2048,
                                use_rope=True, seed=seed + 54),
        "verify32_full": Spec("verify32_full", B=32, L=8, ctx_range=(40000, 80000), dist="coherent",
                              seed=seed + 55),
        "verify32_sliding": Spec("verify32_sliding", B=32, L=8, ctx_range=(40000, 80000),
                                 window=2048, use_rope=True, seed=seed + 56),
        # 16 requests, 8-token causal verify blocks at 80,000 cached keys
        "verify16_sliding": Spec("verify16_sliding", B=16, L=8, ctx=80000, window=2048,
                                 use_rope=True, seed=seed + 31),
        "verify16_full": Spec("verify16_full", B=16, L=8, ctx=80000, dist="coherent", seed=seed + 32),
        # 64-token pages with shuffled ids, cache scale 1/64, gate N(0, 4)
        "paged_full": Spec("paged_full", B=4, L=8, ctx=65536, page_size=64, kv_scale=1 / 64,
                           gate_std=2.0, seed=seed + 41),
        "paged_sliding": Spec("paged_sliding", B=4, L=8, ctx=65536, page_size=64, window=2048,
                              use_rope=True, kv_scale=1 / 64, gate_std=2.0, seed=seed + 42),
        # the page's three "heads dp" gating shapes (128 query, 16 KV heads); their
        # page size is not given, so they take the default pool of 64-token pages
        # ("spread mixed": contexts uniform in [1, ctx])
        "dp8_full_mixed": Spec("dp8_full_mixed", B=8, ctx_range=(1, 8192), page_size=64,
                               hq=DP_HQ, hkv=DP_HKV, seed=seed + 61),
        "dp2_full_v8_soft": Spec("dp2_full_v8_soft", B=2, L=8, ctx=20000, page_size=64,
                                 hq=DP_HQ, hkv=DP_HKV, seed=seed + 62),
        "dp2_full_v8_coherent": Spec("dp2_full_v8_coherent", B=2, L=8, ctx=20000, page_size=64,
                                     dist="coherent", hq=DP_HQ, hkv=DP_HKV, seed=seed + 63),
        # prefill blocks (the page "Prefill layer (muse_prefill_layer)", its load
        # table): 753 new tokens on an 80,000-token context, one or four
        # conversations; a first turn of 16,384 tokens after 0, 32,768 or 65,536
        "prefill1_sliding": Spec("prefill1_sliding", B=1, L=753, ctx=80000, window=2048,
                                 use_rope=True, seed=seed + 71),
        "prefill1_full": Spec("prefill1_full", B=1, L=753, ctx=80000, seed=seed + 72),
        "prefill4_sliding": Spec("prefill4_sliding", B=4, L=753, ctx=80000, window=2048,
                                 use_rope=True, seed=seed + 73),
        "prefill4_full": Spec("prefill4_full", B=4, L=753, ctx=80000, seed=seed + 74),
        "prefill16k_ctx0_full": Spec("prefill16k_ctx0_full", B=1, L=16384, ctx=0, seed=seed + 75),
        "prefill16k_ctx32k_sliding": Spec("prefill16k_ctx32k_sliding", B=1, L=16384, ctx=32768,
                                          window=2048, use_rope=True, seed=seed + 76),
        "prefill16k_ctx32k_full": Spec("prefill16k_ctx32k_full", B=1, L=16384, ctx=32768,
                                       seed=seed + 77),
        "prefill16k_ctx64k_full": Spec("prefill16k_ctx64k_full", B=1, L=16384, ctx=65536,
                                       seed=seed + 78),
    }
    return specs[name]


NAMED = ["pr1", "decode1_sliding", "decode1_full", "decode32_full", "decode32_sliding",
         "verify16_sliding", "verify16_full", "paged_full", "paged_sliding"]

# The page's twelve scored loads (load, layer) -> workload, and the weight the
# page gives each layer kind in its geometric-mean score.
LOAD_SET = [
    ("decode 1", "sliding", "decode1_sliding"), ("decode 1", "full", "decode1_full"),
    ("decode 16", "sliding", "decode16_sliding"), ("decode 16", "full", "decode16_full"),
    ("decode 32", "sliding", "decode32_sliding"), ("decode 32", "full", "decode32_full"),
    ("verify 1", "sliding", "verify1_sliding"), ("verify 1", "full", "verify1_full"),
    ("verify 16", "sliding", "verify16_sliding"), ("verify 16", "full", "verify16_full"),
    ("verify 32", "sliding", "verify32_sliding"), ("verify 32", "full", "verify32_full"),
]
LAYER_WEIGHT = {"sliding": 46.0, "full": 16.0}

# The prefill page's eight scored shapes (load, layer, q_len, ctx) -> workload,
# with the weight it gives each shape inside its load.
PREFILL_SET = [
    ("turn 1", "sliding", "prefill1_sliding", 46.0), ("turn 1", "full", "prefill1_full", 16.0),
    ("turn 4", "sliding", "prefill4_sliding", 46.0), ("turn 4", "full", "prefill4_full", 16.0),
    ("first turn", "full ctx 0", "prefill16k_ctx0_full", 16.0),
    ("first turn", "sliding ctx 32768", "prefill16k_ctx32k_sliding", 138.0),
    ("first turn", "full ctx 32768", "prefill16k_ctx32k_full", 16.0),
    ("first turn", "full ctx 65536", "prefill16k_ctx64k_full", 16.0),
]
