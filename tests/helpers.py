"""Shared test plumbing: move seeded inputs to the GPU, run the library through
its C ABI, run the oracle on the same inputs, compare.

The tolerance on the bf16 output is max |gpu - oracle| <= 2e-2 + 2e-2 |oracle|
element by element, against the oracle's exact (double) output; the cache
bytes written by the step must match bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as O

ATOL = 2e-2
RTOL = 2e-2


def to_device(inp: dict, dev="cuda") -> dict:
    d = dict(inp)
    for k in ("qkv", "positions", "seq_lens", "page_table", "cache_loc", "k_cache", "v_cache"):
        d[k] = inp[k].to(dev)
    d["k_scale_t"] = torch.tensor([inp["k_scale"]], dtype=torch.float32, device=dev)
    d["v_scale_t"] = torch.tensor([inp["v_scale"]], dtype=torch.float32, device=dev)
    return d


def heads(inp: dict) -> tuple[int, int]:
    return inp.get("hq", 16), inp.get("hkv", 2)


def run_gpu(inp: dict, dev="cuda", workspace=None):
    """One step through the C ABI on fresh device copies; returns host arrays
    (out bf16 bits [T, 64 hq], k_cache, v_cache uint8 [rows, 64 hkv])."""
    from paged_fp8_gated_b200 import binding
    hq, hkv = heads(inp)
    d = to_device(inp, dev)
    out = binding.attn_decode(d["qkv"], d["positions"], d["seq_lens"], d["page_table"],
                              d["cache_loc"], d["k_cache"], d["v_cache"], d["k_scale_t"],
                              d["v_scale_t"], inp["page_size"], inp["window"], inp["use_rope"],
                              L=inp["L"], workspace=workspace, hq=hq, hkv=hkv)
    torch.cuda.synchronize()
    T = inp["B"] * inp["L"]
    out_bits = out.view(torch.int16).reshape(T, 64 * hq).cpu().numpy().astype(np.uint16)
    kc = d["k_cache"].reshape(-1, 64 * hkv).cpu().numpy()
    vc = d["v_cache"].reshape(-1, 64 * hkv).cpu().numpy()
    return out_bits, kc, vc


def run_oracle(inp: dict, want=None) -> O.OracleResult:
    hq, hkv = heads(inp)
    qkv = inp["qkv"].view(torch.int16).numpy().astype(np.uint16)
    return O.attn_decode(qkv, inp["positions"], inp["page_table"], inp["cache_loc"],
                         inp["k_cache"].reshape(-1, 64 * hkv), inp["v_cache"].reshape(-1, 64 * hkv),
                         inp["k_scale"], inp["v_scale"], inp["page_size"], inp["window"],
                         inp["use_rope"], want=want, hq=hq, hkv=hkv)


def new_rows(inp: dict) -> np.ndarray:
    return np.unique(inp["cache_loc"].numpy())


def compare(gpu_out_bits: np.ndarray, ref: O.OracleResult, want=None) -> dict:
    """Element-wise check on the selected (token, head) outputs; returns stats."""
    got = O.bf16_bits_to_float(gpu_out_bits)
    exact = ref.out_exact
    T, cols = got.shape
    if want is None:
        mask = np.ones((T, cols), bool)
    else:
        mask = np.repeat(np.asarray(want, bool).reshape(T, cols // 64), 64, axis=1)
    g, e = got[mask], exact[mask]
    err = np.abs(g - e)
    bound = ATOL + RTOL * np.abs(e)
    rel_l2 = float(np.linalg.norm(g - e) / max(np.linalg.norm(e), 1e-30))
    return dict(max_abs=float(err.max()), worst_ratio=float((err / bound).max()),
                n=int(mask.sum()), nonfinite=int((~np.isfinite(g)).sum()), rel_l2=rel_l2,
                ok=bool(np.isfinite(g).all() and (err <= bound).all()))


def sample_want(T: int, n: int, seed: int = 0, hq: int = 16) -> np.ndarray:
    """n (token, head) pairs, always including the first and last token."""
    rng = np.random.default_rng(seed)
    want = np.zeros((T, hq), bool)
    want[0, rng.integers(hq)] = True
    want[T - 1, rng.integers(hq)] = True
    for _ in range(max(0, n - 2)):
        want[rng.integers(T), rng.integers(hq)] = True
    return want
