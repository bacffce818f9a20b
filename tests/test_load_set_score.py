"""The load-set aggregation of bench.py --suite against the page's rule
(task page "Gated attention decode (muse_attention_decode)", section "Shapes",
the paragraph under the load table): a load's time is the weighted sum of its
shapes' times and the score is the plain geometric mean over loads.  CPU only."""
import math

import bench
from paged_fp8_gated_b200 import workloads as W


def _row(load, weight, t, f):
    return {"load": load, "weight": weight, "us_per_step": t, "floor_us_page_model": f}


def test_one_load_is_weighted_sum_ratio():
    rows = [_row("a", 46.0, 10.0, 1.0), _row("a", 16.0, 20.0, 10.0)]
    score, ratios = bench.load_set_score(rows)
    assert ratios["a"] == (46 * 1 + 16 * 10) / (46 * 10 + 16 * 20)
    assert score == ratios["a"]


def test_loads_count_equally_whatever_their_size():
    # a load with ten times the shapes' times and floors has the same ratio and
    # the same say in the score as a small one
    small = [_row("s", 46.0, 10.0, 1.0), _row("s", 16.0, 20.0, 10.0)]
    big = [_row("b", 46.0, 100.0, 10.0), _row("b", 16.0, 200.0, 100.0)]
    other = [_row("o", 46.0, 5.0, 4.0), _row("o", 16.0, 8.0, 8.0)]
    s1, r1 = bench.load_set_score(small + other)
    s2, r2 = bench.load_set_score(big + other)
    assert math.isclose(r1["s"], r2["b"], rel_tol=1e-12)
    assert math.isclose(s1, s2, rel_tol=1e-12)
    assert math.isclose(s1, math.sqrt(r1["s"] * r1["o"]), rel_tol=1e-12)


def test_fixed_cost_comes_off_every_shape_time():
    rows = [_row("a", 46.0, 10.0, 1.0), _row("a", 16.0, 20.0, 10.0)]
    _, ratios = bench.load_set_score(rows, fixed_us=4.0)
    assert ratios["a"] == (46 * 1 + 16 * 10) / (46 * 6 + 16 * 16)


def test_page_load_table_has_six_loads_of_two_shapes():
    loads = {}
    for load, layer, _ in W.LOAD_SET:
        loads.setdefault(load, []).append(W.LAYER_WEIGHT[layer])
    assert len(loads) == 6
    assert all(sorted(w) == [16.0, 46.0] for w in loads.values())
