"""Randomised pins of the oracle (hypothesis): the independent references of
the fixed-seed pins (brute force over all expert subsets, a token-order
simulation of the capacity rule, the half-step quantisation bound) over many
small adversarial cases: logits on a coarse grid so that ties are frequent,
skewed expert choices, capacities from 1 up, rows of mixed magnitudes."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from tests.test_oracle_pins import _brute_topk

SETTINGS = settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])


@SETTINGS
@given(st.data())
def test_topk_equals_brute_force_under_frequent_ties(data):
    E = data.draw(st.integers(2, 8), label="E")
    k = data.draw(st.integers(1, E), label="k")
    T = data.draw(st.integers(1, 5), label="T")
    # quarter steps in [-1, 1]: many exact ties, and sums exact in fp64
    grid = st.integers(-4, 4)
    lg = np.array(data.draw(st.lists(grid, min_size=T * E, max_size=T * E)), np.float32).reshape(T, E) / 4
    bias = None
    if data.draw(st.booleans(), label="bias"):
        bias = np.array(data.draw(st.lists(grid, min_size=E, max_size=E)), np.float32) / 4
    idx, w = oracle.topk_softmax(lg, k, bias)
    eff = lg if bias is None else (lg + bias[None, :]).astype(np.float32)
    for t in range(T):
        assert idx[t].tolist() == _brute_topk(eff[t], k)
    assert np.all(w > 0) and np.all(np.abs(w.astype(np.float64).sum(1) - 1.0) <= 4 * 2.0 ** -24)
    assert np.all(np.diff(w, axis=1) <= 0)


@SETTINGS
@given(st.data())
def test_permute_with_capacity_equals_token_order_simulation(data):
    E = data.draw(st.integers(1, 8), label="E")
    k = data.draw(st.integers(1, min(E, 4)), label="k")
    T = data.draw(st.integers(1, 40), label="T")
    hot = data.draw(st.integers(0, E - 1), label="hot")
    rows = []
    for _ in range(T):
        perm = data.draw(st.permutations(list(range(E))))
        if data.draw(st.booleans()) and hot not in perm[:k]:
            perm = [hot] + [e for e in perm if e != hot]     # skew toward one expert
        rows.append(perm[:k])
    idx = np.array(rows, np.int32)
    cap = data.draw(st.sampled_from([-1, 1, 2, 3, 5, 1000]), label="cap")
    offsets, row2ts, ts2row = oracle.permute(idx, E, cap)
    # simulation: visit (token, slot) in order, keep an expert's first `cap` arrivals
    seen = [0] * E
    kept = []
    for t in range(T):
        for s in range(k):
            e = int(idx[t, s])
            ok = cap < 0 or seen[e] < cap
            seen[e] += ok
            kept.append(ok)
    flat = idx.reshape(-1)
    expect = [i for e in range(E) for i in range(T * k) if flat[i] == e and kept[i]]
    assert row2ts.tolist() == expect
    assert offsets.tolist() == list(np.concatenate([[0], np.cumsum([seen[e] for e in range(E)])]))
    ts = ts2row.reshape(-1)
    assert [bool(v >= 0) for v in ts] == kept
    assert all(row2ts[ts[i]] == i for i in range(T * k) if kept[i])


@SETTINGS
@given(st.data())
def test_quantised_rows_round_to_nearest(data):
    n = data.draw(st.integers(1, 48), label="n")
    mag = data.draw(st.sampled_from([1e-30, 1e-3, 1.0, 1e3, 1e30]), label="magnitude")
    vals = data.draw(st.lists(st.floats(-1.0, 1.0, width=32), min_size=n, max_size=n))
    v = (np.array(vals, np.float32) * np.float32(mag)).astype(np.float32)
    q, s = oracle.quantize_rows(v[None, :])
    amax = np.float32(np.abs(v).max())
    if amax / np.float32(127.0) == 0.0:          # zero row, or a scale that underflows
        assert s[0] == 0.0 and not q.any()
        return
    sc = float(s[0])
    vv = v.astype(np.float64)
    inside = np.abs(vv / sc) <= 127.0        # a subnormal scale can sit well below amax / 127
    err = np.abs(vv - q[0].astype(np.float64) * sc)
    assert np.all(err[inside] <= sc * (0.5 + 1e-5))
    assert np.all(q[0][~inside] == np.where(vv[~inside] > 0, 127, -127))
    if sc >= 2.0 ** -126:                    # a normal scale: the largest value gets the full range
        assert np.abs(q[0]).max() == 127
    assert np.all((q[0] == 0) | (np.sign(q[0]) == np.sign(v)))


@SETTINGS
@given(st.data())
def test_fp8_quantised_rows_round_to_nearest(data):
    n = data.draw(st.integers(1, 48), label="n")
    mag = data.draw(st.sampled_from([1e-30, 1e-3, 1.0, 1e3, 1e30]), label="magnitude")
    vals = data.draw(st.lists(st.floats(-1.0, 1.0, width=32), min_size=n, max_size=n))
    v = (np.array(vals, np.float32) * np.float32(mag)).astype(np.float32)
    q, s = oracle.quantize_rows_fp8(v[None, :])
    if np.float32(np.abs(v).max()) / np.float32(448.0) == 0.0:   # zero row, or a scale that underflows
        assert s[0] == 0.0 and not q.any()
        return
    sc = float(s[0])
    if sc >= 2.0 ** -126:                               # a normal scale: the largest value maps to +-448
        assert (q[0] & 0x7f).max() == 0x7e
    t = v.astype(np.float64) / sc
    dq = oracle.e4m3_decode(q[0]).astype(np.float64)
    inside = np.abs(t) <= 448.0
    # half an E4M3 step of the value's binade (2^-3 of the binade for normals, 2^-9 below 2^-6)
    step = np.where(np.abs(t) >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(t), 1e-30))) - 3),
                    2.0 ** -9)
    assert np.all((np.abs(t - dq) <= step / 2 * (1 + 1e-6) + 1e-7 * np.abs(t))[inside])
    assert np.all(np.abs(dq[~inside]) == 448.0)
    assert np.all((dq == 0) | (np.sign(dq) == np.sign(v)))
