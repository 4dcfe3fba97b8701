"""Pins of the CPU oracle against things other than itself: closed forms,
brute force on tiny inputs, library routines, error bounds and invariants.

Each test names the part of the layer it pins.  A plausible mistake in the
oracle (a dropped term, a wrong sign or index, a transposed operand, a wrong
tie rule) fails at least one of them.
"""
import dataclasses
import itertools
import math

import numpy as np
import pytest

import oracle
import synth

U32 = 2.0 ** -24  # unit roundoff of fp32


def ulp_dist(a, b):
    """Distance in fp32 ulps between two positive fp32 arrays."""
    ai = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ai - bi)


# ----------------------------------------------------------------------------- exp

def test_exp_within_2ulp_of_libm_dense_sweep():
    x = np.linspace(-87.0, 88.0, 2_000_001, dtype=np.float32)
    y = oracle.expf(x)
    ref = np.exp(x.astype(np.float64)).astype(np.float32)  # correctly rounded to fp32 in practice
    assert ulp_dist(y, ref).max() <= 2


def test_exp_special_values_and_clamp():
    assert oracle.expf(np.float32(0.0))[0] == 1.0
    assert ulp_dist(oracle.expf(np.float32(1.0)), np.float32(math.e))[0] <= 1
    # arguments beyond the range are clamped to [-87, 88]
    assert oracle.expf(np.float32(-200.0))[0] == oracle.expf(np.float32(-87.0))[0]
    assert oracle.expf(np.float32(500.0))[0] == oracle.expf(np.float32(88.0))[0]
    # e^a e^-a = 1 within a few ulp on random arguments
    a = synth.uniform(11, 1, (10000,), -40.0, 40.0)
    prod = oracle.expf(a).astype(np.float64) * oracle.expf(-a).astype(np.float64)
    assert np.abs(prod - 1.0).max() < 6 * U32


# ----------------------------------------------------------------------------- quantisation

def test_quant_handcrafted_halves_and_zero_row():
    # amax 127 gives scale exactly 1, so q = rint(v) with ties to even
    row = np.array([127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5, 126.5, -127.0], np.float32)
    q, s = oracle.quantize_rows(row[None, :])
    assert s[0] == 1.0
    assert q[0].tolist() == [127, 2, 4, -2, -4, 0, 0, 2, 126, -127]
    q, s = oracle.quantize_rows(np.zeros((1, 16), np.float32))
    assert s[0] == 0.0 and not q.any()


def test_quant_error_bound_and_full_range():
    v = synth.normal(12, 1, (200, 333), std=3.0)
    v[7] *= 1e-30          # tiny row
    v[9, :] = 0.0
    v[9, 5] = -2.0         # single non-zero entry
    q, s = oracle.quantize_rows(v)
    for r in range(v.shape[0]):
        amax = np.abs(v[r]).max()
        assert s[r] == np.float32(amax) / np.float32(127.0)
        err = np.abs(v[r].astype(np.float64) - q[r].astype(np.float64) * float(s[r]))
        # half a step, plus the rounding of v/s
        assert err.max() <= float(s[r]) * (0.5 + 1e-5)
        assert np.abs(q[r]).max() == 127
    assert q[9, 5] == -127 and np.count_nonzero(q[9]) == 1


def test_quant_tiny_rows_scale_underflow_and_subnormal_scales():
    # amax / 127 underflows to 0 in fp32: scale 0 and codes 0 (like an all-zero row)
    tiny = np.array([1e-44, -3e-45, 0.0, 7e-45], np.float32)
    assert np.float32(np.abs(tiny).max()) / np.float32(127.0) == 0.0
    q, s = oracle.quantize_rows(tiny[None, :])
    assert s[0] == 0.0 and not q.any()
    qf, sf = oracle.quantize_rows_fp8(tiny[None, :])
    assert sf[0] == 0.0 and not qf.any()
    # a subnormal but non-zero scale still rounds to nearest: |v - q s| <= s/2
    for amax in (1e-37, 3e-39, 1e-40, 2e-42):
        v = (synth.normal(40, 1, (1, 300), std=1.0) * np.float32(amax / 4)).astype(np.float32)
        v[0, 0] = np.float32(amax)
        q, s = oracle.quantize_rows(v)
        sc = float(s[0])
        assert 0.0 < sc < 1.2e-38
        vv = v[0].astype(np.float64)
        inside = np.abs(vv / sc) <= 127.0
        err = np.abs(vv - q[0].astype(np.float64) * sc)
        assert np.all(err[inside] <= sc * (0.5 + 2.0 ** -20)), amax
        assert np.all(np.abs(q[0][~inside]) == 127)
        assert np.all(np.sign(q[0]) == np.sign(np.where(np.abs(vv) >= sc / 2, vv, 0.0)))


# ----------------------------------------------------------------------------- activation clip

def test_clip_at_or_above_the_range_changes_nothing():
    x = synth.normal(14, 1, (40, 256), std=2.0)
    inv_s = synth.uniform(14, 2, (256,)) + np.float32(0.5)
    q0, s0 = oracle.quantize_tokens(x, inv_s)
    top = float((np.abs(x * inv_s)).max())
    for clip in (top, top * 2.0, 1e30):
        q, s = oracle.quantize_tokens(x, inv_s, act_clip=clip)
        assert np.array_equal(q, q0) and np.array_equal(s, s0)


def test_clip_saturates_beyond_the_cap_and_keeps_half_step_inside():
    """With the token's range capped at c: the scale is c/127 (one fp32
    division), values within the cap are within half a step, values beyond it
    saturate at +-127 with their sign."""
    x = synth.normal(15, 1, (64, 512), std=1.0)
    x[:, ::50] *= 40.0                       # outlier channels
    c = np.float32(3.0)
    q, s = oracle.quantize_tokens(x, None, act_clip=float(c))
    for t in range(x.shape[0]):
        amax = np.float32(np.abs(x[t]).max())
        cap = min(amax, c)
        assert s[t] == np.float32(cap) / np.float32(127.0)
        inside = np.abs(x[t]) <= cap
        err = np.abs(x[t][inside].astype(np.float64) - q[t][inside].astype(np.float64) * float(s[t]))
        assert err.max() <= float(s[t]) * (0.5 + 1e-5)
        beyond = np.abs(x[t]) > cap * np.float32(1.0001)
        assert np.array_equal(q[t][beyond], np.where(x[t][beyond] > 0, 127, -127).astype(np.int8))
    # a hand-made token: cap 2 -> scale 2/127, 5 and -9 saturate, 1 -> rint(63.5) = 64
    row = np.array([[1.0, 5.0, -9.0, 2.0, -2.0, 0.0]], np.float32)
    q, s = oracle.quantize_tokens(row, None, act_clip=2.0)
    assert s[0] == np.float32(2.0) / np.float32(127.0)
    assert q[0].tolist() == [int(np.rint(np.float32(1.0) / s[0])), 127, -127, 127, -127, 0]


def test_clip_percentile_is_the_nearest_rank_order_statistic():
    x = synth.normal(16, 1, (50, 96), std=1.5)
    inv_s = synth.uniform(16, 2, (96,)) + np.float32(0.25)
    a = np.sort(np.abs((x * inv_s).astype(np.float32)).ravel())
    n = a.size
    for p in (50.0, 99.0, 99.9, 100.0, 1e-9):
        c = oracle.act_clip_percentile(x, inv_s, p)
        rank = max(1, min(n, int(np.ceil(p / 100.0 * n))))
        assert c == a[rank - 1]
        # the defining property, counted directly
        assert (a <= c).sum() >= rank and (a < c).sum() < rank
    assert oracle.act_clip_percentile(x, inv_s, 100.0) == a[-1]


# ----------------------------------------------------------------------------- smoothing

def test_smoothing_identity_fp64():
    """(X diag(s)^-1)(diag(s) W) = X W for the oracle's scales."""
    x = synth.normal(13, 1, (16, 64)).astype(np.float64)
    w = synth.normal(13, 2, (64, 32), std=0.02).astype(np.float64)
    ax = np.abs(x).max(0).astype(np.float32)
    aw = np.abs(w).max(1).astype(np.float32)
    s, inv = oracle.smooth_scales(ax, aw, 0.6)
    s64 = s.astype(np.float64)
    lhs = (x / s64) @ (s64[:, None] * w)
    assert np.abs(lhs - x @ w).max() <= 1e-12 * np.abs(x @ w).max()


def test_smoothing_closed_forms():
    ax = np.array([4.0, 9.0, 0.25, 0.0, 2.0], np.float32)
    aw = np.array([1.0, 4.0, 0.04, 3.0, 0.0], np.float32)
    # alpha = 1: s = max|X|;  alpha = 0: s = 1 / max|W|  (both floored at 1e-5)
    s1, _ = oracle.smooth_scales(ax, aw, 1.0)
    assert np.allclose(s1, np.maximum(ax, np.float32(1e-5)), rtol=1e-7)
    s0, _ = oracle.smooth_scales(ax, aw, 0.0)
    assert np.allclose(s0, 1.0 / np.maximum(aw, np.float32(1e-5)).astype(np.float64), rtol=1e-7)
    # alpha = 1/2 balances the two: max|X_j| / s_j == max|W_j| * s_j
    s, inv = oracle.smooth_scales(ax[:3], aw[:3], 0.5)
    assert np.allclose(ax[:3] / s, aw[:3] * s, rtol=1e-6)
    assert np.allclose(s.astype(np.float64) * inv, 1.0, atol=2 * U32)


def test_channel_absmax_is_the_column_max_of_abs():
    """Calibration statistic ("MiniMax-M3 W8A8 on K100AI" s3.2): per input
    channel, max |x| over the calibration rows; checked against numpy's
    column maximum on a non-square matrix with a negative-only column, a zero
    column and a planted outlier, so a wrong axis or a dropped abs fails."""
    x = synth.normal(21, 1, (37, 48))
    x[:, 5] = -np.abs(x[:, 5]) - 1.0
    x[:, 7] = 0.0
    x[30, 9] = -1e30
    x[0, 47] = 3e-39                          # subnormal, the column's only nonzero
    x[1:, 47] = 0.0
    ref = np.abs(x).max(axis=0)
    assert np.array_equal(oracle.channel_absmax(x), ref)
    assert oracle.channel_absmax(x)[9] == np.float32(1e30)
    assert np.array_equal(oracle.channel_absmax(x[:1]), np.abs(x[0]))
    assert not oracle.channel_absmax(np.zeros((0, 8), np.float32)).any()


def test_gateup_input_absmax_is_the_max_over_experts_and_outputs():
    """Smoothing weight statistic ("MiniMax-M3 W8A8 on K100AI" s6.1, with the
    one-s-per-layer reading): aw_j = max over every expert e and output n of
    |W_gate[e][j][n]| and |W_up[e][j][n]|.  Brute force over (e, n), with each
    row's maximum planted in a different expert, projection, column and sign;
    accumulation over expert chunks equals the one-shot result."""
    E, d, f = 5, 24, 40
    wg = synth.normal(22, 1, (E, d, f), std=0.02)
    wu = synth.normal(22, 2, (E, d, f), std=0.02)
    for j in range(d):
        tgt = wg if j % 2 else wu
        tgt[(3 * j) % E, j, (7 * j) % f] = (-1.0 if j % 3 else 1.0) * (0.5 + j / 100.0)
    brute = np.zeros(d, np.float32)
    for e in range(E):
        for j in range(d):
            for n in range(f):
                brute[j] = max(brute[j], abs(wg[e, j, n]), abs(wu[e, j, n]))
    assert np.array_equal(oracle.gateup_input_absmax(wg, wu), brute)
    aw = np.zeros(d, np.float32)
    for lo, hi in ((0, 2), (2, 3), (3, 5)):
        oracle.gateup_input_absmax(wg[lo:hi], wu[lo:hi], aw)
    assert np.array_equal(aw, brute)
    # every expert and both projections take part: leaving any out changes aw
    assert not np.array_equal(oracle.gateup_input_absmax(wg[:E - 1], wu[:E - 1]), brute)
    assert not np.array_equal(oracle.gateup_input_absmax(wg, np.zeros_like(wu)), brute)
    assert not np.array_equal(oracle.gateup_input_absmax(np.zeros_like(wg), wu), brute)


def test_weight_quant_is_per_output_channel_of_smoothed_weights():
    d, f = 32, 24
    w = synth.normal(14, 3, (d, f), std=0.02)
    s = np.linspace(0.5, 3.0, d).astype(np.float32)
    q, sw = oracle.quantize_gateup_expert(w, s)
    assert q.shape == (f, d)
    ws = (s[:, None] * w).astype(np.float32)           # W'[j][n] = s_j W[j][n]
    for n in range(f):
        assert sw[n] == np.float32(np.abs(ws[:, n]).max()) / np.float32(127.0)
        assert np.abs(ws[:, n] - q[n] * sw[n]).max() <= sw[n] * 0.50001
    qd, swd = oracle.quantize_down_expert(w.T.copy())   # [f][d] -> channels over d
    assert qd.shape == (d, f)
    for n in range(d):
        assert swd[n] == np.float32(np.abs(w.T[:, n]).max()) / np.float32(127.0)


# ----------------------------------------------------------------------------- router

def test_router_logits_within_dot_error_bound():
    T, d, E = 8, 512, 16
    x = synth.normal(15, 1, (T, d))
    x[:, 3] *= 30.0
    wr = synth.normal(15, 2, (d, E), std=0.02)
    lg = oracle.router_logits(x, wr)
    ref = x.astype(np.float64) @ wr.astype(np.float64)
    bound = d * U32 * (np.abs(x).astype(np.float64) @ np.abs(wr).astype(np.float64))
    assert np.all(np.abs(lg - ref) <= bound)


def test_router_logits_order_is_the_stated_one():
    """Hand-made exact cases that tell the stated order (32 lane chains over
    j = 32 i + p, then the xor butterfly 16, 8, 4, 2, 1) apart from a plain
    sequential sum: 2^25 + 1 loses the 1 in fp32, so where a +1 lands decides
    the result."""
    d = 64
    big = 2.0 ** 25

    def logit(prods):
        x = np.zeros((1, d), np.float32)
        w = np.zeros((d, 1), np.float32)
        for j, v in prods.items():
            x[0, j], w[j, 0] = 1.0, v
        return float(oracle.router_logits(x, w)[0, 0])

    # integer partial sums below 2^24 are exact in any order
    x = (np.arange(d) % 7).astype(np.float32)[None, :]
    w = (np.arange(d) % 5).astype(np.float32)[:, None]
    assert oracle.router_logits(x, w)[0, 0] == float((x[0] * w[:, 0]).sum())
    # lane 0 chains j = 0 and j = 32 (cancel exactly), lane 1 holds j = 1
    assert logit({0: big, 32: -big, 1: 1.0}) == 1.0        # sequential j order gives 0
    assert logit({0: big, 1: -big, 32: 1.0}) == 0.0        # sequential j order gives 1
    # butterfly: lane 0 meets lane 16 first, lane 1 only at the last step
    assert logit({0: big, 16: -big, 1: 1.0}) == 1.0        # sequential lane order gives 0
    assert logit({0: big, 1: -big, 16: 1.0}) == 0.0        # sequential lane order gives 1


def _brute_topk(l, k):
    """Brute force over all k-subsets: the chosen set maximises the sum of its
    logits (fp64); among equal sums the lexicographically smallest index tuple
    wins; slots are ordered by logit descending, index ascending."""
    E = len(l)
    best, best_key = None, None
    for S in itertools.combinations(range(E), k):
        key = (-sum(float(l[e]) for e in S), S)
        if best_key is None or key < best_key:
            best, best_key = S, key
    return sorted(best, key=lambda e: (-float(l[e]), e))


def test_topk_brute_force_all_subsets_tiny_config():
    w = synth.WORKLOADS["tiny"]
    data = synth.make_data(w)
    lg = oracle.router_logits(data.x, data.w_router)
    idx, wt = oracle.topk_softmax(lg, w.k)
    for t in range(w.T):
        assert idx[t].tolist() == _brute_topk(lg[t], w.k)


def test_topk_ties_go_to_lowest_index():
    w = synth.WORKLOADS["tiny"]
    data = synth.make_data(w)
    wr = data.w_router.copy()
    wr[:, 5] = wr[:, 2]   # experts 2 and 5 always tie
    wr[:, 7] = wr[:, 2]   # and 7
    lg = oracle.router_logits(data.x, wr)
    assert np.array_equal(lg[:, 2], lg[:, 5]) and np.array_equal(lg[:, 2], lg[:, 7])
    idx, _ = oracle.topk_softmax(lg, 2)
    for t in range(w.T):
        assert idx[t].tolist() == _brute_topk(lg[t], 2)
        if 5 in idx[t] or 7 in idx[t]:
            assert 2 in idx[t]          # 5 or 7 only ever come with (after) 2
    # all-equal logits: slots are 0..k-1 with equal weights 1/k
    idx, wt = oracle.topk_softmax(np.zeros((3, 8), np.float32), 4)
    assert idx.tolist() == [[0, 1, 2, 3]] * 3 and np.all(wt == np.float32(0.25))


def test_gate_weights_softmax_over_selected():
    lg = synth.normal(16, 1, (500, 64), std=2.0)
    bias = synth.zipf_bias(16, 64)
    idx, w = oracle.topk_softmax(lg, 4, bias)
    l = lg.astype(np.float64) + bias.astype(np.float32).astype(np.float64)
    for t in range(0, 500, 7):
        assert idx[t].tolist() == sorted(range(64), key=lambda e: (-np.float32(lg[t, e] + bias[e]), e))[:4]
    sel = np.take_along_axis(l, idx.astype(np.int64), 1)
    ref = np.exp(sel - sel[:, :1])
    ref /= ref.sum(1, keepdims=True)
    assert np.abs(w - ref).max() < 8 * U32
    assert np.abs(w.astype(np.float64).sum(1) - 1.0).max() <= 4 * U32
    assert np.all(np.diff(w, axis=1) <= 0)   # rank order
    # without renormalisation the weights are the full softmax restricted to the k slots
    idx2, w2 = oracle.topk_softmax(lg, 4, bias, renormalize=False)
    full = np.exp(l - l.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    assert np.abs(w2 - np.take_along_axis(full, idx2.astype(np.int64), 1)).max() < 8 * U32


# ----------------------------------------------------------------------------- permutation

def test_permute_matches_stable_sort_and_round_trips():
    T, k, E = 300, 4, 16
    idx = np.stack([synth.permutation(17, 100 + t, E)[:k] for t in range(T)]).astype(np.int32)
    idx[:50] = np.array([3, 0, 1, 2])        # a crowded expert
    offsets, row2ts, ts2row = oracle.permute(idx, E)
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")  # library stable sort by expert
    assert np.array_equal(row2ts, order)
    counts = np.bincount(flat, minlength=E)
    assert np.array_equal(np.diff(offsets), counts) and offsets[-1] == T * k
    assert np.array_equal(row2ts[ts2row.reshape(-1)], np.arange(T * k))
    for e in range(E):
        rows = row2ts[offsets[e]:offsets[e + 1]]
        assert np.all(flat[rows] == e) and np.all(np.diff(rows // k) > 0)


def test_capacity_drops_in_token_order():
    T, k, E = 200, 3, 8
    rng_keys = synth.bits(18, 1, T * k)
    idx = np.zeros((T, k), np.int32)
    for t in range(T):                       # skewed: expert 0 very hot
        choices = []
        for s in range(k):
            c = int(rng_keys[t * k + s] % 4) if s == 0 else int(rng_keys[t * k + s] % E)
            while c in choices:
                c = (c + 1) % E
            choices.append(c)
        idx[t] = choices
    cap = oracle.capacity(1.25, T, k, E)
    assert cap == math.ceil(1.25 * T * k / E)
    offsets, row2ts, ts2row = oracle.permute(idx, E, cap)
    # brute-force simulation in (token, slot) order
    seen = [0] * E
    kept = np.zeros((T, k), bool)
    for t in range(T):
        for s in range(k):
            e = idx[t, s]
            if seen[e] < cap:
                seen[e] += 1
                kept[t, s] = True
    assert np.array_equal(ts2row >= 0, kept)
    counts = np.bincount(idx.reshape(-1), minlength=E)
    assert np.array_equal(np.diff(offsets), np.minimum(counts, cap))
    assert np.array_equal(row2ts[ts2row[kept]], np.flatnonzero(kept.reshape(-1)))
    assert oracle.capacity(0.0, T, k, E) == -1
    assert oracle.capacity(1.25, 4096, 8, 256) == 160


def test_capacity_is_clamped_to_the_row_count():
    """No expert can receive more than T k arrivals, so a capacity factor that
    large keeps everything: the capacity is clamped to T k (also for an
    infinite factor) and the permutation equals the one without a limit."""
    T, k, E = 50, 2, 4
    assert oracle.capacity(1e30, T, k, E) == T * k
    assert oracle.capacity(float("inf"), T, k, E) == T * k
    assert oracle.capacity(float(E), T, k, E) == T * k
    assert oracle.capacity(1.0, T, k, E) == math.ceil(T * k / E)
    keys = synth.bits(19, 1, T * k)
    idx = np.array([[int(keys[t * k]) % E, (int(keys[t * k]) % E + 1 + int(keys[t * k + 1]) % (E - 1)) % E]
                    for t in range(T)], np.int32)
    capped = oracle.permute(idx, E, oracle.capacity(1e30, T, k, E))
    free = oracle.permute(idx, E, -1)
    for a, b in zip(capped, free):
        assert np.array_equal(a, b)


# ----------------------------------------------------------------------------- GEMM

def test_int8_gemm_equals_int64_matmul():
    a = (synth.bits(19, 1, 37 * 300) % 255).astype(np.int64) - 127
    b = (synth.bits(19, 2, 29 * 300) % 255).astype(np.int64) - 127
    a = a.reshape(37, 300)
    b = b.reshape(29, 300)
    a[0] = 127
    b[0] = 127
    b[1] = -127
    c = oracle.gemm_i8(a.astype(np.int8), b.astype(np.int8))
    assert np.array_equal(c.astype(np.int64), a @ b.T)


# ----------------------------------------------------------------------------- whole layer

def _integer_layer(T, d, E, k, f, seed):
    """Inputs on which quantisation is exact: integer-valued X rows with
    |x| max exactly 127, integer weights with every output channel's max 127."""
    def ints(tid, shape):
        v = (synth.bits(seed, tid, int(np.prod(shape))) % 255).astype(np.int64) - 127
        return v.reshape(shape)
    x = ints(1, (T, d))
    x[:, 0] = 127
    wg = ints(2, (E, d, f)); wg[:, 0, :] = 127
    wu = ints(3, (E, d, f)); wu[:, 1, :] = -127
    wd = ints(4, (E, f, d)); wd[:, 0, :] = 127
    # scale the weights so that the dequantised gate/up land in SiLU's interesting range
    return x, wg, wu, wd


def test_whole_layer_closed_form_integer_case():
    T, d, E, k, f = 24, 64, 4, 2, 32
    x, wg, wu, wd = _integer_layer(T, d, E, k, f, 20)
    prep = oracle.prepare(wg.astype(np.float32), wu.astype(np.float32), wd.astype(np.float32),
                          x.astype(np.float32), 0.5, smooth=False)
    assert np.all(prep.sw_gate == 1.0) and np.all(prep.sw_up == 1.0) and np.all(prep.sw_down == 1.0)
    assert np.array_equal(prep.wq_gate.astype(np.int64), wg.transpose(0, 2, 1))
    assert np.array_equal(prep.wq_down.astype(np.int64), wd.transpose(0, 2, 1))
    logits = synth.normal(20, 9, (T, E))
    rt = oracle.route(x.astype(np.float32), k, E, logits=logits)
    y, dbg = oracle.moe_tokens(x.astype(np.float32), prep, rt)
    assert np.all(dbg["sx"] == 1.0) and np.array_equal(dbg["xq"].astype(np.int64), x)
    for t in range(T):
        for s in range(k):
            e = rt.idx[t, s]
            g64 = x[t] @ wg[e]                       # exact integer dot products
            u64 = x[t] @ wu[e]
            assert np.array_equal(dbg["acc1"][t, s, :f], g64)
            assert np.array_equal(dbg["acc1"][t, s, f:], u64)
            # SwiGLU in fp64 from the exact integers (|acc| < 2^24: the fp32 casts are exact)
            g = g64.astype(np.float64)
            with np.errstate(over="ignore"):
                h64 = g / (1.0 + np.exp(-g)) * u64
            sh = float(dbg["sh"][t, s])
            assert abs(sh - np.abs(h64).max() / 127.0) <= 4e-7 * sh
            q64 = h64 / sh
            hq = dbg["hq"][t, s].astype(np.int64)
            near_half = np.abs(np.abs(q64 - np.floor(q64)) - 0.5) < 1e-4
            assert np.all((hq == np.clip(np.rint(q64), -127, 127)) | near_half)
            assert np.abs(hq - q64).max() <= 0.5 + 1e-4
            acc2 = hq @ wd[e]
            assert np.array_equal(dbg["acc2"][t, s], acc2)
            o = acc2.astype(np.float64) * sh * float(rt.w[t, s])
            assert np.allclose(dbg["o"][t, s], o, rtol=4 * U32, atol=0)
        o_sum = dbg["o"][t].astype(np.float64).sum(0)
        assert np.allclose(y[t], o_sum, rtol=1e-6, atol=1e-6 * np.abs(o_sum).max())


def test_dense_special_case_e1_k1():
    """E = 1, k = 1 is a dense W8A8 SwiGLU FFN: routing weight exactly 1, every
    token on expert 0, output = FFN(x) up to W8A8 noise."""
    T, d, f = 16, 128, 64
    x = synth.normal(21, 1, (T, d))
    wg = synth.normal(21, 2, (1, d, f), std=0.2)
    wu = synth.normal(21, 3, (1, d, f), std=0.2)
    wd = synth.normal(21, 4, (1, f, d), std=0.2)
    prep = oracle.prepare(wg, wu, wd, x, 0.5)
    rt = oracle.route(x, 1, 1, logits=np.zeros((T, 1), np.float32))
    assert np.all(rt.w == 1.0) and np.all(rt.idx == 0)
    y, _ = oracle.moe_tokens(x, prep, rt)
    x64 = x.astype(np.float64)
    g = x64 @ wg[0].astype(np.float64)
    u = x64 @ wu[0].astype(np.float64)
    ref = (g / (1 + np.exp(-g)) * u) @ wd[0].astype(np.float64)
    rel = np.abs(y - ref).max() / np.abs(ref).max()
    assert rel < 3e-2, rel


def test_moe_vs_unquantised_fp64_sanity():
    """Tiny config: the W8A8 layer tracks the unquantised fp64 MoE with the same
    routing to within W8A8 noise (normwise ~1e-2)."""
    w = synth.WORKLOADS["tiny"]
    wts = synth.make_weights(w)
    data = synth.make_data(w)
    prep = oracle.prepare(wts.w_gate, wts.w_up, wts.w_down, wts.calib_x, w.alpha)
    rt = oracle.route(data.x, w.k, w.E, w_router=data.w_router)
    y, _ = oracle.moe_tokens(data.x, prep, rt)
    x64 = data.x.astype(np.float64)
    ref = np.zeros_like(x64)
    for t in range(w.T):
        for s in range(w.k):
            e = rt.idx[t, s]
            g = x64[t] @ wts.w_gate[e].astype(np.float64)
            u = x64[t] @ wts.w_up[e].astype(np.float64)
            ref[t] += rt.w[t, s] * ((g / (1 + np.exp(-g)) * u) @ wts.w_down[e].astype(np.float64))
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 5e-2, rel


# ----------------------------------------------------------------------------- FP8 (E4M3)

def _e4m3_table():
    """All finite non-negative E4M3 values by code, from the format definition
    (bias 7, 3 mantissa bits, subnormals m 2^-9, code 0x7f is NaN)."""
    vals = []
    for c in range(0x7f):
        e, m = c >> 3, c & 7
        vals.append(m * 2.0 ** -9 if e == 0 else (8 + m) * 2.0 ** (e - 10))
    return np.array(vals)


def _e4m3_brute(v):
    """Nearest finite E4M3 by exhaustive search; ties go to the even code;
    beyond 448 saturate."""
    tab = _e4m3_table()
    out = np.empty(len(v), np.uint8)
    for i, x in enumerate(np.asarray(v, np.float64)):
        a = abs(x)
        dist = np.abs(tab - a)
        best = np.flatnonzero(dist == dist.min())
        c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        if a >= 448.0:
            c = 0x7e
        out[i] = c | (0x80 if np.signbit(x) else 0)
    return out


def test_e4m3_decode_table():
    v = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    tab = _e4m3_table()
    assert np.array_equal(v[:0x7f].astype(np.float64), tab)
    assert np.isnan(v[0x7f]) and np.isnan(v[0xff])
    assert np.array_equal(v[0x80:0xff], -v[:0x7f])
    assert v[0x7e] == 448.0 and v[1] == 2.0 ** -9 and v[8] == 2.0 ** -6
    assert np.all(np.diff(tab) > 0)


def test_e4m3_encode_matches_exhaustive_nearest_with_ties_to_even():
    tab = _e4m3_table()
    mids = (tab[1:] + tab[:-1]) / 2.0
    rng = np.random.default_rng(7)
    dense = np.exp(rng.uniform(np.log(1e-4), np.log(600.0), 4000)).astype(np.float32)
    special = np.array([0.0, 448.0, 449.0, 464.0, 465.0, 1e6, 2.0 ** -10, 3 * 2.0 ** -11, 1e-30], np.float32)
    v = np.concatenate([tab.astype(np.float32), mids.astype(np.float32), dense, special])
    v = np.concatenate([v, -v])
    assert np.array_equal(oracle.e4m3_encode(v), _e4m3_brute(v))
    # every code decodes and re-encodes to itself (the NaN codes excepted)
    codes = np.array([c for c in range(256) if c & 0x7f != 0x7f], np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)


def test_fp8_quant_rows_scale_and_error_bound():
    v = synth.normal(17, 1, (100, 300), std=2.0)
    v[5] = 0.0
    q, s = oracle.quantize_rows_fp8(v)
    assert s[5] == 0.0 and not q[5].any()
    dq = oracle.e4m3_decode(q).astype(np.float64)
    for r in range(v.shape[0]):
        if r == 5:
            continue
        amax = np.abs(v[r]).max()
        assert s[r] == np.float32(amax) / np.float32(448.0)
        assert (q[r] & 0x7f).max() == 0x7e            # the largest value maps to +-448
        t = v[r].astype(np.float64) / float(s[r])
        # half a step of the value's binade (2^-4 relative for normals, 2^-10 absolute below 2^-6)
        step = np.where(np.abs(t) >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(t), 1e-30))) - 3),
                        2.0 ** -9)
        assert np.all(np.abs(t - dq[r]) <= step / 2 * (1 + 1e-6) + 1e-7 * np.abs(t))


def test_fp8_gemm_is_the_exact_sum_rounded_once():
    rng = np.random.default_rng(18)
    a = rng.integers(0, 256, (7, 333), dtype=np.uint8)
    b = rng.integers(0, 256, (5, 333), dtype=np.uint8)
    a[(a & 0x7f) == 0x7f] = 0
    b[(b & 0x7f) == 0x7f] = 0
    c = oracle.gemm_fp8(a, b)
    va, vb = oracle.e4m3_decode(a), oracle.e4m3_decode(b)
    from fractions import Fraction
    for m in range(a.shape[0]):
        for n in range(b.shape[0]):
            exact = sum(Fraction(float(x)) * Fraction(float(y)) for x, y in zip(va[m], vb[n]))
            assert c[m, n] == np.float32(float(exact))


def test_fp8_dense_special_case_e1_k1():
    """E = 1, k = 1: the layer is one dense SwiGLU FFN; the FP8 chain stays
    within FP8 noise (a few 1e-2 relative) of the unquantised fp64 FFN."""
    d, f, T = 128, 256, 8
    x = synth.normal(19, 1, (T, d))
    wg = synth.normal(19, 2, (1, d, f), std=0.05)
    wu = synth.normal(19, 3, (1, d, f), std=0.05)
    wd = synth.normal(19, 4, (1, f, d), std=0.05)
    prep = oracle.prepare_fp8(wg, wu, wd, x, 0.5)
    rt = oracle.route(x, 1, 1, logits=np.zeros((T, 1), np.float32))
    y, dbg = oracle.moe_tokens_fp8(x, prep, rt)
    x64 = x.astype(np.float64)
    g = x64 @ wg[0].astype(np.float64)
    u = x64 @ wu[0].astype(np.float64)
    h = g / (1.0 + np.exp(-g)) * u
    ref = h @ wd[0].astype(np.float64)
    rel = np.abs(y - ref).max() / np.abs(ref).max()
    assert rel < 0.1
    # every stage's debug output decodes to values of the right scale
    assert np.all(dbg["sx"] > 0) and np.all(dbg["sh"] > 0)


def test_fp8_whole_layer_closed_form_exact_codes():
    """E4M3 counterpart of the integer closed form: X rows and weight columns
    drawn from the E4M3 values with each range exactly 448, smoothing off, so
    every scale is 1 and every code is the value itself.  Then the gate/up
    accumulators are exact rational sums rounded once to fp32, the h codes are
    within half an E4M3 step of h / sh, and the down accumulators are the
    exact sums of the decoded h codes -- each checked against fp64 arithmetic
    written here, not the oracle's routines."""
    T, d, E, k, f = 16, 64, 3, 2, 32
    tab = _e4m3_table()
    vals = np.concatenate([tab[8:0x7e], -tab[8:0x7e]])       # normal E4M3 values below 448
    rng = np.random.default_rng(21)

    def draw(shape, axis):
        a = rng.choice(vals, size=shape)                      # exact E4M3 values, |a| <= 416
        # put an exact 448 on every row (axis=1) / column (axis=-2) so the range is 448
        idx = rng.integers(0, a.shape[axis], size=[s for i, s in enumerate(a.shape) if i != axis % a.ndim])
        np.put_along_axis(a, np.expand_dims(idx, axis), 448.0, axis=axis)
        return a
    x = draw((T, d), 1)
    wg = np.stack([draw((d, f), 0) for _ in range(E)])
    wu = np.stack([draw((d, f), 0) for _ in range(E)])
    wd = np.stack([draw((f, d), 0) for _ in range(E)])
    prep = oracle.prepare_fp8(wg.astype(np.float32), wu.astype(np.float32), wd.astype(np.float32),
                              x.astype(np.float32), 0.5, smooth=False)
    assert np.all(prep.sw_gate == 1.0) and np.all(prep.sw_up == 1.0) and np.all(prep.sw_down == 1.0)
    assert np.array_equal(oracle.e4m3_decode(prep.wq_gate).astype(np.float64), wg.transpose(0, 2, 1))
    logits = synth.normal(21, 9, (T, E))
    rt = oracle.route(x.astype(np.float32), k, E, logits=logits)
    y, dbg = oracle.moe_tokens_fp8(x.astype(np.float32), prep, rt)
    assert np.all(dbg["sx"] == 1.0)
    assert np.array_equal(oracle.e4m3_decode(dbg["xq"]).astype(np.float64), x)
    from fractions import Fraction
    for t in range(T):
        for s in range(k):
            e = rt.idx[t, s]
            g_exact = [sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(x[t], wg[e][:, n]))
                       for n in range(f)]
            assert np.array_equal(dbg["acc1"][t, s, :f], np.array([np.float32(float(v)) for v in g_exact]))
            g = dbg["acc1"][t, s, :f].astype(np.float64)
            u = dbg["acc1"][t, s, f:].astype(np.float64)
            assert np.array_equal(dbg["acc1"][t, s, f:], (x[t] @ wu[e]).astype(np.float32))
            with np.errstate(over="ignore"):
                h64 = g / (1.0 + np.exp(-g)) * u
            sh = float(dbg["sh"][t, s])
            assert abs(sh - np.abs(h64).max() / 448.0) <= 1e-6 * sh
            q = h64 / sh
            dq = oracle.e4m3_decode(dbg["hq"][t, s]).astype(np.float64)
            step = np.where(np.abs(q) >= 2.0 ** -6,
                            2.0 ** (np.floor(np.log2(np.maximum(np.abs(q), 1e-30))) - 3), 2.0 ** -9)
            assert np.all(np.abs(dq - q) <= step / 2 * (1 + 1e-4) + 1e-6 * np.abs(q))
            acc2 = wd[e].T @ dq                                      # exact: products fit fp64
            assert np.array_equal(dbg["acc2"][t, s], acc2.astype(np.float32))


# ----------------------------------------------------------------------------- bf16 output cast

def _bf16_rne_by_distance(v32):
    """Round-to-nearest-even to bf16 written from the definition: the two bf16
    neighbours of |v| (its truncation and the next bf16 above it; above the
    largest finite bf16 the next is 2^128, i.e. infinity) are compared by
    exact distance in fp64, a tie goes to the neighbour whose last significand
    bit is 0, and the sign is put back."""
    bits = v32.view(np.uint32).astype(np.uint64)
    lo_bits = bits & 0x7FFF0000
    hi_bits = lo_bits + 0x10000
    lo = lo_bits.astype(np.uint32).view(np.float32).astype(np.float64)
    hi = np.where(hi_bits >= 0x7F800000, 2.0 ** 128,
                  np.minimum(hi_bits, 0x7F7F0000).astype(np.uint32).view(np.float32).astype(np.float64))
    x = np.abs(v32.astype(np.float64))
    d_lo, d_hi = x - lo, hi - x
    lo_even = ((lo_bits >> 16) & 1) == 0
    out = np.where((d_hi < d_lo) | ((d_hi == d_lo) & ~lo_even), hi_bits, lo_bits)
    return (out | (bits & 0x80000000)).astype(np.uint32)


def test_round_bf16_is_round_to_nearest_even():
    """The final bf16 cast of every bf16 layer: equal, bit for bit, to the
    definition above and to torch's fp32 -> bf16 conversion, on every tie
    pattern (even and odd last kept bit, carries into the exponent, the
    largest finite bf16 and the overflow to infinity), on subnormals and on
    10^6 random finite fp32 values."""
    import torch
    pat = []
    for exp_bits in (0x00, 0x01, 0x3F, 0x7E, 0x80, 0xFE):
        for m7 in (0x00, 0x01, 0x3E, 0x7E, 0x7F):
            for low in (0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF):
                for sign in (0, 1):
                    pat.append((sign << 31) | (exp_bits << 23) | (m7 << 16) | low)
    keys = synth.bits(23, 1, 1_000_000).astype(np.uint64)
    rnd = (keys & 0xFFFFFFFF).astype(np.uint32)
    rnd = rnd[((rnd >> 23) & 0xFF) != 0xFF]                  # finite values only
    near_max = (0x7F7F0000 + (keys[:4096] & 0xFFFF)).astype(np.uint32)
    v = np.concatenate([np.array(pat, np.uint32), rnd, near_max]).view(np.float32)
    got = oracle.round_bf16(v).view(np.uint32)
    assert np.array_equal(got, _bf16_rne_by_distance(v))
    lib = torch.from_numpy(v.copy()).to(torch.bfloat16).to(torch.float32).numpy().view(np.uint32)
    assert np.array_equal(got, lib)
    # hand-worked cases: ties to even, carry into the exponent, overflow
    one = np.float32(1.0).view(np.uint32)
    cases = {one | 0x8000: one, (one | 0x10000) | 0x8000: one + 0x20000,
             0x3F7F8000: 0x3F800000, 0x7F7F7FFF: 0x7F7F0000, 0x7F7F8000: 0x7F800000,
             0x00008000: 0x00000000, 0x00018000: 0x00020000}
    for src, dst in cases.items():
        assert oracle.round_bf16(np.array([src], np.uint32).view(np.float32)).view(np.uint32)[0] == dst, hex(src)


def test_bf16_layer_rounds_each_slot_row_then_sums_in_slot_order():
    """For a bf16-output layer the oracle stores each per-slot expert output
    row in bf16 and sums the rows in slot order in fp32 before the final bf16
    cast; for an fp32-output layer the rows stay fp32.  Rebuilt here from the
    oracle's own accumulators with torch's bf16 conversion and numpy sums."""
    import torch
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=12, data_seed=24)
    wts = synth.make_weights(wl)
    data = synth.make_data(wl)
    prep = oracle.prepare(wts.w_gate, wts.w_up, wts.w_down, wts.calib_x, wl.alpha)
    rt = oracle.route(data.x, wl.k, wl.E, w_router=data.w_router)

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).to(torch.float32).numpy()

    for out_bf16 in (False, True):
        y, dbg = oracle.moe_tokens(data.x, prep, rt, out_bf16=out_bf16)
        want = np.zeros_like(y)
        for t in range(wl.T):
            for s_ in range(wl.k):
                e = rt.idx[t, s_]
                o = oracle.down_epilogue(dbg["acc2"][t, s_], float(dbg["sh"][t, s_]), prep.sw_down[e],
                                         float(rt.w[t, s_]))
                if out_bf16:
                    o = bf16(o)
                assert np.array_equal(dbg["o"][t, s_], o)
                want[t] = (want[t] + o).astype(np.float32)
        if out_bf16:
            want = bf16(want)
        assert np.array_equal(y, want)
