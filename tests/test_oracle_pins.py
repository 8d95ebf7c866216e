"""Pins for the CPU oracle: checks against values and identities that do not come from the oracle.

* the hand-derived worked example built on the pages' PowerInfer single-layer
  example (hot {3,5,7}, predicted {3,4,5}), tests/golden/powerinfer_example.json;
* the identity behind activation sparsity: with the exact active set
  {i : pre-activation > 0} the sparse output equals the dense FFN output,
  because every skipped neuron contributes an exact zero (53ai.com page,
  section "激活稀疏"); the dense FFN is computed independently with numpy;
* brute force over every subset on tiny layers: a set reproduces the dense
  output exactly when it contains the exact active set;
* the predictor's threshold against its definition sigmoid(z) > 0.5 evaluated
  with an exponential, h and z against an independent numpy evaluation;
* the exact fp16 decoding against numpy for all 65536 bit patterns;
* closed forms: one active neuron, the empty set, a tie and a NaN logit;
* the look-ahead stack (layer l+1's set predicted from layer l's input): a
  two-layer example worked by hand where predicting one layer early changes the
  set and the output, and the special cases where it must equal the plain stack;
* int8 and int4 rows: the quantizer's codes and scales worked by hand (ties to even,
  zero rows), its error bound, and the quantized-row step equal to the fp16 step on
  weights that lie exactly on an int8 or int4 grid.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "powerinfer_example.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


class _L:
    """Minimal layer record for the oracle's duck-typed API."""

    def __init__(self, act, w_up, w_gate, b, w_down, A, B, c):
        class C:
            pass
        self.cfg = C()
        self.cfg.act = act
        self.w_up, self.w_gate, self.b, self.w_down, self.A, self.B, self.c = w_up, w_gate, b, w_down, A, B, c


def _golden_layer(g, act, dtype):
    f = lambda k: np.asarray(g[k], dtype=dtype)
    if act == "relu":
        return _L("relu", f("W_relu_nxd"), None, f("b"), f("W_down_dxn"), f("A_dxr"), f("B_rxn"), f("c"))
    return _L("reglu", f("W_up_reglu_nxd"), f("W_relu_nxd"), f("b"), f("W_down_dxn"), f("A_dxr"), f("B_rxn"),
              f("c"))


# ------------------------------------------------------------------ decoding
def test_half_decode_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits.view(np.float16))
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_f32_decode_exact():
    rng = np.random.default_rng(1)
    v = rng.standard_normal(1000).astype(np.float32)
    assert np.array_equal(oracle.decode(v), v.astype(np.float64))


# ------------------------------------------------------------------ golden example
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_golden_powerinfer_relu(dtype):
    g = _golden()
    L = _golden_layer(g, "relu", dtype)
    x = np.asarray(g["x"], dtype=dtype)
    st = oracle.forward(L, x)
    e = g["expected"]
    assert st.h.tolist() == e["h"]
    assert st.z.tolist() == e["z"]
    assert st.idx.tolist() == e["predicted_set"] == [3, 4, 5]
    hot = {i for i, v in enumerate(g["hotness"]) if v > 0.5}
    assert hot == {3, 5, 7}
    assert 7 not in st.idx and 4 in st.idx  # hot is not active, cold can be
    for k, v in e["relu_a"].items():
        assert st.a[int(k)] == v
    assert st.y.tolist() == e["relu_y"]
    gpre = oracle.preact(x, L.w_up, None, L.b, "relu")
    assert np.flatnonzero(gpre > 0).tolist() == e["exact_set_relu"]


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_golden_powerinfer_reglu(dtype):
    g = _golden()
    L = _golden_layer(g, "reglu", dtype)
    x = np.asarray(g["x"], dtype=dtype)
    st = oracle.forward(L, x)
    e = g["expected"]
    assert st.idx.tolist() == [3, 4, 5]
    for k, v in e["reglu_a"].items():
        assert st.a[int(k)] == v
    assert st.y.tolist() == e["reglu_y"]


def test_golden_stack_two_layers():
    g = _golden()
    L = _golden_layer(g, "relu", np.float16)
    e = g["expected"]["stack2_relu"]
    xL, recs = oracle.forward_stack([L, L], np.asarray(g["x"], np.float64))
    assert [r["x_in"].astype(np.float64).tolist() for r in recs] == e["layer_inputs"]
    assert [np.flatnonzero(r["mask"]).tolist() for r in recs] == e["sets"]
    assert xL.tolist() == e["x_out"]


# ------------------------------------------------------------------ look-ahead stack
def _lookahead_hand_layers():
    """Two ReLU layers, d = n = r = 2, every value exact in fp16.

    Layer 0: A = B = I, c = 0, W_up = I, b = 0, W_down = [[-2, 0], [2, 0]].
    Layer 1: A = B = I, c = 0, W_up = -I, b = 0, W_down = I.
    With x0 = (1, -1): h = relu(x0) = (1, 0), so layer 0's set is {0} and
    y_0 = 1 * W_down[:, 0] = (-2, 2), x_1 = (-1, 1).
    Plain stack: layer 1 predicts from x_1: h = (0, 1), set {1}; its activation is
    relu(-x_1[1]) = 0, so x_2 = x_1 = (-1, 1).
    Look-ahead: layer 1 predicts from x0: h = (1, 0), set {0}; its activation is
    relu(-x_1[0]) = 1, so y_1 = (1, 0) and x_2 = (0, 1).
    """
    f = lambda v: np.asarray(v, dtype=np.float16)
    eye = np.eye(2)
    z2 = np.zeros(2)
    l0 = _L("relu", f(eye), None, f(z2), f([[-2, 0], [2, 0]]), f(eye), f(eye), f(z2))
    l1 = _L("relu", f(-eye), None, f(z2), f(eye), f(eye), f(eye), f(z2))
    return [l0, l1]


def test_lookahead_hand_example():
    layers = _lookahead_hand_layers()
    x0 = np.array([1.0, -1.0])
    xl, recs = oracle.forward_stack_lookahead(layers, x0)
    assert [np.flatnonzero(r["mask"]).tolist() for r in recs] == [[0], [0]]
    assert [r["y"].tolist() for r in recs] == [[-2.0, 2.0], [1.0, 0.0]]
    assert xl.tolist() == [0.0, 1.0]
    xs, recs_s = oracle.forward_stack(layers, x0)
    assert [np.flatnonzero(r["mask"]).tolist() for r in recs_s] == [[0], [1]]
    assert xs.tolist() == [-1.0, 1.0]


@pytest.mark.parametrize("act", ["relu", "reglu"])
def test_lookahead_special_cases_equal_the_stack(act):
    rng = np.random.default_rng(31)
    layers = [_rand_layer(rng, 24, 40, 8, act, np.float16) for _ in range(3)]
    x0 = rng.standard_normal(24)
    # one layer: nothing to look ahead of
    a, ra = oracle.forward_stack_lookahead(layers[:1], x0)
    b, rb = oracle.forward_stack(layers[:1], x0)
    assert np.array_equal(a, b) and np.array_equal(ra[0]["mask"], rb[0]["mask"])
    # layers that add nothing keep every input equal to u_0, so predicting from the
    # previous input is predicting from the current one
    for L in layers[:2]:
        L.w_down = np.zeros_like(L.w_down)
    a, ra = oracle.forward_stack_lookahead(layers, x0)
    b, rb = oracle.forward_stack(layers, x0)
    assert np.array_equal(a, b)
    assert all(np.array_equal(p["mask"], q["mask"]) for p, q in zip(ra, rb))
    assert np.any(a != x0)  # the last layer does add something


@pytest.mark.parametrize("bits", [8, 4])
def test_lookahead_with_quantized_rows_is_the_quantized_step(bits):
    """One layer of the look-ahead stack on quantized rows is the single quantized step:
    x_1 = x_0 + y of forward_q on round(x_0)."""
    rng = np.random.default_rng(33)
    lay = _rand_layer(rng, 32, 48, 8, "reglu", np.float16)
    qr = oracle.quantize_layer(lay, bits=bits)
    x0 = rng.standard_normal(32)
    xl, recs = oracle.forward_stack_lookahead([lay], x0, qrows=[qr])
    step = oracle.forward_q(lay, qr, x0.astype(np.float16))
    assert np.array_equal(recs[0]["mask"], step.mask)
    assert np.array_equal(xl, x0 + step.y)


# ------------------------------------------------------------------ dense identity
def _rand_layer(rng, d, n, r, act, dtype):
    s = 1.0 / np.sqrt(d)
    w_up = (rng.standard_normal((n, d)) * s).astype(dtype)
    w_gate = (rng.standard_normal((n, d)) * s).astype(dtype) if act == "reglu" else None
    b = (rng.standard_normal(n) * 0.5).astype(dtype)
    w_down = (rng.standard_normal((d, n)) * s).astype(dtype)
    A = (rng.standard_normal((d, r)) / np.sqrt(r)).astype(dtype)
    B = (rng.standard_normal((r, n)) / np.sqrt(r)).astype(dtype)
    c = (rng.standard_normal(n) * 0.5).astype(dtype)
    return _L(act, w_up, w_gate, b, w_down, A, B, c)


def _dense_numpy(L, x):
    """Textbook dense FFN in float64 with numpy (independent of the oracle's loops)."""
    x = x.astype(np.float64)
    up = L.w_up.astype(np.float64) @ x
    if L.cfg.act == "relu":
        act = np.maximum(up + L.b.astype(np.float64), 0.0)
    else:
        gate = L.w_gate.astype(np.float64) @ x + L.b.astype(np.float64)
        act = np.maximum(gate, 0.0) * up
    return L.w_down.astype(np.float64) @ act


def _close(a, b, rel=1e-12):
    scale = max(1e-300, float(np.max(np.abs(b))))
    return float(np.max(np.abs(a - b))) <= rel * scale


@pytest.mark.parametrize("act", ["relu", "reglu"])
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_exact_set_equals_dense(act, dtype):
    rng = np.random.default_rng(7)
    for trial in range(4):
        L = _rand_layer(rng, 64, 96, 16, act, dtype)
        x = rng.standard_normal(64).astype(dtype)
        g = oracle.preact(x, L.w_up, L.w_gate, L.b, act)
        s_star = (g > 0).astype(np.uint8)
        assert 0 < s_star.sum() < 96
        _, y = oracle.ffn_masked(x, L.w_up, L.w_gate, L.b, L.w_down, s_star, act)
        assert _close(y, _dense_numpy(L, x))


@pytest.mark.parametrize("act", ["relu", "reglu"])
def test_all_ones_mask_equals_dense(act):
    rng = np.random.default_rng(8)
    L = _rand_layer(rng, 48, 80, 8, act, np.float32)
    x = rng.standard_normal(48).astype(np.float32)
    _, y = oracle.ffn_masked(x, L.w_up, L.w_gate, L.b, L.w_down, np.ones(80, np.uint8), act)
    assert _close(y, _dense_numpy(L, x))


@pytest.mark.parametrize("act", ["relu", "reglu"])
def test_bruteforce_subsets_tiny(act):
    """Over all 2^n sets M: sparse(M) == dense  <=>  M contains the exact active set."""
    rng = np.random.default_rng(9)
    d, n = 12, 10
    L = _rand_layer(rng, d, n, 4, act, np.float32)
    x = rng.standard_normal(d).astype(np.float32)
    g = oracle.preact(x, L.w_up, L.w_gate, L.b, act)
    s_star = g > 0
    assert 2 <= s_star.sum() <= n - 2
    dense = _dense_numpy(L, x)
    for m in range(1 << n):
        mask = np.array([(m >> i) & 1 for i in range(n)], dtype=np.uint8)
        _, y = oracle.ffn_masked(x, L.w_up, L.w_gate, L.b, L.w_down, mask, act)
        contains = bool(np.all(mask[s_star] == 1))
        assert _close(y, dense, 1e-12) == contains, m


# ------------------------------------------------------------------ predictor
def test_predictor_against_sigmoid_definition():
    rng = np.random.default_rng(10)
    for dtype in (np.float32, np.float16):
        d, r, n = 40, 12, 200
        A = (rng.standard_normal((d, r)) / np.sqrt(r)).astype(dtype)
        B = (rng.standard_normal((r, n)) / np.sqrt(r)).astype(dtype)
        c = (rng.standard_normal(n) * 0.3).astype(dtype)
        x = rng.standard_normal(d).astype(dtype)
        h, z, mask = oracle.predictor(x, A, B, c)
        h_np = np.maximum(x.astype(np.float64) @ A.astype(np.float64), 0.0)
        z_np = h_np @ B.astype(np.float64) + c.astype(np.float64)
        assert _close(h, h_np) and _close(z, z_np)
        sig = 1.0 / (1.0 + np.exp(-z_np))
        clear = np.abs(z_np) > 1e-9
        assert np.array_equal(mask[clear].astype(bool), (sig > 0.5)[clear])
        assert 0 < mask.sum() < n


def test_tie_and_nan_are_inactive():
    A = np.eye(2, dtype=np.float32)
    B = np.array([[1.0, 1.0, 1.0], [0.0, 0.0, 0.0]], np.float32)
    x = np.array([2.0, -3.0], np.float32)  # h = (2, 0)
    c = np.array([-2.0, np.nan, -1.0], np.float32)  # z = (0, nan, 1)
    h, z, mask = oracle.predictor(x, A, B, c)
    assert h.tolist() == [2.0, 0.0]
    assert z[0] == 0.0 and np.isnan(z[1]) and z[2] == 1.0
    assert mask.tolist() == [0, 0, 1]


def test_single_active_neuron_closed_form():
    rng = np.random.default_rng(11)
    L = _rand_layer(rng, 32, 20, 4, "relu", np.float16)
    x = rng.standard_normal(32).astype(np.float16)
    g = oracle.preact(x, L.w_up, None, L.b, "relu")
    i = int(np.argmax(g))
    mask = np.zeros(20, np.uint8)
    mask[i] = 1
    a, y = oracle.ffn_masked(x, L.w_up, None, L.b, L.w_down, mask, "relu")
    ai = max(0.0, float(L.w_up[i].astype(np.float64) @ x.astype(np.float64)) + float(L.b[i]))
    assert abs(a[i] - ai) <= 1e-12 * abs(ai)
    assert np.array_equal(y, a[i] * L.w_down[:, i].astype(np.float64))
    assert np.count_nonzero(a) == 1


def test_empty_set_gives_zero():
    rng = np.random.default_rng(12)
    L = _rand_layer(rng, 16, 8, 4, "reglu", np.float32)
    x = rng.standard_normal(16).astype(np.float32)
    a, y = oracle.ffn_masked(x, L.w_up, L.w_gate, L.b, L.w_down, np.zeros(8, np.uint8), "reglu")
    assert not a.any() and not y.any()


# ------------------------------------------------------------------ bookkeeping
def test_batch_rows_are_single_token_steps():
    rng = np.random.default_rng(13)
    L = _rand_layer(rng, 24, 30, 6, "relu", np.float32)
    X = rng.standard_normal((3, 24)).astype(np.float32)
    steps = oracle.forward_batch(L, X)
    for t in range(3):
        st = oracle.forward(L, X[t])
        assert np.array_equal(st.y, steps[t].y) and np.array_equal(st.mask, steps[t].mask)


def test_arbitration_rule():
    z = np.array([0.5, -0.0005, 0.0002, -2.0, 1e-4])
    ref = z > 0
    other = np.array([1, 1, 0, 0, 1], bool)
    use, mism = oracle.arbitrate(z, ref, other)
    assert mism.size == 0
    assert use.tolist() == [1, 1, 0, 0, 1]
    other2 = np.array([0, 0, 1, 0, 1], bool)  # disagrees outside the band on neuron 0
    use2, mism2 = oracle.arbitrate(z, ref, other2)
    assert mism2.tolist() == [0]


def test_tolerance_rule():
    y_ref = np.array([1.0, -2.0, 0.5])
    ok, _ = oracle.within_tolerance(y_ref + 3.9e-3, y_ref)
    bad, _ = oracle.within_tolerance(y_ref + 4.1e-3, y_ref)
    assert ok and not bad
    assert oracle.within_tolerance(np.zeros(3), np.zeros(3))[0]
    assert not oracle.within_tolerance(np.array([0, 1e-30, 0]), np.zeros(3))[0]


# ---------------------------------------------------------------- int8 rows
def test_quantizer_hand_values():
    """Scale = absmax / 127 and codes rounded to nearest even, worked by hand: absmax
    127 gives scale 1 (codes = rounded values, 2.5 -> 2), absmax 254 gives scale 2
    (1.5 -> 2, -2.5 -> -2, 0.5 -> 0), an all-zero row gives scale 0 and codes 0."""
    w = np.array([[127, -3.25, 2.5, 0.75, -127], [254, 3, -5, 1, 0], [0, 0, 0, 0, 0]], np.float16)
    q, s = oracle.quantize(w)
    assert q.tolist() == [[127, -3, 2, 1, -127], [127, 2, -2, 0, 0], [0, 0, 0, 0, 0]]
    assert s.tolist() == [1.0, 2.0, 0.0]
    qc, sc = oracle.quantize(np.ascontiguousarray(w.T), units_along_rows=False)
    assert np.array_equal(qc, q) and np.array_equal(sc, s)


def test_quantizer_hand_values_int4():
    """qmax 7: absmax 7 gives scale 1 (-3.25 -> -3, 2.5 -> 2, 0.75 -> 1), absmax 14 gives
    scale 2 (1.5 -> 2, -2.5 -> -2, 0.5 -> 0), an all-zero row scale 0 and codes 0."""
    w = np.array([[7, -3.25, 2.5, 0.75, -7], [14, 3, -5, 1, 0], [0, 0, 0, 0, 0]], np.float16)
    q, s = oracle.quantize(w, bits=4)
    assert q.tolist() == [[7, -3, 2, 1, -7], [7, 2, -2, 0, 0], [0, 0, 0, 0, 0]]
    assert s.tolist() == [1.0, 2.0, 0.0]


@pytest.mark.parametrize("bits", [8, 4])
def test_quantizer_invariants(bits):
    qmax = 127 if bits == 8 else 7
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((40, 96)) * rng.uniform(0.01, 3.0, (40, 1))).astype(np.float16)
    w[5] = 0
    q, s = oracle.quantize(w, bits=bits)
    wf = w.astype(np.float64)
    assert np.all(np.abs(q.astype(int)) <= qmax)
    nz = np.abs(wf).max(axis=1) > 0
    assert np.all(np.abs(q[nz]).max(axis=1) == qmax)
    assert np.all(s[~nz] == 0) and np.all(q[~nz] == 0)
    # |w - q s| <= s / 2, up to the fp32 rounding of w / s
    err = np.abs(wf - q.astype(np.float64) * s[:, None].astype(np.float64))
    assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 1e-5))
    # the scale is the fp32 quotient absmax / qmax
    amax = np.abs(w.astype(np.float32)).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(qmax)).astype(np.float32))


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("act", ["relu", "reglu"])
def test_forward_q_equals_forward_on_an_exact_grid(act, bits):
    """Weights that are codes times 2^-7 (int8) or 2^-3 (int4) for up and gate and twice
    that for down, exact in fp16, each unit reaching +-qmax: quantization gives back those
    codes and scales, and the quantized-row step equals the fp16 step exactly."""
    qmax = 127 if bits == 8 else 7
    unit = 2.0 ** -7 if bits == 8 else 2.0 ** -3
    rng = np.random.default_rng(8)
    d, n, r = 48, 40, 16

    def grid(units, length):
        q = rng.integers(-qmax, qmax + 1, (units, length))
        q[np.arange(units), rng.integers(0, length, units)] = qmax
        return q

    q_up, q_gate, q_down_t = grid(n, d), grid(n, d), grid(n, d)
    w_up = (q_up * unit).astype(np.float16)
    w_gate = (q_gate * unit).astype(np.float16) if act == "reglu" else None
    w_down = np.ascontiguousarray((q_down_t * 2 * unit).astype(np.float16).T)  # another scale than up's
    b = (rng.standard_normal(n) * 0.1).astype(np.float16)
    A = (rng.standard_normal((d, r)) * 0.3).astype(np.float16)
    B = (rng.standard_normal((r, n)) * 0.3).astype(np.float16)
    c = (rng.standard_normal(n) * 0.1).astype(np.float16)
    lay = _L(act, w_up, w_gate, b, w_down, A, B, c)
    qr = oracle.quantize_layer(lay, bits=bits)
    assert np.array_equal(qr.q_up, q_up) and np.all(qr.s_up == np.float32(unit))
    assert np.array_equal(qr.q_down, q_down_t) and np.all(qr.s_down == np.float32(2 * unit))
    for t in range(3):
        x = rng.standard_normal(d).astype(np.float16)
        ref = oracle.forward(lay, x)
        got = oracle.forward_q(lay, qr, x)
        assert np.array_equal(got.mask, ref.mask) and ref.mask.sum() > 0
        assert np.array_equal(got.a, ref.a) and np.array_equal(got.y, ref.y)
