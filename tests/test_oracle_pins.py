"""Pins of the CPU oracle against facts fixed outside the oracle itself:
hand-derived worked examples (tests/golden), closed forms, invariants, brute
force over the unpacked ternary matrix, and a planted-mistake check.

Readings pinned here (stated in oracle/bitnet_oracle.h):
R1 activation quantiser, R2 packed layout, R3 codes and tail, R4 linear.
"""
import os

import numpy as np
import pytest

import oracle
from ternary_weight_i2_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------- quantiser R1

def _read_quant_golden():
    cases, cur = [], {}
    with open(os.path.join(GOLDEN, "quant_small.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            cur[key] = val.split()
            if key == "s":
                cases.append(cur)
                cur = {}
    return cases


def test_quant_golden_examples():
    cases = _read_quant_golden()
    assert len(cases) == 4
    for c in cases:
        x = np.array([float(v) for v in c["x"]], np.float32)[None, :]
        want = np.array([int(v) for v in c["q"]], np.int8)
        num, den = c["s"][0].split("/")
        s_want = np.float32(np.float32(float(num)) / np.float32(float(den)))
        q, s, st = oracle.quant_act(x)
        assert st == oracle.OK
        np.testing.assert_array_equal(q[0, : x.shape[1]], want)
        assert s[0] == s_want


def test_quant_invariants_random():
    rng = np.random.default_rng(1)
    for k in (1, 7, 128, 300, 1536):
        x = synth.normal_outliers(rng, 9, k)
        x[3] *= np.float32(1e-6)
        x[4] *= np.float32(1e6)
        q, s, st = oracle.quant_act(x)
        assert st == oracle.OK
        kp = oracle.kpad(k)
        assert q.shape == (9, kp)
        assert not q[:, k:].any()                         # zero padding
        qv = q[:, :k].astype(np.int64)
        assert np.abs(qv).max() <= 127 and qv.min() >= -127  # never -128
        amax = np.abs(x).max(axis=1)
        for r in range(9):
            i = int(np.argmax(np.abs(x[r])))
            assert abs(int(qv[r, i])) == 127                 # absmax maps to 127
            sgn = np.sign(qv[r])
            assert np.all((sgn == 0) | (sgn == np.sign(x[r])))
            assert s[r] == np.float32(amax[r] / np.float32(127))
            err = np.abs(qv[r] * np.float64(s[r]) - x[r].astype(np.float64))
            assert err.max() <= 0.5 * float(s[r]) * (1 + 1e-4)


def test_quant_special_rows():
    x = np.zeros((6, 200), np.float32)
    x[0] = 3.0                     # constant positive
    x[1] = -2.0                    # constant negative
    # row 2 stays zero
    x[3] = 1.0
    x[3, 17] = np.nan              # non-finite row
    x[4] = 1.0
    x[4, 5] = np.inf               # non-finite row
    x[5, :4] = [1e-38, -5e-39, 0.0, 2e-39]   # 127/amax overflows to inf
    q, s, st = oracle.quant_act(x)
    assert st == oracle.NONFINITE
    assert (q[0, :200] == 127).all() and (q[1, :200] == -127).all()
    assert not q[2].any() and s[2] == 0
    assert not q[3].any() and s[3] == 0
    assert not q[4].any() and s[4] == 0
    assert list(q[5, :5]) == [127, -127, 0, 127, 0]


def test_quant_ties_round_half_even_constructed():
    # amax = 127 makes inv exactly 1, so x*inv = x: every half rounds to even
    halves = np.arange(-126.5, 127.0, 1.0, dtype=np.float32)
    x = np.concatenate([halves, [np.float32(127.0)]])[None, :]
    q, _, _ = oracle.quant_act(x)
    # half-even: floor if floor is even, else ceil
    fl = np.floor(halves).astype(np.int64)
    exp = np.where(fl % 2 == 0, fl, fl + 1)
    np.testing.assert_array_equal(q[0, : halves.size].astype(np.int64), exp)


# ------------------------------------------------------- pack layout R2, R3

def _read_pack_golden():
    spec = {}
    with open(os.path.join(GOLDEN, "pack_k130.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, val = line.split(":", 1)
                spec[key] = val.split()
    return spec


def test_pack_golden_bytes():
    spec = _read_pack_golden()
    k = int(spec["K"][0])
    w = np.zeros((1, k), np.int8)
    for item in spec["w"]:
        pos, val = item.split(":")
        w[0, int(pos)] = int(val)
    want = None
    for item in spec["bytes"]:
        pos, val = item.split(":")
        if pos == "default":
            want = np.full(32 * ((k + 127) // 128), int(val, 16), np.uint8)
    for item in spec["bytes"]:
        pos, val = item.split(":")
        if pos != "default":
            want[int(pos)] = int(val, 16)
    p, st = oracle.pack(w)
    assert st == oracle.OK
    np.testing.assert_array_equal(p[0], want)


@pytest.mark.parametrize("k", list(range(1, 301, 1)) + [1535, 8960, 9024])
def test_pack_unpack_roundtrip_and_tail(k):
    rng = np.random.default_rng(k)
    w = synth.ternary(rng, 3, k, (0.3, 0.4, 0.3))
    p, st = oracle.pack(w)
    assert st == oracle.OK
    assert p.shape == (3, 32 * ((k + 127) // 128))
    np.testing.assert_array_equal(oracle.unpack(p, k), w)
    # every 2-bit field of a position k' >= K holds code 01 (weight 0)
    kp = oracle.kpad(k)
    for kk in range(k, kp):
        byte = 32 * (kk // 128) + kk % 32
        sh = 2 * ((kk % 128) // 32)
        assert ((p[:, byte] >> sh) & 3 == 1).all()
    # no field anywhere holds the unused code 3
    for sh in (0, 2, 4, 6):
        assert not (((p >> sh) & 3) == 3).any()


def test_pack_rejects_non_ternary():
    w = np.zeros((2, 10), np.int8)
    w[1, 3] = 2
    w[0, 9] = -128
    p, st = oracle.pack(w)
    assert st == oracle.NOT_TERNARY
    np.testing.assert_array_equal(oracle.unpack(p, 10), np.zeros((2, 10), np.int8))


def _onehot_check(unpacker, k, k0s):
    """For each k0, a row holding a single +1 at k0 must decode to that row."""
    bad = 0
    for k0 in k0s:
        w = np.zeros((1, k), np.int8)
        w[0, k0] = 1
        p, _ = oracle.pack(w)
        bad += int(not np.array_equal(unpacker(p, k), w))
    return bad


def test_onehot_gather_layout():
    k = 300
    rng = np.random.default_rng(5)
    x = synth.normal(rng, 3, k)
    q, s, _ = oracle.quant_act(x)
    for k0 in range(k):
        w = np.zeros((1, k), np.int8)
        w[0, k0] = 1
        p, _ = oracle.pack(w)
        acc, st = oracle.ternary_matmul(q, p, k)
        assert st == oracle.OK
        np.testing.assert_array_equal(acc[:, 0], q[:, k0].astype(np.int32))


def test_misread64_is_caught():
    """The planted 64-element misreading keeps every 128-span's multiset of
    weights (so sums and non-zero counts agree) but fails the one-hot check."""
    k = kf = 8960
    rng = np.random.default_rng(11)
    w = synth.ternary(rng, 4, k)
    p, _ = oracle.pack(w)
    wm = oracle.unpack_misread64(p, k)
    for j in range(kf // 128):
        a = np.sort(w[:, 128 * j:128 * (j + 1)], axis=1)
        b = np.sort(wm[:, 128 * j:128 * (j + 1)], axis=1)
        np.testing.assert_array_equal(a, b)
    assert not np.array_equal(wm, w[:, :kf])
    assert _onehot_check(oracle.unpack_misread64, 256, range(256)) > 0
    assert _onehot_check(oracle.unpack, 256, range(256)) == 0


# ------------------------------------------------------------- linear R4

@pytest.mark.parametrize("m,n,k", [(1, 1, 1), (2, 3, 5), (5, 9, 127), (3, 9, 128),
                                   (4, 7, 129), (5, 2, 300), (1, 9, 256), (2, 4, 1536)])
def test_linear_matches_bruteforce(m, n, k):
    rng = np.random.default_rng(100 * m + n + k)
    w = synth.ternary(rng, n, k)
    x = synth.normal_outliers(rng, m, k)
    s_w = synth.weight_scale(rng)
    p, _ = oracle.pack(w)
    acc, y64, y32, st = oracle.linear(x, p, n, k, s_w)
    assert st == oracle.OK
    q, s_act, _ = oracle.quant_act(x)
    ref = q[:, :k].astype(np.float64) @ w.astype(np.float64).T   # exact integers
    np.testing.assert_array_equal(acc.astype(np.float64), ref)
    # y against the double-precision sum of dequantised products
    yd = (q[:, :k].astype(np.float64) * np.float64(1) * s_act[:, None].astype(np.float64)) @ \
         (w.astype(np.float64) * np.float64(s_w)).T
    np.testing.assert_allclose(y64, yd, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(y32, y64, rtol=1e-6, atol=0)


def test_linear_special_rows_closed_forms():
    k, n, m = 1000, 4, 3
    rng = np.random.default_rng(2)
    x = synth.normal(rng, m, k)
    w = np.zeros((n, k), np.int8)
    w[1] = 1
    w[2] = -1
    w[3] = synth.ternary(rng, 1, k)[0]
    p, _ = oracle.pack(w)
    acc, y64, _, _ = oracle.linear(x, p, n, k, 0.05)
    q, _, _ = oracle.quant_act(x)
    sq = q[:, :k].astype(np.int64).sum(axis=1)
    assert (acc[:, 0] == 0).all() and (y64[:, 0] == 0).all()
    np.testing.assert_array_equal(acc[:, 1], sq)
    np.testing.assert_array_equal(acc[:, 2], -sq)
    # zero weights contribute nothing: zeroing weight (3, i) moves acc by -w*q
    for i in rng.choice(k, 20, replace=False):
        w2 = w.copy()
        w2[3, i] = 0
        p2, _ = oracle.pack(w2)
        acc2, _, _, _ = oracle.linear(x, p2, n, k, 0.05)
        np.testing.assert_array_equal(acc2[:, 3] - acc[:, 3],
                                      -int(w[3, i]) * q[:, i].astype(np.int32))
        np.testing.assert_array_equal(acc2[:, :3], acc[:, :3])


def test_linear_saturation_max_k():
    k = 9024
    x = np.full((2, k), 3.25, np.float32)
    x[1] = -3.25
    w = np.ones((2, k), np.int8)
    w[1] = -1
    p, _ = oracle.pack(w)
    acc, _, _, st = oracle.linear(x, p, 2, k, 0.1)
    assert st == oracle.OK
    assert acc[0, 0] == 127 * 9024 == 1146048
    assert acc[0, 1] == -1146048 and acc[1, 0] == -1146048 and acc[1, 1] == 1146048


@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 7, 8, 13, 64])
def test_linear_rows_independent_of_m(m):
    """Remainder rows (M = 4, 5, ... as in the blog post's third bug) give the
    same result as computing each token alone."""
    k, n = 257, 33
    rng = np.random.default_rng(m)
    w = synth.ternary(rng, n, k)
    x = synth.normal_outliers(rng, m, k)
    p, _ = oracle.pack(w)
    acc, y64, _, _ = oracle.linear(x, p, n, k, 0.02)
    for r in range(m):
        a1, y1, _, _ = oracle.linear(x[r:r + 1], p, n, k, 0.02)
        np.testing.assert_array_equal(acc[r], a1[0])
        np.testing.assert_array_equal(y64[r], y1[0])


def test_linear_rows_sampled_equals_full():
    k, n, m = 8960, 40, 2
    rng = np.random.default_rng(9)
    w = synth.ternary(rng, n, k)
    x = synth.normal_outliers(rng, m, k)
    p, _ = oracle.pack(w)
    acc, y64, _, _ = oracle.linear(x, p, n, k, 0.07)
    idx = np.array([0, 5, 39, 17])
    a2, y2, _ = oracle.linear_rows(x, p, n, k, 0.07, idx)
    np.testing.assert_array_equal(a2, acc[:, idx])
    np.testing.assert_array_equal(y2, y64[:, idx])


# ------------------------------------------------------ absmean quantiser (R5)

def _read_absmean_golden():
    cases, cur = [], {}
    for line in open(os.path.join(GOLDEN, "absmean_small.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val = line.split(":", 1)
        rows = [[float(v) for v in r.split()] for r in val.split("|")] if key != "s" else float(val)
        cur[key] = rows
        if key == "s":
            cases.append(cur)
            cur = {}
    return cases


def test_absmean_golden_examples():
    cases = _read_absmean_golden()
    assert len(cases) == 4
    for c in cases:
        W = np.array(c["rows"], np.float32)
        w, s, st = oracle.absmean_ternary(W)
        assert st == oracle.OK
        np.testing.assert_array_equal(w, np.array(c["w"], np.int8))
        assert s == np.float32(c["s"])


@pytest.mark.parametrize("p_nonzero", [1.0, 0.75, 0.5, 0.25])
def test_absmean_closed_form_scaled_ternary(p_nonzero):
    """W = c * T with T ternary and a known count of nonzeros: mean|W| = c * p
    exactly, W / scale = T / p has magnitude >= 1 wherever T != 0, so the
    codes give back T."""
    rng = np.random.default_rng(int(p_nonzero * 100))
    n, k = 16, 256
    nz = int(p_nonzero * n * k)
    T = np.zeros(n * k, np.int8)
    T[:nz] = rng.choice([-1, 1], nz)
    rng.shuffle(T)
    T = T.reshape(n, k)
    c = np.float32(0.03125)
    w, s, st = oracle.absmean_ternary(c * T.astype(np.float32))
    assert st == oracle.OK
    assert s == np.float32(c * nz / (n * k))
    np.testing.assert_array_equal(w, T)


def test_absmean_power_of_two_equivariance_and_invariants():
    """Scaling W by 2^e scales the mean exactly and leaves every quotient, so
    every code, unchanged; on random W the codes are ternary, carry W's sign,
    are 0 exactly where |W| / scale <= 1/2 and 1 in magnitude elsewhere."""
    rng = np.random.default_rng(77)
    W = (rng.standard_normal((48, 520)) * 0.02).astype(np.float32)
    w, s, st = oracle.absmean_ternary(W)
    assert st == oracle.OK and s > 0
    for e in (-3, 5):
        w2, s2, _ = oracle.absmean_ternary(W * np.float32(2.0 ** e))
        assert s2 == np.float32(s * 2.0 ** e)
        np.testing.assert_array_equal(w2, w)
    assert set(np.unique(w)) <= {-1, 0, 1}
    assert (np.sign(w[w != 0]) == np.sign(W[w != 0])).all()
    ratio = np.abs(W / s)          # the fp32 quotient the codes are decided on
    assert (w[ratio < 0.5] == 0).all() and (np.abs(w[ratio > 0.5]) == 1).all()


def test_absmean_nonfinite_tensor():
    W = np.ones((3, 7), np.float32)
    for bad in (np.nan, np.inf, -np.inf):
        W2 = W.copy()
        W2[1, 4] = bad
        w, s, st = oracle.absmean_ternary(W2)
        assert st == oracle.NONFINITE and s == 0.0 and not w.any()


def test_ternary_round_at_given_scale_hand_table():
    """The second pass alone, at scale 2, against codes worked by hand from
    clamp(rint(W / 2), -1, 1): quotients exactly +-0.5 round to 0 (half to
    even), just above 0.5 to 1, +-1.5 to +-2 and clamp; scale 0 gives 0."""
    W = np.array([[-3.1, -3.0, -1.0, -0.99, 0.0, 1.0, 1.0000001, 3.0, 100.0]], np.float32)
    want = np.array([[-1, -1, 0, 0, 0, 0, 1, 1, 1]], np.int8)
    np.testing.assert_array_equal(oracle.ternary_round(W, 2.0), want)
    assert not oracle.ternary_round(W, 0.0).any()


def test_absmean_codes_are_the_second_pass_at_its_own_scale():
    rng = np.random.default_rng(78)
    W = (rng.standard_normal((9, 301)) * 0.1).astype(np.float32)
    w, s, _ = oracle.absmean_ternary(W)
    np.testing.assert_array_equal(oracle.ternary_round(W, s), w)


# ----------------------------------------------------- fused epilogue (R6)

def _read_epilogue_golden():
    cases, cur = [], {}
    for line in open(os.path.join(GOLDEN, "epilogue_small.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val = (t.strip() for t in line.split(":", 1))
        if val == "none":
            cur[key] = None
        elif key in ("s_w", "relu"):
            cur[key] = float(val)
        else:
            cur[key] = np.array([[float(v) for v in r.split()] for r in val.split("|")], np.float32)
        if key == "out":
            cases.append(cur)
            cur = {}
    return cases


def test_epilogue_golden_examples():
    cases = _read_epilogue_golden()
    assert len(cases) == 5
    for c in cases:
        w = c["w"].astype(np.int8)
        n, k = w.shape
        packed, _ = oracle.pack(w)
        acc, y64, y32, st = oracle.linear(c["x"], packed, n, k, c["s_w"])
        assert st == oracle.OK
        bias = None if c["bias"] is None else c["bias"][0]
        gamma = None if c["gamma"] is None else c["gamma"][0]
        o32, o64 = oracle.epilogue(y32, y64, bias=bias, gamma=gamma, residual=c["residual"], relu=bool(c["relu"]))
        np.testing.assert_array_equal(o32, c["out"])
        np.testing.assert_array_equal(o64, c["out"].astype(np.float64))


def test_epilogue_step_order():
    """Bias before ReLU, layer scale after ReLU, layer scale not applied to
    the residual -- each single-element case tells one wrong order apart."""
    y = np.array([[-1.0]], np.float32)
    one = np.array([1.0], np.float32)
    # bias then relu: relu(-1 + 2) = 1  (relu first would give 0 + 2 = 2)
    assert oracle.epilogue(y, bias=2 * one, relu=True)[0][0, 0] == 1.0
    # relu then gamma: relu(-1) * -1 = 0  (gamma first would give relu(1) = 1)
    assert oracle.epilogue(y, gamma=-one, relu=True)[0][0, 0] == 0.0
    # residual + gamma * h: 1 + 2 * 1 = 3  (gamma * (r + h) would give 4)
    assert oracle.epilogue(-y, gamma=2 * one, residual=np.array([[1.0]], np.float32))[0][0, 0] == 3.0


def test_epilogue_identities_and_exact_cases():
    rng = np.random.default_rng(61)
    m, n = 5, 77
    y = (rng.standard_normal((m, n)) * 3).astype(np.float32)
    # no operand: bit-for-bit unchanged
    np.testing.assert_array_equal(oracle.epilogue(y)[0].view(np.uint32), y.view(np.uint32))
    # residual = -y, nothing else: every x + (-x) is exactly +0
    out = oracle.epilogue(y, residual=-y)[0]
    assert (out.view(np.uint32) == 0).all()
    # power-of-two layer scale scales exactly (no residual)
    b = rng.standard_normal(n).astype(np.float32)
    base = oracle.epilogue(y, bias=b, relu=True)[0]
    four = oracle.epilogue(y, bias=b, relu=True, gamma=np.full(n, 4.0, np.float32))[0]
    np.testing.assert_array_equal(four, base * np.float32(4))
    # relu: non-negative, +0 (not -0) wherever y + b <= 0, y + b elsewhere
    yb = y + b
    assert (base >= 0).all() and (base.view(np.uint32)[yb <= 0] == 0).all()
    np.testing.assert_array_equal(base[yb > 0], yb[yb > 0])
    negzero = np.full((1, 3), -0.0, np.float32)
    assert (oracle.epilogue(negzero, relu=True)[0].view(np.uint32) == 0).all()


def test_epilogue_fp32_form_within_its_rounding_bound_of_fp64_form():
    """Four rounded fp32 steps: |out32 - out64| <= 4 u (|r| + |g| (|y| + |b|))
    with u = 2^-24, for inputs exactly representable in both forms."""
    rng = np.random.default_rng(62)
    m, n = 7, 301
    y = (rng.standard_normal((m, n)) * 10).astype(np.float32)
    b = rng.standard_normal(n).astype(np.float32)
    g = rng.uniform(0.5, 2.0, n).astype(np.float32)
    r = (rng.standard_normal((m, n)) * 10).astype(np.float32)
    o32, o64 = oracle.epilogue(y, y.astype(np.float64), bias=b, gamma=g, residual=r, relu=True)
    bound = 4 * 2.0 ** -24 * (np.abs(r) + np.abs(g) * (np.abs(y) + np.abs(b))) + 1e-300
    assert (np.abs(o32.astype(np.float64) - o64) <= bound).all()
    # and a single dropped term in either form would break it by far
    assert np.abs(o64 - oracle.epilogue(None, y.astype(np.float64), bias=b, gamma=g, relu=True)[1]).min() > 0


# --------------------------------------------------------- I8_S linear (R7)

def _maddubs_dot(q_row, w_row):
    """The pages' I8_S multiply-add pipeline for one dot product, block by
    block (Q_K = 32): sign trick (unsigned |w| times sign(w)*x), adjacent
    products summed into int16 with saturation, int16 pairs into int32, then
    a horizontal sum.  Written from the pipeline's description, independent
    of the oracle's plain loop."""
    k = len(q_row)
    total = 0
    for b0 in range(0, k, 32):
        wb = w_row[b0:b0 + 32].astype(np.int64)
        xb = q_row[b0:b0 + 32].astype(np.int64)
        u = np.abs(wb)                                   # u8 operand
        s = np.sign(wb) * xb                             # s8 operand
        assert (u <= 255).all() and (s >= -128).all() and (s <= 127).all()
        prod = u * s
        if len(prod) % 2:
            prod = np.append(prod, 0)
        pairs = np.clip(prod[0::2] + prod[1::2], -32768, 32767)   # maddubs: saturating int16
        total += int(pairs.sum())                        # madd with ones + hsum in int32
    return total


def test_i8_matmul_brute_force_and_sign_trick_pipeline():
    rng = np.random.default_rng(71)
    for m, n, k in [(1, 1, 1), (3, 5, 31), (2, 7, 32), (4, 3, 33), (2, 9, 100), (5, 4, 1536)]:
        x = synth.normal_outliers(rng, m, k)
        q, s_act, _ = oracle.quant_act(x)
        w = rng.integers(-127, 128, size=(n, k), dtype=np.int64).astype(np.int8)
        acc, st = oracle.i8_matmul(q, oracle.i8_layout(w), k)
        assert st == oracle.OK
        want = q[:, :k].astype(np.int64) @ w.astype(np.int64).T
        np.testing.assert_array_equal(acc, want)
        for r in range(m):
            for c in range(n):
                assert _maddubs_dot(q[r, :k], w[c]) == acc[r, c]


def test_i8_matmul_closed_forms_pads_and_overflow():
    k = 1000
    q = np.zeros((2, oracle.kpad(k)), np.int8)
    q[0, :k] = 127
    q[1, :k] = np.where(np.arange(k) % 2 == 0, 127, -127)
    w = np.full((3, k), 127, np.int8)
    w[1] = -127
    w[2] = np.where(np.arange(k) % 2 == 0, 1, -1)
    rows = oracle.i8_layout(w)
    acc, _ = oracle.i8_matmul(q, rows, k)
    np.testing.assert_array_equal(acc, [[127 * 127 * k, -127 * 127 * k, 0],
                                        [0, 0, 127 * k]])
    # pads (k..1023 of each row) are never read
    rows2 = rows.copy()
    rows2[:, k:] = 99
    np.testing.assert_array_equal(oracle.i8_matmul(q, rows2, k)[0], acc)
    assert oracle.i8_row_bytes(k) == 1024 and oracle.i8_row_bytes(1) == 32 and oracle.i8_row_bytes(32) == 32
    # past 2^31 / 127^2 = 133,143 elements a saturated sum leaves int32
    kb = 133200
    qb = np.full((1, oracle.kpad(kb)), 127, np.int8)
    wb = np.full((1, kb), 127, np.int8)
    _, st = oracle.i8_matmul(qb, oracle.i8_layout(wb), kb)
    assert st & oracle.OVERFLOW


def test_linear_i8_fp32_form_rounds_large_sums_to_even():
    """x = 127 everywhere gives q = 127 and s_act = 1; with w = 127 and
    s_w = 1, y32 is (float)acc.  K = 1041: acc = 16129 * 1041 = 16,790,289,
    odd and above 2^24, halfway between 16,790,288 and 16,790,290: rounds to
    the even 16,790,288."""
    k = 1041
    x = np.full((1, k), 127.0, np.float32)
    w = np.full((1, k), 127, np.int8)
    acc, y64, y32, st = oracle.linear_i8(x, oracle.i8_layout(w), k, 1.0)
    assert st == oracle.OK
    assert acc[0, 0] == 16790289
    assert y64[0, 0] == 16790289.0
    assert y32[0, 0] == np.float32(16790288.0)


# ---------------------------------------------------- decode chain (R8)

def _identity_like(n, k, sign=1):
    w = np.zeros((n, k), np.int8)
    d = min(n, k)
    w[np.arange(d), np.arange(d)] = sign
    return w


def _chain_layers(shapes_weights, s_w=1.0):
    return [[(oracle.pack(w)[0], w.shape[0], w.shape[1], s_w) for w in layer] for layer in shapes_weights]


def test_chain_carries_codes_only_along_the_true_dependences():
    """Identity weights on the chain's true path (q -> o -> up -> down) and
    zero weights elsewhere (k, v, gate): the codes of the first input come
    back out of every layer's down unchanged, times its scale.  A chain wired
    through k, v or gate would give zeros."""
    rng = np.random.default_rng(81)
    x0 = synth.normal_outliers(rng, 2, 1536)
    layer = [_identity_like(1536, 1536), np.zeros((256, 1536), np.int8), np.zeros((256, 1536), np.int8),
             _identity_like(1536, 1536), np.zeros((8960, 1536), np.int8), _identity_like(8960, 1536),
             _identity_like(1536, 8960)]
    outs, st = oracle.linear_chain(x0, _chain_layers([layer, layer, layer]))
    assert st == oracle.OK
    q0, s0, _ = oracle.quant_act(x0)
    for ys in outs:
        qd, sd, _ = oracle.quant_act(ys[6])
        np.testing.assert_array_equal(qd[:, :1536], q0[:, :1536])
        assert not ys[1].any() and not ys[2].any() and not ys[4].any()
        assert (np.abs(ys[6]) > 0).any()
        # down's output is the first codes dequantised: within a few fp32
        # roundings of q0 * s0 (s_w = 1 everywhere)
        np.testing.assert_allclose(ys[6], q0[:, :1536] * s0[:, None], rtol=1e-5, atol=0)


def test_chain_negating_the_first_linear_negates_everything_downstream():
    """The quantiser is odd (rint is symmetric) and every later linear is
    linear with the same scales, so flipping q's weights flips every later
    output bit for bit in magnitude and exactly in sign."""
    rng = np.random.default_rng(82)
    x0 = synth.normal_outliers(rng, 1, 1536)
    rest = [synth.ternary(rng, n, k) for _, n, k in synth.LAYER_SHAPES[1:]]
    wq = synth.ternary(rng, 1536, 1536)
    scales = [synth.weight_scale(rng) for _ in range(7)]

    def run(wq_):
        ws = [wq_] + rest
        layer = [(oracle.pack(w)[0], w.shape[0], w.shape[1], s) for w, s in zip(ws, scales)]
        return oracle.linear_chain(x0, [layer])[0][0]

    a, b = run(wq), run(-wq)
    for i in (0, 3, 4, 5, 6):      # q and everything that depends on it
        np.testing.assert_array_equal(b[i], -a[i])
    for i in (1, 2):               # k and v read the layer input only
        np.testing.assert_array_equal(b[i], a[i])
