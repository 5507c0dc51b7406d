"""Pins for the oracle: checks against values and facts that do not come from the oracle itself.

- the worked integer matrix product printed on the quantisation primer page;
- brute force over every ternary row of length <= 6 against that pinned dense product;
- exact rational arithmetic (fractions.Fraction) for the absmean scale;
- closed forms for RMSNorm + absmax quantisation, the weight codes, the dequantisation
  and SiLU;
- the half-step rounding bounds of both quantisers;
- hand-derived byte examples of the packing layout.
No GPU is needed.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth
from conftest import read_golden


# ----------------------------------------------------------------------------------------------
# Integer product: the worked example of the primer page, section "具体例".

def _golden_matmul():
    lines = read_golden("matmul_worked_example.txt")
    mats, i = {}, 0
    while i < len(lines):
        name, r, c = lines[i].split()
        r, c = int(r), int(c)
        mats[name] = np.array([[int(v) for v in lines[i + 1 + j].split()] for j in range(r)])
        i += 1 + r
    return mats


def test_dense_matmul_worked_example():
    m = _golden_matmul()
    C = oracle.dense_matmul_i64(m["A"], m["B"])
    np.testing.assert_array_equal(C, m["C"])


def test_dense_matmul_transposes_and_operand_order():
    # (A B)^T = B^T A^T: the page's product, transposed, must come out of the transposed and
    # swapped operands.  The example is rectangular and not symmetric, so an oracle that read
    # either operand with its indices swapped, or walked the inner index of one operand
    # backwards, cannot meet both this and the pin above.
    m = _golden_matmul()
    np.testing.assert_array_equal(oracle.dense_matmul_i64(m["B"].T, m["A"].T), m["C"].T)
    assert not np.array_equal(oracle.dense_matmul_i64(m["A"], m["B"][::-1]), m["C"])
    assert not np.array_equal(oracle.dense_matmul_i64(m["A"][:, ::-1], m["B"]), m["C"])
    # the swapped product B A is the 3x3 matrix worked out by hand from the page's entries
    np.testing.assert_array_equal(oracle.dense_matmul_i64(m["B"], m["A"]),
                                  [[39, 54, 69], [49, 68, 87], [59, 82, 105]])


# ----------------------------------------------------------------------------------------------
# Ternary accumulation equals the dense product with {-1,0,1} weights.

@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 6])
def test_ternary_accumulate_bruteforce_all_rows(K):
    rows = np.array(list(itertools.product([-1, 0, 1], repeat=K)), dtype=np.int8)   # 3^K x K
    grid = np.array([-128, -127, -64, -1, 0, 1, 2, 63, 127], dtype=np.int64)
    rng = np.random.default_rng(K)
    q = rng.choice(grid, size=(11, K)).astype(np.int8)
    q[0, :] = -128
    q[1, :] = 127
    acc = oracle.ternary_accumulate(q, rows)
    dense = oracle.dense_matmul_i64(q.astype(np.int64), rows.T.astype(np.int64))
    np.testing.assert_array_equal(acc.astype(np.int64), dense)


def test_ternary_accumulate_random_rectangular():
    q = synth.int8_codes(1, "acc", 5, 4096)
    c = synth.ternary(1, "acc", 7, 4096)
    acc = oracle.ternary_accumulate(q, c)
    dense = oracle.dense_matmul_i64(q.astype(np.int64), c.T.astype(np.int64))
    np.testing.assert_array_equal(acc.astype(np.int64), dense)
    # single token, single output: a plain signed sum
    s = int(q[0][c[0] == 1].astype(np.int64).sum() - q[0][c[0] == -1].astype(np.int64).sum())
    assert acc[0, 0] == s


# ----------------------------------------------------------------------------------------------
# Packing layout.

def test_pack_hand_examples():
    for ln in read_golden("pack_layout_examples.txt"):
        codes_s, bytes_s = ln.split(";")
        codes = np.array([int(v) for v in codes_s.split()], dtype=np.int8).reshape(1, 16)
        want = np.array([int(v, 16) for v in bytes_s.split()], dtype=np.uint8).reshape(1, 4)
        got = oracle.pack_codes(codes)
        np.testing.assert_array_equal(got, want, err_msg=ln)
        np.testing.assert_array_equal(oracle.unpack_codes(got, 16), codes)


def test_pack_impulses_and_roundtrip():
    K = 64
    for k in range(K):
        for v in (-1, 1):
            c = np.zeros((1, K), dtype=np.int8)
            c[0, k] = v
            p = oracle.pack_codes(c)
            diff = np.nonzero(p[0] != 0x55)[0]
            assert list(diff) == [(k // 16) * 4 + (k % 4)]
    c = synth.ternary(3, "pack", 9, 256)
    p = oracle.pack_codes(c)
    np.testing.assert_array_equal(oracle.unpack_codes(p, 256), c)
    fields = np.stack([(p >> s) & 3 for s in (0, 2, 4, 6)])
    assert not np.any(fields == 3)


# ----------------------------------------------------------------------------------------------
# Absmean scale: exact sum against rational arithmetic.

def _fraction_sum_abs(W):
    return sum((Fraction(float(abs(v))) for v in np.asarray(W, np.float32).reshape(-1)),
               Fraction(0))


def _beta_from_fraction(W):
    s = _fraction_sum_abs(W)
    n = np.asarray(W).size
    b = np.float32(float(s) / n)       # float(Fraction) is correctly rounded
    return max(b, np.float32(1e-5))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_abs_sum_exact_matches_fractions(seed):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal(3000).astype(np.float32) * np.float32(0.02)
    extra = np.array([1e-40, -3e-42, 1.4e-45, 3.0e38, -1e30, 2.5, -0.0, 7e-39],
                     dtype=np.float32)
    W = np.concatenate([W, extra, rng.standard_normal(100).astype(np.float32) * 1e-20])
    rng.shuffle(W)
    assert oracle.abs_sum_exact(W) == float(_fraction_sum_abs(W))


def test_abs_sum_rounding_ties_and_sticky():
    two53 = np.float32(2.0 ** 53)
    # exact sum 2^53 + 1: a tie, rounds to the even neighbour 2^53
    assert oracle.abs_sum_exact(np.array([two53, 1.0], np.float32)) == 2.0 ** 53
    # 2^53 + 3: a tie between 2^53+2 (odd mantissa) and 2^53+4 (even): goes up
    assert oracle.abs_sum_exact(np.array([two53, 3.0], np.float32)) == 2.0 ** 53 + 4
    # 2^53 + 1 + 2^-20: just above the tie, rounds up
    assert oracle.abs_sum_exact(np.array([two53, 1.0, 2.0 ** -20], np.float32)) == 2.0 ** 53 + 2
    # order independence
    W = np.array([two53, 1.0, 2.0 ** -20, 3.0, 1e-30], np.float32)
    assert oracle.abs_sum_exact(W) == oracle.abs_sum_exact(W[::-1].copy())
    assert math.isnan(oracle.abs_sum_exact(np.array([1.0, np.inf], np.float32)))


def test_beta_matches_fractions_and_closed_forms():
    W = synth.weights(0, "beta", 64, 96)
    assert oracle.absmean_beta(W) == _beta_from_fraction(W)
    # W = a * S with S in {+-1}: beta = a exactly and the codes are S
    a = np.float32(0.0173)
    S = np.where(synth.ternary(5, "sign", 32, 64, p_zero=0.0) > 0, 1, -1).astype(np.float32)
    W = (a * S).astype(np.float32)
    assert oracle.absmean_beta(W) == a
    np.testing.assert_array_equal(oracle.ternary_codes(W, a), S.astype(np.int8))
    # zero matrix: beta floors at 1e-5, all codes 0
    Z = np.zeros((16, 32), np.float32)
    assert oracle.absmean_beta(Z) == np.float32(1e-5)
    assert not oracle.ternary_codes(Z, oracle.absmean_beta(Z)).any()


def test_beta_statistics_gaussian():
    sigma = 0.02
    W = synth.weights(7, "stats", 512, 1024, std=sigma)
    beta = float(oracle.absmean_beta(W))
    assert abs(beta / (sigma * math.sqrt(2 / math.pi)) - 1) < 0.01
    c = oracle.ternary_codes(W, beta)
    p0 = float((c == 0).mean())
    # |W| < beta/2 = 0.399 sigma  ->  P = erf(0.399 / sqrt 2) = 0.310
    assert abs(p0 - math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))) < 0.01


# ----------------------------------------------------------------------------------------------
# Weight codes: ties and the half-step bound.

def test_codes_ties_and_clamp():
    beta = np.float32(0.25)
    W = np.array([0.125, -0.125, 0.375, 0.3749, 0.1251, 10.0, -10.0, 0.0], np.float32)
    # W/beta = 0.5 (tie -> 0), -0.5 (-> 0), 1.5 (tie -> 2 -> clamp 1), 1.4996 -> 1,
    # 0.5004 -> 1, 40 -> 1, -40 -> -1, 0 -> 0
    np.testing.assert_array_equal(oracle.ternary_codes(W, beta), [0, 0, 1, 1, 1, 1, -1, 0])


def test_codes_half_step_bound():
    W = synth.weights(11, "half", 128, 256)
    beta = oracle.absmean_beta(W)
    c = oracle.ternary_codes(W, beta)
    assert set(np.unique(c)) <= {-1, 0, 1}
    inner = np.abs(W / beta) <= 1.5
    err = np.abs(W.astype(np.float64) - c.astype(np.float64) * float(beta))
    assert np.all(err[inner] <= float(beta) / 2 * (1 + 1e-6))
    assert np.all(c[~inner] == np.sign(W[~inner]))


# ----------------------------------------------------------------------------------------------
# RMSNorm + absmax activation codes: closed forms and bounds.

def test_actquant_constant_row():
    for v in (0.3, -2.0, 17.0):
        x = np.full((1, 256), v, np.float32)
        q, gamma, rs = oracle.rmsnorm_actquant(x)
        assert np.all(q == (127 if v > 0 else -127))
        assert rs[0] == 127 * 256 * (1 if v > 0 else -1)
        assert abs(float(gamma[0]) - 1.0) < 1e-6          # |x|/sqrt(x^2 + eps) ~ 1


def test_actquant_eps_inside_the_root():
    # x = 1e-4 constant: x / sqrt(x^2 + 1e-8) = 1/sqrt(2); eps outside the root would give ~1
    x = np.full((1, 128), 1e-4, np.float32)
    _, gamma, _ = oracle.rmsnorm_actquant(x, eps=1e-8)
    assert abs(float(gamma[0]) - 1 / math.sqrt(2)) < 1e-6


def test_actquant_one_hot_and_zero_row():
    K = 512
    x = np.zeros((2, K), np.float32)
    x[0, 37] = -3.0
    q, gamma, rs = oracle.rmsnorm_actquant(x)
    assert q[0, 37] == -127 and np.count_nonzero(q[0]) == 1
    assert abs(float(gamma[0]) - math.sqrt(K)) < 1e-3      # |x| / sqrt(x^2/K) = sqrt(K)
    assert not q[1].any() and gamma[1] == np.float32(1e-5) and rs[1] == 0


def test_actquant_scale_invariance_and_norm_weight():
    x = synth.activations(4, "inv", 8, 384, dtype=np.float32)
    q1, g1, _ = oracle.rmsnorm_actquant(x)
    q2, g2, _ = oracle.rmsnorm_actquant(x * np.float32(4.0))   # powers of two: exact scaling
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_allclose(g1, g2, rtol=1e-6)
    # a uniform norm weight of 2 doubles gamma and leaves the codes unchanged
    q3, g3, _ = oracle.rmsnorm_actquant(x, g=np.full(384, 2.0, np.float32))
    np.testing.assert_array_equal(q1, q3)
    np.testing.assert_array_equal(g3, g1 * 2)
    # a norm weight that boosts one column makes that column the row maximum
    g = np.ones(384, np.float32)
    g[5] = 1000.0
    q4, _, _ = oracle.rmsnorm_actquant(x, g=g)
    assert np.all(np.abs(q4[:, 5]) == 127)


def test_actquant_half_step_bound_and_rms():
    x = synth.activations(5, "bound", 16, 1024, dtype=np.float16,
                          outlier_frac=0.01).astype(np.float32)
    g = synth.norm_weight(5, "bound", 1024, ones=False)
    q, gamma, rs = oracle.rmsnorm_actquant(x, g=g)
    assert q.min() >= -127 and q.max() <= 127
    np.testing.assert_array_equal(rs, q.astype(np.int64).sum(axis=1))
    x64 = x.astype(np.float64)
    xhat = x64 / np.sqrt((x64 ** 2).mean(axis=1, keepdims=True) + 1e-8) * g
    np.testing.assert_allclose(gamma, np.abs(xhat).max(axis=1), rtol=2e-6)
    rec = q.astype(np.float64) * gamma[:, None].astype(np.float64) / 127.0
    assert np.all(np.abs(xhat - rec) <= gamma[:, None] / 254.0 * (1 + 1e-5))


# ----------------------------------------------------------------------------------------------
# Dequantisation and GLU.

def test_dequant_closed_form():
    acc = np.array([[127, -254, 0]], np.int32)
    y = oracle.dequant(acc, np.array([2.0], np.float32), np.float32(0.5))
    np.testing.assert_allclose(y, [[1.0, -2.0, 0.0]], rtol=1e-15, atol=0)


def test_silu_glu_closed_forms():
    z = np.array([0.0, 1.0, -1.0, 30.0, -30.0, 2.5], np.float64)
    u = np.array([3.0, 1.0, 1.0, 1.0, 1.0, -2.0], np.float64)
    h = oracle.silu_glu(np.concatenate([z, u])[None, :])[0]
    assert h[0] == 0.0                                      # silu(0) = 0
    assert abs(h[1] - 0.7310585786300049) < 1e-15           # 1 / (1 + e^-1)
    assert abs((h[1] - h[2]) - 1.0) < 1e-15                 # silu(z) - silu(-z) = z
    assert abs(h[3] - 30.0) < 1e-11 and abs(h[4]) < 1e-11
    # the first half is gated, the second is the multiplier
    assert abs(h[5] - (2.5 / (1 + math.exp(-2.5))) * -2.0) < 1e-14


# ----------------------------------------------------------------------------------------------
# Whole projection.

def test_forward_closed_form():
    # x = ones: xhat = 1, gamma = 1, q = 127; W = a*S: beta = a, c = S;
    # y[n] = 127 * sum_k S[n,k] * (1/127) * a = a * sum_k S[n,k]
    K, N = 64, 8
    a = np.float32(0.03)
    S = np.where(synth.ternary(9, "fw", N, K, p_zero=0.0) > 0, 1.0, -1.0).astype(np.float32)
    y, beta = oracle.bitlinear_forward(np.ones((2, K), np.float32), a * S)
    assert beta == a
    np.testing.assert_allclose(y, np.tile(float(a) * S.sum(axis=1).astype(np.float64), (2, 1)), rtol=1e-12)


def test_forward_is_the_composition_of_its_steps():
    x = synth.activations(2, "comp", 5, 256, dtype=np.float16)
    W = synth.weights(2, "comp", 64, 256)
    g = synth.norm_weight(2, "comp", 256, ones=False)
    y, beta = oracle.bitlinear_forward(x, W, g=g)
    q, gamma, _ = oracle.rmsnorm_actquant(x, g=g)
    Wp, beta2, c = oracle.quantize_weights(W)
    assert beta == beta2
    acc = oracle.ternary_accumulate(q, oracle.unpack_codes(Wp, 256))
    np.testing.assert_array_equal(y, oracle.dequant(acc, gamma, beta))
    h, _ = oracle.bitlinear_forward(x, W, g=g, glu=True)
    np.testing.assert_array_equal(h, oracle.silu_glu(y))


# ----------------------------------------------------------------------------------------------
# MLGRU recurrence and the swish gate norm.  The pages give the recurrence in words only (gates
# in (0, 1) weigh the previous state against the current token), so the pins are the limits
# that any such gate must reach, closed forms of the linear recurrence, and structure.
# sigmoid and SiLU on the test side come from scipy's expit, not from the oracle.

from scipy.special import expit  # noqa: E402


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_mlgru_closed_gate_takes_the_token():
    # f -> 0 (F = -40 gives f < 5e-18, and 1 - f rounds to 1): the state is the candidate
    I = _rand((7, 12), 1, 2.0)
    F = np.full((7, 12), -40.0)
    h, hT = oracle.mlgru_scan(I, F, h0=_rand(12, 2))
    np.testing.assert_allclose(h, I * expit(I), rtol=1e-15, atol=1e-16)
    np.testing.assert_array_equal(hT, h[-1])


def test_mlgru_open_gate_keeps_the_state():
    # f -> 1 (F = +40: f rounds to 1 in double): nothing of the tokens enters
    h0 = _rand(9, 3)
    h, hT = oracle.mlgru_scan(_rand((6, 9), 4, 3.0), np.full((6, 9), 40.0), h0=h0)
    np.testing.assert_array_equal(h, np.broadcast_to(h0, (6, 9)))
    np.testing.assert_array_equal(hT, h0)


def test_mlgru_constant_inputs_geometric_series():
    # constant gate f and candidate c from a zero state: h_t = c (1 - f^(t+1))
    T, H = 40, 5
    Fv = np.array([-2.0, -0.3, 0.0, 0.7, 2.5])
    Iv = np.array([1.5, -0.8, 3.0, 0.25, -2.0])
    h, _ = oracle.mlgru_scan(np.tile(Iv, (T, 1)), np.tile(Fv, (T, 1)))
    f, c = expit(Fv), Iv * expit(Iv)
    t = np.arange(1, T + 1)[:, None]
    np.testing.assert_allclose(h, c * (1.0 - f ** t), rtol=1e-12, atol=1e-15)


def test_mlgru_initial_state_enters_through_the_gate_product():
    # the recurrence is affine in h0: h(h0) - h(0) = (prod_{s<=t} f_s) * h0
    T, H = 30, 16
    I, F, h0 = _rand((T, H), 5, 1.5), _rand((T, H), 6, 1.5), _rand(H, 7, 2.0)
    h1, _ = oracle.mlgru_scan(I, F, h0)
    h2, _ = oracle.mlgru_scan(I, F, None)
    np.testing.assert_allclose(h1 - h2, np.cumprod(expit(F), axis=0) * h0, rtol=1e-9,
                               atol=1e-13)


def test_mlgru_split_sequence_carries_the_state():
    # running the first part, then the rest from its final state, equals one run
    T, H, t0 = 25, 11, 9
    I, F, h0 = _rand((T, H), 8), _rand((T, H), 9), _rand(H, 10)
    h, hT = oracle.mlgru_scan(I, F, h0)
    ha, hTa = oracle.mlgru_scan(I[:t0], F[:t0], h0)
    hb, hTb = oracle.mlgru_scan(I[t0:], F[t0:], hTa)
    np.testing.assert_array_equal(np.concatenate([ha, hb]), h)
    np.testing.assert_array_equal(hTb, hT)


def test_mlgru_channels_are_independent():
    # element-wise: permuting the channels permutes the states
    I, F, h0 = _rand((8, 10), 11), _rand((8, 10), 12), _rand(10, 13)
    perm = np.random.default_rng(14).permutation(10)
    h, _ = oracle.mlgru_scan(I, F, h0)
    hp, _ = oracle.mlgru_scan(I[:, perm], F[:, perm], h0[perm])
    np.testing.assert_array_equal(hp, h[:, perm])


def test_swish_gate_norm_unit_rms_with_linear_gate():
    # G = 40: silu(G) = 40 to double precision, so o / (40 w) is h / r, whose mean square over
    # the channels is ms / (ms + eps)
    T, H = 6, 64
    h, w = _rand((T, H), 15), 0.5 + np.abs(_rand(H, 16))
    eps = 1e-3
    o = oracle.swish_gate_norm(h, np.full((T, H), 40.0), w, eps)
    ms = (h * h).mean(axis=1)
    np.testing.assert_allclose(((o / (40.0 * w)) ** 2).mean(axis=1), ms / (ms + eps),
                               rtol=1e-12)
    # and the sign and proportions of h are kept channel by channel
    np.testing.assert_allclose(o / (40.0 * w) * np.sqrt(ms + eps)[:, None], h, rtol=1e-12)


def test_swish_gate_norm_scale_invariance_and_zero_gate():
    T, H = 4, 32
    h, G = _rand((T, H), 17), _rand((T, H), 18)
    o1 = oracle.swish_gate_norm(h, G, None, 0.0)
    o2 = oracle.swish_gate_norm(3.7 * h, G, None, 0.0)
    np.testing.assert_allclose(o2, o1, rtol=1e-13)
    assert np.all(oracle.swish_gate_norm(h, np.zeros((T, H)), None, 1e-8) == 0.0)
    # the gate is SiLU, odd around its own definition: silu(g) - silu(-g) = g
    op = oracle.swish_gate_norm(h, G, None, 1e-8)
    om = oracle.swish_gate_norm(h, -G, None, 1e-8)
    r = np.sqrt((h * h).mean(axis=1) + 1e-8)[:, None]
    np.testing.assert_allclose((op - om) * r / h, G, rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------------------------
# Straight-through backward.  The pins differentiate, by central differences in double, the
# continuous function the straight-through reading differentiates: the RMSNorm followed by the
# bilinear map of dequantised operands, with the codes held fixed.  The loss is L = sum(dy * y),
# so a difference quotient of L is one entry of the gradient; none of it calls the backward.

def _surrogate_parts(T, K, N, seed, with_g=True):
    x = _rand((T, K), seed)
    g = (0.5 + np.abs(_rand((K,), seed + 1))) if with_g else None
    W = _rand((N, K), seed + 2)
    beta = oracle.absmean_beta(W)
    c = oracle.ternary_codes(W, beta)
    q, gamma, _ = oracle.rmsnorm_actquant(x.astype(np.float32), g, 1e-8)
    dy = _rand((T, N), seed + 3)
    return x, g, q, gamma, c, beta, dy


def _norm(x, g, eps):
    r = np.sqrt((x * x).mean(axis=1, keepdims=True) + eps)
    return x / r * (1.0 if g is None else g)


def test_backward_dx_is_the_gradient_of_norm_then_projection():
    # L(x) = sum dy * (norm(x) @ (beta c)^T): the surrogate's input gradient, entry by entry
    T, K, N, eps = 3, 48, 20, 1e-3
    x, g, q, gamma, c, beta, dy = _surrogate_parts(T, K, N, 41)
    dx, _, _ = oracle.bitlinear_backward(x, q, gamma, c, beta, dy, g=g, eps=eps)
    wq = c.astype(np.float64) * float(beta)

    def L(xx):
        return float((dy * (_norm(xx, g, eps) @ wq.T)).sum())
    h = 1e-6
    for t in range(T):
        for k in (0, 7, 19, 47):
            e = np.zeros_like(x)
            e[t, k] = h
            fd = (L(x + e) - L(x - e)) / (2 * h)
            assert abs(dx[t, k] - fd) <= 1e-7 * (1 + abs(fd)), (t, k, dx[t, k], fd)


def test_backward_dw_is_the_gradient_of_the_dequantised_product():
    # L(wq) = sum dy * ((q gamma / 127) @ wq^T) with the activation codes held fixed
    T, K, N = 5, 32, 12
    x, g, q, gamma, c, beta, dy = _surrogate_parts(T, K, N, 43)
    _, dW, _ = oracle.bitlinear_backward(x, q, gamma, c, beta, dy, g=g)
    xq = q.astype(np.float64) * (gamma.astype(np.float64) / 127.0)[:, None]
    wq = c.astype(np.float64) * float(beta)

    def L(w):
        return float((dy * (xq @ w.T)).sum())
    h = 1e-3   # L is linear in w: the quotient is exact up to rounding
    for n, k in [(0, 0), (3, 31), (11, 5), (7, 16)]:
        e = np.zeros_like(wq)
        e[n, k] = h
        fd = (L(wq + e) - L(wq - e)) / (2 * h)
        assert abs(dW[n, k] - fd) <= 1e-9 * (1 + abs(fd)), (n, k, dW[n, k], fd)


def test_backward_dg_is_the_gradient_of_the_norm_weight():
    T, K, N, eps = 4, 40, 9, 1e-8
    x, g, q, gamma, c, beta, dy = _surrogate_parts(T, K, N, 47)
    _, _, dg = oracle.bitlinear_backward(x, q, gamma, c, beta, dy, g=g, eps=eps)
    wq = c.astype(np.float64) * float(beta)

    def L(gg):
        return float((dy * (_norm(x, gg, eps) @ wq.T)).sum())
    h = 1e-6
    for k in (0, 13, 39):
        e = np.zeros_like(g)
        e[k] = h
        fd = (L(g + e) - L(g - e)) / (2 * h)
        assert abs(dg[k] - fd) <= 1e-7 * (1 + abs(fd)), (k, dg[k], fd)


def test_backward_input_gradient_is_orthogonal_to_the_input_without_eps():
    # with eps = 0 the norm is invariant to scaling x, so sum_k x_tk dx_tk = 0 for every token
    T, K, N = 6, 64, 24
    x, g, q, gamma, c, beta, dy = _surrogate_parts(T, K, N, 53)
    dx, _, _ = oracle.bitlinear_backward(x, q, gamma, c, beta, dy, g=g, eps=0.0)
    dots = (x * dx).sum(axis=1)
    assert np.all(np.abs(dots) <= 1e-12 * np.abs(x).sum(axis=1) * np.abs(dx).sum(axis=1))
    # and with eps > 0 it is not (the pin above would catch a dropped eps)
    dx2, _, _ = oracle.bitlinear_backward(x, q, gamma, c, beta, dy, g=g, eps=1.0)
    assert np.abs((x * dx2).sum(axis=1)).max() > 1e-3


def test_backward_identity_norm_and_unit_codes():
    # K = 1, g = 1, eps -> 0: xhat = sign(x), so dx = 0; dW_n = dy_n * q * gamma / 127
    x = np.array([[2.5], [-0.75]])
    q = np.array([[127], [-127]], dtype=np.int8)
    gamma = np.array([1.0, 1.0], dtype=np.float32)
    c = np.array([[1], [-1], [0]], dtype=np.int8)
    dy = np.array([[1.0, 2.0, 3.0], [-1.0, 0.5, 4.0]])
    dx, dW, dg = oracle.bitlinear_backward(x, q, gamma, c, 0.5, dy, eps=0.0)
    assert np.all(np.abs(dx) < 1e-15)
    np.testing.assert_allclose(dW[:, 0], [1.0 * 1 + (-1.0) * -1, 2.0 - 0.5, 3.0 - 4.0], rtol=1e-15)
    # dxh_t = sum_n dy_tn c_n beta = (dy_t0 - dy_t1) * 0.5; dg = sum_t dxh_t * x_t / |x_t|
    np.testing.assert_allclose(dg, [(1.0 - 2.0) * 0.5 * 1 + (-1.0 - 0.5) * 0.5 * -1], rtol=1e-15)
