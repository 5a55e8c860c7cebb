"""Pins for the FP64 CPU oracle, each against something other than the oracle.

Every oracle function is checked against at least one of: exact integer
arithmetic (numpy int64), closed forms, float64 library routines (numpy
matmul, torch cross_entropy / autograd), invariants (shift invariance,
gradient rows summing to zero, the adjoint identity of the two gradient
GEMMs) and the parameters the pages print (tests/golden/).  The cases are
chosen so that a dropped term, a wrong sign or index, or a transposed operand
fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from lm_head_fp32_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _bits(t):
    return synth.bf16_bits(t)


# --------------------------------------------------------------------------
# bf16 conversions
# --------------------------------------------------------------------------

def test_bf16_widening_known_patterns():
    assert oracle.bf16_to_f64(0x3F80) == 1.0
    assert oracle.bf16_to_f64(0xC000) == -2.0
    assert oracle.bf16_to_f64(0x0001) == 2.0 ** -133          # smallest subnormal
    assert oracle.bf16_to_f64(0x7F7F) == (2 - 2 ** -7) * 2.0 ** 127
    assert oracle.bf16_to_f64(0x8000) == 0.0 and math.copysign(1, oracle.bf16_to_f64(0x8000)) < 0


def test_bf16_rounding_matches_torch_on_float_values():
    # For values that are exact in binary32, one-step FP64 -> BF16 RNE must equal
    # torch's binary32 -> BF16 conversion (RNE).
    g = torch.Generator().manual_seed(7)
    parts = [
        torch.randn(20000, generator=g) * 3,
        torch.randn(2000, generator=g) * 1e-38,            # BF16 subnormal range
        torch.randn(2000, generator=g) * 3e38,             # near overflow
        torch.tensor([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.3895314e38, 3.4e38,
                      float("inf"), -float("inf")]),
    ]
    # exact ties: 1 + 2^-8 (tie, even -> 1.0) and 1 + 3*2^-8 (tie, even -> 1 + 2^-6)
    f = torch.cat(parts).to(torch.float32)
    ref = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_bf16(f.double().numpy())
    assert np.array_equal(got, ref)


def test_bf16_rounding_is_single_step():
    # v = 1 + 2^-8 + 2^-30: above the tie, so RNE straight from FP64 gives 1 + 2^-7.
    # Rounding to binary32 first would give exactly 1 + 2^-8 (a tie) and then 1.0.
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert oracle.bf16_to_f64(oracle.f64_to_bf16(v)) == 1.0 + 2.0 ** -7
    assert oracle.bf16_to_f64(oracle.f64_to_bf16(-v)) == -(1.0 + 2.0 ** -7)
    # the largest finite value plus half a spacing overflows (ties to even)
    big = (2 - 2 ** -7) * 2.0 ** 127 + 2.0 ** 119
    assert oracle.f64_to_bf16(big) == 0x7F80


def test_f32_rounding():
    a = np.array([1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, 0.1, -1e-50], dtype=np.float64)
    assert np.array_equal(oracle.round_f32(a), a.astype(np.float32))


# --------------------------------------------------------------------------
# a1 logits
# --------------------------------------------------------------------------

def test_logits_integer_exact_against_int64(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "p1_integer_exactness.json")))
    lo, hi = spec["int_lo"], spec["int_hi"]
    for K in spec["K"]:
        assert K * spec["max_abs_product"] < spec["exact_bound"]
        M, V = spec["activations_rows"], 96          # V cut down for CPU time
        X = synth.int_bf16((M, K), spec["seed"], lo, hi)
        W = synth.int_bf16((V, K), spec["seed"] + 1, lo, hi)
        ref = X.to(torch.int64).numpy() @ W.to(torch.int64).numpy().T
        got = oracle.logits(_bits(X), _bits(W))
        assert np.array_equal(got, ref.astype(np.float64))
        # and the FP32 round of an exact integer is that integer
        assert np.array_equal(oracle.round_f32(got), ref.astype(np.float32))


def test_logits_random_against_numpy_and_transpose_sensitivity():
    M, K, V = 7, 40, 13                 # all different: a swapped operand cannot fit
    X = synth.normal_bf16((M, K), 1.0, 11)
    W = synth.normal_bf16((V, K), 0.5, 12)
    x64, w64 = X.double().numpy(), W.double().numpy()
    got = oracle.logits(_bits(X), _bits(W))
    ref = x64 @ w64.T
    assert got.shape == (M, V)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)
    # the row subset is the same rows of the full product
    sub = oracle.logits(_bits(X), _bits(W), rows=[5, 0, 5])
    assert np.array_equal(sub, got[[5, 0, 5]])


def test_logits_brute_force_python_loops():
    M, K, V = 3, 5, 4
    X = synth.int_bf16((M, K), 3)
    W = synth.normal_bf16((V, K), 1.0, 4)
    xs, ws = X.double().tolist(), W.double().tolist()
    got = oracle.logits(_bits(X), _bits(W))
    for i in range(M):
        for v in range(V):
            s = math.fsum(xs[i][k] * ws[v][k] for k in range(K))
            assert abs(got[i, v] - s) <= 1e-15 * max(1.0, abs(s))


# --------------------------------------------------------------------------
# a2 cross-entropy forward
# --------------------------------------------------------------------------

@pytest.mark.parametrize("V", [1, 2, 3, 32768, 128256, 151936])
def test_ce_uniform_row_gives_log_V(V):
    x = np.full((2, V), 3.25, dtype=np.float32)
    t = np.array([0, V - 1], dtype=np.int64)
    st, code = oracle.ce_fwd(x, t)
    assert (code == oracle.ROW_VALID).all()
    assert (st[:, 0] == 3.25).all() and (st[:, 1] == float(V)).all() and (st[:, 2] == 3.25).all()
    np.testing.assert_allclose(st[:, 3], math.log(V), rtol=0, atol=1e-12)


def test_ce_two_value_closed_form():
    rng = np.random.default_rng(5)
    for _ in range(50):
        a, b = rng.normal(0, 6, size=2).astype(np.float32)
        x = np.array([[a, b]], dtype=np.float32)
        st, _ = oracle.ce_fwd(x, np.array([0]))
        ref = math.log1p(math.exp(float(b) - float(a))) if b < a else \
            (float(b) - float(a)) + math.log1p(math.exp(float(a) - float(b)))
        assert abs(st[0, 3] - ref) <= 1e-12 * max(1.0, ref)


def test_ce_worked_example():
    # row (1, 2, 3), target 2: loss = log(e + e^2 + e^3) - 3 = log(1 + e^-1 + e^-2)
    st, _ = oracle.ce_fwd(np.array([[1, 2, 3]], dtype=np.float32), np.array([2]))
    assert st[0, 0] == 3.0 and st[0, 2] == 3.0
    assert abs(st[0, 1] - (1 + math.exp(-1) + math.exp(-2))) < 1e-15
    assert abs(st[0, 3] - math.log(1 + math.exp(-1) + math.exp(-2))) < 1e-15


def test_ce_fwd_against_torch_float64():
    g = torch.Generator().manual_seed(3)
    for M, V in [(8, 64), (5, 7), (1, 1), (3, 333)]:
        x = (torch.randn(M, V, generator=g) * 4).to(torch.float32)
        t = torch.randint(0, V, (M,), generator=g)
        t[0] = -100
        ref = torch.nn.functional.cross_entropy(x.double(), t, reduction="none", ignore_index=-100)
        st, code = oracle.ce_fwd(x.numpy(), t.numpy())
        np.testing.assert_allclose(st[:, 3], ref.numpy(), rtol=1e-13, atol=1e-13)
        valid = t.numpy() != -100
        xd = x.double().numpy()
        np.testing.assert_array_equal(st[valid, 0], xd[valid].max(axis=1))
        np.testing.assert_allclose(st[valid, 1],
                                   np.exp(xd[valid] - xd[valid].max(axis=1, keepdims=True)).sum(1),
                                   rtol=1e-13)
        np.testing.assert_array_equal(st[valid, 2], xd[valid, t.numpy()[valid]])
        assert code[0] == oracle.ROW_IGNORED and (st[0] == 0).all()


def test_ce_shift_invariance():
    rng = np.random.default_rng(9)
    x = (rng.integers(-400, 400, size=(4, 500)) / 16.0).astype(np.float32)
    t = rng.integers(0, 500, size=4)
    s0, _ = oracle.ce_fwd(x, t)
    s1, _ = oracle.ce_fwd(x + np.float32(3.0), t)    # exact shift (multiples of 1/16)
    np.testing.assert_allclose(s1[:, 3], s0[:, 3], rtol=0, atol=1e-12)
    np.testing.assert_allclose(s1[:, 1], s0[:, 1], rtol=1e-14)
    np.testing.assert_array_equal(s1[:, 0], s0[:, 0] + 3.0)


def test_ce_ignored_and_bad_targets():
    x = np.random.default_rng(1).normal(size=(5, 9)).astype(np.float32)
    t = np.array([-100, 9, -1, 3, 1000], dtype=np.int64)
    st, code = oracle.ce_fwd(x, t, ignore_index=-100)
    assert list(code) == [oracle.ROW_IGNORED, oracle.ROW_BAD_TARGET, oracle.ROW_BAD_TARGET,
                          oracle.ROW_VALID, oracle.ROW_BAD_TARGET]
    assert (st[[0, 1, 2, 4]] == 0).all() and st[3, 3] > 0
    # a different ignore_index value
    st2, code2 = oracle.ce_fwd(x, np.array([7, 7, 3, 3, 3]), ignore_index=7)
    assert list(code2[:2]) == [oracle.ROW_IGNORED] * 2


def test_ce_saved_stats_layout(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "p2_saved_stats.json")))
    st, _ = oracle.ce_fwd(np.zeros((3, 5), np.float32), np.array([0, 1, 2]))
    assert st.shape == (3, spec["stats_cols"])
    assert spec["stats_fields"] == ["m", "d", "x_y", "loss"]


# --------------------------------------------------------------------------
# a3 cross-entropy backward
# --------------------------------------------------------------------------

def test_ce_bwd_against_torch_autograd():
    g = torch.Generator().manual_seed(4)
    M, V = 6, 50
    x = (torch.randn(M, V, generator=g) * 4).to(torch.float32)
    t = torch.randint(0, V, (M,), generator=g)
    t[2] = -100
    gl = torch.rand(M, generator=g).to(torch.float32) + 0.5
    xd = x.double().requires_grad_(True)
    loss = torch.nn.functional.cross_entropy(xd, t, reduction="none", ignore_index=-100)
    (loss * gl.double()).sum().backward()
    got = oracle.ce_bwd(x.numpy(), t.numpy(), gl.numpy())
    np.testing.assert_allclose(got, xd.grad.numpy(), rtol=1e-12, atol=1e-15)
    # scalar upstream gradient (stride 0)
    got1 = oracle.ce_bwd(x.numpy(), t.numpy(), 0.25)
    xd.grad = None
    loss = torch.nn.functional.cross_entropy(xd, t, reduction="none", ignore_index=-100)
    (loss * 0.25).sum().backward()
    np.testing.assert_allclose(got1, xd.grad.numpy(), rtol=1e-12, atol=1e-15)


def test_ce_bwd_rows_sum_to_zero_and_ignored_zero():
    rng = np.random.default_rng(2)
    x = rng.normal(0, 4, size=(4, 1000)).astype(np.float32)
    t = np.array([10, -100, 999, 5000])
    d = oracle.ce_bwd(x, t, 1.0)
    assert abs(d[0].sum()) < 1e-12 and abs(d[2].sum()) < 1e-12
    assert (d[1] == 0).all() and (d[3] == 0).all()
    assert d[0, 10] < 0 and (np.delete(d[0], 10) > 0).all()


def test_ce_bwd_two_value_closed_form_and_finite_difference():
    # V = 2, target 0: d loss / d x0 = sigmoid(x0 - x1) - 1 = -sigmoid(x1 - x0)
    for a, b in [(0.5, -1.25), (3.0, 3.0), (-20.0, 40.0)]:
        d = oracle.ce_bwd(np.array([[a, b]], np.float32), np.array([0]), 1.0)
        s = 1.0 / (1.0 + math.exp(-(b - a)))
        assert abs(d[0, 0] + s) < 1e-15 and abs(d[0, 1] - s) < 1e-15
    # central finite differences of the forward loss, on exactly representable steps
    rng = np.random.default_rng(12)
    x = (rng.integers(-64, 64, size=(1, 12)) / 8.0).astype(np.float32)
    t = np.array([4])
    d = oracle.ce_bwd(x, t, 1.0)[0]
    h = 2.0 ** -10
    for j in range(12):
        xp, xm = x.copy(), x.copy()
        xp[0, j] += h
        xm[0, j] -= h
        fd = (oracle.ce_fwd(xp, t)[0][0, 3] - oracle.ce_fwd(xm, t)[0][0, 3]) / (2 * h)
        assert abs(fd - d[j]) < 1e-6


def _decimal_row(x, y):
    """-log softmax(x)_y and softmax(x)_y - 1 of one row in 60-digit decimal
    arithmetic (exp and ln of the decimal module), as FP64."""
    import decimal
    ctx = decimal.Context(prec=60)
    xs = [decimal.Decimal(float(v)) for v in x]   # exact: every FP32 value is a short decimal
    m = max(xs)
    e = [ctx.exp(ctx.subtract(v, m)) for v in xs]
    d = decimal.Decimal(0)
    for v in e:
        d = ctx.add(d, v)
    loss = ctx.ln(ctx.divide(d, e[y]))
    grad_y = ctx.subtract(ctx.divide(e[y], d), decimal.Decimal(1))
    return float(loss), float(grad_y)


@pytest.mark.parametrize("gap", [0.0, 10.0, 25.0, 40.0, 70.0])
def test_ce_confident_rows_against_decimal_arithmetic(gap):
    """Rows whose target holds nearly all of the mass (the other columns
    `gap` below it, losses from ~1e-2 down to ~1e-28): the loss and the
    target's gradient keep full relative precision against 60-digit decimal
    arithmetic, where m + log(d) - x_y and softmax_y - 1 would cancel."""
    rng = np.random.default_rng(int(gap) + 3)
    V, y = 300, 17
    x = (rng.normal(0, 1, size=V) - gap).astype(np.float32)
    x[y] = np.float32(2.5)
    st, code = oracle.ce_fwd(x[None, :], np.array([y]))
    d = oracle.ce_bwd(x[None, :], np.array([y]), 1.0)
    loss, grad_y = _decimal_row(x, y)
    assert code[0] == oracle.ROW_VALID
    assert abs(st[0, 3] - loss) <= 1e-13 * abs(loss)
    assert abs(d[0, y] - grad_y) <= 1e-13 * abs(grad_y)
    # and the other entries still sum with it to zero
    assert abs(d[0].sum()) <= 1e-12 * abs(grad_y) + 1e-300


# --------------------------------------------------------------------------
# a4/a5 gradient GEMMs
# --------------------------------------------------------------------------

def test_dx_dw_integer_exact():
    M, K, V = 9, 24, 40
    dl = synth.int_bf16((M, V), 21)
    X = synth.int_bf16((M, K), 22)
    W = synth.int_bf16((V, K), 23)
    dl64, X64, W64 = (a.to(torch.int64).numpy() for a in (dl, X, W))
    assert np.array_equal(oracle.dx(_bits(dl), _bits(W)), (dl64 @ W64).astype(np.float64))
    assert np.array_equal(oracle.dw(_bits(dl), _bits(X)), (dl64.T @ X64).astype(np.float64))


def test_dx_dw_random_and_adjoint_identity():
    M, K, V = 11, 19, 29                # all different
    g = 31
    dl = synth.normal_bf16((M, V), 1e-3, g)
    X = synth.normal_bf16((M, K), 1.0, g + 1)
    W = synth.normal_bf16((V, K), 0.02, g + 2)
    dl64, X64, W64 = (a.double().numpy() for a in (dl, X, W))
    dX = oracle.dx(_bits(dl), _bits(W))
    dW = oracle.dw(_bits(dl), _bits(X))
    assert dX.shape == (M, K) and dW.shape == (V, K)
    np.testing.assert_allclose(dX, dl64 @ W64, rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(dW, dl64.T @ X64, rtol=1e-12, atol=1e-18)
    # <dl, X W^T> = <dX, X> = <dW, W>
    L = oracle.logits(_bits(X), _bits(W))
    a = float((dl64 * L).sum())
    assert abs(float((dX * X64).sum()) - a) <= 1e-12 * abs(a) + 1e-18
    assert abs(float((dW * W64).sum()) - a) <= 1e-12 * abs(a) + 1e-18
    # row subsets
    assert np.array_equal(oracle.dx(_bits(dl), _bits(W), rows=[3, 1]), dX[[3, 1]])
    assert np.array_equal(oracle.dw(_bits(dl), _bits(X), vrows=[28, 0]), dW[[28, 0]])


def test_end_to_end_chain_small():
    # the whole path on one tiny case, against torch float64 autograd
    M, K, V = 6, 16, 24
    X = synth.normal_bf16((M, K), 1.0, 41)
    W = synth.normal_bf16((V, K), 0.3, 42)
    t = torch.tensor([0, 5, -100, 23, 7, 7])
    L = oracle.logits(_bits(X), _bits(W))
    Lf = oracle.round_f32(L)
    st, _ = oracle.ce_fwd(Lf, t.numpy())
    g = float(np.float32(0.2))          # the upstream gradient is an FP32 value
    dl = oracle.ce_bwd(Lf, t.numpy(), g)
    dl_b = oracle.round_bf16(dl)
    dX = oracle.dx(dl_b, _bits(W))
    dW = oracle.dw(dl_b, _bits(X))
    xd = torch.from_numpy(Lf.astype(np.float64)).requires_grad_(True)
    loss = torch.nn.functional.cross_entropy(xd, t, reduction="none", ignore_index=-100)
    (loss * g).sum().backward()
    np.testing.assert_allclose(st[:, 3], loss.detach().numpy(), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dl, xd.grad.numpy(), rtol=1e-12, atol=1e-16)
    dlb64 = oracle.bf16_bits_to_f64(dl_b)
    np.testing.assert_allclose(dX, dlb64 @ W.double().numpy(), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(dW, dlb64.T @ X.double().numpy(), rtol=1e-12, atol=1e-18)


def test_synth_generators_are_deterministic_and_shaped():
    X1 = synth.int_bf16((4, 8), 1234)
    X2 = synth.int_bf16((4, 8), 1234)
    assert torch.equal(X1, X2) and X1.min() >= -8 and X1.max() <= 8
    t = synth.targets(1024, 32768, 0.02, 1234)
    assert int((t == -100).sum()) == 20
    x, orows = synth.ce_logits(200, 300, 4.0, 1234, outlier_frac=0.01)
    assert len(orows) == 2
    for r in orows.tolist():
        assert int((x[r].abs() == 80).sum()) == 16
