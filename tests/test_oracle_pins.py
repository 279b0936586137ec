"""Pins for the fp64 oracle, checked against things other than itself.

The pages print no worked example for the MLP block, so the oracle is pinned
by: textbook values of the normal distribution (tests/golden), closed forms
and a hand-worked example, brute-force dot products on tiny shapes, central
finite differences of a scalar loss (pins every gradient and GeLU′ without
using their formulas), the pages' two partition identities (page "Megatron",
section "张量并行 / 数学原理": column-shard concatenation equals X·A, the sum of
row-shard products equals Y·B), special cases, and an independent float64
torch computation with autograd. Mutation tests at the end plant plausible
mistakes in throw-away builds of the oracle and check that the pins catch
them.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import bruteforce

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "normal_distribution_table.txt")


def _table():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(float(v) for v in line.split()))
    return rows


def _rand_problem(rng, T, h, F, scale_w=0.7, scale_b=0.5):
    return dict(X=rng.standard_normal((T, h)), A=rng.standard_normal((h, F)) * scale_w,
                a=rng.standard_normal(F) * scale_b, B=rng.standard_normal((F, h)) * scale_w,
                b=rng.standard_normal(h) * scale_b, dZ=rng.standard_normal((T, h)))


def _all_outputs(orc, P, act=0):
    H, Y, Z = orc.forward(P["X"], P["A"], P["a"], P["B"], P["b"], act)
    g = orc.backward(P["X"], P["A"], P["B"], H, Y, P["dZ"], act)
    return dict(H=H, Y=Y, Z=Z, **g)


def _max_rel(x, y):
    x, y = np.asarray(x, dtype=np.float64), np.asarray(y, dtype=np.float64)
    return float(np.max(np.abs(x - y)) / max(np.max(np.abs(y)), 1e-300))


# ---------------------------------------------------------------- scalar pins

def check_normal_table(orc):
    for x, Phi, phi in _table():
        assert abs(orc.normal_cdf(x) - Phi) < 2e-15, x
        assert abs(orc.normal_pdf(x) - phi) < 2e-15, x
        assert abs(orc.normal_cdf(-x) - (1.0 - Phi)) < 2e-15, x
        # GeLU(x) = x·Φ(x), GeLU′(x) = Φ(x) + x·φ(x), from the table alone
        assert abs(orc.gelu(x) - x * Phi) < 1e-14, x
        assert abs(orc.gelu(-x) - (-x) * (1.0 - Phi)) < 1e-14, x
        assert abs(orc.gelu_grad(x) - (Phi + x * phi)) < 1e-14, x
        assert abs(orc.gelu_grad(-x) - ((1.0 - Phi) - x * phi)) < 1e-14, x


def test_normal_table():
    check_normal_table(oracle.default())


def test_gelu_closed_forms():
    assert oracle.gelu(0.0) == 0.0
    assert oracle.gelu_grad(0.0) == 0.5
    # far tails: Φ(±10) is 1 or 0 to well below double precision
    assert oracle.gelu(10.0) == 10.0 and abs(oracle.gelu(-10.0)) < 1e-20
    assert oracle.gelu_grad(10.0) == 1.0 and abs(oracle.gelu_grad(-10.0)) < 1e-20
    # GeLU(x) − GeLU(−x) = x  (since Φ(x) + Φ(−x) = 1)
    for x in np.linspace(-4, 4, 33):
        assert abs(oracle.gelu(x) - oracle.gelu(-x) - x) < 1e-15


def check_gelu_grad_fd(orc):
    # GeLU′ against a central difference of GeLU itself (error O(ε²) ≈ 1e-10)
    eps = 1e-5
    for x in np.linspace(-5, 5, 41):
        fd = (orc.gelu(x + eps) - orc.gelu(x - eps)) / (2 * eps)
        assert abs(fd - orc.gelu_grad(x)) < 1e-9, x


def test_gelu_grad_matches_finite_difference():
    check_gelu_grad_fd(oracle.default())


def test_gelu_tanh_closed_forms():
    """The tanh form ½x(1 + tanh(√(2/π)(x + 0.044715x³))): value and slope at
    0, the identity g(x) − g(−x) = x (tanh is odd), the tails, its derivative
    against a central difference, and its distance from the exact GeLU (which
    the normal table pins) staying below 5e-4 everywhere."""
    o = oracle.default()
    assert o.gelu_tanh(0.0) == 0.0 and o.gelu_tanh_grad(0.0) == 0.5
    assert o.gelu_tanh(10.0) == 10.0 and abs(o.gelu_tanh(-10.0)) < 1e-20
    xs = np.linspace(-6, 6, 241)
    for x in xs:
        assert abs(o.gelu_tanh(x) - o.gelu_tanh(-x) - x) < 1e-14
        fd = (o.gelu_tanh(x + 1e-5) - o.gelu_tanh(x - 1e-5)) / 2e-5
        assert abs(fd - o.gelu_tanh_grad(x)) < 1e-9, x
    worst = max(abs(o.gelu_tanh(x) - o.gelu(x)) for x in np.linspace(-8, 8, 3201))
    assert 1e-4 < worst < 5e-4
    # at x = 1: u = √(2/π)·1.044715, from the textbook value of √(2/π)
    u = 0.7978845608028654 * 1.044715
    assert abs(o.gelu_tanh(1.0) - 0.5 * (1 + math.tanh(u))) < 1e-15


# --------------------------------------------------------- hand-worked example

def _hand_example():
    """T=2, h=2, F=4 (p=2 shards of 2 columns), chosen so every
    pre-activation is an integer and each output is a short expression in
    Φ(1), Φ(2), φ(1), φ(2)."""
    X = np.array([[1.0, 0.0], [0.0, 2.0]])
    A = np.array([[1.0, -1.0, 0.0, 2.0], [0.0, 1.0, -1.0, 0.0]])
    a = np.array([0.0, 0.0, 1.0, 0.0])
    B = np.array([[1.0, 0.0], [1.0, 1.0], [0.0, -1.0], [0.0, 1.0]])
    b = np.array([0.5, -0.25])
    dZ = np.array([[1.0, 0.0], [0.0, 1.0]])
    return dict(X=X, A=A, a=a, B=B, b=b, dZ=dZ)


def _hand_expected():
    tab = {x: (P, p) for x, P, p in _table()}
    P1, p1 = tab[1.0]
    P2, p2 = tab[2.0]
    # H = X·A + a = [[1, -1, 1, 2], [0, 2, -1, 0]]
    H = np.array([[1, -1, 1, 2], [0, 2, -1, 0]], dtype=float)
    # GeLU(k) = k·Φ(k), Φ(−k) = 1 − Φ(k)
    Y = np.array([[P1, -(1 - P1), P1, 2 * P2], [0.0, 2 * P2, -(1 - P1), 0.0]])
    # Z = Y·B + b, worked out by hand
    Z = np.array([[2 * P1 - 0.5, 2 * P2 - 1.25], [2 * P2 + 0.5, 2 * P2 - P1 + 0.75]])
    # dY = dZ·Bᵀ = [[1, 1, 0, 0], [0, 1, -1, 1]]; GeLU′(k) = Φ(k) + k·φ(k)
    g1, gm1, g2, g0 = P1 + p1, (1 - P1) - p1, P2 + 2 * p2, 0.5
    dH = np.array([[g1, gm1, 0.0, 0.0], [0.0, g2, -gm1, g0]])
    da = dH.sum(axis=0)
    dA = np.array([dH[0], 2 * dH[1]])  # Xᵀ·dH with X = diag(1, 2)
    dB = np.array([[Y[0, f], Y[1, f]] for f in range(4)])  # Yᵀ·I
    dX = np.array([[g1 - gm1, gm1], [-g2 + 2 * g0, g2 + gm1]])  # dH·Aᵀ
    db = np.array([1.0, 1.0])
    return dict(H=H, Y=Y, Z=Z, dH=dH, da=da, dA=dA, dB=dB, dX=dX, db=db)


def check_hand_example(orc):
    got = _all_outputs(orc, _hand_example())
    exp = _hand_expected()
    for k, v in exp.items():
        np.testing.assert_allclose(got[k], v, rtol=0, atol=1e-14, err_msg=k)


def test_hand_worked_example():
    check_hand_example(oracle.default())


# --------------------------------------------------------------- brute force

BRUTE_SHAPES = [(1, 1, 1), (2, 3, 4), (3, 2, 8), (5, 4, 12), (8, 6, 24), (7, 5, 10)]


def check_bruteforce(orc, shapes=BRUTE_SHAPES, seed=0, act=0):
    rng = np.random.default_rng(seed)
    for T, h, F in shapes:
        P = _rand_problem(rng, T, h, F)
        got = _all_outputs(orc, P, act)
        ref = bruteforce.mlp(*(P[k].tolist() for k in ("X", "A", "a", "B", "b", "dZ")), act=act)
        for k, v in ref.items():
            assert _max_rel(got[k], v) <= 1e-12, (k, T, h, F, act)


@pytest.mark.parametrize("act", [0, 1])
def test_bruteforce_tiny(act):
    check_bruteforce(oracle.default(), act=act)


# -------------------------------------------------------- finite differences

def check_finite_differences(orc, seed=1, T=5, h=4, F=8, n_probe=6, act=0):
    """L = Σ dZ ⊙ Z is linear in Z, so ∂L/∂θ is exactly the backward's output
    for θ ∈ {X, A, a, B, b}. Central differences (ε = 1e-6) pin all five
    gradients, GeLU′ included, independently of the backward formulas."""
    rng = np.random.default_rng(seed)
    P = _rand_problem(rng, T, h, F)
    out = _all_outputs(orc, P, act)
    grad_of = {"X": out["dX"], "A": out["dA"], "a": out["da"], "B": out["dB"], "b": out["db"]}

    def loss(Q):
        _, _, Z = orc.forward(Q["X"], Q["A"], Q["a"], Q["B"], Q["b"], act)
        return float(np.sum(P["dZ"] * Z))

    eps = 1e-6
    for name, g in grad_of.items():
        flat = P[name].reshape(-1)
        for idx in rng.choice(flat.size, size=min(n_probe, flat.size), replace=False):
            Qp = {k: v.copy() for k, v in P.items()}
            Qm = {k: v.copy() for k, v in P.items()}
            Qp[name].reshape(-1)[idx] += eps
            Qm[name].reshape(-1)[idx] -= eps
            fd = (loss(Qp) - loss(Qm)) / (2 * eps)
            an = g.reshape(-1)[idx]
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, idx, fd, an)


@pytest.mark.parametrize("act", [0, 1])
def test_finite_differences(act):
    check_finite_differences(oracle.default(), act=act)


# -------------------------------------------------- the pages' two identities

def check_partition_identities(orc, seed=2, T=6, h=5, F=24, act=0):
    rng = np.random.default_rng(seed)
    P = _rand_problem(rng, T, h, F)
    H, Y, Z = orc.forward(P["X"], P["A"], P["a"], P["B"], P["b"], act)
    g = orc.backward(P["X"], P["A"], P["B"], H, Y, P["dZ"], act)
    for p in [d for d in range(1, F + 1) if F % d == 0]:
        Hs, Ys, Zs = orc.forward_sharded(P["X"], P["A"], P["a"], P["B"], P["b"], p, act)
        # column split: concatenation of X·A_i + a_i is X·A + a, column for column
        np.testing.assert_array_equal(Hs, H)
        np.testing.assert_array_equal(Ys, Y)
        # row split: Σ_i Y_i·B_i equals Y·B (rounding order differs)
        assert _max_rel(Zs, Z) < 1e-13, p
        gs = orc.backward_sharded(P["X"], P["A"], P["B"], Hs, Ys, P["dZ"], p, act)
        for k in g:
            assert _max_rel(gs[k], g[k]) < 1e-13, (k, p)
    with pytest.raises(ValueError):
        orc.forward_sharded(P["X"], P["A"], P["a"], P["B"], P["b"], 5)


@pytest.mark.parametrize("act", [0, 1])
def test_partition_identities(act):
    check_partition_identities(oracle.default(), act=act)


def test_shard_split_by_hand():
    """The pages' identities checked on explicit shard matrices: concatenating
    X·A_i gives X·A; summing Y_i·B_i gives Y·B (p = 3)."""
    rng = np.random.default_rng(3)
    T, h, F, p = 4, 3, 9, 3
    P = _rand_problem(rng, T, h, F)
    zero_a, zero_b = np.zeros(F), np.zeros(h)
    H, Y, Z = oracle.forward(P["X"], P["A"], zero_a, P["B"], zero_b)
    Fp = F // p
    for i in range(p):
        Ai = P["A"][:, i * Fp:(i + 1) * Fp]
        Hi, _, _ = oracle.forward(P["X"], Ai, np.zeros(Fp), np.zeros((Fp, h)), zero_b)
        np.testing.assert_array_equal(Hi, H[:, i * Fp:(i + 1) * Fp])
    partial = np.zeros((T, h))
    for i in range(p):
        Bi = P["B"][i * Fp:(i + 1) * Fp]
        # Y_i·B_i via the oracle with an identity first layer on Y_i's columns
        Yi = Y[:, i * Fp:(i + 1) * Fp]
        partial += np.array([[math.fsum(Yi[t, f] * Bi[f, j] for f in range(Fp))
                              for j in range(h)] for t in range(T)])
    assert _max_rel(partial, Z) < 1e-14


# ------------------------------------------------------------ special cases

def check_special_cases(orc, seed=4, T=6, h=4, F=8):
    rng = np.random.default_rng(seed)
    P = _rand_problem(rng, T, h, F)
    # A = 0 ⇒ H = a on every row, Z = GeLU(a)·B + b on every row
    H, Y, Z = orc.forward(P["X"], np.zeros_like(P["A"]), P["a"], P["B"], P["b"])
    np.testing.assert_array_equal(H, np.broadcast_to(P["a"], H.shape))
    za = np.array([math.fsum([orc.gelu(P["a"][f]) * P["B"][f, j] for f in range(F)] + [P["b"][j]])
                   for j in range(h)])
    np.testing.assert_allclose(Z, np.broadcast_to(za, Z.shape), rtol=0, atol=1e-14)
    # B = 0 ⇒ Z = b; dY = 0 ⇒ dH, dA, da, dX vanish; db = column sums of dZ
    Bz = np.zeros_like(P["B"])
    H, Y, Z = orc.forward(P["X"], P["A"], P["a"], Bz, P["b"])
    np.testing.assert_array_equal(Z, np.broadcast_to(P["b"], Z.shape))
    g = orc.backward(P["X"], P["A"], Bz, H, Y, P["dZ"])
    for k in ("dH", "dA", "da", "dX"):
        assert np.all(g[k] == 0.0), k
    np.testing.assert_allclose(g["db"], [math.fsum(P["dZ"][:, j]) for j in range(h)],
                               rtol=0, atol=1e-14)
    # b enters once: Z(b') − Z(b) = b' − b on every row
    _, _, Z1 = orc.forward(P["X"], P["A"], P["a"], P["B"], P["b"])
    _, _, Z2 = orc.forward(P["X"], P["A"], P["a"], P["B"], 2.0 * P["b"])
    np.testing.assert_allclose(Z2 - Z1, np.broadcast_to(P["b"], Z1.shape), rtol=0, atol=1e-13)
    # dZ = 0 ⇒ every gradient vanishes
    H, Y, Z = orc.forward(P["X"], P["A"], P["a"], P["B"], P["b"])
    g = orc.backward(P["X"], P["A"], P["B"], H, Y, np.zeros_like(P["dZ"]))
    for k, v in g.items():
        assert np.all(v == 0.0), k


def test_special_cases():
    check_special_cases(oracle.default())


def test_empty_tokens():
    """T = 0: no rows out, and the weight/bias gradients are zero sums."""
    h, F = 3, 6
    rng = np.random.default_rng(5)
    P = _rand_problem(rng, 0, h, F)
    H, Y, Z = oracle.forward(P["X"], P["A"], P["a"], P["B"], P["b"])
    assert H.shape == (0, F) and Z.shape == (0, h)
    g = oracle.backward(P["X"], P["A"], P["B"], H, Y, P["dZ"])
    for k in ("dA", "da", "dB", "db"):
        assert np.all(g[k] == 0.0), k


# --------------------------------------------------------- subset functions

@pytest.mark.parametrize("act", [0, 1])
def test_rows_and_cols_match_full(act):
    rng = np.random.default_rng(6)
    T, h, F = 9, 5, 12
    P = _rand_problem(rng, T, h, F)
    full = _all_outputs(oracle.default(), P, act)
    R = [0, 3, 8]
    r = oracle.rows(P["X"], P["A"], P["a"], P["B"], P["b"], P["dZ"], R, act)
    for k in ("H", "Y", "Z", "dH", "dX"):
        np.testing.assert_allclose(r[k], full[k][R], rtol=1e-14, atol=1e-15, err_msg=k)
    J = [1, 4, 11]
    c = oracle.cols(P["X"], P["A"], P["a"], P["B"], P["dZ"], J, act)
    for k in ("H", "Y", "dH", "dA"):
        np.testing.assert_allclose(c[k], full[k][:, J], rtol=1e-14, atol=1e-15, err_msg=k)
    np.testing.assert_allclose(c["da"], full["da"][J], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(c["dB"], full["dB"][J], rtol=1e-14, atol=1e-15)


# ------------------------------------------------ torch float64 cross-check

@pytest.mark.parametrize("act", [0, 1])
def test_torch_float64_autograd(act):
    """An independent implementation: torch CPU float64, exact or tanh GeLU, autograd."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    T, h, F = 16, 8, 32
    P = _rand_problem(rng, T, h, F)
    got = _all_outputs(oracle.default(), P, act)
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=k != "dZ") for k, v in P.items()}
    Hh = t["X"] @ t["A"] + t["a"]
    Hh.retain_grad()
    Yy = torch.nn.functional.gelu(Hh, approximate="tanh" if act else "none")
    Zz = Yy @ t["B"] + t["b"]
    (Zz * t["dZ"]).sum().backward()
    ref = dict(H=Hh, Y=Yy, Z=Zz, dH=Hh.grad, dX=t["X"].grad, dA=t["A"].grad, da=t["a"].grad,
               dB=t["B"].grad, db=t["b"].grad)
    for k, v in ref.items():
        assert _max_rel(got[k], v.detach().numpy()) < 1e-12, k


# ------------------------------------------- tensor-parallel linear layers

def _rand_linear(rng, T, K, N):
    return dict(X=rng.standard_normal((T, K)), W=rng.standard_normal((K, N)) * 0.7,
                bias=rng.standard_normal(N) * 0.5, dY=rng.standard_normal((T, N)))


def check_linear_bruteforce(orc, seed=8):
    rng = np.random.default_rng(seed)
    for T, K, N in [(1, 1, 1), (3, 4, 6), (5, 6, 4), (7, 8, 12)]:
        P = _rand_linear(rng, T, K, N)
        Y = orc.linear_forward(P["X"], P["W"], P["bias"])
        dX, dW, db = orc.linear_backward(P["X"], P["W"], P["dY"])
        ref = bruteforce.linear(*(P[k].tolist() for k in ("X", "W", "bias", "dY")))
        for k, v in dict(Y=Y, dX=dX, dW=dW, db=db).items():
            assert _max_rel(v, ref[k]) <= 1e-12, (k, T, K, N)


def test_linear_bruteforce():
    check_linear_bruteforce(oracle.default())


def test_linear_finite_differences():
    """L = Σ dY ⊙ Y; central differences pin dX, dW, dbias."""
    rng = np.random.default_rng(9)
    P = _rand_linear(rng, 4, 5, 6)
    dX, dW, db = oracle.linear_backward(P["X"], P["W"], P["dY"])

    def loss(Q):
        return float(np.sum(P["dY"] * oracle.linear_forward(Q["X"], Q["W"], Q["bias"])))

    for name, g in (("X", dX), ("W", dW), ("bias", db)):
        for idx in rng.choice(P[name].size, size=5, replace=False):
            Qp = {k: v.copy() for k, v in P.items()}
            Qm = {k: v.copy() for k, v in P.items()}
            Qp[name].reshape(-1)[idx] += 1e-6
            Qm[name].reshape(-1)[idx] -= 1e-6
            fd = (loss(Qp) - loss(Qm)) / 2e-6
            assert abs(fd - g.reshape(-1)[idx]) <= 1e-7 * max(1.0, abs(fd)), (name, idx)


@pytest.mark.parametrize("split", ["columns", "rows"])
def test_linear_partition_identities(split):
    """Column split: concatenated X·W_i + bias_i equals X·W + bias bit for bit;
    row split: Σ_i X_i·W_i + bias equals it within rounding; both backward
    partitions give the unsplit gradients."""
    rng = np.random.default_rng(10)
    T, K, N = 6, 12, 24
    P = _rand_linear(rng, T, K, N)
    Y = oracle.linear_forward(P["X"], P["W"], P["bias"])
    dX, dW, db = oracle.linear_backward(P["X"], P["W"], P["dY"])
    dim = N if split == "columns" else K
    for p in [d for d in range(1, dim + 1) if dim % d == 0]:
        Ys = oracle.linear_forward_sharded(P["X"], P["W"], P["bias"], p, split)
        if split == "columns":
            np.testing.assert_array_equal(Ys, Y)
        else:
            assert _max_rel(Ys, Y) < 1e-13, p
        gs = oracle.linear_backward_sharded(P["X"], P["W"], P["dY"], p, split)
        for a, b in zip(gs, (dX, dW, db)):
            assert _max_rel(a, b) < 1e-13, (split, p)
    with pytest.raises(ValueError):
        oracle.linear_forward_sharded(P["X"], P["W"], P["bias"], 5, split)


def test_mlp_is_column_linear_gelu_row_linear():
    """The block composes the two layers: H = column-linear(X; A, a),
    Z = row-linear(GeLU(H); B, b), and the backward chains through GeLU′."""
    rng = np.random.default_rng(11)
    P = _rand_problem(rng, 5, 6, 12)
    full = _all_outputs(oracle.default(), P)
    H = oracle.linear_forward(P["X"], P["A"], P["a"])
    np.testing.assert_allclose(H, full["H"], rtol=0, atol=1e-14)
    Z = oracle.linear_forward(full["Y"], P["B"], P["b"])
    np.testing.assert_allclose(Z, full["Z"], rtol=0, atol=1e-13)
    dY, dB, db = oracle.linear_backward(full["Y"], P["B"], P["dZ"])
    np.testing.assert_allclose(dB, full["dB"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(db, full["db"], rtol=0, atol=1e-13)
    dX, dA, da = oracle.linear_backward(P["X"], P["A"], full["dH"])
    np.testing.assert_allclose(dX, full["dX"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dA, full["dA"], rtol=0, atol=1e-13)


def test_linear_torch_float64_autograd():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(12)
    P = _rand_linear(rng, 9, 7, 11)
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=k != "dY") for k, v in P.items()}
    Y = t["X"] @ t["W"] + t["bias"]
    (Y * t["dY"]).sum().backward()
    got = oracle.linear_forward(P["X"], P["W"], P["bias"])
    dX, dW, db = oracle.linear_backward(P["X"], P["W"], P["dY"])
    assert _max_rel(got, Y.detach().numpy()) < 1e-13
    for a, b in ((dX, t["X"].grad), (dW, t["W"].grad), (db, t["bias"].grad)):
        assert _max_rel(a, b.numpy()) < 1e-13


# ------------------------------------------------------- planted mistakes

MUTANTS = {
    # GeLU′ missing the x·φ(x) term
    "dropped_term": ("return tpo_normal_cdf(x) + x * tpo_normal_pdf(x);", "return tpo_normal_cdf(x);"),
    # wrong sign in GeLU′
    "wrong_sign": ("return tpo_normal_cdf(x) + x * tpo_normal_pdf(x);",
                   "return tpo_normal_cdf(x) - x * tpo_normal_pdf(x);"),
    # tanh-free but wrong constant inside erf (x/2 instead of x/√2)
    "wrong_constant": ("#define TPO_SQRT1_2 0.70710678118654752440", "#define TPO_SQRT1_2 0.5"),
    # transposed operand in dX = dH·Aᵀ (reads A as if it were F×h)
    "transposed_operand": ("mm_nt(T, h, F, dH, A, dX);", "mm_nn(T, h, F, dH, A, dX, 0);"),
    # bias a dropped from the pre-activation
    "dropped_bias": ("H[t * F + f] += a[f];", "H[t * F + f] += 0.0 * a[f];"),
    # wrong cubic coefficient in the tanh form
    "wrong_tanh_constant": ("#define TPO_GELU_TANH_C 0.044715", "#define TPO_GELU_TANH_C 0.04"),
    # linear-layer bias added twice
    "linear_bias_twice": ("for (int64_t n = 0; n < N; ++n) Y[t * N + n] += bias[n];",
                          "for (int64_t n = 0; n < N; ++n) Y[t * N + n] += 2.0 * bias[n];"),
    # db summing the wrong tensor's columns
    "wrong_index": ("tpo_colsum(T, h, dZ, db);\n    mm_tn(F, h, T, Y, dZ, dB);",
                    "tpo_colsum(T, h, dZ, db);\n    mm_tn(F, h, T, H, dZ, dB);"),
}


def _catches(orc):
    checks = [check_hand_example, check_bruteforce, check_finite_differences, check_normal_table,
              check_linear_bruteforce]
    for chk in checks:
        for act in (0, 1):
            try:
                if chk is check_bruteforce:
                    chk(orc, shapes=[(3, 2, 4), (5, 4, 12)], act=act)
                elif chk is check_finite_differences:
                    chk(orc, act=act)
                elif act == 0:
                    chk(orc)
            except AssertionError:
                return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutant = oracle.compile_variant(src.replace(old, new, 1), str(tmp_path / f"mut_{name}.so"))
    assert _catches(mutant), f"planted mistake {name!r} passed every pin"


def test_unmutated_build_passes_all_pins(tmp_path):
    clean = oracle.compile_variant(oracle.source_text(), str(tmp_path / "clean.so"))
    assert not _catches(clean)
