"""Pins of the CPU oracle against facts fixed outside it.

Each check ties an oracle function to something other than itself: a worked
example solved by hand, dense Gaussian elimination (numpy's LAPACK and the
oracle's own LU), central finite differences of the loss, the closed-form
eigenpairs of the Dirichlet Poisson operator, the Krylov-subspace optimality of
conjugate gradients, brute force on tiny inputs, and invariants (symmetry,
gradient pattern, adjoint and Euler identities, permutation equivariance).

The method: Jacobi-preconditioned CG and its implicit-function-theorem adjoint
from "torch-sla: Differentiable Sparse Linear Algebra with Adjoint Solvers and
Sparse Tensor Parallelism for PyTorch" (technical summary, "Methodology" 1-2).
"""
import ctypes
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from differentiable_sparse_linear_csr_b200 import workloads as W
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    d = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (d if d > 0 else 1.0)


def _golden(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split(":", 1)
        out[k.strip()] = [Fraction(t) for t in v.split()]
    return out


def _dense(rp, ci, v, n_cols=None):
    return W.csr_to_dense(rp, ci, v, n_cols)


# ---------------------------------------------------------------------------
# Worked example (hand-derived rational arithmetic)
# ---------------------------------------------------------------------------

def test_worked_2x2_iterates_and_gradient():
    g = _golden("pcg_2x2_worked.txt")
    rp = np.array([int(f) for f in g["rowptr"]], np.int32)
    ci = np.array([int(f) for f in g["colind"]], np.int32)
    v = np.array([float(f) for f in g["values"]])
    b = np.array([float(f) for f in g["b"]])
    x1, i1 = O.pcg(rp, ci, v, b, fixed_iters=1)
    assert i1.iters[0] == 1
    np.testing.assert_allclose(x1, [float(f) for f in g["x1"]], rtol=4e-16, atol=0)
    x2, i2 = O.pcg(rp, ci, v, b, fixed_iters=2)
    np.testing.assert_allclose(x2, [float(f) for f in g["x2"]], rtol=1e-15, atol=0)
    # tolerance mode: finite termination after n = 2 steps
    x, info = O.pcg(rp, ci, v, b, rtol=1e-14)
    assert info.iters[0] == 2 and info.status[0] == O.CONVERGED
    xs = np.array([float(f) for f in g["xstar"]])
    lam, _ = O.cg_adjoint(rp, ci, v, x - xs, rtol=1e-15)
    np.testing.assert_allclose(lam, [float(f) for f in g["lambda"]], rtol=1e-14, atol=0)
    G = O.grad_values(rp, ci, lam, x)
    np.testing.assert_allclose(G, [float(f) for f in g["grad_values"]], rtol=1e-14, atol=0)


def _fp32_example():
    g = _golden("pcg_fp32_policy_3x3.txt")
    rp = np.array([int(f) for f in g["rowptr"]], np.int32)
    ci = np.array([int(f) for f in g["colind"]], np.int32)
    v = np.array([float(f) for f in g["values"]], np.float32)
    b = np.array([float(f) for f in g["b"]], np.float32)
    # the stored iterates are fp32 numbers; float() of the exact fraction is exact
    x1 = np.array([float(f) for f in g["x1"]], np.float32)
    x2 = np.array([float(f) for f in g["x2"]], np.float32)
    assert all(float(np.float32(float(f))) == f for f in g["x1"] + g["x2"])
    return rp, ci, v, b, x1, x2


def test_fp32_precision_policy_worked_example_bit_for_bit():
    """The fp32 oracle reproduces the hand-worked iterates of the 3x3 example
    exactly: every rounding of the stated precision policy is where the
    derivation puts it."""
    rp, ci, v, b, x1, x2 = _fp32_example()
    for k, want in ((1, x1), (2, x2)):
        x, info = O.pcg(rp, ci, v, b, fixed_iters=k)
        assert x.dtype == np.float32 and info.iters[0] == k
        assert np.array_equal(x.view(np.uint32), want.view(np.uint32)), (k, x, want)


# Slips in the fp32 arithmetic that a plausible implementation could make, as
# textual changes of the oracle's source (applied to a copy built on the side).
_FP32_SLIPS = {
    "dots accumulated in fp32": [
        ("    double s = 0.0;\n    if (!reverse) {\n", "    T s = (T)0;\n    if (!reverse) {\n"),
        ("        for (int32_t i = 0; i < n; ++i) s = s + (double)a[i] * (double)b[i];\n",
         "        for (int32_t i = 0; i < n; ++i) s = s + a[i] * b[i];\n"),
        ("        for (int32_t i = n - 1; i >= 0; --i) s = s + (double)a[i] * (double)b[i];",
         "        for (int32_t i = n - 1; i >= 0; --i) s = s + a[i] * b[i];")],
    "alpha kept in fp64 in the x and r updates": [
        ("x[i] = x[i] + a * p[i];", "x[i] = x[i] + alpha * p[i];"),
        ("r[i] = r[i] - a * q[i];", "r[i] = r[i] - alpha * q[i];")],
    "beta kept in fp64 in the direction update": [
        ("p[i] = q[i] + bt * p[i];", "p[i] = q[i] + beta * p[i];")],
    "matrix rows summed in fp64": [
        ("        T s = (T)0;\n        if (!reverse) {\n            for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t)\n"
         "                s = s + vals[t] * x[colind[t]];",
         "        double s = 0.0;\n        if (!reverse) {\n            for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t)\n"
         "                s = s + (double)vals[t] * (double)x[colind[t]];")],
}


def _oracle_variant(tmp_path, edits):
    """liboracle built from a copy of the oracle's source with `edits` applied."""
    import shutil
    import subprocess
    src_dir = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")
    for f in ("oracle.c", "oracle_body.h"):
        shutil.copy(os.path.join(src_dir, f), tmp_path / f)
    body = (tmp_path / "oracle_body.h").read_text()
    for old, new in edits:
        assert body.count(old) == 1, old
        body = body.replace(old, new)
    (tmp_path / "oracle_body.h").write_text(body)
    so = tmp_path / "liboracle_variant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", str(so), str(tmp_path / "oracle.c"), "-lm"])
    lib = ctypes.CDLL(str(so))
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    lib.orc_pcg_f32.argtypes = [i32, P, P, P, P, P, P, P]
    lib.orc_pcg_f32.restype = i32
    return lib


def _variant_pcg_f32(lib, rp, ci, v, b, k):
    x = np.zeros(b.shape[0], np.float32)
    o = O._Opts(0.0, 0.0, k, k, 1, 0, 0)
    r = O._Result()
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    assert lib.orc_pcg_f32(b.shape[0], p(rp), p(ci), p(v), p(b), p(x), ctypes.byref(o), ctypes.byref(r)) == 0
    return x


@pytest.mark.parametrize("slip", sorted(_FP32_SLIPS))
def test_fp32_worked_example_catches_a_planted_slip(slip, tmp_path):
    """Each slip, planted in a copy of the oracle, changes the worked example's
    second iterate, so the bit-for-bit pin above would fail on it; the copy
    without edits reproduces the example."""
    rp, ci, v, b, x1, x2 = _fp32_example()
    (tmp_path / "clean").mkdir()
    (tmp_path / "slip").mkdir()
    clean = _oracle_variant(tmp_path / "clean", [])
    assert np.array_equal(_variant_pcg_f32(clean, rp, ci, v, b, 2).view(np.uint32), x2.view(np.uint32))
    lib = _oracle_variant(tmp_path / "slip", _FP32_SLIPS[slip])
    x = _variant_pcg_f32(lib, rp, ci, v, b, 2)
    assert not np.array_equal(x.view(np.uint32), x2.view(np.uint32)), slip

# ---------------------------------------------------------------------------
# SpMV and dense LU against numpy
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("dtype", [np.float64, np.float32])
def test_spmv_matches_dense_product(dtype):
    rng = np.random.default_rng(11)
    for n_rows, n_cols in [(1, 1), (7, 13), (60, 40), (200, 200)]:
        d = rng.standard_normal((n_rows, n_cols)) * (rng.random((n_rows, n_cols)) < 0.15)
        d[0, :] = 0.0                                    # an empty row
        rp, ci, v = W.dense_to_csr(d, keep_diagonal=False)
        x = rng.standard_normal(n_cols)
        y = O.spmv(rp, ci, v.astype(dtype), x.astype(dtype))
        ref = d.astype(dtype).astype(np.float64) @ x.astype(dtype).astype(np.float64)
        tol = 1e-14 if dtype == np.float64 else 2e-6
        assert np.all(np.abs(y - ref) <= tol * (np.abs(d) @ np.abs(x) + 1e-300))


def test_dense_lu_matches_numpy():
    rng = np.random.default_rng(3)
    for n in (1, 3, 17, 80):
        a = rng.standard_normal((n, n)) + n * np.eye(n) * rng.random()
        b = rng.standard_normal(n)
        assert rel(O.dense_lu_solve(a, b), np.linalg.solve(a, b)) < 1e-12


# ---------------------------------------------------------------------------
# PCG against direct dense solves
# ---------------------------------------------------------------------------

def _spd_cases():
    yield W.random_spd(1, 1.0, 1)
    yield W.random_spd(2, 1.0, 2)
    yield W.random_spd(5, 0.6, 3)
    yield W.random_spd(50, 0.1, 4)
    yield W.random_spd(200, 0.03, 5)
    yield W.poisson2d(8)


def test_pcg_matches_dense_solves():
    for k, (rp, ci, v) in enumerate(_spd_cases()):
        n = rp.shape[0] - 1
        b = W.uniform(100 + k, W.STREAM_B, n, -1, 1)
        x, info = O.pcg(rp, ci, v, b, rtol=1e-14)
        assert info.status[0] == O.CONVERGED
        d = _dense(rp, ci, v)
        assert rel(x, np.linalg.solve(d, b)) < 1e-11
        assert rel(x, O.dense_lu_solve(d, b)) < 1e-11
        x_np, info_np = O.pcg(rp, ci, v, b, rtol=1e-14, precond=False)
        assert rel(x_np, np.linalg.solve(d, b)) < 1e-11


def test_pcg_fp32_follows_fp64():
    rp, ci, v = W.random_spd(300, 0.02, 9)
    b = W.uniform(9, W.STREAM_B, 300, -1, 1)
    x64, _ = O.pcg(rp, ci, v, b, rtol=1e-6)
    x32, i32 = O.pcg(rp, ci, v.astype(np.float32), b.astype(np.float32), rtol=1e-6)
    assert x32.dtype == np.float32 and i32.status[0] == O.CONVERGED
    assert rel(x32, np.linalg.solve(_dense(rp, ci, v), b)) < 1e-5
    assert rel(x32, x64) < 1e-5


def test_initial_guess_and_zero_rhs():
    rp, ci, v = W.random_spd(40, 0.1, 12)
    b = W.uniform(12, W.STREAM_B, 40, -1, 1)
    xs = np.linalg.solve(_dense(rp, ci, v), b)
    x, info = O.pcg(rp, ci, v, b, rtol=1e-10, x0=xs)      # already solved
    assert info.iters[0] == 0 and info.status[0] == O.CONVERGED
    assert rel(x, xs) < 1e-14
    x, info = O.pcg(rp, ci, v, np.zeros(40), rtol=1e-10)
    assert info.iters[0] == 0 and np.all(x == 0)
    x0 = W.uniform(13, W.STREAM_XSTAR, 40, -1, 1)
    x, info = O.pcg(rp, ci, v, b, rtol=1e-13, x0=x0)
    assert info.status[0] == O.CONVERGED and rel(x, xs) < 1e-11


def test_breakdown_and_nonfinite_and_cap():
    # indefinite: diag positive, but not positive definite
    d = np.array([[1.0, 2.0], [2.0, 1.0]])
    rp, ci, v = W.dense_to_csr(d)
    x, info = O.pcg(rp, ci, v, np.array([1.0, -1.0]), rtol=1e-12)
    assert info.status[0] == O.BREAKDOWN
    # non-positive diagonal with Jacobi
    rp, ci, v = W.dense_to_csr(np.array([[-1.0, 0.0], [0.0, 1.0]]))
    _, info = O.pcg(rp, ci, v, np.array([1.0, 1.0]), rtol=1e-12)
    assert info.status[0] == O.BREAKDOWN and info.iters[0] == 0
    # NaN in b
    rp, ci, v = W.random_spd(10, 0.3, 2)
    b = np.ones(10); b[3] = np.nan
    _, info = O.pcg(rp, ci, v, b, rtol=1e-12)
    assert info.status[0] == O.NONFINITE
    # iteration cap
    rp, ci, v = W.poisson2d(16)
    _, info = O.pcg(rp, ci, v, np.ones(256), rtol=1e-14, max_iter=3)
    assert info.status[0] == O.NOT_CONVERGED and info.iters[0] == 3


# ---------------------------------------------------------------------------
# Closed-form eigenpairs of the Dirichlet Poisson operator
# ---------------------------------------------------------------------------

def _sine_vec(N, k):
    i = np.arange(1, N + 1)
    return np.sin(i * k * math.pi / (N + 1))


def _mu(N, k):
    return 4.0 * math.sin(k * math.pi / (2 * (N + 1))) ** 2


def test_poisson1d_eigenvector_rhs_converges_in_one_step():
    N = 64
    rp, ci, v = W.poisson1d(N)
    for k in (1, 7, 33, 64):
        xs = _sine_vec(N, k)
        b = _mu(N, k) * xs
        x, info = O.pcg(rp, ci, v, b, rtol=1e-12)
        assert info.iters[0] == 1 and info.status[0] == O.CONVERGED
        assert rel(x, xs) < 1e-14


def test_poisson2d_eigenvector_rhs_converges_in_one_step():
    N = 64
    rp, ci, v = W.poisson2d(N)
    for k, l in ((1, 1), (5, 60), (64, 2)):
        xs = np.outer(_sine_vec(N, k), _sine_vec(N, l)).reshape(-1)
        b = (_mu(N, k) + _mu(N, l)) * xs
        x, info = O.pcg(rp, ci, v, b, rtol=1e-12)
        assert info.iters[0] == 1
        assert rel(x, xs) < 1e-14


@pytest.mark.parametrize("m", [2, 3, 5])
def test_poisson2d_m_eigenvectors_converge_in_m_steps(m):
    N = 32
    rp, ci, v = W.poisson2d(N)
    pairs = [(1, 1), (3, 2), (6, 7), (10, 4), (20, 20)][:m]
    xs = sum(np.outer(_sine_vec(N, k), _sine_vec(N, l)).reshape(-1) for k, l in pairs)
    b = sum((_mu(N, k) + _mu(N, l)) * np.outer(_sine_vec(N, k), _sine_vec(N, l)).reshape(-1)
            for k, l in pairs)
    # finite termination: the residual collapses at step m, not before
    _, before = O.pcg(rp, ci, v, b, fixed_iters=m - 1)
    x, at = O.pcg(rp, ci, v, b, fixed_iters=m)
    assert before.relres[0] > 1e-3
    assert at.relres[0] < 1e-9
    x, info = O.pcg(rp, ci, v, b, rtol=1e-8)
    assert info.iters[0] == m and info.status[0] == O.CONVERGED
    # ||x - x*|| / ||x*|| <= (mu_max / mu_min) * ||r|| / ||b|| over the components present
    mus = [_mu(N, k) + _mu(N, l) for k, l in pairs]
    assert rel(x, xs) <= (max(mus) / min(mus)) * info.relres[0] * (1 + 1e-6)


def test_poisson2d_matches_sine_transform_solution():
    N = 64
    rp, ci, v = W.poisson2d(N)
    b = W.uniform(1, W.STREAM_B, N * N, -1, 1)
    i = np.arange(1, N + 1)
    S = math.sqrt(2.0 / (N + 1)) * np.sin(np.outer(i, i) * math.pi / (N + 1))   # orthonormal DST-I
    mu = np.array([_mu(N, k) for k in range(1, N + 1)])
    B = b.reshape(N, N)
    X = S @ ((S @ B @ S) / (mu[:, None] + mu[None, :])) @ S
    x, info = O.pcg(rp, ci, v, b, rtol=1e-13)
    kappa = (mu[-1] * 2) / (mu[0] * 2)
    assert rel(x, X.reshape(-1)) < kappa * 1e-13


# ---------------------------------------------------------------------------
# Krylov optimality: the k-th PCG iterate minimises the A-norm error over
# x0 + K_k(M^-1 A, M^-1 r0)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("precond", [True, False])
def test_fixed_k_iterate_is_krylov_minimiser(precond):
    rp, ci, v = W.random_spd(48, 0.12, 21, diag_extra=0.2)
    n = 48
    A = _dense(rp, ci, v)
    b = W.uniform(21, W.STREAM_B, n, -1, 1)
    Minv = 1.0 / np.diag(A) if precond else np.ones(n)
    xstar = np.linalg.solve(A, b)
    basis = [Minv * b]
    for k in range(1, 11):
        Q, _ = np.linalg.qr(np.array(basis).T)
        y = np.linalg.solve(Q.T @ A @ Q, Q.T @ b)
        xk_ref = Q @ y
        xk, info = O.pcg(rp, ci, v, b, fixed_iters=k, precond=precond)
        assert info.iters[0] == k
        err = math.sqrt((xk - xstar) @ A @ (xk - xstar))
        err_ref = math.sqrt((xk_ref - xstar) @ A @ (xk_ref - xstar))
        assert rel(xk, xk_ref) < 1e-9, (k, rel(xk, xk_ref))
        assert err <= err_ref * (1 + 1e-8)
        basis.append(Minv * (A @ basis[-1]))


# ---------------------------------------------------------------------------
# Adjoint and value gradients
# ---------------------------------------------------------------------------

def _loss(A, b, xs):
    x = np.linalg.solve(A, b)
    return 0.5 * float((x - xs) @ (x - xs))


def test_gradient_matches_dense_gradient():
    for k, (rp, ci, v) in enumerate(_spd_cases()):
        n = rp.shape[0] - 1
        b = W.uniform(200 + k, W.STREAM_B, n, -1, 1)
        xs = W.uniform(200 + k, W.STREAM_XSTAR, n, -1, 1)
        x, _ = O.pcg(rp, ci, v, b, rtol=1e-15, max_iter=10 * n + 50)
        lam, _ = O.cg_adjoint(rp, ci, v, x - xs, rtol=1e-15, max_iter=10 * n + 50)
        G = O.grad_values(rp, ci, lam, x)
        A = _dense(rp, ci, v)
        xd = np.linalg.solve(A, b)
        lam_d = np.linalg.solve(A.T, xd - xs)
        Gd = -np.outer(lam_d, xd)                          # dL/dA, dense
        rows = np.repeat(np.arange(n), np.diff(rp))
        assert G.shape == ci.shape                         # pattern of A, no more
        assert rel(G, Gd[rows, ci]) < 1e-10
        assert rel(lam, lam_d) < 1e-10


def test_gradient_matches_central_differences_per_entry():
    rp, ci, v = W.random_spd(12, 0.4, 31)
    n = 12
    b = W.uniform(31, W.STREAM_B, n, -1, 1)
    xs = W.uniform(31, W.STREAM_XSTAR, n, -1, 1)
    x, _ = O.pcg(rp, ci, v, b, rtol=1e-15)
    lam, _ = O.cg_adjoint(rp, ci, v, x - xs, rtol=1e-15)
    G = O.grad_values(rp, ci, lam, x)
    A = _dense(rp, ci, v)
    rows = np.repeat(np.arange(n), np.diff(rp))
    for t in range(ci.shape[0]):                        # one entry at a time (A may lose symmetry)
        h = 1e-6 * max(1.0, abs(v[t]))
        Ap, Am = A.copy(), A.copy()
        Ap[rows[t], ci[t]] += h
        Am[rows[t], ci[t]] -= h
        fd = (_loss(Ap, b, xs) - _loss(Am, b, xs)) / (2 * h)
        assert abs(fd - G[t]) <= 1e-6 * max(abs(fd), 1e-3), (t, fd, G[t])
    for i in range(n):                                  # dL/db = lambda
        h = 1e-6
        bp, bm = b.copy(), b.copy()
        bp[i] += h; bm[i] -= h
        fd = (_loss(A, bp, xs) - _loss(A, bm, xs)) / (2 * h)
        assert abs(fd - lam[i]) <= 1e-6 * max(abs(fd), 1e-3)


def test_symmetric_pair_fd_through_oracle_cg():
    rp, ci, v = W.random_spd(30, 0.15, 41)
    n = 30
    b = W.uniform(41, W.STREAM_B, n, -1, 1)
    xs = W.uniform(41, W.STREAM_XSTAR, n, -1, 1)

    def L(vals):
        x, _ = O.pcg(rp, ci, vals, b, rtol=1e-15, max_iter=1000)
        return 0.5 * float((x - xs) @ (x - xs))

    x, _ = O.pcg(rp, ci, v, b, rtol=1e-15, max_iter=1000)
    lam, _ = O.cg_adjoint(rp, ci, v, x - xs, rtol=1e-15, max_iter=1000)
    G = O.grad_values(rp, ci, lam, x)
    rows = np.repeat(np.arange(n), np.diff(rp))
    pos = {(int(r), int(c)): t for t, (r, c) in enumerate(zip(rows, ci))}
    checked = 0
    for (r, c), t in pos.items():
        if r >= c:
            continue
        t2 = pos[(c, r)]
        h = 1e-6
        vp, vm = v.copy(), v.copy()
        vp[t] += h; vp[t2] += h; vm[t] -= h; vm[t2] -= h
        fd = (L(vp) - L(vm)) / (2 * h)
        assert abs(fd - (G[t] + G[t2])) <= 1e-6 * max(abs(fd), 1e-3)
        checked += 1
    assert checked > 10


@pytest.mark.parametrize("name", ["c1", "c4"])
def test_directional_fd_at_workload_size(name):
    w = W.CONFIGS[name]()
    s = 0 if name == "c1" else 17                       # one system of the batch
    rp, ci, v, b, xs = w.rowptr, w.colind, w.values[s], w.b[s], w.xstar[s]
    x, _ = O.pcg(rp, ci, v, b, rtol=1e-13)
    lam, _ = O.cg_adjoint(rp, ci, v, x - xs, rtol=1e-13)
    G = O.grad_values(rp, ci, lam, x)
    rows = np.repeat(np.arange(w.n), np.diff(rp))
    # symmetric direction on the pattern keeps A symmetric; scale off-diagonals only
    d = W.uniform(77, W.STREAM_POINTS, ci.shape[0], -1, 1)
    tr = {(int(r), int(c)): t for t, (r, c) in enumerate(zip(rows, ci))}
    dsym = np.array([d[min(t, tr[(int(c), int(r))])] for t, (r, c) in enumerate(zip(rows, ci))])
    dsym *= 0.01 * np.abs(v)
    db = W.uniform(78, W.STREAM_POINTS, w.n, -1, 1)

    def L(eps):
        x, _ = O.pcg(rp, ci, v + eps * dsym, b + eps * db, rtol=1e-13)
        return 0.5 * float((x - xs) @ (x - xs))

    h = 1e-5
    fd = (L(h) - L(-h)) / (2 * h)
    ad = float(G @ dsym + lam @ db)
    assert abs(fd - ad) <= 1e-6 * abs(fd)


def test_adjoint_and_euler_identities():
    w = W.c1_poisson64()
    rp, ci, v, b, xs = w.rowptr, w.colind, w.values[0], w.b[0], w.xstar[0]
    x, _ = O.pcg(rp, ci, v, b, rtol=1e-13)
    g = x - xs
    lam, _ = O.cg_adjoint(rp, ci, v, g, rtol=1e-13)
    G = O.grad_values(rp, ci, lam, x)
    assert abs(g @ x - lam @ b) <= 1e-10 * abs(g @ x)    # g.A^-1 b two ways
    euler = float(G @ v)                                  # sum_t G_t v_t = -lambda.(A x)
    assert abs(euler + lam @ b) <= 1e-10 * abs(lam @ b)


def test_adjoint_equals_dense_transposed_solve_on_symmetric_storage():
    rp, ci, v = W.random_spd(64, 0.08, 51)
    g = W.uniform(51, W.STREAM_B, 64, -1, 1)
    lam, _ = O.cg_adjoint(rp, ci, v, g, rtol=1e-14)
    assert rel(lam, np.linalg.solve(_dense(rp, ci, v).T, g)) < 1e-11


def test_permutation_equivariance():
    w = W.c1_poisson64()
    rng = np.random.default_rng(5)
    perm = rng.permutation(w.n)
    rp2, ci2, v2 = W.permute_symmetric(w.rowptr, w.colind, w.values[0], perm)
    x, _ = O.pcg(w.rowptr, w.colind, w.values[0], w.b[0], rtol=1e-13)
    y, _ = O.pcg(rp2, ci2, v2, w.b[0][perm], rtol=1e-13)
    assert rel(y, x[perm]) < 1e-10


def test_gradient_accumulate_adds():
    rp, ci, v = W.random_spd(20, 0.2, 61)
    lam = W.uniform(61, W.STREAM_B, 20, -1, 1)
    x = W.uniform(61, W.STREAM_XSTAR, 20, -1, 1)
    base = W.uniform(62, W.STREAM_B, ci.shape[0], -1, 1)
    G = O.grad_values(rp, ci, lam, x)
    G2 = O.grad_values(rp, ci, lam, x, grad=base)
    assert np.array_equal(G2, base + G)


# ---------------------------------------------------------------------------
# Integer routines: transpose, COO -> CSR, validation (brute force)
# ---------------------------------------------------------------------------

def _random_csr(rng, n_rows, n_cols, density):
    mask = rng.random((n_rows, n_cols)) < density
    d = np.where(mask, rng.standard_normal((n_rows, n_cols)), 0.0)
    rows, cols = np.nonzero(mask)
    rp = np.zeros(n_rows + 1, np.int32)
    np.cumsum(np.bincount(rows, minlength=n_rows), out=rp[1:])
    return rp, cols.astype(np.int32), d[rows, cols]


def test_transpose_against_brute_force_and_involution():
    rng = np.random.default_rng(7)
    for n_rows, n_cols, dens in [(1, 1, 1.0), (5, 9, 0.3), (40, 17, 0.2), (0, 3, 0.5), (30, 30, 0.0)]:
        rp, ci, v = _random_csr(rng, n_rows, n_cols, dens)
        rpT, ciT, vT, perm = O.transpose(rp, ci, v, n_cols)
        # brute force: walk columns, then rows ascending
        rows = np.repeat(np.arange(n_rows), np.diff(rp))
        ent = sorted(zip(ci.tolist(), rows.tolist(), range(ci.shape[0])))
        assert ciT.tolist() == [r for _, r, _ in ent]
        assert perm.tolist() == [t for _, _, t in ent]
        assert np.array_equal(vT, v[[t for _, _, t in ent]])
        assert rpT.tolist() == [0] + np.cumsum(np.bincount(ci, minlength=n_cols)).tolist()
        rp2, ci2, v2, _ = O.transpose(rpT, ciT, vT, n_rows)
        assert np.array_equal(rp2, rp) and np.array_equal(ci2, ci) and np.array_equal(v2, v)


def test_workload_matrices_are_bitwise_symmetric():
    for w in (W.c1_poisson64(), W.c4_batched(B=3)):
        for s in range(w.batch):
            rpT, ciT, vT, _ = O.transpose(w.rowptr, w.colind, w.values[s])
            assert np.array_equal(rpT, w.rowptr) and np.array_equal(ciT, w.colind)
            assert np.array_equal(vT, w.values[s])


def test_coo_to_csr_against_brute_force():
    rng = np.random.default_rng(8)
    for n_rows, n_cols, m in [(1, 1, 3), (6, 4, 30), (50, 70, 400), (10, 10, 0)]:
        row = rng.integers(0, n_rows, m).astype(np.int32)
        col = rng.integers(0, n_cols, m).astype(np.int32)
        val = rng.standard_normal(m)
        rp, ci, vo, slot = O.coo_to_csr(n_rows, n_cols, row, col, val)
        acc = {}
        order = []
        for e in range(m):
            key = (int(row[e]), int(col[e]))
            if key not in acc:
                acc[key] = float(val[e]); order.append(key)
            else:
                acc[key] = acc[key] + float(val[e])
        keys = sorted(acc)
        assert ci.tolist() == [c for _, c in keys]
        assert vo.tolist() == [acc[k] for k in keys]          # bitwise: same left-to-right sums
        counts = np.bincount(np.array([r for r, _ in keys], dtype=np.int64), minlength=n_rows) if keys else np.zeros(n_rows, int)
        assert rp.tolist() == [0] + np.cumsum(counts).tolist()
        pos = {k: i for i, k in enumerate(keys)}
        assert slot.tolist() == [pos[(int(row[e]), int(col[e]))] for e in range(m)]


def test_csr_check_codes():
    rp = np.array([0, 2, 3], np.int32)
    ci = np.array([0, 1, 1], np.int32)
    assert O.csr_check(2, 2, rp, ci, need_diag=True) == (0, -1)
    assert O.csr_check(2, 2, np.array([1, 2, 3], np.int32), ci)[0] == 1
    assert O.csr_check(2, 2, np.array([0, 3, 2], np.int32), ci) == (2, 1)
    assert O.csr_check(2, 2, np.array([0, 2, 2], np.int32), ci)[0] == 3
    assert O.csr_check(2, 2, rp, np.array([0, 2, 1], np.int32)) == (4, 1)
    assert O.csr_check(2, 2, rp, np.array([1, 0, 1], np.int32)) == (5, 1)
    assert O.csr_check(2, 2, rp, np.array([0, 0, 1], np.int32)) == (5, 1)
    assert O.csr_check(2, 2, np.array([0, 1, 2], np.int32)[:3], np.array([1, 0], np.int32), need_diag=True) == (6, 0)
    d = O.diag_positions(rp, ci)
    assert d.tolist() == [0, 2]
