"""GPU (sm_100a) path against the CPU oracle on the same seeded inputs.

Tolerances (relative 2-norm per system unless stated):
  fp64 solutions 1e-8, fp64 adjoint/gradients 1e-6, fp32 solutions 1e-4 (the
  stated parity bars); CSR check/transpose/COO build and the value-gradient
  kernel on identical inputs are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import differentiable_sparse_linear_csr_b200 as sla
from differentiable_sparse_linear_csr_b200 import _lib as L
from differentiable_sparse_linear_csr_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL_X64, TOL_G64, TOL_X32 = 1e-8, 1e-6, 1e-4


def T(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def H(t):
    torch.cuda.synchronize()
    return t.detach().cpu().numpy()


def rel(a, ref):
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / (d if d > 0 else 1.0))


def rel_rows(a, ref):
    return [rel(a[s], ref[s]) for s in range(ref.shape[0])]


def make(rp, ci, B=1, dtype=torch.float64, symmetric=True, n_cols=None):
    return sla.CSR(T(rp), T(ci), n_cols=n_cols, batch=B, dtype=dtype, symmetric=symmetric)


def _random_csr(seed, n_rows, n_cols, per_row, diag=False):
    """Random pattern, about per_row entries a row (row lengths vary), sorted columns."""
    rng = np.random.default_rng(seed)
    k = rng.integers(0, 2 * per_row + 1, n_rows)
    rows = np.repeat(np.arange(n_rows, dtype=np.int64), k)
    cols = rng.integers(0, max(n_cols, 1), rows.shape[0]).astype(np.int64)
    if diag:
        d = np.arange(min(n_rows, n_cols), dtype=np.int64)
        rows, cols = np.concatenate([rows, d]), np.concatenate([cols, d])
    key = np.unique(rows * max(n_cols, 1) + cols)
    rows, cols = key // max(n_cols, 1), key % max(n_cols, 1)
    rp = np.zeros(n_rows + 1, np.int32)
    np.cumsum(np.bincount(rows, minlength=n_rows), out=rp[1:])
    return rp, cols.astype(np.int32)


def _spd_long_rows(n, per_row, seed):
    """Symmetric, strictly diagonally dominant, ~per_row entries a row."""
    rng = np.random.default_rng(seed)
    m = n * per_row // 2
    i = rng.integers(0, n, m)
    j = rng.integers(0, n, m)
    keep = i != j
    i, j = i[keep], j[keep]
    lo, hi = np.minimum(i, j), np.maximum(i, j)
    key = np.unique(lo.astype(np.int64) * n + hi)
    ei, ej = key // n, key % n
    w = W.uniform(seed, W.STREAM_WEIGHTS, ei.shape[0], 0.5, 2.0)
    rp, ci, v = W.weighted_laplacian(n, ei, ej, w, 0.5)
    return rp, ci, v


# ------------------------------------------------------------- integer work ----

def test_csr_check_matches_oracle_bit_exact():
    cases = [
        (2, 2, [0, 2, 3], [0, 1, 1], 1),
        (2, 2, [1, 2, 3], [0, 1, 1], 0),
        (2, 2, [0, 3, 2], [0, 1, 1], 0),
        (2, 2, [0, 2, 2], [0, 1, 1], 0),
        (2, 2, [0, 2, 3], [0, 2, 1], 0),
        (2, 2, [0, 2, 3], [1, 0, 1], 0),
        (2, 2, [0, 2, 3], [0, 0, 1], 0),
        (2, 2, [0, 1, 2], [1, 0], 1),
        (3, 3, [0, 1, 2, 3], [0, -1, 2], 0),
    ]
    rp, ci = _random_csr(5, 3000, 2000, 4)
    cases.append((3000, 2000, rp.tolist(), ci.tolist(), 0))
    bad = ci.copy(); bad[777] = 5000
    cases.append((3000, 2000, rp.tolist(), bad.tolist(), 0))
    for n_rows, n_cols, rp_, ci_, nd in cases:
        rp_ = np.array(rp_, np.int32)
        ci_ = np.array(ci_, np.int32)
        res = torch.zeros(2, dtype=torch.int64, device=DEV)
        L.sla_csr_check(n_rows, n_cols, ci_.shape[0], T(rp_), T(ci_), nd, res)
        assert tuple(H(res).tolist()) == O.csr_check(n_rows, n_cols, rp_, ci_, need_diag=nd)


def test_create_with_validate_rejects_invalid_pattern():
    with pytest.raises(L.SlaError, match="not strictly increasing"):
        make(np.array([0, 2, 3], np.int32), np.array([1, 0, 1], np.int32))


@pytest.mark.parametrize("shape", [(1, 1, 1), (700, 300, 3), (5000, 70000, 6), (40000, 257, 2)])
def test_transpose_bit_exact(shape):
    n_rows, n_cols, per_row = shape
    rp, ci = _random_csr(n_rows + n_cols, n_rows, n_cols, per_row)
    nnz = ci.shape[0]
    B = 3
    vals = W.uniform(7, W.STREAM_WEIGHTS, B * nnz, -1, 1).reshape(B, nnz)
    rpT_o, ciT_o, vT_o, perm_o = O.transpose(rp, ci, vals, n_cols)
    for dt in (torch.float64, torch.float32):
        v = T(vals).to(dt)
        rpT = torch.empty(n_cols + 1, dtype=torch.int32, device=DEV)
        ciT = torch.empty(max(nnz, 1), dtype=torch.int32, device=DEV)
        vT = torch.empty(B, max(nnz, 1), dtype=dt, device=DEV)
        perm = torch.empty(max(nnz, 1), dtype=torch.int32, device=DEV)
        ws = torch.empty(L.sla_transpose_workspace_bytes(n_rows, n_cols, nnz), dtype=torch.uint8, device=DEV)
        L.sla_csr_transpose(n_rows, n_cols, nnz, T(rp), T(ci), B, L.dtype_code(dt), v, rpT, ciT, vT,
                            perm, ws)
        assert np.array_equal(H(rpT), rpT_o)
        assert np.array_equal(H(ciT)[:nnz], ciT_o)
        assert np.array_equal(H(perm)[:nnz], perm_o)
        assert np.array_equal(H(vT)[:, :nnz], vT_o.astype(H(v).dtype))


@pytest.mark.parametrize("dims", [(1, 1, 5), (50, 40, 3000), (3000, 90000, 200000)])
def test_coo_to_csr_bit_exact(dims):
    n_rows, n_cols, m = dims
    rng = np.random.default_rng(m)
    row = rng.integers(0, n_rows, m).astype(np.int32)
    col = rng.integers(0, n_cols, m).astype(np.int32)
    B = 2
    val = W.uniform(9, W.STREAM_WEIGHTS, B * m, -1, 1).reshape(B, m)
    for dt in (torch.float64, torch.float32):
        vnp = val.astype(np.float64 if dt == torch.float64 else np.float32)
        rp_o, ci_o, v_o, slot_o = O.coo_to_csr(n_rows, n_cols, row, col, vnp)
        nnz_o = ci_o.shape[0]
        rp = torch.empty(n_rows + 1, dtype=torch.int32, device=DEV)
        ci = torch.empty(m, dtype=torch.int32, device=DEV)
        vo = torch.empty(B, m, dtype=dt, device=DEV)
        slot = torch.empty(m, dtype=torch.int32, device=DEV)
        nnz = torch.empty(1, dtype=torch.int64, device=DEV)
        ws = torch.empty(L.sla_coo_workspace_bytes(n_rows, n_cols, m), dtype=torch.uint8, device=DEV)
        L.sla_csr_from_coo(n_rows, n_cols, m, T(row), T(col), B, L.dtype_code(dt), T(vnp), rp, ci, vo,
                           slot, nnz, ws)
        assert int(H(nnz)[0]) == nnz_o
        assert np.array_equal(H(rp), rp_o)
        assert np.array_equal(H(ci)[:nnz_o], ci_o)
        assert np.array_equal(H(vo).reshape(B, m)[:, :nnz_o], np.atleast_2d(v_o))
        assert np.array_equal(H(slot), slot_o)


def test_coo_out_of_range_reports_minus_one():
    row = np.array([0, 1, 7], np.int32)
    col = np.array([0, 1, 1], np.int32)
    rp = torch.empty(3, dtype=torch.int32, device=DEV)
    ci = torch.empty(3, dtype=torch.int32, device=DEV)
    nnz = torch.empty(1, dtype=torch.int64, device=DEV)
    ws = torch.empty(L.sla_coo_workspace_bytes(2, 2, 3), dtype=torch.uint8, device=DEV)
    L.sla_csr_from_coo(2, 2, 3, T(row), T(col), 1, 0, None, rp, ci, None, None, nnz, ws)
    assert int(H(nnz)[0]) == -1


# ---------------------------------------------------------------- SpMV ----

def _spmv_bound(rp, ci, v, x):
    rows = np.repeat(np.arange(rp.shape[0] - 1), np.diff(rp))
    s = np.zeros(rp.shape[0] - 1)
    np.add.at(s, rows, np.abs(v) * np.abs(x[ci]))
    return s


def _skewed_csr(seed, n_rows, n_cols):
    """Short rows (mean below the one-thread-a-row limit) with a 3000-entry row
    every 997 rows: the 256-row chunks holding a long row exceed the staged
    kernels' shared memory and walk their rows in global memory instead."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 8, n_rows)
    lens[::997] = 3000
    rows = np.repeat(np.arange(n_rows, dtype=np.int64), lens)
    cols = np.concatenate([np.sort(rng.choice(n_cols, k, replace=False)) for k in lens]).astype(np.int32)
    rp = np.zeros(n_rows + 1, np.int32)
    np.cumsum(np.bincount(rows, minlength=n_rows), out=rp[1:])
    return rp, cols


@pytest.mark.parametrize("pipe", ["1", "0"])
def test_spmv_and_gradients_on_skewed_short_rows(pipe, monkeypatch):
    """Chunks staged in shared memory and chunks too long for it, in one launch
    (the pipelined fp64 SpMV, or one chunk a block)."""
    monkeypatch.setenv("SLA_SPMV_PIPE", pipe)
    n_rows, n_cols, B = 6000, 5000, 2
    rp, ci = _skewed_csr(11, n_rows, n_cols)
    A = make(rp, ci, B=B, symmetric=False, n_cols=n_cols)
    assert A.props.lanes == 1
    v = W.uniform(11, W.STREAM_WEIGHTS, B * ci.shape[0], -1, 1).reshape(B, -1)
    x = W.uniform(11, W.STREAM_B, B * n_cols, -1, 1).reshape(B, n_cols)
    y = H(A.spmv(T(v), T(x)))
    y_o = O.spmv(rp, ci, v, x)
    for s in range(B):
        bound = _spmv_bound(rp, ci, v[s], x[s]) * 64 * np.finfo(np.float64).eps + 1e-300
        assert np.all(np.abs(y[s] - y_o[s]) <= bound)
    lam = W.uniform(12, W.STREAM_B, B * n_rows, -1, 1).reshape(B, n_rows)
    assert np.array_equal(H(A.grad_values(T(lam), T(x))), O.grad_values(rp, ci, lam, x))
    assert np.array_equal(H(A.matvec_grad_values(T(lam), T(x))), -O.grad_values(rp, ci, lam, x))


@pytest.mark.parametrize("per_row,pipe", [(5, "1"), (5, "0"), (30, "1"), (60, "1"), (120, "1"), (250, "1"),
                                          (500, "1")])
def test_spmv_parity_all_row_widths(per_row, pipe, monkeypatch):
    monkeypatch.setenv("SLA_SPMV_PIPE", pipe)
    n_rows, n_cols = 3001, 2503
    rp, ci = _random_csr(per_row, n_rows, n_cols, per_row // 2 + 1)
    B = 2
    v = W.uniform(per_row, W.STREAM_WEIGHTS, B * ci.shape[0], -1, 1).reshape(B, -1)
    x = W.uniform(per_row, W.STREAM_B, B * n_cols, -1, 1).reshape(B, n_cols)
    A = make(rp, ci, B=B, symmetric=False, n_cols=n_cols)
    y = H(A.spmv(T(v), T(x)))
    y_o = O.spmv(rp, ci, v, x)
    for s in range(B):
        bound = _spmv_bound(rp, ci, v[s], x[s]) * 64 * np.finfo(np.float64).eps + 1e-300
        assert np.all(np.abs(y[s] - y_o[s]) <= bound)
    # transposed product through A^T's pattern
    xt = W.uniform(per_row, W.STREAM_XSTAR, B * n_rows, -1, 1).reshape(B, n_rows)
    yt = H(A.spmv(T(v), T(xt), transpose=True))
    rpT, ciT, vT, _ = O.transpose(rp, ci, v, n_cols)
    yt_o = O.spmv(rpT, ciT, vT, xt)
    for s in range(B):
        bound = _spmv_bound(rpT, ciT, vT[s], xt[s]) * 64 * np.finfo(np.float64).eps + 1e-300
        assert np.all(np.abs(yt[s] - yt_o[s]) <= bound)
    # fp32
    A32 = make(rp, ci, B=B, dtype=torch.float32, symmetric=False, n_cols=n_cols)
    y32 = H(A32.spmv(T(v.astype(np.float32)), T(x.astype(np.float32))))
    y32_o = O.spmv(rp, ci, v.astype(np.float32), x.astype(np.float32))
    for s in range(B):
        bound = _spmv_bound(rp, ci, v[s], x[s]) * 64 * np.finfo(np.float32).eps + 1e-30
        assert np.all(np.abs(y32[s].astype(np.float64) - y32_o[s]) <= bound)


def test_spmv_alpha_beta():
    rp, ci, v = W.poisson2d(33)
    A = make(rp, ci)
    x = W.uniform(1, W.STREAM_B, 33 * 33, -1, 1)
    y0 = W.uniform(2, W.STREAM_B, 33 * 33, -1, 1)
    y = T(y0[None, :]).clone()
    L.sla_spmv(A.handle, T(v[None, :]), T(x[None, :]), y, 0, 2.0, -0.5)
    ref = 2.0 * O.spmv(rp, ci, v, x) - 0.5 * y0
    assert rel(H(y)[0], ref) < 1e-15


@pytest.mark.parametrize("B", [1, 3])
def test_pipelined_spmv_batches_and_alpha_beta(B):
    """The pipelined fp64 SpMV over several systems (each system's values on the
    16-byte grid: 7840 entries), with y = alpha A x + beta y."""
    rp, ci, v = W.poisson2d(40)
    n, nnz = 1600, ci.shape[0]
    assert (nnz * 8) % 16 == 0
    A = make(rp, ci, B=B)
    vals = W.uniform(13, W.STREAM_WEIGHTS, B * nnz, -1, 1).reshape(B, nnz)
    x = W.uniform(13, W.STREAM_B, B * n, -1, 1).reshape(B, n)
    y0 = W.uniform(14, W.STREAM_B, B * n, -1, 1).reshape(B, n)
    y = T(y0).clone()
    L.sla_spmv(A.handle, T(vals), T(x), y, 0, 1.5, -0.25)
    for s_ in range(B):
        ref = 1.5 * O.spmv(rp, ci, vals[s_], x[s_]) - 0.25 * y0[s_]
        eps = np.finfo(np.float64).eps
        bound = (1.5 * _spmv_bound(rp, ci, vals[s_], x[s_]) * 64 + 0.25 * np.abs(y0[s_]) * 4) * eps + 1e-300
        assert np.all(np.abs(H(y)[s_] - ref) <= bound)


def test_spmv_values_off_the_16_byte_grid():
    """Values whose address is not a multiple of 16 bytes take the one-chunk-a-block kernel."""
    rp, ci, v = W.poisson2d(40)
    A = make(rp, ci)
    x = W.uniform(5, W.STREAM_B, 1600, -1, 1)
    buf = torch.zeros(ci.shape[0] + 1, dtype=torch.float64, device=DEV)
    vals = buf[1:]
    vals.copy_(T(v))
    assert vals.data_ptr() % 16 == 8
    y = H(A.spmv(vals[None, :], T(x[None, :])))[0]
    bound = _spmv_bound(rp, ci, v, x) * 64 * np.finfo(np.float64).eps + 1e-300
    assert np.all(np.abs(y - O.spmv(rp, ci, v, x)) <= bound)


# ------------------------------------------------------------ gradients ----

@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_grad_values_bit_exact_on_same_inputs(dtype):
    npdt = np.float64 if dtype == torch.float64 else np.float32
    for rp, ci, B in ((*W.poisson2d(45)[:2], 3), (*_random_csr(3, 5000, 5000, 30, diag=True), 2)):
        n = rp.shape[0] - 1
        lam = W.uniform(3, W.STREAM_B, B * n, -1, 1).reshape(B, n).astype(npdt)
        x = W.uniform(3, W.STREAM_XSTAR, B * n, -1, 1).reshape(B, n).astype(npdt)
        base = W.uniform(4, W.STREAM_B, B * ci.shape[0], -1, 1).reshape(B, -1).astype(npdt)
        A = make(rp, ci, B=B, dtype=dtype, symmetric=False)
        g = H(A.grad_values(T(lam), T(x)))
        assert np.array_equal(g, O.grad_values(rp, ci, lam, x))
        gb = T(base).clone()
        A.grad_values(T(lam), T(x), out=gb, accumulate=True)
        assert np.array_equal(H(gb), O.grad_values(rp, ci, lam, x, grad=base))
        # the matvec form gy_i x_j is the exact negation of -lambda_i x_j with lambda = gy
        assert np.array_equal(H(A.matvec_grad_values(T(lam), T(x))), -O.grad_values(rp, ci, lam, x))
        gb = T(base).clone()
        A.matvec_grad_values(T(lam), T(x), out=gb, accumulate=True)
        assert np.array_equal(H(gb), base - O.grad_values(rp, ci, lam, x))


# ------------------------------------------------------------- PCG solves ----

def _cases():
    # (name, rowptr, colind, values[B][nnz], b[B][n])
    w = W.c1_poisson64()
    yield "c1", w.rowptr, w.colind, w.values, w.b
    rp, ci, v = W.poisson2d(37)                       # ragged tail everywhere
    yield "poisson37", rp, ci, v[None, :], W.normal(5, 0, 37 * 37)[None, :]
    rp, ci, v = W.random_spd(3000, 0.002, 8, diag_extra=0.3)   # varying diagonal
    yield "random3000", rp, ci, v[None, :], W.uniform(8, 0, 3000, -1, 1)[None, :]
    # irregular rows in tiles of at least 32 rows: the sorted-window sliced layout
    rp, ci, v = W.random_spd(12000, 0.0005, 9, diag_extra=0.3)
    yield "random12000", rp, ci, v[None, :], W.uniform(9, 0, 12000, -1, 1)[None, :]
    rp, ci, v = _spd_long_rows(6000, 60, 3)              # wide rows: several lanes a row
    yield "wide6000", rp, ci, v[None, :], W.uniform(3, 0, 6000, -1, 1)[None, :]
    w = W.c4_batched(B=24)
    yield "c4x24", w.rowptr, w.colind, w.values, w.b


# (strategy, on-chip grid vectors, sliced short-row layout); on-chip "3" keeps
# the vectors on chip but turns the two-barrier single-system form off; sliced "u" is the sliced
# layout with per-slice widths (uniform widths off), "n" without the rows of
# irregular patterns sorted by length within 32-row windows, "w" with 32-bit
# columns only (no 16-bit offsets)
SOLVER_VARIANTS = [
    (L.SLA_STRATEGY_GRID, "1", "1"), (L.SLA_STRATEGY_GRID, "3", "1"),
    (L.SLA_STRATEGY_GRID, "0", "1"), (L.SLA_STRATEGY_GRID, "1", "0"),
    (L.SLA_STRATEGY_GRID, "0", "0"), (L.SLA_STRATEGY_GRID, "1", "u"),
    (L.SLA_STRATEGY_GRID, "0", "u"), (L.SLA_STRATEGY_GRID, "0", "n"),
    (L.SLA_STRATEGY_GRID, "1", "w"), (L.SLA_STRATEGY_GRID, "0", "w"),
    (L.SLA_STRATEGY_BLOCK, "1", "1"), (L.SLA_STRATEGY_CLUSTER, "1", "1")]


def _variant_env(monkeypatch, onchip, sell):
    monkeypatch.setenv("SLA_GRID_ONCHIP", "0" if onchip == "0" else "1")
    monkeypatch.setenv("SLA_GRID2", "0" if onchip == "3" else "1")
    monkeypatch.setenv("SLA_SELL", "0" if sell == "0" else "1")
    monkeypatch.setenv("SLA_SELL_UNIFORM", "0" if sell == "u" else "1")
    monkeypatch.setenv("SLA_SELL_SORT", "0" if sell == "n" else "1")
    monkeypatch.setenv("SLA_SELL_D16", "0" if sell == "w" else "1")


@pytest.mark.parametrize("strategy,onchip,sell", SOLVER_VARIANTS)
@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_pcg_fixed_iterations_parity(strategy, onchip, sell, dtype, monkeypatch):
    """Every grid variant (x, r, M^-1 on chip or in HBM; sliced or CSR rows) and
    the block solver."""
    _variant_env(monkeypatch, onchip, sell)
    npdt = np.float64 if dtype == torch.float64 else np.float32
    tol = TOL_X64 if dtype == torch.float64 else TOL_X32
    for name, rp, ci, v, b in _cases():
        B = v.shape[0]
        A = make(rp, ci, B=B, dtype=dtype)
        if strategy == L.SLA_STRATEGY_BLOCK and not A.props.block_fits:
            continue
        if strategy == L.SLA_STRATEGY_CLUSTER and not A.props.cluster_fits:
            continue
        if strategy == L.SLA_STRATEGY_GRID and onchip == "0":
            assert A.props.grid_onchip == 0
        if strategy == L.SLA_STRATEGY_GRID and onchip == "3":
            assert A.props.grid_onchip in (0, 1)
        if strategy == L.SLA_STRATEGY_GRID and onchip == "1" and B == 1 and A.props.sliced:
            assert A.props.grid_onchip == 2, name
        if sell == "u":
            assert A.props.sliced in (0, 1, 3), name
        if sell == "n":
            assert A.props.sliced in (0, 1, 2), name
        if sell == "w":
            assert A.props.sliced_col_bytes in (0, 4), name
        if name == "poisson37" and sell == "1":
            assert A.props.sliced_col_bytes == 2, name       # offsets within +-37
        if name == "random12000" and strategy == L.SLA_STRATEGY_GRID and onchip == "0" \
                and sell in ("1", "u"):
            assert A.props.sliced == 3, name            # irregular rows: sorted windows
        for k in (1, 7, 60):
            x, info = A.cg(T(v.astype(npdt)), T(b.astype(npdt)), fixed_iters=k, strategy=strategy)
            xo, io = O.pcg(rp, ci, v.astype(npdt), b.astype(npdt), fixed_iters=k)
            assert np.array_equal(H(info.iters), io.iters), name
            assert np.array_equal(H(info.status), io.status), name
            assert max(rel_rows(H(x), xo)) < tol, (name, k)


@pytest.mark.parametrize("strategy,onchip,sell", SOLVER_VARIANTS)
def test_pcg_tolerance_mode_parity(strategy, onchip, sell, monkeypatch):
    """Iteration counts agree within max(2, 1%); iterates agree at the oracle's count."""
    _variant_env(monkeypatch, onchip, sell)
    for name, rp, ci, v, b in _cases():
        B = v.shape[0]
        A = make(rp, ci, B=B)
        if strategy == L.SLA_STRATEGY_BLOCK and not A.props.block_fits:
            continue
        if strategy == L.SLA_STRATEGY_CLUSTER and not A.props.cluster_fits:
            continue
        xo, io = O.pcg(rp, ci, v, b, rtol=1e-10)
        x, info = A.cg(T(v), T(b), rtol=1e-10, strategy=strategy)
        it = H(info.iters)
        assert np.all(H(info.status) == 0) and np.all(io.status == 0), name
        assert np.all(np.abs(it - io.iters) <= np.maximum(2, 0.01 * io.iters)), (name, it, io.iters)
        assert np.all(H(info.relres) <= 1e-10)
        for s in range(B):
            xk, ik = A.cg(T(v), T(b), fixed_iters=int(io.iters[s]), strategy=strategy)
            assert rel(H(xk)[s], np.atleast_2d(xo)[s]) < TOL_X64, name


def test_grid_and_block_strategies_agree():
    w = W.c4_batched(B=16)
    A = make(w.rowptr, w.colind, B=16)
    xg, ig = A.cg(T(w.values), T(w.b), rtol=1e-10, strategy=L.SLA_STRATEGY_GRID)
    xb, ib = A.cg(T(w.values), T(w.b), rtol=1e-10, strategy=L.SLA_STRATEGY_BLOCK)
    assert max(rel_rows(H(xg), H(xb))) < 1e-9
    assert np.all(np.abs(H(ig.iters) - H(ib.iters)) <= 2)


@pytest.mark.parametrize("onchip", ["1", "0"])
def test_results_are_bitwise_reproducible(onchip, monkeypatch):
    monkeypatch.setenv("SLA_GRID_ONCHIP", onchip)
    w = W.c1_poisson64()
    A = make(w.rowptr, w.colind)
    for strategy in (L.SLA_STRATEGY_GRID, L.SLA_STRATEGY_BLOCK, L.SLA_STRATEGY_CLUSTER):
        x1, i1 = A.cg(T(w.values), T(w.b), rtol=1e-10, strategy=strategy)
        x2, i2 = A.cg(T(w.values), T(w.b), rtol=1e-10, strategy=strategy)
        assert torch.equal(x1, x2) and torch.equal(i1.iters, i2.iters)


@pytest.mark.parametrize("dtype,onchip,grid2", [(torch.float64, "1", "0"), (torch.float32, "1", "1"),
                                                (torch.float64, "0", "0"), (torch.float32, "1", "0")])
def test_row_ahead_column_loads_are_bit_identical(dtype, onchip, grid2, monkeypatch):
    """Loading the next row's column offsets ahead (uniform widths 5 and 7)
    changes no result bit: three-phase on chip, two barriers, vectors in HBM."""
    monkeypatch.setenv("SLA_GRID_ONCHIP", onchip)
    monkeypatch.setenv("SLA_GRID2", grid2)
    npdt = np.float64 if dtype == torch.float64 else np.float32
    w3 = W.c3_diffusion3d(N=40)
    for rp, ci, v in (W.poisson2d(150), (w3.rowptr, w3.colind, w3.values[0])):
        n = rp.shape[0] - 1
        A = make(rp, ci, dtype=dtype)
        assert A.props.sliced == 2 and A.props.sliced_col_bytes == 2
        b = T(W.uniform(7, W.STREAM_B, n, -1, 1).astype(npdt)[None, :])
        vals = T(v.astype(npdt)[None, :])
        out = {}
        for pipe in ("1", "0"):
            monkeypatch.setenv("SLA_SELL_PIPE", pipe)
            x, info = A.cg(vals, b, fixed_iters=40, strategy=L.SLA_STRATEGY_GRID)
            lam, _ = A.cg(vals, x, adjoint=True, fixed_iters=40, strategy=L.SLA_STRATEGY_GRID)
            out[pipe] = (x, lam)
        assert torch.equal(out["1"][0], out["0"][0]) and torch.equal(out["1"][1], out["0"][1])


# ----------------------------------------------------- adjoint + gradient ----

@pytest.mark.parametrize("symmetric_flag", [True, False])
def test_adjoint_and_gradient_parity(symmetric_flag):
    """Forward, adjoint and value gradient at the oracle's iteration counts."""
    for name, rp, ci, v, b in _cases():
        B = v.shape[0]
        n = rp.shape[0] - 1
        xs = W.uniform(11, W.STREAM_XSTAR, B * n, -1, 1).reshape(B, n)
        xo, io = O.pcg(rp, ci, v, b, rtol=1e-10)
        xo = np.atleast_2d(xo)
        lo, lio = O.cg_adjoint(rp, ci, v, xo - xs, rtol=1e-10)
        lo = np.atleast_2d(lo)
        Go = np.atleast_2d(O.grad_values(rp, ci, lo, xo))
        A = make(rp, ci, B=B, symmetric=symmetric_flag)
        for s in range(B):
            sel = slice(s, s + 1)
            # per system, at that system's own oracle counts
            x, _ = A.cg(T(v), T(b), fixed_iters=int(io.iters[s]))
            lam, _ = A.cg(T(v), x - T(xs), adjoint=True, fixed_iters=int(lio.iters[s]))
            G = A.grad_values(lam, x)
            assert rel(H(x)[sel], xo[sel]) < TOL_X64, name
            assert rel(H(lam)[sel], lo[sel]) < TOL_G64, name
            assert rel(H(G)[sel], Go[sel]) < TOL_G64, name
            if B > 4 and s >= 3:
                break


def test_autograd_solve_matches_oracle_and_finite_differences():
    w = W.c1_poisson64()
    rp, ci, v, b, xs = w.rowptr, w.colind, w.values[0], w.b[0], w.xstar[0]
    A = make(rp, ci)
    vals = T(v).requires_grad_(True)
    bt = T(b).requires_grad_(True)
    x = A.solve(vals, bt, rtol=1e-12)
    loss = 0.5 * ((x - T(xs)) ** 2).sum()
    loss.backward()
    xo, _ = O.pcg(rp, ci, v, b, rtol=1e-12)
    lo, _ = O.cg_adjoint(rp, ci, v, xo - xs, rtol=1e-12)
    Go = O.grad_values(rp, ci, lo, xo)
    assert rel(H(bt.grad), lo) < TOL_G64
    assert rel(H(vals.grad), Go) < TOL_G64
    # directional central difference through the GPU forward solve
    rng = np.random.default_rng(0)
    db = rng.uniform(-1, 1, b.shape[0])

    def L_of(eps):
        with torch.no_grad():
            xx = A.solve(T(v), T(b + eps * db), rtol=1e-13)
            return 0.5 * float(((xx - T(xs)) ** 2).sum())

    h = 1e-5
    fd = (L_of(h) - L_of(-h)) / (2 * h)
    assert abs(fd - float(H(bt.grad) @ db)) <= 1e-6 * abs(fd)


def test_autograd_matvec():
    rp, ci = _random_csr(2, 900, 700, 6)
    nnz = ci.shape[0]
    A = make(rp, ci, symmetric=False, n_cols=700)
    v = W.uniform(1, 2, nnz, -1, 1)
    x = W.uniform(1, 0, 700, -1, 1)
    gy = W.uniform(1, 1, 900, -1, 1)
    vt, xt = T(v).requires_grad_(True), T(x).requires_grad_(True)
    y = A.matvec(vt, xt)
    y.backward(T(gy))
    rows = np.repeat(np.arange(900), np.diff(rp))
    assert rel(H(y), O.spmv(rp, ci, v, x)) < 1e-15
    assert np.array_equal(H(vt.grad), gy[rows] * x[ci])
    rpT, ciT, vT, _ = O.transpose(rp, ci, v, 700)
    assert rel(H(xt.grad), O.spmv(rpT, ciT, vT, gy)) < 1e-14


def test_adjoint_memory_does_not_grow_with_iterations():
    rp, ci, v = W.poisson2d(200)
    A = make(rp, ci)
    b = T(W.normal(1, 0, 200 * 200))
    vals = T(v)
    peaks = []
    for k in (10, 10, 1000):   # the first pass warms up library-independent allocations
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
        vv = vals.clone().requires_grad_(True)
        x = A.solve(vv, b, fixed_iters=k)
        (x * x).sum().backward()
        torch.cuda.synchronize()
        peaks.append(torch.cuda.max_memory_allocated() - base)
        del x, vv
    assert peaks[1] == peaks[2]


# ------------------------------------------------------------ edge cases ----

@pytest.mark.parametrize("onchip", ["1", "3", "0"])
def test_edge_cases_match_oracle_outcomes(onchip, monkeypatch):
    _variant_env(monkeypatch, onchip, "1")
    rp, ci, v = W.random_spd(300, 0.02, 4)
    A = make(rp, ci)
    b = W.uniform(4, 0, 300, -1, 1)
    for strategy in (L.SLA_STRATEGY_GRID, L.SLA_STRATEGY_BLOCK, L.SLA_STRATEGY_CLUSTER):
        x, info = A.cg(T(v), T(np.zeros(300)), strategy=strategy)
        assert H(info.iters)[0] == 0 and H(info.status)[0] == L.SLA_CONVERGED and not H(x).any()
        xs = np.linalg.solve(W.csr_to_dense(rp, ci, v), b)
        x, info = A.cg(T(v), T(b), x0=T(xs), rtol=1e-10, strategy=strategy)
        assert H(info.iters)[0] == 0 and rel(H(x)[0], xs) < 1e-15
        x0 = W.uniform(5, 1, 300, -1, 1)
        x, info = A.cg(T(v), T(b), x0=T(x0), fixed_iters=9, strategy=strategy)
        xo, _ = O.pcg(rp, ci, v, b, fixed_iters=9, x0=x0)
        assert rel(H(x)[0], xo) < TOL_X64
        bn = b.copy(); bn[7] = np.nan
        _, info = A.cg(T(v), T(bn), strategy=strategy)
        assert H(info.status)[0] == L.SLA_NONFINITE
        _, info = A.cg(T(v), T(b), rtol=1e-15, max_iter=3, strategy=strategy)
        assert H(info.status)[0] == L.SLA_NOT_CONVERGED and H(info.iters)[0] == 3
        x, info = A.cg(T(v), T(b), rtol=1e-10, precond=False, strategy=strategy)
        xo, io = O.pcg(rp, ci, v, b, rtol=1e-10, precond=False)
        xk, _ = A.cg(T(v), T(b), fixed_iters=int(io.iters[0]), precond=False, strategy=strategy)
        assert abs(int(H(info.iters)[0]) - int(io.iters[0])) <= 2
        assert rel(H(xk)[0], xo) < TOL_X64
    # indefinite matrix: breakdown; negative diagonal: breakdown before any step
    rpi, cii, vi = W.dense_to_csr(np.array([[1.0, 2.0], [2.0, 1.0]]))
    Ai = make(rpi, cii)
    for strategy in (L.SLA_STRATEGY_GRID, L.SLA_STRATEGY_BLOCK, L.SLA_STRATEGY_CLUSTER):
        _, info = Ai.cg(T(vi), T(np.array([1.0, -1.0])), rtol=1e-12, strategy=strategy)
        _, io = O.pcg(rpi, cii, vi, np.array([1.0, -1.0]), rtol=1e-12)
        assert H(info.status)[0] == io.status[0] == L.SLA_BREAKDOWN
        assert H(info.iters)[0] == io.iters[0]
        _, info = Ai.cg(T(-vi), T(np.array([1.0, -1.0])), rtol=1e-12, strategy=strategy)
        assert H(info.status)[0] == L.SLA_BREAKDOWN and H(info.iters)[0] == 0


def test_single_unknown_and_empty_matrix():
    A = make(np.array([0, 1], np.int32), np.array([0], np.int32))
    x, info = A.cg(T(np.array([[4.0]])), T(np.array([[2.0]])), rtol=1e-12)
    assert H(x)[0, 0] == 0.5 and H(info.iters)[0] == 1
    E = sla.CSR(torch.zeros(1, dtype=torch.int32, device=DEV), torch.zeros(0, dtype=torch.int32, device=DEV),
                batch=2)
    x, info = E.cg(torch.zeros(2, 0, dtype=torch.float64, device=DEV),
                   torch.zeros(2, 0, dtype=torch.float64, device=DEV))
    assert x.shape == (2, 0) and np.all(H(info.status) == 0) and np.all(H(info.iters) == 0)


@pytest.mark.parametrize("onchip", ["1", "3", "0"])
def test_bounded_wait_times_out_without_hanging(onchip, monkeypatch):
    _variant_env(monkeypatch, onchip, "1")
    N = 1024                          # one tile a block: tile flags in place of a barrier
    rp, ci, v = W.poisson2d(N)
    A = make(rp, ci)
    b = T(W.normal(2, 0, N * N))
    _, info = A.cg(T(v), b, fixed_iters=500, strategy=L.SLA_STRATEGY_GRID, wait_timeout_ns=1)
    assert H(info.status)[0] == L.SLA_TIMED_OUT
    # the context is still usable and a normal solve is correct afterwards
    x, info = A.cg(T(v), b, fixed_iters=20, strategy=L.SLA_STRATEGY_GRID)
    xo, _ = O.pcg(rp, ci, v, W.normal(2, 0, N * N), fixed_iters=20)
    assert H(info.status)[0] == L.SLA_FIXED_DONE and rel(H(x)[0], xo) < TOL_X64


def test_cluster_bounded_wait_times_out_without_hanging():
    w = W.c1_poisson64()
    A = make(w.rowptr, w.colind)
    assert A.props.cluster_fits
    _, info = A.cg(T(w.values), T(w.b), fixed_iters=400, strategy=L.SLA_STRATEGY_CLUSTER,
                   wait_timeout_ns=1)
    assert H(info.status)[0] == L.SLA_TIMED_OUT
    x, info = A.cg(T(w.values), T(w.b), fixed_iters=20, strategy=L.SLA_STRATEGY_CLUSTER)
    xo, _ = O.pcg(w.rowptr, w.colind, w.values[0], w.b[0], fixed_iters=20)
    assert H(info.status)[0] == L.SLA_FIXED_DONE and rel(H(x)[0], xo) < TOL_X64


def test_auto_strategy_picks_cluster_for_a_small_single_system():
    w = W.c1_poisson64()
    A = make(w.rowptr, w.colind)
    x, info = A.cg(T(w.values), T(w.b), rtol=1e-10)
    xo, io = O.pcg(w.rowptr, w.colind, w.values[0], w.b[0], rtol=1e-10)
    assert abs(int(H(info.iters)[0]) - int(io.iters[0])) <= 2
    xk, _ = A.cg(T(w.values), T(w.b), fixed_iters=int(io.iters[0]), strategy=L.SLA_STRATEGY_CLUSTER)
    assert rel(H(xk)[0], xo) < TOL_X64
