"""Pins for the CPU oracle: each check ties an oracle function to something other than
itself (a printed test vector, a closed form, a library routine, brute force, an
invariant).  The `check_*` helpers take the function under test as an argument; the
mutation tests at the bottom feed them deliberately broken variants (on the CPU) to show
that a plausible mistake fails at least one pin.
"""

import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers

def rand_layer(rng, M, K, nnz, dtype="f32"):
    lin = rng.choice(M * K, size=nnz, replace=False)
    v = rng.normal(0, 1, size=nnz).astype(np.float32)
    if dtype == "bf16":
        v = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return (lin // K).astype(np.int32), (lin % K).astype(np.int32), v


def dense_of(M, K, row, col, v64):
    W = np.zeros((M, K))
    W[row, col] = v64
    return W


# ----------------------------------------------------------------------------- SplitMix64

def read_golden_sm64():
    vals, seed = [], None
    with open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("seed"):
                seed = int(line.split()[1])
            else:
                vals.append(int(line))
    return seed, vals


def test_splitmix64_published_vector():
    seed, vals = read_golden_sm64()
    got = [int(x) for x in oracle.splitmix64(seed, len(vals))]
    assert got == vals


def test_splitmix64_is_counter_based():
    # output i depends only on seed + (i+1)*gamma: shifting the seed by gamma shifts the stream
    gamma = 0x9E3779B97F4A7C15
    a = oracle.splitmix64(12345, 20)
    b = oracle.splitmix64((12345 + gamma) % 2**64, 19)
    assert np.array_equal(a[1:], b)


def test_regrow_position_map_power_of_two():
    # closed form: for M*K = 2^b the multiply-shift map is the top b bits of the draw.
    # On a 2 x 2 grid holding position 0, the accepted draw is the first whose top two
    # bits are nonzero, and every earlier draw has top bits 0.
    M, K = 2, 2
    row = np.array([0], np.int32); col = np.array([0], np.int32)
    v = np.array([1.0], np.float32)
    out = oracle.restructure(M, K, row, col, v, k=1, seed=7)
    draws = oracle.splitmix64(7, out["draws"])
    tops = [int(d) >> 62 for d in draws]
    # the last draw is the accepted one; earlier draws hit position 0 (in S) or repeat
    accepted = tops[-1]
    assert accepted != 0 and all(t == 0 for t in tops[:-1])
    new_lin = set((out["row"].astype(int) * K + out["col"]).tolist())
    assert accepted in new_lin


# ----------------------------------------------------------------------------- O1-O4

def check_build(build_fn, M, K, row, col, vals, P):
    out = build_fn(M, K, row, col, vals, P)
    nnz = row.size
    # O1: unique sorted order by brute force (Python's sort on tuples)
    triples = sorted(zip(row.tolist(), col.tolist(), range(nnz)))
    assert out["row"].tolist() == [t[0] for t in triples]
    assert out["col"].tolist() == [t[1] for t in triples]
    assert out["values"].tobytes() == vals[[t[2] for t in triples]].tobytes()
    # O2: counting
    rp = out["row_ptr"]
    assert rp.tolist() == [sum(1 for r in row.tolist() if r < q) for q in range(M + 1)]
    # O3: perm is a permutation in (col, row) order; csc_row and col_ptr follow
    perm = out["perm"]
    assert sorted(perm.tolist()) == list(range(nnz))
    keys = [(out["col"][j], out["row"][j]) for j in perm.tolist()]
    assert keys == sorted(keys)
    assert out["csc_row"].tolist() == [out["row"][j] for j in perm.tolist()]
    assert out["col_ptr"].tolist() == [sum(1 for c in col.tolist() if c < q) for q in range(K + 1)]
    # O4: part sizes differ by <= 1, cover [0, nnz), part_row = row holding the first entry
    Pe = out["num_parts"]
    assert Pe == min(P, max(nnz, 1))
    for pn, pidx, ptr, dim in ((out["part_nnz"], out["part_row"], rp, M),
                               (out["part_nnz_t"], out["part_col"], out["col_ptr"], K)):
        assert pn[0] == 0 and pn[-1] == nnz and len(pn) == Pe + 1
        sizes = np.diff(pn)
        assert sizes.min() >= (0 if nnz == 0 else 1) and sizes.max() - sizes.min() <= 1
        for p in range(Pe + 1):
            a = int(pn[p])
            if a == nnz:
                assert pidx[p] == dim
            else:
                r = int(pidx[p])
                assert ptr[r] <= a < ptr[r + 1]
    return out


def test_build_exhaustive_2x3():
    rng = np.random.default_rng(1)
    M, K = 2, 3
    for mask in range(1 << (M * K)):
        lin = np.array([i for i in range(M * K) if mask >> i & 1], np.int64)
        lin = lin[rng.permutation(lin.size)]
        row, col = (lin // K).astype(np.int32), (lin % K).astype(np.int32)
        vals = rng.normal(size=lin.size).astype(np.float32)
        for P in (1, 2, 3, 7):
            check_build(oracle.build, M, K, row, col, vals, P)


@pytest.mark.parametrize("seed", range(6))
def test_build_random_small(seed):
    rng = np.random.default_rng(100 + seed)
    M, K = rng.integers(1, 9, size=2)
    nnz = int(rng.integers(0, M * K + 1))
    row, col, v = rand_layer(rng, M, K, nnz, "bf16" if seed % 2 else "f32")
    for P in (1, 3, 16):
        check_build(oracle.build, int(M), int(K), row, col, v, P)


def test_build_errors():
    r = np.array([0, 1], np.int32); c = np.array([0, 3], np.int32); v = np.zeros(2, np.float32)
    with pytest.raises(oracle.OracleError) as e:
        oracle.build(2, 3, r, c, v, 1)
    assert e.value.status == "OUT_OF_RANGE"
    with pytest.raises(oracle.OracleError) as e:
        oracle.build(2, 3, np.array([1, 1], np.int32), np.array([2, 2], np.int32), v, 1)
    assert e.value.status == "DUPLICATE"
    with pytest.raises(oracle.OracleError) as e:
        oracle.build(2, 3, np.array([-1], np.int32), np.array([0], np.int32), v[:1], 1)
    assert e.value.status == "OUT_OF_RANGE"


# ----------------------------------------------------------------------------- O5-O7

def check_products(fwd, bwi, bww, M, K, row, col, v64, X, dY, rng):
    W = dense_of(M, K, row, col, v64)
    Y, A = fwd(M, K, row, col, v64, X)
    # dense fp64 matmul of the scattered W (numpy), and the absolute-term sums
    assert np.allclose(Y, W @ X, rtol=1e-12, atol=1e-12)
    assert np.allclose(A, np.abs(W) @ np.abs(X), rtol=1e-12, atol=1e-12)
    dX, AX = bwi(M, K, row, col, v64, dY)
    assert np.allclose(dX, W.T @ dY, rtol=1e-12, atol=1e-12)
    assert np.allclose(AX, np.abs(W).T @ np.abs(dY), rtol=1e-12, atol=1e-12)
    dW, AW = bww(row, col, dY, X)
    G = dY @ X.T
    assert np.allclose(dW, G[row, col], rtol=1e-12, atol=1e-12)
    assert np.allclose(AW, (np.abs(dY) @ np.abs(X).T)[row, col], rtol=1e-12, atol=1e-12)
    # adjoint identity <W X, dY> = <X, W^T dY>
    lhs, rhs = np.sum(Y * dY), np.sum(X * dX)
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, np.sum(np.abs(Y * dY)))
    # gradient identity sum_e dW_e v_e = <W X, dY>
    assert abs(np.dot(dW, v64) - lhs) <= 1e-12 * max(1.0, np.sum(np.abs(Y * dY)))
    # linearity in X and in the values
    X2 = rng.normal(size=X.shape)
    Ya, _ = fwd(M, K, row, col, v64, 2.0 * X + X2)
    Yb, _ = fwd(M, K, row, col, v64, X2)
    assert np.allclose(Ya, 2.0 * Y + Yb, rtol=1e-10, atol=1e-10)
    v2 = rng.normal(size=v64.shape)
    Yc, _ = fwd(M, K, row, col, v64 + v2, X)
    Yd, _ = fwd(M, K, row, col, v2, X)
    assert np.allclose(Yc, Y + Yd, rtol=1e-10, atol=1e-10)
    # central finite differences of L = <W X, dY> w.r.t. each value and some X entries
    h = 1e-6
    for e in range(min(row.size, 5)):
        vp = v64.copy(); vp[e] += h
        vm = v64.copy(); vm[e] -= h
        fd = (np.sum(fwd(M, K, row, col, vp, X)[0] * dY) - np.sum(fwd(M, K, row, col, vm, X)[0] * dY)) / (2 * h)
        assert abs(fd - dW[e]) <= 1e-5 * max(1.0, abs(dW[e]))
    for (c, n) in [(0, 0), (K - 1, X.shape[1] - 1)]:
        Xp = X.copy(); Xp[c, n] += h
        Xm = X.copy(); Xm[c, n] -= h
        fd = (np.sum(fwd(M, K, row, col, v64, Xp)[0] * dY) - np.sum(fwd(M, K, row, col, v64, Xm)[0] * dY)) / (2 * h)
        assert abs(fd - dX[c, n]) <= 1e-5 * max(1.0, abs(dX[c, n]))


@pytest.mark.parametrize("seed", range(5))
def test_products_random(seed):
    rng = np.random.default_rng(200 + seed)
    M, K, N = (int(x) for x in rng.integers(1, 12, size=3))
    nnz = int(rng.integers(0, M * K + 1))
    row, col, v = rand_layer(rng, M, K, nnz)
    v64 = oracle.widen(v)
    X = rng.normal(size=(K, N)); dY = rng.normal(size=(M, N))
    check_products(oracle.forward, oracle.backward_input, oracle.backward_weight,
                   M, K, row, col, v64, X, dY, rng)


def test_identity_and_permutation_exact():
    rng = np.random.default_rng(3)
    n, N = 37, 5
    X = rng.normal(size=(n, N))
    eye = np.arange(n, dtype=np.int32)
    Y, A = oracle.forward(n, n, eye, eye, np.ones(n), X)
    assert np.array_equal(Y, X) and np.array_equal(A, np.abs(X))
    p = rng.permutation(n).astype(np.int32)
    Y, _ = oracle.forward(n, n, eye, p, np.ones(n), X)  # Y[r] = X[p[r]]
    assert np.array_equal(Y, X[p])
    dX, _ = oracle.backward_input(n, n, eye, p, np.ones(n), X)  # dX[p[r]] = X[r]
    expect = np.empty_like(X); expect[p] = X
    assert np.array_equal(dX, expect)
    dW, _ = oracle.backward_weight(eye, p, X, X)
    assert np.array_equal(dW, np.sum(X * X[p], axis=1))


def test_empty_rows_and_columns_are_zero():
    M, K, N = 6, 5, 3
    row = np.array([1, 1, 4], np.int32); col = np.array([0, 3, 3], np.int32)
    X = np.ones((K, N)); dY = np.ones((M, N))
    Y, A = oracle.forward(M, K, row, col, np.array([1.0, 2.0, 3.0]), X)
    assert np.all(Y[[0, 2, 3, 5]] == 0) and np.all(A[[0, 2, 3, 5]] == 0)
    dX, AX = oracle.backward_input(M, K, row, col, np.array([1.0, 2.0, 3.0]), dY)
    assert np.all(dX[[1, 2, 4]] == 0) and np.allclose(dX[3], 5.0)


# ----------------------------------------------------------------------------- O8

def check_restructure(rs_fn, M, K, row, col, vals, k, seed, regrow=0.0):
    """Invariants plus re-derivation of the drop set (numpy lexsort) and of the accepted
    regrowth (sequential walk over the pinned SplitMix64 stream)."""
    b = oracle.build(M, K, row, col, vals, 1)
    srow, scol, svals = b["row"], b["col"], b["values"]
    out = rs_fn(M, K, srow, scol, svals, k, seed, regrow)
    nnz = srow.size
    lin_old = srow.astype(np.int64) * K + scol
    mag = np.abs(oracle.widen(svals))
    order = np.lexsort((lin_old, mag))
    drop = set(order[:k].tolist())
    S = set(lin_old.tolist())
    # accepted regrowth by a plain sequential walk
    draws = oracle.splitmix64(seed, out["draws"])
    acc, seen = [], set()
    for u in draws.tolist():
        c = (u * (M * K)) >> 64
        if c in S or c in seen:
            continue
        seen.add(c)
        acc.append(c)
        if len(acc) == k:
            break
    assert len(acc) == k
    new_lin = out["row"].astype(np.int64) * K + out["col"]
    assert new_lin.size == nnz
    assert np.all(np.diff(new_lin) > 0)  # sorted, no duplicates
    survivors = [e for e in range(nnz) if e not in drop]
    assert set(new_lin.tolist()) == {int(lin_old[e]) for e in survivors} | set(acc)
    o2n = out["old_to_new"]
    for e in range(nnz):
        if e in drop:
            assert o2n[e] == -1
        else:
            j = int(o2n[e])
            assert new_lin[j] == lin_old[e]
            assert out["values"][j:j + 1].tobytes() == svals[e:e + 1].tobytes()
    # regrown values: regrow rounded to the value type by torch (a library conversion)
    rv = torch.tensor([regrow], dtype=torch.float32)
    if svals.dtype == np.uint16:
        rv_bits = rv.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    else:
        rv_bits = rv.numpy()
    grown_idx = [j for j in range(nnz) if int(new_lin[j]) in set(acc)]
    for j in grown_idx:
        assert out["values"][j:j + 1].tobytes() == rv_bits.tobytes()
    return out


@pytest.mark.parametrize("seed", range(6))
def test_restructure_random(seed):
    rng = np.random.default_rng(300 + seed)
    M, K = (int(x) for x in rng.integers(2, 10, size=2))
    nnz = int(rng.integers(1, M * K // 2 + 1))
    row, col, v = rand_layer(rng, M, K, nnz, "bf16" if seed % 2 else "f32")
    k = int(rng.integers(0, nnz + 1))
    k = min(k, M * K - nnz)
    check_restructure(oracle.restructure, M, K, row, col, v, k, seed=seed * 7919, regrow=1.0 / 3.0)


def test_restructure_ties_and_signed_zero():
    # equal magnitudes (+0 and -0, +x and -x): the lower linear index goes first
    M, K = 3, 4
    row = np.array([0, 0, 1, 2, 2], np.int32); col = np.array([1, 3, 0, 2, 3], np.int32)
    v = np.array([-0.0, 0.0, 0.5, -0.5, 2.0], np.float32)
    out = check_restructure(oracle.restructure, M, K, row, col, v, 3, seed=11)
    assert out["old_to_new"][:3].tolist() == [-1, -1, -1]  # (0,1), (0,3), (1,0) dropped
    out = check_restructure(oracle.restructure, M, K, row, col, v, 4, seed=11)
    assert out["old_to_new"][3] == -1 and out["old_to_new"][4] >= 0


def test_restructure_fills_complement_exactly():
    # M*K - nnz == k: the regrown set must be the whole complement (closed form)
    rng = np.random.default_rng(5)
    M, K = 4, 5
    row, col, v = rand_layer(rng, M, K, 12)
    k = M * K - 12
    out = check_restructure(oracle.restructure, M, K, row, col, v, k, seed=3)
    b = oracle.build(M, K, row, col, v, 1)
    old = set((b["row"].astype(int) * K + b["col"]).tolist())
    new = set((out["row"].astype(int) * K + out["col"]).tolist())
    dropped = {int(b["row"][e]) * K + int(b["col"][e]) for e in range(12) if out["old_to_new"][e] < 0}
    assert new == (set(range(M * K)) - old) | (old - dropped)


def test_restructure_k0_is_identity_and_errors():
    rng = np.random.default_rng(9)
    row, col, v = rand_layer(rng, 5, 6, 10)
    b = oracle.build(5, 6, row, col, v, 1)
    out = oracle.restructure(5, 6, b["row"], b["col"], b["values"], 0, 1)
    assert np.array_equal(out["row"], b["row"]) and np.array_equal(out["col"], b["col"])
    assert out["values"].tobytes() == b["values"].tobytes()
    assert out["old_to_new"].tolist() == list(range(10))
    with pytest.raises(oracle.OracleError) as e:
        oracle.restructure(5, 6, b["row"], b["col"], b["values"], 11, 1)
    assert e.value.status == "INVALID_ARG"  # k > nnz
    r2, c2, v2 = rand_layer(rng, 5, 6, 20)
    b2 = oracle.build(5, 6, r2, c2, v2, 1)
    with pytest.raises(oracle.OracleError) as e:
        oracle.restructure(5, 6, b2["row"], b2["col"], b2["values"], 11, 1)
    assert e.value.status == "NO_ROOM"  # k > M*K - nnz
    bad = b["values"].copy(); bad[3] = np.nan
    with pytest.raises(oracle.OracleError) as e:
        oracle.restructure(5, 6, b["row"], b["col"], bad, 1, 1)
    assert e.value.status == "INVALID_VALUE"


# ----------------------------------------------------------------------------- tolerance metric

def test_normalized_error_metric():
    ref = np.array([1.0, -1.0, 0.0, 3.0]); A = np.array([1.0, 2.0, 0.0, 3.0])
    assert oracle.normalized_error(ref, ref, A) == 0.0
    assert oracle.normalized_error(ref + np.array([0, 0.02, 0, 0]), ref, A) == pytest.approx(0.01)
    assert oracle.normalized_error(ref + np.array([0, 0, 1e-30, 0]), ref, A) == float("inf")


# ----------------------------------------------------------------------------- mutation checks

def _mut_forward_transposed(M, K, row, col, v, X):
    # a swapped row/col index: W^T-like gather (only valid shapes when M == K)
    return oracle.forward(M, K, col, row, v, X)


def _mut_forward_drop_last(M, K, row, col, v, X):
    return oracle.forward(M, K, row[:-1], col[:-1], v[:-1], X)


def _mut_bwi_sign(M, K, row, col, v, dY):
    dX, A = oracle.backward_input(M, K, row, col, v, dY)
    return -dX, A


def _mut_bww_shift(row, col, dY, X):
    dW, A = oracle.backward_weight(row, col, dY, X)
    return np.roll(dW, 1), A


@pytest.mark.parametrize("mut", ["fwd_T", "fwd_drop", "bwi_sign", "bww_shift"])
def test_pins_catch_planted_product_mistakes(mut):
    rng = np.random.default_rng(77)
    M = K = 7
    N = 3
    row, col, v = rand_layer(rng, M, K, 20)
    v64 = oracle.widen(v)
    X = rng.normal(size=(K, N)); dY = rng.normal(size=(M, N))
    fwd, bwi, bww = oracle.forward, oracle.backward_input, oracle.backward_weight
    if mut == "fwd_T":
        fwd = _mut_forward_transposed
    elif mut == "fwd_drop":
        fwd = _mut_forward_drop_last
    elif mut == "bwi_sign":
        bwi = _mut_bwi_sign
    else:
        bww = _mut_bww_shift
    with pytest.raises(AssertionError):
        check_products(fwd, bwi, bww, M, K, row, col, v64, X, dY, rng)


def test_pins_catch_planted_build_and_restructure_mistakes():
    rng = np.random.default_rng(78)
    M, K = 5, 7
    row, col, v = rand_layer(rng, M, K, 15)

    def build_unstable(M, K, r, c, vals, P):
        out = oracle.build(M, K, r, c, vals, P)
        out["values"] = out["values"][::-1].copy()  # values no longer follow their entries
        return out

    def build_bad_parts(M, K, r, c, vals, P):
        out = oracle.build(M, K, r, c, vals, P)
        out["part_row"] = np.maximum(out["part_row"] - 1, 0)
        return out

    def rs_keep_largest(M, K, r, c, vals, k, seed, regrow):
        # drops the largest magnitudes instead of the smallest
        return oracle.restructure(M, K, r, c, (-np.abs(oracle.widen(vals)) - 1).astype(np.float32)
                                  if vals.dtype == np.float32 else vals, k, seed, regrow)

    with pytest.raises(AssertionError):
        check_build(build_unstable, M, K, row, col, v, 3)
    with pytest.raises(AssertionError):
        check_build(build_bad_parts, M, K, row, col, v, 4)
    with pytest.raises(AssertionError):
        check_restructure(rs_keep_largest, M, K, row, col, v, 5, seed=1)
