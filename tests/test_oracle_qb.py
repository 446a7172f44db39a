"""Pins for the oracle's optimal-assignment balancing (QB + exact finish).

Fixed by: brute-force enumeration on tiny instances, scipy's HiGHS LP solver on
the relaxation (integral by the max-min argument), scipy's Hungarian solver
for k = 1, the closed-form minimum of each dual sub-problem, the constraint
sums, and the demo's qualitative claim that the bias evens the load.
Source: "MoE travelogue 6: optimal assignment promotes balance"
(kexue.fm/archives/11619): Linear programming eqs. (3)-(4), Max-min (7),
Divide and conquer (8)-(11), Alternating iteration, Mind the pitfall, Demo code.
"""
import itertools

import numpy as np
import pytest
from scipy.optimize import linear_sum_assignment, linprog

import oracle
import workloads as W


def _objective(s, idx):
    return float(np.take_along_axis(s.astype(np.float64), idx.astype(np.int64), 1).sum())


def _brute(s, k):
    """Best objective and every optimal assignment (as frozensets per token) by enumeration."""
    m, n = s.shape
    C = m * k // n
    combos = list(itertools.combinations(range(n), k))
    best, arg = -np.inf, []
    for choice in itertools.product(combos, repeat=m):
        cnt = np.zeros(n, int)
        for ch in choice:
            cnt[list(ch)] += 1
        if (cnt != C).any():
            continue
        v = sum(float(s[i, list(ch)].astype(np.float64).sum()) for i, ch in enumerate(choice))
        if v > best + 1e-12:
            best, arg = v, [choice]
        elif abs(v - best) <= 1e-12:
            arg.append(choice)
    return best, arg


def _lp(s, k):
    m, n = s.shape
    C = m * k // n
    A = np.zeros((m + n, m * n))
    for i in range(m):
        A[i, i * n:(i + 1) * n] = 1
    for j in range(n):
        A[m + j, j::n] = 1
    r = linprog(-s.astype(np.float64).ravel(), A_eq=A, b_eq=[k] * m + [C] * n, bounds=(0, 1), method="highs")
    assert r.status == 0
    return -r.fun, r.x.reshape(m, n)


def _check_balanced(idx, m, n, k):
    assert idx.shape == (m, k)
    for row in idx:
        assert len(set(row.tolist())) == k and (np.diff(row) > 0).all()
    assert (np.bincount(idx.ravel(), minlength=n) == m * k // n).all()


@pytest.mark.parametrize("case", range(30))
def test_bruteforce_tiny(case):
    shapes = [(8, 4, 1), (6, 3, 1), (6, 4, 2), (4, 4, 2), (8, 2, 1), (6, 3, 2)]
    m, n, k = shapes[case % len(shapes)]
    rng = np.random.default_rng(100 + case)
    s = (rng.standard_normal((m, n)) + 1.5 * rng.standard_normal(n)).astype(np.float32)
    for rule in (oracle.QB_MIDPOINT, oracle.QB_BOUNDARY):
        idx, _, info, rc = oracle.balance_assign(s, k, mode=oracle.QB_SOLVE, rule=rule, max_iters=case % 4)
        assert rc == oracle.OK and info[2] == 0
        _check_balanced(idx, m, n, k)
        best, arg = _brute(s, k)
        assert _objective(s, idx) == pytest.approx(best, abs=1e-9)
        if len(arg) == 1:
            assert [set(r.tolist()) for r in idx] == [set(c) for c in arg[0]]


@pytest.mark.parametrize("m,n,k,iters,seed", [(512, 16, 2, 0, 0), (512, 16, 2, 5, 1), (1024, 8, 1, 3, 2),
                                              (768, 32, 4, 10, 3), (600, 12, 3, 2, 4)])
def test_lp_medium(m, n, k, iters, seed):
    s = W.make_qb_scores(m, n, seed=seed)
    idx, _, info, rc = oracle.balance_assign(s, k, max_iters=iters)
    assert rc == oracle.OK and info[2] == 0
    _check_balanced(idx, m, n, k)
    obj, x = _lp(s, k)
    assert _objective(s, idx) == pytest.approx(obj, rel=1e-12, abs=1e-7)
    # continuous random scores: the LP optimum is a unique 0/1 vertex, equal to ours
    assert np.allclose(x, np.round(x), atol=1e-7)
    ours = np.zeros((m, n))
    np.put_along_axis(ours, idx.astype(np.int64), 1.0, 1)
    assert (ours == np.round(x)).all()
    assert oracle.is_optimal(s, idx)


@pytest.mark.parametrize("m,n,k,seed", [(64, 8, 2, 0), (96, 6, 2, 1), (128, 8, 3, 2), (48, 4, 1, 3), (64, 8, 2, 4)])
def test_solve_with_zero_cost_cycles(m, n, k, seed):
    # half-integer scores with every third row constant: many tokens swap two experts at the same
    # cost, so the expert graph has zero-cost cycles and several arcs into an expert are tight.
    # The exact finish must still follow a path back to an over-full expert (predecessors settled
    # in an earlier Bellman-Ford round) and reach the LP optimum.
    s = (np.round(np.random.default_rng(seed).standard_normal((m, n)) * 2) / 2).astype(np.float32)
    s[::3] = np.float32(0.5)
    idx, _, info, rc = oracle.balance_assign(s, k, max_iters=3)
    assert rc == oracle.OK and info[2] == 0 and info[1] > 0
    _check_balanced(idx, m, n, k)
    obj, _ = _lp(s, k)
    assert _objective(s, idx) == pytest.approx(obj, rel=1e-12, abs=1e-9)
    assert oracle.is_optimal(s, idx)


def test_hungarian_k1():
    m, n = 120, 6
    s = W.make_qb_scores(m, n, seed=7)
    idx, _, info, rc = oracle.balance_assign(s, 1, max_iters=1)
    _check_balanced(idx, m, n, 1)
    C = m // n
    cost = -np.repeat(s.astype(np.float64), C, axis=1)  # each expert column repeated C times
    r, c = linear_sum_assignment(cost)
    assert _objective(s, idx) == pytest.approx(-cost[r, c].sum(), rel=1e-12)
    assert (idx[r, 0] == c // C).all()


def test_dual_subproblem_minima_closed_form():
    # eqs. (10)-(11): min over alpha of k*alpha + sum_j max(0, v_j - alpha) is the sum of the k largest v_j,
    # attained anywhere between the k-th and (k+1)-th largest -- both rules pick such a point.
    m, n, k = 64, 16, 3
    s = W.make_qb_scores(m, n, seed=9)
    beta = np.random.default_rng(1).standard_normal(n).astype(np.float32)
    v = (s - beta[None, :]).astype(np.float32)
    for rule in (oracle.QB_MIDPOINT, oracle.QB_BOUNDARY):
        alpha, idx, _ = oracle.qb_row(s, k, beta, rule)
        vs = -np.sort(-v.astype(np.float64), axis=1)
        g = k * alpha.astype(np.float64) + np.maximum(0, v.astype(np.float64) - alpha[:, None]).sum(1)
        assert np.allclose(g, vs[:, :k].sum(1), rtol=1e-12, atol=1e-9)
        assert ((alpha >= vs[:, k]) & (alpha <= vs[:, k - 1])).all()
        if rule == oracle.QB_BOUNDARY:
            assert (alpha == vs[:, k]).all()  # the page's convention: the (k+1)-th largest
        # the selection is the top-k of s - beta (ties to the lower index), listed best first
        for i in range(m):
            assert idx[i].tolist() == sorted(range(n), key=lambda j: (-v[i, j], j))[:k]
    C = m * k // n
    alpha, _, _ = oracle.qb_row(s, k, beta)
    u = (s - alpha[:, None]).astype(np.float32).astype(np.float64)
    for rule in (oracle.QB_MIDPOINT, oracle.QB_BOUNDARY):
        b = oracle.qb_col(s, k, alpha, rule).astype(np.float64)
        us = -np.sort(-u, axis=0)
        g = C * b + np.maximum(0, u - b[None, :]).sum(0)
        assert np.allclose(g, us[:C].sum(0), rtol=1e-12, atol=1e-9)
        assert ((b >= us[C]) & (b <= us[C - 1])).all()


def test_midpoint_value_is_fp32_mean_of_neighbours():
    s = np.array([[4.0, 1.0, 3.0, 2.0]], np.float32)
    alpha, idx, _ = oracle.qb_row(s, 2, np.zeros(4, np.float32), oracle.QB_MIDPOINT)
    assert alpha[0] == np.float32(2.5) and idx.tolist() == [[0, 2]]
    alpha_b, _, _ = oracle.qb_row(s, 2, np.zeros(4, np.float32), oracle.QB_BOUNDARY)
    assert alpha_b[0] == np.float32(2.0)


def test_step_mode_selects_with_old_beta():
    # Mind the pitfall: x comes from the old beta; beta is updated afterwards.
    m, n, k = 256, 16, 2
    s = W.make_qb_scores(m, n, seed=11)
    beta_old = np.random.default_rng(2).standard_normal(n).astype(np.float32) * np.float32(0.5)
    idx, beta_new, info, rc = oracle.balance_assign(s, k, beta=beta_old, mode=oracle.QB_STEP)
    alpha, sel, _ = oracle.qb_row(s, k, beta_old)
    assert (np.sort(sel, axis=1) == idx).all()
    assert (oracle.qb_col(s, k, alpha) == beta_new).all()
    assert info[0] == 1 and info[1] == 0


def test_solve_balances_and_repair_optimal_on_skewed_scores():
    m, n, k = 2048, 32, 4
    s = W.make_qb_scores(m, n, seed=0)
    _, idx0, _ = oracle.qb_row(s, k, np.zeros(n, np.float32))
    before = np.bincount(idx0.ravel(), minlength=n)
    idx, beta, info, rc = oracle.balance_assign(s, k, max_iters=8)
    assert rc == oracle.OK
    _check_balanced(idx, m, n, k)
    assert before.max() > m * k // n  # plain top-k was unbalanced
    assert oracle.is_optimal(s, idx)
    # repair alone from plain top-k reaches the same optimum
    idx_r, _, info_r, _ = oracle.balance_assign(s, k, max_iters=0)
    assert info_r[1] > 0 and (idx_r == idx).all()


def test_certificate_rejects_a_worse_assignment():
    m, n, k = 256, 8, 2
    s = W.make_qb_scores(m, n, seed=5)
    idx, _, _, _ = oracle.balance_assign(s, k)
    assert oracle.is_optimal(s, idx)
    # swap: token a trades expert p for q and token b trades q for p (counts unchanged) -> a worse objective
    bad = idx.copy()
    for a in range(m):
        for b in range(a + 1, m):
            p = [e for e in bad[a] if e not in bad[b]]
            q = [e for e in bad[b] if e not in bad[a]]
            if p and q:
                pa, qb = p[0], q[0]
                gain = s[a, qb] + s[b, pa] - s[a, pa] - s[b, qb]
                if gain < -1e-3:
                    bad[a][bad[a] == pa] = qb
                    bad[b][bad[b] == qb] = pa
                    break
        else:
            continue
        break
    bad.sort(axis=1)
    assert (np.bincount(bad.ravel(), minlength=n) == m * k // n).all()
    assert _objective(s, bad) < _objective(s, idx)
    assert not oracle.is_optimal(s, bad)


def test_demo_claim_bias_evens_the_load():
    # Demo code: scores rand(m,n) + rand(n); the top-k after subtracting the QB bias is far more even.
    rng = np.random.default_rng(0)
    m, n, k = 20000, 64, 8
    s = (rng.random((m, n)) + rng.random(n)).astype(np.float32)
    _, i0, _ = oracle.qb_row(s, k, np.zeros(n, np.float32))
    v0 = oracle.balance_stats(None, i0, m, n, k, m)["vio"]
    _, beta, _, _ = oracle.balance_assign(s, k, mode=oracle.QB_SOLVE, max_iters=5, max_repair=0, check=False)
    _, i1, _ = oracle.qb_row(s, k, beta)
    v1 = oracle.balance_stats(None, i1, m, n, k, m)["vio"]
    assert v0[0] > 1.0 and v1[0] < 0.1 * v0[0]


def test_argument_errors():
    s = W.make_qb_scores(10, 4, seed=0)
    with pytest.raises(oracle.OracleError):
        oracle.balance_assign(s, 1)  # m*k = 10 not divisible by n = 4
    with pytest.raises(oracle.OracleError):
        oracle.balance_assign(W.make_qb_scores(8, 4), 4)  # k must be < n


# ---------------------------------------------------------------- balancing variants
# "MoE travelogue 6", Related work (BIP: inequality constraints, duals clipped at zero) and
# Gradient descent (SignSGD on beta, eqs. (15)-(17)).

def test_bip_hand_example():
    # m=4, n=2, k=1, C=2. Tokens 0, 1 prefer expert 0; tokens 2, 3 prefer expert 1.
    # All scores negative: alpha_i = max(0, 2nd value) = 0, u = s, and each column's 3rd largest
    # value is negative, so beta = max(0, .) = 0 for both experts.
    s = np.array([[3, 1], [2, 0], [1, 4], [0, 5]], np.float32) - 10
    alpha, idx, _ = oracle.qb_row(s, 1, np.zeros(2, np.float32), rule=oracle.QB_BIP)
    assert (alpha == 0).all() and idx[:, 0].tolist() == [0, 0, 1, 1]
    assert (oracle.qb_col(s, 1, alpha, rule=oracle.QB_BIP) == 0).all()
    # shifted up by 20 (scores [[13, 11], [12, 10], [11, 14], [10, 15]]) the clip is inactive on
    # alpha: the 2nd values 11, 10, 11, 10; column 0 of s - alpha is [2, 2, 0, 0] and column 1 is
    # [0, 0, 3, 5]: both 3rd largest values are 0
    alpha, _, _ = oracle.qb_row(s + 20, 1, np.zeros(2, np.float32), rule=oracle.QB_BIP)
    assert alpha.tolist() == [11, 10, 11, 10]
    assert oracle.qb_col(s + 20, 1, alpha, rule=oracle.QB_BIP).tolist() == [0.0, 0.0]


def test_bip_equals_boundary_when_thresholds_are_positive():
    # the clip max(0, .) only acts on negative thresholds: where the (k+1)-th / (C+1)-th values
    # are positive (scores far above zero, alpha = 0 for the column pass) BIP is the page's
    # boundary rule exactly; where they are negative it returns 0
    s = W.make_qb_scores(2048, 16, seed=3) + np.float32(50)
    b0 = np.zeros(16, np.float32)
    a_b, i_b, _ = oracle.qb_row(s, 2, b0, rule=oracle.QB_BOUNDARY)
    a_p, i_p, _ = oracle.qb_row(s, 2, b0, rule=oracle.QB_BIP)
    assert (a_b > 0).all() and (a_b == a_p).all() and (i_b == i_p).all()
    zero = np.zeros(2048, np.float32)
    beta_b = oracle.qb_col(s, 2, zero, rule=oracle.QB_BOUNDARY)
    assert (beta_b > 0).all() and (oracle.qb_col(s, 2, zero, rule=oracle.QB_BIP) == beta_b).all()
    assert (oracle.qb_col(s - 100, 2, zero, rule=oracle.QB_BIP) == 0).all()
    assert (oracle.qb_row(s - 100, 2, b0, rule=oracle.QB_BIP)[0] == 0).all()


def test_bip_duals_never_negative():
    s = W.make_qb_scores(3000, 24, seed=5) - np.float32(1.0)
    beta = np.zeros(24, np.float32)
    for _ in range(4):
        _, beta, _, _ = oracle.balance_assign(s, 3, beta=beta, mode=oracle.QB_STEP, rule=oracle.QB_BIP)
        assert (beta >= 0).all()
        alpha, _, _ = oracle.qb_row(s, 3, beta, rule=oracle.QB_BIP)
        assert (alpha >= 0).all()


def test_sign_step_hand_example():
    # m=4, n=2, k=1, C=2: tokens 0-2 prefer expert 0 (s = [1, 0]), token 3 expert 1 (s = [0, 1]).
    # MIDPOINT alpha_i = 0.5 for every token. count_0 = #{s_i0 - 0.5 > 0} = 3 > C: the gradient
    # C - 3 < 0, so beta_0 rises by gamma; count_1 = 1 < C: beta_1 falls by gamma.
    s = np.array([[1, 0], [1, 0], [1, 0], [0, 1]], np.float32)
    idx, beta, info = oracle.qb_sign_step(s, 1, np.zeros(2, np.float32), 0.125)
    assert idx[:, 0].tolist() == [0, 0, 0, 1]
    assert beta.tolist() == [0.125, -0.125]
    assert info.tolist() == [1, 0, 1, 0]  # one update, no repair, excess 1, no ties
    # balanced selection: both counts equal C, sign(0) = 0, beta unchanged
    s2 = np.array([[1, 0], [1, 0], [0, 1], [0, 1]], np.float32)
    _, beta2, info2 = oracle.qb_sign_step(s2, 1, np.array([0.25, -0.5], np.float32), 0.125)
    assert beta2.tolist() == [0.25, -0.5] and info2[2] == 0


def test_sign_steps_shrink_the_violation():
    # repeated SignSGD steps move load from the crowded experts to the empty ones (the page puts
    # its effect between Loss-Free and QB)
    m, n, k = 4096, 16, 2
    s = W.make_qb_scores(m, n, seed=7, skew_std=1.0)
    beta = np.zeros(n, np.float32)
    idx0, _, _ = oracle.qb_sign_step(s, k, beta, 0.0)
    v0 = oracle.balance_stats(None, idx0, m, n, k, m)["vio"][0]
    for _ in range(60):
        idx, beta, _ = oracle.qb_sign_step(s, k, beta, 0.05)
    v1 = oracle.balance_stats(None, idx, m, n, k, m)["vio"][0]
    assert v1 < 0.5 * v0


def test_sign_step_with_zero_gamma_is_plain_topk():
    s = W.make_qb_scores(512, 8, seed=2)
    beta = np.linspace(-0.3, 0.3, 8).astype(np.float32)
    idx, beta_out, _ = oracle.qb_sign_step(s, 2, beta, 0.0)
    assert (beta_out == beta).all()
    _, ref, _ = oracle.qb_row(s, 2, beta)
    assert (np.sort(ref, axis=1) == idx).all()


# ---------------------------------------------------------------- mini-batch beta ("Mind the pitfall")
def test_minibatch_step_hand_example():
    # m=4, n=2, k=1, two mini-batches of 2 tokens (C_b = 1), beta_old = 0.
    # row pass: picks [0, 0, 1, 1]; alpha = mid of the two values = [2, 1, 1, 3].
    # batch 0 (tokens 0, 1): u_0 = [3-2, 2-1] = [1, 1] -> beta = mid(1, 1) = 1;
    #                        u_1 = [1-2, 0-1] = [-1, -1] -> -1.
    # batch 1 (tokens 2, 3): u_0 = [0-1, 1-3] = [-1, -2] -> mid = -1.5; u_1 = [2-1, 5-3] = [1, 2] -> 1.5.
    # average: beta = [(1 - 1.5) / 2, (-1 + 1.5) / 2] = [-0.25, 0.25].
    s = np.array([[3, 1], [2, 0], [0, 2], [1, 5]], np.float32)
    idx, beta, info = oracle.balance_step_minibatch(s, 1, np.zeros(2, np.float32), 2)
    assert idx[:, 0].tolist() == [0, 0, 1, 1]
    assert beta.tolist() == [-0.25, 0.25]
    assert info.tolist() == [1, 0, 0, 0]
    # the whole batch as one (C = 2): u_0 = [1, 1, -1, -2] -> mid(1, -1) = 0; u_1 = [-1, -1, 1, 2] -> 0
    _, beta_all, _, _ = oracle.balance_assign(s, 1, mode=oracle.QB_STEP)
    assert beta_all.tolist() == [0.0, 0.0]


def test_minibatch_step_one_batch_is_step():
    s = W.make_qb_scores(1024, 16, seed=5)
    b0 = np.linspace(-0.2, 0.2, 16).astype(np.float32)
    for rule in (oracle.QB_MIDPOINT, oracle.QB_BOUNDARY, oracle.QB_BIP):
        i1, b1, f1 = oracle.balance_step_minibatch(s, 2, b0, 1024, rule=rule)
        i2, b2, f2, _ = oracle.balance_assign(s, 2, beta=b0, mode=oracle.QB_STEP, rule=rule)
        assert (i1 == i2).all() and (b1 == b2).all() and (f1 == f2).all()


def test_minibatch_step_identical_batches_give_the_batch_beta():
    # B copies of the same mini-batch: each beta_b is that batch's beta, and their mean is it exactly
    s0 = W.make_qb_scores(256, 16, seed=6)
    s = np.concatenate([s0] * 8)
    _, b_one, _, _ = oracle.balance_assign(s0, 4, mode=oracle.QB_STEP)
    idx, b_avg, _ = oracle.balance_step_minibatch(s, 4, np.zeros(16, np.float32), 256)
    assert (b_avg == b_one).all()
    # selection is the whole batch's topk(s - beta_old), as in STEP
    i_step, _, _, _ = oracle.balance_assign(s, 4, mode=oracle.QB_STEP)
    assert (idx == i_step).all()


def test_minibatch_step_argument_errors():
    s = np.zeros((12, 4), np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.balance_step_minibatch(s, 1, np.zeros(4, np.float32), 5)   # 5 does not divide 12
    with pytest.raises(oracle.OracleError):
        oracle.balance_step_minibatch(s, 1, np.zeros(4, np.float32), 6)   # 6 * 1 not divisible by 4
