"""Pins of the oracle's acceptance, residual draw, proposals and state update.

Each test checks the oracle against something fixed outside it: the E[acc] /
TPF table printed on the engineering-notes page ("自省扩散语言模型的 token
生成机制与工程实践", section "Token 生成的核心参数与验收机制"), the geometric
closed form stated on the I-DLM project page, exact enumeration of the
losslessness claim, or hand-worked cases.
"""
import math

import numpy as np
import pytest

from oracle import isd_oracle as O


def load_table(golden):
    rows = []
    for line in open(golden("eng_stride_table.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            n, e, t = line.split()
            rows.append((int(n), float(e), float(t)))
    return rows


def plain_probs(z):
    """Direct softmax without a max shift (test-side, independent of the oracle)."""
    e = [math.exp(float(v)) for v in z]
    s = sum(e)
    return [v / s for v in e]


def constructed_pair(rng, V, x, a, scale=0.5):
    """A p-row and a q-row (float32 logits) with p(x)/q(x) = a.

    q equals p except that logit x is raised by delta, with
    e^delta = (1 - P) / (a - P), P = p(x); then q(x) = P / a.
    """
    z = (rng.standard_normal(V) * scale).astype(np.float32)
    P = plain_probs(z)[x]
    assert a > P
    zq = z.copy()
    zq[x] = np.float32(float(z[x]) + math.log((1.0 - P) / (a - P)))
    return z, zq


def eacc_closed_form(a, N):
    return (1.0 - a ** N) / (1.0 - a)


def tpf_restart_model(a, N):
    # Full acceptance (prob a^(N-1)) keeps c = N: one forward per cycle.
    # A rejection adds one restart forward (c = 1) and one replacement token.
    f = a ** (N - 1)
    return (eacc_closed_form(a, N) + 1.0 - f) / (2.0 - f)


def test_table_matches_geometric_closed_form(golden):
    # Geometric acceptance (position k accepted with probability p^(k-1)).
    for N, e_acc, tpf in load_table(golden):
        assert round(eacc_closed_form(0.9, N), 2) == pytest.approx(e_acc, abs=1e-9)
        assert abs(tpf_restart_model(0.9, N) - tpf) < 0.0051


def _run_constructed(rng, B, N, a, V=64):
    Q = 2 * N - 1
    logits = (rng.standard_normal((B, Q, V)) * 0.5).astype(np.float32)
    prev = (rng.standard_normal((B, Q, V)) * 0.5).astype(np.float32)
    tok = rng.integers(0, V, size=(B, N)).astype(np.int32)
    for b in range(B):
        for j in range(2, N + 1):
            z, zq = constructed_pair(rng, V, int(tok[b, j - 1]), a)
            logits[b, j - 2] = z
            prev[b, N + j - 2] = zq
    u = rng.random((B, 2 * N)).astype(np.float32)
    kv = np.full(B, 100, dtype=np.int32)
    nc = np.full(B, N, dtype=np.int32)
    return O.accept(logits, prev, nc, tok, kv, u, N)


@pytest.mark.parametrize("N", [2, 3, 4, 5, 8])
def test_mean_accept_length_matches_table(golden, N):
    table = {n: e for n, e, _ in load_table(golden)}
    rng = np.random.default_rng(1000 + N)
    B = 6000
    res = _run_constructed(rng, B, N, 0.9)
    A = res["accept_len"].astype(np.float64)
    # every evaluated ratio equals the constructed rate
    r = res["ratio"][res["ratio"] >= 0]
    assert np.all(np.abs(r - 0.9) < 1e-5)
    se = A.std(ddof=1) / math.sqrt(B)
    assert abs(A.mean() - eacc_closed_form(0.9, N)) < 4 * se
    assert abs(A.mean() - table[N]) < 0.005 + 4 * se
    # geometric tail: P(A >= k) = 0.9^(k-1)
    for k in range(1, N + 1):
        assert abs((A >= k).mean() - 0.9 ** (k - 1)) < 4 * math.sqrt(0.25 / B) + 1e-12


@pytest.mark.parametrize("N", [2, 4, 8])
def test_closed_loop_tpf_matches_table(golden, N):
    """Run the oracle's state machine in closed loop; tokens per forward must
    equal the table's TPF column (and the TPF^2/Q identity must hold on the
    counters, as derived on the project page, step 6).

    The tolerance is 4 standard errors of the mean TPF, estimated from the
    per-request TPFs (requests are independent; consecutive forwards of one
    request are not, so a per-forward standard error would be too small),
    plus the table's rounding to two decimals."""
    table = {n: t for n, _, t in load_table(golden)}
    rng = np.random.default_rng(77 + N)
    B, steps, V, a = 160, 350, 64, 0.9
    Q = 2 * N - 1
    nc = np.ones(B, dtype=np.int32)
    tok = rng.integers(0, V, size=(B, N)).astype(np.int32)
    kv = np.zeros(B, dtype=np.int32)
    per_request = np.zeros(B)
    for _ in range(steps):
        logits = (rng.standard_normal((B, Q, V)) * 0.5).astype(np.float32)
        prev = (rng.standard_normal((B, Q, V)) * 0.5).astype(np.float32)
        for b in range(B):
            for j in range(2, int(nc[b]) + 1):
                z, zq = constructed_pair(rng, V, int(tok[b, j - 1]), a)
                logits[b, j - 2] = z
                prev[b, N + j - 2] = zq
        u = rng.random((B, 2 * N)).astype(np.float32)
        res = O.accept(logits, prev, nc, tok, kv, u, N)
        per_request += res["accept_len"]
        assert np.array_equal(res["next_kv_len"], kv + res["accept_len"])
        nc, tok, kv = res["next_n_clean"], res["next_clean_tok"], res["next_kv_len"]
        assert set(np.unique(nc)) <= {1, N}
    total_tokens = int(per_request.sum())
    forwards = B * steps
    tpf = total_tokens / forwards
    se = (per_request / steps).std(ddof=1) / math.sqrt(B)
    assert se < 0.02  # the run is long enough for the bound to mean something
    assert abs(tpf - tpf_restart_model(a, N)) < 4 * se, (tpf, se)
    assert abs(tpf - table[N]) < 4 * se + 0.005, (tpf, table[N], se)
    oh = forwards * Q / total_tokens
    assert tpf / oh == pytest.approx(tpf * tpf / Q, rel=1e-12)
    # kv_len counts exactly the emitted tokens
    assert int(kv.sum()) == total_tokens


def test_identical_rows_accept_everything():
    rng = np.random.default_rng(5)
    B, N, V = 50, 4, 33
    Q = 2 * N - 1
    logits = rng.standard_normal((B, Q, V)).astype(np.float32)
    prev = rng.standard_normal((B, Q, V)).astype(np.float32)
    for j in range(2, N + 1):
        prev[:, N + j - 2] = logits[:, j - 2]
    tok = rng.integers(0, V, size=(B, N)).astype(np.int32)
    u = np.nextafter(np.float32(1.0), np.float32(0.0)) * np.ones((B, 2 * N), np.float32)
    res = O.accept(logits, prev, np.full(B, N, np.int32), tok, np.zeros(B, np.int32), u, N)
    assert np.all(res["accept_len"] == N)
    assert np.all(res["next_n_clean"] == N)
    assert np.all(res["ratio"] == 1.0)
    assert np.array_equal(res["out_tok"][:, : N - 1], tok[:, 1:])


def test_replacement_is_lossless_by_enumeration():
    """sum_x q(x) [min(1,p/q) 1{x=v} + (1 - min(1,p/q)) w(v)/sum w] = p(v)."""
    rng = np.random.default_rng(9)
    for _ in range(20):
        V = 16
        zp = rng.standard_normal(V) * 1.5
        zq = rng.standard_normal(V) * 1.5
        p = np.array(plain_probs(zp))
        q = np.array(plain_probs(zq))
        w = O.residual_distribution(zp, zq)
        out = np.zeros(V)
        for x in range(V):
            acc = min(1.0, O.accept_ratio(zp, zq, x))
            out[x] += q[x] * acc
            out += q[x] * (1.0 - acc) * w / w.sum()
        assert np.max(np.abs(out - p)) < 1e-12


def _chi2_pvalue(counts, probs):
    from scipy.stats import chisquare
    n = counts.sum()
    return chisquare(counts, probs * n).pvalue


def test_sampled_outputs_follow_p_chi_square():
    """Sample mode, V = 16: the token emitted at position 2 (accepted proposal
    or replacement) is distributed as p, and the fresh proposal x'_1 as the
    anchor row's softmax."""
    rng = np.random.default_rng(2024)
    V, N, T = 16, 2, 30000
    Q = 2 * N - 1
    zp = (rng.standard_normal(V) * 1.2).astype(np.float32)
    zq = (rng.standard_normal(V) * 1.2).astype(np.float32)
    za = (rng.standard_normal(V) * 1.2).astype(np.float32)
    q = np.array(plain_probs(zq))
    logits = np.zeros((T, Q, V), np.float32)
    prev = np.zeros((T, Q, V), np.float32)
    logits[:, 0] = zp
    logits[:, 1] = za
    logits[:, 2] = za
    prev[:, N] = zq
    # proposals drawn from q by the test itself
    x = np.searchsorted(np.cumsum(q), rng.random(T), side="right").clip(0, V - 1)
    tok = np.stack([rng.integers(0, V, T), x], axis=1).astype(np.int32)
    u = rng.random((T, 2 * N)).astype(np.float32)
    res = O.accept(logits, prev, np.full(T, 2, np.int32), tok, np.zeros(T, np.int32), u, N,
                   mode=O.PROPOSE_SAMPLE)
    pos2 = res["out_tok"][:, 0]
    counts = np.bincount(pos2, minlength=V)
    assert _chi2_pvalue(counts, np.array(plain_probs(zp))) > 1e-3
    full = res["accept_len"] == 2
    x1 = res["out_tok"][full, 1]
    assert _chi2_pvalue(np.bincount(x1, minlength=V), np.array(plain_probs(za))) > 1e-3
    # and the acceptance rate equals sum_x min(p(x), q(x))
    p = np.array(plain_probs(zp))
    expect = np.minimum(p, q).sum()
    assert abs(full.mean() - expect) < 4 * math.sqrt(expect * (1 - expect) / T)


def _log(pr):
    return np.log(np.asarray(pr, dtype=np.float64)).astype(np.float32)


def _hand_case():
    V, N = 4, 3
    Q = 2 * N - 1
    logits = np.zeros((1, Q, V), np.float32)
    prev = np.zeros((1, Q, V), np.float32)
    logits[0, 0] = _log([0.1, 0.2, 0.3, 0.4])      # p for t_2
    prev[0, N + 0] = _log([0.25, 0.25, 0.25, 0.25])  # q for t_2
    logits[0, 1] = _log([0.4, 0.3, 0.2, 0.1])      # p for t_3
    prev[0, N + 1] = _log([0.1, 0.1, 0.1, 0.7])    # q for t_3
    logits[0, 2] = _log([0.1, 0.6, 0.2, 0.1])      # anchor row -> x'_1 = 1
    logits[0, 3] = _log([0.7, 0.1, 0.1, 0.1])      # MASK row 0 -> x'_2 = 0
    logits[0, 4] = _log([0.1, 0.1, 0.1, 0.7])      # MASK row 1 -> x'_3 = 3
    tok = np.array([[1, 2, 3]], np.int32)
    return logits, prev, tok, N


def test_hand_worked_rejection():
    logits, prev, tok, N = _hand_case()
    # r(t_2 = 2) = 0.3/0.25 = 1.2 -> accepted; r(t_3 = 3) = 0.1/0.7 -> u=0.2 rejects.
    # residual max(0, p-q) = [0.3, 0.2, 0.1, 0]; u_res = 0.6 -> target 0.36 -> y = 1.
    u = np.array([[0.5, 0.2, 0.6, 0.0, 0.0, 0.0]], np.float32)
    res = O.accept(logits, prev, np.array([3], np.int32), tok, np.array([10], np.int32), u, N)
    assert res["ratio"][0, 0] == pytest.approx(1.2, rel=1e-6)
    assert res["ratio"][0, 1] == pytest.approx(0.1 / 0.7, rel=1e-6)
    assert res["accept_len"][0] == 2
    assert list(res["out_tok"][0]) == [2, 1, -1]
    assert res["next_n_clean"][0] == 1
    assert list(res["next_clean_tok"][0]) == [1, -1, -1]
    assert res["next_kv_len"][0] == 12
    assert res["rejected_at"][0] == 3


def test_hand_worked_full_accept():
    logits, prev, tok, N = _hand_case()
    u = np.array([[0.5, 0.1, 0.6, 0.0, 0.0, 0.0]], np.float32)
    res = O.accept(logits, prev, np.array([3], np.int32), tok, np.array([10], np.int32), u, N)
    assert res["accept_len"][0] == 3
    assert list(res["out_tok"][0]) == [2, 3, 1]
    assert res["next_n_clean"][0] == 3
    assert list(res["next_clean_tok"][0]) == [1, 0, 3]
    assert res["next_kv_len"][0] == 13


def test_hand_worked_restart_step():
    # c = 1: nothing to verify; emit the anchor proposal from row 0.
    logits, prev, tok, N = _hand_case()
    u = np.zeros((1, 6), np.float32)
    res = O.accept(logits, prev, np.array([1], np.int32), tok, np.array([10], np.int32), u, N)
    assert res["accept_len"][0] == 1
    assert list(res["out_tok"][0]) == [3, -1, -1]          # argmax of row 0 is 3
    assert list(res["next_clean_tok"][0]) == [3, 0, 3]
    assert res["next_kv_len"][0] == 11


def test_stride_one_is_greedy_autoregressive():
    rng = np.random.default_rng(3)
    B, V = 7, 50
    logits = rng.standard_normal((B, 1, V)).astype(np.float32)
    res = O.accept(logits, logits, np.ones(B, np.int32), np.zeros((B, 1), np.int32),
                   np.arange(B, dtype=np.int32), rng.random((B, 2)).astype(np.float32), 1)
    assert np.array_equal(res["out_tok"][:, 0], logits[:, 0].argmax(-1))
    assert np.all(res["accept_len"] == 1)
    assert np.array_equal(res["next_kv_len"], np.arange(B) + 1)


def test_residual_with_point_mass_proposal():
    # q puts (almost) all mass on x; after rejecting x the replacement never is x
    V = 8
    zp = np.zeros(V, np.float32)
    zq = np.full(V, -60.0, np.float32)
    zq[5] = 0.0
    w = O.residual_distribution(zp, zq)
    assert w[5] == 0.0
    assert np.allclose(w / w.sum(), [1 / 7] * 5 + [0] + [1 / 7] * 2)


def test_inverse_cdf_edges():
    w = np.array([0.0, 0.25, 0.0, 0.5, 0.25])
    assert O.inverse_cdf(w, 0.0) == 1
    assert O.inverse_cdf(w, 0.2499) == 1
    assert O.inverse_cdf(w, 0.25) == 3
    assert O.inverse_cdf(w, 0.75) == 4
    assert O.inverse_cdf(w, np.nextafter(1.0, 0.0)) == 4


def test_argmax_ties_go_to_lowest_index():
    z = np.array([1.0, 3.0, 2.0, 3.0, 3.0], np.float32)
    m, s, a = O.row_stats(z)
    assert (m, a) == (3.0, 1)
    assert s == pytest.approx(3.0 + math.exp(-1.0) + math.exp(-2.0), rel=1e-15)
    assert O.row_stats(np.zeros(10))[1] == 10.0


def test_zero_residual_mass_falls_back_to_argmax_p():
    """A proposal with zero probability under both rows: p(x)/q(x) is 0/0
    (NaN), so u < p(x)/q(x) is false for every u and the proposal is rejected;
    p and q are otherwise equal, so max(0, p - q) has no mass and the
    replacement is the argmax of p (the reading taken for the empty residual),
    here worked out by hand: entry 1 holds the largest logit."""
    N, V = 2, 5
    Q = 2 * N - 1
    zp = np.array([0.1, 2.0, -np.inf, 0.5, -1.0], np.float32)
    logits = np.zeros((1, Q, V), np.float32)
    prev = np.zeros((1, Q, V), np.float32)
    logits[0, 0] = zp          # p for t_2
    prev[0, N] = zp            # q for t_2: the same distribution
    tok = np.array([[3, 2]], np.int32)   # t_2 = 2 has p = q = 0
    u = np.array([[0.0, 0.7, 0.2, 0.3]], np.float32)
    with np.errstate(invalid="ignore"):
        res = O.accept(logits, prev, np.array([2], np.int32), tok, np.array([5], np.int32), u, N)
        w = O.residual_distribution(zp, zp)
    assert w.sum() == 0.0
    assert np.isnan(res["ratio"][0, 0])
    assert res["rejected_at"][0] == 2
    assert res["accept_len"][0] == 1
    assert list(res["out_tok"][0]) == [1, -1]
    assert res["next_n_clean"][0] == 1 and list(res["next_clean_tok"][0]) == [1, -1]
    assert res["next_kv_len"][0] == 6


def test_inverse_cdf_falls_back_to_last_positive_weight():
    """When no prefix sum exceeds u * total (u = 1 makes the target equal to
    the total), the draw is the last entry with positive weight -- never a
    trailing zero-weight entry."""
    w = np.array([0.0, 0.25, 0.0, 0.5, 0.25, 0.0, 0.0])
    assert O.inverse_cdf(w, 1.0) == 4
    assert O.inverse_cdf(np.array([0.0, 3.0, 0.0]), 1.0) == 1
    # the main branch just below: the largest uniform in [0, 1) of float32
    assert O.inverse_cdf(w, float(np.nextafter(np.float32(1), np.float32(0)))) == 4


def test_loop_stats_counts_match_the_oracle_loop():
    """The device loop's statistics (speculative_verification_isd_b200.workload.
    loop_stats) rebuild each step's clean count from the accept lengths alone;
    on the oracle's own closed loop their test and acceptance counts equal the
    oracle's (tested = proposals with a ratio, accepted = u < ratio), and
    tokens per forward is the mean accept length."""
    from speculative_verification_isd_b200.workload import loop_stats
    rng = np.random.default_rng(11)
    B, steps, V, N, a = 40, 120, 64, 4, 0.85
    Q = 2 * N - 1
    nc = np.ones(B, dtype=np.int32)
    tok = rng.integers(0, V, size=(B, N)).astype(np.int32)
    kv = np.zeros(B, dtype=np.int32)
    hist = np.zeros((steps, B), np.int64)
    tests = acc = 0
    for s in range(steps):
        logits = (rng.standard_normal((B, Q, V)) * 0.5).astype(np.float32)
        prev = (rng.standard_normal((B, Q, V)) * 0.5).astype(np.float32)
        for b in range(B):
            for j in range(2, int(nc[b]) + 1):
                z, zq = constructed_pair(rng, V, int(tok[b, j - 1]), a)
                logits[b, j - 2] = z
                prev[b, N + j - 2] = zq
        u = rng.random((B, 2 * N)).astype(np.float32)
        res = O.accept(logits, prev, nc, tok, kv, u, N)
        hist[s] = res["accept_len"]
        if s >= 10:
            r = res["ratio"]
            tested = r >= 0
            tests += int(tested.sum())
            acc += int((tested & (u[:, : N - 1] < r)).sum())
        nc, tok, kv = res["next_n_clean"], res["next_clean_tok"], res["next_kv_len"]
    st = loop_stats(hist, N, 10, steps)
    assert st["tests"] == tests
    assert st["accept_rate"] == pytest.approx(acc / tests, abs=1e-12)
    assert st["tpf"] == pytest.approx(hist[10:].mean(), abs=1e-12)
    assert abs(st["accept_rate"] - a) < 0.03
    # starting the count mid-run from the known clean counts gives the same
    c10 = np.ones(B, np.int64)
    for s in range(10):
        c10 = np.where(hist[s] == c10, N, 1)
    assert loop_stats(hist, N, 10, steps, c_start=c10) == st


def test_bench_restart_model_matches_the_closed_form():
    """bench.py's restart-model TPF (reported beside the closed-loop figure)
    is the same function of (a, N) as this file's, and gives the table's
    2.92 at a = 0.9, N = 4; a = 1 keeps every proposal (TPF = N)."""
    import bench
    for N in (2, 3, 4, 8):
        for a in (0.5, 0.8, 0.9, 0.95):
            assert bench.restart_model_tpf(a, N) == pytest.approx(tpf_restart_model(a, N), rel=1e-12)
        assert bench.restart_model_tpf(1.0, N) == pytest.approx(float(N))
    assert round(bench.restart_model_tpf(0.9, 4), 2) == 2.92
