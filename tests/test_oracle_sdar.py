"""Pins of the SDAR-style block-decoding oracle (oracle.sdar_oracle) against
a library routine, the ISD oracle's strict-causal attention, closed forms,
hand-worked decisions and brute force (no GPU needed)."""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import isd_oracle as O
from oracle import sdar_oracle as S
from speculative_verification_isd_b200.inputs import f32_to_bf16_bits


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _paged_case(seed, B=2, N=3, Hq=4, Hkv=2, D=8, P=4, kv_len=(0, 7)):
    """Random dense prefixes scattered into a permuted page pool."""
    rng = np.random.default_rng(seed)
    kv_len = np.array(kv_len, np.int32)
    max_pages = (int(kv_len.max()) + N + P - 1) // P
    num_pages = B * max_pages + 3
    perm = rng.permutation(num_pages)
    table = perm[: B * max_pages].reshape(B, max_pages).astype(np.int32)
    k_pool = bf(rng.standard_normal((num_pages, P, Hkv, D)))
    v_pool = bf(rng.standard_normal((num_pages, P, Hkv, D)))
    q = bf(rng.standard_normal((B, N, Hq, D)))
    k_new = bf(rng.standard_normal((B, N, Hkv, D)))
    v_new = bf(rng.standard_normal((B, N, Hkv, D)))
    return dict(q=q, k_new=k_new, v_new=v_new, k_pool=k_pool, v_pool=v_pool, page_table=table,
                kv_len=kv_len, P=P)


@pytest.mark.parametrize("seed", [0, 1])
def test_block_attention_equals_sdpa_without_mask(seed):
    """R2: every block row sees the prefix and the whole block, which is
    torch's scaled_dot_product_attention with no mask over the dense
    [prefix; block] sequence (float64, then one bf16 rounding)."""
    c = _paged_case(seed)
    B, N, Hq, D = c["q"].shape
    Hkv = c["k_new"].shape[2]
    scale = 1.0 / math.sqrt(D)
    out, k2, v2 = S.block_attention(c["q"], c["k_new"], c["v_new"], c["k_pool"], c["v_pool"],
                                    c["page_table"], c["kv_len"], c["P"], scale)
    for b in range(B):
        L = int(c["kv_len"][b])
        Kp = O.gather_sequence(c["k_pool"], c["page_table"][b], L, c["P"])
        Vp = O.gather_sequence(c["v_pool"], c["page_table"][b], L, c["P"])
        K = torch.from_numpy(O.bf16_to_f64(np.concatenate([Kp, c["k_new"][b]])))  # [L+N,Hkv,D]
        Vv = torch.from_numpy(O.bf16_to_f64(np.concatenate([Vp, c["v_new"][b]])))
        q = torch.from_numpy(O.bf16_to_f64(c["q"][b]))  # [N,Hq,D]
        rep = Hq // Hkv
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.permute(1, 0, 2), K.repeat_interleave(rep, 1).permute(1, 0, 2),
            Vv.repeat_interleave(rep, 1).permute(1, 0, 2), scale=scale)  # [Hq,N,D]
        want = O.f64_to_bf16(ref.permute(1, 0, 2).reshape(N, Hq * D).numpy())
        got = out.reshape(B, N, Hq * D)[b]
        diff = np.abs(O.bf16_to_f64(got) - O.bf16_to_f64(want))
        # one bf16 rounding of values that agree to ~1e-15: equal, or one ulp
        # apart where the float64 sums straddle a rounding boundary
        assert diff.max() <= 2.0 ** -7 * np.abs(O.bf16_to_f64(want)).max()
        assert (diff == 0).mean() > 0.99
        # R3: the block rows were written at kv_len .. kv_len+N-1
        tail = O.gather_sequence(k2, c["page_table"][b], L + N, c["P"])[L:]
        assert np.array_equal(tail, c["k_new"][b])


def test_last_block_row_equals_strict_causal_row():
    """The last block row sees exactly the keys a strict-causal row at the same
    position sees, so it matches the ISD oracle's attention for clean slot
    N-1 of a block whose N clean slots hold the same rows."""
    c = _paged_case(3, kv_len=(5, 12))
    B, N, Hq, D = c["q"].shape
    Hkv = c["k_new"].shape[2]
    Q = 2 * N - 1
    rng = np.random.default_rng(9)
    q_isd = np.concatenate([c["q"], bf(rng.standard_normal((B, N - 1, Hq, D)))], axis=1)
    k_isd = np.concatenate([c["k_new"], bf(rng.standard_normal((B, N - 1, Hkv, D)))], axis=1)
    v_isd = np.concatenate([c["v_new"], bf(rng.standard_normal((B, N - 1, Hkv, D)))], axis=1)
    # the ISD layout needs pages for kv_len + 2N - 1 positions
    P = c["P"]
    max_pages = (int(c["kv_len"].max()) + Q + P - 1) // P
    extra = max_pages - c["page_table"].shape[1]
    pool_k = np.concatenate([c["k_pool"], np.zeros((B * extra,) + c["k_pool"].shape[1:], np.uint16)])
    pool_v = np.concatenate([c["v_pool"], np.zeros_like(pool_k[: B * extra])])
    base = c["k_pool"].shape[0]
    table = np.concatenate([c["page_table"], (base + np.arange(B * extra)).reshape(B, extra)],
                           axis=1).astype(np.int32)
    scale = 1.0 / math.sqrt(D)
    o_sdar, _, _ = S.block_attention(c["q"], c["k_new"], c["v_new"], c["k_pool"], c["v_pool"],
                                     c["page_table"], c["kv_len"], P, scale)
    o_isd, _, _ = O.attention(q_isd, k_isd, v_isd, pool_k, pool_v, table, c["kv_len"],
                              np.full(B, N, np.int32), N, P, scale)
    o_sdar = o_sdar.reshape(B, N, -1)
    o_isd = o_isd.reshape(B, Q, -1)
    assert np.array_equal(o_sdar[:, N - 1], o_isd[:, N - 1])
    # and earlier rows differ from their strict-causal counterparts (they
    # also see the block rows after them)
    assert not np.array_equal(o_sdar[:, 0], o_isd[:, 0])


def test_confidence_closed_forms():
    """R5: the confidence is the largest softmax probability."""
    V = 1000
    # uniform row: every probability 1/V
    m, s, a = O.row_stats(np.zeros(V))
    assert S.confidence(s) == np.float32(1.0 / V) and a == 0
    # one entry g above V-1 equal ones: e^g / (e^g + V - 1)
    for g in [0.5, 3.0, 12.0]:
        z = np.zeros(V)
        z[417] = g
        m, s, a = O.row_stats(z)
        want = math.exp(g) / (math.exp(g) + V - 1)
        assert a == 417
        assert abs(float(S.confidence(s)) - want) <= 1e-6 * want
    # float32 decision precision (R8)
    assert S.confidence(np.array([4.0])).dtype == np.float32


def test_unmask_hand_worked():
    """R6 on hand-worked blocks."""
    cand = np.array([10, 11, 12, 13])
    # two positions clear tau = 0.8: both commit, the others stay MASK
    tok, ch = S.unmask(np.array([-1, -1, -1, -1]), np.float32([0.5, 0.9, 0.2, 0.95]), cand, 0.8)
    assert list(tok) == [-1, 11, -1, 13] and ch == [1, 3]
    # none clears tau: only the most confident uncommitted one (position 2;
    # the committed position 1 with a higher confidence does not count)
    tok, ch = S.unmask(np.array([-1, 7, -1, -1]), np.float32([0.1, 0.99, 0.3, 0.2]), cand, 0.8)
    assert list(tok) == [-1, 7, 12, -1] and ch == [2]
    # ties go to the lowest position
    tok, ch = S.unmask(np.array([-1, -1, -1, -1]), np.float32([0.25, 0.4, 0.4, 0.1]), cand, 0.9)
    assert ch == [1]
    # the threshold is inclusive
    tok, ch = S.unmask(np.array([-1, -1]), np.float32([0.5, 0.25]), cand[:2], 0.5)
    assert ch == [0]
    # a complete block does not change
    tok, ch = S.unmask(np.array([1, 2]), np.float32([0.9, 0.9]), np.array([5, 6]), 0.0)
    assert list(tok) == [1, 2] and ch == []


def test_unmask_threshold_limits():
    """tau > 1 (no confidence reaches it): one position per forward, in
    decreasing confidence, so S_b = N.  tau = 0: the whole block at once."""
    rng = np.random.default_rng(0)
    N = 6
    conf = rng.random(N).astype(np.float32)
    cand = np.arange(N) + 100
    tok = np.full(N, -1)
    order = []
    for _ in range(N):
        tok, ch = S.unmask(tok, conf, cand, 1.5)
        assert len(ch) == 1
        order += ch
    assert order == list(np.argsort(-conf, kind="stable"))
    assert list(tok) == list(cand)
    tok, ch = S.unmask(np.full(N, -1), conf, cand, 0.0)
    assert ch == list(range(N)) and list(tok) == list(cand)


def _scripted_batch(sync):
    """Three requests, blocks of N = 3, tau = 0.5, six forwards.  Forward 0:
    every confidence is high, so every first block completes in one forward
    (forward 1 is their store pass).  From forward 2 on, request 0's second
    block has low confidences until forward 4 (one position per forward);
    requests 1 and 2 stay high."""
    N, tau = 3, 0.5
    hi, lo = 0.9, 0.1
    conf = [[[hi] * 3, [hi] * 3, [hi] * 3],
            [[hi] * 3, [hi] * 3, [hi] * 3],
            [[lo, 0.2, 0.3], [hi] * 3, [hi] * 3],
            [[lo, 0.3, 0.2], [hi] * 3, [hi] * 3],
            [[hi] * 3, [hi] * 3, [hi] * 3],
            [[hi] * 3, [hi] * 3, [hi] * 3]]
    tok = np.full((3, N), -1)
    steps = np.zeros(3, np.int64)
    kv = np.array([10, 20, 30])
    hist = []
    for t in range(6):
        cand = np.full((3, N), 40 + t) + np.arange(3)[:, None] * 100
        r = S.unmask_batch(tok, steps, kv, np.float32(conf[t]), cand, tau, sync)
        hist.append(r)
        tok, steps, kv = r["block_tok"], r["steps"], r["kv_len"]
    return hist


def test_unmask_batch_free_and_sync():
    """R3, R7 on the scripted batch: a complete block leaves after its store
    pass; without sync requests 1 and 2 move on by themselves, with sync they
    wait for request 0's slow second block."""
    free = _scripted_batch(False)
    sync = _scripted_batch(True)
    for h in (free, sync):
        # forward 0 completes every block, forward 1 stores them and they leave
        assert list(h[0]["unmasked"]) == [3, 3, 3] and list(h[0]["block_steps"]) == [0, 0, 0]
        assert list(h[1]["unmasked"]) == [0, 0, 0] and list(h[1]["block_steps"]) == [1, 1, 1]
        assert list(h[1]["kv_len"]) == [13, 23, 33]
        assert list(h[1]["out_tok"][2]) == [240, 240, 240]
        # forward 2: request 0 commits only its most confident position (2)
        assert list(h[2]["unmasked"]) == [1, 3, 3]
        assert list(h[2]["block_tok"][0]) == [-1, -1, 42]
    # forward 3: requests 1 and 2 store; free they leave, synced they wait
    assert list(free[3]["block_steps"]) == [0, 1, 1]
    assert list(free[3]["out_tok"][1]) == [142, 142, 142]
    assert list(free[3]["out_tok"][0]) == [-1, -1, -1]
    assert list(sync[3]["block_steps"]) == [0, 0, 0]
    assert list(sync[3]["unmasked"]) == [1, 0, 0]
    assert list(sync[3]["steps"]) == [2, 1, 1]
    assert list(sync[3]["block_tok"][0]) == [-1, 43, 42]
    # forward 4 completes request 0's block (S = 3); forward 5 is its store
    # pass: synced, the whole batch leaves together
    assert list(sync[4]["block_steps"]) == [0, 0, 0]
    assert list(sync[5]["block_steps"]) == [3, 1, 1]
    assert list(sync[5]["kv_len"]) == [16, 26, 36]
    assert list(sync[5]["out_tok"][0]) == [44, 43, 42]
    # free: requests 1 and 2 completed another block in forward 4 and left in 5
    assert list(free[5]["block_steps"]) == [3, 1, 1]
    assert list(free[5]["kv_len"]) == [16, 29, 39]


def test_sync_round_costs_the_slowest_block():
    """Under sync the round length (forwards between two departures of the
    batch) is the largest S_b of that round plus the store pass, and
    round_stats reports it."""
    rng = np.random.default_rng(4)
    B, N, tau = 5, 4, 0.6
    tok = np.full((B, N), -1)
    steps = np.zeros(B, np.int64)
    kv = np.zeros(B, np.int64)
    hist, last = [], -1
    for t in range(200):
        conf = rng.random((B, N)).astype(np.float32)
        cand = rng.integers(0, 50, (B, N))
        r = S.unmask_batch(tok, steps, kv, conf, cand, tau, True)
        tok, steps, kv = r["block_tok"], r["steps"], r["kv_len"]
        hist.append(r["block_steps"])
        if (r["block_steps"] > 0).any():
            assert (r["block_steps"] > 0).all()
            assert t - last == r["block_steps"].max() + 1
            last = t
    rs = S.round_stats(np.stack(hist), N)
    h = np.stack(hist)
    done = h[(h > 0).any(axis=1)]
    assert rs["rounds"] == done.shape[0] and rs["blocks"] == done.size
    assert rs["mean_max_S"] == pytest.approx(done.max(axis=1).mean())
    assert rs["tpf_sync"] == pytest.approx(N / (done.max(axis=1).mean() + 1))
    assert rs["mean_max_S"] >= rs["mean_S"]


@pytest.mark.parametrize("B", [1, 2, 3, 4])
def test_expected_max_brute_force(B):
    """E[max of B iid] in closed form against enumeration of all B-tuples."""
    pmf = np.array([0.1, 0.4, 0.3, 0.2])
    want = 0.0
    for tup in itertools.product(range(4), repeat=B):
        want += np.prod(pmf[list(tup)]) * (max(tup) + 1)
    assert S.expected_max(pmf, B) == pytest.approx(want, rel=1e-12)
    assert S.expected_max(np.array([0, 0, 1.0]), B) == pytest.approx(3.0)
    if B == 1:
        assert S.expected_max(pmf, 1) == pytest.approx(float(np.dot(pmf, [1, 2, 3, 4])))


def test_sdar_step_tiny_closed_loop():
    """A few whole steps on the table model: decisions, outputs and the KV
    pool evolve as the rules say (uses block_attention, lm_head, row_stats)."""
    rng = np.random.default_rng(1)
    B, N, Hq, Hkv, D, V, P = 2, 3, 4, 2, 8, 64, 4
    tables = dict(Eq=bf(rng.standard_normal((V + 1, Hq, D))),
                  Ek=bf(rng.standard_normal((V + 1, Hkv, D))),
                  Ev=bf(rng.standard_normal((V + 1, Hkv, D))))
    W = bf(rng.standard_normal((V, Hq * D)) * 0.5)
    kv = np.array([3, 9])
    max_pages = 8
    table = np.arange(B * max_pages, dtype=np.int32).reshape(B, max_pages)
    k_pool = bf(rng.standard_normal((B * max_pages, P, Hkv, D)))
    v_pool = bf(rng.standard_normal((B * max_pages, P, Hkv, D)))
    tok = np.full((B, N), -1)
    steps = np.zeros(B, np.int64)
    emitted = 0
    for t in range(8):
        q, kn, vn = S.embed_block(tables, tok, V)
        r = S.sdar_step(q, kn, vn, k_pool, v_pool, table, kv, W, tok, steps, P,
                        D ** -0.5, 0.3, True)
        # each open block commits at least one position per forward
        for b in range(B):
            if (tok[b] == -1).any():
                assert r["unmasked"][b] >= 1
        # confidences are the row stats' 1/S and candidates their argmax
        assert np.array_equal(r["conf"].ravel(), S.confidence(r["row_sumexp"]))
        emitted += int((r["block_steps"] > 0).sum())
        k_pool, v_pool = r["k_pool"], r["v_pool"]
        tok, steps, kv = r["block_tok"], r["steps"], r["kv_len"]
    assert emitted >= B
    assert np.all(kv >= np.array([3, 9]) + N)


def test_product_round_stats_match_the_oracle():
    """The product-side statistics the benchmark reports (workload.py) agree
    with the oracle's on synchronous and free-running decision histories."""
    from speculative_verification_isd_b200.workload import expected_max_of, sdar_round_stats
    rng = np.random.default_rng(8)
    B, N, tau = 6, 4, 0.55
    for sync in (True, False):
        tok = np.full((B, N), -1)
        steps = np.zeros(B, np.int64)
        kv = np.zeros(B, np.int64)
        hist = []
        for t in range(300):
            r = S.unmask_batch(tok, steps, kv, rng.random((B, N)).astype(np.float32),
                               rng.integers(0, 9, (B, N)), tau, sync)
            tok, steps, kv = r["block_tok"], r["steps"], r["kv_len"]
            hist.append(r["block_steps"])
        h = np.stack(hist)
        mine = sdar_round_stats(h, N)
        ref = S.round_stats(h, N)
        assert mine["blocks"] == ref["blocks"]
        assert mine["mean_S"] == pytest.approx(ref["mean_S"], rel=1e-12)
        assert mine["tpf_free"] == pytest.approx(ref["tpf_free"], rel=1e-12)
        if sync:
            assert mine["rounds"] == ref["rounds"]
            assert mine["mean_max_S"] == pytest.approx(ref["mean_max_S"], rel=1e-12)
            assert mine["tpf_sync"] == pytest.approx(ref["tpf_sync"], rel=1e-12)
        assert sum(mine["pmf"]) == pytest.approx(1.0)
    for pmf in ([0.1, 0.4, 0.3, 0.2], [0.0, 1.0], [0.7, 0.2, 0.1, 0.0, 0.0]):
        for Bb in (1, 3, 32):
            assert expected_max_of(pmf, Bb) == pytest.approx(S.expected_max(np.array(pmf), Bb),
                                                             rel=1e-12)


def test_rope_rotation_layout_and_invariants():
    """The stand-in's rotary embedding: rotate-half pairing, the frequency
    ladder base^(-2i/D), identity at position 0, and the relative-position
    property that makes it a rotary embedding."""
    from speculative_verification_isd_b200.inputs import rope_table
    D = 4
    tab = rope_table(64, D, base=1.0e6)
    # unit vectors: e_0 pairs with e_2 at frequency 1, e_1 with e_3 at 1e-3
    p = 5
    r0 = O.bf16_to_f64(S.rope_rotate(bf([1.0, 0, 0, 0]), tab[p]))
    assert np.allclose(r0, [math.cos(p), 0, math.sin(p), 0], atol=2 ** -8)
    r1 = O.bf16_to_f64(S.rope_rotate(bf([0, 1.0, 0, 0]), tab[p]))
    assert np.allclose(r1, [0, math.cos(p * 1e-3), 0, math.sin(p * 1e-3)], atol=2 ** -8)
    r2 = O.bf16_to_f64(S.rope_rotate(bf([0, 0, 1.0, 0]), tab[p]))
    assert np.allclose(r2, [-math.sin(p), 0, math.cos(p), 0], atol=2 ** -8)
    # position 0 is the identity, bit for bit
    rng = np.random.default_rng(0)
    D = 128
    tab = rope_table(4096, D)
    x = bf(rng.standard_normal((3, D)))
    assert np.array_equal(S.rope_rotate(x, tab[0]), x)
    # norms kept (to bf16 rounding); q(p).k(p') depends on p - p' only
    q, k = bf(rng.standard_normal(D)), bf(rng.standard_normal(D))
    nq = np.linalg.norm(O.bf16_to_f64(q))
    for pos in (1, 77, 4000):
        assert np.linalg.norm(O.bf16_to_f64(S.rope_rotate(q, tab[pos]))) == pytest.approx(nq, rel=1e-2)
    dots = []
    for p0 in (0, 100, 2500):
        qa = O.bf16_to_f64(S.rope_rotate(q, tab[p0 + 37]))
        ka = O.bf16_to_f64(S.rope_rotate(k, tab[p0]))
        dots.append(float(qa @ ka))
    scale = nq * np.linalg.norm(O.bf16_to_f64(k))
    assert max(dots) - min(dots) <= 2e-2 * scale
    # a block embedded with the table: committed tokens and MASK rows, rotated by position
    V = 50
    tables = dict(Eq=bf(rng.standard_normal((V + 1, 2, D))), Ek=bf(rng.standard_normal((V + 1, 1, D))),
                  Ev=bf(rng.standard_normal((V + 1, 1, D))))
    tok = np.array([[-1, 7, -1]])
    qq, kk, vv = S.embed_block(tables, tok, V, np.array([10]), tab)
    assert np.array_equal(qq[0, 1], S.rope_rotate(tables["Eq"][7], tab[11]))
    assert np.array_equal(kk[0, 2], S.rope_rotate(tables["Ek"][V], tab[12]))
    assert np.array_equal(vv[0, 0], tables["Ev"][V])
    assert not np.array_equal(qq[0, 0], qq[0, 2])   # MASK rows differ by position
