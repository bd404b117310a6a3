"""Pins of the oracle's slot layout, paged KV append, attention, LoRA and LM
head against brute force and textbook special cases (no GPU needed)."""
import math

import numpy as np
import pytest

from oracle import isd_oracle as O
from speculative_verification_isd_b200.inputs import f32_to_bf16_bits


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def test_slot_positions_layout():
    # c = 2 of N = 4: slots 0,1 clean; 2,3 inactive; 4,5,6 MASK right after t_2.
    assert list(O.slot_positions(100, 2, 4)) == [100, 101, -1, -1, 102, 103, 104]
    assert list(O.slot_positions(0, 4, 4)) == [0, 1, 2, 3, 4, 5, 6]
    assert list(O.slot_positions(7, 1, 1)) == [7]


def test_f64_to_bf16_rounding():
    # exactly representable values survive
    for v in [0.0, 1.0, -2.5, 0.015625, 1.5 * 2.0 ** 100, -1.25 * 2.0 ** -100]:
        assert O.bf16_to_f64(O.f64_to_bf16(np.array([v])))[0] == v
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert O.bf16_to_f64(O.f64_to_bf16(np.array([1.0 + 2 ** -8])))[0] == 1.0
    # 1 + 3*2^-8 is halfway between 1+2^-7 and 1+2^-6: even is 1+2^-6
    assert O.bf16_to_f64(O.f64_to_bf16(np.array([1.0 + 3 * 2 ** -8])))[0] == 1.0 + 2 ** -6
    # just above a tie rounds up (a bit that float32 would have dropped)
    assert O.bf16_to_f64(O.f64_to_bf16(np.array([1.0 + 2 ** -8 + 2 ** -40])))[0] == 1.0 + 2 ** -7
    # nearest-value property on random inputs
    rng = np.random.default_rng(0)
    x = rng.standard_normal(2000) * 10.0 ** rng.integers(-5, 5, 2000)
    r = O.bf16_to_f64(O.f64_to_bf16(x))
    e = np.floor(np.log2(np.abs(x)))
    ulp = 2.0 ** (e - 7)
    assert np.all(np.abs(r - x) <= ulp / 2 * (1 + 1e-12))


def _textbook_attention(qv, keys, vals, scale):
    scores = [scale * sum(a * b for a, b in zip(qv, k)) for k in keys]
    mx = max(scores)
    ws = [math.exp(s - mx) for s in scores]
    z = sum(ws)
    return [sum(w * v[d] for w, v in zip(ws, vals)) / z for d in range(len(vals[0]))]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_paged_attention_equals_dense_textbook(seed):
    """Build each request's dense sequence first, scatter it into a randomly
    permuted page pool, and compare the oracle's paged attention with
    textbook softmax attention over the dense sequence."""
    rng = np.random.default_rng(seed)
    B, N, Hq, Hkv, D, P = 3, 3, 4, 2, 8, 4
    Q = 2 * N - 1
    kv_len = np.array([0, 5, 11], np.int32)
    n_clean = np.array([1, 3, 2], np.int32)
    scale = 1.0 / math.sqrt(D)
    q = bf(rng.standard_normal((B, Q, Hq, D)))
    k_new = bf(rng.standard_normal((B, Q, Hkv, D)))
    v_new = bf(rng.standard_normal((B, Q, Hkv, D)))
    need = (kv_len + Q + P - 1) // P
    num_pages = int(need.sum()) + 2
    perm = rng.permutation(num_pages)
    table = np.full((B, need.max()), -1, np.int32)
    k_pool = bf(rng.standard_normal((num_pages, P, Hkv, D)))   # garbage everywhere
    v_pool = bf(rng.standard_normal((num_pages, P, Hkv, D)))
    dense_k, dense_v = [], []
    off = 0
    for b in range(B):
        table[b, : need[b]] = perm[off: off + need[b]]
        off += need[b]
        pk = bf(rng.standard_normal((kv_len[b], Hkv, D)))
        pv = bf(rng.standard_normal((kv_len[b], Hkv, D)))
        for t in range(kv_len[b]):
            k_pool[table[b, t // P], t % P] = pk[t]
            v_pool[table[b, t // P], t % P] = pv[t]
        # active block slots, in slot order, follow the prefix contiguously
        active = list(range(n_clean[b])) + list(range(N, Q))
        dense_k.append((np.concatenate([pk, k_new[b, active]]), active))
        dense_v.append(np.concatenate([pv, v_new[b, active]]))
    out, kp2, vp2 = O.attention(q, k_new, v_new, k_pool, v_pool, table, kv_len, n_clean, N, P,
                                scale)
    out = O.bf16_to_f64(out).reshape(B, Q, Hq, D)
    for b in range(B):
        dk, active = dense_k[b]
        dv = dense_v[b]
        for s in range(Q):
            if s not in active:
                assert np.all(out[b, s] == 0.0)
                continue
            upto = kv_len[b] + active.index(s) + 1
            for h in range(Hq):
                g = h // (Hq // Hkv)
                keys = O.bf16_to_f64(dk[:upto, g]).tolist()
                vals = O.bf16_to_f64(dv[:upto, g]).tolist()
                ref = _textbook_attention(O.bf16_to_f64(q[b, s, h]).tolist(), keys, vals, scale)
                got = out[b, s, h]
                # the oracle rounds once to bf16: within half a bf16 ulp
                assert np.all(np.abs(got - ref) <= np.abs(np.array(ref)) * 2 ** -8 + 1e-30)
        # cache rows written at the block positions; every other row untouched
        for i, s in enumerate(active):
            t = kv_len[b] + i
            assert np.array_equal(kp2[table[b, t // P], t % P], k_new[b, s])
            assert np.array_equal(vp2[table[b, t // P], t % P], v_new[b, s])
    touched = np.zeros((num_pages, P), bool)
    for b in range(B):
        for i in range(n_clean[b] + N - 1):
            t = kv_len[b] + i
            touched[table[b, t // P], t % P] = True
    assert np.array_equal(kp2[~touched], k_pool[~touched])
    assert np.array_equal(vp2[~touched], v_pool[~touched])


def test_attention_single_key_returns_value():
    # stride 1, empty prefix: the only visible key is the slot itself.
    rng = np.random.default_rng(4)
    q = bf(rng.standard_normal((2, 1, 2, 16)))
    k = bf(rng.standard_normal((2, 1, 1, 16)))
    v = bf(rng.standard_normal((2, 1, 1, 16)))
    pool = np.zeros((2, 4, 1, 16), np.uint16)
    table = np.array([[0], [1]], np.int32)
    out, _, _ = O.attention(q, k, v, pool, pool, table, np.zeros(2, np.int32),
                            np.ones(2, np.int32), 1, 4, 0.3)
    out = out.reshape(2, 2, 16)
    for b in range(2):
        for h in range(2):
            assert np.array_equal(out[b, h], v[b, 0, 0])


def test_attention_equal_keys_average_values():
    # identical keys -> uniform weights -> output is the mean of the visible values
    B, N, Hq, Hkv, D, P = 1, 2, 2, 1, 4, 4
    kv_len = np.array([3], np.int32)
    kvec = bf(np.full(D, 0.5))
    k_pool = np.tile(kvec, (2, P, Hkv, 1)).astype(np.uint16)
    vals = np.arange(2 * P * D, dtype=np.float32).reshape(2, P, 1, D) / 64.0
    v_pool = bf(vals)
    k_new = np.tile(kvec, (B, 3, Hkv, 1)).astype(np.uint16)
    v_new = bf(np.full((B, 3, Hkv, D), 1.0))
    q = bf(np.ones((B, 3, Hq, D)))
    table = np.array([[1, 0]], np.int32)
    out, _, _ = O.attention(q, k_new, v_new, k_pool, v_pool, table, kv_len, np.array([2]), N, P,
                            1.0)
    out = O.bf16_to_f64(out).reshape(B, 3, Hq, D)
    prefix = O.bf16_to_f64(v_pool[1, :3, 0])                  # positions 0..2 live in page 1
    expect0 = (prefix.sum(0) + 1.0) / 4                         # slot 0 sees 3 prefix + itself
    assert np.allclose(out[0, 0, 0], expect0, rtol=2 ** -8)
    expect2 = (prefix.sum(0) + 3.0) / 6                         # MASK slot 2 sees 3 + 3 block rows
    assert np.allclose(out[0, 2, 1], expect2, rtol=2 ** -8)
    assert np.all(out[0, 1] != 0)                               # slot 1 active (c = 2)


def test_lm_head_special_cases():
    rng = np.random.default_rng(6)
    M, H, V = 5, 32, 40
    hidden = bf(rng.standard_normal((M, H)))
    # one-hot vocabulary rows pick single hidden entries exactly
    W = np.zeros((V, H), np.float32)
    cols = rng.integers(0, H, V)
    W[np.arange(V), cols] = 1.0
    z = O.lm_head(hidden, bf(W))
    assert np.array_equal(z, O.bf16_to_f64(hidden)[:, cols].astype(np.float32))
    # all-ones hidden gives row sums of W (a transposed operand would not)
    Wr = bf(rng.standard_normal((V, H)))
    z = O.lm_head(bf(np.ones((M, H))), Wr)
    assert np.allclose(z, np.tile(O.bf16_to_f64(Wr).sum(1), (M, 1)), rtol=1e-6, atol=1e-6)
    # brute-force dot products on a few entries, with vocabulary chunking active
    z = O.lm_head(hidden, Wr, v_chunk=7)
    hh, ww = O.bf16_to_f64(hidden), O.bf16_to_f64(Wr)
    for (i, j) in [(0, 0), (4, 39), (2, 17)]:
        ref = 0.0
        for k in range(H):
            ref += hh[i, k] * ww[j, k]
        assert abs(float(z[i, j]) - ref) <= abs(ref) * 2 ** -23 + 1e-12
        assert O.lm_head_entry(hidden[i], Wr[j]) == pytest.approx(ref, rel=1e-12, abs=1e-12)


def test_gated_lora_touches_only_mask_rows():
    rng = np.random.default_rng(8)
    B, N, H, r = 2, 3, 16, 4
    Q = 2 * N - 1
    hidden = bf(rng.standard_normal((B * Q, H)))
    A = bf(rng.standard_normal((H, r)))
    Bm = bf(rng.standard_normal((r, H)))
    out = O.gated_lora(hidden, A, Bm, B, N).reshape(B, Q, H)
    hid = hidden.reshape(B, Q, H)
    assert np.array_equal(out[:, :N], hid[:, :N])                 # clean rows: base weights
    assert not np.array_equal(out[:, N:], hid[:, N:])
    # zero adapter is the identity
    z = O.gated_lora(hidden, np.zeros_like(A), Bm, B, N)
    assert np.array_equal(z, hidden)
    # A picks hidden entry 0 into rank slot 0, B adds it to column 3:
    A1 = np.zeros((H, r), np.float32)
    A1[0, 0] = 1.0
    B1 = np.zeros((r, H), np.float32)
    B1[0, 3] = 1.0
    o = O.gated_lora(hidden, bf(A1), bf(B1), B, N).reshape(B, Q, H)
    h64 = O.bf16_to_f64(hid)
    for b in range(B):
        for s in range(N, Q):
            exp = h64[b, s].copy()
            exp[3] += h64[b, s, 0]
            assert np.array_equal(o[b, s], O.f64_to_bf16(exp))
