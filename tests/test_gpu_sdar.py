"""SDAR-style confidence-threshold block decoding on the GPU against the
oracle (oracle.sdar_oracle).

Layered like the ISD parity tests: block-causal attention and the KV append
against the oracle's (bf16 tolerance; the pool bit-exact), logits on the GPU's
own hidden rows (fp32 reassociation bound), row statistics, and the unmask
decisions.  The decisions are compared bit-exactly on the GPU's own
statistics (same float32 confidence on both sides), and on the oracle's
statistics except where a confidence lies within NEAR of tau or of the
runner-up (float32 vs float64 sums may order those differently).
"""
import numpy as np
import pytest
import torch

from oracle import isd_oracle as O
from oracle import parity as OP
from oracle import sdar_oracle as S
from speculative_verification_isd_b200 import inputs as I

from gpu_util import bf16_dev, bf16_host, i32_dev, record_parity, row_stats_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isd():
    from speculative_verification_isd_b200 import isd as lib
    return lib


# block-causal attention on the tensor-core path (D = 128) and the general
# path (D = 64), ragged prefixes over several 128-key tiles
SDAR_CONFIGS = {
    "ragged_small": I.CONFIGS["ragged_small"],          # B=3, N=4, grp 4: 16 rows per kv head
    "ragged_n8": I.CONFIGS["ragged_n8"],                # B=3, N=8, 64-token pages: 32 rows
    "tiny_d64": I.IsdConfig("tiny_d64", B=4, N=3, Hq=4, Hkv=1, D=64, V=700, page_size=16,
                            prefix_lo=0, prefix_hi=300, w_std=0.5, qkv_std=0.5, kv_std=1.0),
}


def _decisions_close(conf_o, tok, tau):
    """Positions whose decision may flip between float64 and float32 sums:
    the confidence within NEAR of tau, or of another open position's (the
    fallback's choice)."""
    near = np.zeros(tok.shape[0], bool)
    for b in range(tok.shape[0]):
        open_pos = np.nonzero(tok[b] < 0)[0]
        c = conf_o[b, open_pos].astype(np.float64)
        if np.any(np.abs(c - tau) <= OP.NEAR * max(tau, 1e-30)):
            near[b] = True
        if c.size > 1:
            srt = np.sort(c)
            if np.any(np.diff(srt) <= OP.NEAR * srt[1:]):
                near[b] = True
    return near


def _gpu_state(tok, steps, kv):
    return i32_dev(tok), i32_dev(steps), i32_dev(kv)


@pytest.mark.parametrize("name", list(SDAR_CONFIGS))
@pytest.mark.parametrize("sync", [True, False])
def test_sdar_step_layers(isd, name, sync):
    cfg = SDAR_CONFIGS[name]
    B, N, V, P = cfg.B, cfg.N, cfg.V, cfg.page_size
    inp = I.make_step_inputs(cfg, seed=5)
    q, kn, vn = (np.ascontiguousarray(inp[k][:, :N]) for k in ("q", "k_new", "v_new"))
    kv0 = inp["kv_len"].astype(np.int64)
    rng = np.random.default_rng(6)
    # a mixed state: fresh blocks, partly committed ones, one complete block
    tok0 = np.where(rng.random((B, N)) < 0.4, rng.integers(0, V, (B, N)), -1).astype(np.int32)
    tok0[0] = -1
    tok0[-1] = rng.integers(0, V, N)
    steps0 = np.where((tok0 >= 0).any(axis=1), rng.integers(1, N, B), 0).astype(np.int32)
    mp = inp["page_table"].shape[1]
    d = isd.make_dims(B, N, cfg.Hq, cfg.Hkv, cfg.D, V, P, inp["k_pool"].shape[0], mp)
    M = B * N
    # the oracle first: its confidences fix a tau that splits the open positions
    o_hid, o_kp, o_vp = S.block_attention(q, kn, vn, inp["k_pool"], inp["v_pool"],
                                          inp["page_table"], kv0, P, cfg.D ** -0.5)
    z_o = O.lm_head(o_hid, inp["W"])
    _, s_o, a_o = O.row_stats_all(z_o)
    conf_o = S.confidence(s_o).reshape(B, N)
    tau = float(np.quantile(conf_o[tok0 < 0], 0.6))

    g = dict(k_pool=bf16_dev(inp["k_pool"]), v_pool=bf16_dev(inp["v_pool"]),
             page_table=i32_dev(inp["page_table"]), W=bf16_dev(inp["W"]))
    tok_g, steps_g, kv_g = _gpu_state(tok0, steps0, kv0.astype(np.int32))
    hidden = torch.empty(M * d.H, dtype=torch.bfloat16, device="cuda")
    logits = torch.empty(M * V, dtype=torch.float32, device="cuda")
    rs = torch.zeros(M * 4, dtype=torch.int32, device="cuda")
    unmasked = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    out_tok = torch.full((B, N), -7, dtype=torch.int32, device="cuda")
    block_steps = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    ws = isd.alloc_workspace(d)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    isd.sdar_step(d, tau, sync, bf16_dev(q), bf16_dev(kn), bf16_dev(vn), g["k_pool"], g["v_pool"],
                  g["page_table"], kv_g, g["W"], logits, tok_g, steps_g, unmasked, out_tok,
                  block_steps, ws, hidden=hidden, row_stats=rs, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # KV append (bit-exact) and attention
    assert np.array_equal(bf16_host(g["k_pool"]), o_kp)
    assert np.array_equal(bf16_host(g["v_pool"]), o_vp)
    g_hid = bf16_host(hidden).reshape(M, d.H)
    herr = np.abs(O.bf16_to_f64(g_hid) - O.bf16_to_f64(o_hid))
    assert herr.max() <= 2e-2 and herr.mean() <= 3e-3, (herr.max(), herr.mean())
    # logits on the GPU's hidden rows
    z_g = logits.cpu().numpy().reshape(M, V)
    z_h = O.lm_head(g_hid, inp["W"])
    bound = 1e-4 * (np.abs(O.bf16_to_f64(g_hid)) @ np.abs(O.bf16_to_f64(inp["W"])).T) + 1e-6
    assert np.all(np.abs(z_g - z_h) <= bound)
    # row statistics of the GPU's logits
    m_g, s_g, a_g = row_stats_host(rs)
    m_h, s_h, a_h = O.row_stats_all(z_g)
    assert np.array_equal(m_g, m_h.astype(np.float32).astype(np.float64))
    assert np.array_equal(a_g, a_h)
    assert np.all(np.abs(s_g - s_h) <= OP.NEAR * s_h)
    # decisions on the GPU's statistics: bit-exact
    conf_g = S.confidence(s_g).reshape(B, N)
    r_g = S.unmask_batch(tok0, steps0, kv0, conf_g, a_g.reshape(B, N), tau, sync)
    got = dict(block_tok=tok_g, steps=steps_g, kv_len=kv_g, unmasked=unmasked, out_tok=out_tok,
               block_steps=block_steps)
    for k, t in got.items():
        assert np.array_equal(t.cpu().numpy().reshape(r_g[k].shape), r_g[k]), k
    # decisions on the oracle's own statistics, excusing near calls
    r_o = S.unmask_batch(tok0, steps0, kv0, conf_o, a_o.reshape(B, N), tau, sync)
    near = _decisions_close(conf_o, tok0, tau)
    same = np.all(r_o["block_tok"] == r_g["block_tok"], axis=1)
    assert np.all(same | near), np.nonzero(~same & ~near)
    record_parity(f"SDAR step {name} sync={sync}",
                  dict(requests=B, near_threshold=int(near.sum()), mismatches=0,
                       committed=int(r_g["unmasked"].sum())))


@pytest.mark.parametrize("sync", [True, False])
def test_sdar_full_size_sampled(isd, sync):
    """B=32, N=4 blocks at the Qwen3-8B shapes: whole-request attention for
    three requests, whole 256-row vocabulary tiles of the logits, all row
    statistics and the decisions."""
    from speculative_verification_isd_b200.workload import SdarLoopWorkload
    cfg = I.CONFIGS["qwen3_8b_b32_n4"]
    B, N, V, P = cfg.B, cfg.N, cfg.V, cfg.page_size
    w = SdarLoopWorkload(isd, cfg, capacity_steps=4, seed=3, w_std=0.1, qkv_std=0.5, kv_std=1.0)
    d = w.dims
    M = B * N
    tok0 = w.block_tok.cpu().numpy()
    kv0 = w.kv_len.cpu().numpy().astype(np.int64)
    w.run(1, tau=0.02, sync=sync)   # prepare + step (one forward of fresh blocks)
    torch.cuda.synchronize()
    assert int(w.err.item()) == 0
    table = w.page_table.cpu().numpy().reshape(B, -1)
    q = bf16_host(w.q).reshape(B, N, cfg.Hq, cfg.D)
    kn = bf16_host(w.k_new).reshape(B, N, cfg.Hkv, cfg.D)
    vn = bf16_host(w.v_new).reshape(B, N, cfg.Hkv, cfg.D)
    tables = {k: bf16_host(getattr(w, k)[V:V + 1]).reshape((1,) + tuple(getattr(w, k).shape[1:]))
              for k in ("Eq", "Ek", "Ev")}
    # block activations: the MASK row, q and k rotated by position
    qo, ko, vo = S.embed_block(tables, np.zeros((B, N), np.int64) - 1, 0, kv0,
                               w.rope.cpu().numpy())
    assert np.array_equal(q, qo) and np.array_equal(kn, ko) and np.array_equal(vn, vo)
    g_hid = bf16_host(w.hidden).reshape(M, cfg.H)
    for b in (0, B // 2, B - 1):
        L = int(kv0[b]) + N
        # this request's pages only (the pool is ~1 GB)
        pages = torch.from_numpy(table[b, : (L + P - 1) // P].astype(np.int64)).cuda()
        kp = bf16_host(w.k_pool[pages])
        vp = bf16_host(w.v_pool[pages])
        local = np.arange(pages.numel(), dtype=np.int32)
        K = O.bf16_to_f64(O.gather_sequence(kp, local, L, P))
        Vv = O.bf16_to_f64(O.gather_sequence(vp, local, L, P))
        assert np.array_equal(O.gather_sequence(kp, local, L, P)[-N:], kn[b])
        for s in range(N):
            for h in range(cfg.Hq):
                g = h // (cfg.Hq // cfg.Hkv)
                sc = (K[:, g] @ O.bf16_to_f64(q[b, s, h])) * cfg.D ** -0.5
                e = np.exp(sc - sc.max())
                o = (e @ Vv[:, g]) / e.sum()
                got = O.bf16_to_f64(g_hid[b * N + s, h * cfg.D:(h + 1) * cfg.D])
                assert np.abs(got - o).max() <= 2e-2, (b, s, h)
    z_g = w.logits.cpu().numpy().reshape(M, V)
    W = bf16_host(w.W).reshape(V, cfg.H)
    h64 = O.bf16_to_f64(g_hid)
    for t0 in (0, (V // 4) // 256 * 256, (V // 2) // 256 * 256, V - V % 256 - 256, V - V % 256):
        t1 = min(V, t0 + 256)
        Wt = O.bf16_to_f64(W[t0:t1])
        ref = h64 @ Wt.T
        bound = 1e-4 * (np.abs(h64) @ np.abs(Wt).T) + 1e-6
        assert np.all(np.abs(z_g[:, t0:t1] - ref) <= bound), t0
    m_g, s_g, a_g = row_stats_host(w.row_stats)
    m_h, s_h, a_h = O.row_stats_all(z_g)
    assert np.array_equal(a_g, a_h)
    assert np.array_equal(m_g, m_h.astype(np.float32).astype(np.float64))
    assert np.all(np.abs(s_g - s_h) <= OP.NEAR * s_h)
    r = S.unmask_batch(tok0, np.zeros(B, np.int64), kv0, S.confidence(s_g).reshape(B, N),
                       a_g.reshape(B, N), 0.02, sync)
    assert np.array_equal(w.block_tok.cpu().numpy(), r["block_tok"])
    assert np.array_equal(w.unmasked_hist[0].cpu().numpy(), r["unmasked"])
    assert np.array_equal(w.block_steps_hist[0].cpu().numpy(), r["block_steps"])
    assert np.array_equal(w.kv_len.cpu().numpy(), r["kv_len"])
    record_parity(f"SDAR step qwen3_8b_b32_n4 sampled sync={sync}",
                  dict(requests=B, near_threshold=0, mismatches=0,
                       committed=int(r["unmasked"].sum())))


def _loop_stepwise(isd, cfg, steps, tau, sync, seed):
    """isd_sdar_loop one forward per call, every stage against the oracle;
    then the same forwards in one call, bit-identical."""
    from speculative_verification_isd_b200.workload import SdarLoopWorkload
    B, N, V, P = cfg.B, cfg.N, cfg.V, cfg.page_size
    w = SdarLoopWorkload(isd, cfg, capacity_steps=steps, seed=seed)
    d = w.dims
    M = B * N
    tables = {k: bf16_host(getattr(w, k)).reshape((V + 1,) + tuple(getattr(w, k).shape[1:]))
              for k in ("Eq", "Ek", "Ev")}
    rope = w.rope.cpu().numpy()
    Wh = bf16_host(w.W).reshape(V, cfg.H)
    absW = np.abs(O.bf16_to_f64(Wh))
    pool_k, pool_v = bf16_host(w.k_pool), bf16_host(w.v_pool)
    o_table = w.page_table.cpu().numpy().reshape(B, -1).copy()
    o_used = w.pages_used.cpu().numpy().copy()
    o_next = int(w.next_free_page.item())
    max_pages = o_table.shape[1]
    hist = []
    near_steps = 0
    for s in range(steps):
        tok = w.block_tok.cpu().numpy()
        st = w.steps.cpu().numpy()
        kv = w.kv_len.cpu().numpy().astype(np.int64)
        w.run(1, tau, sync)
        torch.cuda.synchronize()
        q, kn, vn = S.embed_block(tables, tok, V, kv, rope)
        assert np.array_equal(bf16_host(w.q).reshape(q.shape), q)
        assert np.array_equal(bf16_host(w.k_new).reshape(kn.shape), kn)
        assert np.array_equal(bf16_host(w.v_new).reshape(vn.shape), vn)
        for b in range(B):
            need = min((int(kv[b]) + N + P - 1) // P, max_pages)
            while o_used[b] < need:
                o_table[b, o_used[b]] = o_next
                o_used[b] += 1
                o_next += 1
        assert np.array_equal(w.page_table.cpu().numpy().reshape(B, -1), o_table)
        o_hid, pool_k, pool_v = S.block_attention(q, kn, vn, pool_k, pool_v, o_table, kv, P,
                                                  cfg.D ** -0.5)
        g_hid = bf16_host(w.hidden).reshape(M, cfg.H)
        herr = np.abs(O.bf16_to_f64(g_hid) - O.bf16_to_f64(o_hid))
        assert herr.max() <= 2e-2 and herr.mean() <= 3e-3, (s, herr.max())
        if s % 25 == 0 or s == steps - 1:
            assert np.array_equal(bf16_host(w.k_pool), pool_k)
            assert np.array_equal(bf16_host(w.v_pool), pool_v)
        z_g = w.logits.cpu().numpy().reshape(M, V)
        z_h = O.lm_head(g_hid, Wh)
        bound = 1e-4 * (np.abs(O.bf16_to_f64(g_hid)) @ absW.T) + 1e-6
        assert np.all(np.abs(z_g - z_h) <= bound), s
        m_g, s_g, a_g = row_stats_host(w.row_stats)
        _, s_h, a_h = O.row_stats_all(z_g)
        assert np.array_equal(a_g, a_h)
        assert np.all(np.abs(s_g - s_h) <= OP.NEAR * s_h)
        r = S.unmask_batch(tok, st, kv, S.confidence(s_g).reshape(B, N), a_g.reshape(B, N), tau,
                           sync)
        assert np.array_equal(w.block_tok.cpu().numpy(), r["block_tok"]), s
        assert np.array_equal(w.steps.cpu().numpy(), r["steps"]), s
        assert np.array_equal(w.kv_len.cpu().numpy(), r["kv_len"]), s
        assert np.array_equal(w.unmasked_hist[s].cpu().numpy(), r["unmasked"]), s
        assert np.array_equal(w.out_tok_hist[s].cpu().numpy(), r["out_tok"]), s
        assert np.array_equal(w.block_steps_hist[s].cpu().numpy(), r["block_steps"]), s
        near_steps += int(_decisions_close(S.confidence(s_h).reshape(B, N), tok, tau).any())
        hist.append(r["block_steps"])
    assert int(w.err.item()) == 0
    final = {f: getattr(w, f).clone() for f in ("block_tok", "steps", "kv_len", "page_table",
                                                "k_pool", "v_pool", "logits")}
    hists = (w.unmasked_hist.clone(), w.out_tok_hist.clone(), w.block_steps_hist.clone())
    # the same forwards in one call, from the initial state
    # (the pool needs no reset: a block's rows are written before they are read)
    w.reset()
    w.run(steps, tau, sync)
    torch.cuda.synchronize()
    assert int(w.err.item()) == 0
    for f, t in final.items():
        assert torch.equal(getattr(w, f), t), f
    assert torch.equal(w.unmasked_hist, hists[0]) and torch.equal(w.out_tok_hist, hists[1])
    assert torch.equal(w.block_steps_hist, hists[2])
    return np.stack(hist), near_steps


@pytest.mark.parametrize("sync", [True, False])
def test_sdar_loop_stepwise(isd, sync):
    """A small stationary batch over 120 forwards, both scheduling modes."""
    cfg = I.IsdConfig("sdar_loop_small", B=5, N=4, Hq=8, Hkv=2, D=128, V=1000, page_size=16,
                      prefix_lo=1, prefix_hi=300, w_std=0.5, qkv_std=0.5, kv_std=1.0)
    tau = 0.3
    hist, near = _loop_stepwise(isd, cfg, 120, tau, sync, seed=2)
    rs = S.round_stats(hist, cfg.N) if sync else None
    left = hist > 0
    assert left.sum() >= cfg.B * 10
    if sync:
        # every round: all blocks leave together, after max S_b forwards and
        # the store pass
        rows = np.nonzero(left.any(axis=1))[0]
        assert np.all(left[rows].all(axis=1))
        gaps = np.diff(np.concatenate([[-1], rows]))
        assert np.array_equal(gaps, hist[rows].max(axis=1) + 1)
        assert rs["mean_max_S"] >= rs["mean_S"]
    record_parity(f"SDAR loop 120 forwards sync={sync}",
                  dict(requests=int(left.sum()), near_threshold=near, mismatches=0))


def test_sdar_loop_captured_in_cuda_graph(isd):
    """The SDAR loop captured once into a CUDA graph replays bit-identically
    to the eager run from the same state."""
    from speculative_verification_isd_b200.workload import SdarLoopWorkload
    cfg = I.IsdConfig("sdar_graph", B=6, N=4, Hq=8, Hkv=2, D=128, V=1000, page_size=16,
                      prefix_lo=1, prefix_hi=300, w_std=0.5, qkv_std=0.5, kv_std=1.0)
    n = 24
    w = SdarLoopWorkload(isd, cfg, capacity_steps=n, seed=4)
    args = w.args(0, n)
    w.run(n, 0.3, True, args=args)
    torch.cuda.synchronize()
    eager = [t.clone() for t in (w.block_steps_hist, w.out_tok_hist, w.kv_len, w.block_tok,
                                 w.logits)]
    w.reset()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            w.isd.sdar_loop(w.dims, 0.3, True, n, w.ws, err_flag=w.err, stream=s, args=args)
    torch.cuda.synchronize()
    w.reset()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert int(w.err.item()) == 0
    for a, b in zip(eager, (w.block_steps_hist, w.out_tok_hist, w.kv_len, w.block_tok,
                            w.logits)):
        assert torch.equal(a, b)
    del g


@pytest.mark.parametrize("case", ["b1_sync", "n1_block", "tau_above_one", "tau_zero"])
def test_sdar_loop_edge_cases(isd, case):
    """Degenerate batches and thresholds, one forward per call against the
    oracle: a batch of one; blocks of one position (every forward commits it,
    so a block costs 2 forwards with its store pass); tau above every
    confidence (S_b = N: one position per forward); tau = 0 (S_b = 1)."""
    B, N, tau = 4, 4, 0.3
    if case == "b1_sync":
        B = 1
    elif case == "n1_block":
        N = 1
    elif case == "tau_above_one":
        tau = 1.5
    elif case == "tau_zero":
        tau = 0.0
    cfg = I.IsdConfig("sdar_edge", B=B, N=N, Hq=8, Hkv=2, D=128, V=700, page_size=16,
                      prefix_lo=0, prefix_hi=200, w_std=0.5, qkv_std=0.5, kv_std=1.0)
    hist, _ = _loop_stepwise(isd, cfg, 24, tau, True, seed=11)
    left = hist[hist > 0]
    assert left.size > 0
    if case == "n1_block" or case == "tau_zero":
        assert np.all(left == 1)
    if case == "tau_above_one":
        assert np.all(left == N)


def test_sdar_bad_token_raises_flag(isd):
    """A committed block token outside [0, V) is reported through the error
    flag (the block row takes the MASK embedding); nothing faults."""
    from speculative_verification_isd_b200.workload import SdarLoopWorkload
    cfg = I.IsdConfig("sdar_flag", B=3, N=4, Hq=8, Hkv=2, D=128, V=700, page_size=16,
                      prefix_lo=0, prefix_hi=100, w_std=0.5, qkv_std=0.5, kv_std=1.0)
    w = SdarLoopWorkload(isd, cfg, capacity_steps=2, seed=1)
    w.block_tok[1, 2] = cfg.V + 5
    w.run(1, 0.3, True)
    torch.cuda.synchronize()
    assert int(w.err.item()) & isd.FLAG_TOKEN_OOB
    # the row was built from the MASK embedding
    q = bf16_host(w.q).reshape(cfg.B, cfg.N, cfg.Hq * cfg.D)
    Eq = bf16_host(w.Eq).reshape(cfg.V + 1, cfg.Hq, cfg.D)
    want, _, _ = S.embed_block({"Eq": Eq, "Ek": Eq[:, :cfg.Hkv], "Ev": Eq[:, :cfg.Hkv]},
                               np.array([[-1] * cfg.N]), cfg.V, np.array([int(w.kv0[1]) + 0]),
                               w.rope.cpu().numpy())
    assert np.array_equal(q[1, 2], want[0, 2].reshape(-1))
