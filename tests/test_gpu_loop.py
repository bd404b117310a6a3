"""The device-resident stationary-batch loop (isd_loop) against the oracle.

isd_loop runs n ISD steps with no host read in between: each step builds the
block's activations from the requests' state (token -> q, k, v table lookup),
extends each request's page list from a bump allocator, and runs the step,
with state, logits and row statistics in double buffers on the device.

1. Layered parity, every step: the loop is run one step per call; after each
   call the host reads the state and logits and the oracle checks every
   stage on the GPU's own inputs to it -- the block activations (table rows,
   bit-exact), the page table (a mirror of the allocator), the KV pool
   (bit-exact), attention, logits, and the accept decisions and tokens under
   the rules of oracle.parity (near-threshold decisions and rounding-explained
   draws counted and reported).
2. The same steps in ONE isd_loop call are bit-identical to the stepped run:
   every step's accept lengths and tokens, the final state, page table, KV
   pool and the last logits.
"""
import numpy as np
import pytest
import torch

from oracle import isd_oracle as O
from oracle import parity as OP
from speculative_verification_isd_b200 import inputs as I

from gpu_util import bf16_dev, bf16_host, f32_dev, i32_dev, record_parity, row_stats_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isd():
    from speculative_verification_isd_b200 import isd as lib
    return lib


def setup(isd, cfg, steps, seed):
    B, N, Q, V, P = cfg.B, cfg.N, cfg.Q, cfg.V, cfg.page_size
    inp = I.make_step_inputs(cfg, seed=seed, n_clean="one")
    tables = I.make_embedding_tables(cfg, seed=seed)
    kv0 = inp["kv_len"].astype(np.int32)
    # pool: the prefix pages first, then room for every step's growth
    pre = [(int(k) + P - 1) // P for k in kv0]
    max_pages = (int(kv0.max()) + steps * N + Q + P - 1) // P + 1
    num_pages = sum(pre) + B * max_pages
    table = np.full((B, max_pages), -1, np.int32)
    pool_k = np.zeros((num_pages, P, cfg.Hkv, cfg.D), np.uint16)
    pool_v = np.zeros_like(pool_k)
    nxt = 0
    for b in range(B):
        for i in range(pre[b]):
            table[b, i] = nxt
            nxt += 1
        for t in range(int(kv0[b])):
            src = inp["page_table"][b, t // P]
            pool_k[table[b, t // P], t % P] = inp["k_pool"][src, t % P]
            pool_v[table[b, t // P], t % P] = inp["v_pool"][src, t % P]
    rng = np.random.default_rng(seed)
    tok0 = np.full((B, N), -1, np.int32)
    tok0[:, 0] = rng.integers(0, V, B)
    u_all = np.stack([I.step_uniforms(seed, k, B, N) for k in range(steps)])
    d = isd.make_dims(B, N, cfg.Hq, cfg.Hkv, cfg.D, V, P, num_pages, max_pages)
    host = dict(inp=inp, tables=tables, kv0=kv0, pre=pre, max_pages=max_pages, table=table,
                pool_k=pool_k, pool_v=pool_v, nxt=nxt, tok0=tok0, u_all=u_all)
    return d, host


def device_buffers(d, cfg, host, steps):
    B, N, M, V = d.B, d.N, d.M, d.V
    return dict(
        Eq=bf16_dev(host["tables"]["Eq"]), Ek=bf16_dev(host["tables"]["Ek"]),
        Ev=bf16_dev(host["tables"]["Ev"]), W=bf16_dev(host["inp"]["W"]),
        k_pool=bf16_dev(host["pool_k"]), v_pool=bf16_dev(host["pool_v"]),
        page_table=i32_dev(host["table"]), pages_used=i32_dev(np.array(host["pre"], np.int32)),
        next_free_page=i32_dev(np.array([host["nxt"]], np.int32)),
        kv_len=i32_dev(np.stack([host["kv0"], np.zeros(B, np.int32)])),
        n_clean=i32_dev(np.stack([np.ones(B, np.int32), np.zeros(B, np.int32)])),
        clean_tok=i32_dev(np.stack([host["tok0"], np.full((B, N), -1, np.int32)])),
        logits=torch.zeros(2 * M * V, dtype=torch.float32, device="cuda"),
        row_stats=torch.zeros(2 * M * 4, dtype=torch.int32, device="cuda"),
        uniforms=f32_dev(host["u_all"][:steps]),
        q=torch.empty(M * cfg.Hq * cfg.D, dtype=torch.bfloat16, device="cuda"),
        k_new=torch.empty(M * cfg.Hkv * cfg.D, dtype=torch.bfloat16, device="cuda"),
        v_new=torch.empty(M * cfg.Hkv * cfg.D, dtype=torch.bfloat16, device="cuda"),
        hidden=torch.empty(M * d.H, dtype=torch.bfloat16, device="cuda"),
        accept_len_hist=torch.empty(steps * B, dtype=torch.int32, device="cuda"),
        out_tok_hist=torch.empty(steps * B * N, dtype=torch.int32, device="cuda"))


def run_loop(isd, cfg, steps, seed, label):
    B, N, Q, V, P = cfg.B, cfg.N, cfg.Q, cfg.V, cfg.page_size
    d, host = setup(isd, cfg, steps, seed)
    M = d.M
    inp, tables, max_pages = host["inp"], host["tables"], host["max_pages"]
    ws = isd.alloc_workspace(d)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    # ---------------- 1. one step per call, every stage against the oracle
    g = device_buffers(d, cfg, host, 1)
    pool_k, pool_v = host["pool_k"].copy(), host["pool_v"].copy()
    o_table, o_used, o_next = host["table"].copy(), list(host["pre"]), host["nxt"]
    absW = np.abs(O.bf16_to_f64(inp["W"]))
    prev = np.zeros((B, Q, V), np.float32)
    al_step, ot_step = [], []
    near, excused, draws, rejections = 0, 0, 0, 0
    for s in range(steps):
        kv = g["kv_len"][0].cpu().numpy()
        nc = g["n_clean"][0].cpu().numpy()
        tok = g["clean_tok"][0].cpu().numpy()
        g["uniforms"].view(-1).copy_(f32_dev(host["u_all"][s]).view(-1))
        isd.loop(d, 1, ws, err_flag=err, **g)
        torch.cuda.synchronize()
        # block activations and pages
        q, kn, vn = I.embed_block(tables, tok, nc, N, V)
        assert np.array_equal(bf16_host(g["q"]).reshape(q.shape), q)
        assert np.array_equal(bf16_host(g["k_new"]).reshape(kn.shape), kn)
        assert np.array_equal(bf16_host(g["v_new"]).reshape(vn.shape), vn)
        for b in range(B):
            need = min((int(kv[b]) + Q + P - 1) // P, max_pages)
            while o_used[b] < need:
                o_table[b, o_used[b]] = o_next
                o_used[b] += 1
                o_next += 1
        assert np.array_equal(g["page_table"].cpu().numpy().reshape(B, max_pages), o_table)
        # attention and the KV append
        o_hid, pool_k, pool_v = O.attention(q, kn, vn, pool_k, pool_v, o_table, kv, nc, N, P,
                                            cfg.D ** -0.5)
        g_hid = bf16_host(g["hidden"]).reshape(M, d.H)
        herr = np.abs(O.bf16_to_f64(g_hid) - O.bf16_to_f64(o_hid))
        assert herr.max() <= 2e-2 and herr.mean() <= 3e-3, (s, herr.max(), herr.mean())
        if s % 50 == 0 or s == steps - 1:
            assert np.array_equal(bf16_host(g["k_pool"]), pool_k)
            assert np.array_equal(bf16_host(g["v_pool"]), pool_v)
        # logits on the GPU's hidden
        z_g = g["logits"][: M * V].cpu().numpy().reshape(M, V)
        z_o = O.lm_head(g_hid, inp["W"])
        bound = 1e-4 * (np.abs(O.bf16_to_f64(g_hid)) @ absW.T) + 1e-6
        assert np.all(np.abs(z_g - z_o) <= bound), s
        m_g, s_g, a_g = row_stats_host(g["row_stats"][: M * 4])
        m_o, s_o, a_o = O.row_stats_all(z_g)
        assert np.array_equal(m_g, m_o.astype(np.float32).astype(np.float64))
        assert np.array_equal(a_g, a_o)
        assert np.all(np.abs(s_g - s_o) <= OP.NEAR * s_o)
        # acceptance on the GPU's logits
        L = z_g.reshape(B, Q, V)
        ores = O.accept(L, prev, nc, tok, kv, host["u_all"][s], N)
        al = g["accept_len_hist"].cpu().numpy()
        ot = g["out_tok_hist"].cpu().numpy().reshape(B, N)
        # the loop keeps no p/q ratios: its decisions are compared through the
        # accept lengths, states and tokens (the ratio kernel output is
        # covered by the single-step parity tests)
        gpu = dict(accept_len=al, out_tok=ot, next_n_clean=g["n_clean"][1].cpu().numpy(),
                   next_clean_tok=g["clean_tok"][1].cpu().numpy(),
                   next_kv_len=g["kv_len"][1].cpu().numpy(), ratio=ores["ratio"])
        rep = OP.compare_accept(gpu, ores, L, prev, dict(n_clean=nc, uniforms=host["u_all"][s]),
                                N, O.PROPOSE_ARGMAX)
        assert rep["mismatches"] == 0, (s, rep["first_mismatch"])
        near += rep["near_threshold"]
        excused += rep["excused_draws"]
        draws += rep["draws"]
        rejections += int((ores["rejected_at"] > 0).sum())
        al_step.append(al.copy())
        ot_step.append(ot.copy())
        # the next step: this step's next state and logits become the inputs
        for k in ("kv_len", "n_clean", "clean_tok"):
            g[k][0].copy_(g[k][1])
        g["logits"][M * V:].copy_(g["logits"][: M * V])
        g["row_stats"][M * 4:].copy_(g["row_stats"][: M * 4])
        prev = L.copy()
    assert int(err.item()) == 0
    record_parity(f"{label}, one step per call", dict(requests=steps * B, near_threshold=near,
                                                     draws=draws, excused_draws=excused,
                                                     mismatches=0))
    assert near + excused <= max(2, steps * B // 100)

    # ---------------- 2. the same steps in one call
    g2 = device_buffers(d, cfg, host, steps)
    isd.loop(d, steps, ws, err_flag=err, **g2)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(g2["accept_len_hist"].cpu().numpy().reshape(steps, B), np.stack(al_step))
    assert np.array_equal(g2["out_tok_hist"].cpu().numpy().reshape(steps, B, N), np.stack(ot_step))
    fin = steps & 1
    for k in ("kv_len", "n_clean", "clean_tok"):
        assert torch.equal(g2[k][fin], g[k][0]), k
    assert torch.equal(g2["page_table"], g["page_table"])
    assert torch.equal(g2["next_free_page"], g["next_free_page"])
    assert torch.equal(g2["k_pool"], g["k_pool"]) and torch.equal(g2["v_pool"], g["v_pool"])
    last = (steps - 1) & 1
    assert torch.equal(g2["logits"][last * M * V:(last + 1) * M * V], g["logits"][: M * V])
    return np.stack(al_step), rejections, draws


def test_loop_tiny_1000_steps(isd):
    """The tiny configuration (B=2, N=2, V=512), 1000 consecutive steps."""
    al, _, _ = run_loop(isd, I.CONFIGS["tiny"], 1000, 0, "device loop, tiny 1000 steps")
    assert al.sum() >= 1000 * 2


def test_loop_with_rejections(isd):
    """Wider logits (rejections, residual draws, restarts) at B=4, N=4."""
    cfg = I.IsdConfig("loop_ragged", B=4, N=4, Hq=8, Hkv=2, D=128, V=1000, page_size=16,
                      prefix_lo=3, prefix_hi=200, w_std=0.4, qkv_std=0.5, kv_std=1.0)
    al, rejections, draws = run_loop(isd, cfg, 150, 5, "device loop, B=4 N=4 with rejections")
    # every outcome occurs after the first step: restarts (accept length 1),
    # partial and full accepts, and rejections with a residual draw
    later = al[1:]
    assert (later == 1).any() and (later == cfg.N).any() and ((later > 1) & (later < cfg.N)).any()
    assert rejections >= 20 and draws >= 20


def _ids(tok, nc, N, V):
    Q = 2 * N - 1
    ids = np.full((tok.shape[0], Q), V, np.int64)
    for b in range(tok.shape[0]):
        ids[b, : int(nc[b])] = tok[b, : int(nc[b])]
    return ids


def test_loop_full_shape_b32_n4(isd):
    """Headline shape (B=32, N=4, Qwen3-8B sizes, prefixes U[512, 8192], the
    benchmark's closed-loop model).  Ten steps one per call: every block row
    equals its table row, the page table follows the allocator's rule, the KV
    append put each block slot's key/value at its position, the row statistics
    match the GPU's logits, sampled logits match the oracle's dot products,
    and the accept decisions, tokens and next states match the oracle's on the
    GPU's logits.  Then the same ten steps in one call are bit-identical."""
    from speculative_verification_isd_b200.workload import LoopWorkload
    cfg = I.CONFIGS["qwen3_8b_b32_n4"]
    B, N, Q, V, P = cfg.B, cfg.N, cfg.Q, cfg.V, cfg.page_size
    steps = 10
    mk = lambda: LoopWorkload(isd, cfg, capacity_steps=steps, seed=2, w_std=0.1, qkv_std=0.5,
                              kv_std=1.0)
    lw = mk()
    d, M = lw.dims, lw.dims.M
    maxp = d.max_pages_per_req
    t = {f: getattr(lw, f) for f in lw.FIELDS}
    hist_al = torch.zeros(1, B, dtype=torch.int32, device="cuda")
    hist_ot = torch.zeros(1, B, N, dtype=torch.int32, device="cuda")
    o_table = lw.page_table.cpu().numpy().reshape(B, maxp).copy()
    o_used = (lw.kv0.astype(np.int64) + P - 1) // P
    o_next = int(lw.next_free_page.item())
    W_h = bf16_host(lw.W).reshape(V, d.H)
    rng = np.random.default_rng(4)
    prev = np.zeros((B, Q, V), np.float32)
    al_step, ot_step = [], []
    near = excused = draws = 0
    for s in range(steps):
        kv = lw.kv_len[0].cpu().numpy()
        nc = lw.n_clean[0].cpu().numpy()
        tok = lw.clean_tok[0].cpu().numpy()
        u = lw.uniforms[s].cpu().numpy()
        isd.loop(d, 1, lw.ws, err_flag=lw.err, uniforms=lw.uniforms[s:s + 1],
                 accept_len_hist=hist_al, out_tok_hist=hist_ot, **t)
        torch.cuda.synchronize()
        # block rows are table rows
        ids = torch.from_numpy(_ids(tok, nc, N, V).reshape(-1)).cuda()
        assert torch.equal(lw.q.view(M, -1), lw.Eq.view(V + 1, -1)[ids])
        assert torch.equal(lw.k_new.view(M, -1), lw.Ek.view(V + 1, -1)[ids])
        assert torch.equal(lw.v_new.view(M, -1), lw.Ev.view(V + 1, -1)[ids])
        # pages: ceil((kv_len + Q) / P) per request, new ones in request order
        for b in range(B):
            need = min((int(kv[b]) + Q + P - 1) // P, maxp)
            while o_used[b] < need:
                o_table[b, o_used[b]] = o_next
                o_used[b] += 1
                o_next += 1
        table = lw.page_table.cpu().numpy().reshape(B, maxp)
        assert np.array_equal(table, o_table)
        # the KV append: every active block slot's key/value at its position
        rows, pos = [], []
        for b in range(B):
            p_b = O.slot_positions(int(kv[b]), int(nc[b]), N)
            for i in range(Q):
                if p_b[i] >= 0:
                    rows.append(b * Q + i)
                    pos.append(int(p_b[i]))
        rows_t = torch.tensor(rows, dtype=torch.long, device="cuda")
        pos = np.array(pos)
        bidx = np.array(rows) // Q
        pages = torch.from_numpy(table[bidx, pos // P].astype(np.int64)).cuda()
        offs = torch.from_numpy(pos % P).long().cuda()
        assert torch.equal(lw.k_pool[pages, offs].view(len(rows), -1), lw.k_new.view(M, -1)[rows_t])
        assert torch.equal(lw.v_pool[pages, offs].view(len(rows), -1), lw.v_new.view(M, -1)[rows_t])
        # logits: sampled entries against the oracle's dot products on the
        # GPU's hidden, row statistics of every row against the GPU's logits
        z_g = lw.logits[: M * V].view(M, V).cpu().numpy()
        hid = bf16_host(lw.hidden).reshape(M, d.H)
        for m, v in zip(rng.integers(0, M, 48), rng.integers(0, V, 48)):
            ref = O.lm_head_entry(hid[m], W_h[v])
            bound = 1e-4 * float(np.abs(O.bf16_to_f64(hid[m])) @ np.abs(O.bf16_to_f64(W_h[v]))) + 1e-6
            assert abs(float(z_g[m, v]) - ref) <= bound, (s, m, v)
        m_g, s_g, a_g = row_stats_host(lw.row_stats[: M * 4])
        m_o, s_o, a_o = O.row_stats_all(z_g)
        assert np.array_equal(m_g, m_o.astype(np.float32).astype(np.float64))
        assert np.array_equal(a_g, a_o)
        assert np.all(np.abs(s_g - s_o) <= OP.NEAR * s_o)
        # acceptance on the GPU's logits
        L = z_g.reshape(B, Q, V)
        ores = O.accept(L, prev, nc, tok, kv, u, N)
        al = hist_al[0].cpu().numpy()
        ot = hist_ot[0].cpu().numpy()
        gpu = dict(accept_len=al, out_tok=ot, next_n_clean=lw.n_clean[1].cpu().numpy(),
                   next_clean_tok=lw.clean_tok[1].cpu().numpy(),
                   next_kv_len=lw.kv_len[1].cpu().numpy(), ratio=ores["ratio"])
        rep = OP.compare_accept(gpu, ores, L, prev, dict(n_clean=nc, uniforms=u), N,
                                O.PROPOSE_ARGMAX)
        assert rep["mismatches"] == 0, (s, rep["first_mismatch"])
        near += rep["near_threshold"]
        excused += rep["excused_draws"]
        draws += rep["draws"]
        al_step.append(al.copy())
        ot_step.append(ot.copy())
        for k in ("kv_len", "n_clean", "clean_tok"):
            getattr(lw, k)[0].copy_(getattr(lw, k)[1])
        lw.logits[M * V:].copy_(lw.logits[: M * V])
        lw.row_stats[M * 4:].copy_(lw.row_stats[: M * 4])
        prev = L.copy()
    assert int(lw.err.item()) == 0
    record_parity("device loop, B=32 N=4 full shape, one step per call",
                  dict(requests=steps * B, near_threshold=near, draws=draws,
                       excused_draws=excused, mismatches=0))
    assert near <= max(1, steps * B // 50) and excused <= max(1, draws // 50)
    # restarts and full accepts both occur
    al_all = np.stack(al_step)
    assert (al_all[1:] == N).any() and (al_all[2:] < N).any()

    # the same steps in one call
    lw2 = mk()
    lw2.run(steps)
    torch.cuda.synchronize()
    assert int(lw2.err.item()) == 0
    assert np.array_equal(lw2.accept_len_hist.cpu().numpy(), al_all)
    assert np.array_equal(lw2.out_tok_hist.cpu().numpy(), np.stack(ot_step))
    fin = steps & 1
    for k in ("kv_len", "n_clean", "clean_tok"):
        assert torch.equal(getattr(lw2, k)[fin], getattr(lw, k)[0]), k
    assert torch.equal(lw2.page_table, lw.page_table)
    assert torch.equal(lw2.next_free_page, lw.next_free_page)
    assert torch.equal(lw2.k_pool, lw.k_pool) and torch.equal(lw2.v_pool, lw.v_pool)
    last = (steps - 1) & 1
    assert torch.equal(lw2.logits[last * M * V:(last + 1) * M * V], lw.logits[: M * V])


def test_loop_captured_in_cuda_graph(isd):
    """isd_loop captured once in a CUDA graph (the launches are capturable: no
    host reads, allocations or memsets) replays bit-identically to the same
    steps run eagerly from the same state."""
    cfg = I.CONFIGS["tiny"]
    steps = 64
    d, host = setup(isd, cfg, steps, 3)
    ws = isd.alloc_workspace(d)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    eager = device_buffers(d, cfg, host, steps)
    isd.loop(d, steps, ws, err_flag=err, **eager)
    torch.cuda.synchronize()
    cap = device_buffers(d, cfg, host, steps)
    args = isd.loop_args(d, steps, **cap)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        isd.loop(d, steps, ws, err_flag=err, stream=torch.cuda.current_stream(), args=args)
    graph.replay()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for k in eager:
        assert torch.equal(eager[k], cap[k]), k
    assert int(cap["accept_len_hist"].sum().item()) >= steps * cfg.B
