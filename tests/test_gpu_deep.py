"""The full-depth forward (isd_embed_block + isd_layers) on the GPU against
the oracle (oracle.forward_oracle), layer by layer.

Each layer runs alone (one isd_layers call of one layer) on the GPU's own
input to it; the oracle computes that layer from the same bf16 input, the same
bf16 weights and the same cache, with the kernels' rounding points.  The
outputs are bf16 after several fp32 reductions whose order differs from the
oracle's float64 sums, so they are compared to a few bf16 ulps of the value's
magnitude; the K/V rows appended to each layer's pool likewise.  Positions
past the appended rows keep their bytes exactly.
"""
import numpy as np
import pytest
import torch

from oracle import forward_oracle as F
from oracle import isd_oracle as O
from speculative_verification_isd_b200 import inputs as I

from gpu_util import bf16_host, record_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isd():
    from speculative_verification_isd_b200 import isd as lib
    return lib


DEEP = {
    # general attention path (D = 64) and the tensor-core path (D = 128)
    "deep_d64": (I.IsdConfig("deep_d64", B=3, N=4, Hq=4, Hkv=2, D=64, V=1000, page_size=16,
                             prefix_lo=1, prefix_hi=300, w_std=0.5), 2, 512),
    "deep_d128": (I.IsdConfig("deep_d128", B=3, N=4, Hq=8, Hkv=2, D=128, V=1000, page_size=16,
                              prefix_lo=1, prefix_hi=300, w_std=0.5), 2, 1024),
    # a wide MLP (intermediate 8192 against hidden 1024), one layer
    "deep_wide": (I.IsdConfig("deep_wide", B=3, N=4, Hq=8, Hkv=2, D=128, V=1000, page_size=16,
                              prefix_lo=1, prefix_hi=300, w_std=0.5), 1, 8192),
}


def _ulp_close(got, want, what, ulps=4.0, mean_frac=0.01):
    """|got - want| within `ulps` bf16 ulps of the largest |want| of its row,
    and on average within mean_frac of the mean |want|."""
    g = np.asarray(got, np.float64)
    w = np.asarray(want, np.float64)
    scale = np.abs(w).max(axis=-1, keepdims=True) + 1e-30
    ulp = 2.0 ** (np.floor(np.log2(scale)) - 7)
    err = np.abs(g - w)
    assert np.all(err <= ulps * ulp), (what, float((err / ulp).max()))
    assert err.mean() <= mean_frac * np.abs(w).mean() + 1e-30, (what, float(err.mean()))


def _host_layer(L):
    return {k: bf16_host(t).reshape(t.shape) for k, t in L.items()}


def _check_stack(isd, w, N, n_clean, requests=None):
    """Embed, then every layer alone against the oracle, then the final norm.
    requests: the subset the oracle recomputes (all by default)."""
    cfg = w.cfg
    v = w.views[N]
    d = v["dims"]
    B, Q, H, P = cfg.B, v["Q"], w.H, cfg.page_size
    v["n_clean"].copy_(torch.from_numpy(np.asarray(n_clean, np.int32)).cuda())
    isd.embed_block(d, w.E, v["n_clean"], v["clean_tok"], v["x"], err_flag=v["err"])
    torch.cuda.synchronize()
    nc = v["n_clean"].cpu().numpy()
    tok = v["clean_tok"].cpu().numpy()
    Eh = bf16_host(w.E).reshape(cfg.V + 1, H)
    ids = np.full((B, Q), cfg.V)
    for b in range(B):
        ids[b, : nc[b]] = tok[b, : nc[b]]
    assert np.array_equal(bf16_host(v["x"]).reshape(B, Q, H), Eh[ids])
    req = np.arange(B) if requests is None else np.asarray(requests)
    kv = v["kv_len"].cpu().numpy()
    table = w.page_table.cpu().numpy()
    rope = w.rope.cpu().numpy()
    pos = F.block_positions(kv[req], nc[req], N)
    active = np.zeros((len(req), Q), bool)
    for i, b in enumerate(req):
        active[i, : nc[b]] = True
        active[i, N:] = True
    # the oracle's pools: only the pages of the checked requests, renumbered
    pages = [table[b][table[b] >= 0] for b in req]
    flat = np.concatenate(pages)
    loc_table = np.full((len(req), table.shape[1]), -1, np.int32)
    o = 0
    for i, pg in enumerate(pages):
        loc_table[i, : len(pg)] = np.arange(o, o + len(pg))
        o += len(pg)
    flat_t = torch.from_numpy(flat.astype(np.int64)).cuda()
    worst = 0.0
    for l, L in enumerate(w.layers):
        x_in = bf16_host(v["x"]).reshape(B, Q, H)[req]
        Lh = {k: t for k, t in _host_layer(L).items() if k not in ("k_pool", "v_pool")}
        Lh["k_pool"] = O.bf16_to_f64(bf16_host(L["k_pool"][flat_t]))
        Lh["v_pool"] = O.bf16_to_f64(bf16_host(L["v_pool"][flat_t]))
        before_k = bf16_host(L["k_pool"][flat_t])
        arr = isd.layer_array(d, w.inter, [L])
        isd.layers(d, w.inter, w.eps, arr, 1, w.rope, v["x"], w.page_table, v["kv_len"],
                   v["n_clean"], v["ws"], err_flag=v["err"])
        torch.cuda.synchronize()
        assert int(v["err"].item()) == 0
        want, st = F.layer(O.bf16_to_f64(x_in), Lh, active, pos, loc_table, P, cfg.Hq, cfg.Hkv,
                           cfg.D, w.eps, rope, exact=False)
        got = O.bf16_to_f64(bf16_host(v["x"]).reshape(B, Q, H)[req])
        _ulp_close(got, want, f"layer {l} output")
        worst = max(worst, float(np.abs(got - want).max() / np.abs(want).max()))
        # the appended K/V rows (active slots) match; every other row kept its bytes
        after_k = bf16_host(L["k_pool"][flat_t])
        after_v = bf16_host(L["v_pool"][flat_t])
        touched = np.zeros(after_k.shape[:2], bool)
        for i in range(len(req)):
            for s in range(Q):
                if active[i, s]:
                    t = int(pos[i, s])
                    touched[loc_table[i, t // P], t % P] = True
        assert np.array_equal(after_k[~touched], before_k[~touched]), l
        _ulp_close(O.bf16_to_f64(after_k[touched]), Lh["k_pool"][touched], f"layer {l} K rows")
        _ulp_close(O.bf16_to_f64(after_v[touched]), Lh["v_pool"][touched], f"layer {l} V rows")
    # the final norm alone
    isd.layers(d, w.inter, w.eps, isd.layer_array(d, w.inter, []), 0, w.rope, v["x"],
               w.page_table, v["kv_len"], v["n_clean"], v["ws"], final_norm=w.final_norm,
               out=v["out"], err_flag=v["err"])
    torch.cuda.synchronize()
    xr = O.bf16_to_f64(bf16_host(v["x"]).reshape(B, Q, H)[req])
    want = O.bf16_to_f64(O.f64_to_bf16(F.rmsnorm(xr, O.bf16_to_f64(bf16_host(w.final_norm)),
                                                 w.eps)))
    _ulp_close(O.bf16_to_f64(bf16_host(v["out"]).reshape(B, Q, H)[req]), want, "final norm",
               ulps=1.0, mean_frac=0.002)
    return worst


@pytest.mark.parametrize("name", list(DEEP))
@pytest.mark.parametrize("mode", ["full", "mixed"])
def test_layers_against_oracle(isd, name, mode):
    from speculative_verification_isd_b200.workload import DeepWorkload
    cfg, n_layers, inter = DEEP[name]
    w = DeepWorkload(isd, cfg, n_layers, inter, seed=3)
    nc = np.full(cfg.B, cfg.N) if mode == "full" else np.array([1, 3, cfg.N])[: cfg.B]
    worst = _check_stack(isd, w, cfg.N, nc)
    record_parity(f"deep stack {name} n_clean={mode} (max rel err {worst:.2e})",
                  dict(requests=cfg.B, near_threshold=0, mismatches=0))


def test_layers_ar_stride_one(isd):
    """N = 1 (one query per request: autoregressive decoding) on the same stack."""
    from speculative_verification_isd_b200.workload import DeepWorkload
    cfg, n_layers, inter = DEEP["deep_d128"]
    w = DeepWorkload(isd, cfg, n_layers, inter, seed=4)
    w.view(1)
    _check_stack(isd, w, 1, np.ones(cfg.B, np.int32))


@pytest.mark.parametrize("N", [4, 1])
def test_layers_full_size_sampled(isd, N):
    """Two layers at the Qwen3-8B shapes (H 4096, 32/8 heads of 128,
    intermediate 12288) over the B=32 block at stride N (N = 1: AR decoding);
    the oracle recomputes three requests (rows are independent in every GEMM,
    requests in the attention)."""
    from speculative_verification_isd_b200.workload import DeepWorkload
    cfg = I.CONFIGS["qwen3_8b_b32_n4"]
    w = DeepWorkload(isd, cfg, 2, 12288, seed=5)
    w.view(N)
    worst = _check_stack(isd, w, N, np.full(cfg.B, N), requests=[0, 15, 31])
    record_parity(f"deep stack qwen3_8b_b32 N={N} 2 layers sampled (max rel err {worst:.2e})",
                  dict(requests=3, near_threshold=0, mismatches=0))


def test_deep_step_runs_lm_head_and_accept(isd):
    """A whole full-depth step (embed, layers, final norm, LM head, accept)
    runs and its logits are the LM head of its own final hidden rows."""
    from speculative_verification_isd_b200.workload import DeepWorkload
    cfg, n_layers, inter = DEEP["deep_d128"]
    w = DeepWorkload(isd, cfg, n_layers, inter, seed=6)
    v = w.views[cfg.N]
    w.step(cfg.N)
    torch.cuda.synchronize()
    assert int(v["err"].item()) == 0
    h = bf16_host(v["out"]).reshape(v["M"], w.H)
    z = v["logits"].cpu().numpy().reshape(v["M"], cfg.V)
    Wh = bf16_host(w.W).reshape(cfg.V, w.H)
    ref = O.lm_head(h, Wh)
    bound = 1e-4 * (np.abs(O.bf16_to_f64(h)) @ np.abs(O.bf16_to_f64(Wh)).T) + 1e-6
    assert np.all(np.abs(z - ref) <= bound)
    al = v["accept_len"].cpu().numpy()
    assert np.all((al >= 1) & (al <= cfg.N))


def test_short_rope_table_raises_flag(isd):
    """Positions past the rotary table are reported (ISD_FLAG_CAPACITY) and
    use its last row; nothing faults."""
    from speculative_verification_isd_b200.workload import DeepWorkload
    cfg, _, inter = DEEP["deep_d128"]
    w = DeepWorkload(isd, cfg, 1, inter, seed=8)
    v = w.views[cfg.N]
    short = w.rope[:4].contiguous()
    isd.embed_block(v["dims"], w.E, v["n_clean"], v["clean_tok"], v["x"], err_flag=v["err"])
    isd.layers(v["dims"], w.inter, w.eps, v["layer_arr"], 1, short, v["x"], w.page_table,
               v["kv_len"], v["n_clean"], v["ws"], err_flag=v["err"])
    torch.cuda.synchronize()
    assert int(v["err"].item()) & isd.FLAG_CAPACITY
