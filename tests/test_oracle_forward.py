"""Pins of the full-depth forward oracle (oracle.forward_oracle): the decoder
layer against transformers' Qwen3 implementation in float64 (a library
routine), the ISD positions by hand, and the element-wise pieces against
closed forms and torch (no GPU needed)."""
import math

import numpy as np
import pytest
import torch

from oracle import forward_oracle as F
from oracle import isd_oracle as O


def _hf_layers(n_layers, H, I, Hq, Hkv, D, eps, seed):
    from transformers.models.qwen3.modeling_qwen3 import (Qwen3Config, Qwen3DecoderLayer,
                                                          Qwen3RMSNorm, Qwen3RotaryEmbedding)
    cfg = Qwen3Config(hidden_size=H, intermediate_size=I, num_attention_heads=Hq,
                      num_key_value_heads=Hkv, head_dim=D, num_hidden_layers=n_layers,
                      vocab_size=64, rms_norm_eps=eps, rope_theta=1.0e6, attention_bias=False)
    cfg._attn_implementation = "eager"
    torch.manual_seed(seed)
    layers = [Qwen3DecoderLayer(cfg, layer_idx=i).double().eval() for i in range(n_layers)]
    for L in layers:
        for p in L.parameters():
            with torch.no_grad():
                p.copy_(torch.randn_like(p) * (0.2 if p.dim() == 2 else 1.0)
                        + (1.0 if p.dim() == 1 else 0.0))
    norm = Qwen3RMSNorm(H, eps=eps).double()
    with torch.no_grad():
        norm.weight.copy_(torch.rand(H, dtype=torch.float64) + 0.5)
    rot = Qwen3RotaryEmbedding(cfg)
    return cfg, layers, norm, rot


def _ours_from_hf(L, Hkv, D, pages, P):
    a = L.self_attn
    m = L.mlp
    t = lambda p: p.detach().double().numpy().copy()
    return dict(in_norm=t(L.input_layernorm.weight),
                w_qkv=np.concatenate([t(a.q_proj.weight), t(a.k_proj.weight), t(a.v_proj.weight)]),
                q_norm=t(a.q_norm.weight), k_norm=t(a.k_norm.weight), w_o=t(a.o_proj.weight),
                post_norm=t(L.post_attention_layernorm.weight),
                w_gate_up=np.concatenate([t(m.gate_proj.weight), t(m.up_proj.weight)]),
                w_down=t(m.down_proj.weight),
                k_pool=np.zeros((pages, P, Hkv, D)), v_pool=np.zeros((pages, P, Hkv, D)))


def _hf_forward(layers, norm, rot, x, T):
    pos = torch.arange(T)[None]
    cos, sin = rot(x, pos)
    mask = torch.full((T, T), float("-inf"), dtype=torch.float64).triu(1)[None, None]
    h = x
    for L in layers:
        out = L(h, attention_mask=mask, position_ids=pos, position_embeddings=(cos, sin))
        h = out[0] if isinstance(out, tuple) else out
    return norm(h), h, cos, sin


@pytest.mark.parametrize("prefix", [0, 5])
def test_stack_equals_transformers_qwen3(prefix):
    """Two layers and the final norm, float64, no rounding points (exact):
    the oracle's rows equal transformers' Qwen3 decoder layers with a causal
    mask over [prefix; block].  With a prefix, the oracle first runs the
    prefix rows through the same layers (filling each layer's paged pool)
    and then the 7 block rows against the cache."""
    H, I, Hq, Hkv, D, eps = 64, 96, 4, 2, 16, 1e-6
    _, layers, norm, rot = _hf_layers(2, H, I, Hq, Hkv, D, eps, seed=prefix)
    S = 7
    T = prefix + S
    torch.manual_seed(100 + prefix)
    x = torch.randn(1, T, H, dtype=torch.float64)
    want_out, want_res, cos, sin = _hf_forward(layers, norm, rot, x, T)
    # HF's own cos/sin as the rotation table: [T, D/2, 2]
    tab = np.stack([cos[0, :, : D // 2].numpy(), sin[0, :, : D // 2].numpy()], axis=-1)
    P = 4
    pages = (T + P - 1) // P
    table = np.arange(pages, dtype=np.int32)[None] [:, ::-1].copy()  # pages in reverse order
    ours = [_ours_from_hf(L, Hkv, D, pages, P) for L in layers]
    xs = x.numpy()
    if prefix:
        h = xs[:, :prefix]
        act = np.ones((1, prefix), bool)
        pos = np.arange(prefix)[None]
        for L in ours:
            h, _ = F.layer(h, L, act, pos, table, P, Hq, Hkv, D, eps, tab, exact=True)
    h = xs[:, prefix:]
    act = np.ones((1, S), bool)
    pos = np.arange(prefix, T)[None]
    for L in ours:
        h, st = F.layer(h, L, act, pos, table, P, Hq, Hkv, D, eps, tab, exact=True)
    out = F.rmsnorm(h, norm.weight.detach().numpy(), eps)
    # transformers' RMSNorm takes its statistics in float32 whatever the
    # input dtype, so the two agree to float32 precision, not float64; any
    # structural slip (a pair, a norm, a residual, a head mapping) is O(1)
    want_r = want_res[:, prefix:].detach().numpy()
    want_o = want_out[:, prefix:].detach().numpy()
    assert np.abs(h - want_r).max() <= 2e-6 * np.abs(want_r).max()
    assert np.abs(out - want_o).max() <= 2e-6 * np.abs(want_o).max()


def test_block_positions_by_hand():
    # c = 2 of N = 4 at kv_len 100: clean 100..103 (2 inactive), MASK 102..104
    pos = F.block_positions([100], [2], 4)
    assert list(pos[0]) == [100, 101, 102, 103, 102, 103, 104]
    assert list(F.block_positions([0], [4], 4)[0]) == list(range(7))
    # active slots match the single-layer oracle's slot layout
    sp = O.slot_positions(37, 3, 4)
    fp = F.block_positions([37], [3], 4)[0]
    assert all(s < 0 or s == f for s, f in zip(sp, fp))


def test_elementwise_pieces():
    # RMSNorm of a constant vector is the weight (times the sign)
    w = np.linspace(0.5, 2.0, 8)
    assert np.allclose(F.rmsnorm(np.full(8, -3.0), w, 0.0), -w)
    assert np.allclose(F.rmsnorm(np.full(8, 3.0), w, 1e-6), w * 3 / math.sqrt(9 + 1e-6))
    z = np.linspace(-8, 8, 101)
    assert np.allclose(F.silu(z), torch.nn.functional.silu(torch.from_numpy(z)).numpy(), rtol=1e-14)
    # RoPE: position 0 is the identity, pairs are (i, i + D/2)
    x = np.arange(8.0)
    ident = np.stack([np.ones(4), np.zeros(4)], -1)
    assert np.array_equal(F.rope(x, ident), x)
    quarter = np.stack([np.zeros(4), np.ones(4)], -1)   # rotate by pi/2
    assert np.array_equal(F.rope(x, quarter), np.concatenate([-x[4:], x[:4]]))


def test_rounding_points_stay_near_exact():
    """The kernels' rounding points (exact=False) move the result by a few
    bf16 ulps, not more (the same inputs, one layer)."""
    H, I, Hq, Hkv, D, eps = 64, 96, 4, 2, 16, 1e-6
    _, layers, norm, rot = _hf_layers(1, H, I, Hq, Hkv, D, eps, seed=7)
    T, P = 7, 4
    x = O.bf16_to_f64(O.f64_to_bf16(torch.randn(1, T, H, dtype=torch.float64).numpy()))
    _, _, cos, sin = _hf_forward(layers, norm, rot, torch.from_numpy(x), T)
    tab = np.stack([cos[0, :, : D // 2].numpy(), sin[0, :, : D // 2].numpy()], axis=-1)
    table = np.arange(2, dtype=np.int32)[None]
    act, pos = np.ones((1, T), bool), np.arange(T)[None]
    a, _ = F.layer(x, _ours_from_hf(layers[0], Hkv, D, 2, P), act, pos, table, P, Hq, Hkv, D,
                   eps, tab, exact=True)
    b, _ = F.layer(x, _ours_from_hf(layers[0], Hkv, D, 2, P), act, pos, table, P, Hq, Hkv, D,
                   eps, tab, exact=False)
    assert np.abs(a - b).max() <= 0.05 * np.abs(a).max()
    assert np.abs(a - b).mean() <= 0.02 * np.abs(a).mean()   # about one bf16 ulp (2^-8) on average
