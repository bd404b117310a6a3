"""CPU oracle of the full-depth synthetic I-DLM forward over an ISD block.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import or run this module.  The product path
never calls it, and this module imports nothing from the product package.

What the pages fix: I-DLM keeps the autoregressive model's stack and serving
path ([EXP] "I-DLM：扩散模型如何用“自省一致性”追上自回归模型质量", section
"推理：复用 AR 推理栈"); its 8B model is built from Qwen3-8B (the pages'
benchmark tables); every query slot of the 2N-1 block goes through the whole
stack in one forward; and in memory-bound decoding the forward's latency
hardly depends on how many tokens it carries, so the speed-up over AR is about
TPF ([PRJ] I-DLM project page, the TPF paragraphs).  The layer internals are
not in the pages; the plainest reading is the base model's decoder layer
(Qwen3):

  F1  x <- x + O(attn(RoPE(qk_norm(QKV(rmsnorm_in(x))))))
      x <- x + down(silu(gate(h)) * up(h)),  h = rmsnorm_post(x)
      and after the last layer the final RMSNorm feeds the LM head.
  F2  Every layer attends with the ISD slot layout and strict-causal mask of
      the single-layer step (oracle.isd_oracle.slot_positions), each layer
      with its own paged K/V pool under the same page table.
  F3  RoPE at each slot's absolute position, rotate-half pairs (i, i + D/2),
      with a (cos, sin) table given as input; q and k are RMS-normalised per
      head (weights q_norm, k_norm) before the rotation.  Inactive clean
      slots take position kv_len + s like active ones (their outputs are
      never used).
  F4  Rounding points (those of the kernels; exact=True drops them, for the
      pin against a library implementation in float64): every RMSNorm output,
      every GEMM output (the residual added before that rounding for the O
      and down projections), q and k after norm + rotation, the attention
      output, silu(gate) * up.  Everything between two rounding points is
      float64 here.

bf16 tensors are uint16 bit patterns, as in oracle.isd_oracle.
"""
from __future__ import annotations

from typing import Dict, List

import numpy as np

from oracle import isd_oracle as O


def _rounder(exact: bool):
    if exact:
        return lambda a: np.asarray(a, dtype=np.float64)
    return lambda a: O.bf16_to_f64(O.f64_to_bf16(np.asarray(a, dtype=np.float64)))


def f64(bits_or_f64, exact: bool):
    """Weights and inputs: bf16 bit patterns -> float64 (exact inputs pass)."""
    a = np.asarray(bits_or_f64)
    return a.astype(np.float64) if a.dtype != np.uint16 else O.bf16_to_f64(a)


def rmsnorm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * w over the last axis (float64)."""
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * w


def rope(x: np.ndarray, cs: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE of x [..., D] with table rows cs [..., D/2, 2]
    (cos, sin): x_i cos - x_{i+D/2} sin, x_{i+D/2} cos + x_i sin."""
    h = x.shape[-1] // 2
    c = cs[..., 0].astype(np.float64)
    s = cs[..., 1].astype(np.float64)
    lo, hi = x[..., :h], x[..., h:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def block_positions(kv_len, n_clean, N: int) -> np.ndarray:
    """[B, 2N-1] positions of every slot (F3): clean slot s at kv_len + s
    (active or not), MASK slot m at kv_len + c + m."""
    B = len(kv_len)
    pos = np.zeros((B, 2 * N - 1), np.int64)
    for b in range(B):
        kv, c = int(kv_len[b]), int(n_clean[b])
        for s in range(N):
            pos[b, s] = kv + s
        for m in range(N - 1):
            pos[b, N + m] = kv + c + m
    return pos


def attention_rows(q, k, v, active, pos, k_pool, v_pool, page_table, P, sm_scale):
    """Append the active rows' K/V at their positions, then strict-causal GQA
    attention of every active row over keys 0..pos (float64; the pools hold
    float64 values).  q [B,S,Hq,D], k/v [B,S,Hkv,D], active/pos [B,S].
    Inactive rows give zero output.  Pools are modified in place."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    for b in range(B):
        for s in range(S):
            if active[b, s]:
                t = int(pos[b, s])
                page = int(page_table[b, t // P])
                k_pool[page, t % P] = k[b, s]
                v_pool[page, t % P] = v[b, s]
    out = np.zeros((B, S, Hq * D))
    for b in range(B):
        if not active[b].any():
            continue
        length = int(pos[b][active[b]].max()) + 1
        t = np.arange(length)
        pages = page_table[b, t // P]
        K = k_pool[pages, t % P]
        V = v_pool[pages, t % P]
        for s in range(S):
            if not active[b, s]:
                continue
            vis = int(pos[b, s]) + 1
            for h in range(Hq):
                g = h // grp
                sc = (K[:vis, g] @ q[b, s, h]) * sm_scale
                w = np.exp(sc - sc.max())
                out[b, s, h * D:(h + 1) * D] = (w @ V[:vis, g]) / w.sum()
    return out


def layer(x, L: Dict[str, np.ndarray], active, pos, page_table, P, Hq, Hkv, D, eps, rope_tab,
          exact=False):
    """One decoder layer (F1-F4) on rows x [B, S, H] (float64 values).

    L: weights (bf16 bits or float64) in_norm [H], w_qkv [(Hq+2Hkv)D, H],
    q_norm [D], k_norm [D], w_o [H, Hq D], post_norm [H], w_gate_up [2I, H]
    (gate rows first), w_down [H, I]; k_pool / v_pool float64 [pages, P,
    Hkv, D], updated in place.  Returns the new x and the intermediates."""
    r = _rounder(exact)
    B, S, H = x.shape
    w = {k: f64(v, exact) for k, v in L.items() if k not in ("k_pool", "v_pool")}
    h = r(rmsnorm(x, w["in_norm"], eps))
    qkv = r(h @ w["w_qkv"].T)
    q = qkv[..., : Hq * D].reshape(B, S, Hq, D)
    k = qkv[..., Hq * D:(Hq + Hkv) * D].reshape(B, S, Hkv, D)
    v = qkv[..., (Hq + Hkv) * D:].reshape(B, S, Hkv, D)
    cs = rope_tab[pos][:, :, None]  # [B, S, 1, D/2, 2]
    q = r(rope(rmsnorm(q, w["q_norm"], eps), cs))
    k = r(rope(rmsnorm(k, w["k_norm"], eps), cs))
    a = r(attention_rows(q, k, v, active, pos, L["k_pool"], L["v_pool"], page_table, P,
                         D ** -0.5))
    x1 = r(x + a @ w["w_o"].T)
    h2 = r(rmsnorm(x1, w["post_norm"], eps))
    gu = r(h2 @ w["w_gate_up"].T)
    I = gu.shape[-1] // 2
    act = r(silu(gu[..., :I]) * gu[..., I:])
    x2 = r(x1 + act @ w["w_down"].T)
    return x2, dict(h=h, q=q, k=k, v=v, attn=a, x_mid=x1, h2=h2, gate_up=gu, act=act)


def forward(x_bits, layers: List[Dict[str, np.ndarray]], final_norm, kv_len, n_clean, N,
            page_table, P, Hq, Hkv, D, eps, rope_tab, exact=False):
    """The whole stack over an ISD block (F1-F4): x_bits [B*Q, H] bf16 block
    embeddings; returns (final-normed hidden [B*Q, H] float64, the residual
    stream after the last layer, per-layer intermediates)."""
    r = _rounder(exact)
    Q = 2 * N - 1
    B = len(kv_len)
    pos = block_positions(kv_len, n_clean, N)
    active = np.zeros((B, Q), bool)
    for b in range(B):
        active[b, : int(n_clean[b])] = True
        active[b, N:] = True
    x = f64(x_bits, exact).reshape(B, Q, -1)
    inter = []
    for L in layers:
        x, st = layer(x, L, active, pos, page_table, P, Hq, Hkv, D, eps, rope_tab, exact)
        inter.append(st)
    out = r(rmsnorm(x, f64(final_norm, exact), eps))
    return out.reshape(B * Q, -1), x.reshape(B * Q, -1), inter


__all__ = ["rmsnorm", "rope", "silu", "block_positions", "attention_rows", "layer", "forward"]
