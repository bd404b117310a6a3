"""CPU oracle of SDAR-style confidence-threshold block decoding, the
batch-synchronous comparison workload of the I-DLM pages.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import or run this module.  The product path
never calls it, and this module imports nothing from the product package.

Source: [PRJ] I-DLM project page (Traditional-Chinese text,
news.myit.tw/news/ml1xco), the paragraphs on SDAR: SDAR denoises by
confidence; each forward pass of SDAR carries N queries (against 2N-1 for
ISD); a batch must wait for the slowest block, so the forwards spent per block
are E[max(S_1..S_B)], which grows with B and lowers the effective TPF, while
ISD requests advance on their own.  The pages name the rule without spelling
it out.  The readings taken here (plainest ones the text supports):

  R1  Block layout.  A block is N positions kv_len .. kv_len+N-1, and every
      forward computes all N of them (query size N).  A committed position
      carries its token, an uncommitted one the MASK token.
  R2  Attention is block-causal: each row sees the whole cached prefix and
      all N rows of its own block (bidirectional inside the block, causal
      across blocks), the usual mask of block-diffusion models.
  R3  Each forward writes the block's K/V rows (from that forward's inputs)
      at their positions.  A block leaves (kv_len += N, a fresh block of
      MASK) only after a forward whose inputs were its final tokens, so the
      cache keeps K/V computed from them: once its last position is committed,
      the request's next forward is the block's store pass, as block-diffusion
      decoders run one forward over a finished block to extend the cache.
  R4  Row s predicts block position s (no logit shift).
  R5  Confidence of position s = its largest softmax probability,
      1 / sum_i exp(z_i - max z); its candidate token is the argmax (ties to
      the lowest index).
  R6  Unmask rule: every uncommitted position whose confidence is >= tau is
      committed with its candidate; if none is, the one uncommitted position
      of highest confidence is (ties to the lowest position).  A block
      therefore takes S_b in [1, N] denoising forwards, then its store pass.
      Committed tokens never change.
  R7  Batch sync: the batch moves to the next block only once every
      request's block is complete and stored.  A request that finished early
      idles (its rows, final tokens, are still computed) until then.  A round
      of the batch costs max_b S_b + 1 forwards.  Without sync (the ISD way)
      a request moves on after its own block's store pass: S_b + 1 forwards.
  R8  Decisions (>= tau, the highest confidence) are taken on float32
      confidences conf = fl32(1) / fl32(S), the precision the kernel decides
      in; the oracle rounds its float64 sum to float32 first.

Data conventions follow oracle.isd_oracle (bf16 as uint16 bit patterns).
Block tokens are int32 [B, N] with -1 for an uncommitted (MASK) position.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from oracle import isd_oracle as O

MASK = -1


# ---------------------------------------------------------------------------
# R1-R3: KV append and block-causal attention
# ---------------------------------------------------------------------------
def kv_append(k_pool, v_pool, k_new, v_new, page_table, kv_len, P):
    """Write all N block rows of each request at kv_len .. kv_len+N-1 (R1, R3).
    Returns new pools."""
    k_out = np.array(k_pool, copy=True)
    v_out = np.array(v_pool, copy=True)
    B, N = k_new.shape[:2]
    for b in range(B):
        for s in range(N):
            t = int(kv_len[b]) + s
            page = int(page_table[b, t // P])
            k_out[page, t % P] = k_new[b, s]
            v_out[page, t % P] = v_new[b, s]
    return k_out, v_out


def block_attention(q, k_new, v_new, k_pool, v_pool, page_table, kv_len, P, sm_scale):
    """GQA attention of every block row over the prefix plus the whole block.

    R2: row s of request b attends to keys 0 .. kv_len+N-1, whatever s is.
    Query head h reads KV head h // (Hq/Hkv).  Softmax of sm_scale * q.k in
    float64 from the bf16 inputs, one rounding to bf16.

    Returns (out [B*N, Hq*D] bf16, k_pool', v_pool').
    """
    B, N, Hq, D = q.shape
    Hkv = k_new.shape[2]
    grp = Hq // Hkv
    k2, v2 = kv_append(k_pool, v_pool, k_new, v_new, page_table, kv_len, P)
    out = np.zeros((B, N, Hq * D), dtype=np.float64)
    for b in range(B):
        length = int(kv_len[b]) + N
        K = O.bf16_to_f64(O.gather_sequence(k2, page_table[b], length, P))
        Vv = O.bf16_to_f64(O.gather_sequence(v2, page_table[b], length, P))
        for s in range(N):
            for h in range(Hq):
                g = h // grp
                scores = (K[:, g, :] @ O.bf16_to_f64(q[b, s, h])) * sm_scale
                w = np.exp(scores - scores.max())
                out[b, s, h * D:(h + 1) * D] = (w @ Vv[:, g, :]) / w.sum()
    return O.f64_to_bf16(out.reshape(B * N, Hq * D)), k2, v2


# ---------------------------------------------------------------------------
# R5, R6, R8: confidence and the unmask rule
# ---------------------------------------------------------------------------
def confidence(sumexp) -> np.ndarray:
    """R5 + R8: float32 confidence 1 / S from the row's sum exp(z - max)."""
    return np.float32(1.0) / np.asarray(sumexp, dtype=np.float32)


def unmask(block_tok: np.ndarray, conf: np.ndarray, cand: np.ndarray, tau: float):
    """One denoising step of one block (R6).

    block_tok [N] (-1 = uncommitted), conf [N] float32, cand [N] argmax tokens.
    Returns (new block_tok, positions committed in this step)."""
    tok = np.array(block_tok, dtype=np.int64, copy=True)
    open_pos = [s for s in range(len(tok)) if tok[s] == MASK]
    if not open_pos:
        return tok, []
    t32 = np.float32(tau)
    chosen = [s for s in open_pos if np.float32(conf[s]) >= t32]
    if not chosen:
        best = open_pos[0]
        for s in open_pos[1:]:
            if np.float32(conf[s]) > np.float32(conf[best]):
                best = s
        chosen = [best]
    for s in chosen:
        tok[s] = int(cand[s])
    return tok, chosen


def unmask_batch(block_tok, steps, kv_len, conf, cand, tau: float, sync: bool):
    """One decision step of the whole batch (R3, R6, R7).

    block_tok [B, N], steps [B] (denoising forwards spent on the current
    block before this one), kv_len [B]; conf, cand [B, N] of this forward.
    A block that was complete when this forward began had its store pass in
    this forward and may leave.  Returns a dict with the next block_tok /
    steps / kv_len and, per request, unmasked (positions committed now),
    out_tok [N] (the block's tokens when it leaves the batch in this step,
    else -1) and block_steps (its S_b then, else 0)."""
    B, N = block_tok.shape
    tok = np.array(block_tok, dtype=np.int64, copy=True)
    st = np.array(steps, dtype=np.int64, copy=True)
    kv = np.array(kv_len, dtype=np.int64, copy=True)
    unmasked = np.zeros(B, np.int64)
    out_tok = np.full((B, N), -1, np.int64)
    block_steps = np.zeros(B, np.int64)
    stored = ~(tok == MASK).any(axis=1)   # complete at entry: this forward stored it
    for b in range(B):
        if not stored[b]:
            tok[b], ch = unmask(tok[b], conf[b], cand[b], tau)
            unmasked[b] = len(ch)
            st[b] += 1
    leave = np.ones(B, bool) * bool(stored.all()) if sync else stored
    for b in range(B):
        if leave[b]:
            out_tok[b] = tok[b]
            block_steps[b] = st[b]
            kv[b] += N
            tok[b] = MASK
            st[b] = 0
    return dict(block_tok=tok, steps=st, kv_len=kv, unmasked=unmasked, out_tok=out_tok,
                block_steps=block_steps)


# ---------------------------------------------------------------------------
# Whole step and closed loop on the synthetic table model
# ---------------------------------------------------------------------------
def rope_rotate(x_bits: np.ndarray, cs: np.ndarray) -> np.ndarray:
    """Rotary embedding of bf16 head vectors x [..., D] with the (cos, sin)
    table row cs [D/2, 2] of their position: element i pairs with i + D/2
    (the rotate-half layout of Qwen3), x_i' = x_i cos - x_{i+D/2} sin and
    x_{i+D/2}' = x_{i+D/2} cos + x_i sin.  The stand-in model fixes the
    arithmetic: float32, each product and sum rounded, then one bf16 rounding."""
    x = O.bf16_to_f64(x_bits).astype(np.float32)
    h = x.shape[-1] // 2
    c = cs[:, 0].astype(np.float32)
    s = cs[:, 1].astype(np.float32)
    lo, hi = x[..., :h], x[..., h:]
    out = np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1).astype(np.float32)
    return O.f64_to_bf16(out.astype(np.float64))


def embed_block(tables: Dict[str, np.ndarray], block_tok: np.ndarray, V: int,
                kv_len: np.ndarray = None, rope: np.ndarray = None):
    """q, k_new, v_new of the N block rows: a committed position looks up its
    token's row, an uncommitted one the MASK row V (R1).  With a rotary table
    rope [positions, D/2, 2], the q and k rows of block position s are rotated
    by position kv_len + s (v is not)."""
    ids = np.where(block_tok >= 0, block_tok, V).astype(np.int64)
    q, k, v = tables["Eq"][ids], tables["Ek"][ids], tables["Ev"][ids]
    if rope is not None:
        q, k = q.copy(), k.copy()
        B, N = block_tok.shape
        for b in range(B):
            for s in range(N):
                cs = rope[int(kv_len[b]) + s]
                q[b, s] = rope_rotate(q[b, s], cs)
                k[b, s] = rope_rotate(k[b, s], cs)
    return q, k, v


def sdar_step(q, k_new, v_new, k_pool, v_pool, page_table, kv_len, W, block_tok, steps,
              P, sm_scale, tau, sync):
    """R1-R8 in order: append + block attention, LM head, confidences, unmask."""
    B, N = block_tok.shape
    hidden, k2, v2 = block_attention(q, k_new, v_new, k_pool, v_pool, page_table, kv_len, P,
                                     sm_scale)
    logits = O.lm_head(hidden, W)
    m, s, a = O.row_stats_all(logits)
    conf = confidence(s).reshape(B, N)
    res = unmask_batch(block_tok, steps, kv_len, conf, a.reshape(B, N), tau, sync)
    res.update(hidden=hidden, logits=logits, k_pool=k2, v_pool=v2, row_max=m, row_sumexp=s,
               row_argmax=a, conf=conf)
    return res


def round_stats(block_steps_hist: np.ndarray, N: int) -> Dict[str, float]:
    """Forwards per block of a decision history (R3, R7).

    block_steps_hist [steps, B]: S_b of a block that left the batch at that
    step, else 0.  A block costs S_b denoising forwards plus its store pass.
    Under sync every request's block leaves at the same step, so each step
    with leavers closes one round, which cost max_b S_b + 1 forwards.
    Returns the number of blocks and rounds, the mean S_b, the mean of
    max_b S_b over rounds, and the tokens per forward of a request without
    the sync, N / (E[S_b] + 1), and with it, N / (E[max_b S_b] + 1)."""
    h = np.asarray(block_steps_hist)
    rounds = [r[r > 0] for r in h if (r > 0).any()]
    if not rounds:
        return dict(blocks=0, rounds=0, mean_S=float("nan"), mean_max_S=float("nan"),
                    tpf_free=float("nan"), tpf_sync=float("nan"))
    s_all = np.concatenate(rounds).astype(np.float64)
    maxes = np.array([r.max() for r in rounds], dtype=np.float64)
    return dict(blocks=int(s_all.size), rounds=len(rounds), mean_S=float(s_all.mean()),
                mean_max_S=float(maxes.mean()), tpf_free=N / (float(s_all.mean()) + 1.0),
                tpf_sync=N / (float(maxes.mean()) + 1.0))


def expected_max(pmf: np.ndarray, B: int) -> float:
    """E[max(S_1..S_B)] for iid S_b with P(S = s) = pmf[s - 1], s = 1..len(pmf):
    P(max <= s) = F(s)^B (the batch-sync penalty of R7 in closed form)."""
    F = np.cumsum(np.asarray(pmf, dtype=np.float64))
    F = np.minimum(F / F[-1], 1.0)
    prev = np.concatenate([[0.0], F[:-1]])
    s = np.arange(1, len(F) + 1)
    return float(np.sum(s * (F ** B - prev ** B)))


__all__ = ["MASK", "kv_append", "block_attention", "confidence", "unmask", "unmask_batch",
           "rope_rotate", "embed_block", "sdar_step", "round_stats", "expected_max"]
