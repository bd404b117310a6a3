"""CPU oracle of the batched ISD verify-and-propose step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run this module.  The product
path (the CUDA library and its binding) never calls it, and this module
imports nothing from the product package.

Plain, slow, obviously correct numpy in float64, written from the I-DLM pages:

  [PRJ] I-DLM project page, Traditional-Chinese text (news.myit.tw/news/ml1xco)
  [EXP] "I-DLM：扩散模型如何用“自省一致性”追上自回归模型质量" (blog.hypho.cn)
  [ENG] "自省扩散语言模型的 token 生成机制与工程实践" (blog.hotdry.top)

Where the pages leave a step open, the reading taken here is stated at the
function that takes it.  Every function is pinned by a ``-m "not gpu"`` test
against something other than itself (the pages' E[acc]/TPF table, closed
forms, brute force, textbook special cases); none is "parity unpinned".

Data conventions (identical meaning to the C-ABI in include/isd.h):
  bf16 tensors are uint16 bit patterns; logits are float32.
  q [B,Q,Hq,D]; k_new, v_new [B,Q,Hkv,D]; k_pool, v_pool [pages,P,Hkv,D];
  page_table [B,max_pages]; kv_len, n_clean [B]; clean_tok [B,N];
  hidden [B*Q, Hq*D]; W [V,H]; lora_A [H,r]; lora_B [r,H];
  uniforms [B,2N]: u_acc[0..N-2], u_res[N-1], u_prop[N..2N-1].
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

PROPOSE_ARGMAX = 0
PROPOSE_SAMPLE = 1


# ---------------------------------------------------------------------------
# bf16 <-> float64
# ---------------------------------------------------------------------------
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 to bf16 (nearest, ties to even) in one step.

    bf16 keeps 7 of float64's 52 stored mantissa bits; the 45 dropped bits are
    rounded half-to-even.  The result is then exact in float32, whose top 16
    bits are the bf16 pattern.  (Values in float32's subnormal range are not
    produced by this step and are not handled specially.)
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    u = x.view(np.uint64)
    low = np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    keep_lsb = (u >> np.uint64(45)) & np.uint64(1)
    r = (u + (half - np.uint64(1)) + keep_lsb) & ~low
    f32 = r.view(np.float64).astype(np.float32)
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# a0: slot layout of the 2N-1 query block
# ---------------------------------------------------------------------------
def slot_positions(kv_len: int, c: int, N: int) -> np.ndarray:
    """Absolute position of each of the Q = 2N-1 slots, -1 if inactive.

    [ENG §Token 生成的核心参数与验收机制] gives the block size 2N-1 for stride N;
    [PRJ, TPF / acceptance paragraph] states that position 1 is always accepted
    because of the logit shift; [EXP §三项关键训练创新, "Logit 偏移"] says the
    hidden state at position i predicts token i+1.  Reading taken: slots
    0..N-1 are CLEAN, of which the first c hold the clean tokens t_1..t_c at
    positions kv_len..kv_len+c-1 and the rest are inactive; slots N..2N-2 are
    MASK slots at positions kv_len+c .. kv_len+c+N-2.
    """
    pos = np.full(2 * N - 1, -1, dtype=np.int64)
    for s in range(c):
        pos[s] = kv_len + s
    for m in range(N - 1):
        pos[N + m] = kv_len + c + m
    return pos


# ---------------------------------------------------------------------------
# a1: KV append into the paged cache
# ---------------------------------------------------------------------------
def kv_append(k_pool, v_pool, k_new, v_new, page_table, kv_len, n_clean, N, P):
    """Write every active slot's K/V row at its position into the paged pool.

    Position t of request b lives in page page_table[b, t // P], row t % P
    ([EXP §推理：复用 AR 推理栈] and [ENG §服务部署与 SGLang 集成]: paged KV cache).
    Returns new pools (inputs are not modified).
    """
    k_out = np.array(k_pool, copy=True)
    v_out = np.array(v_pool, copy=True)
    B = k_new.shape[0]
    for b in range(B):
        pos = slot_positions(int(kv_len[b]), int(n_clean[b]), N)
        for s, t in enumerate(pos):
            if t < 0:
                continue
            page = int(page_table[b, t // P])
            k_out[page, t % P] = k_new[b, s]
            v_out[page, t % P] = v_new[b, s]
    return k_out, v_out


def gather_sequence(pool, page_table_row, length: int, P: int) -> np.ndarray:
    """Rows 0..length-1 of one request's paged sequence, [length, Hkv, D] bf16."""
    t = np.arange(length)
    pages = page_table_row[t // P]
    return pool[pages, t % P]


# ---------------------------------------------------------------------------
# a2: strict-causal GQA attention over the paged cache plus the block
# ---------------------------------------------------------------------------
def attention(q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean, N, P, sm_scale):
    """Strict-causal grouped-query attention for every active slot.

    [PRJ] and [EXP §三项关键训练创新, "严格因果掩码"]: causal attention is applied
    to clean and MASK slots alike, so slot s at position pos_s attends to all
    keys at positions 0..pos_s (the cached prefix plus the block slots at or
    before it).  Query head h uses KV head h // (Hq/Hkv).  Softmax of
    sm_scale * q.k, weights applied to v; computed in float64 from the bf16
    inputs and rounded once to bf16.  Inactive slots produce zero rows.

    Returns (out [B*Q, Hq*D] bf16, k_pool', v_pool').
    """
    B, Q, Hq, D = q.shape
    Hkv = k_new.shape[2]
    grp = Hq // Hkv
    k_pool2, v_pool2 = kv_append(k_pool, v_pool, k_new, v_new, page_table, kv_len, n_clean, N, P)
    out = np.zeros((B, Q, Hq * D), dtype=np.float64)
    for b in range(B):
        c = int(n_clean[b])
        pos = slot_positions(int(kv_len[b]), c, N)
        length = int(pos.max()) + 1
        K = bf16_to_f64(gather_sequence(k_pool2, page_table[b], length, P))   # [L,Hkv,D]
        Vv = bf16_to_f64(gather_sequence(v_pool2, page_table[b], length, P))
        for s in range(Q):
            if pos[s] < 0:
                continue
            visible = int(pos[s]) + 1
            for h in range(Hq):
                g = h // grp
                qv = bf16_to_f64(q[b, s, h])
                scores = (K[:visible, g, :] @ qv) * sm_scale
                w = np.exp(scores - scores.max())
                o = (w @ Vv[:visible, g, :]) / w.sum()
                out[b, s, h * D:(h + 1) * D] = o
    return f64_to_bf16(out.reshape(B * Q, Hq * D)), k_pool2, v_pool2


# ---------------------------------------------------------------------------
# a3: R-ISD gated LoRA on the MASK rows
# ---------------------------------------------------------------------------
def gated_lora(hidden, lora_A, lora_B, B: int, N: int):
    """h' = bf16(h + bf16(h A) B) on MASK rows, h' = h on clean rows.

    [ENG §Token 生成的核心参数与验收机制] and [PRJ, R-ISD paragraph]: the gated
    LoRA adapter (rank 128) is active at MASK positions only; verify (clean)
    positions use the base weights.  Readings taken (the pages give no
    formula): scale 1; the intermediate h A is rounded to bf16; one final
    rounding of h + delta to bf16.
    """
    Q = 2 * N - 1
    h = bf16_to_f64(hidden).reshape(B, Q, -1)
    A = bf16_to_f64(lora_A)
    Bm = bf16_to_f64(lora_B)
    out = np.array(hidden, copy=True).reshape(B, Q, -1)
    for b in range(B):
        for s in range(N, Q):
            t = bf16_to_f64(f64_to_bf16(h[b, s] @ A))
            out[b, s] = f64_to_bf16(h[b, s] + t @ Bm)
    return out.reshape(B * Q, -1)


# ---------------------------------------------------------------------------
# a4: LM head
# ---------------------------------------------------------------------------
def lm_head(hidden, W, v_chunk: int = 8192) -> np.ndarray:
    """logits = hidden . W^T in float64, stored as float32.  [M,V]

    [EXP §ISD 核心逻辑伪代码]: every slot's final hidden state is mapped to a
    distribution over the vocabulary.  The product is taken in vocabulary
    chunks only to bound host memory; each entry is one float64 dot product.
    """
    h = bf16_to_f64(hidden)
    M = h.shape[0]
    V = W.shape[0]
    out = np.empty((M, V), dtype=np.float32)
    for v0 in range(0, V, v_chunk):
        Wc = bf16_to_f64(W[v0:v0 + v_chunk])
        out[:, v0:v0 + v_chunk] = (h @ Wc.T).astype(np.float32)
    return out


def lm_head_entry(hidden_row, W_row) -> float:
    """One logit, as a float64 dot product (for sampled full-size checks)."""
    return float(np.dot(bf16_to_f64(hidden_row), bf16_to_f64(W_row)))


# ---------------------------------------------------------------------------
# a5: row statistics and argmax
# ---------------------------------------------------------------------------
def row_stats(z: np.ndarray):
    """(max, sum_i exp(z_i - max), argmax) of one logits row, in float64.

    Argmax proposals follow [ENG §服务部署与 SGLang 集成] ("Argmax 提议策略").
    Ties go to the lowest index (reading taken; the pages are silent).
    """
    z = np.asarray(z, dtype=np.float64)
    m = float(z.max())
    return m, float(np.exp(z - m).sum()), int(np.argmax(z))


def softmax(z: np.ndarray) -> np.ndarray:
    """Temperature-1 softmax in float64 (the pages state no temperature)."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - z.max())
    return e / e.sum()


def inverse_cdf(weights: np.ndarray, u: float) -> int:
    """Smallest i with sum_{k<=i} w_k > u * sum_k w_k (weights need not be
    normalised).  If rounding leaves no such i, the last index with positive
    weight is returned."""
    w = np.asarray(weights, dtype=np.float64)
    cum = np.cumsum(w)
    target = float(u) * cum[-1]
    hit = np.nonzero(cum > target)[0]
    if hit.size:
        return int(hit[0])
    return int(np.nonzero(w > 0)[0][-1])


# ---------------------------------------------------------------------------
# a6-a9: p/q acceptance, residual draw, next-stride proposals, state update
# ---------------------------------------------------------------------------
def accept_ratio(p_row, q_row, x: int) -> float:
    """p(x)/q(x), p and q the softmaxes of the anchor and proposal rows."""
    return float(softmax(p_row)[x] / softmax(q_row)[x])


def residual_distribution(p_row, q_row) -> np.ndarray:
    """max(0, p - q) (unnormalised).  The pages call the output lossless
    ([EXP §Introspective Strided Decoding（ISD）], [ENG §从质量差距到自省机制])
    but do not print the replacement rule; this is the rule under which
    min(1, p/q) acceptance reproduces p exactly."""
    return np.maximum(0.0, softmax(p_row) - softmax(q_row))


def propose(row, u: float, mode: int) -> int:
    if mode == PROPOSE_ARGMAX:
        return row_stats(row)[2]
    return inverse_cdf(softmax(row), u)


def accept(logits, prev_logits, n_clean, clean_tok, kv_len, uniforms, N: int,
           mode: int = PROPOSE_ARGMAX) -> Dict[str, np.ndarray]:
    """Verify the previous stride's proposals and propose the next stride.

    logits, prev_logits: [B, Q, V] float32 (this step's and the previous
    step's).  For request b with c = n_clean[b] clean tokens t_1..t_c:

    * Verification ([EXP §ISD 核心逻辑伪代码]; [ENG §从质量差距到自省机制]):
      for j = 2..c in order, x = t_j, p = softmax(this step's row j-2) (the
      clean slot holding t_{j-1}, which predicts position j by the logit
      shift), q = softmax(previous step's MASK row N+j-2, which proposed
      t_j).  Accept iff u_acc[j-2] < p(x)/q(x), i.e. with probability
      min(1, p(x)/q(x)).  Reading taken: the first rejection stops the pass.
    * Geometric acceptance ([PRJ]): t_1 is always accepted, so
      A = 1 + (number of accepted t_j).
    * On a rejection at j: the replacement y is drawn by inverse CDF from
      max(0, p - q) with u_res; if that mass is zero, y = argmax p.  Emitted
      tokens: t_2..t_A, y.  Next stride restarts with c = 1, tokens [y].
    * Without a rejection: proposals x'_1 from this step's row c-1 (the
      anchor slot) and x'_{m+2} from MASK row N+m, m = 0..N-2, by argmax (or
      inverse CDF with u_prop in sample mode).  Emitted: t_2..t_c, x'_1.  Next
      stride has c = N, tokens x'_1..x'_N.
    * kv_len grows by A: the clean slots t_1..t_A were computed on a fully
      accepted context, so their cache rows stay.

    This restart state machine reproduces the E[acc] and TPF columns of
    [ENG §Token 生成的核心参数与验收机制, table] (pinned in the tests).
    """
    B = logits.shape[0]
    V = logits.shape[2]
    accept_len = np.zeros(B, dtype=np.int32)
    out_tok = np.full((B, N), -1, dtype=np.int32)
    next_n_clean = np.zeros(B, dtype=np.int32)
    next_tok = np.full((B, N), -1, dtype=np.int32)
    next_kv_len = np.zeros(B, dtype=np.int32)
    ratio = np.full((B, max(N - 1, 1)), -1.0, dtype=np.float64)
    rejected_at = np.full(B, -1, dtype=np.int32)
    for b in range(B):
        c = int(n_clean[b])
        t = [int(x) for x in clean_tok[b, :c]]
        u = uniforms[b]
        emitted = []
        rej_j = -1
        for j in range(2, c + 1):
            x = t[j - 1]
            r = accept_ratio(logits[b, j - 2], prev_logits[b, N + j - 2], x)
            ratio[b, j - 2] = r
            if float(u[j - 2]) < r:
                emitted.append(x)
            else:
                rej_j = j
                break
        if rej_j > 0:
            p_row = logits[b, rej_j - 2]
            w = residual_distribution(p_row, prev_logits[b, N + rej_j - 2])
            if w.sum() > 0.0:
                y = inverse_cdf(w, float(u[N - 1]))
            else:
                y = row_stats(p_row)[2]
            emitted.append(y)
            next_n_clean[b] = 1
            next_tok[b, 0] = y
            rejected_at[b] = rej_j
        else:
            props = [propose(logits[b, c - 1], float(u[N]), mode)]
            for m in range(N - 1):
                props.append(propose(logits[b, N + m], float(u[N + 1 + m]), mode))
            emitted.append(props[0])
            next_n_clean[b] = N
            next_tok[b, :N] = props
        A = len(emitted)
        accept_len[b] = A
        out_tok[b, :A] = emitted
        next_kv_len[b] = int(kv_len[b]) + A
        assert all(0 <= x < V for x in emitted)
    return dict(accept_len=accept_len, out_tok=out_tok, next_n_clean=next_n_clean,
                next_clean_tok=next_tok, next_kv_len=next_kv_len, ratio=ratio,
                rejected_at=rejected_at)


# ---------------------------------------------------------------------------
# Whole step
# ---------------------------------------------------------------------------
def isd_step(inp: Dict[str, np.ndarray], prev_logits: np.ndarray, N: int, P: int,
             sm_scale: float, mode: int = PROPOSE_ARGMAX,
             lora: bool = False) -> Dict[str, np.ndarray]:
    """a1..a9 in order: append + attention, (LoRA on MASK rows), LM head,
    acceptance.  Returns every intermediate so each stage can be compared."""
    B = inp["q"].shape[0]
    Q = 2 * N - 1
    hidden, k_pool2, v_pool2 = attention(
        inp["q"], inp["k_new"], inp["v_new"], inp["k_pool"], inp["v_pool"],
        inp["page_table"], inp["kv_len"], inp["n_clean"], N, P, sm_scale)
    hidden2 = gated_lora(hidden, inp["lora_A"], inp["lora_B"], B, N) if lora else hidden
    logits = lm_head(hidden2, inp["W"]).reshape(B, Q, -1)
    res = accept(logits, prev_logits, inp["n_clean"], inp["clean_tok"], inp["kv_len"],
                 inp["uniforms"], N, mode)
    res.update(hidden=hidden, hidden_lm=hidden2, logits=logits, k_pool=k_pool2, v_pool=v_pool2)
    return res


def row_stats_all(logits: np.ndarray):
    """row_stats of every row of a [..., V] array: (max, sumexp, argmax)."""
    flat = logits.reshape(-1, logits.shape[-1])
    m = np.empty(flat.shape[0])
    s = np.empty(flat.shape[0])
    a = np.empty(flat.shape[0], dtype=np.int64)
    for i in range(flat.shape[0]):
        m[i], s[i], a[i] = row_stats(flat[i])
    return m, s, a


__all__ = [
    "PROPOSE_ARGMAX", "PROPOSE_SAMPLE", "bf16_to_f64", "f64_to_bf16", "slot_positions",
    "kv_append", "gather_sequence", "attention", "gated_lora", "lm_head", "lm_head_entry",
    "row_stats", "row_stats_all", "softmax", "inverse_cdf", "accept_ratio",
    "residual_distribution", "propose", "accept", "isd_step",
]
