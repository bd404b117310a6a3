"""Comparison of an accept result from the CUDA path with the oracle's.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: used by ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``.

The rule is the acceptance specification of the ISD step (p/q criterion of
"I-DLM：扩散模型如何用“自省一致性”追上自回归模型质量", section "Introspective
Strided Decoding（ISD）", and "自省扩散语言模型的 token 生成机制与工程实践", section
"从质量差距到自省机制"), applied to the two sides fed the SAME fp32 logits:

* accept lengths, next states and next kv lengths identical for every request,
  except a request one of whose tested decisions has |u - p(x)/q(x)| < NEAR
  (a near-threshold decision: fp32 on the GPU and fp64 here may fall on
  different sides of u).  Such requests are counted, not compared;
* every token id identical, except an inverse-CDF draw (residual or sampled
  proposal) whose GPU pick lies within NEAR * sum(w) of the oracle's target
  (the GPU accumulates the weights in fp32).  Such draws are counted;
* the p/q ratios of the tested proposals within NEAR relative.

Everything else is a mismatch.  ``compare_accept`` returns the counts; it
never raises, so callers decide what to assert or report.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from . import isd_oracle as O

NEAR = 1e-5


def ratio_near(b: int, c: int, u: np.ndarray, ores: Dict[str, np.ndarray]) -> bool:
    """Is one of request b's tested accept decisions within NEAR of its uniform?"""
    for j in range(2, c + 1):
        r = ores["ratio"][b, j - 2]
        if abs(float(u[b, j - 2]) - r) < NEAR:
            return True
        if not (float(u[b, j - 2]) < r):
            break
    return False


def draw_explained(w, u: float, y: int) -> bool:
    """Is bucket y within NEAR * sum(w) of the oracle's inverse-CDF target?"""
    cum = np.cumsum(np.asarray(w, dtype=np.float64))
    tot = cum[-1]
    if not (0 <= y < len(w)) or w[y] <= 0 or tot <= 0:
        return False
    t = float(u) * tot
    lo = cum[y - 1] if y > 0 else 0.0
    dist = max(0.0, lo - t, t - cum[y])
    return dist <= NEAR * tot


def compare_accept(gpu: Dict[str, np.ndarray], ores: Dict[str, np.ndarray], logits: np.ndarray,
                   prev: np.ndarray, inp: Dict[str, np.ndarray], N: int, mode: int) -> Dict:
    """Counts of the comparison of the GPU's accept outputs with the oracle's.

    gpu: accept_len, out_tok, next_n_clean, next_clean_tok, next_kv_len, ratio
    (host arrays); ores: ``isd_oracle.accept`` on the same logits; logits,
    prev: [B, Q, V] fp32 (this and the previous step's); inp: n_clean,
    uniforms.  Returns a dict with
      requests        -- B
      near_threshold  -- requests skipped for a decision within NEAR of u
      draws           -- inverse-CDF draws compared (requests not skipped)
      excused_draws   -- draws whose token differs but is rounding-explained
      mismatches      -- everything else that differs (0 for parity)
      first_mismatch  -- description of the first mismatch, or None
    """
    B = logits.shape[0]
    u = inp["uniforms"]
    rep = dict(requests=int(B), near_threshold=0, draws=0, excused_draws=0, mismatches=0,
               first_mismatch=None)

    def bad(what):
        rep["mismatches"] += 1
        if rep["first_mismatch"] is None:
            rep["first_mismatch"] = what

    for b in range(B):
        c = int(inp["n_clean"][b])
        if ratio_near(b, c, u, ores):
            rep["near_threshold"] += 1
            continue
        same_state = True
        for key in ("accept_len", "next_n_clean", "next_kv_len"):
            if int(gpu[key][b]) != int(ores[key][b]):
                bad(f"{key}[{b}]: gpu {int(gpu[key][b])} oracle {int(ores[key][b])}")
                same_state = False
        if not same_state:
            continue
        A = int(ores["accept_len"][b])
        # draws of this request: (out / next, position) -> (weights, uniform)
        draws = {}
        rej = int(ores["rejected_at"][b])
        if rej > 0:
            w = O.residual_distribution(logits[b, rej - 2], prev[b, N + rej - 2])
            if w.sum() > 0.0:
                draws[("out", A - 1)] = (w, u[b, N - 1])
                draws[("next", 0)] = draws[("out", A - 1)]
        elif mode == O.PROPOSE_SAMPLE:
            rows = [c - 1] + [N + m for m in range(N - 1)]
            for k, r in enumerate(rows):
                draws[("next", k)] = (O.softmax(logits[b, r]), u[b, N + k])
            draws[("out", A - 1)] = draws[("next", 0)]
        # a draw shared by out_tok and next_clean_tok counts once
        rep["draws"] += len({id(v) for v in draws.values()})
        excused = set()
        for kind, key in (("out", "out_tok"), ("next", "next_clean_tok")):
            g, o = np.asarray(gpu[key][b]), np.asarray(ores[key][b])
            for i in np.nonzero(g != o)[0]:
                d = draws.get((kind, int(i)))
                if d is not None and draw_explained(d[0], d[1], int(g[i])):
                    excused.add(id(d))
                else:
                    bad(f"{key}[{b}][{int(i)}]: gpu {int(g[i])} oracle {int(o[i])}")
        rep["excused_draws"] += len(excused)
        # ratios of the tested proposals
        for j in range(2, A + 2):
            if j - 2 >= ores["ratio"].shape[1] or not (ores["ratio"][b, j - 2] >= 0):
                break
            rg, ro = float(gpu["ratio"][b, j - 2]), float(ores["ratio"][b, j - 2])
            if not abs(rg - ro) <= NEAR * abs(ro):
                bad(f"ratio[{b}][{j - 2}]: gpu {rg} oracle {ro}")
    return rep


__all__ = ["NEAR", "ratio_near", "draw_explained", "compare_accept"]
