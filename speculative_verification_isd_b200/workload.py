"""Full-size synthetic ISD workloads resident on the GPU.

Used by the benchmark, the smoke run and the full-size parity test.  It only
prepares inputs: the structural ones (prefix lengths, page tables, tokens,
uniforms) come from ``inputs``; the large tensors (KV pool, LM head, block
activations, LoRA) are drawn N(0, std) with a seeded CUDA generator and stored
as bf16.  All step arithmetic runs in libisd.so.

Constructed acceptance: for a target rate a, the previous step's MASK rows
are set so that p(x)/q(x) = a exactly for every proposal x.  This needs this
step's anchor rows p, so one untimed step is run first; then q = p except
at x, whose logit is raised by log((1 - P) / (a - P)), P = p(x).
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np
import torch

from . import inputs as I


def _randn_bf16(shape, std: float, gen: torch.Generator) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    flat = out.view(-1)
    chunk = 1 << 26
    tmp = torch.empty(min(chunk, flat.numel()), dtype=torch.float32, device="cuda")
    for s in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - s)
        t = tmp[:n]
        t.normal_(0.0, std, generator=gen)
        flat[s:s + n].copy_(t)
    return out


class DeviceWorkload:
    """Device buffers of one ISD step at a given config, ready to run."""

    def __init__(self, isd, cfg: I.IsdConfig, seed: int = 0, n_uniform_steps: int = 64,
                 accept_rate: Optional[float] = "cfg", n_clean: str = "full"):
        self.isd = isd
        self.cfg = cfg
        self.seed = seed
        a = cfg.accept_rate if accept_rate == "cfg" else accept_rate
        self.accept_rate = a
        B, N, Q = cfg.B, cfg.N, cfg.Q
        kv_len = I.prefix_lengths(cfg, seed)
        table, num_pages = I.page_layout(cfg, kv_len, seed)
        rng = np.random.default_rng([seed, 31])
        if n_clean == "full":
            nc = np.full(B, N, np.int32)
        else:
            nc = rng.integers(1, N + 1, B).astype(np.int32)
        tok = rng.integers(0, cfg.V, size=(B, N)).astype(np.int32)
        self.kv_len_h, self.page_table_h, self.n_clean_h, self.clean_tok_h = kv_len, table, nc, tok
        self.uniforms_h = np.stack([I.step_uniforms(seed, k, B, N) for k in range(n_uniform_steps)])
        gen = torch.Generator(device="cuda")
        gen.manual_seed(seed)
        self.dims = isd.make_dims(B, N, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, cfg.page_size, num_pages,
                                  table.shape[1], cfg.lora_rank, 0)
        d = self.dims
        self.q = _randn_bf16((B, Q, cfg.Hq, cfg.D), cfg.qkv_std, gen)
        self.k_new = _randn_bf16((B, Q, cfg.Hkv, cfg.D), cfg.qkv_std, gen)
        self.v_new = _randn_bf16((B, Q, cfg.Hkv, cfg.D), cfg.qkv_std, gen)
        self.k_pool = _randn_bf16((num_pages, cfg.page_size, cfg.Hkv, cfg.D), cfg.kv_std, gen)
        self.v_pool = _randn_bf16((num_pages, cfg.page_size, cfg.Hkv, cfg.D), cfg.kv_std, gen)
        self.W = _randn_bf16((cfg.V, cfg.H), cfg.w_std, gen)
        self.lora_A = _randn_bf16((cfg.H, cfg.lora_rank), cfg.lora_std, gen) if cfg.lora_rank else None
        self.lora_B = _randn_bf16((cfg.lora_rank, cfg.H), cfg.lora_std, gen) if cfg.lora_rank else None
        dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
        self.page_table = dev(table)
        self.kv_len = dev(kv_len)
        self.n_clean = dev(nc)
        self.clean_tok = dev(tok)
        self.uniforms_all = dev(self.uniforms_h)
        self.uniforms = self.uniforms_all[0]
        self.ws = isd.alloc_workspace(d)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        M, V = d.M, d.V
        self.hidden = torch.empty(M, d.H, dtype=torch.bfloat16, device="cuda")
        self.logits = torch.empty(M, V, dtype=torch.float32, device="cuda")
        self.row_stats = torch.empty(M, 4, dtype=torch.int32, device="cuda")
        self.prev_logits = torch.zeros(M, V, dtype=torch.float32, device="cuda")
        self.prev_row_stats = torch.empty(M, 4, dtype=torch.int32, device="cuda")
        self.accept_len = torch.empty(B, dtype=torch.int32, device="cuda")
        self.out_tok = torch.empty(B, N, dtype=torch.int32, device="cuda")
        self.next_n_clean = torch.empty(B, dtype=torch.int32, device="cuda")
        self.next_clean_tok = torch.empty(B, N, dtype=torch.int32, device="cuda")
        self.next_kv_len = torch.empty(B, dtype=torch.int32, device="cuda")
        self.ratio = torch.empty(B, max(N - 1, 1), dtype=torch.float32, device="cuda")
        isd.row_stats(d, self.prev_logits, M, self.prev_row_stats, self.ws)
        self._prepare_prev()

    # ------------------------------------------------------------------
    def _prepare_prev(self):
        """Previous step's logits: random rows, with constructed MASK rows."""
        cfg, d = self.cfg, self.dims
        B, N, Q, V = cfg.B, cfg.N, cfg.Q, cfg.V
        gen = torch.Generator(device="cuda")
        gen.manual_seed(self.seed + 1)
        prev = torch.empty(B, Q, V, dtype=torch.float32, device="cuda")
        prev.normal_(0.0, 1.0, generator=gen)
        if self.accept_rate is not None:
            self.step()  # untimed: this step's anchor rows p
            torch.cuda.synchronize()
            cur = self.logits.view(B, Q, V)
            a = float(self.accept_rate)
            for j in range(2, N + 1):
                x = self.clean_tok[:, j - 1].long()
                prow = cur[:, j - 2].double()
                lse = torch.logsumexp(prow, dim=-1)
                zx = prow.gather(1, x[:, None])[:, 0]
                P = torch.exp(zx - lse)
                if torch.any(P >= a):
                    raise ValueError("constructed acceptance needs p(x) < a")
                delta = torch.log((1.0 - P) / (a - P))
                qrow = cur[:, j - 2].clone()
                qrow.scatter_(1, x[:, None], (zx + delta).float()[:, None])
                prev[:, N + j - 2] = qrow
        self.prev_logits.copy_(prev.view(d.M, V))
        self.isd.row_stats(d, self.prev_logits, d.M, self.prev_row_stats, self.ws)
        torch.cuda.synchronize()

    def set_uniforms(self, k: int):
        self.uniforms = self.uniforms_all[k % self.uniforms_all.shape[0]]

    IN_NAMES = ("q", "k_new", "v_new", "kv_len", "n_clean", "clean_tok", "page_table", "uniforms")
    OUT_NAMES = ("accept_len", "out_tok", "next_n_clean", "next_clean_tok", "next_kv_len")

    def pack_io(self):
        """Rebind a step's inputs to views of one device byte buffer and its
        integer results to views of one int32 buffer, so that the host traffic
        of a step is one copy each way.  Returns (in_buf, out_buf, layout) with
        layout = [(name, byte offset, bytes)]."""
        layout, off = [], 0
        for n in self.IN_NAMES:
            t = getattr(self, n)
            nb = t.numel() * t.element_size()
            layout.append((n, off, nb))
            off = (off + nb + 255) // 256 * 256
        buf = torch.empty(off, dtype=torch.uint8, device="cuda")
        for n, o, nb in layout:
            t = getattr(self, n)
            v = buf[o:o + nb].view(t.dtype).view(t.shape)
            v.copy_(t)
            setattr(self, n, v)
        sizes = [getattr(self, n).numel() for n in self.OUT_NAMES]
        obuf = torch.zeros(sum(sizes), dtype=torch.int32, device="cuda")
        o = 0
        for n, sz in zip(self.OUT_NAMES, sizes):
            setattr(self, n, obuf[o:o + sz].view(getattr(self, n).shape))
            o += sz
        return buf, obuf, layout

    def step(self, stream=None, without_lora=False):
        """One isd_step; without_lora runs the same step with the adapter off
        (dims with lora_rank 0), for measuring the adapter's cost."""
        dims, la, lb = self.dims, self.lora_A, self.lora_B
        if without_lora:
            dims = type(self.dims).from_buffer_copy(self.dims)
            dims.lora_rank = 0
            la = lb = None
        self.isd.step(dims, self.q, self.k_new, self.v_new, self.k_pool, self.v_pool,
                      self.page_table, self.kv_len, self.n_clean, self.clean_tok, self.W,
                      self.prev_logits, self.prev_row_stats, self.uniforms, self.logits,
                      self.row_stats, self.accept_len, self.out_tok, self.next_n_clean,
                      self.next_clean_tok, self.next_kv_len, self.ws, hidden=self.hidden,
                      ratio=self.ratio, lora_A=la, lora_B=lb,
                      err_flag=self.err, stream=stream)

    def outputs(self) -> Dict[str, np.ndarray]:
        torch.cuda.synchronize()
        return dict(accept_len=self.accept_len.cpu().numpy(), out_tok=self.out_tok.cpu().numpy(),
                    next_n_clean=self.next_n_clean.cpu().numpy(),
                    next_clean_tok=self.next_clean_tok.cpu().numpy(),
                    next_kv_len=self.next_kv_len.cpu().numpy(), ratio=self.ratio.cpu().numpy())

    def host_view(self) -> Dict[str, np.ndarray]:
        """Small inputs of the current step on the host (for oracle checks)."""
        u = self.uniforms.cpu().numpy()
        return dict(kv_len=self.kv_len_h, n_clean=self.n_clean_h, clean_tok=self.clean_tok_h,
                    page_table=self.page_table_h, uniforms=u, _wl=self)


def _bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def request_slice(host: Dict, cfg: I.IsdConfig, b: int) -> Dict[str, np.ndarray]:
    """Single-request copy of the step's inputs (its own pages renumbered 0..)."""
    wl = host["_wl"]
    pages = host["page_table"][b]
    pages = pages[pages >= 0]
    idx = torch.from_numpy(pages.astype(np.int64)).cuda()
    return dict(
        q=_bf16_host(wl.q[b:b + 1]), k_new=_bf16_host(wl.k_new[b:b + 1]),
        v_new=_bf16_host(wl.v_new[b:b + 1]),
        k_pool=_bf16_host(wl.k_pool.index_select(0, idx)),
        v_pool=_bf16_host(wl.v_pool.index_select(0, idx)),
        page_table=np.arange(len(pages), dtype=np.int32)[None, :],
        kv_len=host["kv_len"][b:b + 1], n_clean=host["n_clean"][b:b + 1])


class LoopWorkload:
    """Device buffers of the stationary-batch loop (isd_loop) at a config.

    The block's activations come from token -> (q, k, v) tables of V + 1 rows
    (row V is the MASK token) drawn N(0, qkv_std); the prefix pages hold
    N(0, kv_std) keys and values; the LM head is N(0, w_std).  The pool has
    room for every request's prefix plus ``capacity_steps`` steps of growth,
    handed out on the device.  Every request starts with one clean token.  With
    a LoRA rank in the config, the gated adapter (N(0, lora_std)) is applied
    to the MASK rows as in the single step.

    The acceptance rate of the loop is a property of this synthetic model: a
    proposal x (argmax of the previous step's MASK row q) is kept with
    probability min(1, p(x)/q(x)), and p and q are the LM head applied to two
    attention outputs over almost the same context; w_std scales the logit
    gap between them, so it sets the rate.
    """

    FIELDS = ("Eq", "Ek", "Ev", "W", "k_pool", "v_pool", "page_table", "pages_used",
              "next_free_page", "kv_len", "n_clean", "clean_tok", "logits", "row_stats", "q",
              "k_new", "v_new", "hidden")

    def __init__(self, isd, cfg: I.IsdConfig, capacity_steps: int, seed: int = 0,
                 w_std: Optional[float] = None, qkv_std: Optional[float] = None,
                 kv_std: Optional[float] = None):
        self.isd, self.cfg, self.seed = isd, cfg, seed
        B, N, Q, V, P = cfg.B, cfg.N, cfg.Q, cfg.V, cfg.page_size
        w_std = cfg.w_std if w_std is None else w_std
        qkv_std = cfg.qkv_std if qkv_std is None else qkv_std
        kv_std = cfg.kv_std if kv_std is None else kv_std
        self.w_std, self.qkv_std, self.kv_std = w_std, qkv_std, kv_std
        kv0 = I.prefix_lengths(cfg, seed)
        pre = (kv0.astype(np.int64) + P - 1) // P
        max_pages = int((kv0.max() + capacity_steps * N + Q + P - 1) // P + 1)
        num_pages = int(pre.sum()) + B * max_pages
        table = np.full((B, max_pages), -1, np.int32)
        nxt = 0
        for b in range(B):
            table[b, : pre[b]] = np.arange(nxt, nxt + pre[b], dtype=np.int32)
            nxt += int(pre[b])
        rng = np.random.default_rng([seed, 37])
        tok0 = np.full((B, N), -1, np.int32)
        tok0[:, 0] = rng.integers(0, V, B)
        self.kv0 = kv0
        self.capacity_steps = capacity_steps
        self.dims = isd.make_dims(B, N, cfg.Hq, cfg.Hkv, cfg.D, V, P, num_pages, max_pages,
                                  cfg.lora_rank)
        d = self.dims
        gen = torch.Generator(device="cuda")
        gen.manual_seed(seed)
        self.Eq = _randn_bf16((V + 1, cfg.Hq, cfg.D), qkv_std, gen)
        self.Ek = _randn_bf16((V + 1, cfg.Hkv, cfg.D), qkv_std, gen)
        self.Ev = _randn_bf16((V + 1, cfg.Hkv, cfg.D), qkv_std, gen)
        self.W = _randn_bf16((V, cfg.H), w_std, gen)
        self.k_pool = _randn_bf16((num_pages, P, cfg.Hkv, cfg.D), kv_std, gen)
        self.v_pool = _randn_bf16((num_pages, P, cfg.Hkv, cfg.D), kv_std, gen)
        r = cfg.lora_rank
        self.lora_A = _randn_bf16((cfg.H, r), cfg.lora_std, gen) if r else None
        self.lora_B = _randn_bf16((r, cfg.H), cfg.lora_std, gen) if r else None
        dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
        self.page_table = dev(table)
        self.pages_used = dev(pre.astype(np.int32))
        self.next_free_page = dev(np.array([nxt], np.int32))
        self.kv_len = dev(np.stack([kv0.astype(np.int32), np.zeros(B, np.int32)]))
        self.n_clean = dev(np.stack([np.ones(B, np.int32), np.zeros(B, np.int32)]))
        self.clean_tok = dev(np.stack([tok0, np.full((B, N), -1, np.int32)]))
        M = d.M
        self.logits = torch.zeros(2 * M * V, dtype=torch.float32, device="cuda")
        self.row_stats = torch.zeros(2 * M * 4, dtype=torch.int32, device="cuda")
        self.q = torch.empty(M * cfg.Hq * cfg.D, dtype=torch.bfloat16, device="cuda")
        self.k_new = torch.empty(M * cfg.Hkv * cfg.D, dtype=torch.bfloat16, device="cuda")
        self.v_new = torch.empty(M * cfg.Hkv * cfg.D, dtype=torch.bfloat16, device="cuda")
        self.hidden = torch.empty(M * d.H, dtype=torch.bfloat16, device="cuda")
        self.uniforms = dev(np.stack([I.step_uniforms(seed, k, B, N)
                                      for k in range(capacity_steps)]))
        self.accept_len_hist = torch.zeros(capacity_steps, B, dtype=torch.int32, device="cuda")
        self.out_tok_hist = torch.zeros(capacity_steps, B, N, dtype=torch.int32, device="cuda")
        self.ws = isd.alloc_workspace(d)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.done = 0
        self._initial = {f: getattr(self, f).clone() for f in self.STATE}

    # the requests' state and the page bookkeeping; the KV pool needs no reset
    # (a position past a request's prefix is appended before it is read)
    STATE = ("page_table", "pages_used", "next_free_page", "kv_len", "n_clean", "clean_tok")

    def reset(self):
        """Back to the state before the first step (stream-ordered copies)."""
        for f in self.STATE:
            getattr(self, f).copy_(self._initial[f])
        self.done = 0

    def args(self, start: int, n: int):
        """Checked isd_loop arguments for steps start .. start+n-1 (start even,
        so that the state and logits of step ``start`` are in buffer 0)."""
        if start % 2 or start + n > self.capacity_steps:
            raise ValueError("loop steps must start even and stay within capacity")
        t = {f: getattr(self, f) for f in self.FIELDS}
        if self.cfg.lora_rank:
            t["lora_A"], t["lora_B"] = self.lora_A, self.lora_B
        t["uniforms"] = self.uniforms[start:start + n]
        t["accept_len_hist"] = self.accept_len_hist[start:start + n]
        t["out_tok_hist"] = self.out_tok_hist[start:start + n]
        return self.isd.loop_args(self.dims, n, **t)

    def run(self, n: int, stream=None, args=None):
        """Enqueue the next n steps (n even keeps the next call's start even)."""
        a = args if args is not None else self.args(self.done, n)
        self.isd.loop(self.dims, n, self.ws, err_flag=self.err, stream=stream, args=a)
        self.done += n

    def state_host(self):
        """n_clean of the current state (buffer 0 after an even number of steps)."""
        return self.n_clean[self.done & 1].cpu().numpy()

    def stats(self, start: int, stop: int, c_start=None) -> Dict[str, float]:
        """Tokens per forward and the proposal acceptance rate of steps
        start .. stop-1 of this loop (see ``loop_stats``)."""
        al = self.accept_len_hist[:stop].cpu().numpy()
        return loop_stats(al, self.cfg.N, start, stop, c_start)


def loop_stats(al: np.ndarray, N: int, start: int, stop: int, c_start=None) -> Dict[str, float]:
    """Tokens per forward and the proposal acceptance rate of steps
    start .. stop-1 from an accept-length history al [steps, B].

    The clean count c of each step follows from the history: every request
    starts at c = 1; a step that keeps all of its c tokens continues with
    c = N, any other with c = 1 (the restart).  A step with c clean tokens
    tests proposals 2..c in order and stops at the first rejection, so it
    accepted A - 1 of them and made one more (rejected) test if A < c.
    c_start: the clean counts at step `start`, when the history before it is
    not the same run."""
    al = np.asarray(al, np.int64)
    c = np.ones(al.shape[1], np.int64)
    first = 0
    if c_start is not None:
        c = np.asarray(c_start, np.int64).copy()
        first = start
    acc = tests = 0
    acc_pos = np.zeros(max(N - 1, 1))
    tests_pos = np.zeros(max(N - 1, 1))
    for s in range(first, stop):
        A = al[s]
        if s >= start:
            full = A == c
            tested = np.where(full, c - 1, A)
            acc += int((A - 1).sum())
            tests += int(tested.sum())
            for j in range(N - 1):
                tests_pos[j] += int((tested > j).sum())
                acc_pos[j] += int((A - 1 > j).sum())
        c = np.where(A == c, N, 1)
    window = al[start:stop]
    tpf = float(window.mean())
    se = float(window.mean(axis=0).std(ddof=1) / math.sqrt(window.shape[1]))
    return dict(tokens=int(window.sum()), tpf=tpf, tpf_se=se,
                accept_rate=acc / max(tests, 1), tests=tests,
                accept_rate_by_position=[float(a / max(t, 1)) for a, t in zip(acc_pos, tests_pos)])


class SdarLoopWorkload:
    """A stationary batch of SDAR-style confidence-threshold block decoding
    (isd_sdar_loop) on the synthetic table model of ``LoopWorkload`` (per-token
    q/k/v tables with a MASK row, a random LM head, random prefixes), with q
    and k rotated by position (rope=True): under the block's bidirectional
    mask, rows that carry the same MASK embedding would otherwise be
    identical and be committed all at once or one by one.  Blocks of N
    positions; tau and sync are arguments of ``run``.  The state (kv_len,
    block_tok, steps, page bookkeeping) is updated in place."""

    FIELDS = ("Eq", "Ek", "Ev", "W", "k_pool", "v_pool", "page_table", "pages_used",
              "next_free_page", "kv_len", "block_tok", "steps", "logits", "row_stats", "q",
              "k_new", "v_new", "hidden")
    STATE = ("page_table", "pages_used", "next_free_page", "kv_len", "block_tok", "steps")

    def __init__(self, isd, cfg: I.IsdConfig, capacity_steps: int, seed: int = 0,
                 w_std: Optional[float] = None, qkv_std: Optional[float] = None,
                 kv_std: Optional[float] = None, rope: bool = True):
        self.isd, self.cfg, self.seed = isd, cfg, seed
        B, N, V, P = cfg.B, cfg.N, cfg.V, cfg.page_size
        w_std = cfg.w_std if w_std is None else w_std
        qkv_std = cfg.qkv_std if qkv_std is None else qkv_std
        kv_std = cfg.kv_std if kv_std is None else kv_std
        self.w_std, self.qkv_std, self.kv_std = w_std, qkv_std, kv_std
        kv0 = I.prefix_lengths(cfg, seed)
        pre = (kv0.astype(np.int64) + P - 1) // P
        # a block advances kv_len by N at most once per forward
        max_pages = int((kv0.max() + (capacity_steps + 1) * N + P - 1) // P + 1)
        num_pages = int(pre.sum()) + B * max_pages
        table = np.full((B, max_pages), -1, np.int32)
        nxt = 0
        for b in range(B):
            table[b, : pre[b]] = np.arange(nxt, nxt + pre[b], dtype=np.int32)
            nxt += int(pre[b])
        self.kv0 = kv0
        self.capacity_steps = capacity_steps
        self.dims = isd.make_dims(B, N, cfg.Hq, cfg.Hkv, cfg.D, V, P, num_pages, max_pages)
        gen = torch.Generator(device="cuda")
        gen.manual_seed(seed)
        self.Eq = _randn_bf16((V + 1, cfg.Hq, cfg.D), qkv_std, gen)
        self.Ek = _randn_bf16((V + 1, cfg.Hkv, cfg.D), qkv_std, gen)
        self.Ev = _randn_bf16((V + 1, cfg.Hkv, cfg.D), qkv_std, gen)
        self.W = _randn_bf16((V, cfg.H), w_std, gen)
        self.k_pool = _randn_bf16((num_pages, P, cfg.Hkv, cfg.D), kv_std, gen)
        self.v_pool = _randn_bf16((num_pages, P, cfg.Hkv, cfg.D), kv_std, gen)
        dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
        self.page_table = dev(table)
        self.pages_used = dev(pre.astype(np.int32))
        self.next_free_page = dev(np.array([nxt], np.int32))
        self.kv_len = dev(kv0.astype(np.int32))
        self.block_tok = dev(np.full((B, N), -1, np.int32))
        self.steps = dev(np.zeros(B, np.int32))
        M = B * N
        self.logits = torch.zeros(M * V, dtype=torch.float32, device="cuda")
        self.row_stats = torch.zeros(M * 4, dtype=torch.int32, device="cuda")
        self.q = torch.empty(M * cfg.Hq * cfg.D, dtype=torch.bfloat16, device="cuda")
        self.k_new = torch.empty(M * cfg.Hkv * cfg.D, dtype=torch.bfloat16, device="cuda")
        self.v_new = torch.empty(M * cfg.Hkv * cfg.D, dtype=torch.bfloat16, device="cuda")
        self.hidden = torch.empty(M * cfg.H, dtype=torch.bfloat16, device="cuda")
        self.unmasked_hist = torch.zeros(capacity_steps, B, dtype=torch.int32, device="cuda")
        self.out_tok_hist = torch.zeros(capacity_steps, B, N, dtype=torch.int32, device="cuda")
        self.block_steps_hist = torch.zeros(capacity_steps, B, dtype=torch.int32, device="cuda")
        # rotary table for every position the run can reach
        self.rope = dev(I.rope_table(max_pages * P, cfg.D)) if rope else None
        self.ws = isd.alloc_workspace(self.dims)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.done = 0
        self._initial = {f: getattr(self, f).clone() for f in self.STATE}

    def reset(self):
        """Back to the state before the first forward (stream-ordered copies)."""
        for f in self.STATE:
            getattr(self, f).copy_(self._initial[f])
        self.done = 0

    def args(self, start: int, n: int):
        """Checked isd_sdar_loop arguments for forwards start .. start+n-1."""
        if start + n > self.capacity_steps:
            raise ValueError("loop steps must stay within capacity")
        t = {f: getattr(self, f) for f in self.FIELDS}
        t["unmasked_hist"] = self.unmasked_hist[start:start + n]
        t["out_tok_hist"] = self.out_tok_hist[start:start + n]
        t["block_steps_hist"] = self.block_steps_hist[start:start + n]
        return self.isd.sdar_loop_args(self.dims, n, rope=self.rope, **t)

    def run(self, n: int, tau: float, sync: bool, stream=None, args=None):
        """Enqueue the next n forwards."""
        a = args if args is not None else self.args(self.done, n)
        self.isd.sdar_loop(self.dims, tau, sync, n, self.ws, err_flag=self.err, stream=stream,
                           args=a)
        self.done += n

    def stats(self, start: int, stop: int) -> Dict[str, float]:
        """Block statistics of forwards start .. stop-1 (see ``sdar_round_stats``)."""
        h = self.block_steps_hist[start:stop].cpu().numpy()
        return sdar_round_stats(h, self.cfg.N)


def sdar_round_stats(block_steps_hist: np.ndarray, N: int) -> Dict[str, float]:
    """Forwards per block from a decision history block_steps_hist [steps, B]
    (S_b of a block that left the batch at that step, else 0).

    S_b counts the denoising forwards request b's block needed on its own;
    every block also takes one store pass.  Under batch sync all blocks of a
    round leave at the same step, so every step with leavers closes a round
    of max_b S_b + 1 forwards; tokens per forward of a request are then
    N / (E[max S_b] + 1) against N / (E[S_b] + 1) without the sync."""
    h = np.asarray(block_steps_hist, np.int64)
    rows = h[(h > 0).any(axis=1)]
    if rows.size == 0:
        return dict(blocks=0, rounds=0, mean_S=float("nan"), mean_max_S=float("nan"),
                    tpf_free=float("nan"), tpf_sync=float("nan"), pmf=[])
    s_b = rows[rows > 0]
    mean_s = float(s_b.mean())
    mean_max = float(rows.max(axis=1).mean())
    pmf = np.bincount(s_b, minlength=N + 1)[1:N + 1] / s_b.size
    return dict(blocks=int(s_b.size), rounds=int(rows.shape[0]), mean_S=mean_s,
                mean_max_S=mean_max, tpf_free=N / (mean_s + 1.0), tpf_sync=N / (mean_max + 1.0),
                pmf=[float(x) for x in pmf])


def expected_max_of(pmf, B: int) -> float:
    """E[max of B independent draws] of S with P(S = s) = pmf[s-1], from the
    distribution function: P(max <= s) = F(s)^B."""
    F = np.cumsum(np.asarray(pmf, np.float64))
    if F.size == 0 or F[-1] <= 0:
        return float("nan")
    F = np.minimum(F / F[-1], 1.0)
    lower = np.concatenate([[0.0], F[:-1]])
    return float(np.sum(np.arange(1, F.size + 1) * (F ** B - lower ** B)))


class DeepWorkload:
    """A full-depth synthetic model over the ISD block, resident on the GPU:
    n_layers Qwen3-style decoder layers (hidden Hq*D, GQA Hkv heads,
    intermediate ``inter``) with random weights, an embedding table with a
    MASK row, the final norm and the LM head, one paged K/V pool per layer
    holding random prefixes, and one batch state (kv_len, n_clean, clean
    tokens).  ``views`` gives other strides N over the same weights and
    pools (N = 1 is autoregressive decoding: one query per request).

    Projections are drawn N(0, 1/K) for K inputs, so each keeps the scale of
    its input; norm weights 1 + N(0, 0.1^2); embeddings N(0, 1)."""

    def __init__(self, isd, cfg: I.IsdConfig, n_layers: int, inter: int, seed: int = 0,
                 n_clean: str = "full", eps: float = 1e-6, max_q: Optional[int] = None):
        self.isd, self.cfg, self.n_layers, self.inter, self.eps = isd, cfg, n_layers, inter, eps
        B, N, V, P, D = cfg.B, cfg.N, cfg.V, cfg.page_size, cfg.D
        H = cfg.Hq * D
        self.H = H
        kv0 = I.prefix_lengths(cfg, seed)
        max_q = max_q or cfg.Q
        need = (kv0.astype(np.int64) + max_q + P - 1) // P
        max_pages = int(need.max())
        num_pages = int(need.sum())
        table = np.full((B, max_pages), -1, np.int32)
        off = 0
        for b in range(B):
            table[b, : need[b]] = np.arange(off, off + need[b], dtype=np.int32)
            off += int(need[b])
        self.kv0 = kv0
        self.num_pages, self.max_pages = num_pages, max_pages
        gen = torch.Generator(device="cuda")
        gen.manual_seed(seed)
        rn = lambda shape, std: _randn_bf16(shape, std, gen)
        ones = lambda n: (1.0 + 0.1 * torch.randn(n, device="cuda", generator=gen)).to(torch.bfloat16)
        qkv_rows = (cfg.Hq + 2 * cfg.Hkv) * D
        self.layers = []
        for _ in range(n_layers):
            self.layers.append(dict(
                in_norm=ones(H), w_qkv=rn((qkv_rows, H), H ** -0.5), q_norm=ones(D), k_norm=ones(D),
                w_o=rn((H, cfg.Hq * D), (cfg.Hq * D) ** -0.5), post_norm=ones(H),
                w_gate_up=rn((2 * inter, H), H ** -0.5), w_down=rn((H, inter), inter ** -0.5),
                k_pool=rn((num_pages, P, cfg.Hkv, D), 1.0), v_pool=rn((num_pages, P, cfg.Hkv, D), 1.0)))
        self.E = rn((V + 1, H), 1.0)
        self.final_norm = ones(H)
        self.W = rn((V, H), cfg.w_std)
        self.rope = torch.from_numpy(I.rope_table(max_pages * P, D)).cuda()
        self.page_table = torch.from_numpy(table).cuda()
        self.views = {}
        self.view(N, n_clean, seed)

    def view(self, N: int, n_clean: str = "full", seed: int = 0):
        """Buffers and state for stride N (Q = 2N-1) over the shared weights."""
        if N in self.views:
            return self.views[N]
        cfg, isd = self.cfg, self.isd
        B, V, P, D = cfg.B, cfg.V, cfg.page_size, cfg.D
        Q = 2 * N - 1
        d = isd.make_dims(B, N, cfg.Hq, cfg.Hkv, D, V, P, self.num_pages, self.max_pages)
        M = B * Q
        rng = np.random.default_rng([seed, 41, N])
        nc = np.full(B, N, np.int32) if n_clean == "full" else np.ones(B, np.int32)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        v = dict(dims=d, Q=Q, M=M,
                 kv_len=dev(self.kv0.astype(np.int32)), n_clean=dev(nc),
                 clean_tok=dev(rng.integers(0, V, (B, N)).astype(np.int32)),
                 x=torch.empty(M * self.H, dtype=torch.bfloat16, device="cuda"),
                 out=torch.empty(M * self.H, dtype=torch.bfloat16, device="cuda"),
                 logits=torch.zeros(M * V, dtype=torch.float32, device="cuda"),
                 prev_logits=torch.zeros(M * V, dtype=torch.float32, device="cuda"),
                 row_stats=torch.zeros(M * 4, dtype=torch.int32, device="cuda"),
                 prev_row_stats=torch.zeros(M * 4, dtype=torch.int32, device="cuda"),
                 uniforms=dev(I.step_uniforms(seed, 0, B, N)),
                 accept_len=torch.zeros(B, dtype=torch.int32, device="cuda"),
                 out_tok=torch.zeros(B * N, dtype=torch.int32, device="cuda"),
                 next_n_clean=torch.zeros(B, dtype=torch.int32, device="cuda"),
                 next_clean_tok=torch.zeros(B * N, dtype=torch.int32, device="cuda"),
                 next_kv_len=torch.zeros(B, dtype=torch.int32, device="cuda"),
                 ws=isd.alloc_layers_workspace(d, self.inter),
                 err=torch.zeros(1, dtype=torch.int32, device="cuda"))
        v["layer_arr"] = isd.layer_array(d, self.inter, self.layers)
        self.views[N] = v
        return v

    def forward(self, N: int, n_layers: Optional[int] = None, stream=None, embed: bool = True):
        """Embeddings (unless embed=False: x as it stands), the first n_layers
        layers (all by default), the final norm into out."""
        v, isd = self.views[N], self.isd
        d = v["dims"]
        if embed:
            isd.embed_block(d, self.E, v["n_clean"], v["clean_tok"], v["x"], err_flag=v["err"],
                            stream=stream)
        n = self.n_layers if n_layers is None else n_layers
        isd.layers(d, self.inter, self.eps, v["layer_arr"], n, self.rope, v["x"], self.page_table,
                   v["kv_len"], v["n_clean"], v["ws"], final_norm=self.final_norm, out=v["out"],
                   err_flag=v["err"], stream=stream)

    def step(self, N: int, stream=None):
        """One whole step at stride N: the forward, the LM head with row
        statistics, the p/q accept against the previous logits buffer (the
        state is not advanced: repeated steps replay the same block)."""
        v, isd = self.views[N], self.isd
        d = v["dims"]
        self.forward(N, stream=stream)
        isd.lm_head(d, v["out"], self.W, v["logits"], v["row_stats"], v["ws"], err_flag=v["err"],
                    stream=stream)
        isd.accept(d, v["logits"], v["row_stats"], v["prev_logits"], v["prev_row_stats"],
                   v["n_clean"], v["clean_tok"], v["kv_len"], v["uniforms"], v["accept_len"],
                   v["out_tok"], v["next_n_clean"], v["next_clean_tok"], v["next_kv_len"], v["ws"],
                   err_flag=v["err"], stream=stream)

    def weight_bytes(self) -> float:
        """Bytes of weights one step streams: every layer's projections and
        norms, the LM head (embedding rows read are negligible)."""
        per = sum(t.numel() * 2 for k, t in self.layers[0].items() if k not in ("k_pool", "v_pool"))
        return float(per * self.n_layers + self.W.numel() * 2)


__all__ = ["DeepWorkload", "DeviceWorkload", "LoopWorkload", "SdarLoopWorkload",
           "expected_max_of", "loop_stats", "request_slice", "sdar_round_stats"]
