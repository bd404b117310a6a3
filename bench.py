#!/usr/bin/env python
"""Benchmark: batched ISD verify-and-propose step on B200.

One step = attention over the paged KV cache (with the KV append) + LM head +
row statistics + p/q accept / residual draw / proposals, for a batch of B
requests, through the C ABI of libisd.so.  Default workload: Qwen3-8B shapes,
B=32, N=4 (Q=7), prefixes U[512, 8192] in 16-token pages, vocab 151936, bf16,
constructed per-position acceptance 0.9.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle
instead (host cores, bounded samples of the same workload).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ISD steps/s and accepted tokens/s at B=32,N=4 (Qwen3-8B shapes); % HBM roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="qwen3_8b_b32_n4")
    ap.add_argument("--accept-rate", type=float, default=None,
                    help="constructed per-proposal acceptance (default: the config's)")
    ap.add_argument("--e2e-steps", type=int, default=2000,
                    help="timed steps of the end-to-end leg (at most --steps; the same count "
                         "keeps both legs in the same clock regime under the power cap)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--sustained-s", type=float, default=2.5,
                    help="seconds of the sustained leg; 0 skips it")
    ap.add_argument("--loop-steps", type=int, default=400,
                    help="timed steps of the closed-loop leg (isd_loop); 0 skips it")
    ap.add_argument("--deep-steps", type=int, default=30,
                    help="timed steps per stride of the full-depth leg (36 layers); 0 skips it")
    ap.add_argument("--deep-layers", type=int, default=36)
    ap.add_argument("--deep-only", action="store_true",
                    help="run only the full-depth leg and print its object")
    ap.add_argument("--sdar-only", action="store_true",
                    help="run only the SDAR-style comparison leg and print its object")
    ap.add_argument("--sdar-steps", type=int, default=400,
                    help="timed forwards of the SDAR-style comparison leg (isd_sdar_loop), "
                         "per scheduling mode; 0 skips it")
    return ap.parse_args()


# ---------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(
            j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        rows = [l.split(", ") for l in self.lines if l]
        if self.bus_id:
            mine = [r for r in rows if len(r) > 1 and r[1].strip().lower().endswith(
                self.bus_id.lower()[-10:])]
            rows = mine or rows
        if not rows:
            return None
        idx0 = rows[0][0]
        rows = [r for r in rows if r[0] == idx0 and len(r) >= 10]
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def profile_traffic(kernel_file: str):
    """dram bytes per launch of the LM-head kernel from the committed ncu summary,
    if the kernel source is unchanged since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "lm_head_traffic.json")
    src = os.path.join(ROOT, "speculative_verification_isd_b200", "csrc", kernel_file)
    if not (os.path.exists(p) and os.path.exists(src)):
        return None
    with open(p) as f:
        j = json.load(f)
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if j.get("source_sha256_16") != h:
        return None
    return j.get("dram_bytes_per_launch_full")


# ---------------------------------------------------------------------------
# CPU oracle sampling (used by the cpu_baseline leg and by --impl reference)
# ---------------------------------------------------------------------------
class OracleSampler:
    """Timed oracle runs on bounded pieces of one ISD step of the workload.

    Inputs are generated on the host from ``inputs`` (seeded; same shapes and
    distributions as the GPU workload) -- nothing here touches the GPU or the
    CUDA library.  One sample times, with the oracle as it stands:
      * the attention of one request (its whole prefix and block);
      * the LM head of all B*Q rows over a ``vs``-entry slice of the vocabulary
        (those rows: the sampled requests' attention outputs, seeded bf16
        rows for requests not sampled yet);
      * the acceptance of one request on full-vocabulary rows (seeded N(0,1)
        logits; the previous step's MASK rows constructed so that p/q = a at
        every proposal, as in the GPU workload).
    A full step is B x attention + (V / vs) x LM-head slice + B x acceptance.
    """

    def __init__(self, cfg, seed=0):
        import numpy as np
        from oracle import isd_oracle as O
        from speculative_verification_isd_b200 import inputs as I
        self.O, self.I, self.np, self.cfg, self.seed = O, I, np, cfg, seed
        self.kv_len = I.prefix_lengths(cfg, seed)
        rng = np.random.default_rng([seed, 41])
        self.clean_tok = rng.integers(0, cfg.V, size=(cfg.B, cfg.N)).astype(np.int32)
        self.hidden = I.f32_to_bf16_bits(
            rng.standard_normal((cfg.M, cfg.H), dtype=np.float32) * np.float32(cfg.qkv_std))
        self._req = {}
        self._w = {}
        self._acc = {}
        self.threads = self._threads()

    @staticmethod
    def _threads():
        try:
            from threadpoolctl import threadpool_info
            n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
            return max(n) if n else 1
        except Exception:
            return os.cpu_count() or 1

    def _bf16(self, rng, shape, std):
        np = self.np
        return self.I.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))

    def request_inputs(self, b):
        """One request's block activations and its own pages (renumbered 0..)."""
        if b not in self._req:
            np, cfg = self.np, self.cfg
            rng = np.random.default_rng([self.seed, 43, b])
            kv = int(self.kv_len[b])
            pages = (kv + cfg.Q + cfg.page_size - 1) // cfg.page_size
            self._req = {b: dict(
                q=self._bf16(rng, (1, cfg.Q, cfg.Hq, cfg.D), cfg.qkv_std),
                k_new=self._bf16(rng, (1, cfg.Q, cfg.Hkv, cfg.D), cfg.qkv_std),
                v_new=self._bf16(rng, (1, cfg.Q, cfg.Hkv, cfg.D), cfg.qkv_std),
                k_pool=self._bf16(rng, (pages, cfg.page_size, cfg.Hkv, cfg.D), cfg.kv_std),
                v_pool=self._bf16(rng, (pages, cfg.page_size, cfg.Hkv, cfg.D), cfg.kv_std),
                page_table=np.arange(pages, dtype=np.int32)[None, :],
                kv_len=self.kv_len[b:b + 1], n_clean=np.full(1, cfg.N, np.int32))}
        return self._req[b]

    def w_slice(self, k, vs):
        if (k, vs) not in self._w:
            rng = self.np.random.default_rng([self.seed, 47, k])
            self._w = {(k, vs): self._bf16(rng, (vs, self.cfg.H), self.cfg.w_std)}
        return self._w[(k, vs)]

    def accept_inputs(self, b):
        """Full-vocabulary logits of one request: this step's rows and the
        previous step's, with p(x)/q(x) = a at every proposal x."""
        if b not in self._acc:
            np, cfg = self.np, self.cfg
            rng = np.random.default_rng([self.seed, 53, b])
            N, Q, V = cfg.N, cfg.Q, cfg.V
            z = rng.standard_normal((1, Q, V), dtype=np.float32)
            zp = rng.standard_normal((1, Q, V), dtype=np.float32)
            a = cfg.accept_rate if cfg.accept_rate is not None else 0.9
            for j in range(2, N + 1):
                x = int(self.clean_tok[b, j - 1])
                row = z[0, j - 2].astype(np.float64)
                P = float(np.exp(row[x] - row.max()) / np.exp(row - row.max()).sum())
                q = z[0, j - 2].copy()
                q[x] = np.float32(row[x] + np.log((1.0 - P) / (a - P)))
                zp[0, N + j - 2] = q
            self._acc = {b: (z, zp)}
        return self._acc[b]

    def sample(self, k, vs):
        """Times one sample; returns (estimated full-step seconds, seconds spent)."""
        cfg, O = self.cfg, self.O
        b = k % cfg.B
        r = self.request_inputs(b)
        w = self.w_slice(k % 4, vs)
        z, zp = self.accept_inputs(b)
        t0 = time.perf_counter()
        hid, _, _ = O.attention(r["q"], r["k_new"], r["v_new"], r["k_pool"], r["v_pool"],
                                r["page_table"], r["kv_len"], r["n_clean"], cfg.N,
                                cfg.page_size, cfg.D ** -0.5)
        t1 = time.perf_counter()
        self.hidden[b * cfg.Q:(b + 1) * cfg.Q] = hid
        O.lm_head(self.hidden, w)
        t2 = time.perf_counter()
        O.accept(z, zp, self.np.full(1, cfg.N, self.np.int32), self.clean_tok[b:b + 1],
                 self.kv_len[b:b + 1], self.I.step_uniforms(self.seed, k, 1, cfg.N), cfg.N)
        t3 = time.perf_counter()
        ta, tl, tc = t1 - t0, t2 - t1, t3 - t2
        return cfg.B * ta + (cfg.V / vs) * tl + cfg.B * tc, t3 - t0


def oracle_rate(cfg, budget_s, max_samples=400, vs=8192):
    """Median extrapolated full-step rate of the oracle over samples that fit
    the time budget."""
    sampler = OracleSampler(cfg)
    ests, spent, k = [], 0.0, 0
    while spent < budget_s and k < max_samples:
        est, used = sampler.sample(k, vs)
        ests.append(est)
        spent += used
        k += 1
    est = statistics.median(ests)
    return est, k, spent, sampler.threads, vs


def cpu_baseline(cfg, budget_s):
    est, k, spent, threads, vs = oracle_rate(cfg, budget_s)
    return {"value": 1.0 / est, "unit": "ISD steps/s", "cores": threads, "kind": "oracle",
            "sample": (f"{k} samples ({spent:.1f} s of CPU work), each: 1 request's attention, "
                       f"the LM head of all {cfg.M} rows over a {vs}-entry vocabulary slice, 1 "
                       f"request's acceptance on full-vocabulary rows; full step extrapolated as "
                       f"{cfg.B} x attention + {cfg.V}/{vs} x LM-head slice + {cfg.B} x "
                       f"acceptance; inputs generated on the host (same recipe and shapes)")}


def accept_parity(wl, cfg, k):
    """The GPU's accept outputs of one step of the timed workload against the
    oracle's acceptance fed the same (GPU) logits: decisions and tokens
    identical except counted near-threshold decisions and rounding-explained
    draws.  Run on rank 0 after the timed region, in the CPU-baseline leg."""
    import numpy as np
    import torch
    from oracle import isd_oracle as O
    from oracle import parity as P
    wl.set_uniforms(k)
    wl.step()
    torch.cuda.synchronize()
    gpu = wl.outputs()
    B, Q, V = cfg.B, cfg.Q, cfg.V
    z = wl.logits.cpu().numpy().reshape(B, Q, V)
    zp = wl.prev_logits.cpu().numpy().reshape(B, Q, V)
    host = dict(n_clean=wl.n_clean.cpu().numpy(), clean_tok=wl.clean_tok.cpu().numpy(),
                kv_len=wl.kv_len.cpu().numpy(), uniforms=wl.uniforms.cpu().numpy())
    t0 = time.perf_counter()
    ores = O.accept(z, zp, host["n_clean"], host["clean_tok"], host["kv_len"], host["uniforms"],
                    cfg.N, O.PROPOSE_ARGMAX)
    rep = P.compare_accept(gpu, ores, z, zp, host, cfg.N, O.PROPOSE_ARGMAX)
    rep.update(step_uniforms_index=int(k), oracle_seconds=round(time.perf_counter() - t0, 2),
               rejections=int((ores["rejected_at"] > 0).sum()),
               rule="decisions, lengths, states, token ids identical; skipped: |u - p/q| < 1e-5; "
                    "excused: draws within 1e-5 * sum(w) of the oracle's inverse-CDF target")
    return rep


# ---------------------------------------------------------------------------
# LM head scale of the closed-loop model.  The proposal acceptance of the loop
# is a property of its synthetic model (see LoopWorkload); at this scale the
# measured rate at B=32, N=4 is about 0.9, the rate of the tokens-per-forward
# table on the engineering page (section on the core parameters of token
# generation).  Attention inputs N(0, 0.5), cache N(0, 1.0).
LOOP_W_STD, LOOP_QKV_STD, LOOP_KV_STD = 0.1, 0.5, 1.0


def restart_model_tpf(a, N):
    """Tokens per forward of the restart state machine when every proposal is
    kept with probability a: a cycle that keeps all N-1 proposals (probability
    a^(N-1)) is one forward; any other adds a restart forward (one clean
    token) and emits one replacement token."""
    f = a ** (N - 1)
    eacc = (1.0 - a ** N) / (1.0 - a) if a < 1.0 else float(N)
    return (eacc + 1.0 - f) / (2.0 - f)


def closed_loop(isd, cfg, R, K, bus, seed):
    """Closed-loop leg: isd_loop runs K steps of a stationary batch on the
    device (block activations by table lookup, pages from the on-device
    allocator, accept state and logits in double buffers; five kernels per
    step), after 16 untimed steps.  Tokens/s counts every token the requests
    emitted in the timed steps, over the slowest rank's time."""
    import torch
    from speculative_verification_isd_b200.workload import LoopWorkload
    W = 16
    K += K % 2
    lw = LoopWorkload(isd, cfg, capacity_steps=W + K, seed=seed, w_std=LOOP_W_STD,
                      qkv_std=LOOP_QKV_STD, kv_std=LOOP_KV_STD)
    stream = torch.cuda.current_stream()
    lw.run(W)
    torch.cuda.synchronize()
    args = lw.args(W, K)
    clocks = ClockSampler(bus)
    clocks.start()
    time.sleep(0.2)
    R.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    lw.run(K, args=args)
    e1.record(stream)
    torch.cuda.synchronize()
    R.barrier()
    clk = clocks.stop()
    ms = R.max(e0.elapsed_time(e1))
    st = lw.stats(W, W + K)
    tokens = R.sum(st["tokens"])
    kv_end = lw.kv_len[0].float().mean().item()
    # the same steps again, the timed K captured once in a CUDA graph: back to
    # the initial state, W steps eagerly, capture, one timed replay (the same
    # work as the eager timed run, and the same results)
    graph = None
    al_eager = lw.accept_len_hist[W:W + K].clone()
    try:
        lw.reset()
        lw.run(W)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            lw.isd.loop(lw.dims, K, lw.ws, err_flag=lw.err, stream=torch.cuda.current_stream(), args=args)
        R.barrier()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        R.barrier()
        gms = R.max(g0.elapsed_time(g1))
        graph = {"steps": K, "ms_per_step": gms / K, "steps_per_s": K * R.world / (gms / 1e3),
                 "tokens_per_s": tokens / (gms / 1e3),
                 "same_accept_lengths_as_eager": bool(torch.equal(al_eager, lw.accept_len_hist[W:W + K])),
                 "err_flags": int(lw.err.item())}
        del g
    except RuntimeError as e:  # capture unsupported in this process: report why
        graph = {"unavailable": str(e).splitlines()[0][:200]}
    out = {"workload": cfg.name + " closed loop", "steps": K, "warmup": W,
           "ms_per_step": ms / K, "steps_per_s": K * R.world / (ms / 1e3),
           "tokens_per_s": tokens / (ms / 1e3), "tpf": st["tpf"], "tpf_se": st["tpf_se"],
           "accept_rate": st["accept_rate"],
           "accept_rate_by_position": st["accept_rate_by_position"],
           "tpf_restart_model_at_measured_rate": restart_model_tpf(st["accept_rate"], cfg.N),
           # compute per output token against AR: TPF^2 / (queries per forward)
           "compute_efficiency_tpf2_over_q": st["tpf"] ** 2 / cfg.Q,
           "model": {"w_std": LOOP_W_STD, "qkv_std": LOOP_QKV_STD, "kv_std": LOOP_KV_STD},
           "mean_kv_len": {"start": float(lw.kv0.mean()), "end": kv_end},
           "gpu_launches": 5 * K, "err_flags": int(lw.err.item()), "clocks": clk,
           "cuda_graph": graph}
    del lw
    torch.cuda.empty_cache()
    return out


# SDAR-style comparison leg: confidence threshold of the unmask rule on the
# same table model (q and k rotated by position).  Confidences of this model
# at V = 151936 are small (flat synthetic logits); tau sits near the median
# confidence of fresh-block rows, so blocks need 1..N forwards.
SDAR_TAU = 1.1e-5


def sdar_leg(isd, cfg, R, K, bus, seed, hbm=None):
    """SDAR-style block decoding on the same batch shape, in both scheduling
    modes: batch-synchronous (a round ends when every request's block is
    complete and stored, so it costs max_b S_b + 1 forwards) and free-running
    (each request moves on by itself after S_b + 1, as ISD requests do).  Each mode: 16 untimed forwards,
    then K timed ones of isd_sdar_loop (five kernels per forward).  Tokens
    count the blocks that left the batch in the timed window."""
    import torch
    from speculative_verification_isd_b200 import inputs as I
    from speculative_verification_isd_b200.workload import (SdarLoopWorkload, expected_max_of,
                                                            sdar_round_stats)
    I_prefix = I.prefix_lengths
    W = 16
    stream = torch.cuda.current_stream()
    out = {"workload": cfg.name + " SDAR-style blocks", "block": cfg.N, "queries_per_forward": cfg.N,
           "tau": SDAR_TAU,
           "model": {"w_std": LOOP_W_STD, "qkv_std": LOOP_QKV_STD, "kv_std": LOOP_KV_STD,
                     "rope_base": 1.0e6}}
    for sync in (True, False):
        sw = SdarLoopWorkload(isd, cfg, capacity_steps=W + K, seed=seed, w_std=LOOP_W_STD,
                              qkv_std=LOOP_QKV_STD, kv_std=LOOP_KV_STD)
        sw.run(W, SDAR_TAU, sync)
        torch.cuda.synchronize()
        kv_start = float(sw.kv_len.float().sum().item())
        args = sw.args(W, K)
        clocks = ClockSampler(bus)
        clocks.start()
        time.sleep(0.2)
        R.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        sw.run(K, SDAR_TAU, sync, args=args)
        e1.record(stream)
        torch.cuda.synchronize()
        R.barrier()
        clk = clocks.stop()
        ms = R.max(e0.elapsed_time(e1))
        st = sdar_round_stats(sw.block_steps_hist[W:W + K].cpu().numpy(), cfg.N)
        tokens = R.sum(st["blocks"] * cfg.N)
        # algorithmic bytes of one forward: the LM head's W and logits, the
        # block's K/V prefix reads (the mean of the window's first and last
        # prefix totals) and the block rows
        kv_mean = 0.5 * (kv_start + float(sw.kv_len.float().sum().item()))
        M = cfg.B * cfg.N
        fwd_bytes = (float(cfg.V) * cfg.H * 2 + float(M) * cfg.V * 4
                     + (kv_mean + M) * cfg.Hkv * cfg.D * 2 * 2 + float(M) * cfg.H * 2 * 2)
        mode = {"forwards": K, "ms_per_forward": ms / K, "forwards_per_s": K * R.world / (ms / 1e3),
                "tokens_per_s": tokens / (ms / 1e3), "blocks": st["blocks"],
                "mean_S": st["mean_S"], "S_pmf": st["pmf"],
                "tokens_per_forward_per_request": st["blocks"] * cfg.N / (K * cfg.B),
                # TPF^2 / (queries per forward), N queries a forward
                "compute_efficiency_tpf2_over_q": (st["blocks"] * cfg.N / (K * cfg.B)) ** 2 / cfg.N,
                "algorithmic_bytes_per_forward": fwd_bytes,
                "achieved_gbs": fwd_bytes / (ms / K / 1e3) / 1e9,
                "err_flags": int(sw.err.item()), "gpu_launches": 5 * K, "clocks": clk}
        if hbm:
            mode["frac_of_hbm"] = mode["achieved_gbs"] / hbm
        if sync:
            # forwards per block with the sync over those without it
            mode.update(rounds=st["rounds"], mean_max_S=st["mean_max_S"],
                        sync_penalty=(st["mean_max_S"] + 1.0) / (st["mean_S"] + 1.0))
        out["sync" if sync else "free"] = mode
        del sw
        torch.cuda.empty_cache()
    # the synchronised batch at smaller batch sizes (same model, the first B
    # requests' prefixes): measured E[max S_b] and tokens per forward
    by_batch = {}
    for Bs in (4, 8, 16):
        cb = dataclasses.replace(cfg, B=Bs, fixed_prefix=tuple(int(x) for x in
                                                                I_prefix(cfg, seed)[:Bs]))
        sw = SdarLoopWorkload(isd, cb, capacity_steps=W + K, seed=seed, w_std=LOOP_W_STD,
                              qkv_std=LOOP_QKV_STD, kv_std=LOOP_KV_STD)
        sw.run(W + K, SDAR_TAU, True)
        torch.cuda.synchronize()
        st = sdar_round_stats(sw.block_steps_hist[W:W + K].cpu().numpy(), cfg.N)
        by_batch[str(Bs)] = {"mean_S": st["mean_S"], "mean_max_S": st["mean_max_S"],
                             "rounds": st["rounds"],
                             "tokens_per_forward_per_request": st["blocks"] * cfg.N / (K * Bs),
                             "err_flags": int(sw.err.item())}
        del sw
        torch.cuda.empty_cache()
    by_batch[str(cfg.B)] = {k: out["sync"][k] for k in ("mean_S", "mean_max_S", "rounds",
                                                       "tokens_per_forward_per_request")}
    out["sync_measured_by_batch"] = by_batch
    # E[max S_b] over a batch of B requests, from the free-running S pmf (the
    # distribution of one request's block on its own), and the tokens per
    # forward of a request that a synchronised batch of B would leave
    pmf = out["free"]["S_pmf"]
    emax = {b: expected_max_of(pmf, b) for b in (1, 2, 4, 8, 16, 32, 64)}
    out["expected_max_S_by_batch"] = {str(b): v for b, v in emax.items()}
    out["sync_tokens_per_forward_by_batch"] = {str(b): cfg.N / (v + 1.0) for b, v in emax.items()}
    return out


QWEN3_8B_INTER = 12288


def deep_leg(isd, cfg, R, K, bus, seed, n_layers, tpf=None, hbm=None):
    """Full-depth leg: the whole step through n_layers Qwen3-8B-shaped decoder
    layers (embed, layers, final norm, LM head, accept), random weights, at
    the ISD stride N (Q = 2N-1 queries per request, every request with c = N)
    and at N = 1 (autoregressive decoding: one query per request) on the same
    weights and caches.  Memory-bound decoding makes the two forwards cost
    about the same, so the speed-up over AR is about TPF; tpf (the closed
    loop's tokens per forward) turns the two step times into that speed-up."""
    import numpy as np
    import torch
    from speculative_verification_isd_b200.workload import DeepWorkload
    W = 3
    dw = DeepWorkload(isd, cfg, n_layers, QWEN3_8B_INTER, seed=seed, max_q=cfg.Q)
    dw.view(1)
    stream = torch.cuda.current_stream()
    out = {"workload": f"{cfg.name} full depth ({n_layers} layers)", "layers": n_layers,
           "hidden": dw.H, "intermediate": QWEN3_8B_INTER,
           "weights": "random, N(0, 1/fan_in); bf16", "gemm": "cuBLASLt bf16 (fp32 accumulate)"}
    weight_bytes = dw.weight_bytes()
    kv_bytes = n_layers * float(np.sum(dw.kv0.astype(np.float64))) * cfg.Hkv * cfg.D * 2 * 2
    times = {}
    for N in (cfg.N, 1):
        v = dw.views[N]
        for _ in range(W):
            dw.step(N)
        torch.cuda.synchronize()
        clocks = ClockSampler(bus)
        clocks.start()
        time.sleep(0.2)
        R.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            dw.step(N)
        e1.record(stream)
        torch.cuda.synchronize()
        R.barrier()
        clk = clocks.stop()
        ms = R.max(e0.elapsed_time(e1)) / K
        times[N] = ms
        # the same step captured once in a CUDA graph and replayed K times
        # (the projections' algorithms were chosen in the eager steps)
        graph = None
        try:
            g = torch.cuda.CUDAGraph()
            gs = torch.cuda.Stream()
            gs.wait_stream(stream)
            with torch.cuda.stream(gs):
                with torch.cuda.graph(g, stream=gs):
                    dw.step(N, stream=gs)
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            R.barrier()
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            for _ in range(K):
                g.replay()
            g1.record(stream)
            torch.cuda.synchronize()
            R.barrier()
            graph = {"ms_per_step": R.max(g0.elapsed_time(g1)) / K,
                     "err_flags": int(v["err"].item())}
            del g
        except RuntimeError as e:  # capture unsupported in this process: report why
            graph = {"unavailable": str(e).splitlines()[0][:200]}
        M = cfg.B * (2 * N - 1)
        logits = float(M) * cfg.V * 4
        byts = weight_bytes + kv_bytes + logits
        out["isd" if N > 1 else "ar"] = {
            "N": N, "queries_per_request": 2 * N - 1, "steps": K, "ms_per_step": ms,
            "steps_per_s": R.world / (ms / 1e3), "algorithmic_bytes": byts,
            "achieved_gbs": byts / (ms / 1e3) / 1e9, "err_flags": int(v["err"].item()),
            # this library's kernels per step: embed; per layer two RMSNorms, q/k
            # norm + rotation, K/V append, attention, SiLU; final norm; LM head and
            # its statistics merge; accept.  Plus four cuBLASLt GEMMs per layer.
            "gpu_launches": K * (1 + 6 * n_layers + 4), "library_gemm_launches": K * 4 * n_layers,
            "clocks": clk, "cuda_graph": graph}
        if hbm:
            out["isd" if N > 1 else "ar"]["frac_of_hbm"] = byts / (ms / 1e3) / 1e9 / hbm
    out["forward_time_ratio_isd_over_ar"] = times[cfg.N] / times[1]
    g_isd, g_ar = (out["isd"].get("cuda_graph") or {}), (out["ar"].get("cuda_graph") or {})
    if "ms_per_step" in g_isd and "ms_per_step" in g_ar:
        out["forward_time_ratio_isd_over_ar_graph"] = g_isd["ms_per_step"] / g_ar["ms_per_step"]
        if tpf is not None:
            out["speedup_over_ar_graph"] = tpf * g_ar["ms_per_step"] / g_isd["ms_per_step"]
    if tpf is not None:
        out["tpf_closed_loop"] = tpf
        out["speedup_over_ar"] = tpf * times[1] / times[cfg.N]
        out["isd_tokens_per_s"] = R.world * cfg.B * tpf / (times[cfg.N] / 1e3)
        out["ar_tokens_per_s"] = R.world * cfg.B / (times[1] / 1e3)
    del dw
    torch.cuda.empty_cache()
    return out


def gpu_bus_id():
    """PCI bus id of the current GPU, for the clock sampler (None if unknown)."""
    import torch
    try:
        pr = torch.cuda.get_device_properties(torch.cuda.current_device())
        return "%08X:%02X:00.0" % (int(getattr(pr, "pci_domain_id", 0)), int(pr.pci_bus_id))
    except Exception:
        return None


def config_dict(cfg, world):
    return {"workload": cfg.name, "B": cfg.B, "N": cfg.N, "Q": cfg.Q, "V": cfg.V,
            "hidden": cfg.H, "heads": f"{cfg.Hq}q/{cfg.Hkv}kv x {cfg.D}",
            "prefix": f"U[{cfg.prefix_lo},{cfg.prefix_hi}]", "page_size": cfg.page_size,
            "accept_rate": cfg.accept_rate, "lora_rank": cfg.lora_rank,
            "global_batch": cfg.B * world,
            "parallelism": f"dp{world} (independent batches)",
            "l2": "no flush; every step streams >1.8 GB (LM head 1.245 GB + KV cache) > 126 MB L2"}


def run_reference(args):
    """--impl reference: the CPU oracle on host cores (rank 0 only), on inputs
    generated on the host; no GPU work and no CUDA library."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from speculative_verification_isd_b200 import inputs as I
    cfg = I.CONFIGS[args.config]
    sampler = OracleSampler(cfg)
    total_budget = 150.0
    per_step = total_budget / max(1, args.steps + args.warmup)
    # vocabulary slice sized to the per-step budget (at least 256 entries)
    t0 = time.perf_counter()
    cfg_O = sampler.O
    cfg_O.lm_head(sampler.hidden, sampler.w_slice(0, 1024))
    t_1k = max(1e-4, time.perf_counter() - t0)
    vs = int(max(256, min(cfg.V, 1024 * max(0.05, per_step * 0.6) / t_1k)))
    for k in range(args.warmup):
        sampler.sample(k, vs)
    ests, spent = [], 0.0
    tstart = time.perf_counter()
    for k in range(args.steps):
        est, used = sampler.sample(k, vs)
        ests.append(est)
        spent += used
        if time.perf_counter() - tstart > total_budget:
            break
    est = statistics.median(ests)
    value = 1.0 / est
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "ISD steps/s",
            "n_gpus": world, "steps": len(ests), "warmup": args.warmup, "ms_per_step": est * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(cfg, world),
            "extrapolated": {
                "samples_timed": len(ests), "sample_seconds_total": round(spent, 3),
                "note": ("ms_per_step is the median full-step time extrapolated from each timed "
                         "sample; the samples themselves ran sample_seconds_total seconds, not "
                         "steps x ms_per_step")},
            "cpu_baseline": {"value": value, "unit": "ISD steps/s", "cores": sampler.threads,
                             "kind": "oracle",
                             "sample": (f"per step: 1 request's attention, LM head of all "
                                        f"{cfg.M} rows over a {vs}-entry vocabulary slice, 1 "
                                        f"request's acceptance on full-vocabulary rows; "
                                        f"extrapolated to the full step; inputs generated on "
                                        f"the host")},
            "e2e": {"value": value, "unit": "ISD steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    import numpy as np
    import torch
    from speculative_verification_isd_b200 import ranks as RK
    R = RK.setup(use_cuda=True)
    world, rank = R.world, R.rank
    from speculative_verification_isd_b200 import build as B
    if rank == 0:
        B.build()
    R.barrier()
    from speculative_verification_isd_b200 import inputs as I
    from speculative_verification_isd_b200 import isd
    from speculative_verification_isd_b200.workload import DeviceWorkload
    cfg = I.CONFIGS[args.config]
    hbm, tf_burst, tf_sus, peak_src = measured_peaks()
    if args.deep_only:
        out = deep_leg(isd, cfg, R, max(args.deep_steps, 1), gpu_bus_id(), RK.rank_seed(0, rank),
                       args.deep_layers, hbm=hbm)
        if rank == 0:
            print(json.dumps({"full_depth": out, "n_gpus": world}), flush=True)
        R.close()
        return 0
    if args.sdar_only:
        out = sdar_leg(isd, cfg, R, max(args.sdar_steps, 1), gpu_bus_id(), RK.rank_seed(0, rank),
                       hbm)
        if rank == 0:
            print(json.dumps({"sdar_comparison": out, "n_gpus": world}), flush=True)
        R.close()
        return 0
    # weak scaling: every rank runs its own batch of B requests (requests are
    # independent), so there is no collective on the data path
    if args.accept_rate is not None:
        cfg = dataclasses.replace(cfg, accept_rate=args.accept_rate)
    wl = DeviceWorkload(isd, cfg, seed=RK.rank_seed(0, rank), n_uniform_steps=max(64, args.warmup + 1))
    d = wl.dims
    K, W = args.steps, args.warmup
    stream = torch.cuda.current_stream()
    acc_hist = torch.zeros(K, cfg.B, dtype=torch.int32, device="cuda")

    def run_step(k, acc_out=None):
        wl.set_uniforms(k)
        if acc_out is not None:
            wl.accept_len = acc_out
        wl.step()

    for k in range(W):
        run_step(k)
    torch.cuda.synchronize()
    bus = gpu_bus_id()
    clocks = ClockSampler(bus)
    clocks.start()
    time.sleep(0.3)
    # ---------------- timed region: K steps through isd_step
    R.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for k in range(K):
        run_step(k, acc_hist[k])
    ev1.record(stream)
    torch.cuda.synchronize()
    R.barrier()
    clk = clocks.stop()
    t_ms = R.max(ev0.elapsed_time(ev1))
    wl.accept_len = torch.empty(cfg.B, dtype=torch.int32, device="cuda")
    accepted = R.sum(float(acc_hist.sum().item()))
    steps_total = K * world
    value = RK.job_throughput(K, R, t_ms)  # all ranks' steps over the slowest rank's time
    tok_s = accepted / (t_ms / 1e3)
    mean_acc = accepted / (steps_total * cfg.B)
    flags = int(wl.err.item())

    # ---------------- sustained: the same step back to back for >= 2.5 s, own clock record
    sustained = None
    if args.sustained_s > 0:
        n_sus = max(K, int(args.sustained_s * 1e3 / max(1e-3, t_ms / K)))
        clocks2 = ClockSampler(bus)
        clocks2.start()
        time.sleep(0.2)
        R.barrier()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for k in range(n_sus):
            run_step(k)
        s1.record(stream)
        torch.cuda.synchronize()
        R.barrier()
        clk_sus = clocks2.stop()
        sus_ms = R.max(s0.elapsed_time(s1))
        sustained = {"value": RK.job_throughput(n_sus, R, sus_ms), "unit": "ISD steps/s",
                     "steps": n_sus, "seconds": sus_ms / 1e3, "ms_per_step": sus_ms / n_sus,
                     "clocks": clk_sus}

    # ---------------- stage breakdown (same work, stage by stage, events between)
    KS = min(K, 300)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(KS)]
    for k in range(KS):
        wl.set_uniforms(k)
        e = evs[k]
        e[0].record(stream)
        isd.attention(d, wl.q, wl.k_new, wl.v_new, wl.k_pool, wl.v_pool, wl.page_table, wl.kv_len,
                      wl.n_clean, wl.hidden, wl.ws, wl.err)
        e[1].record(stream)
        # LM head with its fused row statistics (GEMM kernel + partial merge)
        isd.lm_head(d, wl.hidden, wl.W, wl.logits, wl.row_stats, wl.ws, wl.lora_A, wl.lora_B,
                    wl.err)
        e[2].record(stream)
        isd.accept(d, wl.logits, wl.row_stats, wl.prev_logits, wl.prev_row_stats, wl.n_clean,
                   wl.clean_tok, wl.kv_len, wl.uniforms, wl.accept_len, wl.out_tok,
                   wl.next_n_clean, wl.next_clean_tok, wl.next_kv_len, wl.ws, wl.ratio, wl.err)
        e[3].record(stream)
    torch.cuda.synchronize()
    stage = np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(3)]
                      for k in range(KS)])
    st_ms = stage.mean(axis=0)
    t_attn, t_lm, t_acc = [float(x) for x in st_ms]

    # ---------------- R-ISD gated LoRA: cost of the adapter.  The same steps with
    # the adapter on and off, in alternating rounds (so that clock changes hit
    # both alike); alpha = median of the rounds' time ratios
    lora_alpha = None
    if cfg.lora_rank:
        rounds, per = 10, max(10, min(K, 300) // 10)

        def timed(off):
            for k in range(3):
                wl.set_uniforms(k)
                wl.step(without_lora=off)
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for k in range(per):
                wl.set_uniforms(k)
                wl.step(without_lora=off)
            f1.record(stream)
            torch.cuda.synchronize()
            return R.max(f0.elapsed_time(f1)) / per

        ratios = []
        for rnd in range(rounds):
            if rnd % 2 == 0:
                t_on, t_off = timed(False), timed(True)
            else:
                t_off, t_on = timed(True), timed(False)
            ratios.append(t_on / t_off)
        lora_alpha = statistics.median(ratios)

    # ---------------- e2e: public API with host buffers, copies inside the timed region
    # A step's inputs travel in one pinned host buffer (one host-to-device
    # copy), its integer results come back in one (one device-to-host copy);
    # the caller waits for each step's result before issuing the next step.
    # Inputs are double-buffered, as a serving loop would keep them: while
    # step k runs, step k+1's inputs go up on a copy stream (every step's
    # copy is inside the timed region; the first is not overlapped).
    in_dev, out_dev, layout = wl.pack_io()
    in_devs = [in_dev, in_dev.clone()]
    host_ins = [torch.empty(in_dev.numel(), dtype=torch.uint8, pin_memory=True) for _ in range(2)]
    for h in host_ins:
        h.copy_(in_dev)
    u_off, u_nb = next((o, nb) for n, o, nb in layout if n == "uniforms")
    host_us = [h[u_off:u_off + u_nb].view(torch.float32) for h in host_ins]
    u_steps = wl.uniforms_all.cpu().reshape(wl.uniforms_all.shape[0], -1)
    host_out = torch.empty(out_dev.numel(), dtype=torch.int32, pin_memory=True)
    h2d = in_dev.numel()
    d2h = host_out.numel() * 4
    KE = min(args.e2e_steps, K)

    def step_call(buf):
        v = {n: buf[o:o + nb].view(getattr(wl, n).dtype).view(getattr(wl, n).shape)
             for n, o, nb in layout}
        return isd.StepCall(d, v["q"], v["k_new"], v["v_new"], wl.k_pool, wl.v_pool,
                            v["page_table"], v["kv_len"], v["n_clean"], v["clean_tok"], wl.W,
                            wl.prev_logits, wl.prev_row_stats, v["uniforms"], wl.logits,
                            wl.row_stats, wl.accept_len, wl.out_tok, wl.next_n_clean,
                            wl.next_clean_tok, wl.next_kv_len, wl.ws, hidden=wl.hidden,
                            ratio=wl.ratio, lora_A=wl.lora_A, lora_B=wl.lora_B,
                            err_flag=wl.err, stream=stream)

    calls = [step_call(b) for b in in_devs]
    copy_stream = torch.cuda.Stream()
    uploaded = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]
    for ev in consumed:
        ev.record(stream)

    def upload(k, slot):
        host_us[slot].copy_(u_steps[k % u_steps.shape[0]])  # step k's uniforms
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(consumed[slot])  # the step that last read this buffer is done
            in_devs[slot].copy_(host_ins[slot], non_blocking=True)
            uploaded[slot].record(copy_stream)

    def e2e_run(n):
        upload(0, 0)
        for k in range(n):
            s_ = k & 1
            stream.wait_event(uploaded[s_])
            calls[s_]()
            consumed[s_].record(stream)
            host_out.copy_(out_dev, non_blocking=True)
            if k + 1 < n:
                upload(k + 1, s_ ^ 1)
            stream.synchronize()  # the caller needs this step's result before the next one

    e2e_run(max(3, W))
    R.barrier()
    torch.cuda.synchronize()
    clocks_e2e = ClockSampler(bus)
    clocks_e2e.start()
    time.sleep(0.2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(KE)
    e1.record(stream)
    torch.cuda.synchronize()
    R.barrier()
    clk_e2e = clocks_e2e.stop()
    e2e_ms = R.max(e0.elapsed_time(e1))
    e2e_value = KE * world / (e2e_ms / 1e3)

    loop_line = None
    if args.loop_steps > 0:
        loop_line = closed_loop(isd, cfg, R, args.loop_steps, bus, RK.rank_seed(0, rank))
    sdar_line = None
    if args.sdar_steps > 0:
        sdar_line = sdar_leg(isd, cfg, R, args.sdar_steps, bus, RK.rank_seed(0, rank), hbm)
    deep_line = None
    if args.deep_steps > 0:
        deep_line = deep_leg(isd, cfg, R, args.deep_steps, bus, RK.rank_seed(0, rank),
                             args.deep_layers, loop_line["tpf"] if loop_line else None, hbm)

    # ---------------- roofline of the dominant kernel (LM head)
    lm_bytes = float(cfg.V) * cfg.H * 2 + float(cfg.M) * cfg.H * 2 + float(cfg.M) * cfg.V * 4
    lm_flops = 2.0 * cfg.M * cfg.H * cfg.V
    achieved = lm_bytes / (t_lm / 1e3) / 1e9
    kv_bytes = float(np.sum(wl.kv_len_h.astype(np.float64))) * cfg.Hkv * cfg.D * 4
    step_bytes = lm_bytes + kv_bytes + float(cfg.M) * (cfg.H + 2 * cfg.Hkv * cfg.D) * 2 \
        + float(cfg.M) * cfg.H * 2
    step_ms = t_ms / K
    line = {
        "metric": METRIC, "value": value, "unit": "ISD steps/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "accepted_tokens_per_s": tok_s, "mean_accept_len": mean_acc,
        "config": config_dict(cfg, world),
        "roofline": {"bound": "hbm", "kernel": "lm_head_kernel (+ row-stats merge)",
                     "achieved": achieved,
                     "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": profile_traffic("lm_head.cu"),
                     "bytes_per_launch": lm_bytes, "ms_per_launch": t_lm,
                     "tensor_tflops": lm_flops / (t_lm / 1e3) / 1e12,
                     "tensor_frac_of_sustained": lm_flops / (t_lm / 1e3) / 1e12 / tf_sus,
                     "peak_source": peak_src},
        "step_roofline": {"algorithmic_bytes": step_bytes,
                          "achieved_gbs": step_bytes / (step_ms / 1e3) / 1e9,
                          "frac": step_bytes / (step_ms / 1e3) / 1e9 / hbm,
                          "stage_ms": {"attention": t_attn, "lm_head_and_row_stats": t_lm,
                                       "accept": t_acc}},
        "e2e": {"value": e2e_value, "unit": "ISD steps/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": KE, "warmup": max(3, W),
                "inputs": "double-buffered: step k+1's copy runs on a copy stream during step k",
                "result_read_each_step": True, "clocks": clk_e2e},
        "sustained": sustained,
        # KV append, attention, LM head, accept (+ 3 LoRA kernels)
        "gpu_launches": K * (4 + (3 if cfg.lora_rank else 0)),
        "clocks": clk, "err_flags": flags,
    }
    if loop_line is not None:
        line["closed_loop"] = loop_line
    if sdar_line is not None:
        line["sdar_comparison"] = sdar_line
    if deep_line is not None:
        line["full_depth"] = deep_line
    if lora_alpha is not None:
        # step time with the adapter / without it (the pages report about 1.12)
        line["lora_alpha"] = lora_alpha
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        # the oracle's leg: its timed baseline, and the GPU's accept decisions
        # of one step of this workload checked against it
        line["parity"] = accept_parity(wl, cfg, 0)
        line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_budget_s)
    if rank == 0:
        print(json.dumps(line), flush=True)
    R.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
