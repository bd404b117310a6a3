"""Seeded synthetic inputs for the ISD verify-and-propose step.

This module only *generates* inputs: shapes, seeded value distributions, page
tables, prefix lengths, token ids and the caller-side uniforms.  It holds none
of the step's arithmetic (no attention, softmax, acceptance or sampling), so
both the CPU oracle and the CUDA path can be fed from it without sharing any
of the method.

Uniforms are the one random draw the method consumes.  They are produced here
with Philox4x32-10 (J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel random
numbers: as easy as 1, 2, 3", SC'11), written from that paper's definition:
key = (seed, 0), counter = (step, request, block, 0), and a 32-bit output x
maps to u = (x >> 8) * 2^-24 in [0, 1).

Workload shapes follow the I-DLM pages: Qwen3-8B-shaped attention (32 query
heads, 8 KV heads, head dim 128, hidden 4096, vocab 151936), stride N with a
2N-1 slot query block, paged bf16 KV cache, N(0, 0.02) bf16 weights.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

# --------------------------------------------------------------------------
# Philox4x32-10 (Salmon et al., SC'11, section 3.2 and Table 2 constants)
# --------------------------------------------------------------------------
_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = np.uint64(0x9E3779B9)
_PHILOX_W1 = np.uint64(0xBB67AE85)
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(counter: np.ndarray, key: np.ndarray) -> np.ndarray:
    """Philox4x32 with 10 rounds.

    counter: uint32 array [..., 4]; key: uint32 array [..., 2] (broadcastable).
    Returns uint32 [..., 4].
    """
    c = np.asarray(counter, dtype=np.uint64) & _MASK32
    k = np.asarray(key, dtype=np.uint64) & _MASK32
    c0, c1, c2, c3 = c[..., 0], c[..., 1], c[..., 2], c[..., 3]
    k0, k1 = np.broadcast_to(k[..., 0], c0.shape), np.broadcast_to(k[..., 1], c0.shape)
    for rnd in range(10):
        if rnd:
            k0 = (k0 + _PHILOX_W0) & _MASK32
            k1 = (k1 + _PHILOX_W1) & _MASK32
        p0 = _PHILOX_M0 * c0
        p1 = _PHILOX_M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def step_uniforms(seed: int, step: int, B: int, N: int) -> np.ndarray:
    """Uniforms [B, 2N] float32 for one ISD step.

    Per request: indices 0..N-2 are the acceptance draws for proposals 2..N,
    index N-1 is the residual draw, indices N..2N-1 are the proposal draws
    (used only in sample mode).
    """
    n_blocks = (2 * N + 3) // 4
    b = np.arange(B, dtype=np.uint64)[:, None]
    blk = np.arange(n_blocks, dtype=np.uint64)[None, :]
    ctr = np.stack(np.broadcast_arrays(np.uint64(step & 0xFFFFFFFF), b, blk, np.uint64(0)), axis=-1)
    key = np.array([seed & 0xFFFFFFFF, 0], dtype=np.uint64)
    x = philox4x32_10(ctr, key).reshape(B, n_blocks * 4)[:, : 2 * N]
    return ((x >> np.uint32(8)).astype(np.float64) * (2.0 ** -24)).astype(np.float32)


# --------------------------------------------------------------------------
# bf16 input encoding (inputs are drawn in fp32 and stored as bf16 bit
# patterns, uint16, round-to-nearest-even)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# Workload configurations
# --------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class IsdConfig:
    name: str
    B: int
    N: int
    Hq: int
    Hkv: int
    D: int
    V: int
    page_size: int
    prefix_lo: int
    prefix_hi: int
    lora_rank: int = 0
    fixed_prefix: Optional[tuple] = None   # explicit prefix lengths (overrides lo/hi)
    w_std: float = 0.02
    qkv_std: float = 0.02
    kv_std: float = 0.02
    lora_std: float = 0.01
    accept_rate: Optional[float] = None    # constructed p/q acceptance, if any
    spare_pages: int = 0                   # extra pool pages never referenced

    @property
    def Q(self) -> int:
        return 2 * self.N - 1

    @property
    def H(self) -> int:
        return self.Hq * self.D

    @property
    def M(self) -> int:
        return self.B * self.Q

    def max_pages_per_req(self) -> int:
        hi = max(self.fixed_prefix) if self.fixed_prefix else self.prefix_hi
        return (hi + self.Q + self.page_size - 1) // self.page_size


QWEN3_8B = dict(Hq=32, Hkv=8, D=128, V=151936)

CONFIGS: Dict[str, IsdConfig] = {
    # Tiny closed-loop parity case.
    "tiny": IsdConfig("tiny", B=2, N=2, Hq=4, Hkv=1, D=64, V=512, page_size=16,
                      prefix_lo=17, prefix_hi=40, fixed_prefix=(17, 40)),
    # Qwen3-8B-shaped, B=8, N=4, prefixes U[1024, 4096].
    "qwen3_8b_b8_n4": IsdConfig("qwen3_8b_b8_n4", B=8, N=4, page_size=16,
                                prefix_lo=1024, prefix_hi=4096, **QWEN3_8B),
    # Concurrency case: B=32, N=4, prefixes U[512, 8192], constructed acceptance 0.9.
    "qwen3_8b_b32_n4": IsdConfig("qwen3_8b_b32_n4", B=32, N=4, page_size=16,
                                 prefix_lo=512, prefix_hi=8192, accept_rate=0.9, **QWEN3_8B),
    # Wide stride: B=32, N=8, prefixes U[16384, 32768] in 64-token pages.
    "qwen3_8b_b32_n8": IsdConfig("qwen3_8b_b32_n8", B=32, N=8, page_size=64,
                                 prefix_lo=16384, prefix_hi=32768, accept_rate=0.8, **QWEN3_8B),
    # R-ISD gated LoRA: B=64, N=4, rank 128, prefixes U[512, 4096].
    "qwen3_8b_b64_n4_lora": IsdConfig("qwen3_8b_b64_n4_lora", B=64, N=4, page_size=16,
                                      prefix_lo=512, prefix_hi=4096, lora_rank=128, **QWEN3_8B),
    # Parity cases sized for the oracle: several tiles and ragged tails.
    "ragged_small": IsdConfig("ragged_small", B=3, N=4, Hq=8, Hkv=2, D=128, V=1000, page_size=16,
                              prefix_lo=1, prefix_hi=300, w_std=0.5, qkv_std=0.5, kv_std=1.0,
                              spare_pages=5),
    "ragged_lora": IsdConfig("ragged_lora", B=5, N=3, Hq=8, Hkv=2, D=128, V=2053, page_size=16,
                             prefix_lo=0, prefix_hi=700, lora_rank=128, w_std=0.2, qkv_std=0.5,
                             kv_std=1.0, lora_std=0.05),
    # Stride 8 (60 query rows per kv head) in 64-token pages, ragged prefixes.
    "ragged_n8": IsdConfig("ragged_n8", B=3, N=8, Hq=8, Hkv=2, D=128, V=1000, page_size=64,
                           prefix_lo=1, prefix_hi=400, w_std=0.5, qkv_std=0.5, kv_std=1.0),
    "qwen_medium": IsdConfig("qwen_medium", B=4, N=4, page_size=16, prefix_lo=100, prefix_hi=2500,
                             w_std=0.05, qkv_std=0.3, kv_std=1.0, **QWEN3_8B),
}


def prefix_lengths(cfg: IsdConfig, seed: int) -> np.ndarray:
    if cfg.fixed_prefix is not None:
        return np.asarray(cfg.fixed_prefix, dtype=np.int32)
    rng = np.random.default_rng([seed, 11])
    return rng.integers(cfg.prefix_lo, cfg.prefix_hi + 1, size=cfg.B).astype(np.int32)


def page_layout(cfg: IsdConfig, kv_len: np.ndarray, seed: int):
    """Page table [B, max_pages] int32 (unused entries -1) and pool size.

    Each request gets ceil((kv_len + Q) / P) pages; page ids are a seeded
    permutation of the pool, so consecutive positions live in scattered pages.
    """
    P = cfg.page_size
    need = (kv_len.astype(np.int64) + cfg.Q + P - 1) // P
    num_pages = int(need.sum()) + cfg.spare_pages
    rng = np.random.default_rng([seed, 13])
    perm = rng.permutation(num_pages).astype(np.int32)
    mp = cfg.max_pages_per_req()
    table = np.full((cfg.B, mp), -1, dtype=np.int32)
    off = 0
    for b in range(cfg.B):
        table[b, : need[b]] = perm[off: off + need[b]]
        off += need[b]
    return table, num_pages


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return f32_to_bf16_bits((rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)))


def make_step_inputs(cfg: IsdConfig, seed: int = 0, n_clean: str | np.ndarray = "full",
                     step: int = 0) -> Dict[str, np.ndarray]:
    """Host (numpy) inputs of one ISD step for configs small enough for the host.

    bf16 tensors are returned as uint16 bit patterns.  Layouts:
      q [B,Q,Hq,D]; k_new, v_new [B,Q,Hkv,D]; k_pool, v_pool [pages,P,Hkv,D];
      page_table [B,max_pages]; kv_len, n_clean [B]; clean_tok [B,N];
      W [V,H]; lora_A [H,r]; lora_B [r,H]; uniforms [B,2N] float32.
    """
    rng = np.random.default_rng([seed, 17])
    B, N, Q = cfg.B, cfg.N, cfg.Q
    kv_len = prefix_lengths(cfg, seed)
    table, num_pages = page_layout(cfg, kv_len, seed)
    if isinstance(n_clean, str):
        if n_clean == "full":
            nc = np.full(B, N, dtype=np.int32)
        elif n_clean == "one":
            nc = np.ones(B, dtype=np.int32)
        elif n_clean == "mixed":
            nc = rng.integers(1, N + 1, size=B).astype(np.int32)
        else:
            raise ValueError(n_clean)
    else:
        nc = np.asarray(n_clean, dtype=np.int32)
    out = dict(
        q=_normal_bf16(rng, (B, Q, cfg.Hq, cfg.D), cfg.qkv_std),
        k_new=_normal_bf16(rng, (B, Q, cfg.Hkv, cfg.D), cfg.qkv_std),
        v_new=_normal_bf16(rng, (B, Q, cfg.Hkv, cfg.D), cfg.qkv_std),
        k_pool=_normal_bf16(rng, (num_pages, cfg.page_size, cfg.Hkv, cfg.D), cfg.kv_std),
        v_pool=_normal_bf16(rng, (num_pages, cfg.page_size, cfg.Hkv, cfg.D), cfg.kv_std),
        page_table=table,
        kv_len=kv_len,
        n_clean=nc,
        clean_tok=rng.integers(0, cfg.V, size=(B, N)).astype(np.int32),
        W=_normal_bf16(rng, (cfg.V, cfg.H), cfg.w_std),
        uniforms=step_uniforms(seed, step, B, N),
    )
    if cfg.lora_rank:
        out["lora_A"] = _normal_bf16(rng, (cfg.H, cfg.lora_rank), cfg.lora_std)
        out["lora_B"] = _normal_bf16(rng, (cfg.lora_rank, cfg.H), cfg.lora_std)
    return out


def random_logits(B: int, Q: int, V: int, seed: int, scale: float = 3.0) -> np.ndarray:
    """fp32 logits [B,Q,V] with a spread wide enough for non-trivial softmaxes."""
    rng = np.random.default_rng([seed, 19])
    return (rng.standard_normal((B, Q, V), dtype=np.float32) * np.float32(scale)).astype(np.float32)


# --------------------------------------------------------------------------
# Synthetic single-layer "model" for closed-loop runs: per-token q/k/v
# embedding tables plus one MASK embedding.  The block's activations are a
# table lookup, so a whole decode loop runs without any trained weights.
# --------------------------------------------------------------------------
def make_embedding_tables(cfg: IsdConfig, seed: int = 0) -> Dict[str, np.ndarray]:
    rng = np.random.default_rng([seed, 23])
    V1 = cfg.V + 1  # row V is the MASK embedding
    return dict(
        Eq=_normal_bf16(rng, (V1, cfg.Hq, cfg.D), cfg.qkv_std),
        Ek=_normal_bf16(rng, (V1, cfg.Hkv, cfg.D), cfg.qkv_std),
        Ev=_normal_bf16(rng, (V1, cfg.Hkv, cfg.D), cfg.qkv_std),
    )


def embed_block(tables: Dict[str, np.ndarray], clean_tok: np.ndarray, n_clean: np.ndarray,
                N: int, V: int):
    """q, k_new, v_new for a block: clean slots look up their token, MASK slots
    (N..2N-2) and inactive clean slots look up the MASK row V."""
    B = clean_tok.shape[0]
    Q = 2 * N - 1
    ids = np.full((B, Q), V, dtype=np.int64)
    for b in range(B):
        c = int(n_clean[b])
        ids[b, :c] = clean_tok[b, :c]
    return tables["Eq"][ids], tables["Ek"][ids], tables["Ev"][ids]


def rope_table(n_pos: int, D: int, base: float = 1.0e6) -> np.ndarray:
    """Rotary-embedding table [n_pos, D/2, 2] float32: (cos, sin) of
    pos * base^(-2i/D) for pair i, taken in float64 and rounded once.

    Qwen3 rotates q and k by position with base 1e6; the table model of the
    SDAR-style closed loop does the same, so the N rows of a block, which
    carry the same MASK embedding, differ by position as a real model's do."""
    i = np.arange(D // 2, dtype=np.float64)
    inv = base ** (-2.0 * i / D)
    ang = np.arange(n_pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)


def workload_bytes(cfg: IsdConfig, kv_len: np.ndarray) -> Dict[str, float]:
    """Algorithmic HBM bytes of one step (used for roofline figures)."""
    kv = float(np.sum(kv_len.astype(np.float64))) * cfg.Hkv * cfg.D * 2 * 2
    w = float(cfg.V) * cfg.H * 2
    logits = float(cfg.M) * cfg.V * 4
    act = float(cfg.M) * (cfg.H + 2 * cfg.Hkv * cfg.D) * 2 + float(cfg.M) * cfg.H * 2
    return dict(kv=kv, w=w, logits=logits, act=act, total=kv + w + logits + act)


def lm_head_flops(cfg: IsdConfig) -> float:
    return 2.0 * cfg.M * cfg.H * cfg.V


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [
    "philox4x32_10", "step_uniforms", "f32_to_bf16_bits", "bf16_bits_to_f32", "IsdConfig",
    "CONFIGS", "prefix_lengths", "page_layout", "make_step_inputs", "random_logits",
    "make_embedding_tables", "embed_block", "rope_table", "workload_bytes", "lm_head_flops",
    "ceil_div",
]
