"""Python binding of libisd.so (include/isd.h): argument marshalling only.

Every function takes torch CUDA tensors, checks dtype / shape / contiguity,
and passes raw device pointers plus the current CUDA stream to the C ABI.
All arithmetic of the ISD step runs in the library's kernels; there is no
fallback.  Importing this module raises ImportError when libisd.so has not
been built (``python -m speculative_verification_isd_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libisd.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libisd.so not found at {LIB_PATH}: build it with "
                      "`python -m speculative_verification_isd_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

ISD_OK = 0
ISD_ERR_INVALID_ARG = -1
ISD_ERR_UNSUPPORTED_SHAPE = -2
ISD_ERR_WORKSPACE = -3
ISD_ERR_CUDA = -4
FLAG_PAGE_OOB = 1
FLAG_TOKEN_OOB = 2
FLAG_NCLEAN_RANGE = 4
FLAG_CAPACITY = 8
FLAG_WAIT_TIMEOUT = 16
PROPOSE_ARGMAX = 0
PROPOSE_SAMPLE = 1

EXPORTED = ("isd_workspace_bytes", "isd_status_string", "isd_last_error", "isd_attention",
            "isd_lm_head", "isd_row_stats", "isd_accept", "isd_step", "isd_prepare_block",
            "isd_loop", "isd_attention_noalloc", "isd_sdar_step", "isd_sdar_unmask",
            "isd_sdar_loop", "isd_layers_workspace_bytes", "isd_layers", "isd_embed_block")
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # ISD_NOALLOC_SCRATCH_BYTES in include/isd.h


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("N", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32), ("V", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("max_pages_per_req", ctypes.c_int32), ("lora_rank", ctypes.c_int32),
                ("proposal_mode", ctypes.c_int32), ("sm_scale", ctypes.c_float)]

    @property
    def Q(self):
        return 2 * self.N - 1

    @property
    def H(self):
        return self.Hq * self.D

    @property
    def M(self):
        return self.B * self.Q


ROW_STAT_FIELDS = 4  # isd_row_stat = {float max, float sumexp, int32 argmax, int32 reserved}

LOOP_FIELDS = ("Eq", "Ek", "Ev", "W", "lora_A", "lora_B", "k_pool", "v_pool", "page_table",
               "pages_used", "next_free_page", "kv_len", "n_clean", "clean_tok", "logits",
               "row_stats", "uniforms", "q", "k_new", "v_new", "hidden", "accept_len_hist",
               "out_tok_hist")


class LoopArgs(ctypes.Structure):
    """isd_loop_args (include/isd.h): device pointers, in declaration order."""
    _fields_ = [(n, ctypes.c_void_p) for n in LOOP_FIELDS]


SDAR_LOOP_FIELDS = ("Eq", "Ek", "Ev", "W", "k_pool", "v_pool", "page_table", "pages_used",
                    "next_free_page", "kv_len", "block_tok", "steps", "logits", "row_stats", "q",
                    "k_new", "v_new", "hidden", "unmasked_hist", "out_tok_hist",
                    "block_steps_hist")


class SdarLoopArgs(ctypes.Structure):
    """isd_sdar_loop_args (include/isd.h): device pointers, then the optional
    rotary table and its length, in declaration order."""
    _fields_ = [(n, ctypes.c_void_p) for n in SDAR_LOOP_FIELDS] + [
        ("rope", ctypes.c_void_p), ("rope_positions", ctypes.c_int32)]

_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_i32 = ctypes.c_int32
_dims_p = ctypes.POINTER(Dims)

_lib.isd_workspace_bytes.argtypes = [_dims_p]
_lib.isd_workspace_bytes.restype = _sz
_lib.isd_status_string.argtypes = [_i32]
_lib.isd_status_string.restype = ctypes.c_char_p
_lib.isd_last_error.argtypes = []
_lib.isd_last_error.restype = ctypes.c_char_p
_lib.isd_attention.argtypes = [_dims_p] + [_vp] * 10 + [_sz, _vp, _vp]
_lib.isd_attention.restype = _i32
_lib.isd_lm_head.argtypes = [_dims_p] + [_vp] * 7 + [_sz, _vp, _vp]
_lib.isd_lm_head.restype = _i32
_lib.isd_row_stats.argtypes = [_dims_p, _vp, _i32, _vp, _vp, _sz, _vp]
_lib.isd_row_stats.restype = _i32
_lib.isd_accept.argtypes = [_dims_p] + [_vp] * 15 + [_sz, _vp, _vp]
_lib.isd_accept.restype = _i32
_lib.isd_step.argtypes = [_dims_p] + [_vp] * 25 + [_sz, _vp, _vp]
_lib.isd_step.restype = _i32
_lib.isd_prepare_block.argtypes = [_dims_p] + [_vp] * 14
_lib.isd_prepare_block.restype = _i32
_lib.isd_loop.argtypes = [_dims_p, _i32, ctypes.POINTER(LoopArgs), _vp, _sz, _vp, _vp]
_lib.isd_loop.restype = _i32
_lib.isd_attention_noalloc.argtypes = [_dims_p] + [_vp] * 9 + [_vp, _vp]
_lib.isd_attention_noalloc.restype = _i32
_f32 = ctypes.c_float
_lib.isd_sdar_step.argtypes = [_dims_p, _f32, _i32] + [_vp] * 17 + [_sz, _vp, _vp]
_lib.isd_sdar_step.restype = _i32
_lib.isd_sdar_unmask.argtypes = [_dims_p, _f32, _i32] + [_vp] * 8 + [_sz, _vp, _vp]
_lib.isd_sdar_unmask.restype = _i32
_lib.isd_sdar_loop.argtypes = [_dims_p, _f32, _i32, _i32, ctypes.POINTER(SdarLoopArgs), _vp, _sz,
                               _vp, _vp]
_lib.isd_sdar_loop.restype = _i32


LAYER_FIELDS = ("in_norm", "w_qkv", "q_norm", "k_norm", "w_o", "post_norm", "w_gate_up",
                "w_down", "k_pool", "v_pool")


class Layer(ctypes.Structure):
    """isd_layer (include/isd.h): one decoder layer's device pointers."""
    _fields_ = [(n, ctypes.c_void_p) for n in LAYER_FIELDS]


_lib.isd_layers_workspace_bytes.argtypes = [_dims_p, _i32]
_lib.isd_layers_workspace_bytes.restype = _sz
_lib.isd_layers.argtypes = [_dims_p, _i32, _i32, _f32, ctypes.POINTER(Layer), _vp, _i32] + \
    [_vp] * 6 + [_vp, _sz, _vp, _vp]
_lib.isd_layers.restype = _i32
_lib.isd_embed_block.argtypes = [_dims_p] + [_vp] * 6
_lib.isd_embed_block.restype = _i32


class IsdError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        name = _lib.isd_status_string(status).decode()
        detail = _lib.isd_last_error().decode()
        super().__init__(f"{name}: {detail}")


def library() -> ctypes.CDLL:
    return _lib


def make_dims(B, N, Hq, Hkv, D, V, page_size, num_pages, max_pages_per_req, lora_rank=0,
              proposal_mode=PROPOSE_ARGMAX, sm_scale=None) -> Dims:
    if sm_scale is None:
        sm_scale = D ** -0.5
    return Dims(B, N, Hq, Hkv, D, V, page_size, num_pages, max_pages_per_req, lora_rank,
                proposal_mode, float(sm_scale))


def workspace_bytes(d: Dims) -> int:
    return int(_lib.isd_workspace_bytes(ctypes.byref(d)))


def alloc_workspace(d: Dims, device="cuda") -> torch.Tensor:
    n = workspace_bytes(d)
    if n == 0:
        raise IsdError(ISD_ERR_INVALID_ARG)
    return torch.empty(n, dtype=torch.uint8, device=device)


def _ptr(t: Optional[torch.Tensor], dtype=None, numel=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    return t.data_ptr()


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int):
    if status != ISD_OK:
        raise IsdError(status)


def attention(d: Dims, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean, out, ws,
              err_flag=None, stream=None):
    kvrow = d.page_size * d.Hkv * d.D
    _check(_lib.isd_attention(
        ctypes.byref(d), _ptr(q, _BF16, d.M * d.Hq * d.D, "q"),
        _ptr(k_new, _BF16, d.M * d.Hkv * d.D, "k_new"),
        _ptr(v_new, _BF16, d.M * d.Hkv * d.D, "v_new"),
        _ptr(k_pool, _BF16, d.num_pages * kvrow, "k_pool"),
        _ptr(v_pool, _BF16, d.num_pages * kvrow, "v_pool"),
        _ptr(page_table, torch.int32, d.B * d.max_pages_per_req, "page_table"),
        _ptr(kv_len, torch.int32, d.B, "kv_len"), _ptr(n_clean, torch.int32, d.B, "n_clean"),
        _ptr(out, _BF16, d.M * d.H, "out"), _ptr(ws, torch.uint8, None, "ws"), ws.numel(),
        _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)))


def attention_noalloc(d: Dims, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean, out,
                      err_flag=None, stream=None):
    """isd_attention without a workspace argument, for callers that cannot
    allocate device memory (scratch comes from a fixed array in the library)."""
    kvrow = d.page_size * d.Hkv * d.D
    _check(_lib.isd_attention_noalloc(
        ctypes.byref(d), _ptr(q, _BF16, d.M * d.Hq * d.D, "q"),
        _ptr(k_new, _BF16, d.M * d.Hkv * d.D, "k_new"),
        _ptr(v_new, _BF16, d.M * d.Hkv * d.D, "v_new"),
        _ptr(k_pool, _BF16, d.num_pages * kvrow, "k_pool"),
        _ptr(v_pool, _BF16, d.num_pages * kvrow, "v_pool"),
        _ptr(page_table, torch.int32, d.B * d.max_pages_per_req, "page_table"),
        _ptr(kv_len, torch.int32, d.B, "kv_len"), _ptr(n_clean, torch.int32, d.B, "n_clean"),
        _ptr(out, _BF16, d.M * d.H, "out"), _ptr(err_flag, torch.int32, 1, "err_flag"),
        _stream(stream)))


def lm_head(d: Dims, hidden, W, logits, row_stats, ws, lora_A=None, lora_B=None, err_flag=None,
            stream=None):
    _check(_lib.isd_lm_head(
        ctypes.byref(d), _ptr(hidden, _BF16, d.M * d.H, "hidden"),
        _ptr(W, _BF16, d.V * d.H, "W"),
        _ptr(lora_A, _BF16, d.H * d.lora_rank, "lora_A"),
        _ptr(lora_B, _BF16, d.lora_rank * d.H, "lora_B"),
        _ptr(logits, torch.float32, d.M * d.V, "logits"),
        _ptr(row_stats, (torch.int32, torch.float32), d.M * ROW_STAT_FIELDS, "row_stats"),
        _ptr(ws, torch.uint8, None, "ws"), ws.numel(),
        _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)))


def row_stats(d: Dims, logits, rows: int, out, ws, stream=None):
    _check(_lib.isd_row_stats(
        ctypes.byref(d), _ptr(logits, torch.float32, None, "logits"), int(rows),
        _ptr(out, (torch.int32, torch.float32), None, "row_stats"),
        _ptr(ws, torch.uint8, None, "ws"), ws.numel(), _stream(stream)))


def accept(d: Dims, logits, row_stats, prev_logits, prev_row_stats, n_clean, clean_tok, kv_len,
           uniforms, accept_len, out_tok, next_n_clean, next_clean_tok, next_kv_len, ws,
           ratio=None, err_flag=None, stream=None):
    B, N = d.B, d.N
    _check(_lib.isd_accept(
        ctypes.byref(d), _ptr(logits, torch.float32, d.M * d.V, "logits"),
        _ptr(row_stats, (torch.int32, torch.float32), d.M * ROW_STAT_FIELDS, "row_stats"),
        _ptr(prev_logits, torch.float32, d.M * d.V, "prev_logits"),
        _ptr(prev_row_stats, (torch.int32, torch.float32), d.M * ROW_STAT_FIELDS, "prev_row_stats"),
        _ptr(n_clean, torch.int32, B, "n_clean"), _ptr(clean_tok, torch.int32, B * N, "clean_tok"),
        _ptr(kv_len, torch.int32, B, "kv_len"), _ptr(uniforms, torch.float32, B * 2 * N, "uniforms"),
        _ptr(accept_len, torch.int32, B, "accept_len"), _ptr(out_tok, torch.int32, B * N, "out_tok"),
        _ptr(next_n_clean, torch.int32, B, "next_n_clean"),
        _ptr(next_clean_tok, torch.int32, B * N, "next_clean_tok"),
        _ptr(next_kv_len, torch.int32, B, "next_kv_len"),
        _ptr(ratio, torch.float32, B * max(N - 1, 1), "ratio"),
        _ptr(ws, torch.uint8, None, "ws"), ws.numel(),
        _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)))


def _step_args(d: Dims, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean, clean_tok,
               W, prev_logits, prev_row_stats, uniforms, logits, row_stats, accept_len, out_tok,
               next_n_clean, next_clean_tok, next_kv_len, ws, hidden=None, ratio=None,
               lora_A=None, lora_B=None, err_flag=None, stream=None):
    B, N = d.B, d.N
    kvrow = d.page_size * d.Hkv * d.D
    return [
        ctypes.byref(d), _ptr(q, _BF16, d.M * d.Hq * d.D, "q"),
        _ptr(k_new, _BF16, d.M * d.Hkv * d.D, "k_new"),
        _ptr(v_new, _BF16, d.M * d.Hkv * d.D, "v_new"),
        _ptr(k_pool, _BF16, d.num_pages * kvrow, "k_pool"),
        _ptr(v_pool, _BF16, d.num_pages * kvrow, "v_pool"),
        _ptr(page_table, torch.int32, d.B * d.max_pages_per_req, "page_table"),
        _ptr(kv_len, torch.int32, B, "kv_len"), _ptr(n_clean, torch.int32, B, "n_clean"),
        _ptr(clean_tok, torch.int32, B * N, "clean_tok"), _ptr(W, _BF16, d.V * d.H, "W"),
        _ptr(lora_A, _BF16, d.H * d.lora_rank, "lora_A"),
        _ptr(lora_B, _BF16, d.lora_rank * d.H, "lora_B"),
        _ptr(prev_logits, torch.float32, d.M * d.V, "prev_logits"),
        _ptr(prev_row_stats, (torch.int32, torch.float32), d.M * ROW_STAT_FIELDS, "prev_row_stats"),
        _ptr(uniforms, torch.float32, B * 2 * N, "uniforms"),
        _ptr(hidden, _BF16, d.M * d.H, "hidden"),
        _ptr(logits, torch.float32, d.M * d.V, "logits"),
        _ptr(row_stats, (torch.int32, torch.float32), d.M * ROW_STAT_FIELDS, "row_stats"),
        _ptr(accept_len, torch.int32, B, "accept_len"), _ptr(out_tok, torch.int32, B * N, "out_tok"),
        _ptr(next_n_clean, torch.int32, B, "next_n_clean"),
        _ptr(next_clean_tok, torch.int32, B * N, "next_clean_tok"),
        _ptr(next_kv_len, torch.int32, B, "next_kv_len"),
        _ptr(ratio, torch.float32, B * max(N - 1, 1), "ratio"),
        _ptr(ws, torch.uint8, None, "ws"), ws.numel(),
        _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)]


def step(d: Dims, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean, clean_tok, W,
         prev_logits, prev_row_stats, uniforms, logits, row_stats, accept_len, out_tok,
         next_n_clean, next_clean_tok, next_kv_len, ws, hidden=None, ratio=None, lora_A=None,
         lora_B=None, err_flag=None, stream=None):
    _check(_lib.isd_step(*_step_args(
        d, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean, clean_tok, W,
        prev_logits, prev_row_stats, uniforms, logits, row_stats, accept_len, out_tok,
        next_n_clean, next_clean_tok, next_kv_len, ws, hidden, ratio, lora_A, lora_B, err_flag,
        stream)))


class StepCall:
    """isd_step with its arguments checked and marshalled once.

    For a loop that issues the same step on the same buffers many times (a
    serving loop whose tensors stay in place): the constructor takes the
    arguments of ``step`` (stream included) and validates them; calling the
    object only passes the cached pointers to the library.  The tensors must
    stay alive and in place while the object is used."""

    def __init__(self, d: Dims, *args, **kwargs):
        self._dims = d  # keeps the struct alive: the cached arguments point at it
        self._keep = (args, kwargs)
        self._args = tuple(_step_args(d, *args, **kwargs))
        self._fn = _lib.isd_step

    def __call__(self):
        st = self._fn(*self._args)
        if st != ISD_OK:
            raise IsdError(st)


def prepare_block(d: Dims, Eq, Ek, Ev, n_clean, clean_tok, kv_len, page_table, pages_used,
                  next_free_page, q, k_new, v_new, err_flag=None, stream=None):
    """isd_prepare_block: block activations by table lookup + page bookkeeping."""
    B, N = d.B, d.N
    _check(_lib.isd_prepare_block(
        ctypes.byref(d), _ptr(Eq, _BF16, (d.V + 1) * d.Hq * d.D, "Eq"),
        _ptr(Ek, _BF16, (d.V + 1) * d.Hkv * d.D, "Ek"), _ptr(Ev, _BF16, (d.V + 1) * d.Hkv * d.D, "Ev"),
        _ptr(n_clean, torch.int32, B, "n_clean"), _ptr(clean_tok, torch.int32, B * N, "clean_tok"),
        _ptr(kv_len, torch.int32, B, "kv_len"),
        _ptr(page_table, torch.int32, B * d.max_pages_per_req, "page_table"),
        _ptr(pages_used, torch.int32, B, "pages_used"),
        _ptr(next_free_page, torch.int32, 1, "next_free_page"),
        _ptr(q, _BF16, d.M * d.Hq * d.D, "q"), _ptr(k_new, _BF16, d.M * d.Hkv * d.D, "k_new"),
        _ptr(v_new, _BF16, d.M * d.Hkv * d.D, "v_new"), _ptr(err_flag, torch.int32, 1, "err_flag"),
        _stream(stream)))


def loop_args(d: Dims, n_steps: int, **t) -> LoopArgs:
    """Checked isd_loop_args from tensors named as its fields (lora_A / lora_B
    may be omitted when lora_rank is 0)."""
    B, N, M = d.B, d.N, d.M
    kvrow = d.page_size * d.Hkv * d.D
    want = dict(
        Eq=(_BF16, (d.V + 1) * d.Hq * d.D), Ek=(_BF16, (d.V + 1) * d.Hkv * d.D),
        Ev=(_BF16, (d.V + 1) * d.Hkv * d.D), W=(_BF16, d.V * d.H),
        lora_A=(_BF16, d.H * d.lora_rank), lora_B=(_BF16, d.lora_rank * d.H),
        k_pool=(_BF16, d.num_pages * kvrow), v_pool=(_BF16, d.num_pages * kvrow),
        page_table=(torch.int32, B * d.max_pages_per_req), pages_used=(torch.int32, B),
        next_free_page=(torch.int32, 1), kv_len=(torch.int32, 2 * B), n_clean=(torch.int32, 2 * B),
        clean_tok=(torch.int32, 2 * B * N), logits=(torch.float32, 2 * M * d.V),
        row_stats=((torch.int32, torch.float32), 2 * M * ROW_STAT_FIELDS),
        uniforms=(torch.float32, n_steps * B * 2 * N), q=(_BF16, M * d.Hq * d.D),
        k_new=(_BF16, M * d.Hkv * d.D), v_new=(_BF16, M * d.Hkv * d.D), hidden=(_BF16, M * d.H),
        accept_len_hist=(torch.int32, n_steps * B), out_tok_hist=(torch.int32, n_steps * B * N))
    vals = {}
    for n in LOOP_FIELDS:
        dt, numel = want[n]
        vals[n] = _ptr(t.get(n), dt, numel, n)
    return LoopArgs(**vals)


def loop(d: Dims, n_steps: int, ws, err_flag=None, stream=None, args: Optional[LoopArgs] = None,
         **tensors):
    """isd_loop: n_steps ISD steps of a stationary batch on the device."""
    a = args if args is not None else loop_args(d, n_steps, **tensors)
    _check(_lib.isd_loop(ctypes.byref(d), int(n_steps), ctypes.byref(a),
                         _ptr(ws, torch.uint8, None, "ws"), ws.numel(),
                         _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)))


def row_stats_view(rs: torch.Tensor):
    """(max, sumexp, argmax) views of an isd_row_stat buffer stored as int32 [M, 4]."""
    r = rs.view(-1, ROW_STAT_FIELDS)
    f = r.view(torch.float32) if r.dtype == torch.int32 else r
    i = r if r.dtype == torch.int32 else r.view(torch.int32)
    return f[:, 0], f[:, 1], i[:, 2]


# ---------------------------------------------------------------------------
# SDAR-style confidence-threshold block decoding (blocks of N rows, Q = N)
# ---------------------------------------------------------------------------
def sdar_step(d: Dims, tau: float, sync: bool, q, k_new, v_new, k_pool, v_pool, page_table,
              kv_len, W, logits, block_tok, steps, unmasked, out_tok, block_steps, ws,
              hidden=None, row_stats=None, err_flag=None, stream=None):
    """isd_sdar_step: block-causal attention over the block's N rows, LM head,
    confidence-threshold unmask (state block_tok / steps / kv_len in place)."""
    B, N = d.B, d.N
    M = B * N
    kvrow = d.page_size * d.Hkv * d.D
    _check(_lib.isd_sdar_step(
        ctypes.byref(d), float(tau), int(bool(sync)), _ptr(q, _BF16, M * d.Hq * d.D, "q"),
        _ptr(k_new, _BF16, M * d.Hkv * d.D, "k_new"), _ptr(v_new, _BF16, M * d.Hkv * d.D, "v_new"),
        _ptr(k_pool, _BF16, d.num_pages * kvrow, "k_pool"),
        _ptr(v_pool, _BF16, d.num_pages * kvrow, "v_pool"),
        _ptr(page_table, torch.int32, B * d.max_pages_per_req, "page_table"),
        _ptr(kv_len, torch.int32, B, "kv_len"), _ptr(W, _BF16, d.V * d.H, "W"),
        _ptr(hidden, _BF16, M * d.H, "hidden"), _ptr(logits, torch.float32, M * d.V, "logits"),
        _ptr(row_stats, (torch.int32, torch.float32), M * ROW_STAT_FIELDS, "row_stats"),
        _ptr(block_tok, torch.int32, B * N, "block_tok"), _ptr(steps, torch.int32, B, "steps"),
        _ptr(unmasked, torch.int32, B, "unmasked"), _ptr(out_tok, torch.int32, B * N, "out_tok"),
        _ptr(block_steps, torch.int32, B, "block_steps"),
        _ptr(ws, torch.uint8, None, "ws"), ws.numel(),
        _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)))


def sdar_unmask(d: Dims, tau: float, sync: bool, row_stats, block_tok, steps, kv_len, unmasked,
                out_tok, block_steps, ws, err_flag=None, stream=None):
    """isd_sdar_unmask: the decision alone on given row statistics [B*N]."""
    B, N = d.B, d.N
    _check(_lib.isd_sdar_unmask(
        ctypes.byref(d), float(tau), int(bool(sync)),
        _ptr(row_stats, (torch.int32, torch.float32), B * N * ROW_STAT_FIELDS, "row_stats"),
        _ptr(block_tok, torch.int32, B * N, "block_tok"), _ptr(steps, torch.int32, B, "steps"),
        _ptr(kv_len, torch.int32, B, "kv_len"), _ptr(unmasked, torch.int32, B, "unmasked"),
        _ptr(out_tok, torch.int32, B * N, "out_tok"),
        _ptr(block_steps, torch.int32, B, "block_steps"),
        _ptr(ws, torch.uint8, None, "ws"), ws.numel(),
        _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)))


def sdar_loop_args(d: Dims, n_steps: int, rope=None, **t) -> SdarLoopArgs:
    """Checked isd_sdar_loop_args from tensors named as its fields; rope:
    optional float32 [positions, D/2, 2] rotary table."""
    B, N = d.B, d.N
    M = B * N
    kvrow = d.page_size * d.Hkv * d.D
    want = dict(
        Eq=(_BF16, (d.V + 1) * d.Hq * d.D), Ek=(_BF16, (d.V + 1) * d.Hkv * d.D),
        Ev=(_BF16, (d.V + 1) * d.Hkv * d.D), W=(_BF16, d.V * d.H),
        k_pool=(_BF16, d.num_pages * kvrow), v_pool=(_BF16, d.num_pages * kvrow),
        page_table=(torch.int32, B * d.max_pages_per_req), pages_used=(torch.int32, B),
        next_free_page=(torch.int32, 1), kv_len=(torch.int32, B), block_tok=(torch.int32, B * N),
        steps=(torch.int32, B), logits=(torch.float32, M * d.V),
        row_stats=((torch.int32, torch.float32), M * ROW_STAT_FIELDS),
        q=(_BF16, M * d.Hq * d.D), k_new=(_BF16, M * d.Hkv * d.D), v_new=(_BF16, M * d.Hkv * d.D),
        hidden=(_BF16, M * d.H), unmasked_hist=(torch.int32, n_steps * B),
        out_tok_hist=(torch.int32, n_steps * B * N), block_steps_hist=(torch.int32, n_steps * B))
    vals = {}
    for n in SDAR_LOOP_FIELDS:
        dt, numel = want[n]
        vals[n] = _ptr(t.get(n), dt, numel, n)
    if rope is not None:
        if rope.dim() != 3 or rope.shape[1:] != (d.D // 2, 2):
            raise ValueError(f"rope must be [positions, {d.D // 2}, 2]")
        vals["rope"] = _ptr(rope, torch.float32, None, "rope")
        vals["rope_positions"] = int(rope.shape[0])
    return SdarLoopArgs(**vals)


def sdar_loop(d: Dims, tau: float, sync: bool, n_steps: int, ws, err_flag=None, stream=None,
              args: Optional[SdarLoopArgs] = None, **tensors):
    """isd_sdar_loop: n_steps forwards of an SDAR-style stationary batch on the device."""
    a = args if args is not None else sdar_loop_args(d, n_steps, **tensors)
    _check(_lib.isd_sdar_loop(ctypes.byref(d), float(tau), int(bool(sync)), int(n_steps),
                              ctypes.byref(a), _ptr(ws, torch.uint8, None, "ws"), ws.numel(),
                              _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)))


# ---------------------------------------------------------------------------
# Full-depth forward over the ISD block
# ---------------------------------------------------------------------------
def layers_workspace_bytes(d: Dims, inter: int) -> int:
    return int(_lib.isd_layers_workspace_bytes(ctypes.byref(d), int(inter)))


def alloc_layers_workspace(d: Dims, inter: int, device="cuda") -> torch.Tensor:
    n = layers_workspace_bytes(d, inter)
    if n == 0:
        raise IsdError(ISD_ERR_INVALID_ARG)
    return torch.empty(n, dtype=torch.uint8, device=device)


def layer_array(d: Dims, inter: int, layers) -> ctypes.Array:
    """Checked isd_layer array from dicts of tensors named as its fields."""
    H, D = d.Hq * d.D, d.D
    kvrow = d.page_size * d.Hkv * D
    want = dict(in_norm=H, w_qkv=(d.Hq + 2 * d.Hkv) * D * H, q_norm=D, k_norm=D, w_o=H * d.Hq * D,
                post_norm=H, w_gate_up=2 * inter * H, w_down=H * inter,
                k_pool=d.num_pages * kvrow, v_pool=d.num_pages * kvrow)
    arr = (Layer * max(len(layers), 1))()
    for i, L in enumerate(layers):
        for n in LAYER_FIELDS:
            setattr(arr[i], n, _ptr(L[n], _BF16, want[n], f"layer {i} {n}"))
    return arr


def layers(d: Dims, inter: int, eps: float, layer_arr, n_layers: int, rope, x, page_table,
           kv_len, n_clean, ws, final_norm=None, out=None, err_flag=None, stream=None):
    """isd_layers: n_layers decoder layers over the block (x in/out), then
    the final RMSNorm into out when final_norm is given."""
    M, H = d.M, d.Hq * d.D
    if rope.dim() != 3 or rope.shape[1:] != (d.D // 2, 2):
        raise ValueError(f"rope must be [positions, {d.D // 2}, 2]")
    _check(_lib.isd_layers(
        ctypes.byref(d), int(n_layers), int(inter), float(eps), layer_arr,
        _ptr(rope, torch.float32, None, "rope"), int(rope.shape[0]),
        _ptr(final_norm, _BF16, H, "final_norm"), _ptr(x, _BF16, M * H, "x"),
        _ptr(out, _BF16, M * H, "out"),
        _ptr(page_table, torch.int32, d.B * d.max_pages_per_req, "page_table"),
        _ptr(kv_len, torch.int32, d.B, "kv_len"), _ptr(n_clean, torch.int32, d.B, "n_clean"),
        _ptr(ws, torch.uint8, None, "ws"), ws.numel(),
        _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)))


def embed_block(d: Dims, E, n_clean, clean_tok, x, err_flag=None, stream=None):
    """isd_embed_block: the block's input rows from the embedding table E [V+1, H]."""
    H = d.Hq * d.D
    _check(_lib.isd_embed_block(
        ctypes.byref(d), _ptr(E, _BF16, (d.V + 1) * H, "E"), _ptr(n_clean, torch.int32, d.B, "n_clean"),
        _ptr(clean_tok, torch.int32, d.B * d.N, "clean_tok"), _ptr(x, _BF16, d.M * H, "x"),
        _ptr(err_flag, torch.int32, 1, "err_flag"), _stream(stream)))
