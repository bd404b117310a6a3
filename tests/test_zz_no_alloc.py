"""isd_attention_noalloc: the attention step for callers that cannot hand the
library a workspace (an engine that gave all free device memory to its KV
cache, or code that must not call the CUDA allocator).  Its scratch comes
from a fixed array inside the library; otherwise it launches the same kernels
with the same partition as isd_attention, so its output must be bit-identical
to isd_attention's with a caller-owned workspace -- on consecutive calls,
since every call reuses that array.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from speculative_verification_isd_b200 import inputs as I


def _noalloc_twice_equals_workspace_call(isd, sb_dims, args, hidden_ws, err):
    """Two noalloc calls in a row, each bit-identical to the workspace call."""
    from gpu_util import bf16_host
    ref = bf16_host(hidden_ws)
    for _ in range(2):
        out = torch.full_like(hidden_ws, float("nan"))
        isd.attention_noalloc(sb_dims, *args, out, err)
        torch.cuda.synchronize()
        assert np.array_equal(bf16_host(out), ref)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "ragged_small", "qwen_medium"])
def test_noalloc_attention_matches_workspace_entry_point_twice(name):
    """tiny (head dim 64) runs the general kernel, the others the tensor-core
    kernel; both take their partials and counters from the built-in array."""
    from speculative_verification_isd_b200 import isd
    from gpu_util import StepBuffers, bf16_host

    cfg = I.CONFIGS[name]
    inp = I.make_step_inputs(cfg, seed=21, n_clean="mixed")
    sb = StepBuffers(isd, cfg, inp)
    sb.attention()  # the existing entry point, with a caller-owned workspace
    torch.cuda.synchronize()
    ref_k, ref_v = bf16_host(sb.k_pool), bf16_host(sb.v_pool)
    args = (sb.q, sb.k_new, sb.v_new, sb.k_pool, sb.v_pool, sb.page_table, sb.kv_len, sb.n_clean)
    _noalloc_twice_equals_workspace_call(isd, sb.dims, args, sb.hidden, sb.err)
    assert np.array_equal(bf16_host(sb.k_pool), ref_k)
    assert np.array_equal(bf16_host(sb.v_pool), ref_v)
    assert int(sb.err.item()) == 0


@pytest.mark.gpu
def test_noalloc_attention_at_the_benchmark_shape():
    """Qwen3-8B shapes, B=32, N=4, prefixes up to 8192 tokens: the shape the
    header names as fitting the built-in array.  Its split partials reach
    close to the array's end, so this also checks that the last bytes are
    addressed correctly."""
    from speculative_verification_isd_b200 import isd
    from speculative_verification_isd_b200 import workload as Wk

    cfg = I.CONFIGS["qwen3_8b_b32_n4"]
    wl = Wk.DeviceWorkload(isd, cfg, seed=2, accept_rate=None)
    d = wl.dims
    args = (wl.q, wl.k_new, wl.v_new, wl.k_pool, wl.v_pool, wl.page_table, wl.kv_len, wl.n_clean)
    isd.attention(d, *args, wl.hidden, wl.ws, wl.err)
    torch.cuda.synchronize()
    _noalloc_twice_equals_workspace_call(isd, d, args, wl.hidden, wl.err)
    assert int(wl.err.item()) == 0


def test_noalloc_rejects_dims_beyond_its_scratch():
    """Dims whose scratch would not fit the built-in array are refused on the
    host (nothing is launched, the pointers are never touched)."""
    from speculative_verification_isd_b200 import isd
    lib = isd.library()
    # 256 requests, 8 KV heads, 32 K-token contexts: far more than 32 MiB of partials
    d = isd.make_dims(256, 4, 32, 8, 128, 151936, 16, 1000, 2048)
    fake = ctypes.c_void_p(1 << 20)
    st = lib.isd_attention_noalloc(ctypes.byref(d), *([fake] * 9), None, None)
    assert st == isd.ISD_ERR_WORKSPACE
    msg = lib.isd_last_error().decode()
    assert "scratch" in msg and str(isd.NOALLOC_SCRATCH_BYTES) in msg
