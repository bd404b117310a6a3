"""isd_attention_noalloc: the attention step for callers that cannot hand the
library a workspace (an engine that gave all free device memory to its KV
cache, or code that must not call the CUDA allocator).  Its scratch comes
from a fixed array inside the library, so the same results must come out as
from isd_attention with a caller-owned workspace -- on consecutive calls,
since every call reuses that array.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from speculative_verification_isd_b200 import inputs as I


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["ragged_small", "qwen_medium"])
def test_noalloc_attention_matches_workspace_entry_point_twice(name):
    from speculative_verification_isd_b200 import isd
    from gpu_util import StepBuffers, bf16_host

    cfg = I.CONFIGS[name]
    inp = I.make_step_inputs(cfg, seed=21, n_clean="mixed")
    sb = StepBuffers(isd, cfg, inp)
    sb.attention()  # the existing entry point, with a caller-owned workspace
    torch.cuda.synchronize()
    ref = (bf16_host(sb.hidden).astype(np.uint32) << 16).view(np.float32)
    ref_k, ref_v = bf16_host(sb.k_pool), bf16_host(sb.v_pool)
    for _ in range(2):
        out = torch.full_like(sb.hidden, float("nan"))
        isd.attention_noalloc(sb.dims, sb.q, sb.k_new, sb.v_new, sb.k_pool, sb.v_pool,
                              sb.page_table, sb.kv_len, sb.n_clean, out, sb.err)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert np.all(np.isfinite(got))
        # the attention tolerance used by the parity tests (bf16 outputs)
        assert np.max(np.abs(got - ref.reshape(got.shape))) <= 2e-2
        assert np.array_equal(bf16_host(sb.k_pool), ref_k)
        assert np.array_equal(bf16_host(sb.v_pool), ref_v)
    assert int(sb.err.item()) == 0


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
