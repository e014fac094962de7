"""The allocation-free dense Top-K entry point (dosa_index_dense_topk_static).

Callers that cannot allocate device memory use this entry point; its scratch is
a fixed array inside the library.  Called through the C-ABI twice in a row, it
must return exactly what dosa_index_dense_topk returns (the same kernels run on
the same inputs, so the tolerance is equality), and it must reject sizes beyond
its fixed scratch before launching anything.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from exact_certified_top_b200 import binding
from exact_certified_top_b200.workloads import generate, small_case

pytestmark = pytest.mark.gpu


def _call_static(lib, idx, x, so, K, out):
    so_t = torch.as_tensor(so, dtype=torch.int64).contiguous()
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return lib.dosa_index_dense_topk_static(
        idx._h, ptr(x["q"]), ptr(x["q_scale"]), ptr(x["w"]), ptr(x["k"]), ptr(x["k_scale"]),
        ctypes.c_void_p(so_t.data_ptr()), so_t.shape[0] - 1, K, ptr(out),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("base,T,S,K", [("causal_1k_bf16", 600, 1500, 128),
                                        ("prefill_128k_fp8", 333, 4096, 1000)])
def test_static_entry_matches_dense_topk_twice(cuda_lib, base, T, S, K):
    lib = binding.load()
    wl = small_case(base, T, S, K=K, q_pos0=S - T)
    x = {k: (v.cuda() if torch.is_tensor(v) and k != "seq_offsets" else v)
         for k, v in generate(wl).items()}
    idx = binding.Index(wl.dtype)
    want = idx.dense_topk(x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"], x["seq_offsets"], K)
    for _ in range(2):
        out = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
        assert _call_static(lib, idx, x, x["seq_offsets"], K, out) == 0
        torch.cuda.synchronize()
        # the static call's device error word (expired waits, bounds checks)
        # sits in the fixed array's header: NULL reads it back
        assert lib.dosa_check_device(None, ctypes.c_void_p(
            torch.cuda.current_stream().cuda_stream)) == 0
        assert torch.equal(out, want)


def test_static_entry_rejects_sizes_beyond_its_scratch(cuda_lib):
    lib = binding.load()
    idx = binding.Index("bf16")
    fake = torch.empty(16, dtype=torch.uint8, device="cuda")     # never read
    x = {"q": fake, "q_scale": None, "w": fake, "k": fake, "k_scale": None}
    so = [[0, 0, 1000000 - 8], [8, 1000000, 0]]                   # 1M keys > 524280
    out = torch.empty((8, 16), dtype=torch.int32, device="cuda")
    assert _call_static(lib, idx, x, so, 16, out) == 3           # DOSA_ERR_WORKSPACE
