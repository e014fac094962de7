"""Host-side checks of the C-ABI (no GPU needed): the library loads, exports
every function include/dosa.h declares, validates configs and rejects bad
arguments before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

from exact_certified_top_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "dosa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dosa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return binding.load()


def test_every_declared_function_is_exported(lib):
    names = header_functions()
    assert set(names) == set(binding.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (dosa_\w+)", out))
    for n in names:
        assert n in exported, n
        assert getattr(lib, n) is not None


def test_config_default_and_create(lib):
    cfg = binding.Config()
    lib.dosa_index_config_default(ctypes.byref(cfg))
    assert (cfg.H, cfg.d, cfg.max_K, cfg.seed_first, cfg.seed_last, cfg.r, cfg.G,
            cfg.margin_log2, cfg.screening, cfg.sparse_writeback, cfg.block_bound,
            cfg.probe_sample, cfg.short_dense_keys) == (64, 128, 2048, 64, 512, 4, 2, -12, 2, 1, 1,
                                                        1, 16384)
    h = ctypes.c_void_p()
    assert lib.dosa_index_create(ctypes.byref(cfg), ctypes.byref(h)) == 0 and h.value
    lib.dosa_index_destroy(h)
    lib.dosa_index_destroy(None)


def test_create_accepts_32_heads(lib):
    cfg = binding.Config()
    lib.dosa_index_config_default(ctypes.byref(cfg))
    cfg.H = 32
    h = ctypes.c_void_p()
    assert lib.dosa_index_create(ctypes.byref(cfg), ctypes.byref(h)) == 0 and h.value
    lib.dosa_index_destroy(h)


@pytest.mark.parametrize("field,value,code", [("d", 64, 2), ("H", 48, 2), ("max_K", 0, 1),
                                              ("r", 5, 1), ("G", 3, 1), ("margin_log2", 0, 1),
                                              ("dtype", 7, 1), ("screening", 4, 1),
                                              ("sparse_writeback", 2, 1), ("block_bound", -1, 1),
                                              ("probe_sample", 2, 1), ("short_dense_keys", -1, 1)])
def test_create_rejects_bad_config(lib, field, value, code):
    cfg = binding.Config()
    lib.dosa_index_config_default(ctypes.byref(cfg))
    setattr(cfg, field, value)
    h = ctypes.c_void_p()
    assert lib.dosa_index_create(ctypes.byref(cfg), ctypes.byref(h)) == code
    assert not h.value


def test_workspace_size_dense(lib):
    idx = binding.Index("bf16")
    n = idx.workspace_size(1024, 1024, 256, certified=False)
    assert n == 256 + 1024 * 1024 * 4
    n = idx.workspace_size(131072, 131072, 2048, certified=False)
    assert n == 256 + 8192 * 131072 * 4
    with pytest.raises(binding.DosaError):
        idx.workspace_size(10, 10, 0, certified=False)
    with pytest.raises(binding.DosaError):
        idx.workspace_size(10, 10, 4096, certified=False)


def _call_dense(lib, idx, **over):
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: every case fails validation
    so = (ctypes.c_int64 * 6)(0, 0, 0, 8, 8, 0)
    args = dict(q=fake, q_scale=None, w=fake, k=fake, k_scale=None, so=so, B=1, K=4, out=fake,
                ws=ctypes.c_void_p(1 << 20), ws_bytes=1 << 20)
    args.update(over)
    return lib.dosa_index_dense_topk(idx._h, args["q"], args["q_scale"], args["w"], args["k"],
                                     args["k_scale"], args["so"], args["B"], args["K"],
                                     args["out"], args["ws"], args["ws_bytes"], None)


def test_dense_topk_rejects_bad_arguments_without_launching(lib):
    idx = binding.Index("bf16")
    assert _call_dense(lib, idx, q=None) == 1
    assert _call_dense(lib, idx, K=0) == 1
    assert _call_dense(lib, idx, K=4096) == 1
    assert _call_dense(lib, idx, B=0) == 1
    assert _call_dense(lib, idx, q=ctypes.c_void_p((1 << 20) + 8)) == 1      # misaligned
    assert _call_dense(lib, idx, q_scale=ctypes.c_void_p(1 << 20)) == 1      # bf16 with scales
    bad = (ctypes.c_int64 * 6)(0, 0, 5, 8, 8, 0)                             # 8 rows from pos 5 > 8 keys
    assert _call_dense(lib, idx, so=bad) == 1
    assert _call_dense(lib, idx, ws_bytes=100) == 3                          # workspace too small
    assert _call_dense(lib, idx, ws=ctypes.c_void_p((1 << 20) + 16)) == 1    # misaligned workspace
    fp8 = binding.Index("fp8")
    assert _call_dense(lib, fp8) == 1                                         # fp8 without scales


def test_status_strings(lib):
    assert lib.dosa_status_string(0) == b"ok"
    assert lib.dosa_status_string(5) == b"device wait timed out"
    assert lib.dosa_status_string(99) == b"unknown status"
