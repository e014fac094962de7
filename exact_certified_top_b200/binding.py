"""ctypes binding of libdosa (include/dosa.h).

Argument marshalling only: tensors become device pointers, the current torch
stream becomes the cudaStream_t, status codes become exceptions.  Every step of
the indexer runs in the library's CUDA kernels; there is no CPU fallback, and
loading fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdosa.so")

DOSA_BF16, DOSA_FP8_E4M3 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration",
          3: "workspace too small", 4: "CUDA error", 5: "device wait timed out",
          6: "device bounds check failed"}

# Every function the public header declares (the CPU tests check the export).
EXPORTS = ("dosa_index_config_default", "dosa_index_create", "dosa_index_destroy",
           "dosa_index_workspace_size", "dosa_index_topk", "dosa_index_dense_topk",
           "dosa_index_scores", "dosa_reference_scores", "dosa_index_certificate",
           "dosa_index_dense_topk_static", "dosa_topk_rows", "dosa_check_device",
           "dosa_status_string", "dosa_profile_enable", "dosa_profile_reset",
           "dosa_profile_read", "dosa_index_topk_host", "dosa_index_host_workspace_size",
           "dosa_index_decode_topk", "dosa_index_decode_workspace_size")
KERNELS = {"score": 0, "topk": 1, "reference": 2, "key_prep": 3, "cert_setup": 4,
           "certified": 5, "select": 6, "filter": 7, "decode": 8,
           "fill": 9, "block": 10, "rescore": 11, "rank": 12}


class DosaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({code})")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("d", ctypes.c_int), ("dtype", ctypes.c_int),
                ("max_K", ctypes.c_int), ("seed_first", ctypes.c_int),
                ("seed_last", ctypes.c_int), ("r", ctypes.c_int), ("G", ctypes.c_int),
                ("margin_log2", ctypes.c_int), ("screening", ctypes.c_int),
                ("sparse_writeback", ctypes.c_int), ("block_bound", ctypes.c_int),
                ("probe_sample", ctypes.c_int), ("short_dense_keys", ctypes.c_int)]


class Stats(ctypes.Structure):
    _fields_ = [("visible_pairs", ctypes.c_int64), ("seed_pairs", ctypes.c_int64),
                ("screened_pairs", ctypes.c_int64), ("rejected_pairs", ctypes.c_int64),
                ("exact_pairs", ctypes.c_int64), ("candidates", ctypes.c_int64),
                ("filtered_pairs", ctypes.c_int64), ("block_skipped_pairs", ctypes.c_int64),
                ("rescored_pairs", ctypes.c_int64), ("repaired_rows", ctypes.c_int64),
                ("rescreened_pairs", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {name: int(getattr(self, name)) for name, _ in self._fields_}


_lib = None
_P, _I, _I64, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t


def load(path: str = LIB_PATH):
    """Load libdosa.so and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built: run `python -m exact_certified_top_b200.build`")
    lib = ctypes.CDLL(path)
    lib.dosa_index_config_default.argtypes = [ctypes.POINTER(Config)]
    lib.dosa_index_config_default.restype = None
    lib.dosa_index_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(_P)]
    lib.dosa_index_destroy.argtypes = [_P]
    lib.dosa_index_destroy.restype = None
    lib.dosa_index_workspace_size.argtypes = [_P, _I64, _I64, _I, _I, _I64,
                                              ctypes.POINTER(_SZ)]
    common = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _SZ, _P]
    lib.dosa_index_topk.argtypes = common + [ctypes.POINTER(Stats)]
    lib.dosa_index_dense_topk.argtypes = common
    lib.dosa_index_topk_host.argtypes = common + [ctypes.POINTER(Stats)]
    lib.dosa_index_decode_topk.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P, _SZ,
                                           _P, ctypes.POINTER(Stats)]
    lib.dosa_index_decode_workspace_size.argtypes = [_P, _I64, _I64, _I, ctypes.POINTER(_SZ)]
    lib.dosa_index_host_workspace_size.argtypes = [_P, _I64, _I64, _I64, _I, _I64,
                                                   ctypes.POINTER(_SZ)]
    lib.dosa_index_scores.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _I64,
                                      _P, _P]
    lib.dosa_reference_scores.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P,
                                          _I64, _P]
    lib.dosa_index_dense_topk_static.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P]
    lib.dosa_index_certificate.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _SZ,
                                           _P]
    lib.dosa_topk_rows.argtypes = [_P, _I64, _P, _I64, _I, _P, _P]
    lib.dosa_check_device.argtypes = [_P, _P]
    lib.dosa_profile_enable.argtypes = [_I]
    lib.dosa_profile_reset.argtypes = []
    lib.dosa_profile_read.argtypes = [_I, ctypes.POINTER(_I64), ctypes.POINTER(ctypes.c_double)]
    lib.dosa_status_string.argtypes = [_I]
    lib.dosa_status_string.restype = ctypes.c_char_p
    for fn in EXPORTS:
        f = getattr(lib, fn)
        if f.restype is ctypes.c_int and fn not in ("dosa_index_config_default",):
            f.restype = ctypes.c_int
    _lib = lib
    return lib


def _check(fn: str, code: int):
    if code != 0:
        raise DosaError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _seq_offsets(seq_offsets) -> torch.Tensor:
    so = torch.as_tensor(seq_offsets, dtype=torch.int64).cpu().contiguous()
    if so.dim() != 2 or so.shape[1] != 3:
        raise ValueError("seq_offsets must be [B+1, 3]")
    return so


class Index:
    """A libdosa handle: the certified indexer and its dense reference."""

    def __init__(self, dtype: str = "bf16", H: int = 64, d: int = 128, max_K: int = 2048,
                 **overrides):
        lib = load()
        cfg = Config()
        lib.dosa_index_config_default(ctypes.byref(cfg))
        cfg.H, cfg.d, cfg.max_K = H, d, max_K
        cfg.dtype = DOSA_FP8_E4M3 if dtype == "fp8" else DOSA_BF16
        for k, v in overrides.items():
            setattr(cfg, k, int(v))
        self.cfg = cfg
        self.dtype = dtype
        h = ctypes.c_void_p()
        _check("dosa_index_create", lib.dosa_index_create(ctypes.byref(cfg), ctypes.byref(h)))
        self._h = h
        self._lib = lib

    def close(self):
        if getattr(self, "_h", None):
            self._lib.dosa_index_destroy(self._h)
            self._h = None

    __del__ = close

    def workspace_size(self, Tq: int, S_max: int, K: int, certified: bool,
                       chunk_rows: int = 0) -> int:
        n = ctypes.c_size_t()
        _check("dosa_index_workspace_size",
               self._lib.dosa_index_workspace_size(self._h, Tq, S_max, K, int(certified),
                                                   chunk_rows, ctypes.byref(n)))
        return int(n.value)

    def _workspace(self, q, seq_offsets, K, certified, workspace):
        if workspace is not None:
            return workspace
        so = _seq_offsets(seq_offsets)
        S_max = int((so[1:, 1] - so[:-1, 1]).max())
        n = self.workspace_size(q.shape[0], S_max, K, certified)
        return torch.zeros(n, dtype=torch.uint8, device=q.device)

    def _topk_args(self, q, q_scale, w, k, k_scale, seq_offsets, K, out):
        so = _seq_offsets(seq_offsets)
        if out is None:
            out = torch.empty((q.shape[0], K), dtype=torch.int32, device=q.device)
        return so, out

    def dense_topk(self, q, q_scale, w, k, k_scale, seq_offsets, K, out=None, workspace=None):
        so, out = self._topk_args(q, q_scale, w, k, k_scale, seq_offsets, K, out)
        ws = self._workspace(q, so, K, False, workspace)
        _check("dosa_index_dense_topk", self._lib.dosa_index_dense_topk(
            self._h, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k), _ptr(k_scale),
            ctypes.c_void_p(so.data_ptr()), so.shape[0] - 1, K, _ptr(out), _ptr(ws),
            ws.numel(), _stream()))
        return out

    def topk(self, q, q_scale, w, k, k_scale, seq_offsets, K, out=None, workspace=None,
             stats: bool = False):
        so, out = self._topk_args(q, q_scale, w, k, k_scale, seq_offsets, K, out)
        ws = self._workspace(q, so, K, True, workspace)
        st = Stats()
        _check("dosa_index_topk", self._lib.dosa_index_topk(
            self._h, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k), _ptr(k_scale),
            ctypes.c_void_p(so.data_ptr()), so.shape[0] - 1, K, _ptr(out), _ptr(ws),
            ws.numel(), _stream(), ctypes.byref(st) if stats else None))
        return (out, st.as_dict()) if stats else out

    def host_workspace_size(self, Tq: int, S_total: int, S_max: int, K: int,
                            chunk_rows: int = 0) -> int:
        n = ctypes.c_size_t()
        _check("dosa_index_host_workspace_size",
               self._lib.dosa_index_host_workspace_size(self._h, Tq, S_total, S_max, K,
                                                        chunk_rows, ctypes.byref(n)))
        return int(n.value)

    def topk_host(self, q, q_scale, w, k, k_scale, seq_offsets, K, out=None, workspace=None,
                  stats: bool = False):
        """Certified Top-K with host (CPU, ideally pinned) inputs and output; the
        workspace is a CUDA tensor (host_workspace_size bytes)."""
        so = _seq_offsets(seq_offsets)
        if out is None:
            out = torch.empty((q.shape[0], K), dtype=torch.int32, pin_memory=True)
        if workspace is None:
            S_max = int((so[1:, 1] - so[:-1, 1]).max())
            n = self.host_workspace_size(q.shape[0], int(so[-1, 1]), S_max, K)
            workspace = torch.zeros(n, dtype=torch.uint8, device="cuda")
        st = Stats()
        _check("dosa_index_topk_host", self._lib.dosa_index_topk_host(
            self._h, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k), _ptr(k_scale),
            ctypes.c_void_p(so.data_ptr()), so.shape[0] - 1, K, _ptr(out), _ptr(workspace),
            workspace.numel(), _stream(), ctypes.byref(st) if stats else None))
        return (out, st.as_dict()) if stats else out

    def decode_workspace_size(self, Tq: int, S_max: int, K: int) -> int:
        n = ctypes.c_size_t()
        _check("dosa_index_decode_workspace_size",
               self._lib.dosa_index_decode_workspace_size(self._h, Tq, S_max, K, ctypes.byref(n)))
        return int(n.value)

    def decode_topk(self, q, q_scale, w, k, k_scale, seq_offsets, K, seed_idx, out=None,
                    workspace=None, stats: bool = False):
        """Decode-step Top-K seeded by the previous step's selection seed_idx [Tq, K]."""
        so, out = self._topk_args(q, q_scale, w, k, k_scale, seq_offsets, K, out)
        if workspace is None:
            S_max = int((so[1:, 1] - so[:-1, 1]).max())
            workspace = torch.zeros(self.decode_workspace_size(q.shape[0], S_max, K),
                                    dtype=torch.uint8, device=q.device)
        seed = seed_idx.to(torch.int32).contiguous()
        st = Stats()
        _check("dosa_index_decode_topk", self._lib.dosa_index_decode_topk(
            self._h, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k), _ptr(k_scale),
            ctypes.c_void_p(so.data_ptr()), so.shape[0] - 1, K, _ptr(seed), _ptr(out),
            _ptr(workspace), workspace.numel(), _stream(), ctypes.byref(st) if stats else None))
        return (out, st.as_dict()) if stats else out

    def certificate(self, q, q_scale, w, k, k_scale, seq_offsets, workspace=None,
                    bound_rows: bool = False):
        """Per-query certificate records [Tq, 16] (code domain), retained heads
        [Tq, 4] and, when asked, the bound rows [Tq, 8, d] (codes, q's dtype)."""
        so = _seq_offsets(seq_offsets)
        cert = torch.empty((q.shape[0], 16), dtype=torch.float32, device=q.device)
        ret = torch.empty((q.shape[0], 4), dtype=torch.int32, device=q.device)
        rows = (torch.empty((q.shape[0], 8, q.shape[2]), dtype=q.dtype, device=q.device)
                if bound_rows else None)
        ws = self._workspace(q, so, 1, True, workspace)
        _check("dosa_index_certificate", self._lib.dosa_index_certificate(
            self._h, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k), _ptr(k_scale),
            ctypes.c_void_p(so.data_ptr()), so.shape[0] - 1, _ptr(cert), _ptr(ret), _ptr(rows),
            _ptr(ws), ws.numel(), _stream()))
        return (cert, ret, rows) if bound_rows else (cert, ret)

    def scores(self, q, q_scale, w, k, k_scale, row0, rows, pos0, S, out, ld, scratch):
        _check("dosa_index_scores", self._lib.dosa_index_scores(
            self._h, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k), _ptr(k_scale), row0, rows, pos0,
            S, _ptr(out), ld, _ptr(scratch), _stream()))
        return out

    def reference_scores(self, q, q_scale, w, k, k_scale, row0, rows, pos0, S, out, ld):
        _check("dosa_reference_scores", self._lib.dosa_reference_scores(
            self._h, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k), _ptr(k_scale), row0, rows, pos0,
            S, _ptr(out), ld, _stream()))
        return out


def topk_rows(scores: torch.Tensor, row_len: torch.Tensor, K: int, out=None) -> torch.Tensor:
    lib = load()
    if out is None:
        out = torch.empty((scores.shape[0], K), dtype=torch.int32, device=scores.device)
    _check("dosa_topk_rows", lib.dosa_topk_rows(_ptr(scores), scores.stride(0), _ptr(row_len),
                                                scores.shape[0], K, _ptr(out), _stream()))
    return out


def check_device(workspace: torch.Tensor):
    _check("dosa_check_device", load().dosa_check_device(_ptr(workspace), _stream()))


def profile_enable(on: bool = True):
    _check("dosa_profile_enable", load().dosa_profile_enable(int(on)))


def profile_reset():
    _check("dosa_profile_reset", load().dosa_profile_reset())


def profile_read() -> dict:
    """{kernel kind: (launches, summed device ms)} since the last reset."""
    lib = load()
    out = {}
    for name, kind in KERNELS.items():
        n, ms = ctypes.c_int64(), ctypes.c_double()
        _check("dosa_profile_read", lib.dosa_profile_read(kind, ctypes.byref(n), ctypes.byref(ms)))
        out[name] = (int(n.value), float(ms.value))
    return out
