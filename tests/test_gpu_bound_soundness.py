"""Soundness of the bound the GPU screens with, pair by pair.

The certificate's invariant ("DOSA: Dots Sparse Attention", Daily Paper Cast
transcript, Method: a rejected key could not have entered the Top-K) needs,
for every visible pair, UB(t,s) >= I(t,s).  The GPU's bound is rebuilt here in
fp64 from what the GPU itself screens with -- its folded weights omega, its
beta (with its spectral estimate and rounding slack), its margin coefficient
and its bound rows (the retained heads' codes and the hi/lo rows of the
negative aggregates, dosa_index_certificate) -- and compared with the oracle's
exact score of every pair.  A second check: the margin c ||k|| covers the
fp32 error of evaluating that bound on the GPU (tensor-core dot products of
length d and the few fp32 operations after them), so the bound the kernels
compare with the threshold is never below the exact one."""
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import replace

import numpy as np
import pytest
import torch
from threadpoolctl import threadpool_limits

from exact_certified_top_b200 import binding
from exact_certified_top_b200.workloads import WORKLOADS, codes_numpy, generate, small_case
from oracle import decode_bf16, decode_e4m3, indexer_scores

pytestmark = pytest.mark.gpu


def _decode(codes, dtype):
    return decode_e4m3(codes) if dtype == "fp8" else decode_bf16(codes)


def _check_rows(x, dtype, rows_to_check):
    """Every visible pair of the listed rows: rebuilt GPU bound >= exact score,
    and the margin >= 4x the fp32 evaluation error of the bound."""
    xd = {k: (v.cuda() if torch.is_tensor(v) and k != "seq_offsets" else v) for k, v in x.items()}
    idx = binding.Index(dtype)
    cert, ret, brows = idx.certificate(xd["q"], xd["q_scale"], xd["w"], xd["k"], xd["k_scale"],
                                       x["seq_offsets"], bound_rows=True)
    cert = cert.cpu().numpy().astype(np.float64)
    brows = _decode(codes_numpy(brows), dtype)               # [T, 8, d] code domain
    kc = _decode(codes_numpy(x["k"]), dtype)                  # [S, d] code domain
    ks = np.ones(kc.shape[0]) if x["k_scale"] is None else x["k_scale"].numpy().astype(np.float64)
    qs = np.ones(x["q"].shape[0]) if x["q_scale"] is None else x["q_scale"].numpy().astype(np.float64)
    qc = _decode(codes_numpy(x["q"]), dtype)
    w = x["w"].numpy().astype(np.float64)
    pos = x["positions"].numpy()
    knorm = np.linalg.norm(kc, axis=1)

    def one(t):
        n = int(pos[t]) + 1
        k = kc[:n]
        c = cert[t]
        R = brows[t]
        x4 = k @ R[:4].T                                      # retained heads
        y = k @ R[4:].T                                        # u_1 hi, lo, u_2 hi, lo
        neg1 = c[6] * y[:, 0] + c[7] * y[:, 1]
        neg2 = c[8] * y[:, 2] + c[9] * y[:, 3]
        ub = (np.maximum(x4, 0.0) @ c[0:4] + c[4] * knorm[:n]
              - np.maximum(neg1, 0.0) - np.maximum(neg2, 0.0))
        real = qs[t] * ks[:n]
        # exact score in the real domain (decoded codes times the scales)
        I = indexer_scores(qc[t] * qs[t], w[t], k * ks[:n, None])
        ub_real = ub * real
        slack = 1e-12 * (np.abs(ub_real) + np.abs(I) + 1.0)
        bad = np.nonzero(ub_real < I - slack)[0]
        assert bad.size == 0, (f"row {t}: {bad.size} pairs with bound below the score, first "
                               f"key {bad[0]}: bound {ub_real[bad[0]]} score {I[bad[0]]}")
        # fp32 evaluation error of the bound: the tensor-core dot products
        # (d = 128 terms, error <= d 2^-24 sum |a_i b_i| <= 2^-17 ||a|| ||k||) and
        # about ten fp32 operations on terms of the sizes below
        rn = np.linalg.norm(R, axis=1)
        dot_err = 2.0 ** -17 * knorm[:n] * (np.abs(c[0:4]) @ rn[:4]
                                            + abs(c[6]) * rn[4] + abs(c[7]) * rn[5]
                                            + abs(c[8]) * rn[6] + abs(c[9]) * rn[7])
        terms = (np.maximum(x4, 0.0) @ np.abs(c[0:4]) + c[4] * knorm[:n] + np.abs(neg1)
                 + np.abs(neg2))
        eval_err = dot_err + 16 * 2.0 ** -24 * terms
        margin = c[5] * knorm[:n]
        assert np.all(margin >= 4.0 * eval_err), f"row {t}: margin below the fp32 error bound"
        return n

    with threadpool_limits(1):
        with ThreadPoolExecutor(max(1, os.cpu_count() or 1)) as ex:
            pairs = sum(ex.map(one, rows_to_check))
    return pairs


def test_bound_sound_on_every_pair_of_the_1k_workload(cuda_lib):
    wl = WORKLOADS["causal_1k_bf16"]
    x = generate(wl)
    assert _check_rows(x, wl.dtype, range(wl.T)) == wl.visible_pairs


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_bound_sound_on_every_pair_of_redundant_heads(cuda_lib, dtype):
    """Near-copy heads: the bound is tight (beta small), so an error in omega,
    the projections or the hi/lo split would show here first."""
    base = "redundant_chunk128k_fp8"
    wl = replace(small_case(base, 256, 20000), dtype=dtype)
    x = generate(wl)
    assert _check_rows(x, dtype, range(wl.T)) == wl.visible_pairs


def test_bound_sound_on_every_pair_of_a_2048_row_slice_of_the_128k_prefill(cuda_lib):
    wl = WORKLOADS["prefill_128k_fp8"]
    wl = replace(wl, name="prefill_128k_fp8[last 2048 rows]", T=2048, q_pos0=wl.S - 2048)
    x = generate(wl)
    assert _check_rows(x, wl.dtype, range(wl.T)) == wl.visible_pairs
