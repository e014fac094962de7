"""Seeded synthetic inputs for the indexer workloads.

This module only draws inputs: it holds none of the indexer's arithmetic, and
both the CUDA path and the CPU oracle consume the same tensors it returns.

Generator (one sequence, H heads, head dimension d):
  k[s]   = mu_k + c * A_k z_s + 0.3 eps_s          (A_k: d x 16, entries N(0,1)/4)
  q[t,h] = mu_q + A_q z_{t,h} + 0.3 eps_{t,h}      (its own mu_q, A_q)
  mu ~ N(0, I_d) drawn once; z in R^16 and eps in R^d are i.i.d. N(0,1).
  Sinks: a seeded 1 % of key positions have k scaled by 4.
  w[t,h] ~ N(0,1)/8 i.i.d. (mixed signs); the bound-tightness case instead
  makes a random half of each query's heads negative, w = +-|N(0,1)|/8.
  c = 1, or 0.1 for the nearly isotropic keys of the bound-tightness case.
Redundant heads (head_noise > 0): z and eps are drawn once per query token and
  shared by its heads, and each head adds its own N(0, head_noise^2) per
  coordinate: q[t,h] = mu_q + A_q z_t + 0.3 eps_t + head_noise * n_{t,h}.  The
  weights are w[t,h] = |N(0,1)|/8 with a seeded random quarter of each query's
  heads negated.  This stands in for trained indexers, whose heads are far
  more alike than independent draws (the pages' prune rates are measured on
  such layers).
Storage:
  bf16: round-to-nearest-even from fp32.
  fp8 e4m3: one fp32 scale per token = absmax / 448 (over H x d for a query
  token, over d for a key), code = e4m3(value / scale) after clamping to +-448.
  levels=8: q, k and w are rounded to the 8 integer levels {-4..3} times a
  per-tensor power-of-two step chosen so the levels span about +-2 sigma; every
  score is then an exact dyadic number, so ties are common and fp32 is exact.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

__all__ = ["Workload", "WORKLOADS", "generate", "small_case"]


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                      # query rows
    S: int                      # keys of the sequence
    H: int = 64
    d: int = 128
    dtype: str = "bf16"         # "bf16" or "fp8" (e4m3 + per-token fp32 scales)
    K: int = 2048
    q_pos0: int = 0             # position of query row 0 among the keys
    lowrank_scale: float = 1.0  # c in the key generator
    neg_half: bool = False      # exactly half of each query's heads negative
    levels: int = 0             # 0, or 8 for integer-level quantisation
    seed: int = 0
    sink_frac: float = 0.01
    # decode steps: rows 1.. are row 0 (the previous step) plus N(0, noise^2)
    # per coordinate (w: plus N(0, (noise / 8)^2)), drawn before quantisation
    decode_noise: float = 0.0
    # redundant heads: per-head perturbation of a shared per-token query
    head_noise: float = 0.0

    @property
    def visible_pairs(self) -> int:
        """Causal query-key pairs: sum over rows of (position + 1)."""
        a = self.q_pos0 + 1
        b = self.q_pos0 + self.T
        return (a + b) * self.T // 2


WORKLOADS = {
    "causal_1k_bf16": Workload("causal_1k_bf16", T=1024, S=1024, K=256),
    "causal_16k_bf16": Workload("causal_16k_bf16", T=16384, S=16384, K=2048),
    "prefill_128k_fp8": Workload("prefill_128k_fp8", T=131072, S=131072, dtype="fp8", K=2048),
    # the same prefill with a 32-head indexer (the GLM-style shape)
    "prefill_128k_fp8_h32": Workload("prefill_128k_fp8_h32", T=131072, S=131072, H=32,
                                     dtype="fp8", K=2048),
    "chunk_1m_fp8": Workload("chunk_1m_fp8", T=8192, S=1048576, dtype="fp8", K=2048,
                             q_pos0=1048576 - 8192),
    "tight_64k_bf16_levels": Workload("tight_64k_bf16_levels", T=65536, S=65536, K=2048,
                                      lowrank_scale=0.1, neg_half=True, levels=8),
    # heads of a query nearly alike (trained-indexer stand-in): the certificate
    # is tight and screening rejects most keys.  A prefill chunk of 8,192 rows
    # at the end of a 128K context, and the whole 128K causal prefill.
    "redundant_chunk128k_fp8": Workload("redundant_chunk128k_fp8", T=8192, S=131072,
                                        dtype="fp8", K=2048, q_pos0=131072 - 8192,
                                        head_noise=0.05),
    "redundant_128k_fp8": Workload("redundant_128k_fp8", T=131072, S=131072, dtype="fp8",
                                   K=2048, head_noise=0.05),
    # decode step at ~1M cached keys: the last 5 rows of the sequence; row 0
    # (position S - 5) is the previous step, whose selection seeds rows 1..4
    # (a 4-row multi-token-prediction step)
    "decode_1m_fp8": Workload("decode_1m_fp8", T=5, S=1048576, dtype="fp8", K=2048,
                              q_pos0=1048576 - 5, decode_noise=0.3),
}

# Rows of a decode workload: row 0 is the previous step, rows 1.. are decoded.
DECODE_PREV_ROWS = 1


def small_case(base: str, T: int, S: int | None = None, **kw) -> Workload:
    """A reduced-size copy of a named workload (same generator and dtype)."""
    wl = WORKLOADS[base]
    S = T if S is None else S
    q_pos0 = kw.pop("q_pos0", S - T if wl.q_pos0 else 0)
    return replace(wl, name=f"{base}@T{T}S{S}", T=T, S=S, q_pos0=q_pos0, **kw)


def _randn(g, shape, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _e4m3_per_token(x: torch.Tensor):
    """x: [n, ...] fp32 -> (uint8 codes, fp32 scale [n]); scale = absmax/448."""
    n = x.shape[0]
    amax = x.reshape(n, -1).abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    y = (x / scale.view((n,) + (1,) * (x.dim() - 1))).clamp(-448.0, 448.0)
    return y.to(torch.float8_e4m3fn).view(torch.uint8), scale.to(torch.float32)


def _level_step(sigma: float) -> float:
    """Power-of-two step so that 4 steps cover about 2 sigma."""
    return 2.0 ** round(math.log2(max(2.0 * sigma / 4.0, 1e-30)))


def _to_levels(x: torch.Tensor, step: float) -> torch.Tensor:
    return torch.clamp(torch.floor(x / step + 0.5), -4, 3) * step


def generate(wl: Workload, device="cpu", chunk: int = 4096) -> dict:
    """Draw the inputs of ``wl`` on ``device``.

    Returns a dict: q [T,H,d] (torch.bfloat16, or uint8 e4m3 codes), q_scale [T]
    fp32 or None, w [T,H] fp32, k [S,d], k_scale [S] or None, positions [T]
    int64, seq_offsets [[0, 0, q_pos0], [T, S, 0]] int64 (host), sinks [S] bool.
    The same seed on the same device gives the same bytes."""
    device = torch.device(device)
    # The workload's own constants (means, low-rank maps, sink positions) come
    # from a host generator, so every device draws the same workload; the
    # per-token draws use the device's generator (same seed).
    seed = int(wl.seed) * 1000003 + 17
    gh = torch.Generator(device="cpu")
    gh.manual_seed(seed)
    H, d, T, S = wl.H, wl.d, wl.T, wl.S
    mu_k = _randn(gh, (d,), "cpu").to(device)
    A_k = (_randn(gh, (d, 16), "cpu") / 4.0).to(device)
    mu_q = _randn(gh, (d,), "cpu").to(device)
    A_q = (_randn(gh, (d, 16), "cpu") / 4.0).to(device)
    sinks = (torch.rand((S,), generator=gh) < wl.sink_frac).to(device)
    if device.type == "cpu":
        g = gh
    else:
        g = torch.Generator(device=device)
        g.manual_seed(seed)

    # keys, chunked over tokens
    kf = torch.empty((S, d), dtype=torch.float32, device=device)
    for s0 in range(0, S, chunk):
        n = min(chunk, S - s0)
        z = _randn(g, (n, 16), device)
        eps = _randn(g, (n, d), device)
        kf[s0:s0 + n] = mu_k + wl.lowrank_scale * (z @ A_k.T) + 0.3 * eps
    kf[sinks] *= 4.0

    # head weights
    w = _randn(g, (T, H), device) / 8.0
    if wl.head_noise > 0:
        w = w.abs()
        neg = torch.argsort(torch.rand((T, H), generator=g, device=device), dim=1)[:, : H // 4]
        w.scatter_(1, neg, -w.gather(1, neg))
    if wl.neg_half:
        w = w.abs()
        neg = torch.argsort(torch.rand((T, H), generator=g, device=device), dim=1)[:, : H // 2]
        w.scatter_(1, neg, -w.gather(1, neg))
    if wl.decode_noise > 0:
        assert T <= max(1, chunk // 16), "decode workloads are a few rows"
        w[1:] = w[0:1] + (wl.decode_noise / 8.0) * _randn(g, (T - 1, H), device)

    out = {"positions": torch.arange(wl.q_pos0, wl.q_pos0 + T, dtype=torch.int64, device=device),
           "seq_offsets": torch.tensor([[0, 0, wl.q_pos0], [T, S, 0]], dtype=torch.int64),
           "sinks": sinks}

    # queries, chunked; quantised chunk by chunk to bound memory
    if wl.dtype == "fp8":
        q = torch.empty((T, H, d), dtype=torch.uint8, device=device)
        q_scale = torch.empty((T,), dtype=torch.float32, device=device)
    else:
        q = torch.empty((T, H, d), dtype=torch.bfloat16, device=device)
        q_scale = None
    q_step = None
    for t0 in range(0, T, max(1, chunk // 16)):
        n = min(max(1, chunk // 16), T - t0)
        if wl.head_noise > 0:
            z = _randn(g, (n, 1, 16), device)
            eps = _randn(g, (n, 1, d), device)
            qf = mu_q + z @ A_q.T + 0.3 * eps + wl.head_noise * _randn(g, (n, H, d), device)
        else:
            z = _randn(g, (n, H, 16), device)
            eps = _randn(g, (n, H, d), device)
            qf = mu_q + z @ A_q.T + 0.3 * eps
        if wl.decode_noise > 0:
            qf[1:] = qf[0:1] + wl.decode_noise * _randn(g, (n - 1, H, d), device)
        if wl.dtype == "fp8":
            q[t0:t0 + n], q_scale[t0:t0 + n] = _e4m3_per_token(qf)
        else:
            if wl.levels:
                if q_step is None:
                    q_step = _level_step(float(qf.std()))
                qf = _to_levels(qf, q_step)
            q[t0:t0 + n] = qf.to(torch.bfloat16)

    if wl.dtype == "fp8":
        k, k_scale = _e4m3_per_token(kf)
    else:
        if wl.levels:
            kf = _to_levels(kf, _level_step(float(kf.std())))
            w = _to_levels(w, _level_step(float(w.std())))
        k, k_scale = kf.to(torch.bfloat16), None
    out.update(q=q, q_scale=q_scale, w=w.contiguous(), k=k.contiguous(), k_scale=k_scale)
    return out


def codes_numpy(x: torch.Tensor):
    """Host numpy view of stored codes: uint16 bit patterns for bf16 tensors,
    uint8 for e4m3 codes."""
    x = x.detach().cpu()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view("uint16")
    return x.numpy()
