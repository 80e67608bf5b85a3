"""Seeded synthetic weights and calibration streams.

Everything is generated on the CPU with ``torch.Generator`` objects keyed by
(seed, purpose, index), so any chunk of a long stream can be regenerated alone
and both the GPU path and the oracle see bit-identical values.

Workload shapes follow the NanoQuant pages: calibration is 128 sequences of
2048 tokens (summary page, "Method steps" (方法步骤详情), stage one), i.e.
262144 tokens per stream; layers are Llama-2-7B / 70B shaped.  No dataset is
used: activations and gradients are Gaussian with per-channel log-normal scales,
standing in for WikiText-2 only by their shape.
"""
import hashlib
from dataclasses import dataclass
from typing import Iterator, List, Optional, Tuple

import torch

CALIB_TOKENS = 128 * 2048
CHUNK_TOKENS = 8192

__all__ = [
    "CALIB_TOKENS", "CHUNK_TOKENS", "make_generator", "channel_scales", "stream_chunks",
    "stream_tensor", "gaussian_weight", "student_t_weight", "planted_weight", "LayerSpec",
    "llama2_7b_block", "llama2_70b_block", "planted_problem", "random_problem",
]


def make_generator(seed: int, *keys) -> torch.Generator:
    """A CPU generator whose seed is a hash of (seed, *keys)."""
    h = hashlib.sha256(repr((int(seed),) + tuple(keys)).encode()).digest()
    g = torch.Generator(device="cpu")
    g.manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))
    return g


def channel_scales(seed: int, stream: str, C: int, sigma: float = 1.0) -> torch.Tensor:
    """Per-channel log-normal scales exp(sigma * N(0,1)), float32."""
    g = make_generator(seed, stream, "scales")
    return torch.exp(sigma * torch.randn(C, generator=g, dtype=torch.float32))


def stream_chunks(seed: int, stream: str, T: int, C: int, dtype=torch.bfloat16,
                  sigma: float = 1.0, chunk: int = CHUNK_TOKENS) -> Iterator[torch.Tensor]:
    """Token-major chunks of x_tj = N(0,1) * scale_j, cast to ``dtype`` (RNE)."""
    scales = channel_scales(seed, stream, C, sigma)
    t0 = 0
    idx = 0
    while t0 < T:
        t1 = min(T, t0 + chunk)
        g = make_generator(seed, stream, "chunk", idx)
        x = torch.randn(t1 - t0, C, generator=g, dtype=torch.float32) * scales
        yield x.to(dtype)
        t0 = t1
        idx += 1


def stream_tensor(seed: int, stream: str, T: int, C: int, dtype=torch.bfloat16,
                  sigma: float = 1.0, pin: bool = False) -> torch.Tensor:
    """The whole stream as one contiguous T x C tensor (optionally in pinned memory)."""
    out = torch.empty(T, C, dtype=dtype, pin_memory=pin)
    t0 = 0
    for x in stream_chunks(seed, stream, T, C, dtype, sigma):
        out[t0:t0 + x.shape[0]].copy_(x)
        t0 += x.shape[0]
    return out


def gaussian_weight(seed: int, name: str, m: int, n: int, std: float = 0.02,
                    outlier_frac: float = 0.0, outlier_gain: float = 1.0,
                    dtype=torch.bfloat16) -> torch.Tensor:
    """W ~ N(0, std^2) (m x n); a seeded ``outlier_frac`` of input columns scaled by ``outlier_gain``."""
    g = make_generator(seed, name, "W")
    W = torch.randn(m, n, generator=g, dtype=torch.float32) * std
    k = int(round(outlier_frac * n))
    if k > 0:
        cols = torch.randperm(n, generator=make_generator(seed, name, "outliers"))[:k]
        W[:, cols] *= outlier_gain
    return W.to(dtype)


def student_t_weight(seed: int, name: str, m: int, n: int, std: float = 0.02, nu: int = 3,
                     dtype=torch.bfloat16) -> torch.Tensor:
    """W ~ N(0, std^2) with input column j scaled by max(1, |t_j|), t_j ~ Student-t(nu)."""
    g = make_generator(seed, name, "W")
    W = torch.randn(m, n, generator=g, dtype=torch.float32) * std
    gt = make_generator(seed, name, "t")
    z = torch.randn(n, generator=gt, dtype=torch.float64)
    chi2 = (torch.randn(nu, n, generator=gt, dtype=torch.float64) ** 2).sum(0)
    t = z / torch.sqrt(chi2 / nu)
    W *= torch.clamp(t.abs(), min=1.0).to(torch.float32)[None, :]
    return W.to(dtype)


def planted_weight(seed: int, m: int, n: int, r: int, noise: float = 0.1,
                   scale_sigma: float = 0.5):
    """W = diag(s1) U V^T diag(s2) + noise * rms * N(0,1), float32.

    U, V have Bernoulli(1/2) +-1 entries; s1, s2 = exp(scale_sigma * N(0,1)).
    Returns (W, U, V, s1, s2) with the planted factors for recovery checks.
    """
    g = make_generator(seed, "planted")
    U = torch.where(torch.rand(m, r, generator=g) < 0.5, -1.0, 1.0).to(torch.float64)
    V = torch.where(torch.rand(n, r, generator=g) < 0.5, -1.0, 1.0).to(torch.float64)
    s1 = torch.exp(scale_sigma * torch.randn(m, generator=g, dtype=torch.float64))
    s2 = torch.exp(scale_sigma * torch.randn(n, generator=g, dtype=torch.float64))
    W0 = (s1[:, None] * (U @ V.T)) * s2[None, :]
    rms = torch.sqrt((W0 * W0).mean())
    E = torch.randn(m, n, generator=g, dtype=torch.float64)
    W = (W0 + noise * rms * E).to(torch.float32)
    return W, U, V, s1, s2


@dataclass
class LayerSpec:
    name: str
    m: int            # out features
    n: int            # in features
    stream_in: str    # name of the activation stream feeding the layer


def llama2_7b_block() -> List[LayerSpec]:
    """Linear layers of one Llama-2-7B transformer block (hidden 4096, MLP 11008)."""
    h, f = 4096, 11008
    return [LayerSpec("q_proj", h, h, "attn_in"), LayerSpec("k_proj", h, h, "attn_in"),
            LayerSpec("v_proj", h, h, "attn_in"), LayerSpec("o_proj", h, h, "o_in"),
            LayerSpec("gate_proj", f, h, "mlp_in"), LayerSpec("up_proj", f, h, "mlp_in"),
            LayerSpec("down_proj", h, f, "down_in")]


def llama2_70b_block() -> List[LayerSpec]:
    """Linear layers of one Llama-2-70B block (hidden 8192, GQA kv 1024, MLP 28672)."""
    h, kv, f = 8192, 1024, 28672
    return [LayerSpec("q_proj", h, h, "attn_in"), LayerSpec("k_proj", kv, h, "attn_in"),
            LayerSpec("v_proj", kv, h, "attn_in"), LayerSpec("o_proj", h, h, "o_in"),
            LayerSpec("gate_proj", f, h, "mlp_in"), LayerSpec("up_proj", f, h, "mlp_in"),
            LayerSpec("down_proj", h, f, "down_in")]


def planted_problem(seed: int = 0, m: int = 256, n: int = 512, r: int = 16, noise: float = 0.1,
                    T: int = 4096):
    """The planted 256 x 512 rank-16 FP32 problem with FP32 act/grad streams of T tokens."""
    W, U, V, s1, s2 = planted_weight(seed, m, n, r, noise)
    acts = stream_tensor(seed, "acts", T, n, dtype=torch.float32)
    grads = stream_tensor(seed, "grads", T, m, dtype=torch.float32)
    return dict(W=W, U=U, V=V, s1=s1, s2=s2, acts=acts, grads=grads)


def random_problem(seed: int, m: int, n: int, T: int, dtype=torch.bfloat16,
                   outlier_frac: float = 0.01, outlier_gain: float = 10.0):
    """A Gaussian BF16 layer with outlier columns and BF16 act/grad streams of T tokens."""
    W = gaussian_weight(seed, "W", m, n, 0.02, outlier_frac, outlier_gain, dtype)
    acts = stream_tensor(seed, "acts", T, n, dtype=dtype)
    grads = stream_tensor(seed, "grads", T, m, dtype=dtype)
    return dict(W=W, acts=acts, grads=grads)
