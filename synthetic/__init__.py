"""Seeded synthetic inputs for the quantized linear layers.

Shared by the tests, ``bench.py`` and ``__graft_entry__.smoke()``; it holds
none of the method's arithmetic (no scales, no rounding to codes, no GEMM),
only random draws. Every tensor is drawn in fp32 on the CPU from its own
``torch.Generator`` seeded with ``base + crc32(key)``, then cast to fp16
with round-to-nearest-even (torch's conversion), so any process that asks
for the same key gets the same bytes.

The workloads mirror the diffusion transformer of "A Quantized Native
Runtime for On-Device Semantic Audio Generation" (aria project page,
"Results": 8 denoising steps, the four linears of a DiT block). No trained
checkpoint is available, so weights are N(0, 0.02^2) draws of the same
shapes and activations are N(0, 1) draws.
"""
from __future__ import annotations

import zlib

import torch

# (name, K = in features, N = out features) of one DiT block's linears
def block_linears(d: int, ffn: int | None = None):
    ffn = 4 * d if ffn is None else ffn
    return [("qkv", d, 3 * d), ("out", d, d), ("up", d, ffn), ("down", ffn, d)]


D1024 = block_linears(1024)          # 1024->3072, 1024->1024, 1024->4096, 4096->1024
D1536 = block_linears(1536)          # 1536->4608, 1536->1536, 1536->6144, 6144->1536
REPLAY_BLOCKS = 24
REPLAY_STEPS = 8
REPLAY_M = 432                       # 2 CFG halves x 216 latent frames
REPLAY_STEER_BLOCK = 12
REPLAY_ALPHA = 0.3


def _gen(key: str, base: int = 0) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((base + zlib.crc32(key.encode())) & 0x7FFFFFFFFFFF)
    return g


def normal(key: str, shape, std: float = 1.0, base: int = 0, dtype=torch.float16) -> torch.Tensor:
    """N(0, std^2) draw in fp32, cast to ``dtype`` (RN). CPU tensor."""
    t = torch.randn(*shape, generator=_gen(key, base), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def weight(key: str, N: int, K: int, std: float = 0.02, outlier_frac: float = 0.0,
           outlier_std: float = 0.2, base: int = 0) -> torch.Tensor:
    """fp16 [N, K] weight (out x in). With ``outlier_frac`` > 0, exactly
    round(outlier_frac*N*K) entries at seeded positions are redrawn from
    N(0, outlier_std^2)."""
    w = torch.randn(N, K, generator=_gen(key + "/w", base), dtype=torch.float32).mul_(std)
    n_out = int(round(outlier_frac * N * K))
    if n_out:
        g = _gen(key + "/outliers", base)
        pos = torch.randperm(N * K, generator=g)[:n_out]
        w.view(-1)[pos] = torch.randn(n_out, generator=g, dtype=torch.float32) * outlier_std
    return w.to(torch.float16)


def activation(key: str, M: int, K: int, outlier_channel_frac: float = 0.0,
               outlier_scale: float = 20.0, base: int = 0) -> torch.Tensor:
    """fp16 [M, K] activations ~N(0,1). With ``outlier_channel_frac`` > 0,
    round(frac*K) input channels (seeded randperm, the same columns in every
    row) are multiplied by ``outlier_scale``."""
    x = torch.randn(M, K, generator=_gen(key + "/x", base), dtype=torch.float32)
    n_ch = int(round(outlier_channel_frac * K))
    if n_ch:
        cols = torch.randperm(K, generator=_gen(key + "/cols", base))[:n_ch]
        x[:, cols] *= outlier_scale
    return x.to(torch.float16)


def bias(key: str, N: int, std: float = 0.01, base: int = 0) -> torch.Tensor:
    return normal(key + "/bias", (N,), std, base)


def steer_vec(key: str, N: int, base: int = 0) -> torch.Tensor:
    """fp32 [N] unit-norm direction: g / ||g||_2 with g ~ N(0, 1)."""
    g = torch.randn(N, generator=_gen(key + "/steer", base), dtype=torch.float64)
    return (g / g.norm()).to(torch.float32)


# ------------------------------------------------------------ workloads ---

def tiny_q8():
    """Tiny q8 correctness case: W [256,256] ~N(0,0.02^2), X [64,256] ~N(0,1),
    bias ~N(0,0.01^2), seed base 0."""
    return dict(W=weight("tiny/W", 256, 256), X=activation("tiny", 64, 256),
                bias=bias("tiny", 256))


def q8_block_d1024(name: str, M: int):
    """One linear of the d=1024 block for q8 weight-only: (W [N,K], X [M,K])."""
    K, N = {n: (k, nn) for n, k, nn in D1024}[name]
    return weight(f"q8d1024/{name}", N, K), activation(f"q8d1024/{name}/M{M}", M, K)


def w8a8_d1536(name: str, M: int):
    """One linear of the d=1536 W8A8 case: 1% of input channels scaled x20."""
    K, N = {n: (k, nn) for n, k, nn in D1536}[name]
    return (weight(f"w8a8d1536/{name}", N, K),
            activation(f"w8a8d1536/{name}/M{M}", M, K, outlier_channel_frac=0.01))


def q4_d1536(name: str, M: int):
    """One linear of the d=1536 q4 case: 0.1% of weights redrawn ~N(0,0.2^2)."""
    K, N = {n: (k, nn) for n, k, nn in D1536}[name]
    return (weight(f"q4d1536/{name}", N, K, outlier_frac=0.001),
            activation(f"q4d1536/{name}/M{M}", M, K))


def replay_weight(block: int, name: str) -> torch.Tensor:
    K, N = {n: (k, nn) for n, k, nn in D1536}[name]
    return weight(f"replay/b{block}/{name}", N, K)


def replay_activation(block: int, name: str, M: int = REPLAY_M) -> torch.Tensor:
    K = {n: k for n, k, _ in D1536}[name]
    return activation(f"replay/b{block}/{name}", M, K)


def replay_steer() -> torch.Tensor:
    return steer_vec("replay", 1536)
