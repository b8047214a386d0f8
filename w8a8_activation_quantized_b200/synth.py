"""Seeded synthetic inputs shaped like the workloads on the Cider pages.

This module holds no step of the method: it draws activations and fp32
weights and nothing else.  Both the CUDA path's tests/benchmark and the CPU
oracle take their inputs from here, so the two sides see the same numbers.

Recipe (stand-ins for an LLM layer's hidden states and trained weights; no
dataset or checkpoint is used):

* activations ``x[M, K]``: i.i.d. N(0, 1) in fp32, then a fixed set of
  ``round(frac * K)`` input channels (drawn once per (K, seed) and shared by
  every M) is multiplied by ``outlier_scale`` -- the outlier channels the
  juejin post describes in section "Outlier 问题：激活量化的核心难点" -- and
  the result is rounded to fp16 (or bf16);
* weights ``W[N, K]``: i.i.d. N(0, std) in fp32, quantized later by whoever
  consumes them.

All draws use numpy's PCG64 with an explicit seed.
"""
import numpy as np


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def outlier_channels(K: int, frac: float, seed: int) -> np.ndarray:
    """Sorted indices of the ``round(frac*K)`` outlier input channels."""
    n = int(round(frac * K))
    if n == 0:
        return np.zeros((0,), np.int64)
    return np.sort(_rng(seed * 7919 + 17).choice(K, size=n, replace=False))


def activations_f32(M: int, K: int, seed: int, outlier_frac: float = 0.01,
                    outlier_scale: float = 50.0, channel_seed: int = None) -> np.ndarray:
    x = _rng(seed).standard_normal((M, K), dtype=np.float32)
    idx = outlier_channels(K, outlier_frac, seed if channel_seed is None else channel_seed)
    if idx.size:
        x[:, idx] *= np.float32(outlier_scale)
    return x


def activations(M: int, K: int, seed: int, outlier_frac: float = 0.01,
                outlier_scale: float = 50.0, dtype: str = "f16",
                channel_seed: int = None) -> np.ndarray:
    """fp16 array (dtype='f16') or bf16 bit patterns as uint16 (dtype='bf16')."""
    x = activations_f32(M, K, seed, outlier_frac, outlier_scale, channel_seed)
    if dtype == "f16":
        return x.astype(np.float16)
    if dtype == "bf16":
        import torch
        return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(dtype)


def weights(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    """fp32 [N, K] ~ N(0, std)."""
    return _rng(seed + 1_000_003).normal(0.0, std, size=(N, K)).astype(np.float32)


def weights_device(N: int, K: int, seed: int, std: float = 0.02, device="cuda"):
    """fp32 [N, K] ~ N(0, std) drawn on `device` by torch's seeded generator
    (for weight sets too large to draw on the host; the same seed and device
    give the same numbers, which a CPU check can copy back)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std


# Named workloads (sizes of the Cider single-op tables and of an 8B-class
# decoder's linear stack).  Each entry: kind, M list, N, K, extra.
WORKLOADS = {
    "pc_small": dict(kind="pc", M=[16], N=128, K=256, outlier_frac=0.0),
    "pc_n10240_k2560": dict(kind="pc", M=[1, 128, 1024, 4096, 8192], N=10240, K=2560,
                            outlier_frac=0.01, outlier_scale=50.0),
    "pg_n2560_k10240": dict(kind="pg", M=[1, 128, 1024, 4096, 8192], N=2560, K=10240,
                            gs=[128, 64], outlier_frac=0.01, outlier_scale=50.0),
    "w4a8_n12288_k4096": dict(kind="w4a8", M=[2048], N=12288, K=4096, gs=[64],
                              outlier_frac=0.01, outlier_scale=50.0),
    "stack_8b_m2048": dict(kind="stack", M=[2048], layers=36, hidden=4096, kv=1024,
                           ffn=12288, outlier_frac=0.005, outlier_scale=100.0),
}


def seed_for(workload_index: int, M: int) -> int:
    """Seed = workload index * 1000 + M."""
    return workload_index * 1000 + M
