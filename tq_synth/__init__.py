"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and bench.py.

This module holds no step of the quantization method: it only draws random
numbers (a Haar rotation, a Gaussian sketch matrix, key/value/query tensors
shaped like the workloads on the pages). Both the CUDA path and the float64
oracle receive exactly the tensors produced here.

Every generator takes an explicit seed; tensors are produced with
``torch.Generator`` (CPU by default, or on a CUDA device for the large
workloads, whose sampled rows are then copied to the host for the oracle).
"""

from __future__ import annotations

import dataclasses

import torch

SEED_DATA = 0
SEED_PI = 1
SEED_S = 2
SEED_OUTLIERS = 3


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def rotation(d: int, seed: int = SEED_PI) -> torch.Tensor:
    """Haar-random orthogonal d x d matrix (QR of a seeded Gaussian, column signs
    fixed by sign(diag R)), rounded to float32 on the CPU."""
    a = torch.randn(d, d, generator=_gen(seed), dtype=torch.float64)
    q, r = torch.linalg.qr(a)
    q = q * torch.sign(torch.diagonal(r))[None, :]
    return q.to(torch.float32).contiguous()


def hadamard_signs(d: int, seed: int = SEED_PI) -> torch.Tensor:
    """The seeded random signs s (+-1, float32, CPU) of `randomized_hadamard(d, seed)`."""
    if d < 1 or d & (d - 1):
        raise ValueError(f"d={d} is not a power of two")
    return torch.where(torch.rand(d, generator=_gen(seed), dtype=torch.float64) < 0.5, -1.0, 1.0).to(torch.float32)


def randomized_hadamard(d: int, seed: int = SEED_PI) -> torch.Tensor:
    """Structured orthogonal d x d matrix H diag(s) / sqrt(d): H the Sylvester-Hadamard matrix
    (H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]]), s = `hadamard_signs(d, seed)`; d a power of two.
    Float32 on the CPU; an alternative to `rotation` for the rotation input."""
    s = hadamard_signs(d, seed).to(torch.float64)
    h = torch.ones(1, 1, dtype=torch.float64)
    while h.shape[0] < d:
        h = torch.cat([torch.cat([h, h], 1), torch.cat([h, -h], 1)], 0)
    return (h * s[None, :] / d ** 0.5).to(torch.float32).contiguous()


def sketch(d: int, seed: int = SEED_S) -> torch.Tensor:
    """d x d matrix with i.i.d. N(0, 1) entries, float32 on the CPU."""
    return torch.randn(d, d, generator=_gen(seed), dtype=torch.float32)


def gaussian(shape, seed: int, dtype=torch.float32, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(*shape, generator=g, dtype=torch.float32, device=device).to(dtype)


def outlier_channels(n_heads: int, d: int, k: int = 4, seed: int = SEED_OUTLIERS) -> torch.Tensor:
    """[n_heads, k] distinct channel indices per head (drawn in head order)."""
    g = _gen(seed)
    return torch.stack([torch.randperm(d, generator=g)[:k] for _ in range(n_heads)])


def with_outliers(x: torch.Tensor, channels: torch.Tensor, factor: float = 8.0) -> torch.Tensor:
    """Scale the given channels of each head by `factor`. x: [B, H, T, d] (float32)."""
    scale = torch.ones(x.shape[1], x.shape[3], dtype=x.dtype, device=x.device)
    rows = torch.arange(x.shape[1]).repeat_interleave(channels.shape[1])
    scale[rows, channels.reshape(-1).to(torch.long)] = factor
    return x * scale[None, :, None, :]


def lognormal_sphere(shape, seed: int, sigma: float = 0.5, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """Vectors with norms ~ lognormal(0, sigma) and Haar-uniform directions."""
    g = _gen(seed, device)
    z = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
    z = z / z.norm(dim=-1, keepdim=True)
    r = torch.exp(sigma * torch.randn(*shape[:-1], 1, generator=g, dtype=torch.float32, device=device))
    return (z * r).to(dtype)


def anisotropic_unit(n: int, d: int, seed_sigma: int, seed_x: int, device="cpu") -> torch.Tensor:
    """Unit-normalised rows of N(0, diag(sigma^2)), sigma_k ~ U[0.2, 2] (float32)."""
    sig = 0.2 + 1.8 * torch.rand(d, generator=_gen(seed_sigma), dtype=torch.float32)
    x = torch.randn(n, d, generator=_gen(seed_x, device), dtype=torch.float32, device=device) * sig.to(device)
    return x / x.norm(dim=1, keepdim=True)


# ----------------------------------------------------------------------------
# the workloads
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_seq: int
    n_q_heads: int
    n_kv_heads: int
    d: int
    n_tokens: int
    k_bits: int          # total bits per key coordinate (bits-1 index bits + 1 QJL bit)
    v_bits: int          # index bits per value coordinate (MSE only)
    dtype: torch.dtype

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


PR1 = Workload("pr1-d128-4096keys-16q-b3", 1, 16, 1, 128, 4096, 3, 3, torch.float32)
LLAMA = Workload("llama3-8b-decode-32k-b3", 1, 32, 8, 128, 32768, 3, 3, torch.bfloat16)


def sweep(bits: int) -> Workload:
    return Workload(f"bsweep-b{bits}-8x8x131072", 8, 8, 8, 128, 131072, bits, bits, torch.bfloat16)


def pr1_inputs():
    """PR1: 4096 keys and 16 queries, d=128, fp32 N(0,1) from seed 0 (queries are
    the next 16 rows of the same stream). Values are the following 4096 rows."""
    rows = gaussian((4096 + 16 + 4096, 128), SEED_DATA)
    keys = rows[:4096].reshape(1, 1, 4096, 128)
    q = rows[4096:4112].reshape(1, 16, 128)
    v = rows[4112:].reshape(1, 1, 4096, 128)
    return keys, v, q


def llama_inputs(n_tokens: int = 32768, device="cpu", seed: int = SEED_DATA):
    """Llama-3-8B-shaped decode: K, V [1, 8, T, 128] bf16 N(0,1) with 4 outlier
    channels per head scaled x8 (same channels for K and V), q [1, 32, 128] fp32."""
    ch = outlier_channels(8, 128)
    k = with_outliers(gaussian((1, 8, n_tokens, 128), seed, device=device), ch.to(device)).to(torch.bfloat16)
    v = with_outliers(gaussian((1, 8, n_tokens, 128), seed + 100, device=device), ch.to(device)).to(torch.bfloat16)
    q = gaussian((1, 32, 128), seed + 200, device=device)
    return k, v, q


def sweep_inputs(n_seq: int = 8, n_heads: int = 8, n_tokens: int = 131072, d: int = 128, device="cpu", seed: int = SEED_DATA):
    """b-sweep: K, V [B, H, T, d] bf16 with lognormal(0, 0.5) norms times Haar
    directions; one fp32 N(0,1) query per KV head."""
    k = lognormal_sphere((n_seq, n_heads, n_tokens, d), seed, device=device)
    v = lognormal_sphere((n_seq, n_heads, n_tokens, d), seed + 100, device=device)
    q = gaussian((n_seq, n_heads, d), seed + 200, device=device)
    return k, v, q


def large_layer_inputs(layer: int, n_heads: int = 128, n_tokens: int = 131072, d: int = 128, device="cpu"):
    """One layer of the large-model cache: K, V [1, H, T, d] fp16 N(0,1) with
    4 outlier channels per head x8; one fp32 query per head."""
    ch = outlier_channels(n_heads, d)
    base = 1000 + 10 * layer
    k = with_outliers(gaussian((1, n_heads, n_tokens, d), base, device=device), ch.to(device)).to(torch.float16)
    v = with_outliers(gaussian((1, n_heads, n_tokens, d), base + 1, device=device), ch.to(device)).to(torch.float16)
    q = gaussian((1, n_heads, d), base + 2, device=device)
    return k, v, q


def nn_inputs(n_db: int = 1_000_000, n_q: int = 10_000, d: int = 200, device="cpu"):
    """Nearest-neighbour stand-in: database and queries drawn from one anisotropic
    Gaussian law (per-dimension std ~ U[0.2, 2], seed 10), unit-normalised."""
    db = anisotropic_unit(n_db, d, 10, 11, device=device)
    qs = anisotropic_unit(n_q, d, 10, 12, device=device)
    return db, qs

