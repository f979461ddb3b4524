"""Seeded synthetic inputs for STAR-KV latent decode attention.

This module holds no step of the method: no projection, rotation, quantizer,
page format, RoPE or attention.  It draws random numbers and random
orthonormal frames, and builds the factor matrices that the workload
definitions prescribe (a truncated SVD with a known spectrum), so that both the
oracle and the CUDA path start from identical inputs.

Random numbers come from a counter-based SplitMix64 (Steele, Lea & Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014): output i of a
stream with key k is mix64(k + (i + 1) * 0x9E3779B97F4A7C15).  Uniforms take
the top 53 bits; normals use the Box-Muller transform on pairs of uniforms.
Every tensor has its own stream, keyed by (seed, tensor id, layer, index), so a
sub-range of a tensor (one sequence, one head) can be drawn without drawing the
rest.

Workload shapes follow the STAR-KV pages: a LongChat-7B / LLaMA-2-7B attention
layer (32 heads, head_dim 128, hidden 4096) and a LLaMA-3-8B GQA layer
(32 query heads, 8 KV heads), key ranks with mean 32 (75 % of the channels
removed, "STAR-KV 阅读笔记" section 2.1 and section 8), a joint value rank, and
singular values sigma_i = i^-0.8.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Tensor ids used to key the random streams.
T_RANKS, T_UK, T_VK, T_UV, T_VV, T_WO, T_X, T_Q, T_ZK, T_ZV, T_PERM, T_LEN, T_WK, T_WV = range(14)


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor: int, layer: int = 0, index: int = 0) -> np.uint64:
    """Derive a 64-bit stream key from (seed, tensor id, layer, index)."""
    k = np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    for part in (tensor, layer, index):
        k = _mix(k + np.array([part + 1], dtype=np.uint64) * _GOLDEN)
    return k[0]


def raw64(key: np.uint64, n: int, offset: int = 0) -> np.ndarray:
    i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
    return _mix(np.array([key], dtype=np.uint64) + i * _GOLDEN)


def uniforms(key: np.uint64, n: int, offset: int = 0) -> np.ndarray:
    """n uniforms in [0, 1), 53-bit resolution."""
    return (raw64(key, n, offset) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normals(key: np.uint64, n: int, offset: int = 0) -> np.ndarray:
    """n standard normals (Box-Muller on consecutive uniform pairs)."""
    # normal 2j (2j+1) is the cosine (sine) output of uniform pair (2j, 2j+1)
    lead = offset % 2
    m = (n + lead + 1) // 2
    u = uniforms(key, 2 * m, offset - lead)
    r = np.sqrt(-2.0 * np.log1p(-u[0::2]))  # 1-u in (0, 1]
    a = 2.0 * math.pi * u[1::2]
    out = np.empty(2 * m)
    out[0::2] = r * np.cos(a)
    out[1::2] = r * np.sin(a)
    return out[lead:lead + n]


def haar_frame(key: np.uint64, rows: int, cols: int) -> np.ndarray:
    """rows x cols matrix with orthonormal columns, Haar distributed.

    Householder QR (LAPACK) of a Gaussian matrix, with the signs fixed so that
    diag(R) > 0, which makes the frame exactly Haar.
    """
    g = normals(key, rows * cols).reshape(rows, cols)
    q, r = np.linalg.qr(g)
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    return q * s


def spectrum(n: int, power: float = 0.8) -> np.ndarray:
    return np.arange(1, n + 1, dtype=np.float64) ** (-power)


def ragged_ranks(seed: int, layer: int, n_kv: int, mean: int = 32, lo: int = 16, hi: int = 64,
                 step: int = 8) -> list[int]:
    """Key ranks per KV head: uniform on {lo, lo+step, ..., hi}, rescaled to the mean.

    r_h = step * round_half_up(r~_h * mean * n_kv / sum(r~) / step), clamped to
    [lo, hi]; then the sum is forced to mean * n_kv by moving the largest
    (lowest index first) down, or the smallest up, one step at a time.
    """
    grid = np.arange(lo, hi + 1, step)
    u = uniforms(stream_key(seed, T_RANKS, layer), n_kv)
    raw = grid[np.minimum((u * len(grid)).astype(np.int64), len(grid) - 1)].astype(np.float64)
    target = mean * n_kv
    r = [int(step * math.floor(x * target / raw.sum() / step + 0.5)) for x in raw]
    r = [min(max(x, lo), hi) for x in r]
    while sum(r) > target:
        i = max(range(n_kv), key=lambda j: (r[j], -j))
        if r[i] - step < lo:
            break
        r[i] -= step
    while sum(r) < target:
        i = min(range(n_kv), key=lambda j: (r[j], j))
        if r[i] + step > hi:
            break
        r[i] += step
    return r


@dataclasses.dataclass
class LayerSpec:
    """Shape and storage options of one attention layer."""
    hidden: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    key_ranks: list
    value_rank: int
    dtype: str = "bf16"          # "f32" or "bf16": factors, unquantized latents, q, out
    quantized: bool = False
    top_fraction: float = 0.25
    top_bits: int = 4
    bottom_bits: int = 3
    group_size: int = 32
    hadamard_block: int = 0       # 0 = off, else equal to group_size
    rope: bool = False
    rope_theta: float = 10000.0
    page_size: int = 16
    plain: bool = False           # uncompressed layer (plain K/V, K stored post-RoPE)

    @property
    def latent_widths(self) -> list:
        """Widths of the stored latents of one token: keys per KV head, then values."""
        if self.plain:
            return [self.head_dim] * self.n_kv_heads + [self.n_kv_heads * self.head_dim]
        return list(self.key_ranks) + [self.value_rank]


@dataclasses.dataclass
class LayerFactors:
    """Unrotated factors of one layer, float64.

    Keys (per KV head h): A_k[h] D x r_h, B_k[h] r_h x d.
    Values (joint):       A_v D x r_v,    B_v r_v x (H_kv d).
    Output projection:    W_o (H d) x D.
    Plain layers use W_k, W_v (D x H_kv d) instead of the factors.
    """
    A_k: list = None
    B_k: list = None
    A_v: np.ndarray = None
    B_v: np.ndarray = None
    W_o: np.ndarray = None
    W_k: np.ndarray = None
    W_v: np.ndarray = None
    sigma_k: list = None
    sigma_v: np.ndarray = None


def make_factors(spec: LayerSpec, seed: int, layer: int = 0, power: float = 0.8) -> LayerFactors:
    """Truncated-SVD factors A = U_r diag(sigma_r), B = V_r^T of matrices with
    Gaussian (Haar) singular vectors and spectrum sigma_i = i^-power."""
    D, d, Hkv, H = spec.hidden, spec.head_dim, spec.n_kv_heads, spec.n_heads
    f = LayerFactors()
    f.W_o = normals(stream_key(seed, T_WO, layer), H * d * D).reshape(H * d, D) / math.sqrt(D)
    if spec.plain:
        sig = spectrum(d, power)
        wk, wv = [], []
        for h in range(Hkv):
            U = haar_frame(stream_key(seed, T_UK, layer, h), D, d)
            V = haar_frame(stream_key(seed, T_VK, layer, h), d, d)
            wk.append((U * sig) @ V.T)
            U = haar_frame(stream_key(seed, T_UV, layer, h), D, d)
            V = haar_frame(stream_key(seed, T_VV, layer, h), d, d)
            wv.append((U * sig) @ V.T)
        f.W_k = np.concatenate(wk, axis=1)
        f.W_v = np.concatenate(wv, axis=1)
        return f
    f.A_k, f.B_k, f.sigma_k = [], [], []
    sig = spectrum(d, power)
    for h, r in enumerate(spec.key_ranks):
        U = haar_frame(stream_key(seed, T_UK, layer, h), D, d)
        V = haar_frame(stream_key(seed, T_VK, layer, h), d, d)
        f.A_k.append(U[:, :r] * sig[:r])
        f.B_k.append(V[:, :r].T.copy())
        f.sigma_k.append(sig)
    rv = spec.value_rank
    sv = spectrum(min(D, Hkv * d), power)
    U = haar_frame(stream_key(seed, T_UV, layer), D, rv)
    V = haar_frame(stream_key(seed, T_VV, layer), Hkv * d, rv)
    f.A_v = U * sv[:rv]
    f.B_v = V.T.copy()
    f.sigma_v = sv
    return f


def hidden_states(seed: int, layer: int, seq: int, n_tokens: int, hidden: int, offset: int = 0) -> np.ndarray:
    """Activations X ~ N(0, 1), [n_tokens, hidden], for tokens offset.. of one sequence."""
    key = stream_key(seed, T_X, layer, seq)
    return normals(key, n_tokens * hidden, offset * hidden).reshape(n_tokens, hidden)


def latent_draw(seed: int, layer: int, seq: int, n_tokens: int, sigmas: np.ndarray, latent: int,
                offset: int = 0) -> np.ndarray:
    """Unrotated latents drawn directly, [n_tokens, r]: column j ~ N(0, sigma_j^2).

    For X ~ N(0, I) and A = U_r diag(sigma_r) with orthonormal U_r, the latents
    X A are independent N(0, sigma_j^2) per column; this draws that
    distribution without the D-dimensional activations, for long contexts.
    """
    r = len(sigmas)
    key = stream_key(seed, T_ZK if latent >= 0 else T_ZV, layer, seq * 4096 + max(latent, 0))
    return normals(key, n_tokens * r, offset * r).reshape(n_tokens, r) * sigmas[None, :]


def queries(seed: int, layer: int, batch: int, n_heads: int, head_dim: int, n_pos: int = 1) -> np.ndarray:
    """q ~ N(0, 1) / sqrt(d): [batch, n_pos, n_heads, head_dim] (n_pos = 1 for decode)."""
    q = normals(stream_key(seed, T_Q, layer), batch * n_pos * n_heads * head_dim)
    return q.reshape(batch, n_pos, n_heads, head_dim) / math.sqrt(head_dim)


def page_tables(seed: int, seq_lens: list, page_size: int, extra_pages: int = 0):
    """Seeded random assignment of physical pages to sequences.

    Returns (page_table [B, max_pages] int32, n_pages).  Unused entries hold -1.
    """
    need = [(s + page_size - 1) // page_size for s in seq_lens]
    n_pages = sum(need) + extra_pages
    u = uniforms(stream_key(seed, T_PERM), n_pages)
    perm = np.argsort(u, kind="stable").astype(np.int32)
    max_pages = max(max(need), 1)
    pt = np.full((len(seq_lens), max_pages), -1, dtype=np.int32)
    k = 0
    for b, n in enumerate(need):
        pt[b, :n] = perm[k:k + n]
        k += n
    return pt, n_pages


# ---------------------------------------------------------------------------
# The five workload definitions.
# ---------------------------------------------------------------------------

LAYER_SEED = {0: 0, 1: 1, 2: 1, 3: 3, 4: 4}


def config_spec(cfg: int, quantized: bool | None = None, layer: int = 2, seed: int | None = None) -> LayerSpec:
    """LayerSpec of workload `cfg` (0..4).

    Seeds: workload k uses seed k, except that workload 2 is the layer of
    workload 1 (seed 1) with rotation and quantization added.
    """
    seed = LAYER_SEED[cfg] if seed is None else seed
    if cfg == 0:
        return LayerSpec(hidden=256, n_heads=4, n_kv_heads=4, head_dim=64, key_ranks=[8, 16, 16, 24],
                         value_rank=64, dtype="f32")
    if cfg == 1:
        return LayerSpec(hidden=4096, n_heads=32, n_kv_heads=32, head_dim=128,
                         key_ranks=ragged_ranks(seed, 0, 32), value_rank=1024, dtype="bf16",
                         rope=True, rope_theta=10000.0)
    if cfg == 2:
        return LayerSpec(hidden=4096, n_heads=32, n_kv_heads=32, head_dim=128,
                         key_ranks=ragged_ranks(seed, 0, 32), value_rank=1024, dtype="bf16",
                         quantized=True, hadamard_block=32, rope=True, rope_theta=10000.0)
    if cfg == 3:
        q = bool(quantized)
        return LayerSpec(hidden=4096, n_heads=32, n_kv_heads=8, head_dim=128,
                         key_ranks=ragged_ranks(seed, 0, 8), value_rank=256, dtype="bf16",
                         quantized=q, hadamard_block=32 if q else 0, rope=True, rope_theta=500000.0)
    if cfg == 4:
        if layer in (0, 1, 31):
            return LayerSpec(hidden=4096, n_heads=32, n_kv_heads=32, head_dim=128, key_ranks=[128] * 32,
                             value_rank=4096, dtype="bf16", rope=True, rope_theta=10000.0, plain=True)
        return LayerSpec(hidden=4096, n_heads=32, n_kv_heads=32, head_dim=128,
                         key_ranks=ragged_ranks(seed + layer, layer, 32), value_rank=1024, dtype="bf16",
                         quantized=True, hadamard_block=32, rope=True, rope_theta=10000.0)
    raise ValueError(cfg)


CONFIG_SHAPES = {
    0: dict(batch=1, ctx=256),
    1: dict(batch=16, ctx=4096),
    2: dict(batch=16, ctx=32768),
    3: dict(batch=64, ctx=8192),
    4: dict(batch=16, ctx=32768, prefill=4096, chunk=1024),
}
