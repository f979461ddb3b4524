"""Test/bench harness: seeded inputs for one layer, fed identically to the oracle
and to the library.

The factors, queries and latents come from `synth`; the library receives them
as torch tensors in the layer dtype, and the oracle receives the float64 values
of those same tensors.  Rotated latents are produced by the oracle (the
rotation is a step of the method), rounded once to float32, and then given to
both sides: the library packs them in latent mode, the oracle quantizes them
itself.  No expected value is ever read back from the library.
"""
from __future__ import annotations

import functools
import math

import numpy as np
import torch

from oracle import starkv_oracle as O
from synth import gen

TOL_REL_L2 = 3e-3
TOL_MAX = 1e-2


def tdtype(spec):
    return torch.float32 if spec.dtype == "f32" else torch.bfloat16


def rounded(x: np.ndarray, spec) -> np.ndarray:
    """float64 values of x after conversion to the layer dtype (what the library receives)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(tdtype(spec)).to(torch.float64).numpy()


class Case:
    """One layer with its seeded factors, in the precision the library receives."""

    def __init__(self, spec: gen.LayerSpec, seed: int, layer: int = 0):
        self.spec, self.seed, self.layer = spec, seed, layer
        f = gen.make_factors(spec, seed, layer)
        self.raw = f
        r = functools.partial(rounded, spec=spec)
        self.f = gen.LayerFactors(
            A_k=[r(a) for a in f.A_k] if f.A_k else None, B_k=[r(b) for b in f.B_k] if f.B_k else None,
            A_v=r(f.A_v) if f.A_v is not None else None, B_v=r(f.B_v) if f.B_v is not None else None,
            W_o=r(f.W_o), W_k=r(f.W_k) if f.W_k is not None else None, W_v=r(f.W_v) if f.W_v is not None else None)
        self._B_rot = None

    @property
    def B_rot(self):
        if self._B_rot is None and not self.spec.plain:
            self._B_rot = O.up_projections(self.spec, self.f)
        return self._B_rot

    def rotations(self):
        return [O.rotation(r, self.spec) for r in self.spec.latent_widths]

    # ---- latents ---------------------------------------------------------
    def hidden(self, b: int, T: int, offset: int = 0) -> np.ndarray:
        """bf16/f32-rounded hidden states of sequence b, tokens offset..offset+T-1."""
        return rounded(gen.hidden_states(self.seed, self.layer, b, T, self.spec.hidden, offset), self.spec)

    def latents_from_hidden(self, X: np.ndarray, positions) -> list:
        """Float32 stored-side latents [T, r] per latent from hidden states (oracle projection)."""
        s = self.spec
        if s.plain:
            Z = O.plain_latents(s, self.f, X, positions)
            d = s.head_dim
            return [Z[:, g * d:(g + 1) * d] for g in range(s.n_kv_heads)] + [Z[:, s.n_kv_heads * d:]]
        Rs = self.rotations()
        out = [O.project(X, A, R) for A, R in zip(self.f.A_k, Rs[:-1])]
        out.append(O.project(X, self.f.A_v, Rs[-1]))
        return out

    def latents_direct(self, b: int, T: int, offset: int = 0) -> list:
        """Float32 latents drawn directly (distribution of X A), then rotated by the oracle."""
        s = self.spec
        Rs = self.rotations()
        out = []
        for li, r in enumerate(s.latent_widths[:-1]):
            z = gen.latent_draw(self.seed, self.layer, b, T, self.raw.sigma_k[li][:r], li, offset)
            out.append(O.rotate(z, Rs[li]))
        z = gen.latent_draw(self.seed, self.layer, b, T, self.raw.sigma_v[:s.value_rank], -1, offset)
        out.append(O.rotate(z, Rs[-1]))
        return out

    def stored(self, Z: list) -> list:
        return [O.stored_values_fast(z, z.shape[1], self.spec) for z in Z]

    # ---- oracle ----------------------------------------------------------
    def oracle_decode(self, Zs: list, q: np.ndarray, q_pos: int, seq_len: int) -> np.ndarray:
        s = self.spec
        if s.plain:
            return O.decode_plain(s, self.f, np.concatenate(Zs[:-1], axis=1), Zs[-1], q, seq_len, q_pos)
        return O.decode(s, self.f, Zs, q, q_pos, seq_len, self.B_rot)

    # ---- library ---------------------------------------------------------
    def load(self, dev="cuda", unfused_output=False):
        from decode_attention_rank_b200 import starkv as lib
        s = self.spec
        cfg = lib.LayerConfig.from_spec(s)
        cfg.unfused_output = unfused_output
        dt = tdtype(s)

        def t(x):
            return torch.from_numpy(np.ascontiguousarray(x)).to(dev).to(dt)
        if s.plain:
            return lib.load_factors(cfg, t(self.f.W_k), None, t(self.f.W_v), None, t(self.f.W_o))
        A_k = torch.cat([t(a).reshape(-1) for a in self.f.A_k])
        B_k = torch.cat([t(b).reshape(-1) for b in self.f.B_k])
        L = lib.load_factors(cfg, A_k, B_k, t(self.f.A_v), t(self.f.B_v), t(self.f.W_o))
        torch.cuda.synchronize()
        return L


def queries(case: Case, batch: int, peaky: float = 1.0, n_pos: int = 1) -> np.ndarray:
    s = case.spec
    q = gen.queries(case.seed, case.layer, batch, s.n_heads, s.head_dim, n_pos) * peaky
    return rounded(q, s)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def check_close(got: np.ndarray, want: np.ndarray, what: str = "") -> None:
    e = rel_l2(got, want)
    m = float(np.max(np.abs(got - want)))
    lim = TOL_MAX * float(np.max(np.abs(want)))
    assert e <= TOL_REL_L2 and m <= lim, f"{what}: rel_l2 {e:.3e} (<= {TOL_REL_L2}), max {m:.3e} (<= {lim:.3e})"


class GpuCache:
    """A device pool + page table for a batch of sequences, filled in latent mode."""

    def __init__(self, layer, seq_lens: list, seed: int = 0, extra_pages: int = 3, dev="cuda"):
        self.layer = layer
        self.seq_lens = list(seq_lens)
        pt, n_pages = gen.page_tables(seed, [max(s, 1) for s in seq_lens], 16, extra_pages)
        self.page_table_np = pt
        self.n_pages = n_pages
        self.page_table = torch.from_numpy(pt).to(dev)
        self.pool = torch.empty(n_pages * layer.page_bytes, dtype=torch.uint8, device=dev)
        layer.cache_init(self.pool, n_pages)

    def append_latents(self, b: int, Z: list, start: int = 0, chunk: int = 4096) -> None:
        """Append tokens start.. of sequence b from float32 latents (one [T, r] array per latent)."""
        T = Z[0].shape[0]
        for c0 in range(0, T, chunk):
            n = min(chunk, T - c0)
            zc = np.concatenate([z[c0:c0 + n] for z in Z], axis=1).astype(np.float32)
            zt = torch.from_numpy(zc).cuda()
            seq = torch.full((n,), b, dtype=torch.int32, device="cuda")
            pos = torch.arange(start + c0, start + c0 + n, dtype=torch.int32, device="cuda")
            self.layer.append(self.pool, self.n_pages, self.page_table, seq, pos, zt, True)

    def pool_pages(self) -> np.ndarray:
        torch.cuda.synchronize()
        return self.pool.cpu().numpy().reshape(self.n_pages, -1)
