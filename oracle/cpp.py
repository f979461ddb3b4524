"""ctypes front end of the float64 C++ oracle (oracle/starkv_oracle.cpp).

TEST INFRASTRUCTURE, like the numpy oracle beside it: only the tests, the
package smoke check and the CPU baseline arm of the benchmark use it.  It
shares no code with the CUDA library.  build() compiles the shared library
with g++ (no GPU needed); load() builds it when missing.

The functions take and return numpy arrays with the numpy oracle's shapes
and conventions (see starkv_oracle.py), so the tests can hold the two
implementations equal.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "starkv_oracle.cpp")
LIB = os.path.join(HERE, "liborc.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", "-fno-fast-math",
                        "-ffp-contract=off", "-o", LIB, SRC], check=True)
    return LIB


class _Spec(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("quantized", ctypes.c_int), ("top_fraction", ctypes.c_double),
                ("top_bits", ctypes.c_int), ("bottom_bits", ctypes.c_int), ("group_size", ctypes.c_int),
                ("hadamard", ctypes.c_int), ("rope", ctypes.c_int), ("rope_theta", ctypes.c_double),
                ("page_size", ctypes.c_int)]


_lib = None


def load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        _lib.orc_n_high.argtypes = [ctypes.c_int, ctypes.c_double]
        _lib.orc_groups.argtypes = [ctypes.c_int, ctypes.POINTER(_Spec), P]
        _lib.orc_group_rotation.argtypes = [ctypes.c_int, P]
        _lib.orc_rotation.argtypes = [ctypes.c_int, ctypes.POINTER(_Spec), P]
        _lib.orc_bf16_round.argtypes = [ctypes.c_float]
        _lib.orc_bf16_round.restype = ctypes.c_float
        _lib.orc_fp16_round_up.argtypes = [ctypes.c_float]
        _lib.orc_fp16_round_up.restype = ctypes.c_uint16
        _lib.orc_half_value.argtypes = [ctypes.c_uint16]
        _lib.orc_half_value.restype = ctypes.c_double
        _lib.orc_quantize_group.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P]
        _lib.orc_block_bytes.argtypes = [ctypes.c_int, ctypes.POINTER(_Spec), ctypes.c_int]
        _lib.orc_block_bytes.restype = ctypes.c_size_t
        _lib.orc_pack_block.argtypes = [P, ctypes.c_int, ctypes.POINTER(_Spec), ctypes.c_int, P]
        _lib.orc_stored_values.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.POINTER(_Spec), ctypes.c_int, P]
        _lib.orc_rope.argtypes = [P, ctypes.c_int, ctypes.c_int, P, ctypes.c_double, P]
        _lib.orc_decode.argtypes = [ctypes.POINTER(_Spec), P, P, P, P, ctypes.c_int, P, P, P, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, P]
        _lib.orc_decode_plain.argtypes = [ctypes.POINTER(_Spec), P, P, P, P, ctypes.c_int, ctypes.c_int, P]
    return _lib


def _spec(s) -> _Spec:
    return _Spec(s.hidden, s.n_heads, s.n_kv_heads, s.head_dim, int(bool(s.quantized) and not s.plain),
                 float(s.top_fraction), s.top_bits, s.bottom_bits, s.group_size, int(bool(s.hadamard_block)),
                 int(bool(s.rope)), float(s.rope_theta), s.page_size)


def _p(a: np.ndarray) -> int:
    return a.ctypes.data


def n_high(r: int, top_fraction: float) -> int:
    return load().orc_n_high(r, top_fraction)


def groups(r: int, spec) -> list:
    out = np.zeros(3 * max(r, 1), dtype=np.int32)
    n = load().orc_groups(r, ctypes.byref(_spec(spec)), _p(out))
    return [tuple(int(v) for v in out[3 * k:3 * k + 3]) for k in range(n)]


def group_rotation(n: int) -> np.ndarray:
    out = np.zeros((n, n))
    load().orc_group_rotation(n, _p(out))
    return out


def rotation(r: int, spec) -> np.ndarray:
    out = np.zeros((r, r))
    load().orc_rotation(r, ctypes.byref(_spec(spec)), _p(out))
    return out


def bf16_round(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    f = load().orc_bf16_round
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.float32).reshape(x.shape)


def fp16_round_up(x: float) -> np.float16:
    return np.array([load().orc_fp16_round_up(float(x))], dtype=np.uint16).view(np.float16)[0]


def quantize_group(z, bits: int):
    z = np.ascontiguousarray(np.asarray(z, dtype=np.float32))
    s16 = np.zeros(1, dtype=np.uint16)
    u = np.zeros(max(z.size, 1), dtype=np.uint8)
    if load().orc_quantize_group(_p(z), z.size, bits, _p(s16), _p(u)):
        raise ValueError("scale overflow")
    return s16.view(np.float16)[0], u[:z.size]


def pack_block(Z: np.ndarray, r: int, spec, channel_major: bool = False) -> np.ndarray:
    Z = np.ascontiguousarray(np.asarray(Z, dtype=np.float32))
    sp = _spec(spec)
    out = np.zeros(load().orc_block_bytes(r, ctypes.byref(sp), 2), dtype=np.uint8)
    if load().orc_pack_block(_p(Z), r, ctypes.byref(sp), int(channel_major), _p(out)):
        raise ValueError("scale overflow")
    return out


def stored_values(Z: np.ndarray, r: int, spec) -> np.ndarray:
    Z = np.ascontiguousarray(np.asarray(Z, dtype=np.float32))
    out = np.zeros(Z.shape, dtype=np.float64)
    es = 4 if spec.dtype == "f32" else 2
    if load().orc_stored_values(_p(Z), Z.shape[0], r, ctypes.byref(_spec(spec)), es, _p(out)):
        raise ValueError("scale overflow")
    return out


def rope(x: np.ndarray, pos, theta: float) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    d = x.shape[-1]
    flat = x.reshape(-1, d)
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.float64), x.shape[:-1]).reshape(-1))
    out = np.zeros_like(flat)
    load().orc_rope(_p(flat), flat.shape[0], d, _p(p), theta, _p(out))
    return out.reshape(x.shape)


def up_projections(spec, f) -> list:
    """B' = R^T B per key latent, then for the value latent, with this library's rotation."""
    out = [rotation(r, spec).T @ np.asarray(B, dtype=np.float64) for r, B in zip(spec.key_ranks, f.B_k)]
    out.append(rotation(spec.value_rank, spec).T @ np.asarray(f.B_v, dtype=np.float64))
    return out


def decode(spec, f, Zhat, q, q_pos: int, seq_len: int, B_rot=None, threads: int = 0) -> np.ndarray:
    """Decode attention output [D] of one sequence (the numpy oracle's `decode`, same arguments;
    B_rot = the rotated up-projections [B'_k,0 .. B'_k,Hkv-1, B'_v], built here when absent)."""
    lib = load()
    if B_rot is None:
        B_rot = up_projections(spec, f)
    sp = _spec(spec)
    Hkv = spec.n_kv_heads
    zk = [np.ascontiguousarray(np.asarray(z, dtype=np.float64)[:seq_len]) for z in Zhat[:Hkv]]
    bk = [np.ascontiguousarray(np.asarray(b, dtype=np.float64)) for b in B_rot[:Hkv]]
    zv = np.ascontiguousarray(np.asarray(Zhat[-1], dtype=np.float64)[:seq_len])
    bv = np.ascontiguousarray(np.asarray(B_rot[-1], dtype=np.float64))
    wo = np.ascontiguousarray(np.asarray(f.W_o, dtype=np.float64))
    qq = np.ascontiguousarray(np.asarray(q, dtype=np.float64))
    ranks = np.array([b.shape[0] for b in bk], dtype=np.int32)
    zk_ptrs = (ctypes.c_void_p * Hkv)(*[_p(z) for z in zk])
    bk_ptrs = (ctypes.c_void_p * Hkv)(*[_p(b) for b in bk])
    out = np.zeros(spec.hidden)
    n_threads = threads or len(os.sched_getaffinity(0))
    lib.orc_decode(ctypes.byref(sp), _p(ranks), ctypes.cast(zk_ptrs, ctypes.c_void_p),
                   ctypes.cast(bk_ptrs, ctypes.c_void_p), _p(zv), zv.shape[1], _p(bv), _p(wo), _p(qq), q_pos,
                   seq_len, n_threads, _p(out))
    return out


def decode_plain(spec, f, Khat, Vhat, q, seq_len: int, q_pos: int) -> np.ndarray:
    lib = load()
    K = np.ascontiguousarray(np.asarray(Khat, dtype=np.float64)[:seq_len])
    V = np.ascontiguousarray(np.asarray(Vhat, dtype=np.float64)[:seq_len])
    wo = np.ascontiguousarray(np.asarray(f.W_o, dtype=np.float64))
    qq = np.ascontiguousarray(np.asarray(q, dtype=np.float64))
    out = np.zeros(spec.hidden)
    lib.orc_decode_plain(ctypes.byref(_spec(spec)), _p(K), _p(V), _p(wo), _p(qq), q_pos, seq_len, _p(out))
    return out
