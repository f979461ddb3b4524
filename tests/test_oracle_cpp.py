"""The float64 C++ oracle (oracle/starkv_oracle.cpp) against the same pins as the numpy oracle, and
the two oracles against each other.

The C++ oracle is an independent restatement of the same plain definitions ("STAR-KV 阅读笔记"
sections 2.2, 5.1-5.3, 6.1 and Algorithm 2); it exists so the CPU baseline can run the method's
arithmetic in compiled code on all host cores.  Its pins here do not go through the numpy oracle:
golden bytes, scipy's Hadamard matrices, torch's bf16 cast, exhaustive fp16 enumeration, closed
forms for tiny attention.  The cross-checks then hold it equal to the numpy oracle on seeded cases.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import cpp as C
from oracle import starkv_oracle as O
from synth import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_spec(**kw):
    base = dict(hidden=32, n_heads=2, n_kv_heads=2, head_dim=8, key_ranks=[3, 5], value_rank=6, dtype="f32")
    base.update(kw)
    return gen.LayerSpec(**base)


def _read_golden(name):
    meta, hexes = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            if k == "hex":
                hexes.append((int(v[0]), [int(x, 16) for x in v[1:]]))
            else:
                meta[k] = v
    return meta, hexes


# ---------------------------------------------------------------------------
# Pins (nothing here calls the numpy oracle)
# ---------------------------------------------------------------------------

def test_cpp_bf16_round_matches_torch():
    x = (gen.normals(gen.stream_key(5, 91), 4000) * 10.0 ** np.arange(-3, 3).repeat(667)[:4000]).astype(np.float32)
    x = np.concatenate([x, np.array([0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -9)], dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(C.bf16_round(x), ref)


def test_cpp_fp16_round_up_brute_force():
    halves = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    xs = np.concatenate([gen.uniforms(gen.stream_key(1, 92), 2000) * 70000.0 * (gen.uniforms(gen.stream_key(2, 92), 2000) ** 6),
                         halves[::211].astype(np.float64), [1e-9, 6e-8, 65504.0]]).astype(np.float32)
    for x in xs[xs <= 65504.0]:
        assert np.float32(C.fp16_round_up(x)) == halves[np.searchsorted(halves, x, side="left")], x


@pytest.mark.parametrize("bits", [3, 4])
def test_cpp_quantizer_error_bound_and_grid(bits):
    qmax = 2 ** (bits - 1) - 1
    z = (gen.normals(gen.stream_key(3, 93, bits), 32 * 200) * 3.0).astype(np.float32).reshape(200, 32)
    for row in z:
        s16, u = C.quantize_group(row, bits)
        s = float(s16)
        assert s >= np.max(np.abs(row)) / qmax * (1 - 1e-7)            # the scale is rounded up
        zh = (u.astype(np.float64) - 2 ** (bits - 1)) * s
        assert np.all(u >= 1) and np.all(u <= 2 * qmax + 1)              # symmetric grid, offset binary
        assert np.max(np.abs(zh - row)) <= s / 2 * (1 + 1e-6)            # half a step
    s16, u = C.quantize_group(np.zeros(32, np.float32), bits)
    assert float(s16) == 0.0 and np.all(u == 2 ** (bits - 1))
    with pytest.raises(ValueError):
        C.quantize_group(np.array([1e9] + [0.0] * 31, np.float32), bits)


def test_cpp_hadamard_golden_and_rotation_assembly():
    import scipy.linalg as sl
    rows = []
    with open(os.path.join(GOLDEN, "hadamard_6.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            rows.append([float(x) / float(parts[1]) for x in parts[3:]])
    np.testing.assert_allclose(C.group_rotation(6), np.array(rows), atol=1e-15)

    def sylv(n):
        return sl.hadamard(n) / math.sqrt(n)
    spec = gen.LayerSpec(hidden=1, n_heads=1, n_kv_heads=1, head_dim=128, key_ranks=[20], value_rank=20,
                         quantized=True, hadamard_block=32)
    assert C.n_high(20, 0.25) == 5 and C.n_high(56, 0.25) == 14 and C.n_high(1024, 0.25) == 256
    np.testing.assert_allclose(C.rotation(20, spec), sl.block_diag(sylv(4), sylv(1), sylv(8), sylv(4), sylv(2), sylv(1)),
                               atol=1e-15)
    np.testing.assert_allclose(C.rotation(56, spec), sl.block_diag(sylv(8), sylv(4), sylv(2), sylv(32), sylv(8), sylv(2)),
                               atol=1e-15)
    np.testing.assert_array_equal(C.rotation(20, gen.LayerSpec(**{**spec.__dict__, "hadamard_block": 0})), np.eye(20))
    assert C.groups(56, spec) == [(0, 14, 4), (14, 32, 3), (46, 10, 3)]


@pytest.mark.parametrize("name,cmajor,n_slots", [("pack_r6_two_slots.txt", False, 2),
                                                 ("pack_value_r4_three_slots.txt", True, 3)])
def test_cpp_pack_block_golden_bytes(name, cmajor, n_slots):
    meta, hexes = _read_golden(name)
    r = int(meta["r"][0])
    spec = gen.LayerSpec(hidden=1, n_heads=1, n_kv_heads=1, head_dim=8, key_ranks=[r], value_rank=r,
                         quantized=True, top_fraction=float(meta["top_fraction"][0]))
    Z = np.full((16, r), np.nan, dtype=np.float32)
    for s in range(n_slots):
        Z[s] = [float(x) for x in meta[f"slot{s}"]]
    want = np.zeros(int(meta["bytes"][0]), dtype=np.uint8)
    for off, bs in hexes:
        want[off:off + len(bs)] = bs
    np.testing.assert_array_equal(C.pack_block(Z, r, spec, channel_major=cmajor), want)


def test_cpp_rope_closed_form():
    # pair (p, p + d/2) rotated by pos * theta^(-2p/d); norms kept; relative-position invariance
    d = 8
    x = gen.normals(gen.stream_key(4, 94), d)
    y = C.rope(x, 3.0, 10000.0)
    for p in range(d // 2):
        a = 3.0 * 10000.0 ** (-2 * p / d)
        np.testing.assert_allclose(y[p], x[p] * math.cos(a) - x[p + d // 2] * math.sin(a), rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(y[p + d // 2], x[p + d // 2] * math.cos(a) + x[p] * math.sin(a), rtol=1e-14, atol=1e-15)
    k = gen.normals(gen.stream_key(5, 94), d)
    np.testing.assert_allclose(C.rope(x, 7.0, 1e4) @ C.rope(k, 2.0, 1e4), C.rope(x, 15.0, 1e4) @ C.rope(k, 10.0, 1e4),
                               rtol=1e-12)


def test_cpp_decode_brute_force_tiny():
    spec = gen.LayerSpec(hidden=2, n_heads=1, n_kv_heads=1, head_dim=4, key_ranks=[1], value_rank=1, dtype="f32")
    f = gen.LayerFactors(A_k=[None], B_k=[np.array([[1.0, 0, 0, 0]])], A_v=None,
                         B_v=np.array([[0.0, 2.0, 0, 0]]), W_o=np.array([[1.0, 0], [0, 3.0], [0, 0], [0, 0]]))
    Zh = [np.array([[2.0], [-1.0]]), np.array([[1.0], [5.0]])]
    out = C.decode(spec, f, Zh, np.array([[1.5, 0, 0, 0]]), 1, 2)
    p0 = 1.0 / (1.0 + math.exp(1.5 * -1.0 / 2.0 - 1.5 * 2.0 / 2.0))
    y = p0 * np.array([0, 2.0, 0, 0]) + (1 - p0) * np.array([0, 10.0, 0, 0])
    np.testing.assert_allclose(out, [y[0], 3.0 * y[1]], rtol=1e-14)


def test_cpp_gqa_head_map_brute_force():
    # H = 4 over H_kv = 2, contiguous groups kv(h) = h // 2; identity up-projections, W_o,h = (h + 1) I
    spec = gen.LayerSpec(hidden=2, n_heads=4, n_kv_heads=2, head_dim=2, key_ranks=[2, 2], value_rank=4, dtype="f32")
    Wo = np.zeros((8, 2))
    for h in range(4):
        Wo[2 * h:2 * h + 2] = (h + 1) * np.eye(2)
    f = gen.LayerFactors(A_k=[None, None], B_k=[np.eye(2), np.eye(2)], A_v=None, B_v=np.eye(4), W_o=Wo)
    keys = [np.array([[1.0, 0.0], [0.0, 1.0]]), np.array([[0.0, 4.0], [-2.0, 0.0]])]
    vals = np.array([[1.0, 0.0, 5.0, 0.0], [0.0, 1.0, 0.0, -7.0]])
    q = np.array([[2.0, 0.0], [0.0, 1.0], [1.0, 1.0], [-1.0, 3.0]])
    out = C.decode(spec, f, keys + [vals], q, 1, 2)
    want = np.zeros(2)
    for h in range(4):
        g = h // 2
        s = keys[g] @ q[h] / math.sqrt(2)
        p0 = 1.0 / (1.0 + math.exp(s[1] - s[0]))
        y = p0 * vals[0, 2 * g:2 * g + 2] + (1 - p0) * vals[1, 2 * g:2 * g + 2]
        want += (h + 1) * y
    np.testing.assert_allclose(out, want, rtol=1e-13)


def test_cpp_full_rank_equals_attention_from_w():
    # r = d, RoPE on: attention over latents equals attention with K = X W_k, V = X W_v computed directly
    spec = small_spec(key_ranks=[8, 8], value_rank=16, rope=True)
    T = 9
    f = gen.make_factors(spec, 1)
    X = gen.hidden_states(1, 0, 0, T, spec.hidden)
    Zh = [X @ a for a in f.A_k] + [X @ f.A_v]
    q = gen.queries(1, 0, 1, spec.n_heads, spec.head_dim)[0, 0]
    out = C.decode(spec, f, Zh, q, T - 1, T)
    d = spec.head_dim
    want = np.zeros(spec.hidden)
    V = X @ (f.A_v @ f.B_v)
    pos = np.arange(T)
    for h in range(spec.n_heads):
        K = X @ (f.A_k[h] @ f.B_k[h])
        theta = 10000.0 ** (-2 * np.arange(d // 2) / d)
        ang = pos[:, None] * theta[None]
        Kr = np.concatenate([K[:, :d // 2] * np.cos(ang) - K[:, d // 2:] * np.sin(ang),
                             K[:, d // 2:] * np.cos(ang) + K[:, :d // 2] * np.sin(ang)], axis=1)
        a = (T - 1) * theta
        qr = np.concatenate([q[h, :d // 2] * np.cos(a) - q[h, d // 2:] * np.sin(a),
                             q[h, d // 2:] * np.cos(a) + q[h, :d // 2] * np.sin(a)])
        p = torch.softmax(torch.from_numpy(Kr @ qr / math.sqrt(d)), 0).numpy()
        want += (p @ V[:, h * d:(h + 1) * d]) @ f.W_o[h * d:(h + 1) * d]
    np.testing.assert_allclose(out, want, rtol=1e-11, atol=1e-12)


def test_cpp_plain_layer_single_token_and_sdpa():
    spec = gen.LayerSpec(hidden=16, n_heads=4, n_kv_heads=2, head_dim=8, key_ranks=[], value_rank=0, dtype="f32",
                         plain=True, rope=True)
    T, d = 7, 8
    f = gen.make_factors(spec, 2)
    K = gen.normals(gen.stream_key(6, 95), T * 16).reshape(T, 16)
    V = gen.normals(gen.stream_key(7, 95), T * 16).reshape(T, 16)
    q = gen.normals(gen.stream_key(8, 95), 4 * d).reshape(4, d)
    # one token: the output is that token's value through W_o, whatever the scores
    out1 = C.decode_plain(spec, f, K, V, q, 1, 0)
    want1 = sum(V[0, (h // 2) * d:(h // 2 + 1) * d] @ f.W_o[h * d:(h + 1) * d] for h in range(4))
    np.testing.assert_allclose(out1, want1, rtol=1e-13)
    # q at position 0 is not rotated: torch's SDPA over the stored K/V (GQA expanded) gives the same head outputs
    out = C.decode_plain(spec, f, K, V, q, T, 0)
    Kt = torch.from_numpy(K).reshape(T, 2, d).transpose(0, 1).repeat_interleave(2, 0)
    Vt = torch.from_numpy(V).reshape(T, 2, d).transpose(0, 1).repeat_interleave(2, 0)
    Y = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q)[:, None], Kt, Vt)[:, 0].numpy()
    np.testing.assert_allclose(out, Y.reshape(-1) @ f.W_o, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# The two oracles agree on seeded cases
# ---------------------------------------------------------------------------

def _quant_spec(**kw):
    base = dict(hidden=192, n_heads=4, n_kv_heads=2, head_dim=48, key_ranks=[20, 45], value_rank=72, dtype="f32",
                quantized=True, hadamard_block=32, rope=True)
    base.update(kw)
    return gen.LayerSpec(**base)


def test_cpp_matches_numpy_formats():
    spec = _quant_spec()
    for r in (1, 5, 20, 45, 72, 1024):
        assert [(g.start, g.n, g.bits) for g in O.groups(r, spec)] == C.groups(r, spec)
        np.testing.assert_array_equal(C.rotation(r, spec), O.rotation(r, spec))
    Z = (gen.normals(gen.stream_key(9, 96), 16 * 72) * 2.0).astype(np.float32).reshape(16, 72)
    Z[5] = np.nan
    for cm in (False, True):
        np.testing.assert_array_equal(C.pack_block(Z, 72, spec, cm), O.pack_block(Z, 72, spec, cm))
    Zf = np.nan_to_num(Z)
    np.testing.assert_array_equal(C.stored_values(Zf, 72, spec), O.stored_values(Zf, 72, spec))
    ub = _quant_spec(quantized=False, dtype="bf16")
    np.testing.assert_array_equal(C.stored_values(Zf, 72, ub), O.stored_values(Zf, 72, ub))


@pytest.mark.parametrize("kw", [dict(), dict(rope=False), dict(n_kv_heads=4, key_ranks=[7, 16, 33, 3]),
                                dict(n_kv_heads=1, key_ranks=[40], value_rank=40, hadamard_block=0)])
def test_cpp_decode_matches_numpy(kw):
    spec = _quant_spec(**kw)
    T = 37
    f = gen.make_factors(spec, 4)
    X = gen.hidden_states(4, 0, 0, T, spec.hidden)
    Rs = [O.rotation(r, spec) for r in spec.latent_widths]
    Z = [O.project(X, A, R) for A, R in zip(f.A_k, Rs[:-1])] + [O.project(X, f.A_v, Rs[-1])]
    Zh = [O.stored_values(z, z.shape[1], spec) for z in Z]
    q = gen.queries(4, 0, 1, spec.n_heads, spec.head_dim)[0, 0]
    for seq_len, q_pos in ((T, T - 1), (1, 0), (20, 30)):
        want = O.decode(spec, f, Zh, q, q_pos, seq_len)
        for th in (1, 3):
            np.testing.assert_allclose(C.decode(spec, f, Zh, q, q_pos, seq_len, threads=th), want, rtol=1e-11,
                                       atol=1e-12 * np.max(np.abs(want)))


def test_cpp_decode_plain_matches_numpy():
    spec = gen.LayerSpec(hidden=48, n_heads=8, n_kv_heads=2, head_dim=16, key_ranks=[], value_rank=0, dtype="bf16",
                         plain=True, rope=True)
    f = gen.make_factors(spec, 5)
    X = gen.hidden_states(5, 0, 0, 23, spec.hidden)
    Z = O.plain_latents(spec, f, X, np.arange(23)).astype(np.float64)
    q = gen.queries(5, 0, 1, spec.n_heads, spec.head_dim)[0, 0]
    K, V = Z[:, :32], Z[:, 32:]
    np.testing.assert_allclose(C.decode_plain(spec, f, K, V, q, 23, 22), O.decode_plain(spec, f, K, V, q, 23, 22),
                               rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("top_fraction,top_bits,bottom_bits,group_size,hadamard", [
    (0.25, 4, 3, 32, True), (0.2, 4, 3, 32, True), (1.0, 4, 3, 32, True), (0.0, 4, 3, 32, False),
    (0.25, 8, 2, 16, True), (0.5, 5, 6, 7, False), (0.3, 2, 8, 1, False), (0.25, 4, 3, 24, True)])
def test_cpp_matches_numpy_formats_across_bit_splits(top_fraction, top_bits, bottom_bits, group_size, hadamard):
    # The two oracles agree on group layout, rotation and stored bytes for every bit split, group size and
    # rank tried: the 20:80 and 25:75 splits of the pages, uniform widths, odd group sizes, ragged segments.
    spec = _quant_spec(top_fraction=top_fraction, top_bits=top_bits, bottom_bits=bottom_bits,
                       group_size=group_size, hadamard_block=group_size if hadamard else 0)
    for r in (1, 2, 3, 8, 17, 31, 33, 40, 64, 97, 130):
        assert [(g.start, g.n, g.bits) for g in O.groups(r, spec)] == C.groups(r, spec), r
        np.testing.assert_array_equal(C.rotation(r, spec), O.rotation(r, spec))
        Z = (gen.normals(gen.stream_key(11, r), 16 * r) * 1.5).astype(np.float32).reshape(16, r)
        Z[3, : (r + 1) // 2] = 0.0             # an all-zero head of a token (zero scale)
        for cm in (False, True):
            np.testing.assert_array_equal(C.pack_block(Z, r, spec, cm), O.pack_block(Z, r, spec, cm))
        np.testing.assert_array_equal(C.stored_values(Z, r, spec), O.stored_values(Z, r, spec))
