"""Oracle for STAR-KV latent decode attention: a plain, slow float64 reference.

TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the CPU
baseline arm of the benchmark may import this module.  The library never calls
it, and it shares no code with the CUDA path: both start from the seeded inputs
of the `synth` package and nothing else.

What it computes is the plain definition of attention over the reconstructed,
dequantized low-rank KV cache, with no fusion, no re-association and no split
over tokens:

  keys    K_h = Zhat_{k,h} B'_{k,h}                 (head-wise decomposition)
  values  V_g = Zhat_v B'_{v}[:, g d:(g+1) d]       (joint decomposition)
  scores  s_h = RoPE(q_h) . RoPE(K_{kv(h)})^T / sqrt(d)
  output  out = sum_h softmax(s_h) V_{kv(h)} W_{o,h}

Sources (page titles and sections of the STAR-KV material):
  * "STAR-KV 阅读笔记" (Zhongzhu Zhou's reading notes on arXiv 2606.08382 v1):
      section 2.2  latents Z = X A, factors A = U_r Sigma_r, B = V_r^T;
      section 5.1-5.2  head-wise keys, joint values;
      section 5.3  value-side output fusion M_h = B_{v,h} W_{o,h}, stacked
                   P Z_v, pre-RoPE key latents;
      section 6.1  block-wise Hadamard inserted before quantization and
                   absorbed into the factors; high-magnitude block at 4 bits,
                   ordinary block at 3 bits; average-bit ledger;
      section 6.2  cache ledger with exempt layers;
      Algorithm 2  the decode data flow.
  * "tenosra/longchat-7b-starkv-proxima" model card: top_fraction 0.25,
    top_bits 4, bottom_bits 3; protected layers.
  * The arXiv abstract (as reprinted on the gptget.net summary page).

Readings where the pages are silent:
  * quantizer: symmetric, zero point 0, qmax = 2^(b-1) - 1, one fp16 scale per
    (token, 32-channel group), scale = fp16 rounded toward +inf of amax/qmax
    (IEEE fp32 division), codes = round-half-even(z / scale) clamped to
    [-qmax, qmax], stored offset-binary u = q + 2^(b-1);
  * channel segments: hi = [0, ceil(top_fraction r)), lo = the rest; groups of
    32 from each segment start, the last group shorter;
  * rotation: per group, a direct sum of normalised Sylvester-Hadamard blocks
    over the binary decomposition of the group length (largest first);
  * page format: see `page_layout` and `pack_block`;
  * RoPE: rotate-half pairing (p, p + d/2), theta_p = base^(-2p/d), keys at
    their slot position, the query at q_pos;
  * GQA: kv(h) = h // (H / H_kv).

Parity status: every function below is pinned by tests/test_oracle_pins.py
(closed forms, identities, brute force, and hand-derived golden bytes);
see that file for the pin of each.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


# ---------------------------------------------------------------------------
# Channel segments and groups ("STAR-KV 阅读笔记" section 6.1: the top channels
# by singular value form the high-precision block; SVD order puts them first).
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Group:
    start: int   # first channel of the group in the latent
    n: int       # number of channels
    bits: int    # code width (0 = unquantized)


def n_high(r: int, top_fraction: float) -> int:
    """Channels in the 4-bit segment: ceil(top_fraction * r)."""
    return int(math.ceil(top_fraction * r - 1e-9))


def groups(r: int, spec) -> list:
    """Quantization (and rotation) groups of a latent of width r, hi segment first."""
    if not spec.quantized:
        return [Group(0, r, 0)]
    out = []
    nh = n_high(r, spec.top_fraction)
    for seg_start, seg_len, bits in ((0, nh, spec.top_bits), (nh, r - nh, spec.bottom_bits)):
        k = 0
        while k < seg_len:
            n = min(spec.group_size, seg_len - k)
            out.append(Group(seg_start + k, n, bits))
            k += n
    return out


# ---------------------------------------------------------------------------
# Block-wise Hadamard ("STAR-KV 阅读笔记" section 6.1: rotate the
# high-magnitude block and the ordinary block separately; R orthogonal, so
# inserting R R^T before quantization is exact and both halves are absorbed
# into the down and up projections).
# ---------------------------------------------------------------------------

def sylvester(n: int) -> np.ndarray:
    """Unnormalised Sylvester-Hadamard matrix of order n (a power of two)."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    assert h.shape[0] == n
    return h


def group_rotation(n: int) -> np.ndarray:
    """Direct sum of normalised Sylvester blocks over the binary decomposition of n."""
    out = np.zeros((n, n))
    k = 0
    p = 1 << (n.bit_length() - 1) if n > 0 else 0
    while k < n:
        while p > n - k:
            p >>= 1
        out[k:k + p, k:k + p] = sylvester(p) / math.sqrt(p)
        k += p
    return out


def rotation(r: int, spec) -> np.ndarray:
    """Block-diagonal rotation R (r x r) of one latent; identity when off."""
    R = np.eye(r)
    if spec.quantized and spec.hadamard_block:
        for g in groups(r, spec):
            R[g.start:g.start + g.n, g.start:g.start + g.n] = group_rotation(g.n)
    return R


# ---------------------------------------------------------------------------
# Latent projection ("STAR-KV 阅读笔记" section 2.2; Algorithm 2 steps 1-2).
# ---------------------------------------------------------------------------

def project(X: np.ndarray, A: np.ndarray, R: np.ndarray) -> np.ndarray:
    """Latents of tokens X (rows): Z = X A R in float64, rounded once to float32."""
    return (X @ A @ R).astype(np.float32)


def rotate(Z: np.ndarray, R: np.ndarray) -> np.ndarray:
    """Rotate directly drawn unrotated latents: Z R, rounded once to float32."""
    return (np.asarray(Z, dtype=np.float64) @ R).astype(np.float32)


def rotated_factor(B: np.ndarray, R: np.ndarray) -> np.ndarray:
    """Up-projection with the rotation absorbed: B' = R^T B."""
    return R.T @ B


# ---------------------------------------------------------------------------
# Number formats, written from their IEEE-754 definitions.
# ---------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); returns float32."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return r.astype(np.uint32).view(np.float32)


def fp16_round_up(x32: np.float32) -> np.float16:
    """Smallest binary16 value >= x (rounding toward +infinity); x finite, >= 0."""
    h = np.float16(x32)                      # nearest binary16
    if np.float32(h) < x32:
        h = np.nextafter(h, np.float16(np.inf))
    return h


# ---------------------------------------------------------------------------
# Quantizer ("STAR-KV 阅读笔记" section 6.1: hi block 4-bit, ordinary 3-bit;
# the rest of the definition is the reading stated in the module docstring).
# ---------------------------------------------------------------------------

class ScaleOverflow(ValueError):
    pass


def quantize_group(z: np.ndarray, bits: int):
    """Quantize one (token, group) vector of float32 latents.

    Returns (s16: np.float16, u: uint8 array of offset-binary codes).
    """
    z = np.asarray(z, dtype=np.float32)
    qmax = (1 << (bits - 1)) - 1
    amax = np.float32(np.max(np.abs(z))) if z.size else np.float32(0)
    s32 = np.float32(amax / np.float32(qmax))
    if s32 > np.float32(65504.0):
        raise ScaleOverflow(float(s32))
    s16 = fp16_round_up(s32)
    if s16 == 0:
        q = np.zeros(z.shape, dtype=np.int64)
    else:
        q = np.rint(z / np.float32(s16)).astype(np.int64)
        q = np.clip(q, -qmax, qmax)
    return s16, (q + (1 << (bits - 1))).astype(np.uint8)


def dequantize_group(u: np.ndarray, s16: np.float16, bits: int) -> np.ndarray:
    """Dequantized values (u - 2^(b-1)) * scale, exact in float64."""
    return (u.astype(np.float64) - (1 << (bits - 1))) * float(s16)


# ---------------------------------------------------------------------------
# Page format (16-token pages, as in vLLM-style paged KV blocks on the model
# card; the pages fix no byte layout, so this one is a reading).
#
#   page = latent block 0 | latent block 1 | ... | latent block L-1 | pad to 128 B
#   latents in order: key latent of KV head 0 .. H_kv-1, then the joint value latent
#   unquantized block: element (slot, j) at byte (slot * r + j) * elem_size (key
#                      latents, and every latent of a plain layer), or at byte
#                      (j * P + slot) * elem_size (the value latent of a latent
#                      layer: channel-major); pad to 16 B
#   quantized block:   scales [group][slot] fp16, pad to 16 B; then for each group g
#                      a code block of P * n_g * b_g bits, pad to 16 B, a bitstream
#                      written least significant bit first (stream bit k is bit
#                      (k mod 8) of byte k div 8).  The code of (slot, channel i of g)
#                      occupies stream bits [k, k + b_g) with
#                        key latents (slot-major):     k = (slot * n_g + i) * b_g
#                        value latent (channel-major): k = (i * P + sigma(slot)) * b_g,
#                      sigma(s) = (P/2) (s mod 2) + s div 2: each channel's P codes form
#                      one field, even slots first, then odd slots.
# ---------------------------------------------------------------------------

def _ru(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def elem_size(spec) -> int:
    return 4 if spec.dtype == "f32" else 2


def block_bytes(r: int, spec) -> int:
    P = spec.page_size
    if not spec.quantized or spec.plain:
        return _ru(P * r * elem_size(spec), 16)
    gs = groups(r, spec)
    total = _ru(len(gs) * P * 2, 16)
    for g in gs:
        total += _ru(P * g.n * g.bits // 8, 16)
    return total


def page_layout(spec):
    """(offsets of each latent block, page_bytes)."""
    offs, o = [], 0
    for r in spec.latent_widths:
        offs.append(o)
        o += block_bytes(r, spec)
    return offs, _ru(o, 128)


def write_bits(buf: np.ndarray, bit_offset: int, value: int, nbits: int) -> None:
    """Write `nbits` of `value` into byte buffer `buf`, LSB first, one bit at a time."""
    for t in range(nbits):
        if (value >> t) & 1:
            k = bit_offset + t
            buf[k // 8] |= np.uint8(1 << (k % 8))


def read_bits(buf: np.ndarray, bit_offset: int, nbits: int) -> int:
    v = 0
    for t in range(nbits):
        k = bit_offset + t
        v |= ((int(buf[k // 8]) >> (k % 8)) & 1) << t
    return v


def slot_place(slot: int, P: int) -> int:
    """Place of a slot inside a channel field of the value latent: even slots first."""
    return (P // 2) * (slot % 2) + slot // 2


def code_bit(slot: int, i: int, n: int, bits: int, P: int, channel_major: bool) -> int:
    """First stream bit of the code of (slot, channel i) in a group of n channels."""
    if channel_major:
        return (i * P + slot_place(slot, P)) * bits
    return (slot * n + i) * bits


def pack_block(Z: np.ndarray, r: int, spec, channel_major: bool = False) -> np.ndarray:
    """Bytes of one latent block holding the float32 latents Z [P, r] (rows = slots).

    Rows of Z that are NaN-free are written; a slot that holds no token should
    be passed as None rows (see `pack_page`), which leaves its bytes zero.
    channel_major selects the value latent's order (see the page format above):
    codes by `code_bit`, unquantized elements [channel][slot].
    """
    P = spec.page_size
    out = np.zeros(block_bytes(r, spec), dtype=np.uint8)
    if not spec.quantized or spec.plain:
        if spec.dtype == "f32":
            vals = np.asarray(Z, dtype=np.float32)
        else:
            vals = bf16_round(Z).view(np.uint32) >> np.uint32(16)
            vals = vals.astype(np.uint16)
        es = elem_size(spec)
        for slot in range(P):
            if Z[slot] is None or np.isnan(np.asarray(Z[slot], dtype=np.float64)).any():
                continue
            if channel_major:
                for j in range(r):
                    o = (j * P + slot) * es
                    out[o:o + es] = vals[slot][j:j + 1].view(np.uint8)
            else:
                row = vals[slot].view(np.uint8)
                o = slot * r * es
                out[o:o + row.size] = row
        return out
    gs = groups(r, spec)
    scale_bytes = _ru(len(gs) * P * 2, 16)
    code_off = scale_bytes
    for gi, g in enumerate(gs):
        cb = out[code_off:code_off + _ru(P * g.n * g.bits // 8, 16)]
        for slot in range(P):
            z = Z[slot]
            if z is None or np.isnan(np.asarray(z, dtype=np.float64)).any():
                continue
            s16, u = quantize_group(np.asarray(z, dtype=np.float32)[g.start:g.start + g.n], g.bits)
            sb = np.array([s16], dtype=np.float16).view(np.uint8)
            so = (gi * P + slot) * 2
            out[so:so + 2] = sb
            for i in range(g.n):
                write_bits(cb, code_bit(slot, i, g.n, g.bits, P, channel_major), int(u[i]), g.bits)
        code_off += _ru(P * g.n * g.bits // 8, 16)
    return out


def pack_page(latents_per_slot, spec) -> np.ndarray:
    """Bytes of one page.

    latents_per_slot: list of P entries; each is None (empty slot) or a list of
    float32 vectors, one per latent (keys per KV head, then values).
    """
    offs, pb = page_layout(spec)
    page = np.zeros(pb, dtype=np.uint8)
    P = spec.page_size
    for li, r in enumerate(spec.latent_widths):
        Z = np.full((P, r), np.nan, dtype=np.float32)
        for slot in range(P):
            if latents_per_slot[slot] is not None:
                Z[slot] = latents_per_slot[slot][li]
        last = li == len(spec.latent_widths) - 1
        blk = pack_block(Z, r, spec, channel_major=last and not spec.plain)
        page[offs[li]:offs[li] + blk.size] = blk
    return page


def build_pool(spec, latents, page_table, n_pages) -> np.ndarray:
    """Pool bytes [n_pages, page_bytes] for the float32 latents of every sequence.

    latents[b] is a list (one per latent) of [T_b, r] float32 arrays; token t of
    sequence b lives in page page_table[b][t // P], slot t % P.
    """
    _, pb = page_layout(spec)
    P = spec.page_size
    pool = np.zeros((n_pages, pb), dtype=np.uint8)
    for b, lat in enumerate(latents):
        T = lat[0].shape[0]
        for p in range((T + P - 1) // P):
            slots = []
            for s in range(P):
                t = p * P + s
                slots.append([L[t] for L in lat] if t < T else None)
            pool[page_table[b][p]] = pack_page(slots, spec)
    return pool


# ---------------------------------------------------------------------------
# Dequantized view of the stored latents (what Algorithm 2 step 4a reads).
# ---------------------------------------------------------------------------

def stored_values(Z: np.ndarray, r: int, spec) -> np.ndarray:
    """Values a reader of the cache sees for float32 latents Z [T, r], as float64."""
    Z = np.asarray(Z, dtype=np.float32)
    if not spec.quantized or spec.plain:
        if spec.dtype == "f32":
            return Z.astype(np.float64)
        return bf16_round(Z).astype(np.float64)
    out = np.zeros(Z.shape, dtype=np.float64)
    for g in groups(r, spec):
        for t in range(Z.shape[0]):
            s16, u = quantize_group(Z[t, g.start:g.start + g.n], g.bits)
            out[t, g.start:g.start + g.n] = dequantize_group(u, s16, g.bits)
    return out


def stored_values_fast(Z: np.ndarray, r: int, spec) -> np.ndarray:
    """Same result as `stored_values`, vectorised over tokens (for long contexts).

    Identical arithmetic per element: float32 amax, float32 division by qmax,
    binary16 rounding toward +inf, float32 division, round-half-even, clamp.
    """
    Z = np.asarray(Z, dtype=np.float32)
    if not spec.quantized or spec.plain:
        return stored_values(Z, r, spec)
    out = np.zeros(Z.shape, dtype=np.float64)
    for g in groups(r, spec):
        blk = Z[:, g.start:g.start + g.n]
        qmax = (1 << (g.bits - 1)) - 1
        amax = np.max(np.abs(blk), axis=1).astype(np.float32)
        s32 = (amax / np.float32(qmax)).astype(np.float32)
        if (s32 > np.float32(65504.0)).any():
            raise ScaleOverflow(float(s32.max()))
        s16 = s32.astype(np.float16)
        low = s16.astype(np.float32) < s32
        s16[low] = np.nextafter(s16[low], np.float16(np.inf))
        s = s16.astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.rint(blk / s[:, None])
        q = np.where(s[:, None] == 0, 0.0, q)
        q = np.clip(q, -qmax, qmax)
        out[:, g.start:g.start + g.n] = q.astype(np.float64) * s16.astype(np.float64)[:, None]
    return out


# ---------------------------------------------------------------------------
# RoPE (rotate-half form; "STAR-KV 阅读笔记" section 5.3: the key cache is kept
# before RoPE and each reconstructed key is rotated by its own position).
# ---------------------------------------------------------------------------

def rope(x: np.ndarray, pos, theta: float) -> np.ndarray:
    """Rotate rows of x [..., d] by positions pos (broadcast over leading dims)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    freq = theta ** (-2.0 * np.arange(half) / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


# ---------------------------------------------------------------------------
# Attention ("STAR-KV 阅读笔记" Algorithm 2, written as the plain definition).
# ---------------------------------------------------------------------------

def softmax(s: np.ndarray) -> np.ndarray:
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def kv_of(h: int, spec) -> int:
    return h // (spec.n_heads // spec.n_kv_heads)


def decode(spec, f, Zhat, q, q_pos: int, seq_len: int, B_rot=None) -> np.ndarray:
    """Decode attention output [D] of one sequence, float64.

    Zhat: list of stored-value arrays [T, r] (keys per KV head, then values).
    f: factors (float64 values of what the library receives).
    q: [H, d] query.  Keys at positions 0..seq_len-1 are attended to.
    B_rot: optional list (keys..., value) of rotated up-projections B' = R^T B.
    """
    H, d = spec.n_heads, spec.head_dim
    scale = 1.0 / math.sqrt(d)
    if B_rot is None:
        B_rot = up_projections(spec, f)
    T = seq_len
    pos = np.arange(T)
    Vfull = Zhat[-1][:T] @ B_rot[-1]                      # [T, H_kv d], explicit
    out = np.zeros(spec.hidden)
    for h in range(H):
        g = kv_of(h, spec)
        K = Zhat[g][:T] @ B_rot[g]                        # [T, d], explicit
        qh = np.asarray(q[h], dtype=np.float64)
        if spec.rope:
            K = rope(K, pos, spec.rope_theta)
            qh = rope(qh, q_pos, spec.rope_theta)
        p = softmax((K @ qh) * scale)
        y = p @ Vfull[:, g * d:(g + 1) * d]
        out += y @ f.W_o[h * d:(h + 1) * d]
    return out


def up_projections(spec, f) -> list:
    """B' = R^T B for every key latent and for the value latent."""
    out = []
    for h, r in enumerate(spec.key_ranks):
        out.append(rotated_factor(f.B_k[h], rotation(r, spec)))
    out.append(rotated_factor(f.B_v, rotation(spec.value_rank, spec)))
    return out


def decode_plain(spec, f, Khat, Vhat, q, seq_len: int, q_pos: int) -> np.ndarray:
    """Uncompressed layer: stored K (already rotated by RoPE) and V, [T, H_kv d]."""
    H, d = spec.n_heads, spec.head_dim
    out = np.zeros(spec.hidden)
    for h in range(H):
        g = kv_of(h, spec)
        qh = np.asarray(q[h], dtype=np.float64)
        if spec.rope:
            qh = rope(qh, q_pos, spec.rope_theta)
        p = softmax((Khat[:seq_len, g * d:(g + 1) * d] @ qh) / math.sqrt(d))
        out += (p @ Vhat[:seq_len, g * d:(g + 1) * d]) @ f.W_o[h * d:(h + 1) * d]
    return out


def plain_latents(spec, f, X: np.ndarray, positions) -> np.ndarray:
    """Stored quantities of an uncompressed layer: [RoPE(X W_k) | X W_v], float32."""
    d = spec.head_dim
    K = X @ f.W_k
    if spec.rope:
        K = np.concatenate([rope(K[:, g * d:(g + 1) * d], np.asarray(positions), spec.rope_theta)
                            for g in range(spec.n_kv_heads)], axis=1)
    return np.concatenate([K, X @ f.W_v], axis=1).astype(np.float32)


def prefill(spec, f, Zhat, Q, q_start: int, B_rot=None) -> np.ndarray:
    """Causal attention for queries at positions q_start .. q_start + n - 1.

    Q: [n, H, d].  Query i attends to keys 0 .. q_start + i.  Returns [n, D].
    """
    n = Q.shape[0]
    return np.stack([decode(spec, f, Zhat, Q[i], q_start + i, q_start + i + 1, B_rot)
                     for i in range(n)])


# ---------------------------------------------------------------------------
# Value-side output fusion ("STAR-KV 阅读笔记" section 5.3): M_h = B'_{v,kv(h)} W_{o,h}.
# The oracle's attention does not use it; the identity is pinned in the tests.
# ---------------------------------------------------------------------------

def fused_output_factor(spec, f, h: int) -> np.ndarray:
    d = spec.head_dim
    g = kv_of(h, spec)
    Bv = rotated_factor(f.B_v, rotation(spec.value_rank, spec))
    return Bv[:, g * d:(g + 1) * d] @ f.W_o[h * d:(h + 1) * d]


# ---------------------------------------------------------------------------
# Ledger ("STAR-KV 阅读笔记" section 6.1 and 6.2).
# ---------------------------------------------------------------------------

def average_bits(top_fraction: float, top_bits: int, bottom_bits: int) -> float:
    return top_fraction * top_bits + (1.0 - top_fraction) * bottom_bits


def payload_reduction(rank_kept: float, bits: float, base_bits: int = 16) -> float:
    """Ideal payload reduction vs base_bits at a kept-rank fraction."""
    return base_bits / bits / rank_kept


def mixed_ledger(n_layers: int, exempt: int, compressed_fraction: float) -> float:
    """Whole-cache reduction when `exempt` layers stay uncompressed."""
    return n_layers / (exempt + (n_layers - exempt) * compressed_fraction)


def latent_bytes_per_token(r: int, spec) -> float:
    """Algorithmic bytes of one token of one latent (codes + scales, no padding)."""
    if not spec.quantized or spec.plain:
        return r * elem_size(spec)
    bits = sum(g.n * g.bits for g in groups(r, spec))
    return bits / 8 + 2 * len(groups(r, spec))
