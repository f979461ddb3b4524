"""GPU parity at the workloads' own shapes, on sampled sequences and rows.

The library decodes the whole batch at the workload's batch size and context
(so the kernels run with their real grid, run/partial structure and page
tables); the float64 oracle checks a seeded sample of the sequences (it
would take minutes for all).  Sequences are independent, so the unchecked
ones only need valid latents: they are drawn with the same seeded generator
and not rotated.  Tolerances as in test_parity_gpu.py.
"""
import numpy as np
import pytest
import torch

from oracle import starkv_oracle as O
from synth import gen

from harness import Case, GpuCache, check_close, queries

pytestmark = pytest.mark.gpu


def _case(cfg, quantized=False, layer=2):
    return Case(gen.config_spec(cfg, quantized=quantized, layer=layer), gen.LAYER_SEED[cfg], layer if cfg == 4 else 0)


def _filler_latents(c: Case, b: int, T: int) -> list:
    """Valid float32 latents for a sequence whose output is not checked (seeded, unrotated)."""
    s = c.spec
    out = [gen.latent_draw(c.seed, c.layer, b, T, c.raw.sigma_k[li][:r], li).astype(np.float32)
           for li, r in enumerate(s.latent_widths[:-1])]
    out.append(gen.latent_draw(c.seed, c.layer, b, T, c.raw.sigma_v[:s.value_rank], -1).astype(np.float32))
    return out


def full_shape_decode(c: Case, batch: int, ctx: int, checked: tuple, peaky: float = 1.0):
    L = c.load()
    s = c.spec
    # ragged lengths around ctx (the last page of each sequence partly filled)
    lens = [ctx - (7 * b) % 16 for b in range(batch)]
    cache = GpuCache(L, lens)
    Zs = {}
    for b, T in enumerate(lens):
        if b in checked:
            Z = c.latents_direct(b, T)
            Zs[b] = Z
        else:
            Z = _filler_latents(c, b, T)
        cache.append_latents(b, Z)
    q = queries(c, batch, peaky)[:, 0]
    qt = torch.from_numpy(q).cuda().to(torch.bfloat16)
    out = torch.empty(batch, s.hidden, device="cuda", dtype=torch.bfloat16)
    ws = torch.empty(L.workspace_bytes(batch, cache.page_table.shape[1] * 16), dtype=torch.uint8, device="cuda")
    L.decode(cache.pool, cache.n_pages, cache.page_table, torch.tensor(lens, dtype=torch.int32, device="cuda"), qt,
             out, ws)
    torch.cuda.synchronize()
    assert L.sync_status() == 0
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    for b in checked:
        T = lens[b]
        check_close(got[b], c.oracle_decode(c.stored(Zs[b]), q[b], T - 1, T), f"seq {b} (T={T})")


def test_cfg1_batch16_ctx4096():
    full_shape_decode(_case(1), 16, 4096, checked=(0, 11))


def test_cfg2_batch16_ctx32768():
    full_shape_decode(_case(2), 16, 32768, checked=(3, 15))


@pytest.mark.parametrize("quant", [False, True])
def test_cfg3_batch64_ctx8192(quant):
    full_shape_decode(_case(3, quantized=quant), 64, 8192, checked=(0, 41))


def test_cfg3_batch64_ctx8192_peaky():
    full_shape_decode(_case(3, quantized=True), 64, 8192, checked=(17,), peaky=25.0)


def test_cfg4_prefill_chunk_1024_after_3072():
    """One 1024-query chunk of the 4096-token prefill of a compressed stack layer, after 3072 tokens of
    history (chunks of 1024, appended before their attention), on the tensor cores (keys and values
    rebuilt for the chunk, tiled causal attention, output through W_o): rows at the 128-query tile
    edges checked against the oracle's causal prefill."""
    c = _case(4, layer=2)
    s = c.spec
    L = c.load()
    T0, n = 3072, 1024
    cache = GpuCache(L, [T0 + n])
    Z = c.latents_direct(0, T0 + n)
    cache.append_latents(0, Z)
    Q = queries(c, 1, n_pos=n)[0]
    qt = torch.from_numpy(Q).cuda().to(torch.bfloat16)
    out = torch.empty(n, s.hidden, device="cuda", dtype=torch.bfloat16)
    ws = torch.empty(L.workspace_bytes(1, cache.page_table.shape[1] * 16, n), dtype=torch.uint8, device="cuda")
    L.prefill(cache.pool, cache.n_pages, cache.page_table, [T0], [n], qt, out, ws)
    torch.cuda.synchronize()
    assert L.sync_status() == 0
    got = out.double().cpu().numpy()
    Zs = c.stored(Z)
    for i in (0, 255, 256, 511, 1023):
        want = O.decode(s, c.f, Zs, Q[i], T0 + i, T0 + i + 1, c.B_rot)
        check_close(got[i], want, f"prefill row {i}")


def test_hidden_mode_append_codes_within_one_step():
    """Append from hidden states on the tensor cores (projection with fp16 operands, block FWHT,
    quantizer): every stored value is within one code step of the oracle's float64 projection
    quantized by the oracle, read back from the pool bytes with the oracle's page-format reader."""
    c = _case(2)
    s = c.spec
    L = c.load()
    T = 80
    cache = GpuCache(L, [T])
    X = c.hidden(0, T)
    xt = torch.from_numpy(X).cuda().to(torch.bfloat16)
    ws = torch.empty(L.append_workspace_bytes(T), dtype=torch.uint8, device="cuda")
    seq = torch.zeros(T, dtype=torch.int32, device="cuda")
    pos = torch.arange(T, dtype=torch.int32, device="cuda")
    L.append(cache.pool, cache.n_pages, cache.page_table, seq, pos, xt, False, workspace=ws)
    pool = cache.pool_pages()
    Z = c.latents_from_hidden(X, np.arange(T))
    offs, _ = O.page_layout(s)
    worst = 0.0
    for li, r in enumerate(s.latent_widths):
        cmaj = li == len(s.latent_widths) - 1
        want_vals = O.stored_values(Z[li], r, s)
        gs = O.groups(r, s)
        for t in range(T):
            page = pool[cache.page_table_np[0][t // 16]]
            blk = page[offs[li]:]
            slot = t % 16
            code_off = ((len(gs) * 16 * 2) + 15) // 16 * 16
            for gi, g in enumerate(gs):
                s_gpu = float(blk[(gi * 16 + slot) * 2:(gi * 16 + slot) * 2 + 2].view(np.float16)[0])
                s_or, _ = O.quantize_group(Z[li][t, g.start:g.start + g.n], g.bits)
                cb = blk[code_off:]
                for i in range(g.n):
                    u = O.read_bits(cb, O.code_bit(slot, i, g.n, g.bits, 16, cmaj), g.bits)
                    z_gpu = (u - (1 << (g.bits - 1))) * s_gpu
                    step = max(s_gpu, float(s_or))
                    err = abs(z_gpu - want_vals[t, g.start + i])
                    worst = max(worst, err / step if step > 0 else err)
                    assert err <= 1.02 * step + 1e-30, (li, t, gi, i, err, step)
                code_off += (16 * g.n * g.bits // 8 + 15) // 16 * 16
    assert worst <= 1.02
