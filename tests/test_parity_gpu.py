"""GPU parity of the library against the float64 oracle, through the C ABI.

Inputs are seeded (synth); the oracle never sees a value produced by the
library.  Tolerances (attention outputs): relative L2 <= 3e-3 and
max |err| <= 1e-2 * max |oracle|; packed pages: bit-exact.
"""
import functools

import numpy as np
import pytest
import torch

from oracle import starkv_oracle as O
from synth import gen

from harness import Case, GpuCache, check_close, queries, rel_l2

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=None)
def case(cfg: int, quantized: bool = False, layer: int = 2) -> Case:
    spec = gen.config_spec(cfg, quantized=quantized, layer=layer)
    return Case(spec, gen.LAYER_SEED[cfg], layer if cfg == 4 else 0)


def run_decode(c: Case, lens, peaky=1.0, use_hidden=True, check_pool=True, q_pos=None, page_seed=0, path=0,
               unfused=False):
    """Fill a cache (latent mode), decode one query per sequence, compare with the oracle."""
    L = c.load(unfused_output=unfused)
    if path:
        L.set_decode_path(path)
    s = c.spec
    cache = GpuCache(L, lens, seed=page_seed)
    lat_all = []
    for b, T in enumerate(lens):
        if T == 0:
            lat_all.append(None)
            continue
        if use_hidden:
            X = c.hidden(b, T)
            Z = c.latents_from_hidden(X, np.arange(T))
        else:
            Z = c.latents_direct(b, T)
        lat_all.append(Z)
        cache.append_latents(b, Z)
    if check_pool:
        pool = cache.pool_pages()
        want = O.build_pool(s, [z for z in lat_all if z is not None],
                            cache.page_table_np[[b for b, z in enumerate(lat_all) if z is not None]], cache.n_pages)
        np.testing.assert_array_equal(pool, want)
    B = len(lens)
    q = queries(c, B, peaky)[:, 0]
    qt = torch.from_numpy(q).cuda().to(torch.float32 if s.dtype == "f32" else torch.bfloat16)
    out = torch.empty(B, s.hidden, device="cuda", dtype=qt.dtype)
    ws = torch.empty(L.workspace_bytes(B, cache.page_table.shape[1] * 16), dtype=torch.uint8, device="cuda")
    seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    qp = None if q_pos is None else torch.tensor(q_pos, dtype=torch.int32, device="cuda")
    L.decode(cache.pool, cache.n_pages, cache.page_table, seq_lens, qt, out, ws, q_pos=qp)
    torch.cuda.synchronize()
    assert L.sync_status() == 0
    got = out.to(torch.float64).cpu().numpy()
    for b, T in enumerate(lens):
        if T == 0:
            assert np.all(got[b] == 0)
            continue
        Zs = c.stored(lat_all[b])
        pos = (T - 1) if q_pos is None else q_pos[b]
        want = c.oracle_decode(Zs, q[b], pos, T)
        check_close(got[b], want, f"seq {b} (T={T})")
    return got


def test_cfg0_tiny_fp32():
    run_decode(case(0), [256])


def test_cfg0_ragged_and_empty():
    run_decode(case(0), [1, 0, 37, 130])


def test_cfg1_bf16_rope():
    run_decode(case(1), [300, 17, 1])


def test_cfg1_peaky():
    # logits scaled up (std ~ 3) so attention is far from uniform
    run_decode(case(1), [200, 129], peaky=25.0, check_pool=False)


def test_cfg2_quantized_hadamard():
    run_decode(case(2), [333, 64, 5])


def test_cfg2_peaky_direct_latents():
    run_decode(case(2), [257, 48], peaky=25.0, use_hidden=False)


def test_cfg3_gqa_bf16():
    run_decode(case(3), [200, 33, 96])


def test_cfg3_gqa_quantized():
    run_decode(case(3, quantized=True), [200, 33, 96])


def test_cfg4_plain_layer():
    run_decode(case(4, layer=0), [150, 31])


def test_cfg4_compressed_layer():
    run_decode(case(4, layer=2), [150, 31])


def test_custom_query_positions():
    run_decode(case(1), [100, 64], q_pos=[150, 5], check_pool=False)


def test_page_table_permutation_invariance():
    c = case(2)
    a = run_decode(c, [90, 40], page_seed=1, check_pool=False)
    b = run_decode(c, [90, 40], page_seed=7, check_pool=False)
    np.testing.assert_array_equal(a, b)


def test_hidden_mode_append_matches_oracle_projection():
    """Append from hidden states: the kernel projects, rotates and quantizes.
    Codes may differ from the oracle's float64 projection only at rounding
    boundaries; the decoded output must still meet the attention tolerance."""
    c = case(2)
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
    want = O.build_pool(s, [Z], cache.page_table_np, cache.n_pages)
    diff = np.count_nonzero(pool != want)
    assert diff <= 0.01 * pool.size, diff
    q = queries(c, 1)[:, 0]
    qt = torch.from_numpy(q).cuda().to(torch.bfloat16)
    out = torch.empty(1, s.hidden, device="cuda", dtype=torch.bfloat16)
    wsd = torch.empty(L.workspace_bytes(1, cache.page_table.shape[1] * 16), dtype=torch.uint8, device="cuda")
    L.decode(cache.pool, cache.n_pages, cache.page_table, torch.tensor([T], dtype=torch.int32, device="cuda"), qt, out,
             wsd)
    got = out.double().cpu().numpy()[0]
    check_close(got, c.oracle_decode(c.stored(Z), q[0], T - 1, T), "hidden-mode append")


def test_prefill_causal_small():
    c = case(2)
    s = c.spec
    L = c.load()
    T0, n = 40, 24            # 40 cached tokens, then 24 new queries (chunk of a prefill)
    cache = GpuCache(L, [T0 + n])
    Z = c.latents_direct(0, T0 + n)
    cache.append_latents(0, Z)
    Q = queries(c, 1, n_pos=n)[0]
    qt = torch.from_numpy(Q).cuda().to(torch.bfloat16)
    out = torch.empty(n, s.hidden, device="cuda", dtype=torch.bfloat16)
    ws = torch.empty(L.workspace_bytes(1, T0 + n, n), dtype=torch.uint8, device="cuda")
    L.prefill(cache.pool, cache.n_pages, cache.page_table, [T0], [n], qt, out, ws)
    got = out.double().cpu().numpy()
    want = O.prefill(s, c.f, c.stored(Z), Q, T0, c.B_rot)
    for i in range(n):
        check_close(got[i], want[i], f"prefill query {i}")


def test_batch_40_padded_output_tile():
    # 40 rows -> one 48-row B tile of the tensor-core output kernel (8 zero rows)
    run_decode(case(2), [64] * 3 + [17] * 37, check_pool=False, use_hidden=False)


def test_prefill_two_output_tiles():
    """300 query rows -> two B tiles (256 + 44) of the output kernel; sampled rows checked."""
    c = case(1)
    s = c.spec
    L = c.load()
    T0, n = 20, 300
    cache = GpuCache(L, [T0 + n])
    Z = c.latents_direct(0, T0 + n) if not s.plain else None
    cache.append_latents(0, Z)
    Q = queries(c, 1, n_pos=n)[0]
    qt = torch.from_numpy(Q).cuda().to(torch.bfloat16)
    out = torch.empty(n, s.hidden, device="cuda", dtype=torch.bfloat16)
    ws = torch.empty(L.workspace_bytes(1, T0 + n, n), dtype=torch.uint8, device="cuda")
    L.prefill(cache.pool, cache.n_pages, cache.page_table, [T0], [n], qt, out, ws)
    got = out.double().cpu().numpy()
    Zs = c.stored(Z)
    for i in (0, 1, 255, 256, 299):
        want = O.decode(s, c.f, Zs, Q[i], T0 + i, T0 + i + 1, c.B_rot)
        check_close(got[i], want, f"prefill row {i}")


def test_prefill_tc_row_batches():
    """A quantized RoPE layer's tensor-core prefill (keys and values rebuilt per chunk, tiled causal
    attention): two sequences with different history lengths, 320 rows, rows at the 128-query tile
    and sequence edges and a peaky-attention rerun against the oracle; the CUDA-core path agrees."""
    c = case(2)
    s = c.spec
    starts, ns = [100, 30], [200, 120]
    for peaky in (1.0, 25.0):
        outs = []
        for path in (0, 1):
            L = c.load()
            if path:
                L.set_decode_path(path)
            cache = GpuCache(L, [a + n for a, n in zip(starts, ns)])
            Zs = []
            for b, (a, n) in enumerate(zip(starts, ns)):
                Z = c.latents_direct(b, a + n)
                cache.append_latents(b, Z)
                Zs.append(c.stored(Z))
            Qall = queries(c, 2, peaky=peaky, n_pos=max(ns))
            Q = np.concatenate([Qall[b][:n] for b, n in enumerate(ns)])
            qt = torch.from_numpy(Q).cuda().to(torch.bfloat16)
            out = torch.empty(sum(ns), s.hidden, device="cuda", dtype=torch.bfloat16)
            ws = torch.empty(L.workspace_bytes(2, max(a + n for a, n in zip(starts, ns)), max(ns)), dtype=torch.uint8,
                             device="cuda")
            L.prefill(cache.pool, cache.n_pages, cache.page_table, starts, ns, qt, out, ws)
            outs.append(out.double().cpu().numpy())
        got = outs[0]
        for r in (0, 1, 199, 200, 255, 256, 319):
            b = 0 if r < ns[0] else 1
            i = r if b == 0 else r - ns[0]
            want = O.decode(s, c.f, Zs[b], Q[r], starts[b] + i, starts[b] + i + 1, c.B_rot)
            check_close(got[r], want, f"prefill row {r} (peaky {peaky})")
        assert np.linalg.norm(outs[1] - got) <= 3e-3 * np.linalg.norm(got)


@pytest.mark.parametrize("cfg,quant,lens", [
    (2, False, [600, 257, 256, 1]),
    (3, True, [300, 97]),
    (1, False, [600, 257, 1]),
    (3, False, [300, 97]),
])
def test_tc_scores_feeding_cuda_core_values(cfg, quant, lens):
    """Tensor-core score kernel (path 2) against the oracle, with multiple and
    partial 256-token super-tiles."""
    run_decode(case(cfg, quantized=quant), lens, use_hidden=False, check_pool=False, path=2)
    run_decode(case(cfg, quantized=quant), lens[:2], peaky=25.0, use_hidden=False, check_pool=False, path=2)


@pytest.mark.parametrize("top", [0.2, 1.0])
def test_tc_other_bit_splits(top):
    """The compiled head shapes of the 20 % split (odd group widths in both
    segments) and of all-4-bit latents (full 32-channel 4-bit groups), with
    every rank 16..64, through the tensor-core score path; packed pages
    checked bit for bit."""
    import dataclasses
    spec = dataclasses.replace(gen.config_spec(2, quantized=True), top_fraction=top,
                               key_ranks=[16, 24, 32, 40, 48, 56, 64, 16] * 4)
    c = Case(spec, gen.LAYER_SEED[2], 0)
    run_decode(c, [600, 257, 33], use_hidden=False, check_pool=True)
    run_decode(c, [300, 40], peaky=25.0, use_hidden=False, check_pool=False)


def test_tc_empty_sequences_and_tile_edges():
    """All-tensor-core decode with empty sequences (zero output rows) between
    sequences that end exactly on and just past 128- and 256-token tile edges."""
    run_decode(case(2), [300, 0, 128, 129, 0, 256, 17], use_hidden=False, check_pool=False)


def test_tc_full_rope_table_length():
    """A sequence as long as the RoPE table the layer was loaded with (32768
    positions): the last score tile and the last RoPE tile coincide."""
    run_decode(case(2), [32768, 5], use_hidden=False, check_pool=False)


def test_tc_long_context_runs():
    """All-tensor-core decode with more super-tiles than SMs: CTAs whose unit
    ranges span several super-tiles and cross sequence boundaries."""
    run_decode(case(2), [20000, 9000, 37], use_hidden=False, check_pool=False)
    run_decode(case(2), [12000, 12000], peaky=25.0, use_hidden=False, check_pool=False)


@pytest.mark.parametrize("cfg", [2, 1, 3])
def test_decode_paths_agree(cfg):
    """CUDA-core path (1), tensor-core scores (2) and all tensor-core (0) agree: 4/3-bit latents
    (workload 2) and unquantized bf16 latents (workload 1; workload 3 with GQA)."""
    outs = [run_decode(case(cfg), [700, 300], use_hidden=False, check_pool=False, path=p) for p in (1, 2, 0)]
    for o in outs[1:]:
        assert np.linalg.norm(o - outs[0]) <= 3e-3 * np.linalg.norm(outs[0])


def test_device_status_bad_page():
    """An out-of-range page id is caught by the kernels (status word), not dereferenced."""
    c = case(0)
    L = c.load()
    cache = GpuCache(L, [40])
    cache.append_latents(0, c.latents_direct(0, 40))
    torch.cuda.synchronize()
    assert L.sync_status() == 0
    bad = cache.page_table.clone()
    bad[0, 1] = cache.n_pages + 5
    q = torch.from_numpy(queries(c, 1)[:, 0]).cuda().float()
    out = torch.empty(1, c.spec.hidden, device="cuda")
    ws = torch.empty(L.workspace_bytes(1, bad.shape[1] * 16), dtype=torch.uint8, device="cuda")
    L.decode(cache.pool, cache.n_pages, bad, torch.tensor([40], dtype=torch.int32, device="cuda"), q, out, ws)
    assert L.sync_status() & 0x1
    assert L.sync_status() == 0     # read-and-clear
    # append to a position beyond the page table
    z = torch.zeros(1, L.latent_total, device="cuda")
    L.append(cache.pool, cache.n_pages, cache.page_table, torch.zeros(1, dtype=torch.int32, device="cuda"),
             torch.tensor([cache.page_table.shape[1] * 16], dtype=torch.int32, device="cuda"), z, True)
    assert L.sync_status() & 0x2


def test_bounded_wait_expires_into_the_status_word():
    """A bounded device wait on a barrier that nothing completes gives up after its limit, sets
    STARKV_DEV_TIMEOUT and lets the waiting roles drain; the host reads STARKV_ERR_TIMEOUT and the
    context stays usable for a normal decode afterwards."""
    import time
    from decode_attention_rank_b200 import starkv as lib
    c = case(0)
    L = c.load()
    cache = GpuCache(L, [40])
    Z = c.latents_direct(0, 40)
    cache.append_latents(0, Z)
    torch.cuda.synchronize()
    assert L.sync_status() == 0
    t0 = time.perf_counter()
    L.check_wait_timeout(50000)                 # 50 ms
    st, bits = L.sync_status_code()
    dt = time.perf_counter() - t0
    assert st == 6 and bits == lib.DEV_TIMEOUT, (st, bits)
    assert 0.04 < dt < 5.0, dt
    assert L.sync_status_code() == (0, 0)       # read-and-clear
    q = queries(c, 1)[:, 0]
    out = torch.empty(1, c.spec.hidden, device="cuda")
    ws = torch.empty(L.workspace_bytes(1, cache.page_table.shape[1] * 16), dtype=torch.uint8, device="cuda")
    L.decode(cache.pool, cache.n_pages, cache.page_table, torch.tensor([40], dtype=torch.int32, device="cuda"),
             torch.from_numpy(q).cuda().float(), out, ws)
    assert L.sync_status() == 0
    check_close(out.double().cpu().numpy()[0], c.oracle_decode(c.stored(Z), q[0], 39, 40), "decode after timeout")


@pytest.mark.parametrize("cfg,quant", [(2, False), (3, True), (1, False)])
def test_unfused_value_output(cfg, quant):
    """Output in the unfused order (y_h B'_v,kv(h), then W_o; "STAR-KV 阅读笔记" section 5.3 states the
    fusion as an exact reorder) against the oracle, which uses W_o and the explicit values; GQA
    (workload 3) and the CUDA-core decode path (workload 1, unquantized) included; and the fused
    layer's output agrees within the tolerance."""
    c = case(cfg, quantized=quant)
    lens = [333, 64, 5]
    a = run_decode(c, lens, use_hidden=False, check_pool=False, unfused=True)
    run_decode(c, lens[:2], peaky=25.0, use_hidden=False, check_pool=False, unfused=True)
    b = run_decode(c, lens, use_hidden=False, check_pool=False)
    assert np.linalg.norm(a - b) <= 3e-3 * np.linalg.norm(b)


def test_phase_timing_leaves_results_unchanged():
    """starkv_profile_decode records per-kernel times without changing the output."""
    c = case(2)
    L = c.load()
    lens = [600, 257, 33]
    cache = GpuCache(L, lens, seed=3)
    for b, T in enumerate(lens):
        cache.append_latents(b, c.latents_direct(b, T))
    B = len(lens)
    q = torch.from_numpy(queries(c, B)[:, 0]).cuda().to(torch.bfloat16)
    ws = torch.empty(L.workspace_bytes(B, cache.page_table.shape[1] * 16), dtype=torch.uint8, device="cuda")
    seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    outs = []
    for prof in (0, 3):
        L.profile_decode(prof)
        out = torch.empty(B, c.spec.hidden, device="cuda", dtype=torch.bfloat16)
        for _ in range(3):
            L.decode(cache.pool, cache.n_pages, cache.page_table, seq_lens, q, out, ws)
        torch.cuda.synchronize()
        outs.append(out.float().cpu().numpy())
        if prof:
            ms = L.decode_phase_ms(3)
            assert len(ms) == 3 and all(len(m) == 4 for m in ms)
            assert all(t > 0.0 for m in ms for t in m), ms
            assert all(sum(m) < 1000.0 for m in ms), ms
    L.profile_decode(0)
    assert L.sync_status() == 0
    np.testing.assert_array_equal(outs[0], outs[1])


def _prefill_rows(c, L, starts, ns, peaky=1.0):
    """Append each sequence's latents (history and chunk), run one prefill call, return
    (outputs [sum ns][D] float64, queries, stored latents per sequence)."""
    s = c.spec
    cache = GpuCache(L, [a + n for a, n in zip(starts, ns)])
    Zs = []
    for b, (a, n) in enumerate(zip(starts, ns)):
        T = a + n
        Z = c.latents_from_hidden(c.hidden(b, T), np.arange(T)) if s.plain else c.latents_direct(b, T)
        cache.append_latents(b, Z)
        Zs.append(c.stored(Z))
    Qall = queries(c, len(ns), peaky=peaky, n_pos=max(ns))
    Q = np.concatenate([Qall[b][:n] for b, n in enumerate(ns)])
    qt = torch.from_numpy(Q).cuda().to(torch.bfloat16)
    out = torch.empty(sum(ns), s.hidden, device="cuda", dtype=torch.bfloat16)
    ws = torch.empty(L.workspace_bytes(len(ns), cache.page_table.shape[1] * 16, max(ns)), dtype=torch.uint8,
                     device="cuda")
    L.prefill(cache.pool, cache.n_pages, cache.page_table, starts, ns, qt, out, ws)
    torch.cuda.synchronize()
    assert L.sync_status() == 0
    return out.double().cpu().numpy(), Q, Zs


@pytest.mark.parametrize("cfg,quant,layer", [(2, False, 2), (1, False, 2), (3, False, 2), (3, True, 2), (4, False, 0)])
def test_prefill_tensor_core_tiles(cfg, quant, layer):
    """Tensor-core prefill against the oracle's causal attention: 4/3-bit and bf16 latents, GQA
    (workload 3) and an uncompressed layer (workload 4, layer 0).  Two sequences, one with history
    and a chunk that ends inside a 128-query tile, one a prompt from position 0; rows at the tile
    edges, the first and last rows, and a peaky rerun; all rows agree with the CUDA-core path."""
    c = case(cfg, quantized=quant, layer=layer)
    s = c.spec
    starts, ns = [300, 0], [200, 131]
    for peaky in (1.0, 25.0):
        L = c.load()
        got, Q, Zs = _prefill_rows(c, L, starts, ns, peaky)
        for r in (0, 1, 127, 128, 199, 200, 327, 328, 330):
            b = 0 if r < ns[0] else 1
            i = r if b == 0 else r - ns[0]
            T = starts[b] + i + 1
            if s.plain:
                want = O.decode_plain(s, c.f, np.concatenate(Zs[b][:-1], axis=1), Zs[b][-1], Q[r], T, T - 1)
            else:
                want = O.decode(s, c.f, Zs[b], Q[r], T - 1, T, c.B_rot)
            check_close(got[r], want, f"prefill row {r} (peaky {peaky})")
        if peaky == 1.0:
            L1 = c.load()
            L1.set_decode_path(1)
            ref, _, _ = _prefill_rows(c, L1, starts, ns, peaky)
            assert np.linalg.norm(ref - got) <= 3e-3 * np.linalg.norm(ref)
