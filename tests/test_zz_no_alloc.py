"""Decode without a workspace: starkv_decode_attn_noalloc.

Some callers cannot allocate device memory for a workspace (for example a
plugin inside a serving engine whose allocator already holds the GPU's memory),
so the library offers a decode entry point whose scratch is a fixed device
array inside the library.  This checks, through the C ABI, that two calls in a
row give the same output as the regular entry point with a caller workspace,
and that a size beyond the array is refused before any launch.  Both entry
points run the same kernels on the same inputs and every step of the decode
is deterministic (no floating-point atomics; partial sums are added in a
fixed order), so the outputs must agree bit for bit: a stale or unwritten
scratch element would show up as a difference.  This file is collected last
on purpose.
"""
import numpy as np
import pytest
import torch

from synth import gen

from harness import Case, GpuCache, queries

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode():
    from decode_attention_rank_b200 import starkv as lib
    c = Case(gen.config_spec(2), gen.LAYER_SEED[2])
    L = c.load()
    lens = [700, 33, 256]
    cache = GpuCache(L, lens)
    for b, T in enumerate(lens):
        cache.append_latents(b, c.latents_direct(b, T))
    B = len(lens)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    max_ctx = cache.page_table.shape[1] * 16
    assert L.workspace_bytes(B, max_ctx) <= lib.NOALLOC_SCRATCH_BYTES
    ws = torch.empty(L.workspace_bytes(B, max_ctx), dtype=torch.uint8, device="cuda")
    for call in range(2):
        q = torch.from_numpy(queries(c, B, peaky=1.0 + 7.0 * call)[:, 0]).cuda().to(torch.bfloat16)
        ref = torch.empty(B, c.spec.hidden, dtype=torch.bfloat16, device="cuda")
        got = torch.full_like(ref, float("nan"))
        L.decode(cache.pool, cache.n_pages, cache.page_table, seq_lens, q, ref, ws)
        L.decode_noalloc(cache.pool, cache.n_pages, cache.page_table, seq_lens, q, got)
        torch.cuda.synchronize()
        assert L.sync_status() == 0
        g = got.double().cpu().numpy()
        assert np.isfinite(g).all()
        assert torch.equal(got, ref), f"call {call}: {int((got != ref).sum())} elements differ"


def test_noalloc_refuses_sizes_beyond_the_array():
    from decode_attention_rank_b200 import starkv as lib
    c = Case(gen.config_spec(0), 0)
    L = c.load()
    B, max_pages = 64, 4096          # score buffer alone: 64 * 4 heads * 65536 * 4 B = 64 MiB
    assert L.workspace_bytes(B, max_pages * 16) > lib.NOALLOC_SCRATCH_BYTES
    pool = torch.zeros(L.page_bytes, dtype=torch.uint8, device="cuda")
    pt = torch.zeros(B, max_pages, dtype=torch.int32, device="cuda")
    lens = torch.ones(B, dtype=torch.int32, device="cuda")
    q = torch.zeros(B, 4, 64, device="cuda")
    out = torch.zeros(B, 256, device="cuda")
    with pytest.raises(lib.StarKVError) as e:
        L.decode_noalloc(pool, 1, pt, lens, q, out)
    assert e.value.status == 7 and "scratch" in str(e.value)
