"""The C ABI library on a machine without a GPU: it loads, exports every entry
point declared in include/starkv.h, and rejects bad arguments on the host
before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"STARKV_API\s+[\w\s\*]+?\b(starkv_\w+)\s*\(", text)
    return names


def test_library_exports_every_declared_symbol():
    from decode_attention_rank_b200 import starkv as lib
    names = declared_symbols()
    assert len(names) >= 14
    raw = lib.raw_lib()
    for n in names:
        assert hasattr(raw, n), n
    assert set(lib.EXPORTED) <= set(names)


def test_version_and_status_strings():
    from decode_attention_rank_b200 import starkv as lib
    assert "sm_100a" in lib.version()
    raw = lib.raw_lib()
    for code, text in lib.STATUS.items():
        assert raw.starkv_status_string(code).decode() == text


def test_host_validation_before_cuda():
    from decode_attention_rank_b200 import starkv as lib
    bad = [
        dict(hidden=64, n_heads=3, n_kv_heads=2, head_dim=8, key_ranks=[4, 4], value_rank=8),    # H % Hkv
        dict(hidden=64, n_heads=2, n_kv_heads=2, head_dim=7, key_ranks=[4, 4], value_rank=8),    # odd d
        dict(hidden=64, n_heads=2, n_kv_heads=2, head_dim=8, key_ranks=[9, 4], value_rank=8),    # rank > d
        dict(hidden=64, n_heads=2, n_kv_heads=2, head_dim=8, key_ranks=[4, 4], value_rank=17),   # r_v > Hkv d
        dict(hidden=64, n_heads=2, n_kv_heads=2, head_dim=8, key_ranks=[4, 4], value_rank=8, page_size=8),
        dict(hidden=64, n_heads=2, n_kv_heads=2, head_dim=8, key_ranks=[4, 4], value_rank=8, hadamard_block=32),
        dict(hidden=64, n_heads=2, n_kv_heads=2, head_dim=8, key_ranks=[4, 4], value_rank=8, quantized=True,
             top_bits=9),
    ]
    for kw in bad:
        cfg = lib.LayerConfig(**kw)
        with pytest.raises(lib.StarKVError) as e:
            lib.load_factors(cfg, None, None, None, None, None, stream=0)
        assert e.value.status == 1, kw
    # null factors with a valid config are also rejected on the host
    cfg = lib.LayerConfig(hidden=64, n_heads=2, n_kv_heads=2, head_dim=8, key_ranks=[4, 4], value_rank=8)
    with pytest.raises(lib.StarKVError) as e:
        lib.load_factors(cfg, None, None, None, None, None, stream=0)
    assert e.value.status == 1
    raw = lib.raw_lib()
    assert raw.starkv_decode_attn(None, None, 0, None, 0, 1, None, None, None, None, None, 0, None) == 1
    assert raw.starkv_append(None, None, 0, None, 0, 0, 1, None, None, None, 0, None, 0, None) == 1
    assert raw.starkv_workspace_bytes(None, 1, 1, 1) == 0
    assert raw.starkv_prefill_attn(None, None, 0, None, 0, 1, None, None, None, None, None, 0, None) == 1
    # a top fraction outside [0, 1] is rejected before anything is allocated
    cfg = lib.LayerConfig(hidden=64, n_heads=2, n_kv_heads=2, head_dim=8, key_ranks=[4, 4], value_rank=8,
                          quantized=True, top_fraction=1.5)
    with pytest.raises(lib.StarKVError) as e:
        lib.load_factors(cfg, None, None, None, None, None, stream=0)
    assert e.value.status == 1


def test_page_table_capacity_overflow_rejected_on_the_host():
    # max_pages * 16 must fit in an int: a larger page table is refused before the layer is read
    # or any size is computed from it (dummy non-NULL pointers, never dereferenced).
    from decode_attention_rank_b200 import starkv as lib
    raw = lib.raw_lib()
    dummy = ctypes.create_string_buffer(4096)
    p = ctypes.cast(dummy, ctypes.c_void_p).value
    big = (2 ** 31 - 1) // 16 + 1
    assert raw.starkv_decode_attn(p, p, 1, p, big, 1, p, None, p, p, p, 1 << 20, None) == 1
    assert "overflows" in raw.starkv_last_error().decode()
    assert raw.starkv_decode_attn_noalloc(p, p, 1, p, big, 1, p, None, p, p, None) == 1
    assert "overflows" in raw.starkv_last_error().decode()
    assert raw.starkv_prefill_attn(p, p, 1, p, big, 1, p, p, p, p, p, 1 << 20, None) == 1
    assert "overflows" in raw.starkv_last_error().decode()
    assert raw.starkv_append(p, p, 1, p, 1, big, 1, p, p, p, 1, p, 0, None) == 1
    assert "overflows" in raw.starkv_last_error().decode()


def test_misaligned_buffers_rejected_on_the_host():
    # 16-byte device buffers and 4-byte int32 arrays: a pointer off its boundary is refused with
    # STARKV_ERR_ARG before the layer is read or any CUDA call is made (dummy host pointers, never
    # dereferenced).
    from decode_attention_rank_b200 import starkv as lib
    raw = lib.raw_lib()
    dummy = ctypes.create_string_buffer(4096 + 64)
    p = (ctypes.cast(dummy, ctypes.c_void_p).value + 15) // 16 * 16
    for off in (2, 8):
        m = p + off
        assert raw.starkv_decode_attn(p, p, 1, p, 1, 1, p, None, m, p, p, 1 << 20, None) == 1     # q
        assert "aligned" in raw.starkv_last_error().decode()
        assert raw.starkv_decode_attn(p, p, 1, p, 1, 1, p, None, p, m, p, 1 << 20, None) == 1     # out
        assert raw.starkv_decode_attn(p, p, 1, p, 1, 1, p, None, p, p, m, 1 << 20, None) == 1     # workspace
        assert raw.starkv_decode_attn(p, m, 1, p, 1, 1, p, None, p, p, p, 1 << 20, None) == 1     # pool
        assert raw.starkv_decode_attn_noalloc(p, p, 1, p, 1, 1, p, None, m, p, None) == 1         # q
        assert "aligned" in raw.starkv_last_error().decode()
        assert raw.starkv_prefill_attn(p, p, 1, p, 1, 1, p, p, m, p, p, 1 << 20, None) == 1       # q
        assert "aligned" in raw.starkv_last_error().decode()
        assert raw.starkv_append(p, p, 1, p, 1, 1, 1, p, p, m, 1, p, 0, None) == 1                # input
        assert "aligned" in raw.starkv_last_error().decode()
    # int32 arrays off a 4-byte boundary
    assert raw.starkv_decode_attn(p, p, 1, p + 2, 1, 1, p, None, p, p, p, 1 << 20, None) == 1      # page_table
    assert raw.starkv_decode_attn(p, p, 1, p, 1, 1, p + 1, None, p, p, p, 1 << 20, None) == 1      # seq_lens
    assert raw.starkv_decode_attn(p, p, 1, p, 1, 1, p, p + 2, p, p, p, 1 << 20, None) == 1         # q_pos
    assert raw.starkv_decode_attn_noalloc(p, p, 1, p + 2, 1, 1, p, None, p, p, None) == 1
    assert raw.starkv_prefill_attn(p, p, 1, p + 2, 1, 1, p, p, p, p, p, 1 << 20, None) == 1
    assert raw.starkv_append(p, p, 1, p, 1, 1, 1, p + 2, p, p, 1, p, 0, None) == 1               # seq_idx
    assert raw.starkv_append(p, p, 1, p, 1, 1, 1, p, p + 2, p, 1, p, 0, None) == 1               # positions
    assert "aligned" in raw.starkv_last_error().decode()


def test_binding_argument_counts_match_the_header():
    # Every entry point the binding declares argtypes for takes as many arguments as include/starkv.h says.
    from decode_attention_rank_b200 import starkv as lib
    text = open(os.path.join(ROOT, "include", "starkv.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    sigs = dict(re.findall(r"STARKV_API\s+[\w\s\*]+?\b(starkv_\w+)\s*\(([^)]*)\)", text))
    raw = lib.raw_lib()
    checked = 0
    for name, params in sigs.items():
        argtypes = getattr(raw, name).argtypes
        if argtypes is None:
            continue
        p = params.strip()
        n = 0 if p in ("", "void") else len(p.split(","))
        assert len(argtypes) == n, (name, len(argtypes), n)
        checked += 1
    assert checked >= 15
