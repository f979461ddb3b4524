"""Thin Python binding of the libstarkv C ABI (argument marshalling only).

Every step of the attention path runs in the library's CUDA kernels; this
module converts torch tensors to raw pointers and sizes, calls the C entry
points declared in include/starkv.h, and raises on a non-OK status.  torch is
used only to hold device memory and to name the current CUDA stream.

Importing succeeds on machines without a GPU (the shared library loads without
one); calling into it then fails with the CUDA error the runtime reports.  If
libstarkv.so is missing, the import fails: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libstarkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m decode_attention_rank_b200.build` "
                      "(there is no fallback path)")
_lib = ctypes.CDLL(LIB_PATH)

STARKV_F32, STARKV_BF16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "out of device memory", 4: "CUDA error",
          5: "device status word set", 6: "device wait timed out", 7: "workspace too small"}
DEV_BAD_PAGE, DEV_BAD_POSITION, DEV_SCALE_OVF, DEV_TIMEOUT = 0x1, 0x2, 0x4, 0x8

EXPORTED = ["starkv_load_factors", "starkv_free_layer", "starkv_layer_get_info", "starkv_page_bytes",
            "starkv_cache_init", "starkv_append", "starkv_append_workspace_bytes", "starkv_decode_attn",
            "starkv_prefill_attn", "starkv_workspace_bytes", "starkv_sync_status", "starkv_status_string",
            "starkv_last_error", "starkv_version", "starkv_decode_attn_noalloc", "starkv_set_decode_path",
            "starkv_check_wait_timeout"]
NOALLOC_SCRATCH_BYTES = 32 << 20


class _Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("key_ranks", ctypes.POINTER(ctypes.c_int)),
                ("value_rank", ctypes.c_int), ("dtype", ctypes.c_int), ("quantized", ctypes.c_int),
                ("top_fraction", ctypes.c_float), ("top_bits", ctypes.c_int), ("bottom_bits", ctypes.c_int),
                ("group_size", ctypes.c_int), ("hadamard_block", ctypes.c_int), ("rope", ctypes.c_int),
                ("rope_theta", ctypes.c_double), ("softmax_scale", ctypes.c_float), ("page_size", ctypes.c_int),
                ("plain", ctypes.c_int), ("max_positions", ctypes.c_int), ("unfused_output", ctypes.c_int)]


class _Info(ctypes.Structure):
    _fields_ = [("n_latents", ctypes.c_int), ("latent_total", ctypes.c_int), ("key_rank_total", ctypes.c_int),
                ("page_bytes", ctypes.c_size_t), ("bytes_per_token", ctypes.c_double),
                ("factor_bytes", ctypes.c_size_t)]


_vp, _i32p, _sz, _i64 = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64
_lib.starkv_load_factors.argtypes = [ctypes.POINTER(_Config), _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(_vp)]
_lib.starkv_free_layer.argtypes = [_vp]
_lib.starkv_free_layer.restype = None
_lib.starkv_layer_get_info.argtypes = [_vp, ctypes.POINTER(_Info)]
_lib.starkv_page_bytes.argtypes = [_vp]
_lib.starkv_page_bytes.restype = _sz
_lib.starkv_cache_init.argtypes = [_vp, _vp, _i64, _vp]
_lib.starkv_append.argtypes = [_vp, _vp, _i64, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _i32p, _vp,
                               ctypes.c_int, _vp, _sz, _vp]
_lib.starkv_append_workspace_bytes.argtypes = [_vp, ctypes.c_int]
_lib.starkv_append_workspace_bytes.restype = _sz
_lib.starkv_decode_attn.argtypes = [_vp, _vp, _i64, _i32p, ctypes.c_int, ctypes.c_int, _i32p, _i32p, _vp, _vp, _vp,
                                    _sz, _vp]
_lib.starkv_prefill_attn.argtypes = [_vp, _vp, _i64, _i32p, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _sz,
                                     _vp]
_lib.starkv_decode_attn_noalloc.argtypes = [_vp, _vp, _i64, _i32p, ctypes.c_int, ctypes.c_int, _i32p, _i32p, _vp,
                                            _vp, _vp]
_lib.starkv_workspace_bytes.argtypes = [_vp, ctypes.c_int, ctypes.c_int, ctypes.c_int]
_lib.starkv_workspace_bytes.restype = _sz
_lib.starkv_sync_status.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
_lib.starkv_status_string.argtypes = [ctypes.c_int]
_lib.starkv_status_string.restype = ctypes.c_char_p
_lib.starkv_last_error.argtypes = []
_lib.starkv_last_error.restype = ctypes.c_char_p
_lib.starkv_set_decode_path.argtypes = [_vp, ctypes.c_int]
_lib.starkv_check_wait_timeout.argtypes = [_vp, ctypes.c_uint32, _vp]
_lib.starkv_profile_decode.argtypes = [_vp, ctypes.c_int]
_lib.starkv_decode_phase_ms.argtypes = [_vp, ctypes.POINTER(ctypes.c_float), ctypes.c_int]
N_PHASES = 4   # query preparation + scores, joint values, run merge, output projection
_lib.starkv_version.argtypes = []
_lib.starkv_version.restype = ctypes.c_char_p


class StarKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.starkv_last_error().decode()
        super().__init__(f"{where}: {STATUS.get(status, status)}" + (f" ({msg})" if msg else ""))


def _check(st: int, where: str) -> None:
    if st != 0:
        raise StarKVError(st, where)


def version() -> str:
    return _lib.starkv_version().decode()


def _ptr(t) -> int:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


@dataclass
class LayerConfig:
    """Python mirror of starkv_layer_config (see include/starkv.h)."""
    hidden: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    key_ranks: list = field(default_factory=list)
    value_rank: int = 0
    dtype: str = "bf16"
    quantized: bool = False
    top_fraction: float = 0.25
    top_bits: int = 4
    bottom_bits: int = 3
    group_size: int = 32
    hadamard_block: int = 0
    rope: bool = False
    rope_theta: float = 10000.0
    softmax_scale: float = 0.0
    page_size: int = 16
    plain: bool = False
    max_positions: int = 0
    unfused_output: bool = False

    @classmethod
    def from_spec(cls, spec) -> "LayerConfig":
        return cls(hidden=spec.hidden, n_heads=spec.n_heads, n_kv_heads=spec.n_kv_heads, head_dim=spec.head_dim,
                   key_ranks=list(spec.key_ranks), value_rank=spec.value_rank, dtype=spec.dtype,
                   quantized=spec.quantized, top_fraction=spec.top_fraction, top_bits=spec.top_bits,
                   bottom_bits=spec.bottom_bits, group_size=spec.group_size, hadamard_block=spec.hadamard_block,
                   rope=spec.rope, rope_theta=spec.rope_theta, page_size=spec.page_size, plain=spec.plain)

    def _c(self):
        ranks = (ctypes.c_int * max(1, len(self.key_ranks)))(*self.key_ranks)
        c = _Config(self.hidden, self.n_heads, self.n_kv_heads, self.head_dim,
                    ctypes.cast(ranks, ctypes.POINTER(ctypes.c_int)) if self.key_ranks else None, self.value_rank,
                    STARKV_F32 if self.dtype == "f32" else STARKV_BF16, int(self.quantized), self.top_fraction,
                    self.top_bits, self.bottom_bits, self.group_size, self.hadamard_block, int(self.rope),
                    self.rope_theta, self.softmax_scale, self.page_size, int(self.plain), self.max_positions,
                    int(self.unfused_output))
        return c, ranks


class Layer:
    """One loaded layer (owns its folded factors on the device)."""

    def __init__(self, handle: int, cfg: LayerConfig):
        self._h = handle
        self.cfg = cfg
        info = _Info()
        _check(_lib.starkv_layer_get_info(self._h, ctypes.byref(info)), "starkv_layer_get_info")
        self.n_latents = info.n_latents
        self.latent_total = info.latent_total
        self.key_rank_total = info.key_rank_total
        self.page_bytes = info.page_bytes
        self.bytes_per_token = info.bytes_per_token
        self.factor_bytes = info.factor_bytes

    def __del__(self):
        self.free()

    def free(self) -> None:
        if getattr(self, "_h", None):
            _lib.starkv_free_layer(self._h)
            self._h = None

    @property
    def handle(self) -> int:
        return self._h

    def cache_init(self, pool, n_pages: int, stream=None) -> None:
        _check(_lib.starkv_cache_init(self._h, _ptr(pool), n_pages, _stream(stream)), "starkv_cache_init")

    def append_workspace_bytes(self, n_tokens: int) -> int:
        return _lib.starkv_append_workspace_bytes(self._h, n_tokens)

    def append(self, pool, n_pages: int, page_table, seq_idx, positions, inputs, input_is_latent: bool,
               workspace=None, stream=None) -> None:
        n = int(seq_idx.numel())
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        _check(_lib.starkv_append(self._h, _ptr(pool), n_pages, _ptr(page_table), int(page_table.shape[0]),
                                  int(page_table.shape[1]), n,
                                  _ptr(seq_idx), _ptr(positions), _ptr(inputs), int(input_is_latent),
                                  _ptr(workspace), ws_bytes, _stream(stream)), "starkv_append")

    def workspace_bytes(self, batch: int, max_ctx: int, max_q: int = 1) -> int:
        return _lib.starkv_workspace_bytes(self._h, batch, max_ctx, max_q)

    def decode(self, pool, n_pages: int, page_table, seq_lens, q, out, workspace, q_pos=None, stream=None) -> None:
        _check(_lib.starkv_decode_attn(self._h, _ptr(pool), n_pages, _ptr(page_table), int(page_table.shape[1]),
                                       int(seq_lens.numel()), _ptr(seq_lens), _ptr(q_pos), _ptr(q), _ptr(out),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream)), "starkv_decode_attn")

    def decode_noalloc(self, pool, n_pages: int, page_table, seq_lens, q, out, q_pos=None, stream=None) -> None:
        """Decode without a workspace (scratch in the library's fixed device array)."""
        _check(_lib.starkv_decode_attn_noalloc(self._h, _ptr(pool), n_pages, _ptr(page_table),
                                               int(page_table.shape[1]), int(seq_lens.numel()), _ptr(seq_lens),
                                               _ptr(q_pos), _ptr(q), _ptr(out), _stream(stream)),
               "starkv_decode_attn_noalloc")

    def prefill(self, pool, n_pages: int, page_table, q_start: list, q_len: list, q, out, workspace,
                stream=None) -> None:
        B = len(q_start)
        qs = (ctypes.c_int32 * B)(*q_start)
        ql = (ctypes.c_int32 * B)(*q_len)
        _check(_lib.starkv_prefill_attn(self._h, _ptr(pool), n_pages, _ptr(page_table), int(page_table.shape[1]), B,
                                        ctypes.cast(qs, _vp), ctypes.cast(ql, _vp), _ptr(q), _ptr(out),
                                        _ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream(stream)), "starkv_prefill_attn")

    def set_decode_path(self, path: int) -> None:
        """0 automatic, 1 CUDA-core kernels, 2 tensor-core scores + CUDA-core values (diagnostics)."""
        _check(_lib.starkv_set_decode_path(self._h, path), "starkv_set_decode_path")

    def profile_decode(self, n_calls: int) -> None:
        """Keep CUDA-event timings of the next n_calls tensor-core decodes (0 = off)."""
        _check(_lib.starkv_profile_decode(self._h, n_calls), "starkv_profile_decode")

    def decode_phase_ms(self, n_calls: int) -> list:
        """Per-call lists of the phase times (ms) recorded since profile_decode."""
        buf = (ctypes.c_float * (n_calls * N_PHASES))()
        _check(_lib.starkv_decode_phase_ms(self._h, buf, n_calls), "starkv_decode_phase_ms")
        return [list(buf[c * N_PHASES:(c + 1) * N_PHASES]) for c in range(n_calls)]

    def check_wait_timeout(self, limit_us: int, stream=None) -> None:
        """Run the bounded-wait diagnostic kernel (see starkv_check_wait_timeout)."""
        _check(_lib.starkv_check_wait_timeout(self._h, limit_us, _stream(stream)), "starkv_check_wait_timeout")

    def sync_status_code(self, stream=None) -> tuple:
        """(status code of starkv_sync_status, status bits)."""
        bits = ctypes.c_uint32(0)
        st = _lib.starkv_sync_status(self._h, _stream(stream), ctypes.byref(bits))
        return st, bits.value

    def sync_status(self, stream=None) -> int:
        bits = ctypes.c_uint32(0)
        st = _lib.starkv_sync_status(self._h, _stream(stream), ctypes.byref(bits))
        if st not in (0, 5, 6):
            _check(st, "starkv_sync_status")
        return bits.value


def load_factors(cfg: LayerConfig, A_k, B_k, A_v, B_v, W_o, stream=None) -> Layer:
    """Fold and upload one layer's factors (device tensors in cfg.dtype, unrotated)."""
    c, keep = cfg._c()
    h = _vp()
    _check(_lib.starkv_load_factors(ctypes.byref(c), _ptr(A_k), _ptr(B_k), _ptr(A_v), _ptr(B_v), _ptr(W_o),
                                    _stream(stream), ctypes.byref(h)), "starkv_load_factors")
    del keep
    return Layer(h.value, cfg)


def raw_lib():
    """The ctypes handle of libstarkv.so (for tests of the C ABI itself)."""
    return _lib
